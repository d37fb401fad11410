// bs_linear_no_alloc: the decode path with its scratch memory in a fixed array that
// the library itself holds, for callers that cannot allocate device memory.
//
// Who needs it: some hosts hand a kernel only its input and output buffers and no
// workspace (plugin interfaces of inference engines, for example), and some serving
// loops forbid any device allocation after start-up, because cudaMalloc can
// synchronise the whole device and can fail under memory pressure in the middle of
// a request.  Such callers cannot provide the workspace bs_linear asks for.
//
// How: the scratch is a file-scope __device__ array of kStaticScratchBytes (8 MiB).
// Every GPU that loads this library keeps that much memory until the process exits.
// Host code may not use the array's name as a device address (on the host it is
// only a stand-in symbol), so the first call on each device, with that device
// current, asks the runtime for the array's device address with
// cudaGetSymbolAddress, clears the whole array and caches the address.  That first
// call is synchronous; make it before any stream capture.  Nothing here calls
// cudaMalloc, cudaFree or any other allocating routine.
//
// All calls on a device share the one array, and it keeps whatever the previous call
// left in it; a decode call that completes leaves its row-tile counters at zero, so
// no clearing is needed between calls.  A call that ran out of a bounded wait may
// leave counters behind, and the array belongs to every stack on the device: once
// bs_get_device_error has reported an error on any stack of a device, the next
// no-alloc call on that device, whatever its stack, clears the whole array first (an
// asynchronous memset on the call's stream).  Two calls whose kernels may overlap on
// the GPU (different streams, no ordering between them) race on the array: order them
// on one stream, or give them distinct workspaces through bs_linear.
#include <atomic>
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::atomic<int> g_scratch_dirty[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_static_scratch on the current device; set up on first use.
bs_status scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return BS_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return BS_ERR_CUDA;
    if (cudaMemset(p, 0, kStaticScratchBytes) != cudaSuccess) return BS_ERR_CUDA;
    g_scratch_addr[device] = p;
    g_scratch_dirty[device].store(0);
  }
  *out = g_scratch_addr[device];
  return BS_OK;
}

}  // namespace

namespace bs {
void note_device_error(int device) {
  if (device >= 0 && device < kMaxDevices) g_scratch_dirty[device].store(1);
}
}  // namespace bs

extern "C" bs_status bs_linear_no_alloc(bs_stack_t stack, const void* x, int batch, bs_dtype dt, int n_loaded,
                                        void* y, bs_stream_t stream) {
  if (stack == nullptr || x == nullptr || y == nullptr || batch <= 0) return BS_ERR_INVALID_ARG;
  if (batch > bs::kDecodeMaxBatch || stack->plain) return BS_ERR_INVALID_ARG;
  if (n_loaded < 0 || n_loaded > stack->n_blocks) return BS_ERR_RANGE;
  const size_t need = bs::decode_ws_layout(stack->m, stack->d, n_loaded > 0 ? n_loaded : 1, batch).total;
  if (need > kStaticScratchBytes) return BS_ERR_CAPACITY;
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess) return BS_ERR_NO_DEVICE;
  if (device != stack->device) return BS_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const bs_status st = scratch_address(device, &scratch);
  if (st != BS_OK) return st;
  if (g_scratch_dirty[device].exchange(0) != 0) {
    if (cudaMemsetAsync(scratch, 0, kStaticScratchBytes, stream) != cudaSuccess) {
      g_scratch_dirty[device].store(1);
      return BS_ERR_CUDA;
    }
  }
  return bs_linear(stack, x, batch, dt, n_loaded, y, scratch, kStaticScratchBytes, stream);
}
