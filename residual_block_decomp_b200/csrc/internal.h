// Internal declarations shared by the host API and the kernels of the library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/bitstack.h"

namespace bs {

constexpr int kK = 16;                 // singular vectors per block on the GPU path
constexpr int kTileRows = 128;         // rows of a sign tile / an MMA M tile
constexpr int kTileCols = 256;         // columns of a sign tile / one decode unit
constexpr int kTileBytes = 4096;       // bytes of one sign tile
constexpr int kDecodeMaxBatch = 4;     // batches up to this run the factored decode kernel
constexpr int kDecodeMaxBlocks = 64;   // loaded blocks the decode kernel stages |V| maxima for
constexpr int kMaxGrid = 160;          // cap on the decode kernel's persistent grid
constexpr uint32_t kErrTimeout = 1u;   // device error word bit: a bounded wait ran out

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Decode workspace carve-up (all regions 256-byte aligned).
struct DecodeWs {
  size_t hdr, zq, csum, flags, part, cnt, total;
};
inline DecodeWs decode_ws_layout(int m, int d, int n, int batch) {
  DecodeWs w{};
  const size_t KG = static_cast<size_t>(d) / kTileCols;
  const size_t chunks = static_cast<size_t>(n) * KG;
  size_t off = 0;
  w.hdr = off;   off = 256;  // {epoch, done}: see DecodeParams::hdr
  w.zq = off;    off = align_up(off + chunks * 32u * batch * kTileCols, 256);
  w.csum = off;  off = align_up(off + chunks * 16u * batch * sizeof(float), 256);
  w.flags = off; off = align_up(off + chunks * sizeof(uint32_t), 256);
  w.part = off;  off = align_up(off + static_cast<size_t>(kMaxGrid) * 2 * kTileRows * batch * sizeof(float), 256);
  w.cnt = off;   off = align_up(off + static_cast<size_t>(m / kTileRows) * sizeof(unsigned long long), 256);
  w.total = off;
  return w;
}

struct DecodeParams {
  const uint8_t* blocks;       // record i at blocks + i * block_bytes
  unsigned long long block_bytes;
  const void* x;               // batch x d, f16 or bf16
  void* y;                     // batch x m, same dtype
  const float* inv_s;          // d
  const float* vmax;           // [capacity][16]: max_c |V_i[c, j]|
  uint8_t* zq;                 // [n * KG] activation chunks, int8 planes, UMMA layout
  float* csum;                 // [n * KG][16 * batch] column sums of the dequantised chunk
  uint32_t* flags;             // [n * KG] chunk published at epoch
  float* part;                 // [grid][2][batch][128] partial outputs
  unsigned long long* cnt;     // [m / 128] epoch-tagged arrival counters
  uint32_t* err;               // sticky device error word
  uint32_t* hdr;               // workspace header {epoch, done}: a launch tags its flags and
                               // counters with epoch + 1; the last CTA to exit advances epoch.
                               // Zero before the workspace's first use.
  int m, d, n, KG, RT;
  long long units;             // RT * n * KG
  int stages;                  // shared-memory ring depth
  int x_bf16;
  int inject_unreachable;      // consumers wait for a tag no CTA publishes (timeout test)
  unsigned long long timeout_ns;
};

struct PrefillParams {
  const uint8_t* blocks;
  unsigned long long block_bytes;
  void* y;
  const float* inv_s;
  uint32_t* err;
  int m, d, n, M, KG, NT;
  int xstages, sbufs;
  unsigned long long timeout_ns;
};

// Launchers (decode.cu, prefill.cu, aux_kernels.cu).  They return cudaSuccess or the
// launch error.
cudaError_t launch_decode(const DecodeParams& p, int batch, int grid, int sm_count, cudaStream_t stream);
size_t decode_smem_bytes(int batch, int stages);
int decode_pick_stages(int batch);

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_u,
                           const CUtensorMap& tm_v, int bf16, cudaStream_t stream);
size_t prefill_smem_bytes(int n, int NT, int xstages, int sbufs);

cudaError_t launch_reconstruct(const uint8_t* blocks, unsigned long long block_bytes, const float* inv_s, int m,
                               int d, int n, void* out, int dtype, cudaStream_t stream);
cudaError_t launch_unpack(const uint8_t* record, int m, int d, int8_t* out, cudaStream_t stream);
cudaError_t launch_vmax(const uint8_t* record, int m, int d, float* out16, cudaStream_t stream);

}  // namespace bs

// The handle.  Host memory only.
struct bs_stack_s {
  int m, d, k, capacity, n_blocks;
  uint8_t* blocks;
  size_t block_bytes, dev_bytes;
  const float* inv_s;
  float* vmax;
  uint32_t* err;
  int device, sm_count;
  unsigned long long timeout_ns;
  int inject_unreachable;
  CUtensorMap tm_u, tm_v;  // prefill operand maps over the whole block area
  int tmaps_ready;
};
