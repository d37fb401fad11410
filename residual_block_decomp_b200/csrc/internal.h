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
constexpr int kDecodeMaxBlocks = 64;   // loaded blocks the decode path accepts
constexpr uint32_t kErrTimeout = 1u;   // device error word bit: a bounded wait ran out

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Decode work unit: a segment = one 128-row tile x up to C consecutive 256-column
// chunks of one block (C = decode_chunks_per_segment(batch)); the C chunks of a block
// that share a segment form a chunk group.  Segments are numbered s = cg * RT + rt over
// chunk groups cg = i * NCB + (kg / C) of block i.
__host__ __device__ constexpr int decode_chunks_per_segment(int batch) { return batch == 1 ? 4 : 2; }
inline int decode_groups_per_block(int d, int batch) {
  const int KG = d / kTileCols, C = decode_chunks_per_segment(batch);
  return (KG + C - 1) / C;
}
// Activation operand of one chunk group ("set"), built in shared memory by the decode
// kernel: C chunks of the two int8 planes in the tensor-core operand layout (32 * batch
// operand columns x 256 K-elements, one byte each).
__host__ __device__ constexpr int decode_chunk_operand_bytes(int batch) { return 32 * batch * kTileCols; }

// Decode workspace carve-up (256-byte aligned regions): one arrival counter per row
// tile, then per-segment partial outputs.  The counters come first so that their place
// does not move with n_loaded or batch: a workspace reused by calls with other sizes
// still finds them at zero (every completed call leaves them at zero).
struct DecodeWs {
  size_t cnt, part, total;
};
inline DecodeWs decode_ws_layout(int m, int d, int n, int batch) {
  DecodeWs w{};
  const size_t RT = static_cast<size_t>(m) / kTileRows;
  const size_t segs = RT * static_cast<size_t>(n) * decode_groups_per_block(d, batch);
  size_t off = 0;
  w.cnt = off;  off = align_up(off + RT * sizeof(uint32_t), 256);
  w.part = off; off = align_up(off + segs * batch * kTileRows * sizeof(float), 256);
  w.total = off;
  return w;
}

// One linear of a decode launch.  Segments of all linears of a launch are numbered
// linear after linear (seg0 = the first segment of this linear, cg0 its first chunk group).
struct DecodeLin {
  const uint8_t* blocks;       // record i at blocks + i * block_bytes
  unsigned long long block_bytes;
  const void* x;               // batch x d, f16 or bf16
  void* y;                     // batch x m, same dtype
  const float* inv_s;          // d
  float* part;                 // [segments of this linear][batch][128] partial outputs
  uint32_t* cnt;               // [RT] partials of the row tile that have arrived
  int m, d, n, KG, RT, NCB;    // NCB chunk groups per block
  int seg0, cg0;
};
// A decode launch over G linears at most (kernel parameter block: one linear for
// bs_linear, up to kDecodeGroupMax for bs_linear_group).
constexpr int kDecodeGroupMax = 256;
template <int G>
struct DecodeArgs {
  DecodeLin lin[G];
  int nlin;                    // linears in use, each with at least one segment
  int segs;                    // segments of all linears
  uint32_t* err;               // sticky device error word
  int x_bf16;
  int inject_unreachable;      // CTA 0's first sign copy is never issued (timeout test)
  unsigned long long timeout_ns;
};
using DecodeParams = DecodeArgs<1>;
using DecodeGroupParams = DecodeArgs<kDecodeGroupMax>;
struct PrefillParams {
  const uint8_t* blocks;
  unsigned long long block_bytes;
  void* y;
  const float* inv_s;
  uint32_t* err;
  int m, d, n, M, KG, NT;
  int xstages, sbufs;
  int CN;                      // CTAs per cluster along the tokens sharing the W_hat rebuild (1, 2, 4)
  unsigned long long timeout_ns;
  // Split K (grids that would leave SMs idle): split z takes the K-tiles [z kts, (z + 1) kts)
  // (kts a multiple of 8, the K-tiles of one sign group) and writes an fp32 partial tile;
  // the CTA that counts a tile's last partial sums the ks partials in split order into y.
  int ks, kts, tiles_y;        // splits, K-tiles per split, token tiles that hold tokens
  float* part;                 // [row tile][token tile][split][128 x NT] partial tiles
  uint32_t* cnt;               // [row tile][token tile] arrival counters, zero between calls
};

// Launch shape of the prefill kernel for a call (host side; also sizes its workspace).
struct PrefillConfig {
  int NT, CN, xstages, sbufs;  // token tile, cluster size, x stages, sign buffers
  int ks, kts;                 // K splits and K-tiles per split
  int tiles, gy;               // token tiles holding tokens, and padded to whole clusters
  size_t cnt_bytes, part_bytes;  // workspace: counters (256-aligned), then partials
};
// False when no configuration fits in shared memory (n too large).
bool prefill_config(int m, int d, int n, int batch, int sms, PrefillConfig* cfg);

// "w/o AVD" stacks: blocks that are plain rank-k' factor pairs, record = [U m x k' fp16
// row-major][V d x k' fp16 row-major].  k' is a multiple of 8 (whole 16-byte rows), at
// most kPlainMaxRank; bs_linear takes x in passes of up to kPlainRowsPerPass rows.
constexpr int kPlainMaxRank = 256;
constexpr int kPlainRowsPerPass = 16;
struct PlainWs {
  size_t cnt, t, part, total;   // [n] counters, [n][rows][k'] t, [slices][n][rows][k'] slice parts
};
PlainWs plain_ws_layout(int d, int kp, int n, int batch);
struct PlainParams {
  const uint8_t* blocks;
  unsigned long long block_bytes;
  unsigned long long v_off;    // V inside a record: m * k' * 2
  const void* x;               // batch x d; this pass reads rows row0 .. row0 + nb - 1
  void* y;                     // batch x m, same dtype
  const float* inv_s;
  float* part;
  float* t;
  uint32_t* cnt;
  int m, d, n, kp, row0, nb, x_bf16;
};
cudaError_t launch_plain(const PlainParams& p, cudaStream_t stream);
cudaError_t launch_plain_reconstruct(const uint8_t* blocks, unsigned long long block_bytes, size_t v_off,
                                     const float* inv_s, int m, int d, int kp, int n, void* out, int dtype,
                                     cudaStream_t stream);

// GPU decomposition (decompose.cu): workspace carve-up and arguments.
struct DecomposeWs {
  size_t R, Y, Y2, Z, Z2, Uf, Vf, small, total;
};
DecomposeWs decompose_ws_layout(int m, int d);
struct DecomposeArgs {
  int m, d, n, power_iters;
  const float* W;            // m x d fp32, row-major
  const float* s;            // d fp32: the activation-aware scale
  unsigned long long seed;
  uint8_t* records;          // n records of block_bytes
  unsigned long long block_bytes;
  double* res_norms;         // n + 1 squared Frobenius norms of the scaled residuals
  void* workspace;
};
cudaError_t run_decompose(const DecomposeArgs& a, cudaStream_t stream);

// Launchers (decode.cu, prefill.cu, aux_kernels.cu).  They return cudaSuccess or the
// launch error.
cudaError_t launch_decode(const DecodeParams& p, int batch, int grid, cudaStream_t stream);
cudaError_t launch_decode_group(const DecodeGroupParams& p, int batch, int grid, cudaStream_t stream);
size_t decode_smem_bytes(int batch);

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_u,
                           const CUtensorMap& tm_v, int bf16, cudaStream_t stream);
size_t prefill_smem_bytes(int n, int NT, int xstages, int sbufs, int cn);

// bs_linear_no_alloc keeps its scratch in one array per device, shared by every stack
// on that device: an error reported on any stack marks the device's array for clearing
// before the next no-alloc call there (no_alloc.cu).
void note_device_error(int device);

cudaError_t launch_reconstruct(const uint8_t* blocks, unsigned long long block_bytes, const float* inv_s, int m,
                               int d, int n, void* out, int dtype, cudaStream_t stream);
cudaError_t launch_unpack(const uint8_t* record, int m, int d, int8_t* out, cudaStream_t stream);

}  // namespace bs

// The handle.  Host memory only.
struct bs_stack_s {
  int plain;                   // 1: "w/o AVD" blocks (k holds k'), 0: BitStack blocks
  int m, d, k, capacity, n_blocks;
  uint8_t* blocks;
  size_t block_bytes, dev_bytes;
  const float* inv_s;
  uint32_t* err;
  int device, sm_count;
  unsigned long long timeout_ns;
  int inject_unreachable;
  CUtensorMap tm_u, tm_v;  // prefill operand maps over the whole block area
  int tmaps_ready;
};
