// Host implementation of the C ABI declared in include/bitstack.h: argument checks,
// the stack handle, block append/drop, host packing, and kernel dispatch.  The
// library never allocates device memory; every device buffer comes from the caller.
#include <algorithm>
#include <cstring>
#include <new>

#include "internal.h"

using namespace bs;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr cuuint32_t kKTile = 32;   // K columns per prefill K-tile

bool gpu_shape_ok(int m, int d, int k) {
  return k == kK && m >= kTileRows && d >= kTileCols && m <= 65536 && d <= 65536 && m % kTileRows == 0 &&
         d % kTileCols == 0;
}

// "w/o AVD" stacks: any m, d; k' a multiple of 8 (whole 16-byte factor rows) up to 256.
bool plain_shape_ok(int m, int d, int kp) {
  return m >= 1 && d >= 1 && m <= 65536 && d <= 65536 && kp >= 8 && kp <= kPlainMaxRank && kp % 8 == 0;
}

// After the block area: the stack's device error word (256 bytes reserved).
size_t meta_bytes(int /*capacity*/) { return 256; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor map over a tensor of fp16/bf16 elements; dims / strides innermost first,
// strides in bytes for dims 1.., box in elements.  No swizzle, no interleave.
bool encode(CUtensorMap* map, bool bf16, int rank, void* base, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, static_cast<cuuint32_t>(rank),
         base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool build_factor_maps(bs_stack_s* s) {
  // U: dims {16 (j), m (rows), capacity (blocks)}, box {8, 128, 1}
  // V: dims {16 (j), d (cols), capacity (blocks)}, box {8, 32, 1}
  const cuuint64_t ustr[2] = {kK * 2, static_cast<cuuint64_t>(s->block_bytes)};
  const cuuint64_t udims[3] = {kK, static_cast<cuuint64_t>(s->m), static_cast<cuuint64_t>(s->capacity)};
  const cuuint32_t ubox[3] = {8, kTileRows, 1};
  uint8_t* ubase = s->blocks + static_cast<size_t>(s->m) * s->d / 8;
  const cuuint64_t vdims[3] = {kK, static_cast<cuuint64_t>(s->d), static_cast<cuuint64_t>(s->capacity)};
  const cuuint32_t vbox[3] = {8, 32, 1};
  uint8_t* vbase = ubase + static_cast<size_t>(2) * kK * s->m;
  return encode(&s->tm_u, false, 3, ubase, udims, ustr, ubox) && encode(&s->tm_v, false, 3, vbase, vdims, ustr, vbox);
}

bs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? BS_OK : BS_ERR_CUDA; }

// The per-linear part of a decode launch, without its workspace pointers.
void fill_lin(DecodeLin& L, const bs_stack_s* stack, const void* x, void* y, int n_loaded, int batch) {
  L.blocks = stack->blocks;
  L.block_bytes = stack->block_bytes;
  L.x = x;
  L.y = y;
  L.inv_s = stack->inv_s;
  L.m = stack->m;
  L.d = stack->d;
  L.n = n_loaded;
  L.KG = stack->d / kTileCols;
  L.RT = stack->m / kTileRows;
  L.NCB = decode_groups_per_block(stack->d, batch);
  L.seg0 = 0;
  L.cg0 = 0;
}

// Workspace of a grouped decode launch: all row-tile counters first (their places
// depend only on the shapes, so they stay put as the loaded counts change), then each
// linear's partials.
struct GroupWs {
  size_t cnt_bytes, total;
};
GroupWs group_ws(int n_linears, const bs_stack_t* stacks, const int* n_loaded, int batch) {
  GroupWs g{0, 0};
  for (int l = 0; l < n_linears; ++l) g.cnt_bytes += static_cast<size_t>(stacks[l]->m / kTileRows) * 4;
  g.cnt_bytes = align_up(g.cnt_bytes, 256);
  size_t off = g.cnt_bytes;
  for (int l = 0; l < n_linears; ++l) {
    const size_t segs = static_cast<size_t>(stacks[l]->m / kTileRows) * n_loaded[l] *
                        decode_groups_per_block(stacks[l]->d, batch);
    off = align_up(off + segs * batch * kTileRows * sizeof(float), 256);
  }
  g.total = off;
  return g;
}

}  // namespace

// Token tile: 256 for long inputs, 128 up to 2047 tokens (more CTAs to fill the SMs),
// else the input rounded up to 32.  The CTAs of a row tile are clustered by up to 4 along
// the tokens to share the rebuild of W_hat.  Shared memory: fewer x stages first (down to
// two), then one sign buffer, then smaller token tiles, then a smaller cluster.  A grid
// that would leave SMs idle splits K into as many parts (of whole sign groups) as fit
// beside it in one wave.
bool bs::prefill_config(int m, int d, int n, int batch, int sms, PrefillConfig* c) {
  const size_t limit = 227 * 1024;
  const int NT0 = batch >= 2048 ? 256 : (batch >= 128 ? 128 : ((batch + 31) / 32) * 32);
  const int tiles0 = (batch + NT0 - 1) / NT0;
  int CN = tiles0 >= 4 ? 4 : (tiles0 >= 2 ? 2 : 1);
  int NT = NT0, xs = 4, sb = 2;
  for (;;) {
    xs = 4;
    sb = 2;
    NT = NT0;
    while (prefill_smem_bytes(n, NT, xs, sb, CN) > limit && xs > 2) --xs;
    if (prefill_smem_bytes(n, NT, xs, sb, CN) > limit) sb = 1;
    while (prefill_smem_bytes(n, NT, xs, sb, CN) > limit && NT > 32) NT /= 2;
    if (prefill_smem_bytes(n, NT, xs, sb, CN) <= limit) break;
    if (CN == 1) return false;
    CN /= 2;
  }
  c->NT = NT;
  c->CN = CN;
  c->xstages = xs;
  c->sbufs = sb;
  c->tiles = (batch + NT - 1) / NT;
  c->gy = (c->tiles + CN - 1) / CN * CN;
  const int KT = d / 32;   // 32-column K-tiles (a multiple of 8: d is a multiple of 256)
  const long long ctas = static_cast<long long>(m / kTileRows) * c->gy;
  int ks = 1;
  if (sms > 0 && ctas < sms) ks = std::min(static_cast<int>(sms / ctas), (KT + 7) / 8);
  int kts = ((KT + ks - 1) / ks + 7) / 8 * 8;
  ks = (KT + kts - 1) / kts;
  c->ks = ks;
  c->kts = kts;
  const size_t tiles_all = static_cast<size_t>(m / kTileRows) * c->tiles;
  c->cnt_bytes = ks > 1 ? (tiles_all * 4 + 255) / 256 * 256 : 0;
  c->part_bytes = ks > 1 ? static_cast<size_t>(ks) * tiles_all * kTileRows * NT * 4 : 0;
  return true;
}

extern "C" {

size_t bs_block_bytes(int m, int d, int k) {
  if (m <= 0 || d <= 0 || k <= 0 || d % 8 != 0) return 0;
  return static_cast<size_t>(m) * d / 8 + static_cast<size_t>(2) * k * (static_cast<size_t>(m) + d);
}

size_t bs_stack_device_bytes(int m, int d, int k, int capacity_blocks) {
  if (!gpu_shape_ok(m, d, k) || capacity_blocks <= 0) return 0;
  return align_up(static_cast<size_t>(capacity_blocks) * bs_block_bytes(m, d, k), 256) + meta_bytes(capacity_blocks);
}

size_t bs_workspace_bytes(int m, int d, int k, int n_loaded, int batch) {
  if (!gpu_shape_ok(m, d, k) || n_loaded < 0 || batch <= 0) return 0;
  if (n_loaded == 0) return 0;
  if (batch <= kDecodeMaxBatch) return decode_ws_layout(m, d, n_loaded, batch).total;
  // the prefill's split-K partials, for the current device's SM count (148 without one)
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  PrefillConfig cfg;
  if (!prefill_config(m, d, n_loaded, batch, sms, &cfg)) return 0;
  return cfg.cnt_bytes + cfg.part_bytes;
}

bs_status bs_pack_record(int m, int d, int k, const uint8_t* neg_bits, const uint16_t* U, const uint16_t* V,
                         void* record) {
  if (neg_bits == nullptr || U == nullptr || V == nullptr || record == nullptr || k <= 0) return BS_ERR_INVALID_ARG;
  if (m <= 0 || d <= 0 || m % kTileRows != 0 || d % kTileCols != 0) return BS_ERR_UNSUPPORTED_SHAPE;
  uint8_t* out = static_cast<uint8_t*>(record);
  const size_t row_bytes = static_cast<size_t>(d) / 8;
  const int RT = m / kTileRows, KG = d / kTileCols;
  for (int rt = 0; rt < RT; ++rt) {
    for (int g = 0; g < KG; ++g) {
      uint8_t* tile = out + (static_cast<size_t>(rt) * KG + g) * kTileBytes;
      for (int rr = 0; rr < kTileRows; ++rr) {
        const uint8_t* src = neg_bits + static_cast<size_t>(rt * kTileRows + rr) * row_bytes;
        for (int pw = 0; pw < 8; ++pw) {
          uint32_t word = 0;
          for (int q = 0; q < 4; ++q) {
            for (int t = 0; t < 8; ++t) {
              const int c = g * kTileCols + 32 * t + 4 * pw + q;
              const uint32_t bit = (src[c >> 3] >> (c & 7)) & 1u;
              word |= bit << (8 * q + t);
            }
          }
          const size_t widx = static_cast<size_t>(pw >> 2) * 512 + static_cast<size_t>(rr) * 4 + (pw & 3);
          const uint8_t le[4] = {static_cast<uint8_t>(word), static_cast<uint8_t>(word >> 8),
                                 static_cast<uint8_t>(word >> 16), static_cast<uint8_t>(word >> 24)};
          std::memcpy(tile + widx * 4, le, 4);
        }
      }
    }
  }
  const size_t nsb = static_cast<size_t>(m) * d / 8;
  std::memcpy(out + nsb, U, static_cast<size_t>(m) * k * 2);
  std::memcpy(out + nsb + static_cast<size_t>(m) * k * 2, V, static_cast<size_t>(d) * k * 2);
  return BS_OK;
}

}  // extern "C"

namespace {

bs_status create_stack(int plain, int m, int d, int k, int capacity_blocks, void* dev_blocks, size_t dev_bytes,
                       const float* dev_inv_scale, bs_stream_t stream, bs_stack_t* out) {
  if (out == nullptr || dev_blocks == nullptr || dev_inv_scale == nullptr || capacity_blocks <= 0)
    return BS_ERR_INVALID_ARG;
  *out = nullptr;
  if (plain ? !plain_shape_ok(m, d, k) : !gpu_shape_ok(m, d, k)) return BS_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(dev_blocks, 256) || !aligned(dev_inv_scale, 16)) return BS_ERR_ALIGNMENT;
  const size_t need = plain ? bs_plain_stack_device_bytes(m, d, k, capacity_blocks)
                            : bs_stack_device_bytes(m, d, k, capacity_blocks);
  if (dev_bytes < need) return BS_ERR_CAPACITY;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BS_ERR_NO_DEVICE;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return BS_ERR_NO_DEVICE;
  if (major != 10 || minor != 0) return BS_ERR_NO_DEVICE;
  bs_stack_s* s = new (std::nothrow) bs_stack_s();
  if (s == nullptr) return BS_ERR_INVALID_ARG;
  s->plain = plain;
  s->m = m;
  s->d = d;
  s->k = k;
  s->capacity = capacity_blocks;
  s->n_blocks = 0;
  s->blocks = static_cast<uint8_t*>(dev_blocks);
  s->block_bytes = plain ? bs_plain_block_bytes(m, d, k) : bs_block_bytes(m, d, k);
  s->dev_bytes = dev_bytes;
  s->inv_s = dev_inv_scale;
  s->err = reinterpret_cast<uint32_t*>(s->blocks + align_up(static_cast<size_t>(capacity_blocks) * s->block_bytes, 256));
  s->device = dev;
  s->sm_count = sms;
  s->timeout_ns = 500000000ull;
  s->inject_unreachable = 0;
  s->tmaps_ready = plain ? 0 : (build_factor_maps(s) ? 1 : 0);
  const cudaError_t e = cudaMemsetAsync(s->err, 0, meta_bytes(capacity_blocks), stream);
  if (e != cudaSuccess) {
    delete s;
    return BS_ERR_CUDA;
  }
  *out = s;
  return BS_OK;
}

// bs_linear for a "w/o AVD" stack: x in passes of up to kPlainRowsPerPass rows.
bs_status plain_linear(bs_stack_t stack, const void* x, int batch, bs_dtype dt, int n_loaded, void* y,
                       void* workspace, size_t workspace_bytes, bs_stream_t stream) {
  const PlainWs L = plain_ws_layout(stack->d, stack->k, n_loaded, batch);
  if (workspace == nullptr || workspace_bytes < L.total) return BS_ERR_CAPACITY;
  if (!aligned(workspace, 256)) return BS_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  PlainParams p{};
  p.blocks = stack->blocks;
  p.block_bytes = stack->block_bytes;
  p.v_off = static_cast<unsigned long long>(stack->m) * stack->k * 2;
  p.x = x;
  p.y = y;
  p.inv_s = stack->inv_s;
  p.part = reinterpret_cast<float*>(ws + L.part);
  p.t = reinterpret_cast<float*>(ws + L.t);
  p.cnt = reinterpret_cast<uint32_t*>(ws + L.cnt);
  p.m = stack->m;
  p.d = stack->d;
  p.n = n_loaded;
  p.kp = stack->k;
  p.x_bf16 = dt == BS_BF16 ? 1 : 0;
  for (int row0 = 0; row0 < batch; row0 += kPlainRowsPerPass) {
    p.row0 = row0;
    p.nb = batch - row0 < kPlainRowsPerPass ? batch - row0 : kPlainRowsPerPass;
    const cudaError_t e = launch_plain(p, stream);
    if (e != cudaSuccess) return BS_ERR_CUDA;
  }
  return BS_OK;
}

}  // namespace

extern "C" {

bs_status bs_stack_create(int m, int d, int k, int capacity_blocks, void* dev_blocks, size_t dev_bytes,
                          const float* dev_inv_scale, bs_stream_t stream, bs_stack_t* out) {
  return create_stack(0, m, d, k, capacity_blocks, dev_blocks, dev_bytes, dev_inv_scale, stream, out);
}

int bs_plain_rank(int m, int d, int k) {
  if (m <= 0 || d <= 0 || k <= 0) return 0;
  const long long kp = k + (static_cast<long long>(m) * d) / (16ll * (static_cast<long long>(m) + d));
  return static_cast<int>(kp - kp % 8);
}

size_t bs_plain_block_bytes(int m, int d, int k_prime) {
  if (!plain_shape_ok(m, d, k_prime)) return 0;
  return static_cast<size_t>(2) * k_prime * (static_cast<size_t>(m) + d);
}

size_t bs_plain_stack_device_bytes(int m, int d, int k_prime, int capacity_blocks) {
  if (!plain_shape_ok(m, d, k_prime) || capacity_blocks <= 0) return 0;
  return align_up(static_cast<size_t>(capacity_blocks) * bs_plain_block_bytes(m, d, k_prime), 256) +
         meta_bytes(capacity_blocks);
}

size_t bs_plain_workspace_bytes(int m, int d, int k_prime, int n_loaded, int batch) {
  if (!plain_shape_ok(m, d, k_prime) || n_loaded <= 0 || batch <= 0) return 0;
  return plain_ws_layout(d, k_prime, n_loaded, batch).total;
}

bs_status bs_plain_stack_create(int m, int d, int k_prime, int capacity_blocks, void* dev_blocks, size_t dev_bytes,
                                const float* dev_inv_scale, bs_stream_t stream, bs_stack_t* out) {
  return create_stack(1, m, d, k_prime, capacity_blocks, dev_blocks, dev_bytes, dev_inv_scale, stream, out);
}

bs_status bs_stack_destroy(bs_stack_t stack) {
  if (stack == nullptr) return BS_ERR_INVALID_ARG;
  delete stack;
  return BS_OK;
}

bs_status bs_stack_num_blocks(bs_stack_t stack, int* n_blocks) {
  if (stack == nullptr || n_blocks == nullptr) return BS_ERR_INVALID_ARG;
  *n_blocks = stack->n_blocks;
  return BS_OK;
}

bs_status bs_append_block(bs_stack_t stack, const void* host_record, bs_stream_t stream) {
  if (stack == nullptr || host_record == nullptr) return BS_ERR_INVALID_ARG;
  if (stack->n_blocks >= stack->capacity) return BS_ERR_CAPACITY;
  uint8_t* slot = stack->blocks + static_cast<size_t>(stack->n_blocks) * stack->block_bytes;
  const cudaError_t e = cudaMemcpyAsync(slot, host_record, stack->block_bytes, cudaMemcpyDefault, stream);
  if (e != cudaSuccess) return BS_ERR_CUDA;
  stack->n_blocks += 1;
  return BS_OK;
}

bs_status bs_drop_block(bs_stack_t stack) {
  if (stack == nullptr) return BS_ERR_INVALID_ARG;
  if (stack->n_blocks <= 0) return BS_ERR_RANGE;
  stack->n_blocks -= 1;
  return BS_OK;
}

bs_status bs_linear(bs_stack_t stack, const void* x, int batch, bs_dtype dt, int n_loaded, void* y,
                    void* workspace, size_t workspace_bytes, bs_stream_t stream) {
  if (stack == nullptr || x == nullptr || y == nullptr || batch <= 0) return BS_ERR_INVALID_ARG;
  if (dt != BS_F16 && dt != BS_BF16) return BS_ERR_INVALID_ARG;
  if (n_loaded < 0 || n_loaded > stack->n_blocks) return BS_ERR_RANGE;
  if (!aligned(x, 16) || !aligned(y, 16)) return BS_ERR_ALIGNMENT;
  const int m = stack->m, d = stack->d;
  if (n_loaded == 0) return cuda_status(cudaMemsetAsync(y, 0, static_cast<size_t>(batch) * m * 2, stream));
  if (stack->plain) return plain_linear(stack, x, batch, dt, n_loaded, y, workspace, workspace_bytes, stream);

  if (batch <= kDecodeMaxBatch) {
    if (n_loaded > kDecodeMaxBlocks) return BS_ERR_RANGE;
    const DecodeWs W = decode_ws_layout(m, d, n_loaded, batch);
    if (workspace == nullptr || workspace_bytes < W.total) return BS_ERR_CAPACITY;
    if (!aligned(workspace, 256)) return BS_ERR_ALIGNMENT;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecodeParams p{};
    DecodeLin& L = p.lin[0];
    fill_lin(L, stack, x, y, n_loaded, batch);
    L.part = reinterpret_cast<float*>(ws + W.part);
    L.cnt = reinterpret_cast<uint32_t*>(ws + W.cnt);
    const long long segs = static_cast<long long>(L.RT) * n_loaded * L.NCB;
    if (segs > (1ll << 30)) return BS_ERR_UNSUPPORTED_SHAPE;
    p.nlin = 1;
    p.segs = static_cast<int>(segs);
    p.err = stack->err;
    p.x_bf16 = dt == BS_BF16 ? 1 : 0;
    p.inject_unreachable = stack->inject_unreachable;
    stack->inject_unreachable = 0;
    p.timeout_ns = stack->timeout_ns;
    // One CTA per SM, with a few SMs left over: calls chained on a stream start while the
    // CTAs of the call ahead that add its last partials still reduce and write y, so the
    // next call's CTAs find free SMs at once instead of queueing behind them.
    const int slack = stack->sm_count > 32 ? 4 : 0;
    const int ctas = stack->sm_count - slack;
    const int grid = segs < ctas ? static_cast<int>(segs) : ctas;
    return cuda_status(launch_decode(p, batch, grid, stream));
  }

  // prefill: W_hat tiles rebuilt in shared memory, tcgen05 GEMM
  if (!stack->tmaps_ready) return BS_ERR_CUDA;
  PrefillParams p{};
  p.blocks = stack->blocks;
  p.block_bytes = stack->block_bytes;
  p.y = y;
  p.inv_s = stack->inv_s;
  p.err = stack->err;
  p.m = m;
  p.d = d;
  p.n = n_loaded;
  p.M = batch;
  p.KG = d / kTileCols;
  p.timeout_ns = stack->timeout_ns;
  PrefillConfig cfg;
  if (!prefill_config(m, d, n_loaded, batch, stack->sm_count, &cfg)) return BS_ERR_CAPACITY;
  p.NT = cfg.NT;
  p.CN = cfg.CN;
  p.xstages = cfg.xstages;
  p.sbufs = cfg.sbufs;
  p.tiles_y = cfg.tiles;
  p.ks = 1;
  p.kts = d / 32;           // one split: all 32-column K-tiles
  // split K only with a workspace that holds the partials (else one pass over K)
  if (cfg.ks > 1 && workspace != nullptr && workspace_bytes >= cfg.cnt_bytes + cfg.part_bytes) {
    if (!aligned(workspace, 256)) return BS_ERR_ALIGNMENT;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.ks = cfg.ks;
    p.kts = cfg.kts;
    p.cnt = reinterpret_cast<uint32_t*>(ws);
    p.part = reinterpret_cast<float*>(ws + cfg.cnt_bytes);
  }
  CUtensorMap tm_x;
  const cuuint64_t xdims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(batch)};
  const cuuint64_t xstr[1] = {static_cast<cuuint64_t>(d) * 2};
  // one 32-column K-tile of NT tokens per copy: rows of 64 bytes in the 64-byte swizzle
  // layout the GEMM reads x in
  const cuuint32_t xbox[2] = {kKTile, static_cast<cuuint32_t>(p.NT)};
  if (!encode(&tm_x, dt == BS_BF16, 2, const_cast<void*>(x), xdims, xstr, xbox, CU_TENSOR_MAP_SWIZZLE_64B))
    return BS_ERR_CUDA;
  return cuda_status(launch_prefill(p, tm_x, stack->tm_u, stack->tm_v, dt == BS_BF16 ? 1 : 0, stream));
}

size_t bs_group_workspace_bytes(int n_linears, const bs_stack_t* stacks, const int* n_loaded, int batch) {
  if (n_linears <= 0 || n_linears > kDecodeGroupMax || stacks == nullptr || n_loaded == nullptr || batch <= 0 ||
      batch > kDecodeMaxBatch)
    return 0;
  for (int l = 0; l < n_linears; ++l)
    if (stacks[l] == nullptr || stacks[l]->plain || n_loaded[l] < 0) return 0;
  return group_ws(n_linears, stacks, n_loaded, batch).total;
}

bs_status bs_linear_group(int n_linears, const bs_stack_t* stacks, const void* const* x, void* const* y,
                          const int* n_loaded, int batch, bs_dtype dt, void* workspace, size_t workspace_bytes,
                          bs_stream_t stream) {
  if (n_linears <= 0 || n_linears > kDecodeGroupMax || stacks == nullptr || x == nullptr || y == nullptr ||
      n_loaded == nullptr || batch <= 0 || batch > kDecodeMaxBatch)
    return BS_ERR_INVALID_ARG;
  if (dt != BS_F16 && dt != BS_BF16) return BS_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BS_ERR_NO_DEVICE;
  for (int l = 0; l < n_linears; ++l) {
    const bs_stack_s* st = stacks[l];
    if (st == nullptr || st->plain || x[l] == nullptr || y[l] == nullptr || st->device != dev) return BS_ERR_INVALID_ARG;
    if (n_loaded[l] < 0 || n_loaded[l] > st->n_blocks || n_loaded[l] > kDecodeMaxBlocks) return BS_ERR_RANGE;
    if (!aligned(x[l], 16) || !aligned(y[l], 16)) return BS_ERR_ALIGNMENT;
  }
  const GroupWs W = group_ws(n_linears, stacks, n_loaded, batch);
  if (workspace == nullptr || workspace_bytes < W.total) return BS_ERR_CAPACITY;
  if (!aligned(workspace, 256)) return BS_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the table is ~22 KB: keep it off the thread's stack
  static thread_local DecodeGroupParams p;
  p = DecodeGroupParams{};
  size_t cnt_off = 0, part_off = W.cnt_bytes;
  long long segs = 0;
  int cgs = 0, nlin = 0;
  for (int l = 0; l < n_linears; ++l) {
    const bs_stack_s* st = stacks[l];
    const size_t RT = static_cast<size_t>(st->m / kTileRows);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(ws + cnt_off);
    cnt_off += RT * 4;
    if (n_loaded[l] == 0) {   // no blocks: y is zero
      const cudaError_t e = cudaMemsetAsync(y[l], 0, static_cast<size_t>(batch) * st->m * 2, stream);
      if (e != cudaSuccess) return BS_ERR_CUDA;
      continue;
    }
    DecodeLin& L = p.lin[nlin++];
    fill_lin(L, st, x[l], y[l], n_loaded[l], batch);
    L.cnt = cnt;
    L.part = reinterpret_cast<float*>(ws + part_off);
    const long long ls = static_cast<long long>(L.RT) * L.n * L.NCB;
    part_off = align_up(part_off + static_cast<size_t>(ls) * batch * kTileRows * sizeof(float), 256);
    L.seg0 = static_cast<int>(segs);
    L.cg0 = cgs;
    segs += ls;
    cgs += L.n * L.NCB;
    if (segs > (1ll << 30)) return BS_ERR_UNSUPPORTED_SHAPE;
  }
  if (nlin == 0) return BS_OK;
  p.nlin = nlin;
  p.segs = static_cast<int>(segs);
  p.err = stacks[0]->err;
  p.x_bf16 = dt == BS_BF16 ? 1 : 0;
  p.inject_unreachable = 0;
  p.timeout_ns = stacks[0]->timeout_ns;
  const int slack = stacks[0]->sm_count > 32 ? 4 : 0;
  const int ctas = stacks[0]->sm_count - slack;
  const int grid = segs < ctas ? static_cast<int>(segs) : ctas;
  return cuda_status(launch_decode_group(p, batch, grid, stream));
}

size_t bs_decompose_workspace_bytes(int m, int d, int k) {
  if (!gpu_shape_ok(m, d, k)) return 0;
  return decompose_ws_layout(m, d).total;
}

bs_status bs_decompose(int m, int d, int k, int n_blocks, const float* W, const float* s, unsigned long long seed,
                       int power_iters, void* records, size_t records_bytes, double* res_norms_sq, void* workspace,
                       size_t workspace_bytes, bs_stream_t stream) {
  if (W == nullptr || s == nullptr || records == nullptr || res_norms_sq == nullptr || workspace == nullptr ||
      n_blocks <= 0 || n_blocks > 4096 || power_iters < 0 || power_iters > 64)
    return BS_ERR_INVALID_ARG;
  if (!gpu_shape_ok(m, d, k)) return BS_ERR_UNSUPPORTED_SHAPE;
  const size_t bb = bs_block_bytes(m, d, k);
  if (records_bytes < bb * static_cast<size_t>(n_blocks) || workspace_bytes < decompose_ws_layout(m, d).total)
    return BS_ERR_CAPACITY;
  if (!aligned(records, 256) || !aligned(workspace, 256) || !aligned(W, 16) || !aligned(s, 16) ||
      !aligned(res_norms_sq, 8))
    return BS_ERR_ALIGNMENT;
  DecomposeArgs a{};
  a.m = m;
  a.d = d;
  a.n = n_blocks;
  a.power_iters = power_iters;
  a.W = W;
  a.s = s;
  a.seed = seed;
  a.records = static_cast<uint8_t*>(records);
  a.block_bytes = bb;
  a.res_norms = res_norms_sq;
  a.workspace = workspace;
  return cuda_status(run_decompose(a, stream));
}

bs_status bs_reconstruct(bs_stack_t stack, int n, void* W_out, bs_dtype dt, bs_stream_t stream) {
  if (stack == nullptr || W_out == nullptr) return BS_ERR_INVALID_ARG;
  if (dt != BS_F16 && dt != BS_BF16 && dt != BS_F32) return BS_ERR_INVALID_ARG;
  if (n < 0 || n > stack->n_blocks) return BS_ERR_RANGE;
  if (!aligned(W_out, 16)) return BS_ERR_ALIGNMENT;
  const size_t elems = static_cast<size_t>(stack->m) * stack->d;
  if (n == 0) return cuda_status(cudaMemsetAsync(W_out, 0, elems * (dt == BS_F32 ? 4 : 2), stream));
  if (stack->plain)
    return cuda_status(launch_plain_reconstruct(stack->blocks, stack->block_bytes,
                                                static_cast<size_t>(stack->m) * stack->k * 2, stack->inv_s, stack->m,
                                                stack->d, stack->k, n, W_out, dt, stream));
  return cuda_status(
      launch_reconstruct(stack->blocks, stack->block_bytes, stack->inv_s, stack->m, stack->d, n, W_out, dt, stream));
}

bs_status bs_unpack_signs(bs_stack_t stack, int block, int8_t* out, bs_stream_t stream) {
  if (stack == nullptr || out == nullptr || stack->plain) return BS_ERR_INVALID_ARG;
  if (block < 0 || block >= stack->n_blocks) return BS_ERR_RANGE;
  return cuda_status(launch_unpack(stack->blocks + static_cast<size_t>(block) * stack->block_bytes, stack->m,
                                   stack->d, out, stream));
}

bs_status bs_get_device_error(bs_stack_t stack) {
  if (stack == nullptr) return BS_ERR_INVALID_ARG;
  uint32_t v = 0;
  if (cudaMemcpy(&v, stack->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return BS_ERR_CUDA;
  if (v == 0) return BS_OK;
  bs::note_device_error(stack->device);
  if (cudaMemset(stack->err, 0, sizeof(v)) != cudaSuccess) return BS_ERR_CUDA;
  return (v & kErrTimeout) ? BS_ERR_TIMEOUT : BS_ERR_CUDA;
}

const char* bs_status_string(bs_status status) {
  switch (status) {
    case BS_OK: return "ok";
    case BS_ERR_INVALID_ARG: return "invalid argument";
    case BS_ERR_UNSUPPORTED_SHAPE:
      return "unsupported shape (BitStack blocks: m % 128 == 0, d % 256 == 0, k == 16; plain blocks: k' a multiple "
             "of 8 up to 256)";
    case BS_ERR_ALIGNMENT: return "misaligned pointer";
    case BS_ERR_CAPACITY: return "capacity or buffer size exceeded";
    case BS_ERR_RANGE: return "block count or index out of range";
    case BS_ERR_CUDA: return "CUDA error";
    case BS_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case BS_ERR_NO_DEVICE: return "no usable sm_100 device";
  }
  return "unknown status";
}

bs_status bs_debug_set_wait(bs_stack_t stack, long long timeout_ns, int unreachable_flag) {
  if (stack == nullptr || timeout_ns <= 0) return BS_ERR_INVALID_ARG;
  stack->timeout_ns = static_cast<unsigned long long>(timeout_ns < 1000 ? 1000 : timeout_ns);
  stack->inject_unreachable = unreachable_flag ? 1 : 0;
  return BS_OK;
}

}  // extern "C"
