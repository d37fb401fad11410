// Decode kernel of the BitStack linear: y = sum_i U_i (S_i ((x (.) 1/s) (.) V_i)).
//
// The weight of a BitStack layer is the sum of the loaded residual blocks, each a
// +-1 sign matrix times the rank-k product of its singular vectors, with the
// activation-aware scale undone per input channel (weight restoration snippet of the
// OpenReview discussion of "BitStack: Any-Size Compression of Large Language Models in
// Variable Memory Environments"; review page "BitStack: Fine-Grained Size Control...",
// Figs. 3 and 5).  For a few rows of x the kernel never forms that weight: by
// associativity  y[b, r] = sum_i sum_j U_i[r, j] T_i[r, (j, b)],
// T_i = S_i Z_i,  Z_i[c, (j, b)] = x[b, c] / s_c * V_i[c, j],  a +-1 contraction with
// N = 16 * batch columns per block.
//
// How it maps to sm_100a:
//  * Work is cut into segments: one 128-row tile of one block times C consecutive
//    256-column chunks (C = 4 for one row of x, 2 for more).  Segments are numbered
//    chunk-group-major (s = cg * RT + rt) and every CTA of the persistent grid takes
//    a contiguous run of them, so a CTA touches one or two chunk groups.
//  * Each CTA quantises the activation chunks of its own chunk groups (no exchange
//    between CTAs): Z = (x / s) (.) V for the group's columns, per column (b, j) a
//    step sigma = max |Z| / 32512 over the group, q = rint(Z / sigma) split exactly
//    into two int8 planes q = 256 hi + lo.  So S_i Z_i runs on the int8 tensor cores
//    (tcgen05.mma kind::i8) with exact int32 accumulation.  S = 1 - 2 Sb with Sb in
//    {0, 1} the stored bit; the 1 part is the group's column sum, added in the epilogue.
//  * Sign tiles (4 KiB per 128 x 256 unit, contiguous along a segment) stream from HBM
//    by one 1-D bulk copy per segment into a ring of shared-memory stages.  Eight
//    expander warps, two teams taking alternate unit pairs, turn each row's sign bits
//    into u8 operands in registers (K-step t = bit t of every byte, one shift and one
//    AND per 4 columns) and store them to a ring of A-buffer pairs in tensor memory
//    (tcgen05.st).  Four threads in four warps issue the MMAs (K-steps w and w + 4 of
//    every unit) into the segment's accumulator, which the epilogue zeroes after
//    reading it, so every MMA accumulates; the two accumulators alternate between
//    segments.  Expanders hand pairs to the issuers, and the epilogue hands
//    accumulators back, through per-warp release counters in shared memory; MMA
//    completion comes back through tcgen05.commit to mbarriers.
//  * The epilogue (four more warps) turns a segment's accumulator into one partial
//    output per row and batch row, with the row's U_i entries from a ring of U tiles.
//    When a CTA is done it counts its segments into per-row-tile counters; CTA rt mod
//    grid waits for all partials of row tile rt, sums them in fixed chunk-group order
//    (deterministic), writes y and resets the counter.
//  * The launch allows programmatic dependent launch: the prologue (barriers, TMEM,
//    the first sign copies, V rows) runs before the previous kernel in the stream has
//    finished; x, s, the workspace and y are touched only after griddepcontrol.wait.
//  * Every wait is bounded; a wait that runs out sets the device error word, and the
//    CTA drains its copies and MMAs, frees tensor memory and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace bs {
namespace {

constexpr int kThreads = 544;   // 17 warps
constexpr int kExpWarps = 8;    // warps 0..7: sign expanders, two teams of four (alternate unit pairs)
constexpr int kWarpEpi0 = 8;    // warps 8..11: epilogue and activation-chunk production
constexpr int kWarpIss0 = 12;   // warps 12..15: MMA issuers (lane 0 each)
constexpr int kWarpCopy = 16;   // sign-tile copies; allocates TMEM
constexpr int kNI = 4;          // MMA issuers: issuer w issues K-steps w and w + 4 of every unit
constexpr int kMaxStages = 16;
constexpr int kBarProd = 1;     // named barrier: warps 8-15 (the first chunk group)
constexpr int kBarEpi = 2;      // named barrier: warps 8-11
constexpr int kGroup = 2;       // units per A-buffer pair (the hand-over granularity)
constexpr int kSmemLimit = 227 * 1024;
constexpr int kSetHdr = 512;    // per chunk-group set: sigma_lo[64], column sums[64]
constexpr int kURing = 4;       // U tiles (4 KiB each) in flight ahead of the epilogue
constexpr int kMaxPairs = 3;    // A-buffer pairs in tensor memory (one batch row: 3)

struct Ctl {
  uint64_t sfull[kMaxStages], sempty[kMaxStages];
  uint64_t ufull[kURing];
  uint64_t aempty[kMaxPairs];   // A-buffer pair free again: the MMAs that read it completed
  uint64_t accfull[2], zfull[2], drain[4];
  uint64_t vfull;         // V rows of the first chunk group
  uint32_t a_ready[kExpWarps];  // A-buffer pairs stored, per expander warp (a sum could let
                                // a fast warp stand in for a slow one)
  uint32_t acc_free[2];   // accumulator zeroed by the epilogue: +1 per epilogue warp per release
  uint32_t tmem_base;
  int abort;
  int abort_snap;
  int red_ok;
  int amaxi[16 * kDecodeMaxBatch];   // max |Z| per column (float bits; values >= 0)
  int zsum[16 * kDecodeMaxBatch];    // sum of q per column
};

template <int B>
struct Cfg {
  static constexpr int NB = 32 * B;                 // MMA N: [hi plane 16B | lo plane 16B]
  static constexpr int ZB = NB * kTileCols;         // operand bytes of one chunk
  // Tensor memory: two accumulators of NB columns (double buffered across segments),
  // then the A-buffer ring, 64 columns (128 lanes x 256 bytes) per unit, in pairs.
  static constexpr uint32_t ACOL0 = 2 * NB;
  static constexpr int NPAIRS = (512 - 2 * NB) / (64 * kGroup);
  static constexpr int C = decode_chunks_per_segment(B);
  static constexpr int COLS = C * kTileCols;        // columns of a chunk group
  static constexpr int SET = kSetHdr + C * ZB;      // one chunk-group set
  static constexpr int VSCR = COLS * kK * 2;        // V rows of a group (fp16)
  static constexpr int XSCR = COLS * B * 2 + COLS * 4;   // x rows (fp16/bf16), then 1/s (fp32)
  static constexpr int XSF = COLS * B * 4;          // x (.) 1/s of the group (fp32)
  static constexpr int URING = kURing * kTileBytes; // U rows of a row tile (128 x 16 fp16) per slot
  static constexpr int STAGE = C * kTileBytes;
  static constexpr int CTL = static_cast<int>((sizeof(Ctl) + 127) / 128 * 128);
  static constexpr int FIXED = 2 * SET + VSCR + XSCR + XSF + URING + CTL;
  static constexpr int NS0 = (kSmemLimit - FIXED) / STAGE;
  static constexpr int NS = NS0 < kMaxStages ? NS0 : kMaxStages;
  static constexpr int SMEM = NS * STAGE + FIXED;
  static_assert(NS >= 2, "sign ring too small");
  static_assert(NPAIRS >= 2 && NPAIRS <= kMaxPairs, "A-buffer ring");
  static_assert(XSCR % 128 == 0 && VSCR % 128 == 0 && XSF % 128 == 0, "scratch alignment");
};

struct Seg {
  int i, rt, kgA, len, cg;
};
__device__ __forceinline__ Seg seg_of(int s, const DecodeParams& p, int C) {
  Seg g;
  g.cg = s / p.RT;
  g.rt = s - g.cg * p.RT;
  g.i = g.cg / p.NCB;
  g.kgA = (g.cg - g.i * p.NCB) * C;
  g.len = min(C, p.KG - g.kgA);
  return g;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void store_y(void* y, int bf16, size_t idx, float v) {
  if (bf16) static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(y)[idx] = __float2half_rn(v);
}
__device__ __forceinline__ float x_at(const uint16_t* xr, int bf16, int idx) {
  const uint16_t h = xr[idx];
  return bf16 ? __uint_as_float(static_cast<uint32_t>(h) << 16) : __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ void set_error(const DecodeParams& p, Ctl* ctl) {
  ctl->abort = 1;
  atomicOr(p.err, kErrTimeout);
}

// Byte addresses of a chunk group's inputs in the stack and in x.
__device__ __forceinline__ const uint8_t* v_rows(const DecodeParams& p, const Seg& sg) {
  return p.blocks + static_cast<size_t>(sg.i) * p.block_bytes + static_cast<size_t>(p.m) * p.d / 8 +
         static_cast<size_t>(2) * kK * p.m + static_cast<size_t>(sg.kgA) * kTileCols * kK * 2;
}
__device__ __forceinline__ const uint8_t* u_tile(const DecodeParams& p, int i, int rt) {
  return p.blocks + static_cast<size_t>(i) * p.block_bytes + static_cast<size_t>(p.m) * p.d / 8 +
         static_cast<size_t>(rt) * kTileRows * kK * 2;
}

// Loads the inputs of chunk group `sg` into the scratch with plain loads (the later
// groups of a CTA; the first one arrives by bulk copies).  Called by the 128 epilogue
// threads after griddep_wait.
template <int B>
__device__ void load_set_inputs(const DecodeParams& p, uint8_t* vscr, uint8_t* xscr, const Seg& sg, int tid) {
  using K = Cfg<B>;
  const int cols = sg.len * kTileCols, col0 = sg.kgA * kTileCols;
  const uint4* vsrc = reinterpret_cast<const uint4*>(v_rows(p, sg));
  for (int v = tid; v < cols * 2; v += 128) reinterpret_cast<uint4*>(vscr)[v] = __ldg(vsrc + v);
  uint16_t* xr = reinterpret_cast<uint16_t*>(xscr);
  for (int idx = tid; idx < B * cols; idx += 128) {
    const int b = idx / cols, c = idx - b * cols;
    xr[b * K::COLS + c] = static_cast<const uint16_t*>(p.x)[static_cast<size_t>(b) * p.d + col0 + c];
  }
  float* isv = reinterpret_cast<float*>(xscr + K::COLS * B * 2);
  for (int c = tid; c < cols; c += 128) isv[c] = __ldg(p.inv_s + col0 + c);
}

// Quantises the activation chunks of chunk group `sg` (inputs already in the scratch:
// V rows, x rows, 1/s) into `set`: operand planes in the UMMA no-swizzle K-major
// layout, the per-column step sigma_lo and the dequantised column sum.  Run by NT
// threads that share named barrier `bar`; it has no other wait, so every thread passes
// the same barriers.  `zfull` is signalled unless `skip`.
template <int B, int NT>
__device__ void produce_set(uint8_t* set, const uint8_t* vscr, const uint8_t* xscr, float* xsf, int bf16, Ctl* ctl,
                            const Seg& sg, int tid, int bar, uint64_t* zfull, bool skip) {
  using K = Cfg<B>;
  const int cols = sg.len * kTileCols;
  const __half* vh = reinterpret_cast<const __half*>(vscr);
  const uint16_t* xr = reinterpret_cast<const uint16_t*>(xscr);
  const float* isv = reinterpret_cast<const float*>(xscr + K::COLS * B * 2);
  // x' = x (.) 1/s, once per column and batch row
  for (int idx = tid; idx < B * cols; idx += NT) {
    const int b = idx / cols, c = idx - b * cols;
    xsf[b * K::COLS + c] = __fmul_rn(x_at(xr, bf16, b * K::COLS + c), isv[c]);
  }
  named_sync(bar, NT);
  const int items = (cols / 16) * 16 * B;   // (16-column group, column (b, j)), column fastest
  if (!skip) {
    // pass 1: max |Z| per column over the group; a thread folds its items of one
    // column before touching shared memory
    int lcol = -1;
    float lmx = 0.0f;
    for (int it = tid; it < items; it += NT) {
      const int c16 = it / (16 * B), col = it - c16 * 16 * B;
      const int b = col >> 4, j = col & 15;
      const float* xp = xsf + b * K::COLS + c16 * 16;
      const __half* vp = vh + c16 * 16 * kK + j;
      float mx = 0.0f;
#pragma unroll
      for (int kin = 0; kin < 16; ++kin) mx = fmaxf(mx, fabsf(__fmul_rn(xp[kin], __half2float(vp[kin * kK]))));
      if (col != lcol) {
        if (lcol >= 0) atomicMax(&ctl->amaxi[lcol], __float_as_int(lmx));
        lcol = col;
        lmx = mx;
      } else {
        lmx = fmaxf(lmx, mx);
      }
    }
    if (lcol >= 0) atomicMax(&ctl->amaxi[lcol], __float_as_int(lmx));
  }
  named_sync(bar, NT);
  if (!skip) {
    // pass 2: q = rint(Z / sigma_lo), |q| <= 127 * 256, q = 256 hi + lo
    uint8_t* ops = set + kSetHdr;
    int lcol = -1, lsum = 0;
    float rlo = 1.0f;
    for (int it = tid; it < items; it += NT) {
      const int c16 = it / (16 * B), col = it - c16 * 16 * B;
      const int b = col >> 4, j = col & 15;
      if (col != lcol) {
        if (lcol >= 0) atomicAdd(&ctl->zsum[lcol], lsum);
        lcol = col;
        lsum = 0;
        const float amax = __int_as_float(ctl->amaxi[col]);
        const float slo = amax > 0.0f ? __fmul_rn(amax, 1.0f / 32512.0f) : 1.0f;
        rlo = 1.0f / slo;
      }
      const float* xp = xsf + b * K::COLS + c16 * 16;
      const __half* vp = vh + c16 * 16 * kK + j;
      uint32_t hw[4] = {0, 0, 0, 0}, lw[4] = {0, 0, 0, 0};
#pragma unroll
      for (int kin = 0; kin < 16; ++kin) {
        const float z = __fmul_rn(xp[kin], __half2float(vp[kin * kK]));
        int qv = __float2int_rn(z * rlo);
        qv = max(-32512, min(32512, qv));
        const int qh = (qv + 128) >> 8;
        const int ql = qv - (qh << 8);
        lsum += qv;
        hw[kin >> 2] |= (static_cast<uint32_t>(qh) & 0xFFu) << (8 * (kin & 3));
        lw[kin >> 2] |= (static_cast<uint32_t>(ql) & 0xFFu) << (8 * (kin & 3));
      }
      // chunk cc, K-step t (32 columns), K half kc, 8-row core matrix n / 8
      const int cc = c16 >> 4, g16 = c16 & 15;
      const int t = g16 >> 1, kc = g16 & 1;
      const int nh = col, nl = 16 * B + col;
      uint8_t* base = ops + static_cast<size_t>(cc) * K::ZB;
      *reinterpret_cast<uint4*>(base + ((t * (K::NB / 8) + nh / 8) * 2 + kc) * 128 + (nh % 8) * 16) =
          make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(base + ((t * (K::NB / 8) + nl / 8) * 2 + kc) * 128 + (nl % 8) * 16) =
          make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    if (lcol >= 0) atomicAdd(&ctl->zsum[lcol], lsum);
    fence_proxy_async_smem();   // the MMAs read the operands through the async proxy
  }
  named_sync(bar, NT);
  if (tid < 16 * B) {
    if (!skip) {
      const float amax = __int_as_float(ctl->amaxi[tid]);
      const float slo = amax > 0.0f ? __fmul_rn(amax, 1.0f / 32512.0f) : 1.0f;
      float* hdr = reinterpret_cast<float*>(set);
      hdr[tid] = slo;
      hdr[64 + tid] = __fmul_rn(slo, static_cast<float>(ctl->zsum[tid]));
    }
    ctl->amaxi[tid] = 0;
    ctl->zsum[tid] = 0;
  }
  named_sync(bar, NT);
  if (tid == 0 && !skip) mbar_arrive(zfull);
}

template <int B>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
  using K = Cfg<B>;
  constexpr int NB = K::NB, C = K::C, NS = K::NS, NPAIRS = K::NPAIRS;
  constexpr uint32_t IDESC = make_idesc(2u, 0u, 1u, 128u, NB);  // s32 <- u8 x s8, M=128, N=NB

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stages = smem;
  uint8_t* sets = smem + NS * K::STAGE;
  uint8_t* vscr = sets + 2 * K::SET;
  uint8_t* xscr = vscr + K::VSCR;
  float* xsf = reinterpret_cast<float*>(xscr + K::XSCR);
  uint8_t* uring = xscr + K::XSCR + K::XSF;
  Ctl* ctl = reinterpret_cast<Ctl*>(uring + K::URING);
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, grid = gridDim.x;
  const int s0 = static_cast<int>(static_cast<long long>(cta) * p.segs / grid);
  const int s1 = static_cast<int>(static_cast<long long>(cta + 1) * p.segs / grid);
  const int nseg = s1 - s0;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  const int NC = p.n * p.NCB;   // chunk groups = partials per row tile
  const Seg sg0 = seg_of(s0, p, C);

  griddep_launch_dependents();

  // ------------------------------------------------------------------ set-up -----
  if (warp == kWarpCopy) {
    tmem_alloc(&ctl->tmem_base, 512);
    if (lane == 0) {
      for (int s = 0; s < kMaxStages; ++s) {
        mbar_init(&ctl->sfull[s], 1);
        mbar_init(&ctl->sempty[s], kExpWarps);
      }
      for (int u = 0; u < kURing; ++u) mbar_init(&ctl->ufull[u], 1);
      for (int q = 0; q < kMaxPairs; ++q) mbar_init(&ctl->aempty[q], kNI);
      for (int q = 0; q < 2; ++q) {
        mbar_init(&ctl->accfull[q], kNI);
        mbar_init(&ctl->zfull[q], 1);
      }
      for (int w = 0; w < 4; ++w) mbar_init(&ctl->drain[w], 1);
      mbar_init(&ctl->vfull, 1);
      ctl->abort = 0;
      for (int w = 0; w < kExpWarps; ++w) ctl->a_ready[w] = 0;
      ctl->acc_free[0] = 0;
      ctl->acc_free[1] = 0;
      for (int c = 0; c < 16 * kDecodeMaxBatch; ++c) {
        ctl->amaxi[c] = 0;
        ctl->zsum[c] = 0;
      }
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < kExpWarps) {
    // ------------------------------------------------ expanders (rows = lanes) -----
    // Units are walked in order in pairs: pair g goes to A-buffer pair g mod NPAIRS and
    // is expanded by team g & 1 (warps 0-3 or 4-7; warp % 4 is the TMEM lane quadrant).
    // Every expander warp walks all units (so all agree on the sign stages, each of
    // which all eight release) but expands only its team's pairs; warp e adds 1 to
    // a_ready[e] (release) once its rows of a pair are in tensor memory, and the
    // issuers wait for the four warps of the pair's team.  A warp whose wait ran out
    // stops signalling (the issuers' bounded waits then run out too); failure is
    // decided per warp by vote.
    const int team = warp >> 2;
    const int tid = (warp & 3) * 32 + lane;   // row within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool failed = false;
    auto check = [&](bool ok) {
      if (!__all_sync(0xffffffffu, ok)) failed = true;
    };
    int j = 0, c = 0, waited = -1;
    Seg sg = sg0;
    for (int g = 0; j < nseg && !failed; ++g) {
      const int pr = g % NPAIRS;
      const bool mine = (g & 1) == team;
      if (mine && g >= NPAIRS)
        check(mbar_wait(&ctl->aempty[pr], static_cast<uint32_t>((g / NPAIRS - 1) & 1), deadline, abort_flag));
      for (int q = 0; q < kGroup && j < nseg && !failed; ++q) {
        const int st = j % NS;
        if (mine) {
          if (waited != j) {
            check(mbar_wait(&ctl->sfull[st], static_cast<uint32_t>((j / NS) & 1), deadline, abort_flag));
            waited = j;
          }
          if (failed) break;
          const uint8_t* tile = stages + st * K::STAGE + c * kTileBytes;
          const uint4 wa = *reinterpret_cast<const uint4*>(tile + tid * 16);
          const uint4 wb = *reinterpret_cast<const uint4*>(tile + 2048 + tid * 16);
          const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
          const uint32_t abase = tmem + lane_base + K::ACOL0 + 64u * static_cast<uint32_t>(kGroup * pr + q);
          // K-step t holds bit t of every byte of the unit's words: byte q of word pw is
          // sign column 32 t + 4 pw + q (the device tile order), value 0 or 1
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t r[32];
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
#pragma unroll
              for (int pw = 0; pw < 8; ++pw) r[tt * 8 + pw] = (w[pw] >> (4 * h + tt)) & 0x01010101u;
            }
            tmem_st32(abase + 32 * h, r);
          }
        }
        if (++c == sg.len) {
          // segment done (its words are in registers): release the stage to the copy warp
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->sempty[st]);
          c = 0;
          ++j;
          if (j < nseg) sg = seg_of(s0 + j, p, C);
        }
      }
      if (failed) break;
      if (mine) {
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) red_release_shared_add(&ctl->a_ready[warp], 1u);
      }
    }
    if (failed) set_error(p, ctl);
  } else if (warp < kWarpIss0 + 4) {
    // --------- warps 8-15: the first chunk group's activation chunks, together ------
    const int tp = threadIdx.x - kWarpEpi0 * 32;   // 0..255
    bool pfailed = false;
    if (warp < kWarpIss0) {
      // accumulators start at zero (the MMAs only accumulate); release both
      const uint32_t lane_base = static_cast<uint32_t>((warp - kWarpEpi0) * 32) << 16;
      uint32_t zr[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) zr[q] = 0u;
#pragma unroll
      for (int cc = 0; cc < 2 * NB; cc += 32) tmem_st32(tmem + lane_base + cc, zr);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        red_release_shared_add(&ctl->acc_free[0], 1u);
        red_release_shared_add(&ctl->acc_free[1], 1u);
      }
    }
    if (nseg > 0) {
      // x and 1/s of the first group by plain loads (only after the previous kernel in
      // the stream has finished: it may have written them), V rows by a bulk copy
      griddep_wait();
      {
        const int cols = sg0.len * kTileCols, col0 = sg0.kgA * kTileCols;
        uint16_t* xr = reinterpret_cast<uint16_t*>(xscr);
        for (int idx = tp; idx < B * cols; idx += 256) {
          const int b = idx / cols, c = idx - b * cols;
          xr[b * K::COLS + c] = static_cast<const uint16_t*>(p.x)[static_cast<size_t>(b) * p.d + col0 + c];
        }
        float* isv = reinterpret_cast<float*>(xscr + K::COLS * B * 2);
        for (int c = tp; c < cols; c += 256) isv[c] = __ldg(p.inv_s + col0 + c);
      }
      const bool ok = mbar_wait(&ctl->vfull, 0, deadline, abort_flag);
      pfailed = !__all_sync(0xffffffffu, ok);
      // a warp that timed out still runs the set's barriers, skipping the work; the
      // others see the abort flag it set
      if (pfailed) set_error(p, ctl);
      named_sync(kBarProd, 256);
      produce_set<B, 256>(sets, vscr, xscr, xsf, p.x_bf16, ctl, sg0, tp, kBarProd, &ctl->zfull[0],
                          *abort_flag != 0);
    }
    if (warp < kWarpIss0) {
      // ------------------------------- epilogue, later chunk groups, row tiles -----
      const int tid = threadIdx.x - kWarpEpi0 * 32;   // row within the tile = TMEM lane
      const uint32_t lane_base = static_cast<uint32_t>((warp - kWarpEpi0) * 32) << 16;
      bool failed = pfailed;
      auto check = [&](bool ok) {
        if (!__all_sync(0xffffffffu, ok)) failed = true;
      };
      griddep_wait();   // the workspace and y belong to this launch only from here on
      // chunk groups of this CTA: zk counts them; the set of group zk is zk & 1
      int zk = 0;
      int cur_cg = nseg > 0 ? sg0.cg : -1;
      const int last_cg = nseg > 0 ? seg_of(s1 - 1, p, C).cg : -1;
      if (nseg > 0 && last_cg > cur_cg) {   // second group: produce it now
        const Seg sg2 = seg_of((cur_cg + 1) * p.RT, p, C);
        load_set_inputs<B>(p, vscr, xscr, sg2, tid);
        named_sync(kBarEpi, 128);
        produce_set<B, 128>(sets + K::SET, vscr, xscr, xsf, p.x_bf16, ctl, sg2, tid, kBarEpi, &ctl->zfull[1], false);
      }
      uint32_t zr[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) zr[q] = 0u;
      for (int j = 0; j < nseg; ++j) {
        const Seg sg = seg_of(s0 + j, p, C);
        if (sg.cg != cur_cg) {
          cur_cg = sg.cg;
          ++zk;
        }
        const float* hdr = reinterpret_cast<const float*>(sets + (zk & 1) * K::SET);
        const int acc = j & 1;
        const int us = j % kURing;
        // this row's U_i entries (16 fp16), from the U ring
        if (!failed) check(mbar_wait(&ctl->ufull[us], static_cast<uint32_t>((j / kURing) & 1), deadline, abort_flag));
        uint4 ua = make_uint4(0, 0, 0, 0), ub = make_uint4(0, 0, 0, 0);
        if (!failed) {
          ua = *reinterpret_cast<const uint4*>(uring + us * kTileBytes + tid * 32);
          ub = *reinterpret_cast<const uint4*>(uring + us * kTileBytes + tid * 32 + 16);
        }
        if (!failed) check(mbar_wait(&ctl->accfull[acc], static_cast<uint32_t>((j >> 1) & 1), deadline, abort_flag));
        if (!failed) {
          tc_fence_after();
          const __half* uh = reinterpret_cast<const __half*>(&ua);
          const __half* uh2 = reinterpret_cast<const __half*>(&ub);
          const uint32_t abase = tmem + lane_base + static_cast<uint32_t>(acc * NB);
          float part[B];
#pragma unroll
          for (int b = 0; b < B; ++b) {
            uint32_t vh[16], vl[16];
            tmem_ld16(abase + b * 16, vh);
            tmem_ld16(abase + 16 * B + b * 16, vl);
            tc_wait_ld();
            float sacc = 0.0f;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const float slo = hdr[b * 16 + jj];
              const float sbz = 256.0f * slo * static_cast<float>(static_cast<int>(vh[jj])) +
                                slo * static_cast<float>(static_cast<int>(vl[jj]));
              // S = 1 - 2 Sb (bit 1 = sign -1):  T = sum_c Z - 2 sum_c Sb Z
              const float tval = hdr[64 + b * 16 + jj] - 2.0f * sbz;
              const float uj = __half2float(jj < 8 ? uh[jj] : uh2[jj - 8]);
              sacc = fmaf(uj, tval, sacc);
            }
            part[b] = sacc;
          }
          // zero the accumulator for segment j + 2 and hand it back to the issuers
#pragma unroll
          for (int cc = 0; cc < NB; cc += 32) tmem_st32(abase + cc, zr);
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) red_release_shared_add(&ctl->acc_free[acc], 1u);
          float* dst = p.part + static_cast<size_t>(s0 + j) * B * kTileRows;
#pragma unroll
          for (int b = 0; b < B; ++b) dst[b * kTileRows + tid] = part[b];
        }
        // U slot us is read by every epilogue thread: refill it for segment j + kURing
        named_sync(kBarEpi, 128);
        if (tid == 0 && j + kURing < nseg) {
          const Seg sn = seg_of(s0 + j + kURing, p, C);
          mbar_arrive_expect_tx(&ctl->ufull[us], kTileBytes);
          bulk_g2s(uring + us * kTileBytes, u_tile(p, sn.i, sn.rt), kTileBytes, &ctl->ufull[us]);
        }
        // The last segment of group zk is done: its MMAs have completed, so the set of
        // zk can take group zk + 2 if this CTA has one.
        const bool group_end = (j + 1 == nseg) || seg_of(s0 + j + 1, p, C).cg != cur_cg;
        if (group_end && cur_cg + 2 <= last_cg) {
          const Seg sg3 = seg_of((cur_cg + 2) * p.RT, p, C);
          load_set_inputs<B>(p, vscr, xscr, sg3, tid);
          named_sync(kBarEpi, 128);
          produce_set<B, 128>(sets + (zk & 1) * K::SET, vscr, xscr, xsf, p.x_bf16, ctl, sg3, tid, kBarEpi,
                              &ctl->zfull[zk & 1], false);
        }
      }
      if (failed) set_error(p, ctl);

      // ------------- row tiles: count the segments, then reduce the owned row tiles ---
      // Row tile rt is reduced by CTA rt mod grid once all NC partials have arrived:
      // fixed chunk-group order, so the sum is deterministic.
      __threadfence();
      named_sync(kBarEpi, 128);
      if (tid == 0) ctl->abort_snap = *abort_flag;
      named_sync(kBarEpi, 128);
      if (!ctl->abort_snap) {
        for (int e = tid; e < nseg; e += 128) atomicAdd(p.cnt + seg_of(s0 + e, p, C).rt, 1u);
        const size_t stride = static_cast<size_t>(p.RT) * B * kTileRows;
        for (int rt = cta; rt < p.RT; rt += grid) {
          if (tid == 0) {
            bool ok = true;
            while (ld_acquire_u32(p.cnt + rt) != static_cast<uint32_t>(NC)) {
              if (*abort_flag || globaltimer_ns() > deadline) {
                ok = false;
                break;
              }
              __nanosleep(64);
            }
            ctl->red_ok = ok ? 1 : 0;
            if (!ok) set_error(p, ctl);
          }
          named_sync(kBarEpi, 128);
          if (ctl->red_ok) {
            __threadfence();
            const float* pp = p.part + static_cast<size_t>(rt) * B * kTileRows + tid;
            constexpr int kBatch = 32 / B;   // loads in flight per thread
            float acc[B];
#pragma unroll
            for (int b = 0; b < B; ++b) acc[b] = 0.0f;
            for (int c0 = 0; c0 < NC; c0 += kBatch) {
              float v[kBatch][B];
#pragma unroll
              for (int u = 0; u < kBatch; ++u)
#pragma unroll
                for (int b = 0; b < B; ++b)
                  v[u][b] = c0 + u < NC ? __ldcg(pp + (c0 + u) * stride + b * kTileRows) : 0.0f;
#pragma unroll
              for (int u = 0; u < kBatch; ++u)
#pragma unroll
                for (int b = 0; b < B; ++b) acc[b] += v[u][b];
            }
#pragma unroll
            for (int b = 0; b < B; ++b)
              store_y(p.y, p.x_bf16, static_cast<size_t>(b) * p.m + static_cast<size_t>(rt) * kTileRows + tid, acc[b]);
            if (tid == 0) p.cnt[rt] = 0u;   // the next call starts from zero
          }
          named_sync(kBarEpi, 128);
        }
      }
    } else if (lane == 0) {
      // ---------------------------------------------------------- MMA issuers -------
      // Lane 0 of warp 8 + w issues K-steps w and w + 4 of every unit into the
      // segment's accumulator (which the epilogue zeroes, so every MMA accumulates) and
      // commits once per A-buffer pair and once per segment.  It waits for the
      // expanders and the epilogue by polling shared counters: an mbarrier wait, or a
      // whole warp walking the loop, costs the issuing thread more than its MMAs.
      const int w = warp - kWarpIss0;
      bool ok = !pfailed;
      bool any = false;
      int j = 0, c = 0, zk = -1, cur_cg = -1;
      Seg sg = sg0;
      uint32_t zbase = 0;
      for (int g = 0; j < nseg && ok; ++g) {
        const int pr = g % NPAIRS;
        ok = poll_geq4(ctl->a_ready + 4 * (g & 1), static_cast<uint32_t>((g >> 1) + 1), deadline, abort_flag);
        if (!ok) break;
        tc_fence_after();
        for (int q = 0; q < kGroup && j < nseg && ok; ++q) {
          const int acc = j & 1;
          if (c == 0) {   // segment j starts: its accumulator must be zeroed
            ok = poll_geq(&ctl->acc_free[acc], 4u * static_cast<uint32_t>((j >> 1) + 1), deadline, abort_flag);
            tc_fence_after();
            if (sg.cg != cur_cg) {
              cur_cg = sg.cg;
              ++zk;
              if (ok) ok = mbar_wait(&ctl->zfull[zk & 1], static_cast<uint32_t>((zk >> 1) & 1), deadline, abort_flag);
              zbase = smem_u32(sets + (zk & 1) * K::SET + kSetHdr);
            }
            if (!ok) break;
          }
          const uint32_t zaddr = zbase + static_cast<uint32_t>(c * K::ZB);
          const uint32_t acol = K::ACOL0 + 64u * static_cast<uint32_t>(kGroup * pr + q);
          const uint32_t dcol = static_cast<uint32_t>(acc * NB);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int t = w + kNI * h;
            const uint64_t bdesc = smem_desc_noswizzle(zaddr + t * (NB / 8) * 256, 128, 256);
            mma_i8_ts(tmem + dcol, tmem + acol + 8 * t, bdesc, IDESC, 1u);
          }
          any = true;
          if (++c == sg.len) {
            tc_commit(&ctl->accfull[acc]);
            c = 0;
            ++j;
            if (j < nseg) sg = seg_of(s0 + j, p, C);
          }
        }
        if (ok) tc_commit(&ctl->aempty[pr]);
      }
      if (!ok) set_error(p, ctl);
      if (any) {
        tc_commit(&ctl->drain[w]);
        mbar_wait(&ctl->drain[w], 0, globaltimer_ns() + 100000000ull, nullptr);
      }
    }
  } else if (warp == kWarpCopy && lane == 0) {
    // ------------------------------------------------------ sign-tile copies -------
    // Stack memory only (it may be read before the previous kernel in the stream has
    // finished): V rows of the first chunk group, the first sign stages and U tiles.
    int issued = 0;
    if (nseg > 0) {
      const uint32_t vb = static_cast<uint32_t>(sg0.len) * kTileCols * kK * 2;
      mbar_arrive_expect_tx(&ctl->vfull, vb);
      bulk_g2s(vscr, v_rows(p, sg0), vb, &ctl->vfull);
    }
    for (; issued < NS && issued < nseg; ++issued) {
      if (p.inject_unreachable && issued == 0) continue;
      const Seg sg = seg_of(s0 + issued, p, C);
      const uint32_t bytes = static_cast<uint32_t>(sg.len) * kTileBytes;
      mbar_arrive_expect_tx(&ctl->sfull[issued], bytes);
      bulk_g2s(stages + issued * K::STAGE,
               p.blocks + static_cast<size_t>(sg.i) * p.block_bytes +
                   (static_cast<size_t>(sg.rt) * p.KG + sg.kgA) * kTileBytes,
               bytes, &ctl->sfull[issued]);
    }
    for (int j = 0; j < kURing && j < nseg; ++j) {
      const Seg sg = seg_of(s0 + j, p, C);
      mbar_arrive_expect_tx(&ctl->ufull[j], kTileBytes);
      bulk_g2s(uring + j * kTileBytes, u_tile(p, sg.i, sg.rt), kTileBytes, &ctl->ufull[j]);
    }
    for (; issued < nseg; ++issued) {
      const int st = issued % NS;
      if (!mbar_wait(&ctl->sempty[st], static_cast<uint32_t>((issued / NS - 1) & 1), deadline, abort_flag)) {
        set_error(p, ctl);
        break;
      }
      const Seg sg = seg_of(s0 + issued, p, C);
      const uint32_t bytes = static_cast<uint32_t>(sg.len) * kTileBytes;
      mbar_arrive_expect_tx(&ctl->sfull[st], bytes);
      bulk_g2s(stages + st * K::STAGE,
               p.blocks + static_cast<size_t>(sg.i) * p.block_bytes +
                   (static_cast<size_t>(sg.rt) * p.KG + sg.kgA) * kTileBytes,
               bytes, &ctl->sfull[st]);
    }
    // No copy may be in flight when the CTA exits: wait for the last use of every
    // stage and for the first-group inputs (each bounded).
    const uint64_t drain_by = globaltimer_ns() + 100000000ull;
    for (int q = (issued > NS ? issued - NS : 0); q < issued; ++q) {
      if (p.inject_unreachable && q == 0) continue;
      mbar_wait(&ctl->sfull[q % NS], static_cast<uint32_t>((q / NS) & 1), drain_by, nullptr);
    }
    if (nseg > 0) mbar_wait(&ctl->vfull, 0, drain_by, nullptr);
  }

  // U-ring copies are issued by epilogue thread 0 (and the copy thread): drain them too.
  if (warp == kWarpEpi0 && lane == 0) {
    const uint64_t drain_by = globaltimer_ns() + 100000000ull;
    for (int j = (nseg > kURing ? nseg - kURing : 0); j < nseg; ++j)
      mbar_wait(&ctl->ufull[j % kURing], static_cast<uint32_t>((j / kURing) & 1), drain_by, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpCopy) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int B>
cudaError_t launch_b(const DecodeParams& p, int grid, cudaStream_t stream) {
  auto kern = decode_kernel<B>;
  constexpr int smem = Cfg<B>::SMEM;
  static bool configured[64] = {};   // the attribute is set once per device, outside any capture
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

size_t decode_smem_bytes(int batch) {
  switch (batch) {
    case 1: return Cfg<1>::SMEM;
    case 2: return Cfg<2>::SMEM;
    case 3: return Cfg<3>::SMEM;
    case 4: return Cfg<4>::SMEM;
    default: return 0;
  }
}

cudaError_t launch_decode(const DecodeParams& p, int batch, int grid, cudaStream_t stream) {
  switch (batch) {
    case 1: return launch_b<1>(p, grid, stream);
    case 2: return launch_b<2>(p, grid, stream);
    case 3: return launch_b<3>(p, grid, stream);
    case 4: return launch_b<4>(p, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace bs
