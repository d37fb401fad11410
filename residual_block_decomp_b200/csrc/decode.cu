// Decode path of the BitStack linear (a few rows of x):
//     y = sum_i U_i (S_i ((x (.) 1/s) (.) V_i)).
//
// The weight of a BitStack layer is the sum of the loaded residual blocks, each a +-1
// sign matrix times the rank-k product of its singular vectors, with the
// activation-aware scale undone per input channel (weight restoration snippet of the
// OpenReview discussion of "BitStack: Any-Size Compression of Large Language Models in
// Variable Memory Environments"; review page "BitStack: Fine-Grained Size Control...",
// Figs. 3 and 5).  For a few rows of x the weight is never formed: by associativity
//     y[b, r] = sum_i sum_j U_i[r, j] T_i[r, (b, j)],   T_i = S_i Z_i,
//     Z_i[c, (b, j)] = x[b, c] / s_c * V_i[c, j],
// a +-1 contraction with 16 * batch columns per block.
//
// One persistent launch, one CTA per SM, walking a contiguous run of segments (one
// 128-row tile x one chunk group of C 256-column chunks of one block), numbered
// chunk-group-major; with no more chunk groups than CTAs, each CTA's run lies inside
// one chunk group:
//  * Activation sets.  Z of a chunk group is quantised per column (b, j): a step
//    sigma = max |Z| / 32512 over the group, q = rint(Z / sigma) split exactly into two
//    int8 planes q = 256 hi + lo, written to shared memory in the tensor-core operand
//    layout, with sigma and the integer column sums of q kept aside.  The CTA's first
//    group is built by all its warps at the start from shared-memory copies of its V
//    rows, 1/s and x (bulk-copied by the copy thread; V and 1/s before the kernel ahead
//    has finished); maxima and sums are warp reduce-scatters; its second group by the epilogue
//    warps while the first is being contracted, and later groups by the epilogue warps
//    into the slot a finished group frees.
//  * Signs.  A copy thread streams each segment's sign tiles (C x 4 KiB, contiguous in
//    the record) into a ring of shared-memory stages with 1-D bulk copies, starting
//    before the kernel ahead in the stream has finished (it reads only the block area).
//  * Expansion.  T teams of four warps (one warp per tensor-memory lane quadrant) take
//    the units (128 x 256 signs) in turn: each thread turns its row's 256 sign bits into
//    s8 operands -128 Sb (K-step t = bit t of every byte moved to bit 7 by a multiply,
//    which runs on the FMA pipe, then one AND per four columns; the device tile order)
//    and stores them to one of its team's two slots in tensor memory; each warp then
//    arrives on the slot's mbarrier.  No barrier inside a team.
//  * MMA.  NI issuer warps take the units in turn (warp-uniform, one elected lane
//    issues): the unit's eight tcgen05.mma.kind::i8 (M = 128, N = 32 * batch, K = 32,
//    s32 accumulate) into the segment's accumulator, then one commit that frees the slot
//    and one that counts the unit into the segment's accumulator barrier.
//  * Epilogue.  S = 1 - 2 Sb with Sb the stored bit, so T = colsum(Z) - 2 Sb Z; four
//    warps read a finished accumulator (hi and lo planes), form T with the group's sigma
//    and column sums, apply the row's U_i entries and store one fp32 partial per row and
//    batch row; they zero the accumulator for reuse (every MMA accumulates; int32 sums
//    are exact, so the order of the units does not matter).
//  * Reduction.  At the end every CTA counts its partials into per-row-tile arrival
//    counters (acquire-release atomics at GPU scope, which publish the partials and
//    make the others' visible to the last arrival); the CTA that adds a tile's last
//    partial sums all of them in fixed chunk-group order and writes y: deterministic,
//    and no CTA ever waits for another.
//  * Hand-overs between roles are mbarriers, waited on with the suspending try_wait so
//    that a waiting warp takes no issue slots from the warps that expand signs.
//  * Every wait is bounded; a wait that runs out sets the device error word, and the
//    CTA drains its copies and MMAs, frees tensor memory and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace bs {
namespace {

constexpr int kMaxStages = 16;
constexpr int kSlots = 2;              // tensor-memory A slots per team
constexpr int kNI = 3;                 // the most issuer warps (20 warps in all at batch <= 2: 96 registers each)
constexpr int kBarZ = 4;               // named barriers: 4 = all warps but the copy warp, 5 = epilogue
constexpr int kBarEpi = 5;
constexpr float kQMax = 32512.0f;      // |q| <= 127 * 256: q = 256 hi + lo with hi, lo in int8
// Rounding to an integer by addition: for |v| < 2^22, the float nearest to 1.5 * 2^23 + v
// lies in [2^23, 2^24), where floats are the integers, so it is 1.5 * 2^23 + rint(v)
// (ties to even: 1.5 * 2^23 is even), and its bit pattern is kRoundBits + rint(v).
// kRoundBias adds 128 more, so the pattern is kRoundBits + q + 128.
constexpr uint32_t kRoundBits = 0x4B400000u;   // bit pattern of 1.5 * 2^23
constexpr float kRoundBias = 12583040.0f;      // 1.5 * 2^23 + 128

template <int B>
struct Cfg {
  static constexpr int NB = 32 * B;                 // MMA N: hi plane (16 B columns) | lo plane
  static constexpr int NCOL = 16 * B;               // columns (b, j) of Z
  static constexpr int C = decode_chunks_per_segment(B);
  static constexpr int ZB = decode_chunk_operand_bytes(B);
  static constexpr int SET = C * ZB;                // one activation set (operand planes only)
  static constexpr int T = B <= 2 ? 3 : 2;          // teams of four warps
  static constexpr int NACC = B == 1 ? 4 : 2;       // segment accumulators in tensor memory
  static constexpr uint32_t ACOL0 = NACC * NB;      // first A-slot column (64 columns per slot)
  // Issuer warps.  Issuer u % NI takes unit u, and unit u fills A slot
  // ((u / T) % kSlots) of team u % T: NI divides T * kSlots, so every use of a slot goes
  // to the same issuer, which therefore waits for the slot's uses one by one (a waiter
  // that skipped a use could take an earlier phase of the same parity for the one it
  // wants).
  static constexpr int NI = B <= 2 ? 3 : 2;
  static constexpr int WISS = 4 * T;                // issuer warps WISS .. WISS + NI - 1
  static constexpr int WEPI = 4 * T + NI;           // epilogue warps WEPI .. WEPI + 3
  static constexpr int WCTL = WEPI + 4;             // copy thread, tensor-memory owner (last warp)
  static constexpr int THREADS = 32 * (WCTL + 1);
  static constexpr int ZTHREADS = THREADS - 32;     // warps that build the first sets
  static constexpr int STAGE = C * kTileBytes;
  static constexpr int CTL = 8192;
  // staging for the first group's x rows and 1/s (its V rows go to the second set slot)
  static constexpr int STG = B * C * kTileCols * 2 + C * kTileCols * 4;
  static constexpr int STG_AL = (STG + 1023) / 1024 * 1024;
  static constexpr int FIXED = 2 * SET + CTL + STG_AL;
  static constexpr int NS0 = (227 * 1024 - FIXED) / STAGE;
  static constexpr int NS = NS0 < kMaxStages ? NS0 : kMaxStages;
  static constexpr int SMEM = NS * STAGE + FIXED;
  static_assert(ACOL0 + T * kSlots * 64 <= 512, "tensor memory columns");
  static_assert((T * kSlots) % NI == 0 && NI <= kNI, "each A slot has one issuer");
  static_assert(NS >= 4, "sign ring too small");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  // each decode CTA allocates all 512 tensor-memory columns: two must never share an SM
  static_assert(2 * (SMEM + 1024) > 228 * 1024, "two decode CTAs would fit one SM");
  static_assert(THREADS <= 1024, "threads per CTA");
  static_assert(ZTHREADS / 32 <= 20, "per-warp partials of the set builders");
  static_assert(4 * (THREADS / kTileRows) * B * kTileRows * 4 + THREADS * 4 <= NS * STAGE,
                "the reduction's scratch fits the drained sign stages");
  static_assert(C * kTileCols * 32 <= SET, "the first group's V rows fit the second set slot");
};

struct Ctl {
  uint64_t sfull[kMaxStages], sempty[kMaxStages];
  uint64_t aempty[3][kSlots];   // a slot's MMAs completed (one commit per unit)
  uint64_t accfull[4];          // a segment's MMAs completed (one commit per unit)
  uint64_t zready[2];           // a set built by the epilogue warps (groups 1, 2, ...)
  uint64_t drain[kNI];
  uint64_t ready[3][kSlots];    // a slot's four quadrants stored (one arrival per team warp)
  uint64_t acc_free[4];         // an accumulator read and zeroed (one arrival per epilogue warp)
  uint64_t vstage, xstage;      // the first group's V rows and 1/s / its x rows, in shared memory
  uint32_t tmem_base;
  int abort;
  int nred;                     // row tiles this CTA completed in the current counting round
  int count_ok;                 // the epilogue finished without error: count the partials
  int amax[2][64];              // per set slot and column: max |Z| (float bits, >= 0)
  int csum[2][64];              // per set slot and column: the group's integer sum of q
  float sig[2][64];             // per set slot and column: the quantisation step
  float rlo[2][64];             // per set slot and column: 1 / step
  int wpart[20][64];            // per warp and column: a set builder's partial max / sum
};
static_assert(sizeof(Ctl) <= 8192, "control block");

struct Seg {
  int i, rt, kgA, len, cg;
  int cgb;   // chunk group within block i
  int l;     // linear of the launch
  int sl;    // segment within linear l
};
// Linear l of a launch (the last one for an index past the end, which walks reach only
// after their last segment).
template <int G>
__device__ __forceinline__ const DecodeLin& lin_at(const DecodeArgs<G>& p, int l) {
  return p.lin[G == 1 ? 0 : (l < p.nlin ? l : p.nlin - 1)];
}
// The linear holding global segment s: the last one whose first segment is <= s.
template <int G>
__device__ __forceinline__ int lin_of_seg(const DecodeArgs<G>& p, int s) {
  if (G == 1) return 0;
  int lo = 0, hi = p.nlin - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.lin[mid].seg0 <= s) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}
template <int G>
__device__ __forceinline__ Seg seg_of(int s, const DecodeArgs<G>& p, int C) {
  Seg g;
  g.l = lin_of_seg(p, s);
  const DecodeLin& L = lin_at(p, g.l);
  g.sl = s - L.seg0;
  g.cg = g.sl / L.RT;
  g.rt = g.sl - g.cg * L.RT;
  g.i = g.cg / L.NCB;
  g.cgb = g.cg - g.i * L.NCB;
  g.kgA = g.cgb * C;
  g.len = min(C, L.KG - g.kgA);
  return g;
}
// The segment after g (chunk-group-major within a linear, linears one after another),
// without divisions.
template <int G>
__device__ __forceinline__ void seg_next(Seg& g, const DecodeArgs<G>& p, int C) {
  ++g.sl;
  const DecodeLin& L = lin_at(p, g.l);
  if (++g.rt == L.RT) {
    g.rt = 0;
    ++g.cg;
    if (++g.cgb == L.NCB) {
      g.cgb = 0;
      ++g.i;
      if (G > 1 && g.i == L.n) {   // on to the next linear (each has at least one block)
        ++g.l;
        g.i = 0;
        g.cg = 0;
        g.sl = 0;
      }
    }
    g.kgA = g.cgb * C;
    g.len = min(C, lin_at(p, g.l).KG - g.kgA);
  }
}
// Chunk group cg of linear l, and the one after it.
struct GroupRef {
  int l, cg;
};
template <int G>
__device__ __forceinline__ GroupRef group_next(GroupRef r, const DecodeArgs<G>& p) {
  const DecodeLin& L = lin_at(p, r.l);
  if (++r.cg == L.n * L.NCB && G > 1) {
    ++r.l;
    r.cg = 0;
  }
  return r;
}

// The run of segments [s0, s1) of CTA `cta`.  For one linear with at most as many chunk
// groups as CTAs, every group gets floor or ceil(grid / groups) CTAs and splits its RT
// segments evenly among them, so no CTA spans two groups (building a group's activation
// set is paid once per CTA); otherwise (more groups, or several linears) the segments
// are split contiguously and a CTA spans several groups, whose sets after the first
// are built in the background.
template <int G>
__device__ __forceinline__ void cta_range(const DecodeArgs<G>& p, int cta, int grid, int& s0, int& s1) {
  const DecodeLin& L = p.lin[0];
  const int NG = L.n * L.NCB;
  if (G == 1 && NG <= grid) {
    const int base = grid / NG, extra = grid - base * NG;
    int g, w, k;
    if (cta < extra * (base + 1)) {
      g = cta / (base + 1);
      w = cta - g * (base + 1);
      k = base + 1;
    } else {
      const int c2 = cta - extra * (base + 1);
      g = extra + c2 / base;
      w = c2 - (g - extra) * base;
      k = base;
    }
    s0 = g * L.RT + (w * L.RT) / k;
    s1 = g * L.RT + ((w + 1) * L.RT) / k;
  } else {
    s0 = static_cast<int>(static_cast<long long>(cta) * p.segs / grid);
    s1 = static_cast<int>(static_cast<long long>(cta + 1) * p.segs / grid);
  }
}

__device__ __forceinline__ void store_y(void* y, int bf16, size_t idx, float v) {
  if (bf16) static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(y)[idx] = __float2half_rn(v);
}
__device__ __forceinline__ float x_at(const void* x, int bf16, size_t idx) {
  const uint16_t h = static_cast<const uint16_t*>(x)[idx];
  return bf16 ? __uint_as_float(static_cast<uint32_t>(h) << 16) : __half2float(__ushort_as_half(h));
}
template <int G>
__device__ __forceinline__ void set_error(const DecodeArgs<G>& p, Ctl* ctl) {
  ctl->abort = 1;
  atomicOr(p.err, kErrTimeout);
}

// Byte offsets inside one block record.
__device__ __forceinline__ const uint8_t* record(const DecodeLin& L, int i) {
  return L.blocks + static_cast<size_t>(i) * L.block_bytes;
}
__device__ __forceinline__ size_t u_offset(const DecodeLin& L) { return static_cast<size_t>(L.m) * L.d / 8; }
__device__ __forceinline__ size_t v_offset(const DecodeLin& L) {
  return u_offset(L) + static_cast<size_t>(2) * kK * L.m;
}

// K-step t of a unit from one sign word: bit t of every byte moved to bit 7 and the
// rest cleared, i.e. the s8 operand -128 * Sb.  The shift is a multiply, which runs on
// the FMA pipe; only the AND takes the (half-rate) integer pipe.
__device__ __forceinline__ uint32_t sign_bytes(uint32_t w, int t) {
  uint32_t v = w;
  if (t < 7) asm("mul.lo.u32 %0, %1, %2;" : "=r"(v) : "r"(w), "r"(1u << (7 - t)));
  return v & 0x80808080u;
}

// The quantisation step of a column from the largest |Z| of its chunk group.
__device__ __forceinline__ float step_of(float amax) {
  return amax > 0.0f ? __fmul_rn(amax, 1.0f / kQMax) : 1.0f;
}

// Reduce-scatter of 16 values over the 32 lanes of a warp (pairwise exchanges, 16
// shuffles): afterwards lane l holds, in its return value, the reduction over all
// lanes of value index scatter_index(l); lanes l and l ^ 1 hold the same index.
__device__ __forceinline__ int scatter_index(int lane) {
  return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}
template <typename Tv, typename Op>
__device__ __forceinline__ Tv warp_reduce_scatter16(Tv (&v)[16], int lane, Op op) {
  constexpr uint32_t FULL = 0xffffffffu;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const bool up = (lane & 16) != 0;
    const Tv send = up ? v[e] : v[e + 8], keep = up ? v[e + 8] : v[e];
    v[e] = op(keep, __shfl_xor_sync(FULL, send, 16));
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const bool up = (lane & 8) != 0;
    const Tv send = up ? v[e] : v[e + 4], keep = up ? v[e + 4] : v[e];
    v[e] = op(keep, __shfl_xor_sync(FULL, send, 8));
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const bool up = (lane & 4) != 0;
    const Tv send = up ? v[e] : v[e + 2], keep = up ? v[e + 2] : v[e];
    v[e] = op(keep, __shfl_xor_sync(FULL, send, 4));
  }
  {
    const bool up = (lane & 2) != 0;
    const Tv send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
    v[0] = op(keep, __shfl_xor_sync(FULL, send, 2));
  }
  return op(v[0], __shfl_xor_sync(FULL, v[0], 1));
}
struct MaxOp {
  __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct UAddOp {
  __device__ __forceinline__ uint32_t operator()(uint32_t a, uint32_t b) const { return a + b; }
};

// The 16 fp16 entries of one V row (32 bytes) as fp32, from global memory (read-only
// path) or from shared memory.
template <bool kGlobal>
__device__ __forceinline__ void v_row(const uint8_t* row, float (&v)[16]) {
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  const uint4 a = kGlobal ? __ldg(r4) : r4[0], b = kGlobal ? __ldg(r4 + 1) : r4[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}

// Input columns of chunk group cg: block i, columns [col0, col0 + gcols).
struct Group {
  int i, col0, gcols;
};
__device__ __forceinline__ Group group_of(const DecodeLin& L, int cg, int C) {
  Group g;
  g.i = cg / L.NCB;
  const int k0 = (cg - g.i * L.NCB) * C;
  g.col0 = k0 * kTileCols;
  g.gcols = min(C, L.KG - k0) * kTileCols;
  return g;
}

// Where a set builder reads the group's inputs: V row of group column c at v + 32 c,
// x[b] at x[b * xs + c], 1/s at is[c] -- global memory for sets built in the
// background, shared-memory copies (bulk-copied by the copy thread) for the first set.
struct SetSrc {
  const uint8_t* v;
  const uint16_t* x;
  const float* is;
  int xs;
};

// The activation set of chunk group cg is built in two passes by NT threads (index
// zt, whole warps) that share a named barrier; thread zt owns group columns zt,
// zt + NT, ... (whole V rows):
//   set_max    Z = (x (.) 1/s) (.) V_i over its columns, max |Z| per column (b, j);
//   set_quant  q = rint(Z / sigma), sigma = max |Z| / 32512, into the operand layout
//              as the two int8 planes q = 256 hi + lo, and the integer sums of q;
// with ctl->{amax, csum, sig}[slot] as the shared state.  Per-column maxima and sums
// are warp reduce-scatters and one shared atomic per column and warp.
template <bool kGlobal, typename P>
__device__ __forceinline__ float x_scaled(const P& p, const SetSrc& S, int c, int b) {
  const uint16_t h = S.x[b * S.xs + c];
  const float xv = p.x_bf16 ? __uint_as_float(static_cast<uint32_t>(h) << 16) : __half2float(__ushort_as_half(h));
  return __fmul_rn(xv, kGlobal ? __ldg(S.is + c) : S.is[c]);
}

template <int B, bool kGlobal, typename P>
__device__ void set_max(const P& p, Ctl* ctl, int slot, const SetSrc& S, int gcols, int zt, int NT) {
  const int lane = zt & 31;
#pragma unroll
  for (int b = 0; b < B; ++b) {
    float mx[16];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) mx[jj] = 0.0f;
    for (int c = zt; c < gcols; c += NT) {
      const float xv = x_scaled<kGlobal>(p, S, c, b);
      float v[16];
      v_row<kGlobal>(S.v + static_cast<size_t>(c) * 32, v);
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) mx[jj] = fmaxf(mx[jj], fabsf(__fmul_rn(xv, v[jj])));
    }
    const float m = warp_reduce_scatter16(mx, lane, MaxOp());
    if ((lane & 1) == 0) ctl->wpart[zt >> 5][b * 16 + scatter_index(lane)] = __float_as_int(m);
  }
}

template <int B, bool kGlobal, typename P>
__device__ void set_quant(const P& p, Ctl* ctl, int slot, uint8_t* set, const SetSrc& S, int gcols, int zt,
                          int NT) {
  using K = Cfg<B>;
  constexpr int NB = K::NB, NCOL = K::NCOL;
  const int lane = zt & 31;
#pragma unroll
  for (int b = 0; b < B; ++b) {
    // 1 / step of the 16 columns in registers (the stores below go to shared memory too,
    // so reads through a pointer would be repeated after every store)
    float rl[16];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) rl[jj] = ctl->rlo[slot][b * 16 + jj];
    uint32_t zs[16];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) zs[jj] = 0u;
    for (int c = zt; c < gcols; c += NT) {
      const float xv = x_scaled<kGlobal>(p, S, c, b);
      float v[16];
      v_row<kGlobal>(S.v + static_cast<size_t>(c) * 32, v);
      // operand layout: no-swizzle K-major core matrices of 8 operand columns x 16 K;
      // K-step t at t * NB * 32, core matrices adjacent in K 128 bytes apart, in N 256
      const int cc = c >> 8, cl = c & 255;
      uint8_t* base = set + cc * K::ZB + ((cl >> 5) * (NB / 8) * 2 + ((cl >> 4) & 1)) * 128 + (cl & 15);
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        // q = rint(Z / sigma), |q| <= 32512 (the step makes |Z| / sigma <= 32512 up to a
        // rounding far below 1/2): one fused multiply-add with kRoundBias leaves the bit
        // pattern bq = kRoundBits + q + 128 (see kRoundBias), whose byte 1 is the hi
        // plane (q + 128) >> 8 and whose byte 0, with bit 7 flipped, the lo plane q mod 256
        const uint32_t bq = __float_as_uint(__fmaf_rn(__fmul_rn(xv, v[jj]), rl[jj], kRoundBias));
        zs[jj] += bq;
        const int nh = b * 16 + jj, nl = NCOL + nh;
        base[(nh >> 3) * 256 + (nh & 7) * 16] = static_cast<uint8_t>(bq >> 8);      // hi
        base[(nl >> 3) * 256 + (nl & 7) * 16] = static_cast<uint8_t>(bq ^ 0x80u);   // lo = q - 256 hi, mod 256
      }
    }
    const uint32_t sum = warp_reduce_scatter16(zs, lane, UAddOp());
    if ((lane & 1) == 0) ctl->wpart[zt >> 5][b * 16 + scatter_index(lane)] = static_cast<int>(sum);
  }
}

template <int B, bool kGlobal, typename P>
__device__ void build_set(const P& p, Ctl* ctl, int slot, uint8_t* set, const SetSrc& S, int gcols, int zt,
                          int NT, int bar) {
  constexpr int NCOL = Cfg<B>::NCOL;
  const int nw = NT >> 5;
  // pass 1; each warp leaves its per-column maxima in wpart, then one thread per column
  // folds them (no two warps update one shared word)
  set_max<B, kGlobal>(p, ctl, slot, S, gcols, zt, NT);
  bar_named(bar, NT);
  if (zt < NCOL) {
    int m = 0;
    for (int w = 0; w < nw; ++w) m = max(m, ctl->wpart[w][zt]);   // max |Z| as float bits, all >= 0
    ctl->amax[slot][zt] = m;
    const float sg = step_of(__int_as_float(m));
    ctl->sig[slot][zt] = sg;
    ctl->rlo[slot][zt] = 1.0f / sg;
  }
  bar_named(bar, NT);
  set_quant<B, kGlobal>(p, ctl, slot, set, S, gcols, zt, NT);
  fence_proxy_async_smem();   // the MMAs read the operand through the async proxy
  bar_named(bar, NT);
  if (zt < NCOL) {
    // the partials hold sums of bq = q + kRoundBits + 128 (mod 2^32); the sum of q itself
    // is below 2^31 in magnitude (at most 1024 columns of |q| <= 32512)
    uint32_t sum = 0u;
    for (int w = 0; w < nw; ++w) sum += static_cast<uint32_t>(ctl->wpart[w][zt]);
    sum -= static_cast<uint32_t>(gcols) * (kRoundBits + 128u);
    ctl->csum[slot][zt] = static_cast<int>(sum);
  }
  bar_named(bar, NT);
}

// A set built from global memory (the epilogue warps, in the background).
template <int B, int G>
__device__ void build_set_global(const DecodeArgs<G>& p, Ctl* ctl, int slot, uint8_t* set, GroupRef gr, int zt,
                                 int NT, int bar) {
  const DecodeLin& L = lin_at(p, gr.l);
  const Group g = group_of(L, gr.cg, Cfg<B>::C);
  SetSrc S;
  S.v = record(L, g.i) + v_offset(L) + static_cast<size_t>(g.col0) * 32;
  S.x = static_cast<const uint16_t*>(L.x) + g.col0;
  S.is = L.inv_s + g.col0;
  S.xs = L.d;
  build_set<B, true>(p, ctl, slot, set, S, g.gcols, zt, NT, bar);
}

// MMA issued by the elected lane of a warp whose lanes hold the same operands.
__device__ __forceinline__ void mma_i8_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, 1;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

template <int B, int G>
__global__ void __launch_bounds__(Cfg<B>::THREADS, 1) decode_kernel(const __grid_constant__ DecodeArgs<G> p) {
  using K = Cfg<B>;
  constexpr int NB = K::NB, NCOL = K::NCOL, C = K::C, NS = K::NS, T = K::T, NACC = K::NACC;
  constexpr uint32_t IDESC = make_idesc(2u, 1u, 1u, 128u, NB);   // s32 <- s8 x s8, M = 128, N = NB
  constexpr uint32_t FULL = 0xffffffffu;

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sets = smem;                              // 2 activation sets (1024-aligned)
  uint8_t* stages = smem + 2 * K::SET;               // sign stages
  Ctl* ctl = reinterpret_cast<Ctl*>(stages + NS * K::STAGE);
  uint8_t* stg = reinterpret_cast<uint8_t*>(ctl) + K::CTL;   // first group: x rows, then 1/s
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, grid = gridDim.x;
  int s0, s1;
  cta_range(p, cta, grid, s0, s1);
  const int nseg = s1 - s0;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  const Seg sg0 = seg_of(s0, p, C);
  const Seg sgz = seg_of(s1 - 1, p, C);
  // chunk groups this CTA touches (consecutive in the launch's numbering)
  const int NZ = (lin_at(p, sgz.l).cg0 + sgz.cg) - (lin_at(p, sg0.l).cg0 + sg0.cg) + 1;
  const DecodeLin& L0 = lin_at(p, sg0.l);            // the linear of the first segment

  griddep_launch_dependents();

  // ------------------------------------------------------------------ set-up -----
  if (warp == K::WCTL) {
    tmem_alloc(&ctl->tmem_base, 512);
    if (lane == 0) {
      for (int s = 0; s < NS; ++s) {
        mbar_init(&ctl->sfull[s], 1);
        mbar_init(&ctl->sempty[s], 4 * C);          // four warps per unit, C units per stage
      }
      for (int t = 0; t < 3; ++t)
        for (int q = 0; q < kSlots; ++q) {
          mbar_init(&ctl->aempty[t][q], 1);
          mbar_init(&ctl->ready[t][q], 4);
        }
      for (int a = 0; a < 4; ++a) {
        mbar_init(&ctl->accfull[a], C);              // one commit per unit
        mbar_init(&ctl->acc_free[a], 4);
      }
      mbar_init(&ctl->vstage, 1);
      mbar_init(&ctl->xstage, 1);
      for (int z = 0; z < 2; ++z) mbar_init(&ctl->zready[z], 1);
      for (int w = 0; w < K::NI; ++w) mbar_init(&ctl->drain[w], 1);
      ctl->abort = 0;
      ctl->nred = 0;
      ctl->count_ok = 0;
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == K::WCTL) {
    // ------------------------------------------------------------- copy warp ---------
    // Issuing a bulk copy costs the issuing thread a few hundred cycles, so the first
    // stages (and the first group's inputs) are issued by the lanes in parallel, one copy
    // each; later stages, which wait for freed slots, by lane 0.
    const bool skip_first = p.inject_unreachable && cta == 0;   // timeout test: see below
    auto issue_stage = [&](int jj, const Seg& sg) {
      const int st = jj % NS;
      const uint32_t bytes = static_cast<uint32_t>(sg.len) * kTileBytes;
      mbar_arrive_expect_tx(&ctl->sfull[st], bytes);
      const DecodeLin& L = lin_at(p, sg.l);
      bulk_g2s(stages + st * K::STAGE,
               record(L, sg.i) + (static_cast<size_t>(sg.rt) * L.KG + sg.kgA) * kTileBytes, bytes, &ctl->sfull[st]);
    };
    // The first group's V rows (into the second set slot) and 1/s, and the first stages:
    // stack memory and the scale vector, read before the previous kernel has finished.
    // (Timeout test: CTA 0 leaves out its first stage, so its waits run out while the
    // other CTAs complete and count their partials.)
    const Group G0 = group_of(L0, sg0.cg, C);
    const int first = min(NS, nseg);
    if (lane == 31) {
      mbar_arrive_expect_tx(&ctl->vstage, static_cast<uint32_t>(G0.gcols) * 36u);
      bulk_g2s(sets + K::SET, record(L0, G0.i) + v_offset(L0) + static_cast<size_t>(G0.col0) * 32,
               static_cast<uint32_t>(G0.gcols) * 32u, &ctl->vstage);
      bulk_g2s(stg + B * C * kTileCols * 2, L0.inv_s + G0.col0, static_cast<uint32_t>(G0.gcols) * 4u, &ctl->vstage);
    }
    if (lane < first && !(skip_first && lane == 0)) issue_stage(lane, seg_of(s0 + lane, p, C));
    // x only after the kernel ahead has finished (it may have written x)
    griddep_wait();
    if (lane == 0) mbar_arrive_expect_tx(&ctl->xstage, static_cast<uint32_t>(B * G0.gcols) * 2u);
    __syncwarp();
    if (lane < B)
      bulk_g2s(stg + lane * C * kTileCols * 2, static_cast<const uint16_t*>(L0.x) + static_cast<size_t>(lane) * L0.d + G0.col0,
               static_cast<uint32_t>(G0.gcols) * 2u, &ctl->xstage);
    if (lane == 0) {
      Seg sc = seg_of(s0 + first, p, C);   // the segment of the next stage to issue
      int issued = first;
      bool ok = true;
      for (; issued < nseg; ++issued) {
        ok = mbar_wait(&ctl->sempty[issued % NS], static_cast<uint32_t>((issued / NS - 1) & 1), deadline, abort_flag);
        if (!ok) break;
        issue_stage(issued, sc);
        seg_next(sc, p, C);
      }
      if (!ok) set_error(p, ctl);
      // no copy may still be landing in shared memory when the CTA exits
      const uint64_t drain_by = globaltimer_ns() + 100000000ull;
      for (int e = (issued > NS ? issued - NS : 0); e < issued; ++e) {
        if (skip_first && e == 0) continue;
        mbar_wait(&ctl->sfull[e % NS], static_cast<uint32_t>((e / NS) & 1), drain_by, nullptr);
      }
      mbar_wait(&ctl->vstage, 0, drain_by, nullptr);
      mbar_wait(&ctl->xstage, 0, drain_by, nullptr);
    }
  } else {
    // ---- every other warp: build the first activation set together --------------------
    {
      const int zt = threadIdx.x;   // 0 .. ZTHREADS - 1
      // warm L2 with the V rows of the second group (stack memory, read before the kernel
      // ahead has finished); the first group's inputs arrive in shared memory
      if (NZ > 1) {
        const GroupRef g1 = group_next(GroupRef{sg0.l, sg0.cg}, p);
        const DecodeLin& L1 = lin_at(p, g1.l);
        const Group G1 = group_of(L1, g1.cg, C);
        for (int c = zt; c < G1.gcols; c += K::ZTHREADS)
          prefetch_l2(record(L1, G1.i) + v_offset(L1) + static_cast<size_t>(G1.col0 + c) * 32);
      }
      griddep_wait();   // the workspace, y and x belong to this launch only from here on
      bool ok = mbar_wait(&ctl->vstage, 0, deadline, abort_flag);
      ok = ok && mbar_wait(&ctl->xstage, 0, deadline, abort_flag);
      if (!ok) set_error(p, ctl);   // the set is then garbage; every later wait sees the abort flag
      const Group G0 = group_of(L0, sg0.cg, C);
      SetSrc S;
      S.v = sets + K::SET;
      S.x = reinterpret_cast<const uint16_t*>(stg);
      S.is = reinterpret_cast<const float*>(stg + B * C * kTileCols * 2);
      S.xs = C * kTileCols;
      build_set<B, false>(p, ctl, 0, sets, S, G0.gcols, zt, K::ZTHREADS, kBarZ);
    }

    if (warp < K::WISS) {
      // ---------------------------------- teams: expand signs into tensor memory -----
      const int team = warp >> 2, q = warp & 3;
      const int tid = 32 * q + lane;                              // row of the unit = TMEM lane
      const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
      int j = 0, c = 0, u = 0, k = 0;
      Seg sg = sg0;
      while (j < nseg) {
        if (u % T == team) {
          const int slot = k % kSlots, use = k / kSlots;
          const int st = j % NS;
          bool ok = true;
          if (use > 0) ok = mbar_wait(&ctl->aempty[team][slot], static_cast<uint32_t>((use - 1) & 1), deadline, abort_flag);
          if (ok) ok = mbar_wait(&ctl->sfull[st], static_cast<uint32_t>((j / NS) & 1), deadline, abort_flag);
          ok = __all_sync(FULL, ok);
          if (!ok) {
            set_error(p, ctl);
            break;
          }
          const uint8_t* tile = stages + st * K::STAGE + c * kTileBytes;
          const uint4 wa = *reinterpret_cast<const uint4*>(tile + tid * 16);
          const uint4 wb = *reinterpret_cast<const uint4*>(tile + 2048 + tid * 16);
          const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
          const uint32_t acol = K::ACOL0 + 64u * static_cast<uint32_t>(team * kSlots + slot);
          // byte q of word pw is sign column 32 t + 4 pw + q in bit t: K-step t of the
          // unit is bit t of every byte (the device tile order), moved to bit 7
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t r[32];
#pragma unroll
            for (int tt = 0; tt < 4; ++tt)
#pragma unroll
              for (int pw = 0; pw < 8; ++pw) r[tt * 8 + pw] = sign_bytes(w[pw], 4 * h + tt);
            tmem_st32(tmem + lane_base + acol + 32u * h, r);
          }
          __syncwarp();
          if (lane == 0) {   // this warp's rows of the stage are in registers
            mbar_arrive(&ctl->sempty[st]);
            if (c == sg.len - 1)
              for (int e = sg.len; e < C; ++e) mbar_arrive(&ctl->sempty[st]);
          }
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->ready[team][slot]);
          ++k;
        }
        ++u;
        if (++c == sg.len) {
          c = 0;
          ++j;
          seg_next(sg, p, C);
        }
      }
    } else if (warp < K::WEPI) {
      // ------------------------------------------ MMA issuers (warp-uniform, elect) -----
      const int w = warp - K::WISS;
      int j = 0, c = 0, u = 0, zk = 0, waited_zk = 0, checked_j = -1;
      bool ok = true, any = false;
      Seg sg = sg0;
      while (j < nseg && ok) {
        if (u % K::NI == w) {
          const int team = u % T, k = u / T, slot = k % kSlots, use = k / kSlots;
          const int a = j % NACC;
          // the slot's four quadrants are stored
          ok = mbar_wait(&ctl->ready[team][slot], static_cast<uint32_t>(use & 1), deadline, abort_flag);
          // the sets of groups 1, 2, ... are built by the epilogue warps
          if (ok && zk > waited_zk) {
            ok = mbar_wait(&ctl->zready[zk & 1], static_cast<uint32_t>(((zk - 1) >> 1) & 1), deadline, abort_flag);
            waited_zk = zk;
          }
          // the segment's accumulator has been read and zeroed
          if (ok && checked_j != j) {
            ok = mbar_wait(&ctl->acc_free[a], static_cast<uint32_t>((j / NACC) & 1), deadline, abort_flag);
            checked_j = j;
          }
          ok = __all_sync(FULL, ok);
          if (!ok) break;
          tc_fence_after();
          // K-step t of the chunk starts t * NB * 32 bytes further (the descriptor's address
          // field counts 16-byte units; shared-memory addresses stay below 256 KB)
          const uint64_t bdesc0 = smem_desc_noswizzle(smem_u32(sets + (zk & 1) * K::SET + c * K::ZB), 128, 256);
          const uint32_t adst = tmem + static_cast<uint32_t>(a * NB);
          const uint32_t asrc = tmem + K::ACOL0 + 64u * static_cast<uint32_t>(team * kSlots + slot);
#pragma unroll
          for (int t = 0; t < 8; ++t)
            mma_i8_elect(adst, asrc + 8u * t, bdesc0 + static_cast<uint64_t>((t * (NB / 8) * 256) >> 4), IDESC);
          commit_elect(&ctl->aempty[team][slot]);
          commit_elect(&ctl->accfull[a]);
          if (c == sg.len - 1 && lane == 0)
            for (int e = sg.len; e < C; ++e) mbar_arrive(&ctl->accfull[a]);
          any = true;
        }
        ++u;
        if (++c == sg.len) {
          c = 0;
          ++j;
          const int cg = sg.cg, l = sg.l;
          seg_next(sg, p, C);
          if (sg.cg != cg || sg.l != l) ++zk;
        }
      }
      if (!ok) set_error(p, ctl);
      if (any) {   // no MMA may still read or write tensor memory at exit
        commit_elect(&ctl->drain[w]);
        mbar_wait(&ctl->drain[w], 0, globaltimer_ns() + 100000000ull, nullptr);
      }
    } else {
      // ------------------------------------- epilogue, partials, row-tile reduction -----
      const int q = warp & 3;
      const int et = threadIdx.x - 32 * K::WEPI;                   // 0 .. 127
      const int tid = 32 * q + lane;                               // row of the tile = TMEM lane
      const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
      uint32_t zr[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) zr[e] = 0u;
      // accumulators start at zero (the MMAs only accumulate): zero and release them all
#pragma unroll
      for (int cc = 0; cc < NACC * NB; cc += 32) tmem_st32(tmem + lane_base + cc, zr);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        for (int a = 0; a < NACC; ++a) mbar_arrive(&ctl->acc_free[a]);
      // the CTA's second chunk group (if any) is built here, while the teams and issuers
      // work through the first
      if (NZ > 1) {
        build_set_global<B>(p, ctl, 1, sets + K::SET, group_next(GroupRef{sg0.l, sg0.cg}, p), et, 128, kBarEpi);
        if (et == 0) mbar_arrive(&ctl->zready[1]);
      }
      bool failed = false;
      int zk = 0;
      Seg sg = sg0;
      for (int j = 0; j < nseg; ++j, seg_next(sg, p, C)) {
        const int a = j % NACC;
        const DecodeLin& L = lin_at(p, sg.l);
        const uint4* urow = reinterpret_cast<const uint4*>(record(L, sg.i) + u_offset(L) +
                                                           static_cast<size_t>(sg.rt * kTileRows + tid) * kK * 2);
        const uint4 ua = __ldg(urow), ub = __ldg(urow + 1);
        bool ok = !failed && mbar_wait(&ctl->accfull[a], static_cast<uint32_t>((j / NACC) & 1), deadline, abort_flag);
        ok = __all_sync(FULL, ok);
        if (ok) {
          tc_fence_after();
          const float* sig = ctl->sig[zk & 1];
          const int* cs = ctl->csum[zk & 1];
          const __half* uh = reinterpret_cast<const __half*>(&ua);
          const __half* uh2 = reinterpret_cast<const __half*>(&ub);
          const uint32_t abase = tmem + lane_base + static_cast<uint32_t>(a * NB);
          float part[B];
#pragma unroll
          for (int b = 0; b < B; ++b) {
            uint32_t vh[16], vl[16];
            tmem_ld16(abase + b * 16, vh);
            tmem_ld16(abase + NCOL + b * 16, vl);
            tc_wait_ld();
            float acc = 0.0f;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int col = b * 16 + jj;
              // the accumulators hold -128 sum_c Sb hi and -128 sum_c Sb lo (exact
              // multiples); S = 1 - 2 Sb:  T / sigma = sum_c q - 2 sum_c Sb q, in int32
              const int sh = -static_cast<int>(vh[jj]) >> 7, sl = -static_cast<int>(vl[jj]) >> 7;
              const int tq = cs[col] - 2 * (256 * sh + sl);
              const float uj = __half2float(jj < 8 ? uh[jj] : uh2[jj - 8]);
              acc = fmaf(__fmul_rn(uj, sig[col]), static_cast<float>(tq), acc);
            }
            part[b] = acc;
          }
          // zero the accumulator for the segment NACC later and hand it back
#pragma unroll
          for (int cc = 0; cc < NB; cc += 32) tmem_st32(abase + cc, zr);
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->acc_free[a]);
          float* dst = L.part + static_cast<size_t>(sg.sl) * B * kTileRows;
#pragma unroll
          for (int b = 0; b < B; ++b) dst[b * kTileRows + tid] = part[b];
        } else {
          set_error(p, ctl);
          failed = true;   // keep walking: every warp must pass the same barriers below
        }
        const bool group_end = (j + 1 == nseg) || sg.rt + 1 == L.RT;
        if (group_end) {
          // this group's set and its sig / csum are no longer read: build group zk + 2
          // (if the CTA has one) into the same slot
          if (bar_any(kBarEpi, 128, failed || *abort_flag != 0)) {
            failed = true;
          } else if (zk + 2 < NZ) {
            build_set_global<B>(p, ctl, zk & 1, sets + (zk & 1) * K::SET,
                                group_next(group_next(GroupRef{sg.l, sg.cg}, p), p), et, 128, kBarEpi);
            if (et == 0) mbar_arrive(&ctl->zready[zk & 1]);
          }
          ++zk;
        }
      }
      const bool stop = bar_any(kBarEpi, 128, failed || *abort_flag != 0);
      if (et == 0) ctl->count_ok = stop ? 0 : 1;
    }
  }

  // --------------------------------------------------- row tiles: count and reduce -----
  // Every warp of the CTA takes part.  The CTA counts its partials into the row tiles'
  // arrival counters; the CTA that adds a tile's last partial sums all of them and
  // writes y.  No CTA waits for another; a CTA that failed counts nothing.  The sum has
  // a fixed association whichever CTA runs it: thread (row r, slice k) of the K =
  // threads / 128 slices adds the partials of chunk groups k, k + K, ... in order, and
  // the K slice sums are added in slice order.
  tc_fence_before();
  __syncthreads();
  if (ctl->count_ok) {
    constexpr int KS = K::THREADS / kTileRows;   // slices per row tile
    const int r = threadIdx.x % kTileRows, ks = threadIdx.x / kTileRows;
    // the sign stages are drained by now: [4 tiles][KS][B][128] slice sums, then the row
    // tiles (linear << 16 | row tile) this CTA completed in the current round
    float* red = reinterpret_cast<float*>(stages);
    int* red_rt = reinterpret_cast<int*>(stages + 4 * KS * B * kTileRows * 4);
    for (int base = 0; base < nseg; base += K::THREADS) {
      const int e = base + static_cast<int>(threadIdx.x);
      if (e < nseg) {
        const Seg se = seg_of(s0 + e, p, C);
        const DecodeLin& L = lin_at(p, se.l);
        // acquire-release at GPU scope: releases this CTA's partials (the barrier above
        // orders every thread's stores before it) and, for the last arrival, acquires
        // all the others' (the barrier below orders this CTA's reads after it)
        if (atom_add_acq_rel_gpu(L.cnt + se.rt, 1u) == static_cast<uint32_t>(L.n * L.NCB - 1)) {
          const int idx = atomicAdd(&ctl->nred, 1);
          red_rt[idx] = (se.l << 16) | se.rt;
        }
      }
      __syncthreads();
      const int nred = ctl->nred;
      // up to kTB row tiles per pass, their loads all in flight together
      constexpr int kTB = 4;
      for (int q0 = 0; q0 < nred; q0 += kTB) {
        const int nq = min(kTB, nred - q0);
        if (ks < KS) {
          const float* pp[kTB];
          size_t stride[kTB];
          int nc[kTB];
          int ncmax = 0;
#pragma unroll
          for (int t = 0; t < kTB; ++t) {
            const int code = t < nq ? red_rt[q0 + t] : red_rt[q0];
            const DecodeLin& L = lin_at(p, code >> 16);
            pp[t] = L.part + static_cast<size_t>(code & 0xffff) * B * kTileRows + r;
            stride[t] = static_cast<size_t>(L.RT) * B * kTileRows;
            nc[t] = t < nq ? L.n * L.NCB : 0;   // partials of the row tile
            ncmax = max(ncmax, nc[t]);
          }
          float acc[kTB][B];
#pragma unroll
          for (int t = 0; t < kTB; ++t)
#pragma unroll
            for (int b = 0; b < B; ++b) acc[t][b] = 0.0f;
          for (int c0 = ks; c0 < ncmax; c0 += 4 * KS) {
            float v[kTB][4][B];
#pragma unroll
            for (int t = 0; t < kTB; ++t) {
#pragma unroll
              for (int e2 = 0; e2 < 4; ++e2)
#pragma unroll
                for (int b = 0; b < B; ++b) {
                  const int cg = c0 + e2 * KS;
                  v[t][e2][b] = cg < nc[t] ? __ldcg(pp[t] + cg * stride[t] + b * kTileRows) : 0.0f;
                }
            }
#pragma unroll
            for (int t = 0; t < kTB; ++t)
#pragma unroll
              for (int e2 = 0; e2 < 4; ++e2)
#pragma unroll
                for (int b = 0; b < B; ++b) acc[t][b] += v[t][e2][b];
          }
#pragma unroll
          for (int t = 0; t < kTB; ++t)
#pragma unroll
            for (int b = 0; b < B; ++b) red[((t * KS + ks) * B + b) * kTileRows + r] = acc[t][b];
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < nq * kTileRows; idx += K::THREADS) {
          const int t = idx / kTileRows, rr = idx - t * kTileRows;
          const int code = red_rt[q0 + t], rt = code & 0xffff;
          const DecodeLin& L = lin_at(p, code >> 16);
#pragma unroll
          for (int b = 0; b < B; ++b) {
            float sum = 0.0f;
            for (int k = 0; k < KS; ++k) sum += red[((t * KS + k) * B + b) * kTileRows + rr];
            store_y(L.y, p.x_bf16, static_cast<size_t>(b) * L.m + static_cast<size_t>(rt) * kTileRows + rr, sum);
          }
          if (rr == 0) L.cnt[rt] = 0u;   // the next call starts from zero
        }
        __syncthreads();
      }
      if (threadIdx.x == 0) ctl->nred = 0;
      __syncthreads();
    }
  }

  if (warp == K::WCTL) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int B, int G>
cudaError_t launch_b(const DecodeArgs<G>& p, int grid, cudaStream_t stream) {
  using K = Cfg<B>;
  auto kern = decode_kernel<B, G>;
  static bool configured[64] = {};   // the attribute is set once per device, outside any capture
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = stream;
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(K::THREADS);
  cfg.dynamicSmemBytes = K::SMEM;
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
    case 1: return launch_b<1, 1>(p, grid, stream);
    case 2: return launch_b<2, 1>(p, grid, stream);
    case 3: return launch_b<3, 1>(p, grid, stream);
    case 4: return launch_b<4, 1>(p, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_group(const DecodeGroupParams& p, int batch, int grid, cudaStream_t stream) {
  switch (batch) {
    case 1: return launch_b<1, kDecodeGroupMax>(p, grid, stream);
    case 2: return launch_b<2, kDecodeGroupMax>(p, grid, stream);
    case 3: return launch_b<3, kDecodeGroupMax>(p, grid, stream);
    case 4: return launch_b<4, kDecodeGroupMax>(p, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace bs
