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
//  * Z_i is quantised to two int8 planes (hi, lo) per column with a per-column scale
//    sigma = max_c|x'[b,c]| * max_c|V_i[c,j]| / 127, so S_i Z_i runs on the int8 tensor
//    cores (tcgen05.mma kind::i8) with exact int32 accumulation.  S = 1 - 2 Sb with
//    Sb in {0, 1} the stored bit; the 1 part is a column sum added in the epilogue.
//  * Sign bits are expanded in registers straight into u8 operands: one AND (and a
//    shift for G < 8) per 4 columns gives bytes {0, 2^g}, g = K-step mod G; each g has
//    its own TMEM accumulator and the epilogue recombines them exactly in int32.  The
//    expanded A operand goes to tensor memory (tcgen05.st), never to shared memory.
//  * One persistent launch: CTA c first quantises its share of the (block, 256-column)
//    activation chunks and publishes each with an epoch flag; then it walks a
//    contiguous range of units (row tile, block, 256-column group) in stream-K order:
//    sign tiles (4 KiB) and activation chunks arrive by bulk copies into a ring of
//    shared-memory stages, four warps expand signs into TMEM, one thread issues MMAs.
//    Row tiles split across CTAs are reduced in fixed CTA order by the last CTA to
//    arrive (an epoch-tagged counter), so results are deterministic.
//  * Every wait is bounded; a wait that runs out sets the device error word, and the
//    CTA drains its copies and MMAs, frees tensor memory and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace bs {
namespace {

constexpr int kThreads = 288;
constexpr int kWarpIss0 = 4;   // warps 4..7: MMA issuers (lane 0 each)
constexpr int kWarpZ = 8;      // activation-chunk copies; allocates TMEM
constexpr int kABufs = 4;      // A-operand buffers in TMEM (64 columns each, from column 256)
constexpr uint32_t kAcol0 = 256;
constexpr int kBarExp = 1;     // named barrier: the four expander warps (128 threads)
constexpr int kBarA = 2;       // named barrier: expander + issuer warps (256 threads), phase A
constexpr int kMaxBlocks = kDecodeMaxBlocks;  // blocks whose |V| column maxima are staged in smem
// Sign tiles stream through shared memory by per-thread 16-byte asynchronous copies
// (each expander thread copies and later reads only its own row's 32 bytes), kSignAhead
// units ahead, one commit group per unit (at most 8 groups outstanding per thread).
// 1-D bulk copies of 4-16 KiB moved far less than HBM bandwidth here.
constexpr int kSignAhead = 8;
// Activation chunks come from L2 by 1-D bulk copies (the TMA engine), in groups of
// consecutive units of one segment (contiguous in memory).  Keeping them off the
// load/store path matters: behind the HBM-latency sign copies on that path, these L2
// hits waited microseconds.
__host__ __device__ constexpr int zgroup(int B) { return B == 1 ? 2 : 1; }       // units per chunk copy
__host__ __device__ constexpr int zstages(int B) { return B == 1 ? 4 : (B == 2 ? 4 : (B == 3 ? 3 : 2)); }

struct Ctl {
  uint64_t afull[kABufs], aempty[kABufs], accfull, accempty, drain[4];
  uint32_t tmem_base;
  uint32_t tag, wait_tag, epoch;
  int abort;
  int is_last;
  float amax[kDecodeMaxBatch];
  float cseg[16 * kDecodeMaxBatch];
  float sig_lo[16 * kDecodeMaxBatch];
  int zsum[16 * kDecodeMaxBatch];
  float vmax[kMaxBlocks * kK];
};

// Shared-memory carve-up:
//   [kSignAhead sign slots of 4 KiB][zstages activation stages][phase-A scratch]
//   [barriers][Ctl];  activation stage = [chunk ZB][column sums 64 B per batch row]
constexpr int kScratchBytes = kTileCols * kK * 2 + kTileCols * kDecodeMaxBatch * 4;  // V chunk + x' chunk
__host__ __device__ constexpr int zstage_bytes(int B) {
  return (zgroup(B) * (32 * B * kTileCols + 64 * B) + 127) / 128 * 128;
}
// Units [u, end) of the group that starts at unit u: at most `gs` units, never past
// the end of u's segment (same row tile and block) or of the CTA's range.
__device__ __forceinline__ int group_len(long long u, long long u1, int KG, int gs) {
  const int kg = static_cast<int>(u % KG);  // per_rt is a multiple of KG
  long long end = u - kg + KG;
  if (end > u1) end = u1;
  const long long len = end - u;
  return static_cast<int>(len < gs ? len : gs);
}

__device__ __forceinline__ void exp_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBarExp), "n"(128) : "memory"); }
__device__ __forceinline__ void phase_a_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBarA), "n"(256) : "memory"); }

__device__ __forceinline__ void store_y(void* y, int bf16, size_t idx, float v) {
  if (bf16) static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(y)[idx] = __float2half_rn(v);
}
__device__ __forceinline__ void unpack8(const uint4& v, int bf16, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (bf16) {
      const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
      f[2 * e] = __bfloat162float(h.x);
      f[2 * e + 1] = __bfloat162float(h.y);
    } else {
      const __half2 h = *reinterpret_cast<const __half2*>(&w[e]);
      f[2 * e] = __half2float(h.x);
      f[2 * e + 1] = __half2float(h.y);
    }
  }
}
// Per-column quantisation step of the activation chunks: z ~ sigma_lo * q with
// |q| <= 127 * 256, split exactly into q = 256 * hi + lo, hi in [-127, 127],
// lo in [-128, 127]; so sigma_hi = 256 * sigma_lo.  The producer of a chunk and every
// consumer evaluate the same expression, so they agree bit for bit.
__device__ __forceinline__ float sigma_lo_of(float amax, float vmax) {
  const float s = __fmul_rn(__fmul_rn(amax, vmax), 1.0f / 32512.0f);
  return s > 0.0f ? s : 1.0f;
}

__device__ __forceinline__ void set_error(const DecodeParams& p, Ctl* ctl) {
  ctl->abort = 1;
  atomicOr(p.err, kErrTimeout);
}

// CTA owning unit u under the split u0(c) = floor(c U / grid).
__device__ __forceinline__ int cta_of(long long u, long long U, int grid) {
  return static_cast<int>(((u + 1) * grid + U - 1) / U) - 1;
}

template <int B, int G>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
  constexpr int NB = 32 * B;                 // MMA N: [hi plane 16B | lo plane 16B]
  constexpr int ZB = NB * kTileCols;         // bytes of one activation chunk
  constexpr int CB = 64 * B;                 // bytes of one chunk's column sums
  constexpr int ZST = zstage_bytes(B);
  constexpr int ZS = zstages(B);
  constexpr int GZ = zgroup(B);
  constexpr int NI = G < 4 ? G : 4;          // MMA issuers: issuer w owns groups g with g % NI == w
  constexpr uint32_t IDESC = make_idesc(2u, 0u, 1u, 128u, NB);  // s32 <- u8 x s8, M=128, N=NB
  static_assert(G * NB <= 256, "accumulators must fit below the A buffers");

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* zst_base = smem + kSignAhead * kTileBytes;
  uint8_t* scratch = zst_base + ZS * ZST;
  uint64_t* zfull = reinterpret_cast<uint64_t*>(scratch + kScratchBytes);
  uint64_t* zempty = zfull + ZS;
  Ctl* ctl = reinterpret_cast<Ctl*>(zempty + ZS);
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, grid = gridDim.x;
  const long long U = p.units;
  const long long u0 = static_cast<long long>(cta) * U / grid;
  const long long u1 = static_cast<long long>(cta + 1) * U / grid;
  const int KG = p.KG;
  const int per_rt = p.n * KG;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  const size_t sign_bytes = static_cast<size_t>(p.m) * p.d / 8;

  // Expander threads start streaming their sign rows before anything else.
  auto sign_src = [&](long long u) {
    const long long rt = u / per_rt, rem = u % per_rt;
    const int i = static_cast<int>(rem / KG), kg = static_cast<int>(rem % KG);
    return p.blocks + static_cast<size_t>(i) * p.block_bytes + (static_cast<size_t>(rt) * KG + kg) * kTileBytes;
  };
  if (warp < 4) {
    for (int j = 0; j < kSignAhead; ++j) {
      if (u0 + j < u1) {
        const uint8_t* src = sign_src(u0 + j);
        uint8_t* dst = smem + j * kTileBytes;
        cp_async16(dst + threadIdx.x * 16, src + threadIdx.x * 16);
        cp_async16(dst + 2048 + threadIdx.x * 16, src + 2048 + threadIdx.x * 16);
      }
      cp_async_commit();
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < ZS; ++s) {
      mbar_init(&zfull[s], 1);
      mbar_init(&zempty[s], NI);
    }
    for (int a = 0; a < kABufs; ++a) {
      mbar_init(&ctl->afull[a], 128);
      mbar_init(&ctl->aempty[a], NI);
    }
    mbar_init(&ctl->accfull, NI);
    mbar_init(&ctl->accempty, 128);
    for (int w = 0; w < 4; ++w) mbar_init(&ctl->drain[w], 1);
    ctl->abort = 0;
    const uint32_t e = *reinterpret_cast<volatile uint32_t*>(p.hdr);
    ctl->epoch = e;
    ctl->tag = e + 1u;
    ctl->wait_tag = p.inject_unreachable ? ((e + 1u) ^ 0x80000000u) : (e + 1u);
    for (int i = 0; i < 16 * kDecodeMaxBatch; ++i) ctl->zsum[i] = 0;
    for (int b = 0; b < kDecodeMaxBatch; ++b) ctl->amax[b] = 0.0f;
    fence_barrier_init();
  }
  if (warp == kWarpZ) tmem_alloc(&ctl->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t tag = ctl->tag, wait_tag = ctl->wait_tag;

  if (warp == kWarpZ) {
    // ---------------------------------------------- activation-chunk producer -----
    // All 32 lanes first wait, in parallel, for every chunk this CTA will read; then
    // each chunk is copied by all lanes (16-byte cp.async), whose arrivals complete
    // the stage's barrier.
    const long long count = u1 - u0;
    const int distinct = static_cast<int>(count < per_rt ? count : per_rt);
    bool ok = true;
    for (int idx = lane; idx < distinct && ok; idx += 32) {
      const int q = static_cast<int>((u0 + idx) % per_rt);
      while (ld_acquire_u32(p.flags + q) != wait_tag) {
        if (*abort_flag || globaltimer_ns() > deadline) { ok = false; break; }
        __nanosleep(32);
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) set_error(p, ctl);
    if (lane == 0) {
      long long g = 0;
      if (ok) {
        fence_proxy_async_global();   // the chunks were written by generic stores
        for (long long u = u0; u < u1; ++g) {
          const int len = group_len(u, u1, KG, GZ);
          const int s = static_cast<int>(g % ZS);
          const long long ph = g / ZS;
          if (ph > 0 && !mbar_wait(&zempty[s], static_cast<uint32_t>((ph - 1) & 1), deadline, abort_flag)) {
            set_error(p, ctl);
            break;
          }
          const int q = static_cast<int>(u % per_rt);  // chunk index i * KG + kg
          uint8_t* st = zst_base + static_cast<size_t>(s) * ZST;
          mbar_arrive_expect_tx(&zfull[s], static_cast<uint32_t>(len) * (ZB + CB));
          bulk_g2s(st, p.zq + static_cast<size_t>(q) * ZB, static_cast<uint32_t>(len) * ZB, &zfull[s]);
          bulk_g2s(st + GZ * ZB, p.csum + static_cast<size_t>(q) * 16 * B, static_cast<uint32_t>(len) * CB, &zfull[s]);
          u += len;
        }
      }
      const long long issued = g;
      for (long long j = (issued > ZS ? issued - ZS : 0); j < issued; ++j)
        mbar_wait(&zfull[j % ZS], static_cast<uint32_t>((j / ZS) & 1), globaltimer_ns() + 100000000ull, nullptr);
    }
  } else {
    // --------- warps 0-7: phase A (quantise and publish the owned activation chunks) ---
    const int ta = threadIdx.x;  // 0..255
    const int chunks = p.n * KG;
    // Inputs of the first chunk this CTA owns are loaded before the |x| scan so that
    // both round trips to memory overlap.
    uint4 vv0 = make_uint4(0, 0, 0, 0), vv1 = make_uint4(0, 0, 0, 0);
    float xsv[B];
    auto load_chunk = [&](int q) {
      const int i = q / KG, c0 = (q % KG) * kTileCols;
      const uint8_t* vsrc = p.blocks + static_cast<size_t>(i) * p.block_bytes + sign_bytes +
                            static_cast<size_t>(2) * kK * p.m;
      const uint4* v4 = reinterpret_cast<const uint4*>(vsrc + static_cast<size_t>(c0) * kK * 2);
      vv0 = __ldg(v4 + ta);
      vv1 = __ldg(v4 + ta + 256);                                              // 512 x 16 B = 8 KiB
      const float is = __ldg(p.inv_s + c0 + ta);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const size_t xi = static_cast<size_t>(b) * p.d + c0 + ta;
        const float xv = p.x_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.x)[xi])
                                  : __half2float(static_cast<const __half*>(p.x)[xi]);
        xsv[b] = __fmul_rn(xv, is);
      }
    };
    if (cta < chunks) load_chunk(cta);
    {
      for (int e = ta; e < p.n * kK && e < kMaxBlocks * kK; e += 256) ctl->vmax[e] = __ldg(p.vmax + e);
      // max_c |x[b, c] / s_c| for every row b of x, 8 columns per load
      float mx[B];
#pragma unroll
      for (int b = 0; b < B; ++b) mx[b] = 0.0f;
      const int nvec = p.d / 8;
      for (int v0 = ta; v0 < nvec; v0 += 256 * 2) {
        uint4 xv[2][B];
        float4 sv[2][2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int v = v0 + r * 256;
          if (v < nvec) {
            sv[r][0] = __ldg(reinterpret_cast<const float4*>(p.inv_s) + 2 * v);
            sv[r][1] = __ldg(reinterpret_cast<const float4*>(p.inv_s) + 2 * v + 1);
#pragma unroll
            for (int b = 0; b < B; ++b)
              xv[r][b] = __ldg(reinterpret_cast<const uint4*>(p.x) + static_cast<size_t>(b) * nvec + v);
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (v0 + r * 256 < nvec) {
            const float is[8] = {sv[r][0].x, sv[r][0].y, sv[r][0].z, sv[r][0].w,
                                 sv[r][1].x, sv[r][1].y, sv[r][1].z, sv[r][1].w};
#pragma unroll
            for (int b = 0; b < B; ++b) {
              float f[8];
              unpack8(xv[r][b], p.x_bf16, f);
#pragma unroll
              for (int e = 0; e < 8; ++e) mx[b] = fmaxf(mx[b], fabsf(__fmul_rn(f[e], is[e])));
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float v = mx[b];
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) atomicMax(reinterpret_cast<int*>(&ctl->amax[b]), __float_as_int(v));
      }
      phase_a_sync();
    }
    float amax[B];
#pragma unroll
    for (int b = 0; b < B; ++b) amax[b] = ctl->amax[b];
    {
      __half* vs = reinterpret_cast<__half*>(scratch);                       // [256][16]
      float* xs = reinterpret_cast<float*>(scratch + kTileCols * kK * 2);     // [B][256]
      for (int q = cta; q < chunks; q += grid) {
        const int i = q / KG;
        if (q != cta) load_chunk(q);
        reinterpret_cast<uint4*>(vs)[ta] = vv0;
        reinterpret_cast<uint4*>(vs)[ta + 256] = vv1;
#pragma unroll
        for (int b = 0; b < B; ++b) xs[b * kTileCols + ta] = xsv[b];
        phase_a_sync();
        uint8_t* zdst = p.zq + static_cast<size_t>(q) * ZB;
        for (int it = ta; it < 16 * B * 16; it += 256) {
          const int cg = it / (16 * B);          // 16-column group of the chunk
          const int col = it % (16 * B);         // b * 16 + j
          const int b = col / 16, j = col % 16;
          const float slo = sigma_lo_of(amax[b], ctl->vmax[i * 16 + j]);
          const float rlo = 1.0f / slo;
          uint32_t hw[4] = {0, 0, 0, 0}, lw[4] = {0, 0, 0, 0};
          int sq = 0;
#pragma unroll
          for (int kin = 0; kin < 16; ++kin) {
            const int cl = cg * 16 + kin;
            const float z = __fmul_rn(xs[b * kTileCols + cl], __half2float(vs[cl * kK + j]));
            int qv = __float2int_rn(z * rlo);
            qv = max(-32512, min(32512, qv));
            const int qh = (qv + 128) >> 8;
            const int ql = qv - (qh << 8);
            sq += qv;
            hw[kin >> 2] |= (static_cast<uint32_t>(qh) & 0xFFu) << (8 * (kin & 3));
            lw[kin >> 2] |= (static_cast<uint32_t>(ql) & 0xFFu) << (8 * (kin & 3));
          }
          // B operand layout: K-step t (32 columns), 8-row group n/8, K half kc.
          const int t = cg >> 1, kc = cg & 1;
          const int nh = col, nl = 16 * B + col;
          uint8_t* ph = zdst + ((t * (NB / 8) + nh / 8) * 2 + kc) * 128 + (nh % 8) * 16;
          uint8_t* pl = zdst + ((t * (NB / 8) + nl / 8) * 2 + kc) * 128 + (nl % 8) * 16;
          *reinterpret_cast<uint4*>(ph) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(pl) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          atomicAdd(&ctl->zsum[col], sq);
        }
        phase_a_sync();
        if (ta < 16 * B) {
          const int b = ta / 16, j = ta % 16;
          const float slo = sigma_lo_of(amax[b], ctl->vmax[i * 16 + j]);
          p.csum[static_cast<size_t>(q) * 16 * B + ta] = __fmul_rn(slo, static_cast<float>(ctl->zsum[ta]));
          ctl->zsum[ta] = 0;
        }
        phase_a_sync();
        if (ta == 0) {   // publish: every write of the chunk happens before the release
          __threadfence();
          st_release_u32(p.flags + q, tag);
        }
      }
    }

    if (warp >= kWarpIss0) {
      // ---------------------------------------------------------- MMA issuers -----
      const int w = warp - kWarpIss0;
      if (lane == 0 && w < NI) {
        long long k = 0;
        int seg = 0;
        bool issued_any = false;
        long long zg = -1;   // chunk group of the current unit, its length and position
        int zlen = 0, zpos = 0;
        for (long long u = u0; u < u1; ++u, ++k) {
          if (zpos == zlen) {
            ++zg;
            zpos = 0;
            zlen = group_len(u, u1, KG, GZ);
          }
          const int zs = static_cast<int>(zg % ZS);
          const uint32_t zph = static_cast<uint32_t>((zg / ZS) & 1);
          const int a = static_cast<int>(k % kABufs);
          const uint32_t pa = static_cast<uint32_t>((k / kABufs) & 1);
          const int kg = static_cast<int>((u % per_rt) % KG);
          const bool seg_start = (u == u0) || (kg == 0);
          const bool seg_end = (u + 1 == u1) || (kg == KG - 1);
          if (!mbar_wait(&zfull[zs], zph, deadline, abort_flag) ||
              !mbar_wait(&ctl->afull[a], pa, deadline, abort_flag) ||
              (seg_start && seg > 0 &&
               !mbar_wait(&ctl->accempty, static_cast<uint32_t>((seg - 1) & 1), deadline, abort_flag))) {
            set_error(p, ctl);
            break;
          }
          tc_fence_after();
          const uint32_t zaddr = smem_u32(zst_base + static_cast<size_t>(zs) * ZST + static_cast<size_t>(zpos) * ZB);
          const uint32_t acol = kAcol0 + 64u * static_cast<uint32_t>(a);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int g = t % G;
            if (g % NI != w) continue;
            const uint64_t bdesc = smem_desc_noswizzle(zaddr + t * (NB / 8) * 256, 128, 256);
            mma_i8_ts(tmem + g * NB, tmem + acol + 8 * t, bdesc, IDESC, (seg_start && t < G) ? 0u : 1u);
          }
          issued_any = true;
          if (++zpos == zlen) tc_commit(&zempty[zs]);   // the group's chunks are consumed
          tc_commit(&ctl->aempty[a]);
          if (seg_end) {
            tc_commit(&ctl->accfull);
            ++seg;
          }
        }
        if (issued_any) {
          tc_commit(&ctl->drain[w]);
          mbar_wait(&ctl->drain[w], 0, globaltimer_ns() + 100000000ull, nullptr);
        }
      }
    } else {
      // ------------------------------------------ warps 0-3: expand, epilogue -----
      const int tid = threadIdx.x;  // 0..127 = row within the tile = TMEM lane
      const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
      // Control flow is uniform across the 128 threads: a thread whose wait ran out
      // keeps walking the loop in "failed" mode, skipping work but passing every
      // named barrier; each warp decides failure by vote so warp-collective tcgen05
      // ops stay uniform.
      float ypart[B];
#pragma unroll
      for (int b = 0; b < B; ++b) ypart[b] = 0.0f;
      float cacc = 0.0f;  // column-sum accumulator of this segment (threads < 16B)
      uint4 ua = make_uint4(0, 0, 0, 0), ub = make_uint4(0, 0, 0, 0);   // this row of U_i
      long long k = 0;
      int seg = 0;
      long long zg = -1;   // chunk group of the current unit, its length and position
      int zlen = 0, zpos = 0;
      bool failed = false;
      auto check = [&](bool ok) {
        if (!__all_sync(0xffffffffu, ok)) failed = true;
      };
      for (long long u = u0; u < u1; ++u, ++k) {
        const bool new_zgroup = (zpos == zlen);
        if (new_zgroup) {
          ++zg;
          zpos = 0;
          zlen = group_len(u, u1, KG, GZ);
        }
        const int slot = static_cast<int>(k % kSignAhead);
        const int zs = static_cast<int>(zg % ZS);
        const uint32_t zph = static_cast<uint32_t>((zg / ZS) & 1);
        const int a = static_cast<int>(k % kABufs);
        const long long pa = k / kABufs;
        const long long rt = u / per_rt, rem = u % per_rt;
        const int i = static_cast<int>(rem / KG), kg = static_cast<int>(rem % KG);
        const bool seg_start = (u == u0) || (kg == 0);
        if (seg_start) {
          cacc = 0.0f;
          const uint8_t* urow = p.blocks + static_cast<size_t>(i) * p.block_bytes + sign_bytes +
                                (static_cast<size_t>(rt) * kTileRows + tid) * kK * 2;
          ua = __ldg(reinterpret_cast<const uint4*>(urow));
          ub = __ldg(reinterpret_cast<const uint4*>(urow + 16));
        }
        // this unit's sign words (own row, own copies) and the next prefetch
        cp_async_wait<kSignAhead - 1>();
        uint8_t* sdst = smem + slot * kTileBytes;
        const uint4 wa = *reinterpret_cast<const uint4*>(sdst + tid * 16);
        const uint4 wb = *reinterpret_cast<const uint4*>(sdst + 2048 + tid * 16);
        if (u + kSignAhead < u1) {
          const uint8_t* src = sign_src(u + kSignAhead);
          cp_async16(sdst + tid * 16, src + tid * 16);
          cp_async16(sdst + 2048 + tid * 16, src + 2048 + tid * 16);
        }
        cp_async_commit();
        const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
        if (!failed) {
          if (new_zgroup) check(mbar_wait(&zfull[zs], zph, deadline, abort_flag));
          if (!failed && tid < 16 * B)
            cacc += reinterpret_cast<const float*>(zst_base + static_cast<size_t>(zs) * ZST + GZ * ZB)[zpos * 16 * B + tid];
          if (!failed && pa > 0)
            check(mbar_wait(&ctl->aempty[a], static_cast<uint32_t>((pa - 1) & 1), deadline, abort_flag));
        }
        if (!failed) {
          const uint32_t abase = tmem + lane_base + kAcol0 + 64u * static_cast<uint32_t>(a);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t r[32];
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
              const int t = 4 * h + tt;
              const int g = t % G;
              const uint32_t mask = 0x01010101u << g;
#pragma unroll
              for (int pw = 0; pw < 8; ++pw) r[tt * 8 + pw] = (w[pw] >> (t - g)) & mask;
            }
            tmem_st32(abase + 32 * h, r);
          }
          tc_wait_st();
          tc_fence_before();
          mbar_arrive(&ctl->afull[a]);
        }
        ++zpos;

        const bool seg_end = (u + 1 == u1) || (kg == KG - 1);
        if (seg_end) {
          if (tid < 16 * B) {
            const int b = tid / 16, j = tid % 16;
            ctl->cseg[tid] = cacc;
            ctl->sig_lo[tid] = sigma_lo_of(amax[b], ctl->vmax[i * 16 + j]);
          }
          exp_sync();
          if (!failed) check(mbar_wait(&ctl->accfull, static_cast<uint32_t>(seg & 1), deadline, abort_flag));
          if (!failed) {
            tc_fence_after();
            const __half* uh = reinterpret_cast<const __half*>(&ua);
            const __half* uh2 = reinterpret_cast<const __half*>(&ub);
            const float ginv = 1.0f / static_cast<float>(1 << (G - 1));
#pragma unroll
            for (int b = 0; b < B; ++b) {
              int ch[16], cl[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) { ch[j] = 0; cl[j] = 0; }
#pragma unroll
              for (int g = 0; g < G; ++g) {
                uint32_t vh[16], vl[16];
                tmem_ld16(tmem + lane_base + g * NB + b * 16, vh);
                tmem_ld16(tmem + lane_base + g * NB + 16 * B + b * 16, vl);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  ch[j] = 2 * ch[j] + static_cast<int>(vh[j]);
                  cl[j] = 2 * cl[j] + static_cast<int>(vl[j]);
                }
              }
              float acc = 0.0f;
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float slo = ctl->sig_lo[b * 16 + j];
                const float sbz = (256.0f * slo * static_cast<float>(ch[j]) + slo * static_cast<float>(cl[j])) * ginv;
                // S = 1 - 2 Sb (bit 1 = sign -1):  T = sum_c Z - 2 sum_c Sb Z
                const float tval = ctl->cseg[b * 16 + j] - 2.0f * sbz;
                const float uj = __half2float(j < 8 ? uh[j] : uh2[j - 8]);
                acc = fmaf(uj, tval, acc);
              }
              ypart[b] += acc;
            }
            tc_fence_before();
            mbar_arrive(&ctl->accempty);
          }
          exp_sync();  // cseg and the scales are rewritten by the next segment
          ++seg;
        }

        const bool rt_end = (u + 1 == u1) || (rem == per_rt - 1);
        if (rt_end) {
          const long long first_u = rt * per_rt, last_u = first_u + per_rt - 1;
          const size_t row = static_cast<size_t>(rt) * kTileRows + tid;
          if (first_u >= u0 && last_u < u1) {
            if (!failed) {
#pragma unroll
              for (int b = 0; b < B; ++b) store_y(p.y, p.x_bf16, static_cast<size_t>(b) * p.m + row, ypart[b]);
            }
          } else {
            const int slot2 = (rt == u0 / per_rt) ? 0 : 1;
            float* mine = p.part + (static_cast<size_t>(cta) * 2 + slot2) * B * kTileRows;
#pragma unroll
            for (int b = 0; b < B; ++b) mine[b * kTileRows + tid] = ypart[b];
            __threadfence();
            exp_sync();
            const int c_first = cta_of(first_u, U, grid), c_last = cta_of(last_u, U, grid);
            if (tid == 0) {
              unsigned long long* cp = p.cnt + rt;
              unsigned long long expect = *reinterpret_cast<volatile unsigned long long*>(cp);
              unsigned long long now = 0;
              while (true) {
                const bool same = static_cast<uint32_t>(expect >> 32) == tag;
                const unsigned long long nv =
                    same ? expect + 1ull : ((static_cast<unsigned long long>(tag) << 32) | 1ull);
                const unsigned long long prev = atomicCAS(cp, expect, nv);
                if (prev == expect) { now = nv; break; }
                expect = prev;
              }
              ctl->is_last = static_cast<int>(now & 0xffffffffull) == (c_last - c_first + 1);
            }
            exp_sync();
            if (ctl->is_last && !*abort_flag) {
              __threadfence();
              float acc[B];
#pragma unroll
              for (int b = 0; b < B; ++b) acc[b] = 0.0f;
              for (int c = c_first; c <= c_last; ++c) {
                const long long cu0 = static_cast<long long>(c) * U / grid;
                const int cslot = (rt == cu0 / per_rt) ? 0 : 1;
                const float* pp = p.part + (static_cast<size_t>(c) * 2 + cslot) * B * kTileRows;
#pragma unroll
                for (int b = 0; b < B; ++b) acc[b] += __ldcg(pp + b * kTileRows + tid);
              }
#pragma unroll
              for (int b = 0; b < B; ++b) store_y(p.y, p.x_bf16, static_cast<size_t>(b) * p.m + row, acc[b]);
            }
            exp_sync();  // is_last is rewritten by the next row tile
          }
#pragma unroll
          for (int b = 0; b < B; ++b) ypart[b] = 0.0f;
        }
      }
      if (failed) set_error(p, ctl);
    }
  }
  if (warp < 4) cp_async_wait<0>();   // no sign copy is in flight at exit

  __syncthreads();
  if (warp == kWarpZ) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // The last CTA to leave advances the workspace epoch for the next launch.
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t done = atomicAdd(p.hdr + 1, 1u);
    if (done == static_cast<uint32_t>(grid) - 1u) {
      p.hdr[1] = 0u;
      __threadfence();
      atomicExch(p.hdr, ctl->epoch + 1u);
    }
  }
}

template <int B>
cudaError_t launch_b(const DecodeParams& p, int grid, cudaStream_t stream) {
  // G groups of K-steps, limited by the 256 TMEM accumulator columns (G * 32B <= 256).
  constexpr int G = (B == 1) ? 8 : (B == 2 ? 4 : 2);
  auto kern = decode_kernel<B, G>;
  const size_t smem = decode_smem_bytes(B, p.stages);
  static int configured = 0;  // the attribute is set once (stream capture never sees it)
  if (configured < static_cast<int>(smem)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured = static_cast<int>(smem);
  }
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t decode_smem_bytes(int batch, int /*stages*/) {
  const int zs = zstages(batch);
  return static_cast<size_t>(kSignAhead) * kTileBytes + static_cast<size_t>(zs) * zstage_bytes(batch) + kScratchBytes +
         2 * zs * sizeof(uint64_t) + sizeof(Ctl) + 64;
}

int decode_pick_stages(int /*batch*/) { return kSignAhead; }

cudaError_t launch_decode(const DecodeParams& p, int batch, int grid, int /*sm_count*/, cudaStream_t stream) {
  switch (batch) {
    case 1: return launch_b<1>(p, grid, stream);
    case 2: return launch_b<2>(p, grid, stream);
    case 3: return launch_b<3>(p, grid, stream);
    case 4: return launch_b<4>(p, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace bs
