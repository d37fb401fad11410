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

constexpr int kThreads = 224;
constexpr int kWarpSign = 4;   // issues sign-tile bulk copies
constexpr int kWarpMma = 5;    // allocates TMEM, issues MMAs
constexpr int kWarpZ = 6;      // waits for activation chunks, issues their bulk copies
constexpr uint32_t kAcol0 = 256, kAcol1 = 384;  // TMEM columns of the two A buffers
constexpr int kBarExp = 1;     // named barrier of the four expander warps

struct Ctl {
  uint64_t afull[2], aempty[2], accfull, accempty, drain;
  uint32_t tmem_base;
  uint32_t tag, wait_tag, epoch;
  int abort;
  int is_last;
  float amax[kDecodeMaxBatch];
  float cseg[16 * kDecodeMaxBatch];
  int zsum[2][16 * kDecodeMaxBatch];
};

constexpr int kScratchBytes = kTileCols * kK * 2 + kTileCols * kDecodeMaxBatch * 4;  // V chunk + x' chunk

__device__ __forceinline__ void exp_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBarExp), "n"(128) : "memory"); }

__device__ __forceinline__ float load_x(const void* x, int x_bf16, size_t idx) {
  if (x_bf16) return __bfloat162float(static_cast<const __nv_bfloat16*>(x)[idx]);
  return __half2float(static_cast<const __half*>(x)[idx]);
}
__device__ __forceinline__ void store_y(void* y, int bf16, size_t idx, float v) {
  if (bf16) static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(y)[idx] = __float2half_rn(v);
}
// Per-column scales; the producer of a chunk and every consumer evaluate the same
// expressions, so they agree bit for bit.
__device__ __forceinline__ float sigma_hi(float amax, float vmax) {
  float s = __fmul_rn(__fmul_rn(amax, vmax), 1.0f / 127.0f);
  return s > 0.0f ? s : 1.0f;
}
__device__ __forceinline__ float sigma_lo(float shi) { return __fmul_rn(shi, 1.0f / 254.0f); }

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
  constexpr int STAGE = kTileBytes + ZB;
  constexpr uint32_t IDESC = make_idesc(2u, 0u, 1u, 128u, NB);  // s32 <- u8 x s8, M=128, N=NB
  static_assert(G * NB <= 256, "accumulators must fit below the A buffers");

  extern __shared__ __align__(1024) uint8_t smem[];
  const int S = p.stages;
  uint64_t* sfull = reinterpret_cast<uint64_t*>(smem + S * STAGE + kScratchBytes);
  uint64_t* zfull = sfull + S;
  uint64_t* sempty = zfull + S;
  Ctl* ctl = reinterpret_cast<Ctl*>(sempty + S);
  uint8_t* scratch = smem + S * STAGE;
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, grid = gridDim.x;
  const long long U = p.units;
  const long long u0 = static_cast<long long>(cta) * U / grid;
  const long long u1 = static_cast<long long>(cta + 1) * U / grid;
  const int KG = p.KG;
  const int per_rt = p.n * KG;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&zfull[s], 1);
      mbar_init(&sempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl->afull[a], 128);
      mbar_init(&ctl->aempty[a], 1);
    }
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->accempty, 128);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    const uint32_t e = *reinterpret_cast<volatile uint32_t*>(p.hdr);
    ctl->epoch = e;
    ctl->tag = e + 1u;
    ctl->wait_tag = p.inject_unreachable ? ((e + 1u) ^ 0x80000000u) : (e + 1u);
    for (int i = 0; i < 2 * 16 * kDecodeMaxBatch; ++i) (&ctl->zsum[0][0])[i] = 0;
    for (int b = 0; b < kDecodeMaxBatch; ++b) ctl->amax[b] = 0.0f;
    fence_barrier_init();
  }
  if (warp == kWarpMma) tmem_alloc(&ctl->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t tag = ctl->tag, wait_tag = ctl->wait_tag;

  if (warp == kWarpSign) {
    // ------------------------------------------------ sign-tile producer ----------
    if (lane == 0) {
      long long k = 0;
      for (long long u = u0; u < u1; ++u, ++k) {
        const int s = static_cast<int>(k % S);
        const long long ph = k / S;
        if (ph > 0 && !mbar_wait(&sempty[s], static_cast<uint32_t>((ph - 1) & 1), deadline, abort_flag)) {
          set_error(p, ctl);
          break;
        }
        const long long rt = u / per_rt, rem = u % per_rt;
        const int i = static_cast<int>(rem / KG), kg = static_cast<int>(rem % KG);
        const uint8_t* src = p.blocks + static_cast<size_t>(i) * p.block_bytes +
                             (static_cast<size_t>(rt) * KG + kg) * kTileBytes;
        mbar_arrive_expect_tx(&sfull[s], kTileBytes);
        bulk_g2s(smem + static_cast<size_t>(s) * STAGE, src, kTileBytes, &sfull[s]);
      }
      // drain: the latest phase issued on every stage must land before exit
      const long long issued = k;
      for (long long j = (issued > S ? issued - S : 0); j < issued; ++j) {
        const int s = static_cast<int>(j % S);
        mbar_wait(&sfull[s], static_cast<uint32_t>((j / S) & 1), globaltimer_ns() + 100000000ull, nullptr);
      }
    }
  } else if (warp == kWarpZ) {
    // ---------------------------------------------- activation-chunk producer -----
    if (lane == 0) {
      long long k = 0;
      for (long long u = u0; u < u1; ++u, ++k) {
        const int s = static_cast<int>(k % S);
        const long long ph = k / S;
        if (ph > 0 && !mbar_wait(&sempty[s], static_cast<uint32_t>((ph - 1) & 1), deadline, abort_flag)) {
          set_error(p, ctl);
          break;
        }
        const long long rem = u % per_rt;
        const int q = static_cast<int>(rem);  // chunk index i * KG + kg
        bool ok = true;
        while (ld_acquire_u32(p.flags + q) != wait_tag) {
          if (*abort_flag || globaltimer_ns() > deadline) { ok = false; break; }
          __nanosleep(64);
        }
        if (!ok) {
          set_error(p, ctl);
          break;
        }
        fence_proxy_async_global();
        mbar_arrive_expect_tx(&zfull[s], ZB);
        bulk_g2s(smem + static_cast<size_t>(s) * STAGE + kTileBytes, p.zq + static_cast<size_t>(q) * ZB, ZB,
                 &zfull[s]);
      }
      const long long issued = k;
      for (long long j = (issued > S ? issued - S : 0); j < issued; ++j) {
        const int s = static_cast<int>(j % S);
        mbar_wait(&zfull[s], static_cast<uint32_t>((j / S) & 1), globaltimer_ns() + 100000000ull, nullptr);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      long long k = 0;
      int seg = 0;
      bool issued_any = false;
      for (long long u = u0; u < u1; ++u, ++k) {
        const int s = static_cast<int>(k % S);
        const uint32_t ph = static_cast<uint32_t>((k / S) & 1);
        const int a = static_cast<int>(k & 1);
        const uint32_t pa = static_cast<uint32_t>((k >> 1) & 1);
        const int kg = static_cast<int>((u % per_rt) % KG);
        const bool seg_start = (u == u0) || (kg == 0);
        const bool seg_end = (u + 1 == u1) || (kg == KG - 1);
        if (!mbar_wait(&zfull[s], ph, deadline, abort_flag) || !mbar_wait(&ctl->afull[a], pa, deadline, abort_flag) ||
            (seg_start && seg > 0 &&
             !mbar_wait(&ctl->accempty, static_cast<uint32_t>((seg - 1) & 1), deadline, abort_flag))) {
          set_error(p, ctl);
          break;
        }
        tc_fence_after();
        const uint32_t zaddr = smem_u32(smem + static_cast<size_t>(s) * STAGE + kTileBytes);
        const uint32_t acol = a ? kAcol1 : kAcol0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int g = t % G;
          const uint64_t bdesc = smem_desc_noswizzle(zaddr + t * (NB / 8) * 256, 128, 256);
          mma_i8_ts(tmem + g * NB, tmem + acol + 8 * t, bdesc, IDESC, (seg_start && t < G) ? 0u : 1u);
        }
        issued_any = true;
        tc_commit(&sempty[s]);
        tc_commit(&ctl->aempty[a]);
        if (seg_end) {
          tc_commit(&ctl->accfull);
          ++seg;
        }
      }
      if (issued_any) {
        tc_commit(&ctl->drain);
        mbar_wait(&ctl->drain, 0, globaltimer_ns() + 100000000ull, nullptr);
      }
    }
  } else {
    // ------------------------------------- warps 0-3: quantise, expand, epilogue ---
    const int tid = threadIdx.x;  // 0..127 = row within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

    // Phase A.1: max_c |x[b, c] / s_c| for every row b of x.
    {
      float mx[B];
#pragma unroll
      for (int b = 0; b < B; ++b) mx[b] = 0.0f;
      for (int c = tid; c < p.d; c += 128) {
        const float is = __ldg(p.inv_s + c);
#pragma unroll
        for (int b = 0; b < B; ++b)
          mx[b] = fmaxf(mx[b], fabsf(__fmul_rn(load_x(p.x, p.x_bf16, static_cast<size_t>(b) * p.d + c), is)));
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float v = mx[b];
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) atomicMax(reinterpret_cast<int*>(&ctl->amax[b]), __float_as_int(v));
      }
      exp_sync();
    }
    float amax[B];
#pragma unroll
    for (int b = 0; b < B; ++b) amax[b] = ctl->amax[b];

    // Phase A.2: quantise and publish the activation chunks this CTA owns.
    {
      __half* vs = reinterpret_cast<__half*>(scratch);                       // [256][16]
      float* xs = reinterpret_cast<float*>(scratch + kTileCols * kK * 2);     // [B][256]
      const int chunks = p.n * KG;
      for (int q = cta; q < chunks; q += grid) {
        const int i = q / KG, kg = q % KG;
        const int c0 = kg * kTileCols;
        const uint8_t* vsrc = p.blocks + static_cast<size_t>(i) * p.block_bytes +
                              static_cast<size_t>(p.m) * p.d / 8 + static_cast<size_t>(2) * kK * p.m;
        const uint4* v4 = reinterpret_cast<const uint4*>(vsrc + static_cast<size_t>(c0) * kK * 2);
        for (int e = tid; e < kTileCols * kK * 2 / 16; e += 128) reinterpret_cast<uint4*>(vs)[e] = v4[e];
        for (int e = tid; e < B * kTileCols; e += 128) {
          const int b = e / kTileCols, cl = e % kTileCols;
          xs[e] = __fmul_rn(load_x(p.x, p.x_bf16, static_cast<size_t>(b) * p.d + c0 + cl), __ldg(p.inv_s + c0 + cl));
        }
        exp_sync();
        uint8_t* zdst = p.zq + static_cast<size_t>(q) * ZB;
        for (int it = tid; it < 16 * B * 16; it += 128) {
          const int cg = it / (16 * B);          // 16-column group of the chunk
          const int col = it % (16 * B);         // b * 16 + j
          const int b = col / 16, j = col % 16;
          const float vmx = __ldg(p.vmax + i * 16 + j);
          const float shi = sigma_hi(amax[b], vmx), slo = sigma_lo(shi);
          uint32_t hw[4] = {0, 0, 0, 0}, lw[4] = {0, 0, 0, 0};
          int sh = 0, sl = 0;
#pragma unroll
          for (int kin = 0; kin < 16; ++kin) {
            const int cl = cg * 16 + kin;
            const float z = __fmul_rn(xs[b * kTileCols + cl], __half2float(vs[cl * kK + j]));
            int qh = __float2int_rn(__fdiv_rn(z, shi));
            qh = max(-127, min(127, qh));
            const float r = __fsub_rn(z, __fmul_rn(static_cast<float>(qh), shi));
            int ql = __float2int_rn(__fdiv_rn(r, slo));
            ql = max(-127, min(127, ql));
            sh += qh;
            sl += ql;
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
          atomicAdd(&ctl->zsum[0][col], sh);
          atomicAdd(&ctl->zsum[1][col], sl);
        }
        exp_sync();
        if (tid < 16 * B) {
          const int b = tid / 16, j = tid % 16;
          const float shi = sigma_hi(amax[b], __ldg(p.vmax + i * 16 + j)), slo = sigma_lo(shi);
          p.csum[static_cast<size_t>(q) * 16 * B + tid] =
              __fadd_rn(__fmul_rn(shi, static_cast<float>(ctl->zsum[0][tid])),
                        __fmul_rn(slo, static_cast<float>(ctl->zsum[1][tid])));
          ctl->zsum[0][tid] = 0;
          ctl->zsum[1][tid] = 0;
        }
        fence_proxy_async_global();
        __threadfence();
        exp_sync();
        if (tid == 0) st_release_u32(p.flags + q, tag);
      }
    }

    // Main loop: expand signs into TMEM, run the epilogue at segment ends.  Control
    // flow is uniform across the 128 threads: a thread whose wait ran out keeps
    // walking the loop in "failed" mode, skipping work but passing every named
    // barrier, and each warp decides failure by vote so warp-collective tcgen05 ops
    // stay uniform.
    float ypart[B];
#pragma unroll
    for (int b = 0; b < B; ++b) ypart[b] = 0.0f;
    long long k = 0;
    int seg = 0;
    bool failed = false;
    auto check = [&](bool ok) {
      if (!__all_sync(0xffffffffu, ok)) failed = true;
    };
    for (long long u = u0; u < u1; ++u, ++k) {
      const int s = static_cast<int>(k % S);
      const uint32_t ph = static_cast<uint32_t>((k / S) & 1);
      const int a = static_cast<int>(k & 1);
      const long long pa = k >> 1;
      const long long rt = u / per_rt, rem = u % per_rt;
      const int i = static_cast<int>(rem / KG), kg = static_cast<int>(rem % KG);
      if (!failed) check(mbar_wait(&sfull[s], ph, deadline, abort_flag));
      uint32_t w[8];
      if (!failed) {
        const uint8_t* stile = smem + static_cast<size_t>(s) * STAGE;
        const uint4 wa = *reinterpret_cast<const uint4*>(stile + tid * 16);
        const uint4 wb = *reinterpret_cast<const uint4*>(stile + 2048 + tid * 16);
        w[0] = wa.x; w[1] = wa.y; w[2] = wa.z; w[3] = wa.w;
        w[4] = wb.x; w[5] = wb.y; w[6] = wb.z; w[7] = wb.w;
        if (pa > 0) check(mbar_wait(&ctl->aempty[a], static_cast<uint32_t>((pa - 1) & 1), deadline, abort_flag));
      }
      if (!failed) {
        const uint32_t abase = tmem + lane_base + (a ? kAcol1 : kAcol0);
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

      const bool seg_end = (u + 1 == u1) || (kg == KG - 1);
      if (seg_end) {
        // column sums of the dequantised chunks of this segment
        const int kg_start = (u - kg >= u0) ? 0 : static_cast<int>((u0 % per_rt) % KG);
        if (!failed && tid < 16 * B) {
          float c = 0.0f;
          bool ok = true;
          for (int g2 = kg_start; g2 <= kg && ok; ++g2) {
            const int q = i * KG + g2;
            while (ld_acquire_u32(p.flags + q) != wait_tag) {
              if (*abort_flag || globaltimer_ns() > deadline) { ok = false; break; }
            }
            if (ok) c = __fadd_rn(c, __ldcg(p.csum + static_cast<size_t>(q) * 16 * B + tid));
          }
          ctl->cseg[tid] = c;
          if (!ok) set_error(p, ctl);
        }
        exp_sync();
        if (!failed) check(*abort_flag == 0);
        if (!failed) check(mbar_wait(&ctl->accfull, static_cast<uint32_t>(seg & 1), deadline, abort_flag));
        if (!failed) {
          tc_fence_after();
          const size_t row = static_cast<size_t>(rt) * kTileRows + tid;
          const uint8_t* urow = p.blocks + static_cast<size_t>(i) * p.block_bytes +
                                static_cast<size_t>(p.m) * p.d / 8 + row * kK * 2;
          const uint4 ua = *reinterpret_cast<const uint4*>(urow);
          const uint4 ub = *reinterpret_cast<const uint4*>(urow + 16);
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
              const float shi = sigma_hi(amax[b], __ldg(p.vmax + i * 16 + j)), slo = sigma_lo(shi);
              const float sbz = (shi * static_cast<float>(ch[j]) + slo * static_cast<float>(cl[j])) * ginv;
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
        exp_sync();  // cseg is rewritten by the next segment
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
          const int slot = (rt == u0 / per_rt) ? 0 : 1;
          float* mine = p.part + (static_cast<size_t>(cta) * 2 + slot) * B * kTileRows;
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

  __syncthreads();
  if (warp == kWarpMma) {
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

size_t decode_smem_bytes(int batch, int stages) {
  const size_t stage = kTileBytes + static_cast<size_t>(32) * batch * kTileCols;
  return stage * stages + kScratchBytes + 3 * stages * sizeof(uint64_t) + sizeof(Ctl) + 64;
}

int decode_pick_stages(int batch) {
  const size_t budget = 200 * 1024;
  int s = 16;
  while (s > 2 && decode_smem_bytes(batch, s) > budget) --s;
  return s;
}

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
