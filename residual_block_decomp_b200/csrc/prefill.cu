// Prefill kernel of the BitStack linear: y = x W_hat_n^T for many rows of x.
//
// The weight is the sum of the loaded residual blocks, sign_i (.) (U_i V_i^T), with
// the activation-aware scale undone per input channel (weight restoration snippet of
// the OpenReview discussion of "BitStack: Any-Size Compression of Large Language
// Models in Variable Memory Environments"; review page "BitStack: Fine-Grained Size
// Control...", Figs. 3 and 5).  With many rows of x the dense contraction dominates,
// so each CTA rebuilds tiles of W_hat on chip and never writes them to device memory:
//
//   for each 32-column K-tile of its 128 output rows:
//     P_i = U_i[rows] V_i[cols]^T          rank-16 tcgen05 MMA (fp16) -> TMEM, per block
//     W_t = (sum_i sign_i (.) P_i) / s     TMEM -> registers, sign applied by XOR
//     W_t -> fp16/bf16 -> shared memory    the A operand of the GEMM
//     y_tile += W_t x_tile^T               tcgen05 MMA, M = 128 rows, N = NT tokens
//
// Operands arrive by TMA (x tiles, U and V tiles; no multicast) and 1-D bulk copies
// (sign tiles).  Warp roles: warps 0-3 rebuild and write the epilogue (thread = row =
// TMEM lane), warp 4 issues copies, warp 5 owns TMEM and issues MMAs.  All waits are
// bounded; a wait that runs out sets the device error word and the CTA unwinds.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace bs {
namespace {

constexpr int kThreads = 192;
constexpr int kWarpLoad = 4, kWarpMma = 5;
constexpr int kKT = 32;              // K columns per tile
constexpr int kPRound = 8;           // blocks whose P tiles fit TMEM at once
constexpr uint32_t kPcol = 256;      // TMEM column of the P region (acc at 0..NT)
constexpr int kBarRb = 1;

struct Ctl {
  uint64_t ubar, pfull, pempty, accfull, drain;
  uint64_t wfull[2], wempty[2];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void rb_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBarRb), "n"(128) : "memory"); }

template <typename DT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <typename DT>
__device__ __forceinline__ DT cvt_out(float v);
template <>
__device__ __forceinline__ __half cvt_out<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 cvt_out<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

struct Layout {
  int u_off, s_off, x_off, v_off, w_off, ctl_off, total;
  int s_stride, x_stride, v_stride;
};
__host__ __device__ inline Layout prefill_layout(int n, int NT, int xstages, int sbufs) {
  Layout L{};
  int off = 0;
  L.u_off = off;  off += n * 4096;                          // U tiles, 128 x 16 fp16 per block
  L.s_stride = n * kTileBytes;
  L.s_off = off;  off += sbufs * L.s_stride;                // sign tiles of one 256-column group
  L.x_stride = NT * kKT * 2;
  L.x_off = off;  off += xstages * L.x_stride;              // x tiles, NT x 32
  L.v_stride = n * 1024;
  L.v_off = off;  off += xstages * L.v_stride;              // V tiles, 32 x 16 per block
  L.w_off = off;  off += 2 * kTileRows * kKT * 2;           // W_hat tiles, 128 x 32, double buffered
  off = (off + 7) & ~7;
  L.ctl_off = off;
  off += static_cast<int>(sizeof(Ctl)) + 2 * xstages * 8 + 2 * sbufs * 8;
  L.total = off;
  return L;
}

template <typename DT>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int n = p.n, NT = p.NT, XS = p.xstages, SB = p.sbufs;
  const Layout L = prefill_layout(n, NT, XS, SB);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + L.ctl_off);
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + L.ctl_off + sizeof(Ctl));
  uint64_t* xempty = xfull + XS;
  uint64_t* sgfull = xempty + XS;
  uint64_t* sgempty = sgfull + SB;
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rt = blockIdx.x;
  const int tok0 = blockIdx.y * NT;
  const int KT = p.d / kKT;
  const int rounds = (n + kPRound - 1) / kPRound;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  const uint32_t is_bf16 = std::is_same<DT, __nv_bfloat16>::value ? 1u : 0u;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->ubar, 1);
    mbar_init(&ctl->pfull, 1);
    mbar_init(&ctl->pempty, 128);
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->drain, 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(&ctl->wfull[w], 128);
      mbar_init(&ctl->wempty[w], 1);
    }
    for (int s = 0; s < XS; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&sgfull[s], 1);
      mbar_init(&sgempty[s], 128);
    }
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) tmem_alloc(&ctl->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == kWarpLoad) {
    // ----------------------------------------------------------------- loader -----
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_u);
      prefetch_tmap(&tm_v);
      bool ok = true;
      mbar_arrive_expect_tx(&ctl->ubar, static_cast<uint32_t>(n) * 4096u);
      for (int i = 0; i < n; ++i) {
        tma_load_3d(smem + L.u_off + i * 4096, &tm_u, 0, rt * kTileRows, i, &ctl->ubar);
        tma_load_3d(smem + L.u_off + i * 4096 + 2048, &tm_u, 8, rt * kTileRows, i, &ctl->ubar);
      }
      int kt = 0;
      for (; kt < KT && ok; ++kt) {
        if (kt % 8 == 0) {
          const int grp = kt / 8, sb = grp % SB, use = grp / SB;
          if (use > 0 && !mbar_wait(&sgempty[sb], static_cast<uint32_t>((use - 1) & 1), deadline, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sgfull[sb], static_cast<uint32_t>(n) * kTileBytes);
          for (int i = 0; i < n; ++i) {
            const uint8_t* src = p.blocks + static_cast<size_t>(i) * p.block_bytes +
                                 (static_cast<size_t>(rt) * p.KG + grp) * kTileBytes;
            bulk_g2s(smem + L.s_off + sb * L.s_stride + i * kTileBytes, src, kTileBytes, &sgfull[sb]);
          }
        }
        const int s = kt % XS, use = kt / XS;
        if (use > 0 && !mbar_wait(&xempty[s], static_cast<uint32_t>((use - 1) & 1), deadline, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&xfull[s], static_cast<uint32_t>(n) * 1024u + static_cast<uint32_t>(NT) * kKT * 2u);
        uint8_t* vb = smem + L.v_off + s * L.v_stride;
        for (int i = 0; i < n; ++i) {
          tma_load_3d(vb + i * 1024, &tm_v, 0, kt * kKT, i, &xfull[s]);
          tma_load_3d(vb + i * 1024 + 512, &tm_v, 8, kt * kKT, i, &xfull[s]);
        }
        uint8_t* xb = smem + L.x_off + s * L.x_stride;
        for (int kc = 0; kc < 4; ++kc) tma_load_2d(xb + kc * NT * 16, &tm_x, kt * kKT + 8 * kc, tok0, &xfull[s]);
      }
      if (!ok) {
        ctl->abort = 1;
        atomicOr(p.err, kErrTimeout);
      }
      // drain the copies issued last on every barrier
      mbar_wait(&ctl->ubar, 0, globaltimer_ns() + 100000000ull, nullptr);
      const int issued = kt;
      for (int j = (issued > XS ? issued - XS : 0); j < issued; ++j)
        mbar_wait(&xfull[j % XS], static_cast<uint32_t>((j / XS) & 1), globaltimer_ns() + 100000000ull, nullptr);
      const int groups = (issued + 7) / 8;
      for (int g = (groups > SB ? groups - SB : 0); g < groups; ++g)
        mbar_wait(&sgfull[g % SB], static_cast<uint32_t>((g / SB) & 1), globaltimer_ns() + 100000000ull, nullptr);
    }
  } else if (warp == kWarpMma) {
    // -------------------------------------------------------------- MMA issuer -----
    if (lane == 0) {
      const uint32_t idesc_p = make_idesc(1u, 0u, 0u, 128u, 32u);                 // f32 <- f16 x f16
      const uint32_t idesc_g = make_idesc(1u, is_bf16, is_bf16, 128u, static_cast<uint32_t>(NT));
      bool ok = mbar_wait(&ctl->ubar, 0, deadline, abort_flag);
      bool issued_any = false;
      int prounds = 0;  // P rounds issued so far (parity of pfull / pempty)
      for (int kt = 0; kt < KT && ok; ++kt) {
        const int s = kt % XS;
        const int w = kt & 1;
        if (!mbar_wait(&xfull[s], static_cast<uint32_t>((kt / XS) & 1), deadline, abort_flag)) { ok = false; break; }
        const uint32_t vaddr = smem_u32(smem + L.v_off + s * L.v_stride);
        const uint32_t uaddr = smem_u32(smem + L.u_off);
        for (int r = 0; r < rounds && ok; ++r) {
          if (prounds > 0 &&
              !mbar_wait(&ctl->pempty, static_cast<uint32_t>((prounds - 1) & 1), deadline, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int i1 = min(n, (r + 1) * kPRound);
          for (int i = r * kPRound; i < i1; ++i) {
            const uint64_t adesc = smem_desc_noswizzle(uaddr + i * 4096, 2048, 128);
            const uint64_t bdesc = smem_desc_noswizzle(vaddr + i * 1024, 512, 128);
            mma_f16_ss(tmem + kPcol + (i - r * kPRound) * 32, adesc, bdesc, idesc_p, 0u);
          }
          issued_any = true;
          tc_commit(&ctl->pfull);
          ++prounds;
        }
        if (!ok) break;
        if (!mbar_wait(&ctl->wfull[w], static_cast<uint32_t>((kt >> 1) & 1), deadline, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t waddr = smem_u32(smem + L.w_off + w * kTileRows * kKT * 2);
        const uint32_t xaddr = smem_u32(smem + L.x_off + s * L.x_stride);
        for (int kk = 0; kk < 2; ++kk) {
          const uint64_t adesc = smem_desc_noswizzle(waddr + kk * 2 * 2048, 2048, 128);
          const uint64_t bdesc = smem_desc_noswizzle(xaddr + kk * 2 * NT * 16, NT * 16, 128);
          mma_f16_ss(tmem, adesc, bdesc, idesc_g, (kt > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&ctl->wempty[w]);
        tc_commit(&xempty[s]);
      }
      if (ok) {
        tc_commit(&ctl->accfull);
      } else {
        ctl->abort = 1;
        atomicOr(p.err, kErrTimeout);
      }
      if (issued_any) {
        tc_commit(&ctl->drain);
        mbar_wait(&ctl->drain, 0, globaltimer_ns() + 100000000ull, nullptr);
      }
    }
  } else {
    // ------------------------------------------ warps 0-3: rebuild, epilogue -------
    const int tid = threadIdx.x;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    bool failed = false;
    auto check = [&](bool ok) {
      if (!__all_sync(0xffffffffu, ok)) failed = true;
    };
    int prounds = 0;
    for (int kt = 0; kt < KT; ++kt) {
      const int grp = kt / 8, t = kt % 8, sb = grp % SB;
      const int w = kt & 1;
      if (t == 0 && !failed) check(mbar_wait(&sgfull[sb], static_cast<uint32_t>((grp / SB) & 1), deadline, abort_flag));
      float acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0.0f;
      const uint8_t* sbase = smem + L.s_off + sb * L.s_stride;
      for (int r = 0; r < rounds; ++r) {
        if (!failed) check(mbar_wait(&ctl->pfull, static_cast<uint32_t>(prounds & 1), deadline, abort_flag));
        if (!failed) {
          tc_fence_after();
          const int i1 = min(n, (r + 1) * kPRound);
          for (int i = r * kPRound; i < i1; ++i) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + kPcol + (i - r * kPRound) * 32, v);
            const uint4 wa = *reinterpret_cast<const uint4*>(sbase + i * kTileBytes + tid * 16);
            const uint4 wb = *reinterpret_cast<const uint4*>(sbase + i * kTileBytes + 2048 + tid * 16);
            const uint32_t wd[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              // column c of the K-tile is bit 8 (c % 4) + t of word c / 4
              const uint32_t sgn = (wd[c >> 2] << (31 - (8 * (c & 3) + t))) & 0x80000000u;
              acc[c] += __uint_as_float(v[c] ^ sgn);
            }
          }
          tc_fence_before();
          mbar_arrive(&ctl->pempty);
        }
        ++prounds;
      }
      if (!failed && t == 7) mbar_arrive(&sgempty[sb]);
      uint32_t packed[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float s0 = __ldg(p.inv_s + kt * kKT + c), s1 = __ldg(p.inv_s + kt * kKT + c + 1);
        packed[c / 2] = pack2<DT>(acc[c] * s0, acc[c + 1] * s1);
      }
      if (kt >= 2 && !failed) check(mbar_wait(&ctl->wempty[w], static_cast<uint32_t>(((kt >> 1) - 1) & 1), deadline, abort_flag));
      if (!failed) {
        uint8_t* wb = smem + L.w_off + w * kTileRows * kKT * 2;
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) {
          *reinterpret_cast<uint4*>(wb + kc * 2048 + (tid >> 3) * 128 + (tid & 7) * 16) =
              make_uint4(packed[4 * kc], packed[4 * kc + 1], packed[4 * kc + 2], packed[4 * kc + 3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&ctl->wfull[w]);
      }
    }
    // epilogue: accumulator row `tid` holds NT token outputs
    if (!failed) check(mbar_wait(&ctl->accfull, 0, deadline, abort_flag));
    if (!failed) {
      tc_fence_after();
      DT* y = static_cast<DT*>(p.y);
      const size_t row = static_cast<size_t>(rt) * kTileRows + tid;
      for (int ch = 0; ch < NT / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + ch * 32, v);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int tok = tok0 + ch * 32 + j;
          if (tok < p.M) y[static_cast<size_t>(tok) * p.m + row] = cvt_out<DT>(__uint_as_float(v[j]));
        }
      }
      tc_fence_before();
    }
    if (failed) {
      ctl->abort = 1;
      atomicOr(p.err, kErrTimeout);
    }
  }

  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t prefill_smem_bytes(int n, int NT, int xstages, int sbufs) {
  return static_cast<size_t>(prefill_layout(n, NT, xstages, sbufs).total) + 64;
}

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_u,
                           const CUtensorMap& tm_v, int bf16, cudaStream_t stream) {
  const size_t smem = prefill_smem_bytes(p.n, p.NT, p.xstages, p.sbufs);
  dim3 grid(p.m / kTileRows, (p.M + p.NT - 1) / p.NT);
  // the attribute is per device and kernel: set it once for each (device, dtype), outside
  // any stream capture (the first call on a device must not be captured)
  static bool configured[64][2] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev][bf16 ? 1 : 0]) {
    e = bf16 ? cudaFuncSetAttribute(prefill_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(227 * 1024))
             : cudaFuncSetAttribute(prefill_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(227 * 1024));
    if (e != cudaSuccess) return e;
    configured[dev][bf16 ? 1 : 0] = true;
  }
  if (bf16) {
    prefill_kernel<__nv_bfloat16><<<grid, kThreads, smem, stream>>>(p, tm_x, tm_u, tm_v);
  } else {
    prefill_kernel<__half><<<grid, kThreads, smem, stream>>>(p, tm_x, tm_u, tm_v);
  }
  return cudaGetLastError();
}

}  // namespace bs
