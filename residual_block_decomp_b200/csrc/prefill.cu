// Prefill kernel of the BitStack linear: y = x W_hat_n^T for many rows of x.
//
// The weight is the sum of the loaded residual blocks, sign_i (.) (U_i V_i^T), with
// the activation-aware scale undone per input channel (weight restoration snippet of
// the OpenReview discussion of "BitStack: Any-Size Compression of Large Language
// Models in Variable Memory Environments"; review page "BitStack: Fine-Grained Size
// Control...", Figs. 3 and 5).  With many rows of x the dense contraction dominates,
// so tiles of W_hat are rebuilt on chip and never written to device memory:
//
//   for each 32-column K-tile of 128 output rows:
//     P_i = U_i[rows] V_i[cols]^T          rank-16 tcgen05 MMA (fp16) -> TMEM, per block,
//                                          four blocks per round, two rounds in flight
//     W_t = (sum_i sign_i (.) P_i) / s     TMEM -> registers, sign applied by XOR
//     W_t -> fp16/bf16 -> shared memory    the A operand of the GEMM
//     y_tile += W_t x_tile^T               tcgen05 MMA, M = 128 rows, N = NT tokens
//
// The CTAs of one 128-row tile that take different token tiles form a cluster of CN
// (1, 2 or 4) and share the rebuild: CTA rank r rebuilds the K-tiles kt = r (mod CN)
// and writes each rebuilt tile into the W ring of every CTA of the cluster (distributed
// shared memory), so a W tile is rebuilt once per cluster instead of once per CTA.
// Ring slot kt mod WS (WS = 2 CN, so each rank owns two slots and can fill one while the
// cluster still reads the other) is always filled by the same rank; a consumer's GEMM
// hands the slot back to that rank with a multicast tcgen05.commit.
//
// Operands arrive by TMA (x tiles in the 64-byte swizzle layout, U and V tiles; no
// multicast) and 1-D bulk copies (sign tiles).  Warp roles: warps 0-7 rebuild (two warps per TMEM lane quadrant, each
// taking half of a K-tile's columns; thread = row = TMEM lane) and write the epilogue,
// warp 8 copies x tiles, warp 10 copies the rebuild's U, V and sign tiles (so that
// neither stream waits behind the other's flow control), warp 9 owns TMEM and issues the
// GEMM, warp 11 issues the rank-16 products (two MMA streams that never wait on each
// other).  All mbarrier waits are
// bounded; a wait that runs out sets the device error word and the CTA unwinds.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace bs {
namespace {

constexpr int kThreads = 384;
constexpr int kWarpLoad = 8, kWarpMma = 9;    // warps 0-7 rebuild (two per TMEM lane quadrant)
constexpr int kWarpRbLoad = 10;               // U, V and sign tiles for the rebuild
constexpr int kWarpP = 11;                    // issues the rank-16 products of the rebuild
constexpr int kRb = 256;                      // rebuild threads
constexpr int kKT = 32;              // K columns per tile
constexpr int kPRound = 4;           // blocks per P round (one TMEM region of 128 columns)
constexpr uint32_t kPcol = 256;      // TMEM columns of the two P regions (acc at 0..NT)
constexpr int kVS = 2;               // V stages (the CTA's own K-tiles only)
constexpr int kMaxWS = 8;            // W ring slots at most
constexpr int kWTile = kTileRows * kKT * 2;   // bytes of one W tile

struct Ctl {
  uint64_t ubar, accfull, drain, drain_p;
  uint64_t pfull[2], pempty[2];      // P regions: products ready / read by the rebuild warps
  uint64_t wfull[kMaxWS];            // W slot filled (armed with the tile's bytes, completed by its copy)
  uint64_t wempty[kMaxWS];           // W slot read by every CTA of the cluster (one commit each)
  uint64_t vfull[kVS], vempty[kVS];  // V stages of the own K-tiles
  uint32_t tmem_base;
  int abort;
  int last;                          // split K: this CTA counted its tile's last partial
};

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
__host__ __device__ inline Layout prefill_layout(int n, int NT, int xstages, int sbufs, int ws) {
  Layout L{};
  int off = 0;
  L.u_off = off;  off += n * 4096;                          // U tiles, 128 x 16 fp16 per block
  L.s_stride = n * kTileBytes;
  L.s_off = off;  off += sbufs * L.s_stride;                // sign tiles of one 256-column group
  L.x_stride = NT * kKT * 2;
  L.x_off = off;  off += xstages * L.x_stride;              // x tiles, NT x 32
  L.v_stride = n * 1024;
  L.v_off = off;  off += kVS * L.v_stride;                  // V tiles of own K-tiles, 32 x 16 per block
  L.w_off = off;  off += ws * kWTile;                       // W_hat tiles, 128 x 32, a ring of ws
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
  const int n = p.n, NT = p.NT, XS = p.xstages, SB = p.sbufs, CN = p.CN;
  const int WS = CN > 1 ? 2 * CN : 2;               // W ring slots: two per rank of the cluster
  const Layout L = prefill_layout(n, NT, XS, SB, WS);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + L.ctl_off);
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + L.ctl_off + sizeof(Ctl));
  uint64_t* xempty = xfull + XS;
  uint64_t* sgfull = xempty + XS;
  uint64_t* sgempty = sgfull + SB;
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rt = blockIdx.x;
  const int tok0 = blockIdx.y * NT;
  const int rank = CN > 1 ? static_cast<int>(cluster_rank()) : 0;
  // this split's K-tiles kt0 .. kt0 + KT - 1 (kt0 a multiple of 8: whole sign groups);
  // below, kl = kt - kt0 indexes them
  const int kt0 = static_cast<int>(blockIdx.z) * p.kts;
  const int KT = min(p.kts, p.d / kKT - kt0);
  const int n_own = (KT - rank + CN - 1) / CN;      // own K-tiles kl = rank, rank + CN, ...
  const int rounds = (n + kPRound - 1) / kPRound;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  const uint32_t is_bf16 = std::is_same<DT, __nv_bfloat16>::value ? 1u : 0u;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->ubar, 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(&ctl->pfull[g], 1);
      mbar_init(&ctl->pempty[g], kRb);
    }
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->drain, 1);
    mbar_init(&ctl->drain_p, 1);
    for (int w = 0; w < kMaxWS; ++w) {
      mbar_init(&ctl->wfull[w], 1);        // armed by this CTA's MMA thread, filled by the producer's copy
      mbar_init(&ctl->wempty[w], CN);      // one commit from every CTA of the cluster
    }
    for (int v = 0; v < kVS; ++v) {
      mbar_init(&ctl->vfull[v], 1);
      mbar_init(&ctl->vempty[v], 1);
    }
    for (int s = 0; s < XS; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&sgfull[s], 1);
      mbar_init(&sgempty[s], kRb);
    }
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) tmem_alloc(&ctl->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // every CTA's barriers are initialised before any CTA of the cluster arrives on them
  if (CN > 1) cluster_sync();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------ x-tile loader -----
    // x tiles for every K-tile (the GEMM's B operand), into a ring of XS stages; lane 0
    // waits for a free stage, the lanes issue the tile's four copies in parallel.
    const uint32_t FULL = 0xffffffffu;
    if (lane == 0) prefetch_tmap(&tm_x);
    bool ok = true;
    int kl = 0;
    for (; kl < KT && ok; ++kl) {
      const int s = kl % XS, use = kl / XS;
      if (lane == 0) {
        if (use > 0) ok = mbar_wait(&xempty[s], static_cast<uint32_t>((use - 1) & 1), deadline, abort_flag);
        if (ok) mbar_arrive_expect_tx(&xfull[s], static_cast<uint32_t>(NT) * kKT * 2u);
      }
      ok = __shfl_sync(FULL, ok, 0);
      if (!ok) break;
      if (lane == 0) tma_load_2d(smem + L.x_off + s * L.x_stride, &tm_x, (kt0 + kl) * kKT, tok0, &xfull[s]);
    }
    if (lane == 0) {
      if (!ok) {
        ctl->abort = 1;
        atomicOr(p.err, kErrTimeout);
      }
      const uint64_t drain_by = globaltimer_ns() + 100000000ull;
      for (int j = (kl > XS ? kl - XS : 0); j < kl; ++j)
        mbar_wait(&xfull[j % XS], static_cast<uint32_t>((j / XS) & 1), drain_by, nullptr);
    }
  } else if (warp == kWarpRbLoad) {
    // ---------------------------------------------------------- rebuild loader -----
    // U tiles once; then, in K order, the sign group of every 8 K-tiles (all of the
    // group's 8 K-tiles share its words; CN divides 8, so every group holds own K-tiles)
    // and the V tiles of the CTA's own K-tiles, each as soon as its ring slot is free.
    const uint32_t FULL = 0xffffffffu;
    if (lane == 0) {
      prefetch_tmap(&tm_u);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&ctl->ubar, static_cast<uint32_t>(n) * 4096u);
    }
    __syncwarp();
    for (int e = lane; e < 2 * n; e += 32)
      tma_load_3d(smem + L.u_off + (e >> 1) * 4096 + (e & 1) * 2048, &tm_u, 8 * (e & 1), rt * kTileRows, e >> 1,
                  &ctl->ubar);
    bool ok = true;
    int oi = 0, groups = 0;
    for (; oi < n_own && ok; ++oi) {
      const int kl = rank + oi * CN, kt = kt0 + kl;
      if (oi == 0 || (kl - CN) / 8 != kl / 8) {   // the first own K-tile of a sign group
        // buffers and phases count the split's groups; the source is the global group
        const int grp = kt / 8, lg = kl / 8, sb = lg % SB, use = lg / SB;
        if (lane == 0) {
          if (use > 0) ok = mbar_wait(&sgempty[sb], static_cast<uint32_t>((use - 1) & 1), deadline, abort_flag);
          if (ok) mbar_arrive_expect_tx(&sgfull[sb], static_cast<uint32_t>(n) * kTileBytes);
        }
        ok = __shfl_sync(FULL, ok, 0);
        if (!ok) break;
        for (int i = lane; i < n; i += 32) {
          const uint8_t* src = p.blocks + static_cast<size_t>(i) * p.block_bytes +
                               (static_cast<size_t>(rt) * p.KG + grp) * kTileBytes;
          bulk_g2s(smem + L.s_off + sb * L.s_stride + i * kTileBytes, src, kTileBytes, &sgfull[sb]);
        }
        ++groups;
      }
      const int vs = oi % kVS, vuse = oi / kVS;
      if (lane == 0) {
        if (vuse > 0) ok = mbar_wait(&ctl->vempty[vs], static_cast<uint32_t>((vuse - 1) & 1), deadline, abort_flag);
        if (ok) mbar_arrive_expect_tx(&ctl->vfull[vs], static_cast<uint32_t>(n) * 1024u);
      }
      ok = __shfl_sync(FULL, ok, 0);
      if (!ok) break;
      uint8_t* vb = smem + L.v_off + vs * L.v_stride;
      for (int e = lane; e < 2 * n; e += 32)
        tma_load_3d(vb + (e >> 1) * 1024 + (e & 1) * 512, &tm_v, 8 * (e & 1), kt * kKT, e >> 1, &ctl->vfull[vs]);
    }
    if (lane == 0) {
      if (!ok) {
        ctl->abort = 1;
        atomicOr(p.err, kErrTimeout);
      }
      // drain the copies issued last on every barrier
      const uint64_t drain_by = globaltimer_ns() + 100000000ull;
      mbar_wait(&ctl->ubar, 0, drain_by, nullptr);
      for (int j = (oi > kVS ? oi - kVS : 0); j < oi; ++j)
        mbar_wait(&ctl->vfull[j % kVS], static_cast<uint32_t>((j / kVS) & 1), drain_by, nullptr);
      for (int g = (groups > SB ? groups - SB : 0); g < groups; ++g)
        mbar_wait(&sgfull[g % SB], static_cast<uint32_t>((g / SB) & 1), drain_by, nullptr);
    }
  } else if (warp == kWarpP) {
    // ------------------------------------------------------- product issuer -----
    // P round pr = (own K-tile oi, round r) into TMEM region pr & 1: rank-16 products of
    // up to kPRound blocks, once the tile's V rows have landed and the rebuild warps have
    // read the region's previous round.  After a tile's last round its V stage is handed
    // back (the commit fires when these MMAs are done).  Runs ahead of the GEMM as far as
    // the V stages and the two regions allow.
    if (lane == 0) {
      const uint32_t idesc_p = make_idesc(1u, 0u, 0u, 128u, 32u);                 // f32 <- f16 x f16
      bool ok = mbar_wait(&ctl->ubar, 0, deadline, abort_flag);
      bool issued_any = false;
      const uint32_t uaddr = smem_u32(smem + L.u_off);
      const int PR = n_own * rounds;
      for (int pr = 0; pr < PR && ok; ++pr) {
        const int oip = pr / rounds, r = pr - oip * rounds, g = pr & 1, vs = oip % kVS;
        if (r == 0) ok = mbar_wait(&ctl->vfull[vs], static_cast<uint32_t>((oip / kVS) & 1), deadline, abort_flag);
        if (ok && pr >= 2)
          ok = mbar_wait(&ctl->pempty[g], static_cast<uint32_t>(((pr >> 1) - 1) & 1), deadline, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t vaddr = smem_u32(smem + L.v_off + vs * L.v_stride);
        const int i1 = min(n, (r + 1) * kPRound);
        for (int i = r * kPRound; i < i1; ++i) {
          const uint64_t adesc = smem_desc_noswizzle(uaddr + i * 4096, 2048, 128);
          const uint64_t bdesc = smem_desc_noswizzle(vaddr + i * 1024, 512, 128);
          mma_f16_ss(tmem + kPcol + 128u * g + (i - r * kPRound) * 32, adesc, bdesc, idesc_p, 0u);
        }
        issued_any = true;
        tc_commit(&ctl->pfull[g]);
        if (r == rounds - 1) tc_commit(&ctl->vempty[vs]);
      }
      if (!ok) {
        ctl->abort = 1;
        atomicOr(p.err, kErrTimeout);
      }
      if (issued_any) {   // no product may still write tensor memory at exit
        tc_commit(&ctl->drain_p);
        mbar_wait(&ctl->drain_p, 0, globaltimer_ns() + 100000000ull, nullptr);
      }
    }
  } else if (warp == kWarpMma) {
    // ----------------------------------------------------------- GEMM issuer -----
    // The GEMM of K-tile kg once its W_hat tile is in this CTA's ring and its x tile has
    // landed; the slot goes back to its producer (rank kg mod CN) when the GEMM is done.
    // Every wait is for an event that depends only on smaller K-tiles.
    if (lane == 0) {
      const uint32_t idesc_g = make_idesc(1u, is_bf16, is_bf16, 128u, static_cast<uint32_t>(NT));
      bool ok = true;
      bool issued_any = false;
      // every W slot expects one tile's bytes for its first use
      for (int w = 0; w < WS && w < KT; ++w) mbar_arrive_expect_tx(&ctl->wfull[w], kWTile);   // split-local
      // ring positions kept as counters (no divisions in the loop): W slot w of use wu,
      // x stage s of use su, producer rank pk = kg mod CN
      const uint64_t adesc0 = smem_desc_noswizzle(smem_u32(smem + L.w_off), 2048, 128);
      const uint64_t bdesc0 = smem_desc_sw64(smem_u32(smem + L.x_off), 8 * 64);
      int w = 0, wu = 0, s = 0, su = 0, pk = 0;
      for (int kg = 0; kg < KT && ok; ++kg) {
        ok = mbar_wait_cluster(&ctl->wfull[w], static_cast<uint32_t>(wu & 1), deadline, abort_flag);
        if (!ok) break;
        if (kg + WS < KT) mbar_arrive_expect_tx(&ctl->wfull[w], kWTile);   // the slot's next use
        ok = mbar_wait(&xfull[s], static_cast<uint32_t>(su & 1), deadline, abort_flag);
        if (!ok) break;
        tc_fence_after();
        // descriptor start addresses count 16-byte units: W slot w at w * kWTile, K-step kk
        // of the W tile 4096 bytes on; x stage s at s * x_stride, K-step kk 32 bytes on
        const uint64_t adesc = adesc0 + static_cast<uint64_t>((w * kWTile) >> 4);
        const uint64_t bdesc = bdesc0 + static_cast<uint64_t>((s * L.x_stride) >> 4);
        mma_f16_ss(tmem, adesc, bdesc, idesc_g, kg > 0 ? 1u : 0u);
        mma_f16_ss(tmem, adesc + (4096 >> 4), bdesc + (32 >> 4), idesc_g, 1u);
        issued_any = true;
        tc_commit(&xempty[s]);
        if (kg + WS < KT) {
          if (CN > 1) tc_commit_multicast(&ctl->wempty[w], static_cast<uint16_t>(1u << pk));
          else tc_commit(&ctl->wempty[w]);
        }
        if (++w == WS) { w = 0; ++wu; }
        if (++s == XS) { s = 0; ++su; }
        if (++pk == CN) pk = 0;
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
    // ---------------------- warps 0-7: rebuild (half a K-tile each), epilogue -------
    const int half = warp >> 2;                          // K-tile columns 16 half .. 16 half + 15
    const int tid = (warp & 3) * 32 + lane;              // row of the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool failed = false;
    auto check = [&](bool ok) {
      if (!__all_sync(0xffffffffu, ok)) failed = true;
    };
    int prounds = 0;
    // the CTA's own K-tiles kl = rank, rank + CN, ... of the split; each is written into
    // ring slot kl mod WS of every CTA of the cluster
    for (int oi = 0; oi < n_own; ++oi) {
      const int kl = rank + oi * CN, kt = kt0 + kl;
      const int lg = kl / 8, t = kl % 8, sb = lg % SB;   // the split's group, K-tile in it
      const int w = kl % WS;
      const bool first_in_group = oi == 0 || (kl - CN) / 8 != lg;
      const bool last_in_group = oi + 1 == n_own || (kl + CN) / 8 != lg;
      if (first_in_group && !failed)
        check(mbar_wait(&sgfull[sb], static_cast<uint32_t>((lg / SB) & 1), deadline, abort_flag));
      // column c of the K-tile is bit 8 (c % 4) + t of word c / 4 of the row; a multiply by
      // 2^(31 - 8 (c % 4) - t) moves it to bit 31 on the FMA pipe, leaving one AND-XOR
      // (the integer pipe) and one add per element and block
      uint32_t mq[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) mq[q] = 1u << (31 - 8 * q - t);
      // 1/s of this thread's 16 columns, loaded before the waits so that their latency
      // hides behind the rounds
      float isv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) isv[c] = __ldg(p.inv_s + kt * kKT + 16 * half + c);
      float acc[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] = 0.0f;
      const uint8_t* sbase = smem + L.s_off + sb * L.s_stride + half * 2048 + tid * 16;
      for (int r = 0; r < rounds; ++r) {
        const int g = prounds & 1;   // P rounds alternate between the two TMEM regions
        if (!failed) check(mbar_wait(&ctl->pfull[g], static_cast<uint32_t>((prounds >> 1) & 1), deadline, abort_flag));
        if (!failed) {
          tc_fence_after();
          // the round's products and sign words all in flight before one wait
          const int nbr = min(kPRound, n - r * kPRound);
          uint32_t v[kPRound][16];
          uint4 wq[kPRound];
#pragma unroll
          for (int ii = 0; ii < kPRound; ++ii) {
            if (ii < nbr) {
              tmem_ld16(tmem + lane_base + kPcol + 128u * g + ii * 32 + 16 * half, v[ii]);
              wq[ii] = *reinterpret_cast<const uint4*>(sbase + (r * kPRound + ii) * kTileBytes);
            }
          }
          tc_wait_ld();
#pragma unroll
          for (int ii = 0; ii < kPRound; ++ii) {
            if (ii < nbr) {
              const uint32_t wd[4] = {wq[ii].x, wq[ii].y, wq[ii].z, wq[ii].w};
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                uint32_t x;
                asm("mul.lo.u32 %0, %1, %2;" : "=r"(x) : "r"(wd[c >> 2]), "r"(mq[c & 3]));
                acc[c] += __uint_as_float(v[ii][c] ^ (x & 0x80000000u));
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&ctl->pempty[g]);
        }
        ++prounds;
      }
      if (!failed && last_in_group) mbar_arrive(&sgempty[sb]);
      uint32_t packed[8];
#pragma unroll
      for (int c = 0; c < 16; c += 2) packed[c / 2] = pack2<DT>(acc[c] * isv[c], acc[c + 1] * isv[c + 1]);
      // the slot is free in every CTA of the cluster once all their GEMMs of the tile
      // WS earlier (also this rank's) are done
      if (kl >= WS && !failed)
        check(mbar_wait_cluster(&ctl->wempty[w], static_cast<uint32_t>(((kl / WS) - 1) & 1), deadline, abort_flag));
      if (!failed) {
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int kc = 2 * half + k2;   // 8-column K chunk of the tile
          *reinterpret_cast<uint4*>(smem + L.w_off + w * kWTile + kc * 2048 + (tid >> 3) * 128 + (tid & 7) * 16) =
              make_uint4(packed[4 * k2], packed[4 * k2 + 1], packed[4 * k2 + 2], packed[4 * k2 + 3]);
        }
        fence_proxy_async_smem();   // read next by the copy engine and the tensor cores
      }
      // all rebuild warps pass here whatever failed (one decision for all of them); then
      // one thread sends the tile from this CTA's slot to the same slot of every other CTA
      // of the cluster, each copy completing the receiver's barrier, and completes its own
      if (bar_any(1, kRb, failed)) {
        failed = true;
      } else if (threadIdx.x < CN) {
        // lane c of warp 0 serves rank c, the copies issued in parallel
        const int c = threadIdx.x;
        const uint8_t* src = smem + L.w_off + w * kWTile;
        if (c == rank) {
          mbar_complete_tx(&ctl->wfull[w], kWTile);
        } else {
          bulk_s2cluster(mapa_shared(smem_u32(src), static_cast<uint32_t>(c)), src, kWTile,
                         mapa_shared(smem_u32(&ctl->wfull[w]), static_cast<uint32_t>(c)));
        }
      }
    }
    // epilogue: accumulator row `tid` holds NT token outputs; the two halves take
    // alternate 32-column chunks.  Without a K split they go to y; with one, to this
    // split's fp32 partial tile (token-major, rows contiguous).  The CTAs that pad the
    // token tiles to whole clusters store nothing.
    if (!failed) check(mbar_wait(&ctl->accfull, 0, deadline, abort_flag));
    const bool real = tok0 < p.M;
    DT* y = static_cast<DT*>(p.y);
    const size_t row = static_cast<size_t>(rt) * kTileRows + tid;
    const size_t tile = static_cast<size_t>(rt) * p.tiles_y + blockIdx.y;
    if (!failed && real) {
      tc_fence_after();
      float* part = p.ks > 1 ? p.part + (tile * p.ks + blockIdx.z) * (kTileRows * NT) : nullptr;
      for (int ch = half; ch < NT / 32; ch += 2) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + ch * 32, v);
        tc_wait_ld();
        if (part != nullptr) {
#pragma unroll
          for (int j = 0; j < 32; ++j) part[(ch * 32 + j) * kTileRows + tid] = __uint_as_float(v[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = tok0 + ch * 32 + j;
            if (tok < p.M) y[static_cast<size_t>(tok) * p.m + row] = cvt_out<DT>(__uint_as_float(v[j]));
          }
        }
      }
      tc_fence_before();
    }
    if (p.ks > 1 && real) {
      // count this partial; the CTA that adds the tile's last one sums all of them in
      // split order (the same association whichever CTA it is) and writes y.  No CTA
      // waits for another.  A CTA that failed counts nothing: its tile is never written
      // and the error word tells the caller (who zeroes the workspace again).  The count
      // is an acquire-release atomic at GPU scope: after the barrier it releases every
      // rebuild thread's partial stores, and for the last arrival it acquires the other
      // CTAs' (the barrier after it orders this CTA's reads behind it).
      if (bar_any(1, kRb, failed)) {
        failed = true;
      } else {
        if (threadIdx.x == 0)
          ctl->last = atom_add_acq_rel_gpu(p.cnt + tile, 1u) == static_cast<uint32_t>(p.ks - 1) ? 1 : 0;
        bar_named(1, kRb);
        if (ctl->last) {
          const float* part = p.part + tile * p.ks * (kTileRows * NT);
          for (int ch = half; ch < NT / 32; ch += 2) {
            for (int j = 0; j < 32; ++j) {
              const int tl = ch * 32 + j;
              if (tok0 + tl >= p.M) break;
              float acc = 0.0f;
              for (int z = 0; z < p.ks; ++z) acc += __ldcg(part + (static_cast<size_t>(z) * NT + tl) * kTileRows + tid);
              y[static_cast<size_t>(tok0 + tl) * p.m + row] = cvt_out<DT>(acc);
            }
          }
          if (threadIdx.x == 0) p.cnt[tile] = 0u;   // left at zero for the next call
        }
      }
    }
    if (failed) {
      ctl->abort = 1;
      atomicOr(p.err, kErrTimeout);
    }
  }

  __syncthreads();
  // no CTA leaves while another CTA of the cluster may still write its ring or arrive on
  // its barriers
  if (CN > 1) cluster_sync();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t prefill_smem_bytes(int n, int NT, int xstages, int sbufs, int cn) {
  return static_cast<size_t>(prefill_layout(n, NT, xstages, sbufs, cn > 1 ? 2 * cn : 2).total) + 64;
}

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_u,
                           const CUtensorMap& tm_v, int bf16, cudaStream_t stream) {
  const size_t smem = prefill_smem_bytes(p.n, p.NT, p.xstages, p.sbufs, p.CN);
  // token tiles padded to a whole number of clusters (the extra CTAs rebuild their share
  // and store nothing)
  const int tiles = (p.M + p.NT - 1) / p.NT;
  const int gy = (tiles + p.CN - 1) / p.CN * p.CN;
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(p.CN);
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = stream;
  cfg.gridDim = dim3(static_cast<unsigned>(p.m / kTileRows), static_cast<unsigned>(gy), static_cast<unsigned>(p.ks));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  if (bf16) return cudaLaunchKernelEx(&cfg, prefill_kernel<__nv_bfloat16>, p, tm_x, tm_u, tm_v);
  return cudaLaunchKernelEx(&cfg, prefill_kernel<__half>, p, tm_x, tm_u, tm_v);
}

}  // namespace bs
