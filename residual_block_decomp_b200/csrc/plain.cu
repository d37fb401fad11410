// "w/o AVD" blocks: the BitStack linear when every residual block is a plain rank-k'
// factor pair U_i V_i^T (vanilla SVD of the residual, no sign matrix), the ablation of
// the review page "BitStack: Fine-Grained Size Control...", Fig. 5 caption, which sets
// k' = k + m n / (16 (m + n)) so that such a block takes the bytes of a BitStack
// block.  The product needs no weight either:
//     y[b, :] = sum_i t_i[b, :] U_i^T,   t_i[b, :] = (x[b, :] (.) 1/s) V_i,
// two thin contractions over the loaded factors, both bound by the bytes of U and V
// (2 k' (m + d) per block), which are read once.  Two launches per group of up to 16
// rows of x:
//   plain_proj   grid (d / 128 row slices of V, loaded blocks): each CTA forms the
//                slice's part of t_i in fp32 and stores it; the CTA that stores the
//                last slice of block i (arrival counter) adds the slices in slice
//                order and writes t_i.  No CTA waits for another.
//   plain_out    grid (m / 32 rows): lane = row, warp = block (and every 8th after
//                it); U_i rows are read once, t_i is warp-uniform; per-warp partial
//                rows are added in warp order.  Launched as a programmatic dependent
//                of plain_proj: its CTAs start as plain_proj's finish and wait on
//                griddepcontrol before they read t.
// All sums have a fixed association, so results do not depend on scheduling.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace bs {
namespace {

constexpr int kSlice = 128;          // rows of V per plain_proj CTA
constexpr int kProjThreads = 256;
constexpr int kOutRows = 32;         // rows of y per plain_out CTA
constexpr int kOutWarps = 8;

__device__ __forceinline__ float load_x(const void* x, int bf16, size_t idx) {
  const uint16_t h = static_cast<const uint16_t*>(x)[idx];
  return bf16 ? __uint_as_float(static_cast<uint32_t>(h) << 16) : __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ void half8(const uint4& w, float (&v)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}

// Dynamic shared memory of plain_proj: x / s of the slice, then the row groups' sums.
__host__ __device__ inline size_t proj_smem(int BT, int kp) {
  const int CH = kp / 8, RG = kProjThreads / CH;
  return static_cast<size_t>(BT) * kSlice * 4 + static_cast<size_t>(RG) * kp * BT * 4;
}

template <int BT>
__global__ void __launch_bounds__(kProjThreads) plain_proj(const PlainParams p) {
  extern __shared__ __align__(16) float psm[];
  __shared__ int last;
  float* xs = psm;                       // [BT][kSlice]
  float* red = psm + BT * kSlice;        // [RG][kp][BT]
  const int sl = blockIdx.x, i = blockIdx.y, tid = threadIdx.x;
  const int kp = p.kp, CH = kp / 8, RG = kProjThreads / CH, nb = p.nb;
  const int c0 = sl * kSlice, rows = min(kSlice, p.d - c0);
  griddep_launch_dependents();
  griddep_wait();   // x may have been written by the kernel ahead
  for (int e = tid; e < BT * kSlice; e += kProjThreads) {
    const int b = e / kSlice, c = e - b * kSlice;
    xs[e] = (b < nb && c < rows)
                ? __fmul_rn(load_x(p.x, p.x_bf16, static_cast<size_t>(p.row0 + b) * p.d + c0 + c), p.inv_s[c0 + c])
                : 0.0f;
  }
  __syncthreads();
  const int ch = tid % CH, rg = tid / CH;
  if (rg < RG) {
    float acc[8][BT];
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int b = 0; b < BT; ++b) acc[e][b] = 0.0f;
    const uint4* vrow = reinterpret_cast<const uint4*>(p.blocks + static_cast<size_t>(i) * p.block_bytes + p.v_off +
                                                       static_cast<size_t>(c0) * kp * 2) + ch;
#pragma unroll 4
    for (int c = rg; c < rows; c += RG) {
      float v[8];
      half8(__ldg(vrow + static_cast<size_t>(c) * CH), v);
#pragma unroll
      for (int b = 0; b < BT; ++b) {
        const float xb = xs[b * kSlice + c];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e][b] = fmaf(v[e], xb, acc[e][b]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int b = 0; b < BT; ++b) red[(static_cast<size_t>(rg) * kp + ch * 8 + e) * BT + b] = acc[e][b];
  }
  __syncthreads();
  // this slice's part of t_i, row groups added in order
  float* part = p.part + (static_cast<size_t>(sl) * p.n + i) * nb * kp;
  for (int e = tid; e < nb * kp; e += kProjThreads) {
    const int b = e / kp, j = e - b * kp;
    float s = 0.0f;
    for (int g = 0; g < RG; ++g) s += red[(static_cast<size_t>(g) * kp + j) * BT + b];
    part[e] = s;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(p.cnt + i, 1u) == static_cast<uint32_t>(gridDim.x - 1) ? 1 : 0;
  __syncthreads();
  if (last) {
    __threadfence();
    float* t = p.t + static_cast<size_t>(i) * nb * kp;
    for (int e = tid; e < nb * kp; e += kProjThreads) {
      float s = 0.0f;
      for (int g = 0; g < static_cast<int>(gridDim.x); ++g)
        s += __ldcg(p.part + (static_cast<size_t>(g) * p.n + i) * nb * kp + e);
      t[e] = s;
    }
    if (tid == 0) p.cnt[i] = 0u;   // the next call starts from zero
  }
}

template <int BT>
__global__ void __launch_bounds__(kOutRows * kOutWarps) plain_out(const PlainParams p) {
  __shared__ float red[kOutWarps][BT][kOutRows];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = blockIdx.x * kOutRows + lane;
  const int kp = p.kp, CH = kp / 8, nb = p.nb;
  const bool row_ok = r < p.m;
  float acc[BT];
#pragma unroll
  for (int b = 0; b < BT; ++b) acc[b] = 0.0f;
  griddep_wait();   // t of every block is complete
  for (int i = w; i < p.n; i += kOutWarps) {
    const uint4* urow = reinterpret_cast<const uint4*>(p.blocks + static_cast<size_t>(i) * p.block_bytes) +
                        static_cast<size_t>(row_ok ? r : 0) * CH;
    const float* t = p.t + static_cast<size_t>(i) * nb * kp;   // warp-uniform reads
#pragma unroll 2
    for (int ch = 0; ch < CH; ++ch) {
      float u[8];
      half8(__ldg(urow + ch), u);
#pragma unroll
      for (int b = 0; b < BT; ++b) {
        if (b < nb) {
          const float4 t0 = __ldg(reinterpret_cast<const float4*>(t + b * kp + ch * 8));
          const float4 t1 = __ldg(reinterpret_cast<const float4*>(t + b * kp + ch * 8 + 4));
          float a = acc[b];
          a = fmaf(u[0], t0.x, a);
          a = fmaf(u[1], t0.y, a);
          a = fmaf(u[2], t0.z, a);
          a = fmaf(u[3], t0.w, a);
          a = fmaf(u[4], t1.x, a);
          a = fmaf(u[5], t1.y, a);
          a = fmaf(u[6], t1.z, a);
          a = fmaf(u[7], t1.w, a);
          acc[b] = a;
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < BT; ++b) red[w][b][lane] = acc[b];
  __syncthreads();
  for (int e = threadIdx.x; e < nb * kOutRows; e += kOutRows * kOutWarps) {
    const int b = e / kOutRows, rr = e - b * kOutRows, row = blockIdx.x * kOutRows + rr;
    if (row >= p.m) continue;
    float s = 0.0f;
#pragma unroll
    for (int g = 0; g < kOutWarps; ++g) s += red[g][b][rr];
    const size_t idx = static_cast<size_t>(p.row0 + b) * p.m + row;
    if (p.x_bf16) static_cast<__nv_bfloat16*>(p.y)[idx] = __float2bfloat16_rn(s);
    else static_cast<__half*>(p.y)[idx] = __float2half_rn(s);
  }
}

// W_hat = (sum_i U_i V_i^T) diag(1/s), one 32 x 32 tile of W per CTA (test path).
template <typename OT>
__global__ void __launch_bounds__(256) plain_reconstruct(const uint8_t* blocks, unsigned long long block_bytes,
                                                         size_t v_off, const float* inv_s, int m, int d, int kp,
                                                         int n, OT* out) {
  __shared__ float us[32][33], vs[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int i = 0; i < n; ++i) {
    const __half* U = reinterpret_cast<const __half*>(blocks + static_cast<size_t>(i) * block_bytes);
    const __half* V = reinterpret_cast<const __half*>(blocks + static_cast<size_t>(i) * block_bytes + v_off);
    for (int j0 = 0; j0 < kp; j0 += 32) {
      for (int e = threadIdx.x; e < 32 * 32; e += 256) {
        const int a = e >> 5, jj = e & 31, j = j0 + jj;
        us[a][jj] = (r0 + a < m && j < kp) ? __half2float(U[static_cast<size_t>(r0 + a) * kp + j]) : 0.0f;
        vs[a][jj] = (c0 + a < d && j < kp) ? __half2float(V[static_cast<size_t>(c0 + a) * kp + j]) : 0.0f;
      }
      __syncthreads();
#pragma unroll 8
      for (int jj = 0; jj < 32; ++jj) {
        const float v = vs[tx][jj];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = fmaf(us[ty + 8 * q][jj], v, acc[q]);
      }
      __syncthreads();
    }
  }
  const int c = c0 + tx;
  if (c >= d) return;
  const float is = inv_s[c];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int r = r0 + ty + 8 * q;
    if (r >= m) continue;
    const float v = acc[q] * is;
    if constexpr (std::is_same<OT, float>::value) out[static_cast<size_t>(r) * d + c] = v;
    else if constexpr (std::is_same<OT, __half>::value) out[static_cast<size_t>(r) * d + c] = __float2half_rn(v);
    else out[static_cast<size_t>(r) * d + c] = __float2bfloat16_rn(v);
  }
}

template <int BT>
cudaError_t launch_bt(const PlainParams& p, cudaStream_t stream) {
  static bool configured[64] = {};   // the attribute is set once per device, outside any capture
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const size_t smem = proj_smem(BT, p.kp);
  if (!configured[dev]) {
    // row groups x rank <= 256 / (k' / 8) x k' <= 2048 for every k': one bound for all
    e = cudaFuncSetAttribute(plain_proj<BT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(static_cast<size_t>(BT) * (kSlice + 2048) * 4));
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
  cfg.gridDim = dim3(static_cast<unsigned>((p.d + kSlice - 1) / kSlice), static_cast<unsigned>(p.n));
  cfg.blockDim = dim3(kProjThreads);
  cfg.dynamicSmemBytes = smem;
  e = cudaLaunchKernelEx(&cfg, plain_proj<BT>, p);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(static_cast<unsigned>((p.m + kOutRows - 1) / kOutRows));
  cfg.blockDim = dim3(kOutRows * kOutWarps);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, plain_out<BT>, p);
}

}  // namespace

PlainWs plain_ws_layout(int d, int kp, int n, int batch) {
  PlainWs w{};
  const size_t nb = static_cast<size_t>(batch < kPlainRowsPerPass ? batch : kPlainRowsPerPass);
  const size_t slices = (static_cast<size_t>(d) + kSlice - 1) / kSlice;
  size_t off = 0;
  w.cnt = off;  off = align_up(off + static_cast<size_t>(n) * sizeof(uint32_t), 256);
  w.t = off;    off = align_up(off + static_cast<size_t>(n) * nb * kp * sizeof(float), 256);
  w.part = off; off = align_up(off + slices * n * nb * kp * sizeof(float), 256);
  w.total = off;
  return w;
}

cudaError_t launch_plain(const PlainParams& p, cudaStream_t stream) {
  if (p.nb <= 1) return launch_bt<1>(p, stream);
  if (p.nb <= 2) return launch_bt<2>(p, stream);
  if (p.nb <= 4) return launch_bt<4>(p, stream);
  if (p.nb <= 8) return launch_bt<8>(p, stream);
  return launch_bt<16>(p, stream);
}

cudaError_t launch_plain_reconstruct(const uint8_t* blocks, unsigned long long block_bytes, size_t v_off,
                                     const float* inv_s, int m, int d, int kp, int n, void* out, int dtype,
                                     cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((d + 31) / 32), static_cast<unsigned>((m + 31) / 32));
  if (dtype == BS_F32)
    plain_reconstruct<float><<<grid, 256, 0, stream>>>(blocks, block_bytes, v_off, inv_s, m, d, kp, n,
                                                       static_cast<float*>(out));
  else if (dtype == BS_F16)
    plain_reconstruct<__half><<<grid, 256, 0, stream>>>(blocks, block_bytes, v_off, inv_s, m, d, kp, n,
                                                        static_cast<__half*>(out));
  else
    plain_reconstruct<__nv_bfloat16><<<grid, 256, 0, stream>>>(blocks, block_bytes, v_off, inv_s, m, d, kp, n,
                                                               static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace bs
