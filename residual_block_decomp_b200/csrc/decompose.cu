// GPU decomposition of a weight into BitStack residual blocks: the offline step that
// produces the records the linear reads.
//
// The method (review page "BitStack: Fine-Grained Size Control...", Figs. 3 and 5;
// OpenReview discussion, reply A3; README "Decomposition"): scale the weight per input
// channel, R_0 = W diag(s), then for every block take the sign of the residual and a
// rank-k SVD of its absolute value, store sign bits and the factors with sqrt(sigma)
// folded into both, and subtract S (.) (U V^T), formed from the stored fp16 factors,
// from the residual.
//
// The rank-k SVD of A = |R| is randomized subspace iteration (Halko, Martinsson and
// Tropp, "Finding structure with randomness", SIAM Review 2011, Algs. 4.4 and 5.1) with
// l = k + 16 columns: a Gaussian sketch (counter-based: SplitMix64 of (seed, block, row,
// column), Box-Muller), q power iterations, each side re-orthonormalised by Cholesky QR
// done twice (the l x l Gram matrix in fp64, factored by one CTA), then the small
// l x l problem B B^T with B = Q^T A solved by cyclic Jacobi rotations in fp64.
// A is never formed: every kernel reads R and takes |R| on the fly.  Tall-skinny
// products run on CUDA cores in fp32 (R is read once per product, the products are
// bound by HBM); only the l x l matrices are fp64.
#include <cuda_fp16.h>

#include <algorithm>

#include "internal.h"

namespace bs {
namespace {

constexpr int kL = 32;           // sketch width: k + 16 (k = 16)
constexpr int kTileR = 64;       // rows of R per CTA in the products
constexpr int kTileK = 32;       // inner tile

// ----------------------------------------------------------------- element-wise ----
__global__ void scale_kernel(const float* W, const float* s, float* R, int m, int d) {
  const size_t total = static_cast<size_t>(m) * d;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * blockDim.x)
    R[e] = W[e] * s[e % d];
}

// sum of squares of R into *out (fp64; *out zeroed by the caller)
__global__ void sumsq_kernel(const float* R, size_t total, double* out) {
  double acc = 0.0;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const double v = R[e];
    acc += v * v;
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ double part[32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += part[w];
    atomicAdd(out, t);
  }
}

// The block's sign words in the device tile order: bit 1 where R < 0 (S = -1).  One
// thread per 32-bit word: word p of row rr of tile (rt, g) holds, in bit 8 q + t, the
// sign of column 32 t + 4 p + q of the tile.
__global__ void pack_signs_kernel(const float* R, int m, int d, uint32_t* words) {
  const size_t nwords = static_cast<size_t>(m) * d / 32;
  const int KG = d / kTileCols;
  for (size_t wi = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; wi < nwords;
       wi += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t tile = wi / 1024;
    const int w = static_cast<int>(wi % 1024);
    const int rt = static_cast<int>(tile / KG), g = static_cast<int>(tile % KG);
    const int h = w / 512, rr = (w % 512) / 4, pp = w % 4;
    const int p = 4 * h + pp;
    const float* row = R + static_cast<size_t>(rt * kTileRows + rr) * d + g * kTileCols;
    uint32_t bits = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (!(row[32 * t + 4 * p + q] >= 0.0f)) bits |= 1u << (8 * q + t);
    words[wi] = bits;
  }
}

// Gaussian sketch X[c][j] (d x l) from a counter-based generator.
__device__ __forceinline__ uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__global__ void sketch_kernel(float* X, int d, uint64_t seed, int block) {
  const size_t total = static_cast<size_t>(d) * kL;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint64_t h = splitmix64(seed ^ splitmix64((static_cast<uint64_t>(block) << 40) ^ e));
    // two uniforms in (0, 1] and [0, 1) from the two halves, then Box-Muller
    const double u1 = (static_cast<double>(h >> 40) + 1.0) * (1.0 / 16777216.0);
    const double u2 = static_cast<double>((h >> 16) & 0xFFFFFFull) * (1.0 / 16777216.0);
    X[e] = static_cast<float>(sqrt(-2.0 * log(u1)) * cospi(2.0 * u2));
  }
}

// ------------------------------------------------------------ tall-skinny products ----
// Y (m x l) = |R| (m x d) X (d x l): a CTA takes 64 rows of R; thread (row group, j)
// keeps 8 outputs.  R is read once, along its rows.
__global__ void __launch_bounds__(256) gemm_a_kernel(const float* R, const float* X, float* Y, int m, int d) {
  __shared__ float As[kTileR][kTileK + 1];
  __shared__ float Xs[kTileK][kL];
  const int r0 = blockIdx.x * kTileR, tid = threadIdx.x;
  const int j = tid & 31, tr = tid >> 5;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  for (int c0 = 0; c0 < d; c0 += kTileK) {
    for (int e = tid; e < kTileR * kTileK; e += 256) {
      const int rr = e / kTileK, cc = e % kTileK;
      As[rr][cc] = fabsf(R[static_cast<size_t>(r0 + rr) * d + c0 + cc]);
    }
    for (int e = tid; e < kTileK * kL; e += 256) Xs[e / kL][e % kL] = X[static_cast<size_t>(c0 + e / kL) * kL + e % kL];
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kTileK; ++kk) {
      const float x = Xs[kk][j];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(As[tr * 8 + e][kk], x, acc[e]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) Y[static_cast<size_t>(r0 + tr * 8 + e) * kL + j] = acc[e];
}

// Z (d x l) = |R|^T (d x m) Y (m x l): a CTA takes 64 columns of R and walks its rows.
__global__ void __launch_bounds__(256) gemm_at_kernel(const float* R, const float* Y, float* Z, int m, int d) {
  __shared__ float As[kTileK][kTileR + 1];
  __shared__ float Ys[kTileK][kL];
  const int c0 = blockIdx.x * kTileR, tid = threadIdx.x;
  const int j = tid & 31, tc = tid >> 5;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  for (int r0 = 0; r0 < m; r0 += kTileK) {
    for (int e = tid; e < kTileK * kTileR; e += 256) {
      const int rr = e / kTileR, cc = e % kTileR;
      As[rr][cc] = fabsf(R[static_cast<size_t>(r0 + rr) * d + c0 + cc]);
    }
    for (int e = tid; e < kTileK * kL; e += 256) Ys[e / kL][e % kL] = Y[static_cast<size_t>(r0 + e / kL) * kL + e % kL];
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kTileK; ++kk) {
      const float y = Ys[kk][j];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(As[kk][tc * 8 + e], y, acc[e]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) Z[static_cast<size_t>(c0 + tc * 8 + e) * kL + j] = acc[e];
}

// G (l x l, fp64, zeroed by the caller) += X^T X over rows of X (N x l).
__global__ void __launch_bounds__(256) gram_kernel(const float* X, int N, double* G) {
  __shared__ float Xs[kTileR][kL];
  const int tid = threadIdx.x, a = tid >> 3, b0 = (tid & 7) * 4;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int r0 = blockIdx.x * kTileR; r0 < N; r0 += gridDim.x * kTileR) {
    const int rows = min(kTileR, N - r0);
    for (int e = tid; e < kTileR * kL; e += 256)
      Xs[e / kL][e % kL] = (e / kL < rows) ? X[static_cast<size_t>(r0 + e / kL) * kL + e % kL] : 0.0f;
    __syncthreads();
    for (int r = 0; r < rows; ++r) {
      const double xa = Xs[r][a];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] += xa * static_cast<double>(Xs[r][b0 + q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) atomicAdd(&G[a * kL + b0 + q], acc[q]);
}

// Xout (N x lo) = Xin (N x l) M (l x lo), M fp64 (row-major, l x ldm), lo <= l.
__global__ void __launch_bounds__(256) apply_kernel(const float* Xin, const double* M, int ldm, int lo, float* Xout,
                                                    int ldo, int N) {
  __shared__ float Ms[kL][kL];
  for (int e = threadIdx.x; e < kL * kL; e += 256)
    Ms[e / kL][e % kL] = (e % kL < lo) ? static_cast<float>(M[(e / kL) * ldm + e % kL]) : 0.0f;
  __syncthreads();
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < static_cast<size_t>(N) * lo;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = e / lo;
    const int j = static_cast<int>(e % lo);
    const float* xr = Xin + r * kL;
    float acc = 0.0f;
#pragma unroll 8
    for (int i = 0; i < kL; ++i) acc = fmaf(xr[i], Ms[i][j], acc);
    Xout[r * ldo + j] = acc;
  }
}

// ------------------------------------------------------------- l x l problems (fp64) ----
// T = L^{-T} for the Cholesky factor L of the Gram matrix G = X^T X (one thread; l = 32),
// so that X T has orthonormal columns.  A pivot below 1e-13 trace(G) (a rank-deficient
// sketch) is raised to that floor, which keeps T finite.
__global__ void chol_inv_kernel(const double* G, double* T) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double L[kL][kL], Li[kL][kL];
  double tr = 0.0;
  for (int i = 0; i < kL; ++i) tr += G[i * kL + i];
  const double floor = 1e-13 * (tr > 0.0 ? tr : 1.0);
  for (int i = 0; i < kL; ++i)
    for (int j = 0; j < kL; ++j) L[i][j] = 0.0;
  for (int j = 0; j < kL; ++j) {
    double dsum = G[j * kL + j];
    for (int p = 0; p < j; ++p) dsum -= L[j][p] * L[j][p];
    const double ljj = sqrt(dsum > floor ? dsum : floor);
    L[j][j] = ljj;
    for (int i = j + 1; i < kL; ++i) {
      double sum = G[i * kL + j];
      for (int p = 0; p < j; ++p) sum -= L[i][p] * L[j][p];
      L[i][j] = sum / ljj;
    }
  }
  // Li = L^{-1} (lower triangular), by forward substitution column by column
  for (int j = 0; j < kL; ++j) {
    for (int i = 0; i < kL; ++i) Li[i][j] = 0.0;
    Li[j][j] = 1.0 / L[j][j];
    for (int i = j + 1; i < kL; ++i) {
      double sum = 0.0;
      for (int p = j; p < i; ++p) sum += L[i][p] * Li[p][j];
      Li[i][j] = -sum / L[i][i];
    }
  }
  for (int i = 0; i < kL; ++i)
    for (int j = 0; j < kL; ++j) T[i * kL + j] = Li[j][i];   // T = Li^T (upper)
}

// Eigen-decomposition of the symmetric G (l x l) by cyclic Jacobi rotations; one warp,
// lane t updating row / column t.  Outputs the eigenvalues in descending order and the
// matching eigenvectors as the columns of Wv (row-major l x l).
__global__ void jacobi_kernel(const double* G, double* evals, double* Wv) {
  __shared__ double A[kL][kL + 1], V[kL][kL + 1];
  __shared__ double cs[2];
  __shared__ int order[kL];
  const int t = threadIdx.x;
  for (int j = 0; j < kL; ++j) {
    A[t][j] = G[t * kL + j];
    V[t][j] = (t == j) ? 1.0 : 0.0;
  }
  __syncwarp();
  for (int sweep = 0; sweep < 30; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int j = 0; j < kL; ++j) {
      const double a = A[t][j] * A[t][j];
      tot += a;
      if (j != t) off += a;
    }
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if (off <= 1e-30 * tot || off == 0.0) break;
    for (int p = 0; p < kL - 1; ++p) {
      for (int q = p + 1; q < kL; ++q) {
        if (t == 0) {
          const double apq = A[p][q];
          double c = 1.0, s = 0.0;
          if (fabs(apq) > 1e-300) {
            // rotation angle that zeroes A[p][q] (Golub and Van Loan, Alg. 8.4.1)
            const double tau = (A[q][q] - A[p][p]) / (2.0 * apq);
            const double tt = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
            c = 1.0 / sqrt(1.0 + tt * tt);
            s = tt * c;
          }
          cs[0] = c;
          cs[1] = s;
        }
        __syncwarp();
        const double c = cs[0], s = cs[1];
        if (s != 0.0) {
          // A <- J^T A J: columns p, q, then rows p, q; V <- V J
          const double atp = A[t][p], atq = A[t][q];
          A[t][p] = c * atp - s * atq;
          A[t][q] = s * atp + c * atq;
          __syncwarp();
          const double apt = A[p][t], aqt = A[q][t];
          A[p][t] = c * apt - s * aqt;
          A[q][t] = s * apt + c * aqt;
          const double vtp = V[t][p], vtq = V[t][q];
          V[t][p] = c * vtp - s * vtq;
          V[t][q] = s * vtp + c * vtq;
        }
        __syncwarp();
      }
    }
  }
  if (t == 0) {
    for (int i = 0; i < kL; ++i) order[i] = i;
    for (int i = 0; i < kL; ++i)
      for (int j = i + 1; j < kL; ++j)
        if (A[order[j]][order[j]] > A[order[i]][order[i]]) {
          const int tmp = order[i];
          order[i] = order[j];
          order[j] = tmp;
        }
  }
  __syncwarp();
  evals[t] = A[order[t]][order[t]];
  for (int j = 0; j < kL; ++j) Wv[t * kL + j] = V[t][order[j]];
}

// M (l x k): column j of the eigenvectors divided by sigma_j = sqrt(lambda_j), so that
// Z M = B^T W Sigma^{-1} = the right singular vectors of B.
__global__ void vscale_kernel(const double* Wv, const double* evals, int k, double* M, double* sigma) {
  const int t = threadIdx.x;   // row of Wv
  for (int j = 0; j < k; ++j) {
    const double lam = evals[j] > 0.0 ? evals[j] : 0.0;
    const double sg = sqrt(lam);
    if (t == 0) sigma[j] = sg;
    M[t * k + j] = sg > 0.0 ? Wv[t * kL + j] / sg : 0.0;
  }
}

// Column sums of U (N x k, stride ldu) into cs (fp64, zeroed by the caller).
__global__ void colsum_kernel(const float* U, int ldu, int N, int k, double* cs) {
  double acc = 0.0;
  const int j = threadIdx.x % k;
  for (size_t r = blockIdx.x * static_cast<size_t>(blockDim.x / k) + threadIdx.x / k; r < static_cast<size_t>(N);
       r += static_cast<size_t>(gridDim.x) * (blockDim.x / k))
    acc += U[r * ldu + j];
  atomicAdd(&cs[j], acc);
}

// fp16 factors into the record: F[r][j] = fp16(X[r][j] * flip_j * sqrt(sigma_j)), where
// flip_j makes the column sum of U non-negative.
__global__ void write_factor_kernel(const float* X, int N, int k, const double* sigma, const double* cs,
                                    __half* out) {
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < static_cast<size_t>(N) * k;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(e % k);
    const double f = (cs[j] < 0.0 ? -1.0 : 1.0) * sqrt(sigma[j]);
    out[e] = __float2half_rn(static_cast<float>(static_cast<double>(X[e]) * f));
  }
}

// R <- S (.) (|R| - U V^T) with U, V the stored fp16 factors (m x 16, d x 16): the
// residual of what the block holds.  A CTA takes 32 rows x 128 columns.
__global__ void __launch_bounds__(256) residual_kernel(float* R, const __half* U, const __half* V, int m, int d) {
  __shared__ float us[32][kK + 1], vs[128][kK + 1];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 128;
  for (int e = threadIdx.x; e < 32 * kK; e += 256)
    us[e / kK][e % kK] = __half2float(U[static_cast<size_t>(r0 + e / kK) * kK + e % kK]);
  for (int e = threadIdx.x; e < 128 * kK; e += 256)
    vs[e / kK][e % kK] = __half2float(V[static_cast<size_t>(c0 + e / kK) * kK + e % kK]);
  __syncthreads();
  const int cl = threadIdx.x & 127;
  for (int rl = threadIdx.x >> 7; rl < 32; rl += 2) {
    float p = 0.0f;
#pragma unroll
    for (int j = 0; j < kK; ++j) p = fmaf(us[rl][j], vs[cl][j], p);
    float* x = R + static_cast<size_t>(r0 + rl) * d + c0 + cl;
    const float v = *x;
    *x = (v >= 0.0f) ? (v - p) : (v + p);   // S (|R| - P) with S = +1 where R >= 0
  }
}

}  // namespace

DecomposeWs decompose_ws_layout(int m, int d) {
  DecomposeWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  w.R = take(static_cast<size_t>(m) * d * 4);
  w.Y = take(static_cast<size_t>(m) * kL * 4);
  w.Y2 = take(static_cast<size_t>(m) * kL * 4);
  w.Z = take(static_cast<size_t>(d) * kL * 4);
  w.Z2 = take(static_cast<size_t>(d) * kL * 4);
  w.Uf = take(static_cast<size_t>(m) * kK * 4);
  w.Vf = take(static_cast<size_t>(d) * kK * 4);
  w.small = take((3 * kL * kL + kL + kL * kK + 2 * kK) * 8);
  w.total = off;
  return w;
}

cudaError_t run_decompose(const DecomposeArgs& a, cudaStream_t st) {
  const int m = a.m, d = a.d, k = kK;
  const DecomposeWs L = decompose_ws_layout(m, d);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  float* R = reinterpret_cast<float*>(ws + L.R);
  float* Y = reinterpret_cast<float*>(ws + L.Y);
  float* Y2 = reinterpret_cast<float*>(ws + L.Y2);
  float* Z = reinterpret_cast<float*>(ws + L.Z);
  float* Z2 = reinterpret_cast<float*>(ws + L.Z2);
  float* Uf = reinterpret_cast<float*>(ws + L.Uf);
  float* Vf = reinterpret_cast<float*>(ws + L.Vf);
  double* G = reinterpret_cast<double*>(ws + L.small);
  double* T = G + kL * kL;
  double* Wv = T + kL * kL;
  double* evals = Wv + kL * kL;
  double* M = evals + kL;
  double* sigma = M + kL * kK;
  double* cs = sigma + kK;
  const size_t md = static_cast<size_t>(m) * d;
  const int ew_grid = static_cast<int>(std::min<size_t>((md + 255) / 256, 148 * 16));
  cudaError_t e = cudaSuccess;
  auto ck = [&]() {
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess;
  };
  auto gram = [&](const float* X, int N) {
    e = cudaMemsetAsync(G, 0, kL * kL * 8, st);
    if (e != cudaSuccess) return;
    gram_kernel<<<std::min(N / kTileR > 0 ? N / kTileR : 1, 148 * 4), 256, 0, st>>>(X, N, G);
  };
  auto apply = [&](const float* X, const double* Mat, int ldm, int lo, float* out, int ldo, int N) {
    const size_t tot = static_cast<size_t>(N) * lo;
    apply_kernel<<<static_cast<int>(std::min<size_t>((tot + 255) / 256, 148 * 16)), 256, 0, st>>>(X, Mat, ldm, lo, out,
                                                                                                    ldo, N);
  };
  // X (N x l) <- an orthonormal basis of its columns: Cholesky QR twice
  auto orth = [&](float* X, float* tmp, int N) {
    gram(X, N);
    chol_inv_kernel<<<1, 1, 0, st>>>(G, T);
    apply(X, T, kL, kL, tmp, kL, N);
    gram(tmp, N);
    chol_inv_kernel<<<1, 1, 0, st>>>(G, T);
    apply(tmp, T, kL, kL, X, kL, N);
  };

  scale_kernel<<<ew_grid, 256, 0, st>>>(a.W, a.s, R, m, d);
  if (!ck()) return e;
  if ((e = cudaMemsetAsync(a.res_norms, 0, (a.n + 1) * sizeof(double), st)) != cudaSuccess) return e;
  sumsq_kernel<<<ew_grid, 256, 0, st>>>(R, md, a.res_norms);
  if (!ck()) return e;
  for (int i = 0; i < a.n; ++i) {
    uint8_t* rec = a.records + static_cast<size_t>(i) * a.block_bytes;
    __half* Urec = reinterpret_cast<__half*>(rec + md / 8);
    __half* Vrec = Urec + static_cast<size_t>(m) * k;
    const size_t nwords = md / 32;
    pack_signs_kernel<<<static_cast<int>(std::min<size_t>((nwords + 255) / 256, 148 * 16)), 256, 0, st>>>(
        R, m, d, reinterpret_cast<uint32_t*>(rec));
    sketch_kernel<<<static_cast<int>((static_cast<size_t>(d) * kL + 255) / 256), 256, 0, st>>>(Z, d, a.seed, i);
    gemm_a_kernel<<<m / kTileR, 256, 0, st>>>(R, Z, Y, m, d);
    for (int q = 0; q < a.power_iters; ++q) {
      orth(Y, Y2, m);
      gemm_at_kernel<<<d / kTileR, 256, 0, st>>>(R, Y, Z, m, d);
      orth(Z, Z2, d);
      gemm_a_kernel<<<m / kTileR, 256, 0, st>>>(R, Z, Y, m, d);
    }
    orth(Y, Y2, m);                                              // Q
    gemm_at_kernel<<<d / kTileR, 256, 0, st>>>(R, Y, Z, m, d);   // B^T = A^T Q
    gram(Z, d);                                                  // B B^T
    jacobi_kernel<<<1, 32, 0, st>>>(G, evals, Wv);
    apply(Y, Wv, kL, k, Uf, k, m);                               // U = Q W_k
    vscale_kernel<<<1, 32, 0, st>>>(Wv, evals, k, M, sigma);
    apply(Z, M, k, k, Vf, k, d);                                 // V = B^T W_k Sigma_k^{-1}
    if ((e = cudaMemsetAsync(cs, 0, kK * 8, st)) != cudaSuccess) return e;
    colsum_kernel<<<std::max(1, std::min(m / 16, 148 * 4)), 256, 0, st>>>(Uf, k, m, k, cs);
    write_factor_kernel<<<static_cast<int>(std::min<size_t>((static_cast<size_t>(m) * k + 255) / 256, 4096)), 256, 0,
                          st>>>(Uf, m, k, sigma, cs, Urec);
    write_factor_kernel<<<static_cast<int>(std::min<size_t>((static_cast<size_t>(d) * k + 255) / 256, 4096)), 256, 0,
                          st>>>(Vf, d, k, sigma, cs, Vrec);
    residual_kernel<<<dim3(d / 128, m / 32), 256, 0, st>>>(R, Urec, Vrec, m, d);
    sumsq_kernel<<<ew_grid, 256, 0, st>>>(R, md, a.res_norms + i + 1);
    if (!ck()) return e;
  }
  return e;
}

}  // namespace bs
