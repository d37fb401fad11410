// Auxiliary kernels: dense reconstruction of W_hat and sign unpacking.
//
// Reconstruction follows the weight restoration snippet of the OpenReview discussion
// of "BitStack: Any-Size Compression of Large Language Models in Variable Memory
// Environments": starting from zero, every loaded block adds unpack(sign) (.) (U V^T);
// the activation-aware scale is then undone per input channel (review page "BitStack:
// Fine-Grained Size Control...", Fig. 5).  These kernels run on CUDA cores; they are
// the library's dense-weight export and its test paths, not the hot path.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace bs {
namespace {

// Word index and bit of sign (r, c) in the device tile order.
__device__ __forceinline__ void sign_pos(int r, int c, int d, size_t* word, int* bit) {
  const int rt = r >> 7, rr = r & 127;
  const int g = c >> 8, cl = c & 255;
  const int t = cl >> 5, rem = cl & 31;
  const int pw = rem >> 2, q = rem & 3;
  const size_t tile = static_cast<size_t>(rt) * (d >> 8) + g;
  *word = tile * 1024 + (pw >> 2) * 512 + rr * 4 + (pw & 3);
  *bit = 8 * q + t;
}

constexpr int kRcRows = 32, kRcCols = 64;

__global__ void __launch_bounds__(256) reconstruct_kernel(const uint8_t* blocks, unsigned long long bb,
                                                          const float* inv_s, int m, int d, int n, void* out,
                                                          int dtype) {
  __shared__ float us[kRcRows][kK + 1];
  __shared__ float vs[kRcCols][kK + 1];
  const int c = blockIdx.x * kRcCols + (threadIdx.x & 63);
  const int r0 = blockIdx.y * kRcRows + (threadIdx.x >> 6) * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  for (int i = 0; i < n; ++i) {
    const uint8_t* rec = blocks + static_cast<size_t>(i) * bb;
    const __half* U = reinterpret_cast<const __half*>(rec + static_cast<size_t>(m) * d / 8);
    const __half* V = U + static_cast<size_t>(m) * kK;
    const uint32_t* words = reinterpret_cast<const uint32_t*>(rec);
    __syncthreads();
    for (int e = threadIdx.x; e < kRcRows * kK; e += 256)
      us[e / kK][e % kK] = __half2float(U[static_cast<size_t>(blockIdx.y * kRcRows + e / kK) * kK + e % kK]);
    for (int e = threadIdx.x; e < kRcCols * kK; e += 256)
      vs[e / kK][e % kK] = __half2float(V[static_cast<size_t>(blockIdx.x * kRcCols + e / kK) * kK + e % kK]);
    __syncthreads();
    const int cl = threadIdx.x & 63;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int rl = (threadIdx.x >> 6) * 8 + e;
      float dot = 0.0f;
#pragma unroll
      for (int j = 0; j < kK; ++j) dot = fmaf(us[rl][j], vs[cl][j], dot);
      size_t wi;
      int bit;
      sign_pos(r0 + e, c, d, &wi, &bit);
      const bool neg = (words[wi] >> bit) & 1u;
      acc[e] += neg ? -dot : dot;
    }
  }
  const float is = inv_s[c];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const size_t idx = static_cast<size_t>(r0 + e) * d + c;
    const float v = acc[e] * is;
    if (dtype == BS_F32) static_cast<float*>(out)[idx] = v;
    else if (dtype == BS_F16) static_cast<__half*>(out)[idx] = __float2half_rn(v);
    else static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  }
}

__global__ void unpack_kernel(const uint32_t* words, int m, int d, int8_t* out) {
  const size_t total = static_cast<size_t>(m) * d;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(e / d), c = static_cast<int>(e % d);
    size_t wi;
    int bit;
    sign_pos(r, c, d, &wi, &bit);
    out[e] = ((words[wi] >> bit) & 1u) ? int8_t(-1) : int8_t(1);
  }
}

}  // namespace

cudaError_t launch_reconstruct(const uint8_t* blocks, unsigned long long block_bytes, const float* inv_s, int m,
                               int d, int n, void* out, int dtype, cudaStream_t stream) {
  dim3 grid(d / kRcCols, m / kRcRows);
  reconstruct_kernel<<<grid, 256, 0, stream>>>(blocks, block_bytes, inv_s, m, d, n, out, dtype);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const uint8_t* record, int m, int d, int8_t* out, cudaStream_t stream) {
  const size_t total = static_cast<size_t>(m) * d;
  const int blocks = static_cast<int>((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  unpack_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const uint32_t*>(record), m, d, out);
  return cudaGetLastError();
}

}  // namespace bs
