// Prefill GEMM: Y[M][N] = A[M][K] * W[N][K]^T, fp16 operands, fp32 accumulate.
// (VPTQ page, "The dequantization interface": dequantisation feeds the prefill
// GEMM.)  The weight operand is the exact fp16 dequantised weight.
#include "vqlin_internal.cuh"

namespace vqlin {

// Straightforward shared-memory tiled kernel: 64x64 output tile, 256 threads,
// 4x4 outputs per thread.
__global__ void __launch_bounds__(256) k_gemm_simt(const __half* __restrict__ A, const __half* __restrict__ W,
                                                   int64_t M, int N, int K, void* __restrict__ Y,
                                                   vqlin_dtype yt) {
  __shared__ float As[16][64 + 1];
  __shared__ float Ws[16][64 + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = (int64_t)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int t = threadIdx.x; t < 16 * 64; t += 256) {
      int r = t / 16, kk = t % 16;
      int64_t m = m0 + r;
      int n = n0 + r;
      As[kk][r] = (m < M && k0 + kk < K) ? __half2float(A[m * K + k0 + kk]) : 0.f;
      Ws[kk][r] = (n < N && k0 + kk < K) ? __half2float(W[(int64_t)n * K + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Ws[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int64_t m = m0 + ty * 4 + i;
      int n = n0 + tx * 4 + j;
      if (m < M && n < N) store_from_float(Y, yt, m * N + n, acc[i][j]);
    }
}

cudaError_t launch_gemm_f16(const __half* A, const __half* W, int64_t M, int N, int K, void* Y, vqlin_dtype yt,
                            cudaStream_t s) {
  dim3 grid((N + 63) / 64, (unsigned)((M + 63) / 64));
  k_gemm_simt<<<grid, 256, 0, s>>>(A, W, M, N, K, Y, yt);
  return cudaGetLastError();
}

}  // namespace vqlin
