// Nearest-centroid assignment: the encoding step before the decode path (VPTQ page, "Step 3:
// Vector quantization of column n": Q_V(v) = argmin_i ||v - C_i||^2, plain Euclidean distance;
// "Residual Vector Quantization": i1 = Q_1(v), then i2 = argmin_j ||(v - C[i1]) - Cres_j||^2).
//
// One thread per sub-vector holds v in registers; the block stages the codebook tile by tile
// in shared memory as fp32, so every centroid read is a broadcast.  The decision is taken in
// binary32: each difference is one rounded subtraction and the running sum one fused
// multiply-add per element (acc = fma(diff, diff, acc)), elements in order 0..d-1, centroids
// from index 0 up, and a centroid replaces the best one only when strictly closer, so ties
// keep the lowest index.  The residual is the binary32 difference v - C1[i1].  The work is
// d subtractions, d fused multiply-adds and one comparison per (sub-vector, centroid):
// CUDA-core ALU bound.  Each computed distance lies within (d + 3) 2^-24 of the exact one
// (relative), so the index returned is a nearest centroid up to that rounding: exactly the
// argmin wherever the exact minimum is unique beyond it.
#include "vqlin_internal.cuh"

namespace vqlin {

namespace asg {

constexpr int THREADS = 256;
constexpr int TILE_BYTES = 64 * 1024;

template <int D>
__device__ __forceinline__ void scan_codebook(const __half* __restrict__ C, int k, float* tile, const float* v,
                                              bool active, uint32_t& best_i) {
  constexpr int TK = TILE_BYTES / (4 * D);
  float best_d = 0.f;
  best_i = 0;
  for (int base = 0; base < k; base += TK) {
    const int nt = min(TK, k - base);
    __syncthreads();                                       // the previous tile is no longer read
    for (int e = threadIdx.x; e < nt * D; e += THREADS) tile[e] = __half2float(C[(size_t)base * D + e]);
    __syncthreads();
    if (active) {
      for (int i = 0; i < nt; ++i) {
        const float* c = tile + i * D;
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < D; ++t) {
          const float diff = __fsub_rn(v[t], c[t]);
          acc = __fmaf_rn(diff, diff, acc);
        }
        if ((base == 0 && i == 0) || acc < best_d) { best_d = acc; best_i = (uint32_t)(base + i); }
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(THREADS) k_assign(const __half* __restrict__ V, int64_t n, const __half* __restrict__ C1,
                                                    int k1, const __half* __restrict__ C2, int k2,
                                                    uint32_t* __restrict__ idx1, uint32_t* __restrict__ idx2) {
  extern __shared__ __align__(16) float tile[];
  const int64_t s = (int64_t)blockIdx.x * THREADS + threadIdx.x;
  const bool active = s < n;
  float v[D];
#pragma unroll
  for (int t = 0; t < D; ++t) v[t] = active ? __half2float(V[s * D + t]) : 0.f;
  uint32_t i1;
  scan_codebook<D>(C1, k1, tile, v, active, i1);
  if (active) idx1[s] = i1;
  if (k2 > 0) {
#pragma unroll
    for (int t = 0; t < D; ++t) v[t] = __fsub_rn(v[t], __half2float(C1[(size_t)i1 * D + t]));
    uint32_t i2;
    scan_codebook<D>(C2, k2, tile, v, active, i2);
    if (active) idx2[s] = i2;
  }
}

template <int D>
static cudaError_t launch(const __half* V, int64_t n, const __half* C1, int k1, const __half* C2, int k2,
                          uint32_t* i1, uint32_t* i2, cudaStream_t s) {
  const int64_t blocks = (n + THREADS - 1) / THREADS;
  cudaError_t e = cudaFuncSetAttribute(k_assign<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, TILE_BYTES);
  if (e != cudaSuccess) return e;
  note_launches(1);
  k_assign<D><<<(unsigned)blocks, THREADS, TILE_BYTES, s>>>(V, n, C1, k1, C2, k2, i1, i2);
  return cudaGetLastError();
}

}  // namespace asg

}  // namespace vqlin

using namespace vqlin;

extern "C" vqlin_status vqlin_assign(const uint16_t* V, int64_t n, int32_t d, const uint16_t* C1, int32_t k1,
                                     const uint16_t* C2, int32_t k2, uint32_t* idx1, uint32_t* idx2, void* stream) {
  if (n < 0 || k1 < 1 || k2 < 0) { set_error("bad size (n >= 0, k1 >= 1, k2 >= 0)"); return VQLIN_ERR_INVALID_ARG; }
  if (d != 4 && d != 6 && d != 8 && d != 12) { set_error("d = %d: must be 4, 6, 8 or 12", d); return VQLIN_ERR_UNSUPPORTED; }
  if (n == 0) return VQLIN_OK;
  if (!V || !C1 || !idx1 || (k2 > 0 && (!C2 || !idx2))) { set_error("NULL argument"); return VQLIN_ERR_INVALID_ARG; }
  if ((n + asg::THREADS - 1) / asg::THREADS > 0x7fffffff) { set_error("n too large"); return VQLIN_ERR_UNSUPPORTED; }
  const __half* v = reinterpret_cast<const __half*>(V);
  const __half* c1 = reinterpret_cast<const __half*>(C1);
  const __half* c2 = reinterpret_cast<const __half*>(C2);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  switch (d) {
    case 4: e = asg::launch<4>(v, n, c1, k1, c2, k2, idx1, idx2, s); break;
    case 6: e = asg::launch<6>(v, n, c1, k1, c2, k2, idx1, idx2, s); break;
    case 8: e = asg::launch<8>(v, n, c1, k1, c2, k2, idx1, idx2, s); break;
    default: e = asg::launch<12>(v, n, c1, k1, c2, k2, idx1, idx2, s); break;
  }
  return cuda_status(e, "assign launch");
}
