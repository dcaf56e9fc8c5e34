// Field unpacking and exact dequantisation to fp16.
//
// VPTQ: Extreme Low-bit Vector Post-Training Quantization for Large Language
// Models, "The dequantization interface": W = C[indices] (single stage) and
// C[indices1] + Cres[indices2] (residual); "Outlier Elimination": the outlier
// columns decode through their own codebook.  SCVQ: Sparse-Compensated Vector
// Quantization for Large Language Models, summary step 1: row and column
// scales.  HAS-VQ abstract: sparse positions reconstruct exactly.
//
// Exactness.  C1 + C2 of two fp16 values spans at most 41 significant bits,
// so it is exact in double, and so is its product with an 11-bit row scale
// (<= 52 bits).  Only the product with the column scale can be inexact; it is
// computed rounded toward zero with its exact error from an FMA, and the last
// bit is forced to 1 when inexact (round-to-odd, Boldo & Melquiond, "Emulation
// of FMA and correctly rounded sums: proved algorithms using rounding to odd",
// IEEE TC 2008).  A 53-bit round-to-odd value rounds to the 11-bit fp16 exactly
// as the real value would, so one RNE conversion gives the correctly rounded
// result.
#include "vqlin_internal.cuh"

namespace vqlin {

__device__ __forceinline__ double round_to_odd_mul(double a, double b) {
  double p = __dmul_rz(a, b);
  double err = fma(a, b, -p);
  if (err != 0.0) p = __longlong_as_double(__double_as_longlong(p) | 1ll);
  return p;
}

// fp16 bits of r*c*S, S = C1 (+ C2) already summed exactly in double.
__device__ __forceinline__ unsigned short exact_f16(double S, const __half* rs, const __half* cs, int i, int j) {
  if (rs) S = S * (double)__half2float(rs[i]);           // exact
  if (cs) S = round_to_odd_mul(S, (double)__half2float(cs[j]));
  return __half_as_ushort(__double2half(S));
}

__global__ void k_unpack(const uint8_t* __restrict__ codes, int64_t stride, int n_rows, int n_fields, int w,
                         uint32_t* __restrict__ out) {
  int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t total = (int64_t)n_rows * n_fields;
  for (; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    int64_t i = t / n_fields, s = t - i * n_fields;
    out[t] = read_field(codes + i * stride, s, w);
  }
}

// One thread per (row, sub-vector), main block then outlier block.
template <int D>
__global__ void __launch_bounds__(256) k_dequant_body(Layer L, __half* __restrict__ W, int64_t ldw) {
  const int n_sub_all = L.n_sub + L.n_sub_o;
  int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)L.n_out * n_sub_all;
  const uint32_t m1 = (1u << L.bits1) - 1u;
  for (; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(t / n_sub_all);
    const int s = (int)(t - (int64_t)i * n_sub_all);
    __half* Wrow = W + (int64_t)i * ldw;
    if (s < L.n_sub) {
      uint32_t f = read_field(L.codes + (int64_t)i * L.stride, s, L.w);
      const __half* e1 = L.cb1 + (size_t)(f & m1) * D;
      const __half* e2 = L.cb2 ? L.cb2 + (size_t)(f >> L.bits1) * D : nullptr;
      int q0 = s * D;
      unsigned short outv[D];
#pragma unroll
      for (int k = 0; k < D; ++k) {
        int q = q0 + k;
        int j = q < L.n_main ? (L.colmap ? L.colmap[q] : q) : 0;
        double S = (double)__half2float(e1[k]);
        if (e2) S = S + (double)__half2float(e2[k]);
        outv[k] = exact_f16(S, L.rs, L.cs, i, j);
      }
      if (!L.colmap && q0 + D <= L.n_main && (((reinterpret_cast<uintptr_t>(Wrow + q0)) & (2 * D - 1)) == 0)) {
        if (D == 8) {
          uint4 v = make_uint4(outv[0] | (uint32_t(outv[1]) << 16), outv[2] | (uint32_t(outv[3]) << 16),
                               outv[4] | (uint32_t(outv[5]) << 16), outv[6] | (uint32_t(outv[7]) << 16));
          *reinterpret_cast<uint4*>(Wrow + q0) = v;
        } else {
          uint2 v = make_uint2(outv[0] | (uint32_t(outv[1]) << 16), outv[2] | (uint32_t(outv[3]) << 16));
          *reinterpret_cast<uint2*>(Wrow + q0) = v;
        }
      } else {
#pragma unroll
        for (int k = 0; k < D; ++k) {
          int q = q0 + k;
          if (q < L.n_main) Wrow[L.colmap ? L.colmap[q] : q] = __ushort_as_half(outv[k]);
        }
      }
    } else {
      const int so = s - L.n_sub;
      uint32_t f = read_field(L.codes_o + (int64_t)i * L.stride_o, so, L.bits_o);
      const __half* e = L.cbo + (size_t)f * D;
#pragma unroll
      for (int k = 0; k < D; ++k) {
        int p = so * D + k;
        if (p < L.n_ocols) {
          int j = L.colmap[L.n_main + p];
          Wrow[j] = __ushort_as_half(exact_f16((double)__half2float(e[k]), L.rs, L.cs, i, j));
        }
      }
    }
  }
}

// REPLACE: sparse positions take the stored value bit for bit.  One warp per row.
__global__ void k_dequant_sparse(Layer L, __half* __restrict__ W, int64_t ldw) {
  const int warps = (blockDim.x >> 5) * gridDim.x;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < L.n_out; i += warps) {
    for (int e = L.row_ptr[i] + (threadIdx.x & 31); e < L.row_ptr[i + 1]; e += 32)
      W[(int64_t)i * ldw + L.col[e]] = __ushort_as_half(L.val[e]);
  }
}

__global__ void k_convert_f16(const unsigned short* __restrict__ X, vqlin_dtype xt, int64_t n,
                              __half* __restrict__ out) {
  int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    float v = xt == VQLIN_BF16 ? __bfloat162float(__ushort_as_bfloat16(X[t])) : __half2float(__ushort_as_half(X[t]));
    out[t] = __float2half_rn(v);
  }
}

static int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  if (g > 148 * 32) g = 148 * 32;
  return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_unpack(const Layer& L, int which, uint32_t* out, cudaStream_t s) {
  int n_fields = which ? L.n_sub_o : L.n_sub;
  if (n_fields == 0) return cudaSuccess;
  note_launches(1);
  k_unpack<<<grid_for((int64_t)L.n_out * n_fields, 256), 256, 0, s>>>(
      which ? L.codes_o : L.codes, which ? L.stride_o : L.stride, L.n_out, n_fields, which ? L.bits_o : L.w, out);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const Layer& L, __half* W, int64_t ldw, cudaStream_t s) {
  int64_t work = (int64_t)L.n_out * (L.n_sub + L.n_sub_o);
  if (work > 0) {
    note_launches(1);
    if (L.d == 8) k_dequant_body<8><<<grid_for(work, 256), 256, 0, s>>>(L, W, ldw);
    else k_dequant_body<4><<<grid_for(work, 256), 256, 0, s>>>(L, W, ldw);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (L.nnz > 0) {
    note_launches(1);
    k_dequant_sparse<<<grid_for((int64_t)L.n_out * 32, 256), 256, 0, s>>>(L, W, ldw);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_convert_to_f16(const void* X, vqlin_dtype xt, int64_t n, __half* out, cudaStream_t s) {
  note_launches(1);
  k_convert_f16<<<grid_for(n, 256), 256, 0, s>>>(reinterpret_cast<const unsigned short*>(X), xt, n, out);
  return cudaGetLastError();
}

}  // namespace vqlin
