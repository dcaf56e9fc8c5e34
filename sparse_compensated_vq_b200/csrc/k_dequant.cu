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
      const size_t g = (size_t)group_of(L, s);        // codebook group of position s
      const __half* e1 = L.cb1 + (g * L.k1 + (f & m1)) * D;
      const __half* e2 = L.cb2 ? L.cb2 + (g * L.k2 + (f >> L.bits1)) * D : nullptr;
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
      // vector stores of the D outputs: 16-byte units for D = 8, 8-byte for D = 4 and 12,
      // 4-byte for D = 6, when the destination is aligned to that unit
      constexpr int VB = D % 8 == 0 ? 16 : (D % 4 == 0 ? 8 : 4);
      if (!L.colmap && q0 + D <= L.n_main && (((reinterpret_cast<uintptr_t>(Wrow + q0)) & (VB - 1)) == 0)) {
        uint32_t pk[D / 2];
#pragma unroll
        for (int k = 0; k < D / 2; ++k) pk[k] = outv[2 * k] | (uint32_t(outv[2 * k + 1]) << 16);
        if constexpr (VB == 16) {
#pragma unroll
          for (int i = 0; i < D / 8; ++i)
            reinterpret_cast<uint4*>(Wrow + q0)[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        } else if constexpr (VB == 8) {
#pragma unroll
          for (int i = 0; i < D / 4; ++i) reinterpret_cast<uint2*>(Wrow + q0)[i] = make_uint2(pk[2 * i], pk[2 * i + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < D / 2; ++i) reinterpret_cast<uint32_t*>(Wrow + q0)[i] = pk[i];
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

// VSR blocks REPLACE whole sub-vectors bit for bit.  One warp per row, lanes over its blocks.
__global__ void k_dequant_vsr(Layer L, __half* __restrict__ W, int64_t ldw) {
  const int warps = (blockDim.x >> 5) * gridDim.x;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < L.n_out; i += warps) {
    for (int b = L.vsr_rp[i] + (threadIdx.x & 31); b < L.vsr_rp[i + 1]; b += 32) {
      const int q0 = L.vsr_pos[b] * L.d;
      for (int t = 0; t < L.d && q0 + t < L.n_main; ++t) {
        const int j = L.colmap ? L.colmap[q0 + t] : q0 + t;
        W[(int64_t)i * ldw + j] = __ushort_as_half(L.vsr_val[(int64_t)b * L.d + t]);
      }
    }
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

// bf16 -> fp16, eight elements per thread with 16-byte loads and stores (n % 8 == 0, both
// buffers 16-byte aligned).
__global__ void k_convert_bf16_f16_x8(const uint4* __restrict__ X, int64_t n8, uint4* __restrict__ out) {
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n8; t += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(X + t);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);   // bf16 -> fp32 exact
      o[k] = (uint32_t)__half_as_ushort(__float2half_rn(lo)) | ((uint32_t)__half_as_ushort(__float2half_rn(hi)) << 16);
    }
    out[t] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Exact dequantisation on the codebook-stationary layout (single-stage codebook, no outlier
// block, W rows 16-byte aligned).  Block (p, h) holds codebook slice p as 8 interleaved
// copies, the column scales as fp32 and the row scales of half h; every entry (row, position,
// index) of its bucket becomes one 16-byte store of eight fp16 weights.
//
// Exactness in fp32: a centroid element C and the row scale r are fp16, so C*r has at most
// 22 significant bits and is exact in fp32.  The product with the column scale is taken
// rounded toward zero with its exact error from an FMA, and the last bit is forced to 1 when
// inexact (round-to-odd, Boldo & Melquiond, IEEE TC 2008); a 24-bit round-to-odd value
// rounds to the 11-bit fp16 exactly as the real value would.  Null entries are skipped.
__device__ __forceinline__ float round_to_odd_mul_f32(float a, float b) {
  float p = __fmul_rz(a, b);
  const float err = fmaf(a, b, -p);
  if (err != 0.f) p = __int_as_float(__float_as_int(p) | 1);
  return p;
}

template <int EPW>
__global__ void __launch_bounds__(512, 1) k_dequant_cs(Layer L, __half* __restrict__ W, int64_t ldw) {
  constexpr int THREADS = 512, COPIES = 8;
  constexpr int SLOT = EPW == 3 ? 21 : 32;
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = L.cs_H, E = L.cs_E, RPP = L.cs_rpp;
  const int c = blockIdx.x;
  const int p = c / H, h = c - p * H;
  const int row0 = h * RPP;
  const int nrows = min(RPP, L.n_out - row0);
  const int slice0 = p * E, E_p = max(0, min(E, L.n_groups * L.k1 - slice0));   // virtual codebook of all groups
  uint4* cbs = reinterpret_cast<uint4*>(smem);                                        // [E + 1][8]
  float* cf = reinterpret_cast<float*>(smem + (size_t)(E + 1) * COPIES * 16);         // [n_sub * 8]
  float* rf = cf + (size_t)L.n_sub * 8;                                               // [RPP]
  const int rot = threadIdx.x & (COPIES - 1);
  for (int k = threadIdx.x; k < E_p; k += THREADS) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(L.cb1) + slice0 + k);
#pragma unroll
    for (int cc = 0; cc < COPIES; ++cc) cbs[k * COPIES + ((cc + rot) & (COPIES - 1))] = v;
  }
  for (int j = threadIdx.x; j < L.n_sub * 8; j += THREADS) cf[j] = (L.cs && j < L.n_main) ? __half2float(L.cs[j]) : 1.f;
  for (int r = threadIdx.x; r < nrows; r += THREADS) rf[r] = L.rs ? __half2float(L.rs[row0 + r]) : 1.f;
  __syncthreads();
  const uint32_t lmask = (1u << L.cs_local_bits) - 1u;
  const uint64_t emask = (1ull << L.cs_ebits) - 1ull;
  const int lbits = L.cs_local_bits;
  const int64_t w_begin = L.cs_start[c];
  const int n_words = (int)(L.cs_start[c + 1] - w_begin);
  const bool has_cs = L.cs != nullptr;
  for (int wi = threadIdx.x; wi < n_words; wi += THREADS) {
    const uint64_t wv = __ldg(reinterpret_cast<const unsigned long long*>(L.cs_words) + w_begin + wi);
    const int s = __ldg(L.cs_wpos + w_begin + wi);
    const float4 c0 = *reinterpret_cast<const float4*>(cf + s * 8), c1 = *reinterpret_cast<const float4*>(cf + s * 8 + 4);
    const float cc8[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int u = 0; u < EPW; ++u) {
      const uint32_t ent = (uint32_t)((wv >> (u * SLOT)) & emask);
      const uint32_t k = ent & lmask;
      if (k == (uint32_t)E) continue;                        // null entry
      const int row_l = (int)(ent >> lbits);
      const uint4 cen = cbs[k * COPIES + (threadIdx.x & (COPIES - 1))];
      const __half* ch = reinterpret_cast<const __half*>(&cen);
      const float r = rf[row_l];
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float a = __half2float(ch[2 * q + e]) * r;   // exact
          v2[e] = has_cs ? round_to_odd_mul_f32(a, cc8[2 * q + e]) : a;
        }
        o[q] = (uint32_t)__half_as_ushort(__float2half_rn(v2[0])) | ((uint32_t)__half_as_ushort(__float2half_rn(v2[1])) << 16);
      }
      *reinterpret_cast<uint4*>(W + (int64_t)(row0 + row_l) * ldw + (int64_t)s * 8) = make_uint4(o[0], o[1], o[2], o[3]);
    }
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
  const bool cs_ok = L.cs_words && !L.colmap && L.k2 == 0 && (ldw & 7) == 0 && (L.n_main & 7) == 0 &&
                     (reinterpret_cast<uintptr_t>(W) & 15) == 0;
  const size_t cs_smem = (size_t)(L.cs_E + 1) * 8 * 16 + (size_t)L.n_sub * 8 * 4 + (size_t)L.cs_rpp * 4;
  if (cs_ok && cs_smem <= 227 * 1024) {
    cudaError_t e;
    if (L.cs_epw == 3) {
      e = cudaFuncSetAttribute(k_dequant_cs<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cs_smem);
      if (e != cudaSuccess) return e;
      note_launches(1);
      k_dequant_cs<3><<<L.cs_P * L.cs_H, 512, cs_smem, s>>>(L, W, ldw);
    } else {
      e = cudaFuncSetAttribute(k_dequant_cs<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cs_smem);
      if (e != cudaSuccess) return e;
      note_launches(1);
      k_dequant_cs<2><<<L.cs_P * L.cs_H, 512, cs_smem, s>>>(L, W, ldw);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    work = 0;                                   // the main block is done (no outlier block here)
  }
  if (work > 0) {
    note_launches(1);
    switch (L.d) {
      case 8: k_dequant_body<8><<<grid_for(work, 256), 256, 0, s>>>(L, W, ldw); break;
      case 4: k_dequant_body<4><<<grid_for(work, 256), 256, 0, s>>>(L, W, ldw); break;
      case 6: k_dequant_body<6><<<grid_for(work, 256), 256, 0, s>>>(L, W, ldw); break;
      default: k_dequant_body<12><<<grid_for(work, 256), 256, 0, s>>>(L, W, ldw); break;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (L.nnz > 0) {
    note_launches(1);
    k_dequant_sparse<<<grid_for((int64_t)L.n_out * 32, 256), 256, 0, s>>>(L, W, ldw);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (L.vsr_nb > 0) {
    note_launches(1);
    k_dequant_vsr<<<grid_for((int64_t)L.n_out * 32, 256), 256, 0, s>>>(L, W, ldw);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_convert_to_f16(const void* X, vqlin_dtype xt, int64_t n, __half* out, cudaStream_t s) {
  if (xt == VQLIN_BF16 && (n & 7) == 0 && (reinterpret_cast<uintptr_t>(X) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(out) & 15) == 0) {
    note_launches(1);
    k_convert_bf16_f16_x8<<<grid_for(n / 8, 256), 256, 0, s>>>(reinterpret_cast<const uint4*>(X), n / 8,
                                                              reinterpret_cast<uint4*>(out));
    return cudaGetLastError();
  }
  note_launches(1);
  k_convert_f16<<<grid_for(n, 256), 256, 0, s>>>(reinterpret_cast<const unsigned short*>(X), xt, n, out);
  return cudaGetLastError();
}

}  // namespace vqlin
