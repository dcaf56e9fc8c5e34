// Fused dequantise + GEMV ("QGemv" on the VPTQ page, "The dequantization
// interface": dequantisation fused into the decode matvec so the fp16 weight
// is never written or re-read), with the sparse correction fused into the same
// pass (SCVQ summary step 4; HAS-VQ abstract).
//
//   y[b,i] = r_i * sum_s <C1[i1(i,s)] (+ C2[i2(i,s)]), x'[b, s*d : s*d+d]>
//          + r_i * sum_s' <Co[io(i,s')], x'_o[b, s'*d : s'*d+d]>
//          + sum_{e in row i} delta_e * x[b, col_e],      x' = c (.) x,
//
// where delta_e = v_e - (decoded value at that position) is prepared at create
// time, so the sparse entries replace the decoded weight exactly (up to the
// fp32 products).  All products and sums are fp32.
#include "vqlin_internal.cuh"

namespace vqlin {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One centroid of D fp16 elements (D in {4, 6, 8, 12}) as floats, with the widest vector
// loads the entry alignment allows: D*2 bytes per entry, so 16-byte loads for D = 8, 8-byte
// loads for D = 4 and 12, 4-byte loads for D = 6.
template <int D, bool SMEM>
__device__ __forceinline__ void load_centroid_any(const __half* base, uint32_t idx, float* c) {
  uint32_t w[D / 2];
  if constexpr (D % 8 == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(base + (size_t)idx * D);
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const uint4 u = SMEM ? p[i] : __ldg(p + i);
      w[4 * i] = u.x; w[4 * i + 1] = u.y; w[4 * i + 2] = u.z; w[4 * i + 3] = u.w;
    }
  } else if constexpr (D % 4 == 0) {
    const uint2* p = reinterpret_cast<const uint2*>(base + (size_t)idx * D);
#pragma unroll
    for (int i = 0; i < D / 4; ++i) {
      const uint2 u = SMEM ? p[i] : __ldg(p + i);
      w[2 * i] = u.x; w[2 * i + 1] = u.y;
    }
  } else {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(base + (size_t)idx * D);
#pragma unroll
    for (int i = 0; i < D / 2; ++i) w[i] = SMEM ? p[i] : __ldg(p + i);
  }
#pragma unroll
  for (int k = 0; k < D / 2; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
    c[2 * k] = f.x; c[2 * k + 1] = f.y;
  }
}

template <int D>
__device__ __forceinline__ void load_centroid(const __half* base, uint32_t idx, float* c) {
  load_centroid_any<D, false>(base, idx, c);
}

template <int D>
__device__ __forceinline__ void load_centroid_smem(const __half* base, uint32_t idx, float* c) {
  load_centroid_any<D, true>(base, idx, c);
}

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRPW = 2;                 // rows per warp
constexpr int kRowsPerCta = kWarps * kRPW;

// Generic kernel: any field width <= 32, d in {4, 6, 8, 12}, residual and outlier
// blocks, batch <= NB.  x' is staged through shared memory in column chunks.
template <int D, int NB, bool CB_SMEM>
__global__ void __launch_bounds__(kThreads) k_gemv_generic(Layer L, const void* __restrict__ x, vqlin_dtype xt,
                                                           int batch, void* __restrict__ y, vqlin_dtype yt,
                                                           int chunk) {
  extern __shared__ __align__(16) unsigned char smem[];
  float* xs = reinterpret_cast<float*>(smem);                       // [NB][chunk]
  __half* cb1s = reinterpret_cast<__half*>(xs + NB * chunk);
  __half* cb2s = cb1s + (size_t)L.n_groups * L.k1 * D;
  __half* cbos = cb2s + (size_t)L.n_groups * L.k2 * D;
  const __half* cb1 = L.cb1;
  const __half* cb2 = L.cb2;
  const __half* cbo = L.cbo;
  if (CB_SMEM) {
    const uint4* srcs[3] = {reinterpret_cast<const uint4*>(L.cb1), reinterpret_cast<const uint4*>(L.cb2),
                            reinterpret_cast<const uint4*>(L.cbo)};
    int lens[3] = {L.n_groups * L.k1 * D * 2, L.n_groups * L.k2 * D * 2, L.ko * D * 2};   // whole 4-byte units
    unsigned char* dst = reinterpret_cast<unsigned char*>(cb1s);
    for (int part = 0; part < 3; ++part) {
      // copy in 4-byte units (an entry is 2*d bytes, d even), eight loads in flight per thread
      const uint32_t* s4 = reinterpret_cast<const uint32_t*>(srcs[part]);
      uint32_t* d4 = reinterpret_cast<uint32_t*>(dst);
      const int n4 = lens[part] / 4;
      for (int t0 = threadIdx.x; t0 < n4; t0 += 8 * kThreads) {
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldg(s4 + min(t0 + u * kThreads, n4 - 1));
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (t0 + u * kThreads < n4) d4[t0 + u * kThreads] = v[u];
      }
      dst += lens[part];
    }
    cb1 = cb1s; cb2 = L.cb2 ? cb2s : nullptr; cbo = cbos;
  }
  pdl_wait();      // x and y belong to the previous grid until it completes
  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRowsPerCta + warp * kRPW;
  const uint32_t m1 = (1u << L.bits1) - 1u;
  float acc[kRPW][NB];
#pragma unroll
  for (int r = 0; r < kRPW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;

  auto stage = [&](int col_base, int ncols, bool outlier) {
    __syncthreads();
    for (int t = threadIdx.x; t < NB * chunk; t += kThreads) {
      int b = t / chunk, q = t - b * chunk;
      float v = 0.f;
      if (b < batch && q < ncols) {
        int qq = col_base + q;
        int j = outlier ? L.colmap[L.n_main + qq] : (L.colmap ? L.colmap[qq] : qq);
        v = load_as_float(x, xt, (int64_t)b * L.n_in + j);
        if (L.cs) v *= __half2float(L.cs[j]);
      }
      xs[t] = v;
    }
    __syncthreads();
  };

  for (int q0 = 0; q0 < L.n_main; q0 += chunk) {
    const int qn = min(chunk, L.n_main - q0);
    stage(q0, qn, false);
    const int s0 = q0 / D, s1 = s0 + (qn + D - 1) / D;
#pragma unroll
    for (int r = 0; r < kRPW; ++r) {
      const int row = row0 + r;
      if (row >= L.n_out) break;
      const uint8_t* rowp = L.codes + (int64_t)row * L.stride;
      // four sub-vectors per lane and round: their fields are read (clamped) before any use
      constexpr int UF = 4;
      for (int sb = s0 + lane; sb < s1; sb += 32 * UF) {
        uint32_t fs[UF];
#pragma unroll
        for (int u = 0; u < UF; ++u) fs[u] = read_field(rowp, min(sb + 32 * u, s1 - 1), L.w);
#pragma unroll
        for (int u = 0; u < UF; ++u) {
          const int s = sb + 32 * u;
          if (s >= s1) break;
          const uint32_t f = fs[u];
          const int g = group_of(L, s);
          float c[D];
          const uint32_t e1 = (uint32_t)g * L.k1 + (f & m1);
          if (CB_SMEM) load_centroid_smem<D>(cb1, e1, c); else load_centroid<D>(cb1, e1, c);
          if (cb2) {
            float c2[D];
            const uint32_t e2 = (uint32_t)g * L.k2 + (f >> L.bits1);
            if (CB_SMEM) load_centroid_smem<D>(cb2, e2, c2); else load_centroid<D>(cb2, e2, c2);
#pragma unroll
            for (int k = 0; k < D; ++k) c[k] += c2[k];
          }
          const float* xv = xs + (s - s0) * D;
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            float a = acc[r][b];
#pragma unroll
            for (int k = 0; k < D; ++k) a = fmaf(c[k], xv[b * chunk + k], a);
            acc[r][b] = a;
          }
        }
      }
    }
  }
  if (L.n_ocols > 0) {
    stage(0, L.n_ocols, true);
#pragma unroll
    for (int r = 0; r < kRPW; ++r) {
      const int row = row0 + r;
      if (row >= L.n_out) break;
      const uint8_t* rowp = L.codes_o + (int64_t)row * L.stride_o;
      for (int s = lane; s < L.n_sub_o; s += 32) {
        uint32_t f = read_field(rowp, s, L.bits_o);
        float c[D];
        if (CB_SMEM) load_centroid_smem<D>(cbo, f, c); else load_centroid<D>(cbo, f, c);
        const float* xv = xs + s * D;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float a = acc[r][b];
#pragma unroll
          for (int k = 0; k < D; ++k) a = fmaf(c[k], xv[b * chunk + k], a);
          acc[r][b] = a;
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRPW; ++r) {
    const int row = row0 + r;
    if (row >= L.n_out) break;
    float sp[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) sp[b] = 0.f;
    if (L.nnz > 0) sparse_row_terms<NB>(L, x, xt, batch, row, lane, 32, sp);
    if (L.vsr_nb > 0) vsr_row_terms<NB>(L, x, xt, batch, row, lane, 32, sp);
    const float rsc = L.rs ? __half2float(L.rs[row]) : 1.f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float body = warp_sum(acc[r][b]);
      float spb = warp_sum(sp[b]);
      if (lane == 0 && b < batch) store_from_float(y, yt, (int64_t)b * L.n_out + row, fmaf(rsc, body, spb));
    }
  }
}

template <int D, int NB>
static cudaError_t launch_generic_nb(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y,
                                     vqlin_dtype yt, cudaStream_t s) {
  // x' chunk: at most 48 KB, a multiple of 32*D columns, at least the outlier block
  int chunk = (48 * 1024) / (4 * NB);
  chunk = (chunk / (32 * D)) * (32 * D);
  int need = ((L.n_main + D - 1) / D) * D;
  if (need < chunk) chunk = ((need + 32 * D - 1) / (32 * D)) * (32 * D);
  int need_o = L.n_sub_o * D;
  if (need_o > chunk) chunk = ((need_o + 32 * D - 1) / (32 * D)) * (32 * D);
  size_t xs_bytes = (size_t)NB * chunk * 4;
  size_t cb_bytes = ((size_t)L.n_groups * (L.k1 + L.k2) + L.ko) * D * 2;
  bool cb_smem = xs_bytes + cb_bytes <= 200 * 1024;
  size_t smem = xs_bytes + (cb_smem ? cb_bytes : 0);
  dim3 grid((L.n_out + kRowsPerCta - 1) / kRowsPerCta);
  if (cb_smem) {
    auto k = k_gemv_generic<D, NB, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), kThreads, smem, s, L, x, xt, batch, y, yt, chunk);
  } else {
    auto k = k_gemv_generic<D, NB, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), kThreads, smem, s, L, x, xt, batch, y, yt, chunk);
  }
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_generic(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y,
                                  vqlin_dtype yt, cudaStream_t s) {
  if (batch <= 1) return launch_generic_nb<D, 1>(L, x, xt, batch, y, yt, s);
  if (batch <= 2) return launch_generic_nb<D, 2>(L, x, xt, batch, y, yt, s);
  if (batch <= 4) return launch_generic_nb<D, 4>(L, x, xt, batch, y, yt, s);
  if (batch <= 8) return launch_generic_nb<D, 8>(L, x, xt, batch, y, yt, s);
  return launch_generic_nb<D, 16>(L, x, xt, batch, y, yt, s);
}

cudaError_t launch_gemv_generic(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                                cudaStream_t s) {
  switch (L.d) {
    case 8: return launch_generic<8>(L, x, xt, batch, y, yt, s);
    case 4: return launch_generic<4>(L, x, xt, batch, y, yt, s);
    case 6: return launch_generic<6>(L, x, xt, batch, y, yt, s);
    default: return launch_generic<12>(L, x, xt, batch, y, yt, s);
  }
}

cudaError_t launch_gemv(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                        void* ws, size_t ws_bytes, cudaStream_t s) {
  bool handled = false;
  cudaError_t e = launch_gemv_cs(L, x, xt, batch, y, yt, ws, ws_bytes, s, &handled);
  if (e != cudaSuccess || handled) return e;
  e = launch_gemv_tc(L, x, xt, batch, y, yt, ws, ws_bytes, s, &handled);
  if (e != cudaSuccess || handled) return e;
  return launch_gemv_generic(L, x, xt, batch, y, yt, s);
}

}  // namespace vqlin
