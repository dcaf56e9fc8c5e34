// Internal definitions of libvqlin (device buffer layout of a handle, kernel
// launchers).  Not part of the public ABI (include/vqlin.h).
#pragma once

#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "vqlin.h"

namespace vqlin {

// Everything a kernel needs to decode a layer.  Device pointers; the handle
// owns them.  Rows of `codes` / `codes_o` are re-laid out at a 16-byte stride.
struct Layer {
  int32_t n_out, n_in, d;
  int32_t k1, bits1, k2, bits2, w;      // w = bits1 + bits2 (field width)
  int32_t n_main, n_sub;                // main columns, main sub-vectors per row
  int32_t n_ocols, n_sub_o, ko, bits_o;
  int64_t stride, stride_o;             // bytes, multiples of 16
  const uint8_t* codes;                 // [n_out][stride]
  const uint8_t* codes_o;               // [n_out][stride_o] or null
  const __half* cb1;                    // [k1][d]
  const __half* cb2;                    // [k2][d] or null
  const __half* cbo;                    // [ko][d] or null
  const __half* rs;                     // [n_out] or null (= 1)
  const __half* cs;                     // [n_in]  or null (= 1)
  const int32_t* colmap;                // [n_in]: main column ids (q order) then outlier ids (p order); null if no outliers
  // Codebook groups: main sub-vector position s decodes with codebook s / g_size (cb1 holds
  // n_groups * k1 entries, cb2 n_groups * k2).  A symmetric codebook is expanded at create time
  // into its k1 entries per group, so the kernels index cb1 the same way.
  int32_t n_groups, g_size;
  uint32_t g_magic;                     // ceil(2^32 / g_size): s / g_size = umulhi(s, g_magic) for s < 65536
  int64_t nnz;
  const int32_t* row_ptr;               // [n_out+1] (null if nnz == 0)
  const int32_t* col;                   // [nnz]
  const uint16_t* val;                  // [nnz] fp16 bits (exact replacement values)
  const float* delta;                   // [nnz] v - body, for the fused products
  const uint16_t* col16;                // [nnz] column ids as u16 when n_in <= 65536, else null
  // The CSR entries by 64-column K-block, for the fused prefill GEMM (null unless it applies):
  // entries of row i in K-block kb are kb_start[i*(n_kb+1)+kb] .. kb_start[i*(n_kb+1)+kb+1]-1, and
  // kb_entry[e] = (col_e mod 64) << 16 | val_e.
  const int32_t* kb_start;              // [n_out][n_kb + 1]
  const uint32_t* kb_entry;             // [nnz]
  // VSR blocks (whole main-column sub-vectors, REPLACE): block b of row i is sub-vector
  // vsr_pos[b], b in [vsr_rp[i], vsr_rp[i+1]); vsr_val its fp16 values [nb][d]; vsr_delta the
  // fused-product form v - decoded body [nb][d] (fp32, 0 past the last main column)
  int64_t vsr_nb;
  const int32_t* vsr_rp;
  const int32_t* vsr_pos;
  const uint16_t* vsr_val;
  const float* vsr_delta;
  // Tensor-core decode layout (d = 8, w in {8,12,16,24,32}; null otherwise): rows padded
  // to a multiple of 16; per row and per slab of 64 sub-vectors, for t = 0..3 the 16
  // fields of sub-vectors 64*slab + 4*ps + t (ps = 0..15), packed LSB-first.
  // With codebook groups the fields of this layout hold g * k1 + i1 (and g * k2 + i2 above
  // tc_bits1), widened to tc_w bits, so these kernels index the concatenated codebooks directly;
  // with one group tc_w = w and tc_bits1 = bits1.
  // For d != 8 (no outlier block) the layout works on 8-wide parts: tc_nsub = n_sub * ceil(d/8)
  // parts per row, decoded with the zero-padded codebooks tc_cb1 / tc_cb2 (tc_k1 / tc_k2 entries,
  // entry k part h at k * ceil(d/8) + h), and x' staged through tc_colmap (layout column -> layer
  // column or -1).  At d = 8: tc_nsub = n_sub, tc_cb = cb, tc_colmap = null.
  const uint8_t* tcodes;
  int32_t tc_w, tc_bits1, tc_nsub, tc_k1, tc_k2;
  const __half* tc_cb1;
  const __half* tc_cb2;
  const int32_t* tc_colmap;
  int32_t n_ls;                         // layout slabs per row
  int32_t tcodes_rows;                  // rows allocated in tcodes (n_out rounded up to 16)
  int64_t tstride;                      // bytes per row = n_ls * 8 * tc_w
  // Codebook-stationary layout (large single-stage codebooks, d = 8; null otherwise):
  // block c = p * cs_H + h owns codebook slice p (entries [p*cs_E, (p+1)*cs_E), cs_E < 1024)
  // and row half h (rows [h*cs_rpp, ...)); its entries (row - h*cs_rpp) << cs_local_bits |
  // (index - p*cs_E), cs_ebits wide, cs_epw per 64-bit word in slots of 21 (cs_epw = 3) or 32
  // bits (cs_epw = 2), sorted by position then row.  Every run of one position is padded to
  // whole words with the null entry (row 0, local index cs_E: a zero centroid), so all
  // entries of a word share the position cs_wpos[word]; block c's words are
  // [cs_start[c], cs_start[c+1]) (multiples of 32, padded with null words).  Within each
  // aligned group of 32 words the entries of a run are dealt to the slots so that a slot
  // column's rows spread over the 32 banks.
  const uint64_t* cs_words;
  const int64_t* cs_start;              // [cs_P*cs_H + 1], in words
  const uint16_t* cs_wpos;              // position of every word
  const float* cs_bound;                // [cs_P*cs_H]: (most entries of one row) * max l1(centroid)
  int32_t cs_P, cs_H, cs_E, cs_rpp, cs_local_bits, cs_ebits, cs_epw;
  int64_t cs_max_words;                 // largest block's word count
};

// Last-error plumbing (thread-local detail string).
void set_error(const char* fmt, ...);
// Counts every kernel the library enqueues (exported as vqlin_kernel_launches).
void note_launches(int n);
vqlin_status cuda_status(cudaError_t e, const char* what);

// Kernel launchers (return cudaGetLastError() of the launch).
cudaError_t launch_unpack(const Layer& L, int which, uint32_t* out, cudaStream_t s);
cudaError_t launch_dequant(const Layer& L, __half* W, int64_t ldw, cudaStream_t s);
cudaError_t launch_gemv(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                        void* ws, size_t ws_bytes, cudaStream_t s);
bool tc_supported(const Layer& L);
size_t gemv_workspace_bytes(const Layer& L, int batch);
cudaError_t launch_gemv_tc(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                           void* ws, size_t ws_bytes, cudaStream_t s, bool* handled);
cudaError_t launch_gemv_generic(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                                cudaStream_t s);
cudaError_t launch_convert_to_f16(const void* X, vqlin_dtype xt, int64_t n, __half* out, cudaStream_t s);
int read_and_clear_device_error();
int read_and_clear_cs_error();
size_t gemv_cs_workspace_bytes(const Layer& L, int batch);
cudaError_t launch_gemv_cs(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                           void* ws, size_t ws_bytes, cudaStream_t s, bool* handled);
cudaError_t launch_gemm_f16(const __half* A, const __half* W, int64_t M, int N, int K, void* Y, vqlin_dtype yt,
                            cudaStream_t s);
// Fused prefill: weight tiles dequantised in shared memory and fed to the tensor cores
// (d = 8, one codebook, no outlier block, n_in % 8 == 0).  X is fp16 [M][n_in], 16-byte aligned.
bool gemm_fused_supported(const Layer& L);
cudaError_t launch_gemm_vq(const Layer& L, const __half* X, int64_t M, void* Y, vqlin_dtype yt, cudaStream_t s);

// ---- small device helpers shared by the library's kernels -----------------
__device__ __forceinline__ float load_as_float(const void* p, vqlin_dtype t, int64_t i) {
  if (t == VQLIN_F32) return __ldg(reinterpret_cast<const float*>(p) + i);
  unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
  if (t == VQLIN_F16) return __half2float(__ushort_as_half(h));
  return __bfloat162float(__ushort_as_bfloat16(h));
}

// Same with the dtype fixed at compile time, so loads in a loop can be issued together.
template <int XT>
__device__ __forceinline__ float ldx(const void* p, int64_t i) {
  if constexpr (XT == VQLIN_F32) {
    return __ldg(reinterpret_cast<const float*>(p) + i);
  } else {
    unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    if constexpr (XT == VQLIN_F16) return __half2float(__ushort_as_half(h));
    else return __bfloat162float(__ushort_as_bfloat16(h));
  }
}

template <int V>
struct dtype_tag { static constexpr int value = V; };

// Calls f(dtype_tag<XT>{}) with XT the runtime dtype t (a uniform branch outside the caller's loops).
template <class F>
__device__ __forceinline__ void with_dtype(vqlin_dtype t, F&& f) {
  if (t == VQLIN_F32) f(dtype_tag<VQLIN_F32>{});
  else if (t == VQLIN_F16) f(dtype_tag<VQLIN_F16>{});
  else f(dtype_tag<VQLIN_BF16>{});
}

__device__ __forceinline__ void store_from_float(void* p, vqlin_dtype t, int64_t i, float v) {
  if (t == VQLIN_F32) reinterpret_cast<float*>(p)[i] = v;
  else if (t == VQLIN_F16) reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  else reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

// Field s (width w <= 32) of a packed row whose base is 16-byte aligned and whose
// buffer extends at least 8 bytes past the last field's byte (guaranteed by the
// 16-byte row stride plus an 16-byte tail pad on the buffer).
__device__ __forceinline__ uint32_t read_field(const uint8_t* row, int64_t s, int w) {
  int64_t bit = s * (int64_t)w;
  const uint8_t* p = row + (bit >> 3);
  uintptr_t a = reinterpret_cast<uintptr_t>(p);
  const uint32_t* q = reinterpret_cast<const uint32_t*>(a & ~uintptr_t(3));
  uint64_t lo = __ldg(q), hi = __ldg(q + 1);
  uint64_t v = lo | (hi << 32);
  int sh = int((a & 3) * 8 + (bit & 7));
  v >>= sh;
  return w >= 32 ? (uint32_t)v : (uint32_t)(v & ((1ull << w) - 1ull));
}

// Fused sparse term of one row, sum_e delta_e * x[b][col_e], over the row's CSR entries
// sub, sub + stride, ... (the caller reduces over its `stride` lanes).  Eight entries per
// round with clamped indices, so the eight loads of each kind issue together; x is read with
// its compile-time dtype.
template <int BP>
__device__ __forceinline__ void sparse_row_terms(const Layer& L, const void* x, vqlin_dtype xt, int B, int64_t row,
                                                 int sub, int stride, float* spv) {
  const int e_beg = L.row_ptr[row], e_end = L.row_ptr[row + 1];
  with_dtype(xt, [&](auto tag) {
    constexpr int XT = decltype(tag)::value;
    for (int e0 = e_beg + sub; e0 < e_end; e0 += 8 * stride) {
      float dl[8];
      int jj[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = min(e0 + u * stride, e_end - 1);
        dl[u] = L.delta[e];
        jj[u] = L.col16 ? (int)L.col16[e] : L.col[e];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) if (e0 + u * stride >= e_end) dl[u] = 0.f;
#pragma unroll
      for (int b = 0; b < BP; ++b)
        if (b < B) {
          float xv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) xv[u] = ldx<XT>(x, (int64_t)b * L.n_in + jj[u]);
#pragma unroll
          for (int u = 0; u < 8; ++u) spv[b] = fmaf(dl[u], xv[u], spv[b]);
        }
    }
  });
}

// The same term split in two for a kernel's layer-only prologue: sparse_prefetch reads the
// row's CSR bounds and its first eight entries of this lane (layer data, before the kernel
// waits for the previous grid); sparse_finish gathers x for them and walks the rest.
struct SparsePre {
  int e0, e_end;
  float dl[8];
  int jj[8];
};

__device__ __forceinline__ void sparse_prefetch(const Layer& L, int64_t row, int sub, int stride, SparsePre& p) {
  p.e0 = L.row_ptr[row] + sub;
  p.e_end = L.row_ptr[row + 1];
  const int last = max(p.e_end - 1, 0);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int e = min(p.e0 + u * stride, last);
    p.dl[u] = L.delta[e];
    p.jj[u] = L.col16 ? (int)L.col16[e] : L.col[e];
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) if (p.e0 + u * stride >= p.e_end) { p.dl[u] = 0.f; p.jj[u] = 0; }
}

template <int BP>
__device__ __forceinline__ void sparse_finish(const Layer& L, const void* x, vqlin_dtype xt, int B, const SparsePre& p,
                                              int stride, float* spv) {
  with_dtype(xt, [&](auto tag) {
    constexpr int XT = decltype(tag)::value;
#pragma unroll
    for (int b = 0; b < BP; ++b)
      if (b < B) {
        float xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) xv[u] = ldx<XT>(x, (int64_t)b * L.n_in + p.jj[u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) spv[b] = fmaf(p.dl[u], xv[u], spv[b]);
      }
    for (int e0 = p.e0 + 8 * stride; e0 < p.e_end; e0 += 8 * stride) {
      float dl[8];
      int jj[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = min(e0 + u * stride, p.e_end - 1);
        dl[u] = L.delta[e];
        jj[u] = L.col16 ? (int)L.col16[e] : L.col[e];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) if (e0 + u * stride >= p.e_end) dl[u] = 0.f;
#pragma unroll
      for (int b = 0; b < BP; ++b)
        if (b < B) {
          float xv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) xv[u] = ldx<XT>(x, (int64_t)b * L.n_in + jj[u]);
#pragma unroll
          for (int u = 0; u < 8; ++u) spv[b] = fmaf(dl[u], xv[u], spv[b]);
        }
    }
  });
}

// Codebook group of main sub-vector position s (0 with one codebook).  Layout padding past the
// last position (the tensor-core layout rounds positions up to whole slabs; their x' is 0) is
// clamped to the last group, so every index stays inside the codebooks.
__device__ __forceinline__ int group_of(const Layer& L, int s) {
  if (L.n_groups <= 1) return 0;
  const int g = L.g_size == 1 ? s : (s < 65536 ? (int)__umulhi((uint32_t)s, L.g_magic) : s / L.g_size);
  return g < L.n_groups ? g : L.n_groups - 1;
}

// VSR term of one row, sum over its blocks b (sub, sub + stride, ...) of sum_t delta[b][t] *
// x[batch][main column s*d + t]: the fused form of the block REPLACE (the caller reduces over its
// `stride` lanes).
template <int BP>
__device__ __forceinline__ void vsr_row_terms(const Layer& L, const void* x, vqlin_dtype xt, int B, int64_t row,
                                              int sub, int stride, float* spv) {
  const int b_beg = L.vsr_rp[row], b_end = L.vsr_rp[row + 1];
  const int d = L.d;
  with_dtype(xt, [&](auto tag) {
    constexpr int XT = decltype(tag)::value;
    for (int b = b_beg + sub; b < b_end; b += stride) {
      const int q0 = L.vsr_pos[b] * d;
      const float* dl = L.vsr_delta + (int64_t)b * d;
      if (XT != VQLIN_F32 && d == 8 && !L.colmap && q0 + 8 <= L.n_main && (L.n_in & 7) == 0) {
        const float4 d0 = __ldg(reinterpret_cast<const float4*>(dl)), d1 = __ldg(reinterpret_cast<const float4*>(dl) + 1);
        const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
        for (int bb = 0; bb < BP; ++bb)
          if (bb < B) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(x) +
                                                                (int64_t)bb * L.n_in + q0));
            const unsigned short* hs = reinterpret_cast<const unsigned short*>(&u);
            float a = spv[bb];
#pragma unroll
            for (int t = 0; t < 8; ++t)
              a = fmaf(dv[t], XT == VQLIN_F16 ? __half2float(__ushort_as_half(hs[t])) : __bfloat162float(__ushort_as_bfloat16(hs[t])), a);
            spv[bb] = a;
          }
      } else {
        for (int t = 0; t < d; ++t) {
          const int q = q0 + t;
          if (q >= L.n_main) break;
          const int j = L.colmap ? L.colmap[q] : q;
          const float dv = dl[t];
#pragma unroll
          for (int bb = 0; bb < BP; ++bb)
            if (bb < B) spv[bb] = fmaf(dv, ldx<XT>(x, (int64_t)bb * L.n_in + j), spv[bb]);
        }
      }
    }
  });
}

// Programmatic dependent launch.  Decode kernels are launched so that they may start
// while the previous grid on the stream is still running; everything they do before
// pdl_wait() reads only the layer (immutable after create) and writes only shared memory.
// pdl_wait() returns once the previous grid has completed and its writes are visible;
// pdl_release() then lets the next grid start its own layer-only prologue (that grid
// still waits for this one before it reads anything this one writes).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <class K, class... A>
cudaError_t launch_pdl(K kernel, dim3 grid, int threads, size_t smem, cudaStream_t s, A... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launches(1);
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace vqlin

// The public handle.
struct vqlin_handle {
  vqlin::Layer L;
  int device;
  // info
  vqlin_info info;
  // allocations to free
  void* allocs[32];
  int n_allocs;
};
