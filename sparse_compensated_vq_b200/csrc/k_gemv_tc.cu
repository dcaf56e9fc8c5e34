// Tensor-core decode GEMV (d = 8): the fused dequant + GEMV of the VPTQ page
// ("The dequantization interface", QGemv) with the gathered centroids as the
// A operand of mma.sync m16n8k16 and the activations as the B operand.
//
//   A[16 rows][16 k]  = fp16 centroids of 16 weight rows (one per sub-vector);
//                       the scales are not applied to A, so A is exact;
//   B[16 k][8 n]      = x' = c (.) x split into fp16 hi + lo parts (columns of
//                       B are (batch, part) pairs), so hi*A + lo*A keeps the
//                       fp32 product to ~2^-22 relative;
//   D[16 rows][8 n]   fp32 accumulators; y = r * (D_hi + D_lo) + sparse term.
//
// A residual codebook (VPTQ "Residual Vector Quantization": C1[i1] + C2[i2])
// issues a second MMA with the C2 centroids as A (no fp16 rounding of the sum).
//
// Index layout.  At create time the packed fields are re-laid out per row so
// that the lane that needs them can fetch them with one vector load: for each
// "layout slab" of 64 sub-vectors and each t in 0..3, the 16 fields of the
// sub-vectors 64*slab + 4*ps + t (ps = 0..15) are stored consecutively
// (LSB-first, same width w).  Thread (g, t) of a warp then owns sub-vector t of
// every group of four, which is exactly the k-range (2t, 2t+1, 2t+8, 2t+9) the
// m16n8k16 fragments give it once the eight elements of a centroid are mapped
// to k = {2t, 2t+1} (elements 0,1 / 4,5) and {2t+8, 2t+9} (elements 2,3 / 6,7).
//
// Work.  A CTA task is (RTT row tiles of 16 rows) x (a chunk of kernel slabs);
// each warp owns one (row tile, kernel slab) pair per chunk, keeps that slab's
// B fragments in registers, and accumulates its D fragment.  Warps of a task
// are reduced through shared memory and the epilogue adds the fused sparse
// correction (delta_e * x_j) and the outlier-column block on CUDA cores.  With
// more columns than one task covers, either the CTA loops over the chunks
// (no scratch), or tasks are split by chunk and accumulate in fp32 with
// atomics (caller workspace, or y itself when y is fp32).
#include "vqlin_internal.cuh"

namespace vqlin {

namespace tcg {

constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;

__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Load the fields one kernel slab needs from a (row, layout slab, t) block:
// 16/NT fields of W bits = 2W/NT bytes, with the widest naturally aligned vector.
template <int W, int NT>
__device__ __forceinline__ void load_sub(const uint8_t* p, uint32_t* w) {
  constexpr int BYTES = 2 * W / NT;
  constexpr int VW = (BYTES % 16 == 0) ? 16 : (BYTES % 8 == 0) ? 8 : (BYTES % 4 == 0) ? 4 : 2;
  if constexpr (VW == 16) {
#pragma unroll
    for (int i = 0; i < BYTES / 16; ++i) {
      uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (VW == 8) {
#pragma unroll
    for (int i = 0; i < BYTES / 8; ++i) {
      uint2 v = __ldg(reinterpret_cast<const uint2*>(p) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else if constexpr (VW == 4) {
#pragma unroll
    for (int i = 0; i < BYTES / 4; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(p) + i);
  } else {
#pragma unroll
    for (int i = 0; i < BYTES / 2; ++i) {
      uint32_t h = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
      if (i & 1) w[i >> 1] |= h << 16; else w[i >> 1] = h;
    }
  }
}

template <int W>
__device__ __forceinline__ uint32_t field_of(const uint32_t* w, int k) {
  const int bit = k * W;
  if constexpr (W == 8 || W == 16 || W == 32) {
    return W == 32 ? w[k] : (w[bit >> 5] >> (bit & 31)) & ((1u << W) - 1u);
  } else {
    const int lo = bit >> 5, sh = bit & 31;
    uint32_t v = (sh + W <= 32) ? (w[lo] >> sh) : __funnelshift_r(w[lo], w[lo + 1], sh);
    return v & ((1u << W) - 1u);
  }
}

struct Args {
  Layer L;
  const void* x;
  vqlin_dtype xt;
  int batch;
  void* y;
  vqlin_dtype yt;
  float* acc;         // split mode: fp32 [batch][n_out] accumulator (may alias y when yt == F32)
  int split;          // 0: a task covers every chunk; 1: tasks are (row group, chunk)
  int n_kslabs;       // kernel slabs over the main columns
  int ks;             // kernel slabs per chunk handled together (<= WARPS)
  int rtt;            // row tiles per task (WARPS / ks)
  int n_chunks;       // ceil(n_kslabs / ks)
  int xs_cols;        // columns of x' held in shared memory (chunk columns, or all)
  int xs_all;         // 1: x' for all main columns staged once per CTA
  // warp-task kernel: the main columns split into wt_nch chunks of wt_cs kernel slabs; block b
  // serves chunk b / wt_bpc (staging its x' once) and a task is one row tile over wt_spt slabs
  int wt_cs, wt_nch, wt_bpc, wt_spt;
};

template <int NT, int W, bool CB_SMEM, int COPIES>
__global__ void __launch_bounds__(THREADS, 1) k_gemv_tc(Args a) {
  constexpr int PS = 16 / NT;            // pair-steps (4 sub-vectors each) per kernel slab
  constexpr int KSV = 4 * PS;            // sub-vectors per kernel slab
  constexpr int BP = 4 * NT;             // batch slots
  constexpr int ACC = NT == 1 ? 4 : 2;   // independent MMA accumulator sets
  const Layer& L = a.L;
  extern __shared__ __align__(16) unsigned char smem[];
  // ---- shared memory carve-up
  unsigned char* sp = smem;
  uint4* cb1s = reinterpret_cast<uint4*>(sp);
  uint4* cb2s = cb1s + (CB_SMEM ? (size_t)L.tc_k1 * COPIES : 0);
  sp = reinterpret_cast<unsigned char*>(cb2s + (CB_SMEM ? (size_t)L.tc_k2 * COPIES : 0));
  __half* xh = reinterpret_cast<__half*>(sp);                      // [batch][xs_cols]
  __half* xl = xh + (size_t)a.batch * a.xs_cols;
  float* red = reinterpret_cast<float*>(xl + (size_t)a.batch * a.xs_cols);   // [rtt][16][8*NT]
  float* xo = red + (size_t)a.rtt * 16 * 8 * NT;                        // outlier x' [BP][n_sub_o*8]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int B = a.batch;
  const uint32_t m1 = (1u << L.tc_bits1) - 1u;   // first-stage bits of the tensor-core layout

  // ---- codebooks into shared memory (COPIES interleaved copies: entry k of copy c at k*COPIES + c)
  if (CB_SMEM) {
    const uint4* c1 = reinterpret_cast<const uint4*>(L.tc_cb1);
    for (int i = threadIdx.x; i < L.tc_k1 * COPIES; i += THREADS) cb1s[i] = __ldg(c1 + i / COPIES);
    if (L.k2) {
      const uint4* c2 = reinterpret_cast<const uint4*>(L.tc_cb2);
      for (int i = threadIdx.x; i < L.tc_k2 * COPIES; i += THREADS) cb2s[i] = __ldg(c2 + i / COPIES);
    }
  }
  // ---- layer-only prefetch for this block's first task, before the wait: the index words of
  //      each warp's first (row tile, kernel slab) and the CSR bounds and first entries of each
  //      thread's epilogue row
  const int n_rt = (L.n_out + 15) / 16;
  const int n_rg = (n_rt + a.rtt - 1) / a.rtt;
  const int n_tasks = a.split ? n_rg * a.n_chunks : n_rg;
  const int my_rt_local = warp / a.ks;            // which of the task's row tiles this warp serves
  const int my_ks = warp - my_rt_local * a.ks;    // which kernel slab of the chunk
  const bool warp_active = my_rt_local < a.rtt;
  const int rows = a.rtt * 16;
  const int lanes_per_row = THREADS / rows;       // rows * lanes_per_row == THREADS
  const int rl = threadIdx.x / lanes_per_row, sub = threadIdx.x - rl * lanes_per_row;
  constexpr int NWORDS = (2 * W / NT + 3) / 4 + 1;
  const int task0 = blockIdx.x;
  uint32_t pw0[NWORDS], pw1[NWORDS];
  pw0[NWORDS - 1] = pw1[NWORDS - 1] = 0;
  SparsePre spre;
  bool spre_ok = false;
  float rsc0 = 1.f;                               // row scale of the first task's epilogue row
  if (task0 < n_tasks) {
    const int rg0 = a.split ? task0 % n_rg : task0;
    const int ch00 = a.split ? task0 / n_rg : 0;
    const int rt0 = rg0 * a.rtt + my_rt_local, kslab0 = ch00 * a.ks + my_ks;
    if (warp_active && rt0 < n_rt && kslab0 < a.n_kslabs) {
      const int ls = kslab0 / NT, ps0 = (kslab0 - ls * NT) * PS;
      const uint8_t* blk0 = L.tcodes + ((int64_t)rt0 * 16 + g) * L.tstride + (int64_t)ls * (8 * W) + t * (2 * W) + ps0 * W / 8;
      load_sub<W, NT>(blk0, pw0);
      load_sub<W, NT>(blk0 + 8 * L.tstride, pw1);
    }
    const int64_t row0 = (int64_t)rg0 * rows + rl;
    if (L.rs && row0 < L.n_out) rsc0 = __half2float(L.rs[row0]);
    if (ch00 == 0 && row0 < L.n_out && L.nnz > 0) {
      sparse_prefetch(L, row0, sub, lanes_per_row, spre);
      spre_ok = true;
    }
  }
  // x (and the accumulator) belong to the previous grid until it completes
  pdl_wait();
  pdl_release();
  float spv0[BP];
#pragma unroll
  for (int b = 0; b < BP; ++b) spv0[b] = 0.f;
  if (spre_ok) sparse_finish<BP>(L, a.x, a.xt, B, spre, lanes_per_row, spv0);
  // ---- outlier-block x' (fp32), once per CTA
  const int n_o = L.n_sub_o * 8;
  for (int i = threadIdx.x; i < BP * n_o; i += THREADS) {
    int b = i / n_o, p = i - b * n_o;
    float v = 0.f;
    if (b < B && p < L.n_ocols) {
      int j = L.colmap[L.n_main + p];
      v = load_as_float(a.x, a.xt, (int64_t)b * L.n_in + j);
      if (L.cs) v *= __half2float(L.cs[j]);
    }
    xo[i] = v;
  }

  // x' = c (.) x for main columns [col0, col0 + ncols) of every batch row, split
  // into fp16 hi + lo; eight consecutive columns per thread, all loads first.
  auto stage_x = [&](int col0, int ncols) {
    const int groups = ncols / 8;
    for (int i = threadIdx.x; i < B * groups; i += THREADS) {
      const int b = i / groups, q = (i - b * groups) * 8;
      const int qq = col0 + q;
      float v[8];
      if (!L.colmap && !L.tc_colmap && a.xt != VQLIN_F32 && qq + 8 <= L.n_main && (L.n_in & 7) == 0) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(a.x) +
                                                        (int64_t)b * L.n_in + qq));
        const unsigned short* hs = reinterpret_cast<const unsigned short*>(&u);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          v[k] = a.xt == VQLIN_F16 ? __half2float(__ushort_as_half(hs[k])) : __bfloat162float(__ushort_as_bfloat16(hs[k]));
        if (L.cs) {
          uint4 cu = __ldg(reinterpret_cast<const uint4*>(L.cs + qq));
          const __half* cv = reinterpret_cast<const __half*>(&cu);
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] *= __half2float(cv[k]);
        }
      } else {
        int jj[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int c = qq + k;
          jj[k] = L.tc_colmap ? (c < L.tc_nsub * 8 ? L.tc_colmap[c] : -1) : (c < L.n_main ? (L.colmap ? L.colmap[c] : c) : -1);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = jj[k] >= 0 ? load_as_float(a.x, a.xt, (int64_t)b * L.n_in + jj[k]) : 0.f;
        if (L.cs) {
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] *= jj[k] >= 0 ? __half2float(L.cs[jj[k]]) : 0.f;
        }
      }
      uint32_t ph[4], pl[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __half h0 = __float2half_rn(v[2 * k]), h1 = __float2half_rn(v[2 * k + 1]);
        __half l0 = __float2half_rn(v[2 * k] - __half2float(h0)), l1 = __float2half_rn(v[2 * k + 1] - __half2float(h1));
        ph[k] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
        pl[k] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
      }
      *reinterpret_cast<uint4*>(xh + (size_t)b * a.xs_cols + q) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(xl + (size_t)b * a.xs_cols + q) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    }
  };

  const int chunk_cols = a.ks * KSV * 8;
  int staged = -1;
  if (a.xs_all) {
    stage_x(0, a.xs_cols);
    staged = 0;
  }
  __syncthreads();

  for (int task = blockIdx.x; task < n_tasks; task += gridDim.x) {
    const int rg = a.split ? task % n_rg : task;
    const int ch0 = a.split ? task / n_rg : 0;
    const int ch1 = a.split ? ch0 + 1 : a.n_chunks;
    for (int i = threadIdx.x; i < a.rtt * 16 * 8 * NT; i += THREADS) red[i] = 0.f;
    // sparse correction (prefetched for the first task) and outlier block of this thread's row
    const bool first_chunk = ch0 == 0;
    const int64_t row = (int64_t)rg * rows + rl;
    const bool row_ok = row < L.n_out;
    float spv[BP], ov[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b) { spv[b] = task == task0 ? spv0[b] : 0.f; ov[b] = 0.f; }
    if (first_chunk && row_ok) {
      if (L.nnz > 0 && task != task0) sparse_row_terms<BP>(L, a.x, a.xt, B, row, sub, lanes_per_row, spv);
      if (L.vsr_nb > 0) vsr_row_terms<BP>(L, a.x, a.xt, B, row, sub, lanes_per_row, spv);
      for (int s = sub; s < L.n_sub_o; s += lanes_per_row) {
        uint32_t f = read_field(L.codes_o + row * L.stride_o, s, L.bits_o);
        uint4 u = __ldg(reinterpret_cast<const uint4*>(L.cbo) + f);
        const __half2* h = reinterpret_cast<const __half2*>(&u);
        float c[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) { float2 f2 = __half22float2(h[k]); c[2 * k] = f2.x; c[2 * k + 1] = f2.y; }
#pragma unroll
        for (int b = 0; b < BP; ++b)
          if (b < B) {
            float acc = ov[b];
#pragma unroll
            for (int k = 0; k < 8; ++k) acc = fmaf(c[k], xo[b * n_o + s * 8 + k], acc);
            ov[b] = acc;
          }
      }
    }
    // ACC independent accumulator sets, so consecutive MMAs do not wait on each other
    float dacc[ACC][NT][4];
#pragma unroll
    for (int q = 0; q < ACC; ++q)
#pragma unroll
      for (int n = 0; n < NT; ++n) dacc[q][n][0] = dacc[q][n][1] = dacc[q][n][2] = dacc[q][n][3] = 0.f;
    const int rt = rg * a.rtt + my_rt_local;
    for (int ch = ch0; ch < ch1; ++ch) {
      if (!a.xs_all && staged != ch) {
        __syncthreads();
        stage_x(ch * chunk_cols, chunk_cols);
        staged = ch;
      }
      __syncthreads();
      const int kslab = ch * a.ks + my_ks;
      if (!warp_active || rt >= n_rt || kslab >= a.n_kslabs) continue;
      const int ls = kslab / NT, part = kslab - ls * NT;
      const int ps0 = part * PS;
      // B fragments of this kernel slab: x'[batch][sub-vector 64 ls + 4 ps + t], hi and lo
      uint4 bf[PS][NT];
      const int col_base = (a.xs_all ? kslab * KSV : (kslab - ch * a.ks) * KSV) * 8;
#pragma unroll
      for (int ps = 0; ps < PS; ++ps) {
        const int col = col_base + (4 * ps + t) * 8;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          int bb, part_lo;
          if constexpr (NT == 1) { bb = g & 3; part_lo = g >> 2; }
          else { part_lo = n / (NT / 2); bb = (n % (NT / 2)) * 8 + g; }
          uint4 v = make_uint4(0, 0, 0, 0);
          if (bb < B) v = *reinterpret_cast<const uint4*>((part_lo ? xl : xh) + (size_t)bb * a.xs_cols + col);
          bf[ps][n] = v;
        }
      }
      // this kernel slab's fields of rows g and g+8 of the row tile (prefetched for the first one)
      uint32_t w0[NWORDS], w1[NWORDS];
      if (task == task0 && ch == ch0) {
#pragma unroll
        for (int i = 0; i < NWORDS; ++i) { w0[i] = pw0[i]; w1[i] = pw1[i]; }
      } else {
        w0[NWORDS - 1] = w1[NWORDS - 1] = 0;
        const uint8_t* blk0 = L.tcodes + ((int64_t)rt * 16 + g) * L.tstride + (int64_t)ls * (8 * W) + t * (2 * W) + ps0 * W / 8;
        load_sub<W, NT>(blk0, w0);
        load_sub<W, NT>(blk0 + 8 * L.tstride, w1);
      }
      // gathers of G pair-steps are issued before their MMAs (hides L2 / shared latency)
      constexpr int G = (W >= 24 || PS < 8) ? (PS < 4 ? PS : 4) : 8;
      static_assert(PS % G == 0 && G <= PS, "pair-step batches must tile the kernel slab");
#pragma unroll
      for (int p0 = 0; p0 < PS; p0 += G) {
        uint4 c0[G], c1[G], e0[G], e1[G];
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const uint32_t f0 = field_of<W>(w0, p0 + j), f1 = field_of<W>(w1, p0 + j);
          // tensor-core layout fields already hold g * k + i for codebook group g
          if (CB_SMEM) {
            c0[j] = cb1s[(f0 & m1) * COPIES + (lane & (COPIES - 1))];
            c1[j] = cb1s[(f1 & m1) * COPIES + (lane & (COPIES - 1))];
          } else {
            c0[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb1) + (f0 & m1));
            c1[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb1) + (f1 & m1));
          }
          if (L.k2) {
            if (CB_SMEM) {
              e0[j] = cb2s[(f0 >> L.tc_bits1) * COPIES + (lane & (COPIES - 1))];
              e1[j] = cb2s[(f1 >> L.tc_bits1) * COPIES + (lane & (COPIES - 1))];
            } else {
              e0[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb2) + (f0 >> L.tc_bits1));
              e1[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb2) + (f1 >> L.tc_bits1));
            }
          }
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const int q = (j % (ACC / 2)) * 2;
            mma16816(dacc[q][n], c0[j].x, c1[j].x, c0[j].y, c1[j].y, bf[p0 + j][n].x, bf[p0 + j][n].y);
            mma16816(dacc[q + 1][n], c0[j].z, c1[j].z, c0[j].w, c1[j].w, bf[p0 + j][n].z, bf[p0 + j][n].w);
            if (L.k2) {
              mma16816(dacc[q][n], e0[j].x, e1[j].x, e0[j].y, e1[j].y, bf[p0 + j][n].x, bf[p0 + j][n].y);
              mma16816(dacc[q + 1][n], e0[j].z, e1[j].z, e0[j].w, e1[j].w, bf[p0 + j][n].z, bf[p0 + j][n].w);
            }
          }
        }
      }
    }
    float d[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float v = dacc[0][n][k];
#pragma unroll
        for (int q = 1; q < ACC; ++q) v += dacc[q][n][k];
        d[n][k] = v;
      }
    // ---- reduce the warps' D fragments: red[rt_local][row][col]
    if (warp_active) {
      float* r0 = red + ((size_t)my_rt_local * 16 + g) * (8 * NT);
      float* r1 = r0 + 8 * (8 * NT);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        atomicAdd(r0 + n * 8 + 2 * t, d[n][0]);
        atomicAdd(r0 + n * 8 + 2 * t + 1, d[n][1]);
        atomicAdd(r1 + n * 8 + 2 * t, d[n][2]);
        atomicAdd(r1 + n * 8 + 2 * t + 1, d[n][3]);
      }
    }
    __syncthreads();
    // ---- epilogue: (rtt*16 rows) x batch, sparse correction and outlier block (computed above)
    {
      // reduce over the lanes of this row (they are consecutive threads)
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        for (int o = 1; o < lanes_per_row; o <<= 1) {
          spv[b] += __shfl_xor_sync(0xffffffffu, spv[b], o);
          ov[b] += __shfl_xor_sync(0xffffffffu, ov[b], o);
        }
      }
      const float rsc = task == task0 ? rsc0 : ((L.rs && row_ok) ? __half2float(L.rs[row]) : 1.f);
      const float* rr = red + (size_t)rl * (8 * NT);
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        if (!row_ok || b >= B || (b & (lanes_per_row - 1)) != sub) continue;
        int nh, nl;
        if (NT == 1) { nh = b; nl = 4 + b; }
        else { nh = (b / 8) * 8 + (b % 8); nl = (NT / 2 + b / 8) * 8 + (b % 8); }
        float body = rr[nh] + rr[nl];
        float v = fmaf(rsc, body + ov[b], spv[b]);
        if (a.split) atomicAdd(a.acc + (int64_t)b * L.n_out + row, v);
        else store_from_float(a.y, a.yt, (int64_t)b * L.n_out + row, v);
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Warp-task variant.  Every (16-row tile, kernel slab) is an independent warp
// task that adds r * (its partial dot products) to a zeroed fp32 accumulator
// with atomics; every group of 8 rows has a task for the fused sparse term and
// the outlier block.  The sparse tasks come first in the task order so their
// dependent loads overlap the MMA tasks.  Shared memory holds the codebooks and
// x' for every column, written once; after that no block-wide barrier is needed,
// so warps overlap each other's memory latency freely.  B fragments are read
// from shared memory per pair-step, which keeps registers low enough for two
// blocks per SM.
template <int NT, int W, bool CB_SMEM, int COPIES, int NW>
__global__ void __launch_bounds__(NW * 32, 16 / NW) k_gemv_wt(Args a) {
  constexpr int WT_THREADS = NW * 32;   // NW warps per block: 8 (two blocks per SM) or 16 (one)
  constexpr int PS = 16 / NT;
  constexpr int KSV = 4 * PS;
  constexpr int BP = 4 * NT;
  constexpr int ACC = NT == 1 ? 4 : 2;   // independent MMA accumulator sets
  const Layer& L = a.L;
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* cb1s = reinterpret_cast<uint4*>(smem);
  uint4* cb2s = cb1s + (CB_SMEM ? (size_t)L.tc_k1 * COPIES : 0);
  __half* xh = reinterpret_cast<__half*>(cb2s + (CB_SMEM ? (size_t)L.tc_k2 * COPIES : 0));   // [batch][xs_cols]
  __half* xl = xh + (size_t)a.batch * a.xs_cols;
  float* xo = reinterpret_cast<float*>(xl + (size_t)a.batch * a.xs_cols);               // [BP][n_sub_o*8]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int B = a.batch;
  const uint32_t m1 = (1u << L.tc_bits1) - 1u;   // first-stage bits of the tensor-core layout

  if (CB_SMEM) {
    const uint4* c1 = reinterpret_cast<const uint4*>(L.tc_cb1);
    for (int i = threadIdx.x; i < L.tc_k1 * COPIES; i += WT_THREADS) cb1s[i] = __ldg(c1 + i / COPIES);
    if (L.k2) {
      const uint4* c2 = reinterpret_cast<const uint4*>(L.tc_cb2);
      for (int i = threadIdx.x; i < L.tc_k2 * COPIES; i += WT_THREADS) cb2s[i] = __ldg(c2 + i / COPIES);
    }
  }
  // x (and the accumulator) belong to the previous grid until it completes
  pdl_wait();
  pdl_release();
  const int n_o = L.n_sub_o * 8;
  for (int i = threadIdx.x; i < BP * n_o; i += WT_THREADS) {
    int b = i / n_o, p = i - b * n_o;
    float v = 0.f;
    if (b < B && p < L.n_ocols) {
      int j = L.colmap[L.n_main + p];
      v = load_as_float(a.x, a.xt, (int64_t)b * L.n_in + j);
      if (L.cs) v *= __half2float(L.cs[j]);
    }
    xo[i] = v;
  }
  // this block's column chunk: kernel slabs [ks_beg, ks_end), main columns from col0
  const int ch = blockIdx.x / a.wt_bpc, jb = blockIdx.x - ch * a.wt_bpc;
  const int ks_beg = ch * a.wt_cs, ks_end = min(ks_beg + a.wt_cs, a.n_kslabs);
  const int col0 = ks_beg * KSV * 8;
  // x' hi/lo for the chunk's main columns, eight columns per thread, loads first
  {
    const int groups = a.xs_cols / 8;
    for (int i = threadIdx.x; i < B * groups; i += WT_THREADS) {
      const int b = i / groups, q = (i - b * groups) * 8;
      const int qq = col0 + q;                         // main-column index of this group
      float v[8];
      if (!L.colmap && !L.tc_colmap && a.xt != VQLIN_F32 && qq + 8 <= L.n_main && (L.n_in & 7) == 0) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(a.x) +
                                                        (int64_t)b * L.n_in + qq));
        const unsigned short* hs = reinterpret_cast<const unsigned short*>(&u);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          v[k] = a.xt == VQLIN_F16 ? __half2float(__ushort_as_half(hs[k])) : __bfloat162float(__ushort_as_bfloat16(hs[k]));
        if (L.cs) {
          uint4 cu = __ldg(reinterpret_cast<const uint4*>(L.cs + qq));
          const __half* cv = reinterpret_cast<const __half*>(&cu);
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] *= __half2float(cv[k]);
        }
      } else {
        int jj[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          jj[k] = L.tc_colmap ? (qq + k < L.tc_nsub * 8 ? L.tc_colmap[qq + k] : -1)
                              : (qq + k < L.n_main ? (L.colmap ? L.colmap[qq + k] : qq + k) : -1);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = jj[k] >= 0 ? load_as_float(a.x, a.xt, (int64_t)b * L.n_in + jj[k]) : 0.f;
        if (L.cs) {
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] *= jj[k] >= 0 ? __half2float(L.cs[jj[k]]) : 0.f;
        }
      }
      uint32_t ph[4], pl[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __half h0 = __float2half_rn(v[2 * k]), h1 = __float2half_rn(v[2 * k + 1]);
        __half l0 = __float2half_rn(v[2 * k] - __half2float(h0)), l1 = __float2half_rn(v[2 * k + 1] - __half2float(h1));
        ph[k] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
        pl[k] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
      }
      *reinterpret_cast<uint4*>(xh + (size_t)b * a.xs_cols + q) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(xl + (size_t)b * a.xs_cols + q) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    }
  }
  __syncthreads();

  const int n_rt = (L.n_out + 15) / 16;
  const bool has_side = L.nnz > 0 || L.n_ocols > 0 || L.vsr_nb > 0;
  const int n_side = has_side ? (L.n_out + 7) / 8 : 0;      // sparse / outlier tasks of 8 rows
  const int gpc = (ks_end - ks_beg + a.wt_spt - 1) / a.wt_spt;   // slab groups of this chunk
  const int n_mt = n_rt * gpc;                                    // this chunk's MMA tasks
  // One task space per chunk, dealt round-robin over the chunk's warps: first the chunk's share of
  // the sparse / outlier tasks (side task ch, ch + nch, ...), then its MMA tasks, so every warp
  // gets the same number of tasks whichever kind they are.
  const int nch = a.wt_nch;
  const int n_side_c = n_side / nch + (ch < n_side % nch ? 1 : 0);
  const int total_c = n_side_c + n_mt;
  for (int tk = jb * NW + warp; tk < total_c; tk += a.wt_bpc * NW) {
    if (tk < n_side_c) {
      const int task = ch + tk * nch;                   // side task: rows 8 task .. +7
      // ---- fused sparse correction and outlier block for rows 8*task .. +8 (4 lanes per row)
      const int64_t row = (int64_t)task * 8 + (lane >> 2);
      const int sub = lane & 3;
      const bool ok = row < L.n_out;
      float spv[BP], ov[BP];
#pragma unroll
      for (int b = 0; b < BP; ++b) spv[b] = ov[b] = 0.f;
      if (ok && L.nnz > 0) sparse_row_terms<BP>(L, a.x, a.xt, B, row, sub, 4, spv);
      if (ok && L.vsr_nb > 0) vsr_row_terms<BP>(L, a.x, a.xt, B, row, sub, 4, spv);
      if (ok) {
        for (int so = sub; so < L.n_sub_o; so += 4) {
          uint32_t f = read_field(L.codes_o + row * L.stride_o, so, L.bits_o);
          uint4 u = __ldg(reinterpret_cast<const uint4*>(L.cbo) + f);
          const __half2* h = reinterpret_cast<const __half2*>(&u);
          float c[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) { float2 f2 = __half22float2(h[k]); c[2 * k] = f2.x; c[2 * k + 1] = f2.y; }
#pragma unroll
          for (int b = 0; b < BP; ++b)
            if (b < B) {
              float acc = ov[b];
#pragma unroll
              for (int k = 0; k < 8; ++k) acc = fmaf(c[k], xo[b * n_o + so * 8 + k], acc);
              ov[b] = acc;
            }
        }
      }
      const float rsc = (ok && L.rs) ? __half2float(L.rs[row]) : 1.f;
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        float v = fmaf(rsc, ov[b], spv[b]);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if (ok && b < B && sub == (b & 3) && v != 0.f) atomicAdd(a.acc + (int64_t)b * L.n_out + row, v);
      }
      continue;
    }
    // ---- MMA task: row tile rt over the kernel slabs of slab group sg of this chunk
    const int mt = tk - n_side_c;
    const int rt = mt / gpc, sg = mt - rt * gpc;
    // one slab per task at batch <= 8 (NT <= 2), known at compile time; several at batch > 8
    const int kb0 = ks_beg + sg * a.wt_spt, kb1 = NT <= 2 ? kb0 + 1 : min(kb0 + a.wt_spt, ks_end);
    const int64_t R0 = (int64_t)rt * 16 + g;
    constexpr int NWORDS = (2 * W / NT + 3) / 4 + 1;
    const float r0 = (L.rs && R0 < L.n_out) ? __half2float(L.rs[R0]) : 1.f;
    const float r1 = (L.rs && R0 + 8 < L.n_out) ? __half2float(L.rs[R0 + 8]) : 1.f;
    // ACC independent accumulator sets, so consecutive MMAs do not wait on each other
    float dacc[ACC][NT][4];
#pragma unroll
    for (int q = 0; q < ACC; ++q)
#pragma unroll
      for (int n = 0; n < NT; ++n) dacc[q][n][0] = dacc[q][n][1] = dacc[q][n][2] = dacc[q][n][3] = 0.f;
    for (int kslab = kb0; kslab < kb1; ++kslab) {
    const int ls = kslab / NT, part = kslab - ls * NT;
    uint32_t w0[NWORDS], w1[NWORDS];
    w0[NWORDS - 1] = w1[NWORDS - 1] = 0;
    const uint8_t* blk0 = L.tcodes + R0 * L.tstride + (int64_t)ls * (8 * W) + t * (2 * W) + part * PS * W / 8;
    load_sub<W, NT>(blk0, w0);
    load_sub<W, NT>(blk0 + 8 * L.tstride, w1);
    const int col_base = (kslab - ks_beg) * KSV * 8;   // inside the staged chunk
    // gathers per batch: never more than the slab's pair-steps (PS is 4 when NT = 4)
    constexpr int G = ((W >= 24) ? 4 : 8) < PS ? ((W >= 24) ? 4 : 8) : PS;
    static_assert(PS % G == 0, "pair-step batches must tile the kernel slab");
#pragma unroll
    for (int p0 = 0; p0 < PS; p0 += G) {
      uint4 c0[G], c1[G], e0[G], e1[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const uint32_t f0 = field_of<W>(w0, p0 + j), f1 = field_of<W>(w1, p0 + j);
        // tensor-core layout fields already hold g * k + i for codebook group g
        if (CB_SMEM) {
          c0[j] = cb1s[(f0 & m1) * COPIES + (lane & (COPIES - 1))];
          c1[j] = cb1s[(f1 & m1) * COPIES + (lane & (COPIES - 1))];
        } else {
          c0[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb1) + (f0 & m1));
          c1[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb1) + (f1 & m1));
        }
        if (L.k2) {
          if (CB_SMEM) {
            e0[j] = cb2s[(f0 >> L.tc_bits1) * COPIES + (lane & (COPIES - 1))];
            e1[j] = cb2s[(f1 >> L.tc_bits1) * COPIES + (lane & (COPIES - 1))];
          } else {
            e0[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb2) + (f0 >> L.tc_bits1));
            e1[j] = __ldg(reinterpret_cast<const uint4*>(L.tc_cb2) + (f1 >> L.tc_bits1));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const int col = col_base + (4 * (p0 + j) + t) * 8;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          int bb, part_lo;
          if constexpr (NT == 1) { bb = g & 3; part_lo = g >> 2; }
          else { part_lo = n / (NT / 2); bb = (n % (NT / 2)) * 8 + g; }
          uint4 bv = make_uint4(0, 0, 0, 0);
          if (bb < B) bv = *reinterpret_cast<const uint4*>((part_lo ? xl : xh) + (size_t)bb * a.xs_cols + col);
          const int q = (j % (ACC / 2)) * 2;
          mma16816(dacc[q][n], c0[j].x, c1[j].x, c0[j].y, c1[j].y, bv.x, bv.y);
          mma16816(dacc[q + 1][n], c0[j].z, c1[j].z, c0[j].w, c1[j].w, bv.z, bv.w);
          if (L.k2) {
            mma16816(dacc[q][n], e0[j].x, e1[j].x, e0[j].y, e1[j].y, bv.x, bv.y);
            mma16816(dacc[q + 1][n], e0[j].z, e1[j].z, e0[j].w, e1[j].w, bv.z, bv.w);
          }
        }
      }
    }
    }  // kernel slabs of the task
    float d[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float v = dacc[0][n][k];
#pragma unroll
        for (int q = 1; q < ACC; ++q) v += dacc[q][n][k];
        d[n][k] = v;
      }
    // hi + lo, times the row scale, into the accumulator
    if (NT == 1) {
      // columns 0-3 hold hi of batches 0-3, columns 4-7 lo: lanes t and t^2 pair up
#pragma unroll
      for (int k = 0; k < 4; ++k) d[0][k] += __shfl_xor_sync(0xffffffffu, d[0][k], 2);
      if (t < 2) {
        const int b0 = 2 * t, b1 = 2 * t + 1;
        if (b0 < B && R0 < L.n_out) atomicAdd(a.acc + (int64_t)b0 * L.n_out + R0, r0 * d[0][0]);
        if (b1 < B && R0 < L.n_out) atomicAdd(a.acc + (int64_t)b1 * L.n_out + R0, r0 * d[0][1]);
        if (b0 < B && R0 + 8 < L.n_out) atomicAdd(a.acc + (int64_t)b0 * L.n_out + R0 + 8, r1 * d[0][2]);
        if (b1 < B && R0 + 8 < L.n_out) atomicAdd(a.acc + (int64_t)b1 * L.n_out + R0 + 8, r1 * d[0][3]);
      }
    } else {
#pragma unroll
      for (int h = 0; h < NT / 2; ++h) {
        const int b0 = h * 8 + 2 * t, b1 = b0 + 1;
        const float v00 = d[h][0] + d[NT / 2 + h][0], v01 = d[h][1] + d[NT / 2 + h][1];
        const float v10 = d[h][2] + d[NT / 2 + h][2], v11 = d[h][3] + d[NT / 2 + h][3];
        if (b0 < B && R0 < L.n_out) atomicAdd(a.acc + (int64_t)b0 * L.n_out + R0, r0 * v00);
        if (b1 < B && R0 < L.n_out) atomicAdd(a.acc + (int64_t)b1 * L.n_out + R0, r0 * v01);
        if (b0 < B && R0 + 8 < L.n_out) atomicAdd(a.acc + (int64_t)b0 * L.n_out + R0 + 8, r1 * v10);
        if (b1 < B && R0 + 8 < L.n_out) atomicAdd(a.acc + (int64_t)b1 * L.n_out + R0 + 8, r1 * v11);
      }
    }
  }
}

template <int NT, int W, bool CB_SMEM, int COPIES>
static cudaError_t launch_wt_cfg(const Args& args, size_t smem, int grid, cudaStream_t s) {
  // one block per SM (shared memory) runs 16 warps; otherwise two blocks of 8
  const bool wide = 2 * (smem + 1024) > 227 * 1024;
  auto k = wide ? k_gemv_wt<NT, W, CB_SMEM, COPIES, 16> : k_gemv_wt<NT, W, CB_SMEM, COPIES, 8>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), wide ? 512 : 256, smem, s, args);
}

template <int NT, int W>
static cudaError_t launch_wt_w(const Args& args, bool cb_smem, int copies, size_t smem, int grid, cudaStream_t s) {
  if (!cb_smem) return launch_wt_cfg<NT, W, false, 1>(args, smem, grid, s);
  switch (copies) {
    case 8: return launch_wt_cfg<NT, W, true, 8>(args, smem, grid, s);
    case 4: return launch_wt_cfg<NT, W, true, 4>(args, smem, grid, s);
    case 2: return launch_wt_cfg<NT, W, true, 2>(args, smem, grid, s);
    default: return launch_wt_cfg<NT, W, true, 1>(args, smem, grid, s);
  }
}

template <int NT>
static cudaError_t launch_wt_nt(const Args& args, bool cb_smem, int copies, size_t smem, int grid, cudaStream_t s) {
  switch (args.L.tc_w) {
    case 8: return launch_wt_w<NT, 8>(args, cb_smem, copies, smem, grid, s);
    case 12: return launch_wt_w<NT, 12>(args, cb_smem, copies, smem, grid, s);
    case 16: return launch_wt_w<NT, 16>(args, cb_smem, copies, smem, grid, s);
    case 24: return launch_wt_w<NT, 24>(args, cb_smem, copies, smem, grid, s);
    default: return launch_wt_w<NT, 32>(args, cb_smem, copies, smem, grid, s);
  }
}

__global__ void k_finalize(const float* __restrict__ acc, int64_t n, void* __restrict__ y, vqlin_dtype yt) {
  pdl_wait();
  pdl_release();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    store_from_float(y, yt, i, acc[i]);
}

template <int NT, int W, bool CB_SMEM, int COPIES>
static cudaError_t launch_cfg(const Args& args, size_t smem, int grid, cudaStream_t s) {
  auto k = k_gemv_tc<NT, W, CB_SMEM, COPIES>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), THREADS, smem, s, args);
}

template <int NT, int W>
static cudaError_t launch_w(const Args& args, bool cb_smem, int copies, size_t smem, int grid, cudaStream_t s) {
  if (!cb_smem) return launch_cfg<NT, W, false, 1>(args, smem, grid, s);
  switch (copies) {
    case 8: return launch_cfg<NT, W, true, 8>(args, smem, grid, s);
    case 4: return launch_cfg<NT, W, true, 4>(args, smem, grid, s);
    case 2: return launch_cfg<NT, W, true, 2>(args, smem, grid, s);
    default: return launch_cfg<NT, W, true, 1>(args, smem, grid, s);
  }
}

template <int NT>
static cudaError_t launch_nt(const Args& args, bool cb_smem, int copies, size_t smem, int grid, cudaStream_t s) {
  switch (args.L.tc_w) {
    case 8: return launch_w<NT, 8>(args, cb_smem, copies, smem, grid, s);
    case 12: return launch_w<NT, 12>(args, cb_smem, copies, smem, grid, s);
    case 16: return launch_w<NT, 16>(args, cb_smem, copies, smem, grid, s);
    case 24: return launch_w<NT, 24>(args, cb_smem, copies, smem, grid, s);
    default: return launch_w<NT, 32>(args, cb_smem, copies, smem, grid, s);
  }
}

}  // namespace tcg

// fp32 [batch][n_out] accumulator of the column-split decode (256-byte multiple)
static size_t gemv_acc_bytes(const Layer& L, int batch) {
  return ((size_t)batch * L.n_out * 4 + 255) & ~size_t(255);
}

bool tc_supported(const Layer& L) {
  return L.tcodes != nullptr && (L.tc_w == 8 || L.tc_w == 12 || L.tc_w == 16 || L.tc_w == 24 || L.tc_w == 32);
}

size_t gemv_workspace_bytes(const Layer& L, int batch) {
  const size_t acc = gemv_acc_bytes(L, batch);
  const size_t cs = gemv_cs_workspace_bytes(L, batch);
  return acc > cs ? acc : cs;
}

// Clears an fp32 accumulator once the previous grid has completed.
__global__ void k_zero(float* __restrict__ p, int64_t n) {
  pdl_wait();
  pdl_release();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) p[i] = 0.f;
}

static int small_grid(int64_t n) { return (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024); }

// Plan and launch.  acc_ws: caller workspace for split accumulation (may be null).
cudaError_t launch_gemv_tc(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                           void* ws, size_t ws_bytes, cudaStream_t s, bool* handled) {
  using namespace tcg;
  *handled = false;
  if (!tc_supported(L) || batch < 1 || batch > 16) return cudaSuccess;
  const int NT = batch <= 4 ? 1 : (batch <= 8 ? 2 : 4);
  const int KSV = 64 / NT;
  // the split accumulator needs only [batch][n_out] fp32, whatever else the workspace is sized for
  const size_t acc_bytes = gemv_acc_bytes(L, batch);
  const int BP = 4 * NT;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem_max = 227 * 1024;
  // codebooks: as many interleaved copies (<= 8) as fit next to x'
  const size_t cb_entries = (size_t)L.tc_k1 + L.tc_k2;
  Args a;
  a.L = L; a.x = x; a.xt = xt; a.batch = batch; a.y = y; a.yt = yt; a.acc = nullptr;
  a.wt_cs = 0; a.wt_nch = 1; a.wt_bpc = 1; a.wt_spt = 1;   // set by the warp-task plan below
  a.n_kslabs = (L.tc_nsub + KSV - 1) / KSV;
  a.ks = a.n_kslabs < WARPS ? a.n_kslabs : WARPS;
  // round ks down to a divisor of WARPS so that rtt * ks == WARPS when several row tiles share a CTA
  while (WARPS % a.ks) --a.ks;
  a.rtt = WARPS / a.ks;
  a.n_chunks = (a.n_kslabs + a.ks - 1) / a.ks;
  const size_t red_bytes = (size_t)a.rtt * 16 * 8 * NT * 4;
  const size_t xo_bytes = (size_t)BP * L.n_sub_o * 8 * 4;
  const int all_cols = a.n_kslabs * KSV * 8;
  const int chunk_cols = a.ks * KSV * 8;
  const size_t x_all = (size_t)batch * all_cols * 4, x_chunk = (size_t)batch * chunk_cols * 4;
  // choose codebook placement and x' staging
  int copies = 0;
  bool cb_smem = false;
  for (int c = 8; c >= 1; c >>= 1) {
    size_t need = cb_entries * 16 * c + red_bytes + xo_bytes + x_chunk + 256;
    if (need <= smem_max && cb_entries * 16 * c <= 160 * 1024) { copies = c; cb_smem = true; break; }
  }
  const size_t cb_bytes = cb_smem ? cb_entries * 16 * copies : 0;
  a.xs_all = (cb_bytes + red_bytes + xo_bytes + x_all + 256 <= smem_max) ? 1 : 0;
  a.xs_cols = a.xs_all ? all_cols : chunk_cols;
  const size_t smem = cb_bytes + (size_t)batch * a.xs_cols * 4 + red_bytes + xo_bytes + 64;
  if (smem > smem_max) return cudaSuccess;   // does not fit: caller uses the generic kernel
  const int n_rt = (L.n_out + 15) / 16;
  // Plan checks on the host: the kernels read index fields of rows up to n_rt * 16 (the layout
  // pads rows to 16), x' columns up to the staged width (every slab when staged once, one chunk
  // of ks slabs otherwise), and at most WARPS kernel slabs per chunk.  Refuse a plan that breaks
  // any of them.
  if ((int64_t)n_rt * 16 > L.tcodes_rows || a.ks < 1 || a.ks > WARPS || a.rtt * a.ks != WARPS ||
      a.xs_cols < (a.xs_all ? all_cols : chunk_cols) || (int64_t)a.n_chunks * a.ks < a.n_kslabs) {
    set_error("tensor-core decode: inconsistent launch plan (refused)");
    return cudaErrorInvalidConfiguration;
  }
  const int n_rg = (n_rt + a.rtt - 1) / a.rtt;
  // ---- warp-task kernel: needs an fp32 accumulator (y itself, or the caller's workspace)
  //      and x' for every column next to the codebooks.  When one block task already
  //      covers every column and the tasks fit in one wave (the block-task kernel runs one
  //      block per SM), the block-task kernel below writes y in a single grid.
  if (a.n_chunks > 1 || n_rg > sms) {
    float* acc = nullptr;
    if (yt == VQLIN_F32) acc = reinterpret_cast<float*>(y);
    else if (ws && ws_bytes >= acc_bytes) acc = reinterpret_cast<float*>(ws);
    // x' for every column next to the codebooks (as many interleaved copies as fit) when that
    // fits; otherwise the columns are split into chunks of whole kernel slabs, each staged once
    // by the blocks that serve it
    int wcopies = 0;
    bool wcb = false;
    int cs = a.n_kslabs;                              // kernel slabs per chunk
    const size_t slab_x = (size_t)batch * KSV * 8 * 4;   // x' (hi + lo fp16) of one kernel slab
    for (int c = 8; c >= 1; c >>= 1) {
      if (cb_entries * 16 * c <= 160 * 1024 && cb_entries * 16 * c + x_all + xo_bytes + 256 <= smem_max) {
        wcopies = c; wcb = true; break;
      }
    }
    if (!wcb) {
      int fit = 0;
      for (int c = 8; c >= 1; c >>= 1) {
        const size_t cbb = cb_entries * 16 * c;
        if (cbb > 160 * 1024 || cbb + xo_bytes + 256 + slab_x > smem_max) continue;
        fit = (int)((smem_max - cbb - xo_bytes - 256) / slab_x);
        if (c == 1 || fit >= 4) { wcopies = c; wcb = true; break; }
      }
      if (!wcb) fit = (int)((smem_max - xo_bytes - 256) / slab_x);   // codebook gathered from L2
      cs = fit < a.n_kslabs ? fit : a.n_kslabs;
    }
    const int nch = cs > 0 ? (a.n_kslabs + cs - 1) / cs : 0;
    const size_t wsmem = (wcb ? cb_entries * 16 * wcopies : 0) + (size_t)batch * cs * KSV * 8 * 4 + xo_bytes + 64;
    if (acc && cs > 0 && wsmem <= smem_max) {
      Args w = a;
      w.acc = acc;
      w.xs_all = 1;
      w.xs_cols = cs * KSV * 8;
      const int n_side = (L.nnz > 0 || L.n_ocols > 0 || L.vsr_nb > 0) ? (L.n_out + 7) / 8 : 0;
      const int per_sm = (int)(smem_max / (wsmem + 1024)) >= 2 ? 2 : 1;
      const int nw = per_sm == 2 ? 8 : 16;             // warps per block (launch_wt_cfg's choice)
      int grid, bpc, spt = 1;
      if (nch == 1) {
        const int total = n_side + n_rt * a.n_kslabs;
        grid = sms * per_sm;
        if (grid > (total + WARPS - 1) / WARPS) grid = (total + WARPS - 1) / WARPS;
        bpc = grid;
      } else {
        bpc = sms * per_sm / nch;
        if (bpc < 1) bpc = 1;
        grid = nch * bpc;
        // a task covers spt slabs of one row tile: about three tasks per warp
        const int64_t slab_tasks = (int64_t)n_rt * a.n_kslabs, target = 3ll * grid * nw;
        spt = (int)((slab_tasks + target - 1) / target);
        if (spt > cs) spt = cs;
        if (spt < 1 || NT <= 2) spt = 1;               // the NT <= 2 kernels take one slab per task
      }
      w.wt_cs = cs; w.wt_nch = nch; w.wt_bpc = bpc; w.wt_spt = spt;
      // plan checks: every chunk's slabs are staged, and the grid is whole chunks of blocks
      if (grid != nch * bpc || (int64_t)nch * cs < a.n_kslabs || w.xs_cols < cs * KSV * 8) {
        set_error("warp-task decode: inconsistent launch plan (refused)");
        return cudaErrorInvalidConfiguration;
      }
      cudaError_t e = launch_pdl(k_zero, dim3(small_grid((int64_t)batch * L.n_out)), 256, 0, s, acc,
                                 (int64_t)batch * L.n_out);
      if (e != cudaSuccess) return e;
      if (NT == 1) e = launch_wt_nt<1>(w, wcb, wcopies, wsmem, grid, s);
      else if (NT == 2) e = launch_wt_nt<2>(w, wcb, wcopies, wsmem, grid, s);
      else e = launch_wt_nt<4>(w, wcb, wcopies, wsmem, grid, s);
      if (e != cudaSuccess) return e;
      if (yt != VQLIN_F32) {
        int64_t n = (int64_t)batch * L.n_out;
        e = launch_pdl(k_finalize, dim3(small_grid(n)), 256, 0, s, (const float*)acc, n, y, yt);
      }
      *handled = (e == cudaSuccess);
      return e;
    }
  }
  // ---- block-task kernel (no scratch needed); split by chunk when there is more than one chunk
  //      and an fp32 accumulator is available
  a.split = 0;
  if (a.n_chunks > 1) {
    if (yt == VQLIN_F32) { a.split = 1; a.acc = reinterpret_cast<float*>(y); }
    else if (ws && ws_bytes >= acc_bytes) { a.split = 1; a.acc = reinterpret_cast<float*>(ws); }
    // otherwise every task loops over the chunks itself (no scratch needed)
  }
  const int n_tasks = a.split ? n_rg * a.n_chunks : n_rg;
  const int per_sm = (int)(smem_max / (smem + 1024)) < 1 ? 1 : (int)(smem_max / (smem + 1024));
  int grid = sms * (per_sm > 2 ? 2 : per_sm);
  if (grid > n_tasks) grid = n_tasks;
  cudaError_t e;
  if (a.split) {
    e = launch_pdl(k_zero, dim3(small_grid((int64_t)batch * L.n_out)), 256, 0, s, a.acc, (int64_t)batch * L.n_out);
    if (e != cudaSuccess) return e;
  }
  if (NT == 1) e = launch_nt<1>(a, cb_smem, copies, smem, grid, s);
  else if (NT == 2) e = launch_nt<2>(a, cb_smem, copies, smem, grid, s);
  else e = launch_nt<4>(a, cb_smem, copies, smem, grid, s);
  if (e != cudaSuccess) return e;
  if (a.split && yt != VQLIN_F32) {
    int64_t n = (int64_t)batch * L.n_out;
    e = launch_pdl(k_finalize, dim3(small_grid(n)), 256, 0, s, (const float*)a.acc, n, y, yt);
  }
  *handled = (e == cudaSuccess);
  return e;
}

}  // namespace vqlin
