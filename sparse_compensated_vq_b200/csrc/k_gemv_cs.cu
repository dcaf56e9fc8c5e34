// Codebook-stationary decode GEMV for codebooks too large for one SM's shared
// memory (K = 65536 entries of d = 8 fp16 = 1 MiB): the fused dequant + GEMV of
// the VPTQ page ("The dequantization interface", QGemv) reorganised so that
// every centroid gather is a bank-conflict-free shared-memory load.
//
// At create time every sub-vector (row i, position s) of the main block is put
// in the bucket of thread block (p, h): p = the codebook slice holding its index
// (slices of E < 1024 consecutive entries), h = the half of the rows holding i.
// Inside a bucket the entries are sorted by position s, then row; an entry keeps
// (row - first row of the half, index - first index of the slice) in a 21-bit
// slot, three per 64-bit word (32-bit slots, two per word, when it needs more
// bits).  Each run of one position is padded to whole words with a null entry
// (local index E, a zero centroid), so every word carries one position, which is
// stored beside it.
//
// A block holds its slice as 8 interleaved copies (entry k of copy c at k*8+c, so
// the eight lanes of a quarter-warp, which read copies 0..7, always hit eight
// different bank groups; 4 copies, half the conflict-free width, when 8 would leave no room
// for the whole entry stream next to a batch of 3-4), x' = c (.) x for every position in
// fp32, and a
// shared-memory accumulator for the rows of its half.  Its entry words and their
// positions arrive by bulk asynchronous copies while it stages the rest.  Each
// lane then takes one word (EPW entries of one position) at a time: x'[s] is a
// broadcast load, each centroid is one conflict-free 16-byte load, and each
// product is added to its row with a 32-bit integer shared-memory atomic.
//
// The row accumulator is fixed point (float shared-memory atomics are several
// times slower than integer ones).  The block's scale S = 2^e is the largest power
// of two with S * bound * max|x'| < 2^30, where bound = (most entries of one row in
// the block) * (largest l1 norm of a centroid in the slice) comes with the layout.
// Since |c . x'| <= l1(c) * max|x'|, no row sum can leave int32, and each product
// is rounded to a multiple of 1/S, i.e. by at most 2^-31 * bound * max|x'|.  Summed
// over all blocks a row's error is below n_sub * (most entries of one row) * 2^-31
// times the largest possible single product (the layout is built only while that
// factor is <= 2^-11).  Integer sums do not depend on the order of the atomics,
// so the result is deterministic.  x must be finite.
//
// The block writes its row sums to its own fp32 plane of the caller's workspace, and k_cs_finalize
// sums the planes per row, applies the row scale and adds the fused sparse
// correction and the outlier-column block (SCVQ summary step 4; HAS-VQ abstract:
// sparse entries exact), at full occupancy.  No global atomics.  Waits are
// bounded.
#include "vqlin_internal.cuh"

namespace vqlin {

namespace csg {

constexpr int WARPS = 16;
constexpr int THREADS = WARPS * 32;
constexpr unsigned long long WAIT_NS = 1000000000ull;

__device__ int g_cs_error = 0;

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(su32(dst)), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__host__ __device__ inline size_t r16(size_t v) { return (v + 15) & ~size_t(15); }

// Shared-memory layout of a block (byte offsets, every region 16-byte aligned).
struct Carve {
  size_t xs, yp, bar, words;
  __host__ __device__ Carve(int E, int n_sub, int NB, int rpp, int copies) {
    xs = r16((size_t)(E + 1) * copies * 16);            // slice + the null entry
    yp = r16(xs + (size_t)n_sub * NB * 8 * 4);
    bar = r16(yp + (size_t)NB * rpp * 4);
    words = bar + 16 + WARPS * 4;                     // mbarrier, abort flag, per-warp max|x'|
  }
  // entry words then their positions (u16), for a buffer of `cap` words (cap % 32 == 0)
  __host__ __device__ size_t wpos(int cap) const { return words + (size_t)cap * 8; }
  __host__ __device__ size_t total(int cap) const { return wpos(cap) + (size_t)cap * 2; }
};

struct Args {
  Layer L;
  const void* x;
  vqlin_dtype xt;
  int batch;
  float* planes;        // [P][batch][n_out]
  int words_cap;        // words the shared buffer holds (a multiple of 32)
};

template <int NB, int EPW, int COPIES>
__global__ void __launch_bounds__(THREADS, 1) k_gemv_cs(Args a) {
  constexpr int SLOT = EPW == 3 ? 21 : 32;
  const Layer& L = a.L;
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = L.cs_H, E = L.cs_E, RPP = L.cs_rpp;
  const int c = blockIdx.x;
  const int p = c / H, h = c - p * H;
  const int row0 = h * RPP;
  const int nrows = min(RPP, L.n_out - row0);
  const int slice0 = p * E, E_p = max(0, min(E, L.n_groups * L.k1 - slice0));   // virtual codebook of all groups
  const int n_sub = L.n_sub;
  const int B = a.batch;
  const Carve cv(E, n_sub, NB, RPP, COPIES);
  uint4* cbs = reinterpret_cast<uint4*>(smem);                        // [E][8]
  float* xs = reinterpret_cast<float*>(smem + cv.xs);                 // [n_sub][NB][8]
  int* yp = reinterpret_cast<int*>(smem + cv.yp);                     // [NB][RPP] fixed point
  float* wmax = reinterpret_cast<float*>(smem + cv.bar + 16);         // [WARPS]
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + cv.bar);         // mbarrier + abort flag
  uint64_t* words = reinterpret_cast<uint64_t*>(smem + cv.words);     // [cap]
  uint16_t* wpos = reinterpret_cast<uint16_t*>(smem + cv.wpos(a.words_cap));   // [cap]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this block's words [cs_start[c], cs_start[c+1]), a multiple of 32
  const int64_t w_begin = L.cs_start[c];
  const int n_words = (int)(L.cs_start[c + 1] - w_begin);
  const bool one_chunk = n_words <= a.words_cap;
  auto issue_chunk = [&](int w0) {      // thread 0: words [w0, w0 + n) and their positions
    const int n = min(a.words_cap, n_words - w0);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(bar)), "r"((uint32_t)(n * 10))
                 : "memory");
    bulk_load(words, L.cs_words + w_begin + w0, (uint32_t)(n * 8), su32(bar));
    bulk_load(wpos, L.cs_wpos + w_begin + w0, (uint32_t)(n * 2), su32(bar));
  };
  // Launched as a programmatic dependent: everything before griddepcontrol.wait reads only
  // the layer (immutable) and writes only shared memory, so it may overlap the previous grid.
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(bar)) : "memory");
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (one_chunk && n_words > 0) issue_chunk(0);   // overlaps the staging below
  }
  float fx_scale, fx_inv;                            // fixed-point scale S and 1/S
  // ---- codebook slice (8 interleaved copies), then x' per position
  {
    const float bound = L.cs_bound[c];
    float xmax = 0.f;
    const uint4* cb = reinterpret_cast<const uint4*>(L.cb1) + slice0;
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    const int k0 = threadIdx.x, k1 = threadIdx.x + THREADS;
    v0 = __ldg(cb + min(k0, E_p - 1));                  // every slice holds at least one entry
    v1 = __ldg(cb + min(k1, E_p - 1));
    // the copies are written in a lane-rotated order: at every store the eight lanes of a
    // quarter-warp write eight different copies, i.e. eight different bank groups
    const int rot = ((threadIdx.x & 7) / (8 / COPIES)) & (COPIES - 1);
    if (k0 < E_p)
#pragma unroll
      for (int cc = 0; cc < COPIES; ++cc) cbs[k0 * COPIES + ((cc + rot) & (COPIES - 1))] = v0;
    if (k1 < E_p)
#pragma unroll
      for (int cc = 0; cc < COPIES; ++cc) cbs[k1 * COPIES + ((cc + rot) & (COPIES - 1))] = v1;
    for (int k = threadIdx.x + 2 * THREADS; k < E_p; k += THREADS) {   // slices wider than 2*THREADS
      const uint4 v = __ldg(cb + k);
#pragma unroll
      for (int cc = 0; cc < COPIES; ++cc) cbs[k * COPIES + ((cc + rot) & (COPIES - 1))] = v;
    }
    if (threadIdx.x < COPIES) cbs[E * COPIES + threadIdx.x] = make_uint4(0, 0, 0, 0);   // the null entry
    for (int i = threadIdx.x; i < NB * RPP; i += THREADS) yp[i] = 0;

    // column scales of every (position, batch) item, before the wait (layer data), parked in
    // the item's x' slot; item i fills 32 bytes, and lanes 4..7 of each quarter-warp write
    // their two halves in the other order, so every store covers eight different bank groups
    const int sw = (threadIdx.x >> 2) & 1;
    for (int i = threadIdx.x; i < n_sub * NB; i += THREADS) {
      const int s = i / NB, b = i - s * NB;
      const int q0 = s * 8;
      float cvv[8];
      if (!L.cs) {
#pragma unroll
        for (int k = 0; k < 8; ++k) cvv[k] = 1.f;
      } else if (!L.colmap && q0 + 8 <= L.n_main) {
        const uint4 cu = __ldg(reinterpret_cast<const uint4*>(L.cs + q0));
        const __half* ch = reinterpret_cast<const __half*>(&cu);
#pragma unroll
        for (int k = 0; k < 8; ++k) cvv[k] = __half2float(ch[k]);
      } else {
        int jj[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int q = min(q0 + k, L.n_main - 1);
          jj[k] = L.colmap ? L.colmap[q] : q;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) cvv[k] = __half2float(L.cs[jj[k]]);
      }
      float4* dst = reinterpret_cast<float4*>(xs + ((size_t)s * NB + b) * 8);
      const float4 lo = make_float4(cvv[0], cvv[1], cvv[2], cvv[3]), hi = make_float4(cvv[4], cvv[5], cvv[6], cvv[7]);
      dst[sw] = sw ? hi : lo;
      dst[sw ^ 1] = sw ? lo : hi;
    }

    // x is written by the previous grid: wait for it.  Only then may the finalize grid start
    // (its sparse and outlier terms read x before they wait for this grid).
    pdl_wait();
    pdl_release();
    // x' = c (.) x for every item (the same thread owns the same items as above): 16-byte loads
    // of x when the main columns are contiguous and 8-aligned, else eight clamped scalar loads
    const bool vec = !L.colmap && a.xt != VQLIN_F32 && (L.n_in & 7) == 0;
    with_dtype(a.xt, [&](auto tag) {
      constexpr int XT = decltype(tag)::value;
      for (int i = threadIdx.x; i < n_sub * NB; i += THREADS) {
        const int s = i / NB, b = i - s * NB;
        const int q0 = s * 8;
        float v[8];
        if (XT != VQLIN_F32 && vec && b < B && q0 + 8 <= L.n_main) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(a.x) +
                                                              (int64_t)b * L.n_in + q0));
          const unsigned short* hs = reinterpret_cast<const unsigned short*>(&u);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            v[k] = XT == VQLIN_F16 ? __half2float(__ushort_as_half(hs[k])) : __bfloat162float(__ushort_as_bfloat16(hs[k]));
        } else {
          int jj[8];
          bool ok[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int q = q0 + k;
            ok[k] = b < B && q < L.n_main;
            jj[k] = ok[k] ? (L.colmap ? L.colmap[q] : q) : 0;
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = ldx<XT>(a.x, (int64_t)(b < B ? b : 0) * L.n_in + jj[k]);
#pragma unroll
          for (int k = 0; k < 8; ++k) if (!ok[k]) v[k] = 0.f;
        }
        float4* dst = reinterpret_cast<float4*>(xs + ((size_t)s * NB + b) * 8);
        const float4 c0 = dst[0], c1 = dst[1];
        const float4 lo = make_float4(v[0] * c0.x, v[1] * c0.y, v[2] * c0.z, v[3] * c0.w);
        const float4 hi = make_float4(v[4] * c1.x, v[5] * c1.y, v[6] * c1.z, v[7] * c1.w);
        xmax = fmaxf(xmax, fmaxf(fmaxf(fmaxf(fabsf(lo.x), fabsf(lo.y)), fmaxf(fabsf(lo.z), fabsf(lo.w))),
                                 fmaxf(fmaxf(fabsf(hi.x), fabsf(hi.y)), fmaxf(fabsf(hi.z), fabsf(hi.w)))));
        dst[sw] = sw ? hi : lo;
        dst[sw ^ 1] = sw ? lo : hi;
      }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, o));
    if (lane == 0) wmax[warp] = xmax;
    __syncthreads();
    xmax = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) xmax = fmaxf(xmax, wmax[w]);
    // S = 2^(30 - ex) with bound * max|x'| = m * 2^ex, 0.5 <= m < 1
    int ex = 0;
    const float t = bound * xmax;
    if (t > 0.f) (void)frexpf(t, &ex);
    const int es = t > 0.f ? max(-126, min(126, 30 - ex)) : 0;
    fx_scale = ldexpf(1.f, es);
    fx_inv = ldexpf(1.f, -es);
  }

  // ---- main loop over the entry words (one chunk when they fit, else chunk by chunk)
  const uint32_t lmask = (1u << L.cs_local_bits) - 1u;
  const uint64_t emask = (1ull << L.cs_ebits) - 1ull;
  const int lbits = L.cs_local_bits;
  uint32_t phase = 0;
  for (int w0 = 0; w0 < n_words; w0 += a.words_cap) {
    if (!one_chunk) {
      __syncthreads();
      if (threadIdx.x == 0) issue_chunk(w0);
    }
    if (!one_chunk || w0 == 0) {
      bool ok = mbar_try(su32(bar), phase);
      if (!ok) {
        const uint64_t t0 = now_ns();
        while (!(ok = mbar_try(su32(bar), phase)))
          if (now_ns() - t0 > WAIT_NS) { atomicExch(&g_cs_error, 6); *abort_flag = 1; break; }
      }
      phase ^= 1u;
    }
    __syncthreads();
    if (*abort_flag) break;
    // warps take whole groups of 32 words, so one instruction covers one layout group
    const int ng = min(a.words_cap, n_words - w0) >> 5;
    const int wb = (ng * warp / WARPS) << 5, we = (ng * (warp + 1) / WARPS) << 5;
    for (int wi = wb + lane; wi < we; wi += 32) {
      const uint64_t wv = words[wi];
      const int s = wpos[wi];
      uint32_t ent[EPW];
      uint4 cen[EPW];
#pragma unroll
      for (int u = 0; u < EPW; ++u) {
        ent[u] = (uint32_t)((wv >> (u * SLOT)) & emask);
        cen[u] = cbs[(ent[u] & lmask) * COPIES + (lane & (COPIES - 1))];
      }
      float xr[NB][8];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float4* xv = reinterpret_cast<const float4*>(xs + ((size_t)s * NB + b) * 8);
        const float4 x0 = xv[0], x1 = xv[1];
        xr[b][0] = x0.x; xr[b][1] = x0.y; xr[b][2] = x0.z; xr[b][3] = x0.w;
        xr[b][4] = x1.x; xr[b][5] = x1.y; xr[b][6] = x1.z; xr[b][7] = x1.w;
      }
#pragma unroll
      for (int u = 0; u < EPW; ++u) {
        const __half2* h2 = reinterpret_cast<const __half2*>(&cen[u]);
        float cf[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) { const float2 f2 = __half22float2(h2[k]); cf[2 * k] = f2.x; cf[2 * k + 1] = f2.y; }
        const int row_l = (int)(ent[u] >> lbits);
        const bool real = (ent[u] & lmask) != (uint32_t)E;   // null entries add nothing
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b >= B || !real) continue;
          float p0 = cf[0] * xr[b][0], p1 = cf[1] * xr[b][1];
          p0 = fmaf(cf[2], xr[b][2], p0); p1 = fmaf(cf[3], xr[b][3], p1);
          p0 = fmaf(cf[4], xr[b][4], p0); p1 = fmaf(cf[5], xr[b][5], p1);
          p0 = fmaf(cf[6], xr[b][6], p0); p1 = fmaf(cf[7], xr[b][7], p1);
          atomicAdd(yp + (size_t)b * RPP + row_l, __float2int_rn((p0 + p1) * fx_scale));
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {   // a copy still in flight must land before the block exits
    const uint64_t t0 = now_ns();
    while (!mbar_try(su32(bar), phase ^ 1u) && now_ns() - t0 < WAIT_NS) {}
  }
  // ---- this block's plane: row sums of half h (the row scale is applied at the end)
  float* plane = a.planes + (size_t)p * B * L.n_out;
  const bool aborted = *abort_flag;
  for (int r = threadIdx.x; r < nrows; r += THREADS)
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (b < B) plane[(size_t)b * L.n_out + row0 + r] = aborted ? 0.f : (float)yp[(size_t)b * RPP + r] * fx_inv;
}

// y[b][i] = r_i * (sum_p planes[p][b][i] + outlier block) + sum_e delta_e x[b][col_e].
// A block takes 32 rows.  It is launched as a programmatic dependent of the
// codebook-stationary grid, so it first computes the terms that do not need that
// grid's output (sparse term: each warp takes four consecutive rows as one range
// of CSR entries, loads issued eight at a time; outlier block: a warp per row),
// then waits for the grid and sums the planes: 8 groups of 32 threads, group g
// adds the planes p = g, g+8, ... (loads issued together, coalesced over the
// rows), then a shared-memory reduction.
template <int NB>
__global__ void __launch_bounds__(256) k_cs_finalize(Layer L, const float* __restrict__ planes, int P,
                                                     const void* __restrict__ x, vqlin_dtype xt, int batch,
                                                     void* __restrict__ y, vqlin_dtype yt) {
  constexpr int PG = 16;                              // planes per group and round (loads in flight)
  __shared__ float part[8][NB][32], spv[NB][32], ovv[NB][32];
  const int i0 = blockIdx.x * 32;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  // the next grid may start its layer-only prologue; it waits for this grid before reading x
  pdl_release();
  with_dtype(xt, [&](auto tag) {
    constexpr int XT = decltype(tag)::value;
    // sparse term of rows i0 + 4*warp .. +3
    const int r0 = warp * 4, ib = i0 + r0;
    float sp[4][NB];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int b = 0; b < NB; ++b) sp[q][b] = 0.f;
    if (L.nnz > 0 && ib < L.n_out) {
      const int rows = min(4, L.n_out - ib);
      int bnd[5];
#pragma unroll
      for (int q = 0; q < 5; ++q) bnd[q] = L.row_ptr[ib + min(q, rows)];
      const int e_end = bnd[4];                      // rows past the last one repeat its end
      for (int e0 = bnd[0] + lane; e0 < e_end; e0 += 32 * 8) {
        float dl[8];
        int jj[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {   // clamped indices: the eight loads issue together
          const int e = min(e0 + 32 * u, e_end - 1);
          dl[u] = L.delta[e];
          jj[u] = L.col16 ? (int)L.col16[e] : L.col[e];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) if (e0 + 32 * u >= e_end) dl[u] = 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b >= batch) continue;
          float xv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) xv[u] = ldx<XT>(x, (int64_t)b * L.n_in + jj[u]);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int e = e0 + 32 * u;
            const float pr = dl[u] * xv[u];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (e >= bnd[q] && e < bnd[q + 1]) sp[q][b] += pr;
          }
        }
      }
    }
    // VSR blocks of the same four rows (lanes over each row's blocks)
    if (L.vsr_nb > 0) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t row = ib + q;
        float tv[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) tv[b] = 0.f;
        if (row < L.n_out) vsr_row_terms<NB>(L, x, xt, batch, row, lane, 32, tv);
#pragma unroll
        for (int b = 0; b < NB; ++b) sp[q][b] += tv[b];
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sp[q][b] += __shfl_xor_sync(0xffffffffu, sp[q][b], o);
        if (lane == 0) spv[b][r0 + q] = sp[q][b];
      }
    // outlier block: a warp per row (rows warp, warp + 8, ...)
    for (int rr = warp; rr < 32; rr += 8) {
      const int i = i0 + rr;
      float ov[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) ov[b] = 0.f;
      if (i < L.n_out) {
        for (int so = lane; so < L.n_sub_o; so += 32) {
          const uint32_t f = read_field(L.codes_o + (int64_t)i * L.stride_o, so, L.bits_o);
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(L.cbo) + f);
          const __half* hv = reinterpret_cast<const __half*>(&u);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int pcol = so * 8 + k;
            if (pcol >= L.n_ocols) break;
            const int j = L.colmap[L.n_main + pcol];
            const float cj = L.cs ? __half2float(L.cs[j]) : 1.f;
            const float ck = __half2float(hv[k]);
#pragma unroll
            for (int b = 0; b < NB; ++b)
              if (b < batch) ov[b] = fmaf(ck, cj * ldx<XT>(x, (int64_t)b * L.n_in + j), ov[b]);
          }
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ov[b] += __shfl_xor_sync(0xffffffffu, ov[b], o);
        if (lane == 0) ovv[b][rr] = ov[b];
      }
    }
  });
  // row scale of this thread's output row (layer data, read before the wait)
  float rsc = 1.f;
  {
    const int i = i0 + (t & 31);
    if (L.rs && (t >> 5) < NB && i < L.n_out) rsc = __half2float(L.rs[i]);
  }
  // the planes are written by the preceding codebook-stationary grid
  pdl_wait();
  {
    const int g = warp, r = lane, i = i0 + r;
    const size_t stride = (size_t)batch * L.n_out;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float acc = 0.f;
      if (b < batch && i < L.n_out) {
        const float* pp = planes + (size_t)b * L.n_out + i;
        for (int q0 = g; q0 < P; q0 += 8 * PG) {
          float v[PG];
#pragma unroll
          for (int k = 0; k < PG; ++k) {
            const int q = q0 + 8 * k;
            v[k] = __ldcg(pp + (size_t)min(q, P - 1) * stride);   // clamped: every load issues at once
          }
#pragma unroll
          for (int k = 0; k < PG; ++k) acc += (q0 + 8 * k < P) ? v[k] : 0.f;
        }
      }
      part[g][b][r] = acc;
    }
  }
  __syncthreads();
  {
    const int b = t >> 5, r = t & 31;
    const int i = i0 + r;
    if (b < NB && b < batch && i < L.n_out) {
      float body = 0.f;
#pragma unroll
      for (int g = 0; g < 8; ++g) body += part[g][b][r];
      store_from_float(y, yt, (int64_t)b * L.n_out + i, fmaf(rsc, body + ovv[b][r], spv[b][r]));
    }
  }
}

template <int NB, int EPW, int COPIES>
static cudaError_t launch_cfg(const Args& a, size_t smem, cudaStream_t s) {
  auto k = k_gemv_cs<NB, EPW, COPIES>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(a.L.cs_P * a.L.cs_H), THREADS, smem, s, a);
}

}  // namespace csg

// Failure-detection self-test: one thread waits on a freshly initialised mbarrier that nothing
// will ever complete, with the same bounded try-wait loop the decode kernel uses but the
// caller's limit.  When the limit passes it records code 7 and returns; no copy is in flight.
namespace csg {
__global__ void k_wait_probe(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const uint64_t t0 = now_ns();
    while (!mbar_try(su32(&bar), 0u))
      if (now_ns() - t0 > limit_ns) { atomicExch(&g_cs_error, 7); break; }
  }
}

}  // namespace csg

int read_and_clear_cs_error() {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, csg::g_cs_error, sizeof v) != cudaSuccess) return -1;
  if (v) cudaMemcpyToSymbol(csg::g_cs_error, &zero, sizeof zero);
  return v;
}

size_t gemv_cs_workspace_bytes(const Layer& L, int batch) {
  if (!L.cs_words || batch > 4) return 0;
  return ((size_t)L.cs_P * batch * L.n_out * 4 + 255) & ~size_t(255);
}

cudaError_t launch_gemv_cs(const Layer& L, const void* x, vqlin_dtype xt, int batch, void* y, vqlin_dtype yt,
                           void* ws, size_t ws_bytes, cudaStream_t s, bool* handled) {
  using namespace csg;
  *handled = false;
  if (!L.cs_words || batch < 1 || batch > 4) return cudaSuccess;
  const size_t need = gemv_cs_workspace_bytes(L, batch);
  if (!ws || ws_bytes < need) return cudaSuccess;
  const int NB = batch == 1 ? 1 : (batch == 2 ? 2 : 4);
  const size_t smem_max = 227 * 1024;
  // 8 codebook copies (conflict-free gathers) unless that forces the entry stream into
  // several chunks while 4 copies would hold it whole
  const int need_words = (int)((L.cs_max_words + 31) & ~31ll);
  int copies = 8;
  {
    const Carve c8(L.cs_E, L.n_sub, NB, L.cs_rpp, 8), c4(L.cs_E, L.n_sub, NB, L.cs_rpp, 4);
    if (c8.total(need_words) > smem_max && c4.total(need_words) <= smem_max) copies = 4;
  }
  const Carve cv(L.cs_E, L.n_sub, NB, L.cs_rpp, copies);
  if (cv.total(64) > smem_max) return cudaSuccess;
  Args a;
  a.L = L; a.x = x; a.xt = xt; a.batch = batch; a.planes = reinterpret_cast<float*>(ws);
  int cap = (int)(((smem_max - cv.words) / 10) & ~31ll);     // 8 + 2 bytes per word, whole groups of 32
  if (need_words < cap) cap = need_words;
  a.words_cap = cap < 32 ? 32 : cap;
  const size_t smem = cv.total(a.words_cap);
  // Plan checks on the host, before anything is launched: the carve must lie inside the dynamic
  // shared memory requested, the word buffer must hold whole 32-word groups, every slot's local
  // index and row must fit the slice and the row half, and the partial planes must fit the
  // workspace.  A plan that fails any of them is refused instead of launched.
  if (smem > smem_max || a.words_cap % 32 != 0 || (int64_t)L.cs_P * L.cs_E < (int64_t)L.n_groups * L.k1 ||
      (int64_t)L.cs_H * L.cs_rpp < L.n_out || (1ll << L.cs_local_bits) <= L.cs_E ||
      (size_t)(L.cs_E + 1) * copies * 16 > cv.xs || (size_t)L.cs_P * batch * L.n_out * 4 > ws_bytes) {
    set_error("codebook-stationary decode: inconsistent launch plan (refused)");
    return cudaErrorInvalidConfiguration;
  }
  cudaError_t e;
  if (copies == 8) {
    if (L.cs_epw == 3) {
      if (NB == 1) e = launch_cfg<1, 3, 8>(a, smem, s);
      else if (NB == 2) e = launch_cfg<2, 3, 8>(a, smem, s);
      else e = launch_cfg<4, 3, 8>(a, smem, s);
    } else {
      if (NB == 1) e = launch_cfg<1, 2, 8>(a, smem, s);
      else if (NB == 2) e = launch_cfg<2, 2, 8>(a, smem, s);
      else e = launch_cfg<4, 2, 8>(a, smem, s);
    }
  } else {
    if (L.cs_epw == 3) {
      if (NB == 1) e = launch_cfg<1, 3, 4>(a, smem, s);
      else if (NB == 2) e = launch_cfg<2, 3, 4>(a, smem, s);
      else e = launch_cfg<4, 3, 4>(a, smem, s);
    } else {
      if (NB == 1) e = launch_cfg<1, 2, 4>(a, smem, s);
      else if (NB == 2) e = launch_cfg<2, 2, 4>(a, smem, s);
      else e = launch_cfg<4, 2, 4>(a, smem, s);
    }
  }
  if (e != cudaSuccess) return e;
  const float* planes = a.planes;
  const int P = L.cs_P;
  const dim3 fgrid((L.n_out + 31) / 32);
  if (NB == 1) e = launch_pdl(k_cs_finalize<1>, fgrid, 256, 0, s, L, planes, P, x, xt, batch, y, yt);
  else if (NB == 2) e = launch_pdl(k_cs_finalize<2>, fgrid, 256, 0, s, L, planes, P, x, xt, batch, y, yt);
  else e = launch_pdl(k_cs_finalize<4>, fgrid, 256, 0, s, L, planes, P, x, xt, batch, y, yt);
  if (e == cudaSuccess) e = cudaGetLastError();
  *handled = (e == cudaSuccess);
  return e;
}

}  // namespace vqlin

extern "C" vqlin_status vqlin_selftest_wait_timeout(int32_t limit_us, void* stream) {
  using namespace vqlin;
  if (limit_us < 1 || limit_us > 1000000) { set_error("limit_us = %d: must be 1..1000000", limit_us); return VQLIN_ERR_INVALID_ARG; }
  note_launches(1);
  csg::k_wait_probe<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_us * 1000ull);
  return cuda_status(cudaGetLastError(), "self-test launch");
}
