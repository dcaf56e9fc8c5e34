// Prefill GEMM on the 5th-generation tensor cores:
//   Y[M][N] = A[M][K] * W[N][K]^T,  A = fp16 activations, W = the exact fp16
//   dequantised weight (VPTQ page, "The dequantization interface": the
//   dequantised weight feeds the prefill GEMM), fp32 accumulation in TMEM.
//
// One CTA computes a 128 x 256 tile of Y:
//   warp 0      TMA producer: A and W K-blocks (64 fp16 = one 128-byte swizzle
//               row) into a 4-stage shared-memory ring, completion on mbarriers;
//   warp 1      allocates 256 TMEM columns and, from one lane, issues
//               tcgen05.mma.kind::f16 (M=128, N=256, K=16) per K-step, returning
//               each ring slot with tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane TMEM quadrant, convert, store.
// Every mbarrier wait is bounded (1 s of %globaltimer): on expiry the kernel
// records an error code in vqlin_device_error, stops issuing work, waits (again
// bounded) for its own copies in flight, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "vqlin_internal.cuh"

namespace vqlin {

__device__ int g_device_error = 0;

namespace tc {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_BYTES = BN * BK * 2;       // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 256;
constexpr unsigned long long WAIT_NS = 1000000000ull;   // 1 s
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; false on timeout (and records the error).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int code) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  while (!mbar_try(bar, parity)) {
    if (now_ns() - t0 > WAIT_NS) {
      atomicExch(&g_device_error, code);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Shared-memory matrix descriptor, K-major operand in the 128-byte swizzle
// layout: 8-row atoms of 8 x 128 B, atoms 1024 B apart (stride byte offset);
// the leading byte offset is not used by this layout; version 1; layout 2.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor, kind::f16: D = f32 (bits 4-5 = 1), A = B = f16
// (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_w, int64_t M,
              int N, int K, void* __restrict__ Y, vqlin_dtype yt) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned ring (the 128-byte swizzle atoms need it)
  unsigned char* ring = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + (size_t)STAGES * STAGE_BYTES);
  // bars[0..S): full, bars[S..2S): empty, bars[2S]: accumulator ready
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int num_kb = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[STAGES + s]), 1);
    }
    mbar_init(smem_u32(&bars[2 * STAGES]), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_holder;
  int issued = 0;   // producer: K-blocks whose copies were issued

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
      if (*abort_flag || !mbar_wait(smem_u32(&bars[STAGES + s]), ph ^ 1u, 1)) { *abort_flag = 1; break; }
      const uint32_t full = smem_u32(&bars[s]);
      mbar_expect_tx(full, STAGE_BYTES);
      unsigned char* a = ring + (size_t)s * STAGE_BYTES;
      tma_load_2d(smem_u32(a), &map_a, full, kb * BK, (int)m0);
      tma_load_2d(smem_u32(a + A_BYTES), &map_w, full, kb * BK, n0);
      issued = kb + 1;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = idesc_f16(BM, BN);
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
      if (*abort_flag || !mbar_wait(smem_u32(&bars[s]), ph, 2)) { *abort_flag = 1; break; }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a = smem_u32(ring + (size_t)s * STAGE_BYTES);
      const uint64_t da = desc_sw128(a), db = desc_sw128(a + A_BYTES);
#pragma unroll
      for (int k = 0; k < BK / 16; ++k)   // 16 fp16 = 32 bytes per step along K inside the swizzle row
        mma_f16(tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc, (kb | k) != 0);
      mma_commit(smem_u32(&bars[STAGES + s]));
    }
    mma_commit(smem_u32(&bars[2 * STAGES]));
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int q = warp & 3;                        // TMEM lane quadrant this warp may access
    const int64_t row = m0 + q * 32 + lane;
    bool ok = mbar_wait(smem_u32(&bars[2 * STAGES]), 0, 3);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // tcgen05.ld is warp-wide: the whole warp reads, or none of it
    if (__all_sync(0xffffffffu, ok && !*abort_flag)) {
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, r);
        if (row < M) {
          const int nb = n0 + c;
          if (yt == VQLIN_F32) {
            float* yp = reinterpret_cast<float*>(Y) + row * N + nb;
            if (nb + 32 <= N && (N % 4) == 0) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(yp + j) = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                                 __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
            } else {
              for (int j = 0; j < 32; ++j) if (nb + j < N) yp[j] = __uint_as_float(r[j]);
            }
          } else {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float lo = __uint_as_float(r[2 * j]), hi = __uint_as_float(r[2 * j + 1]);
              if (yt == VQLIN_F16) {
                __half2 h = __floats2half2_rn(lo, hi);
                packed[j] = *reinterpret_cast<uint32_t*>(&h);
              } else {
                __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
                packed[j] = *reinterpret_cast<uint32_t*>(&h);
              }
            }
            unsigned short* yp = reinterpret_cast<unsigned short*>(Y) + row * N + nb;
            if (nb + 32 <= N && (N % 8) == 0) {
#pragma unroll
              for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<uint4*>(yp + 2 * j) = make_uint4(packed[j], packed[j + 1], packed[j + 2], packed[j + 3]);
            } else {
              for (int j = 0; j < 32; ++j)
                if (nb + j < N) yp[j] = (unsigned short)((packed[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
            }
          }
        }
      }
    }
  }
  // ---------------- teardown
  if (warp == 0 && lane == 0 && *abort_flag) {
    // let the copies this CTA issued land before its shared memory goes away
    for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
      mbar_wait(smem_u32(&bars[kb % STAGES]), (uint32_t)(kb / STAGES) & 1u, 4);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    // the MMAs must have finished with TMEM before it is released (the final
    // commit covers every MMA this CTA issued; a no-op wait on the normal path)
    if (lane == 0) mbar_wait(smem_u32(&bars[2 * STAGES]), 0, 5);
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}


// ---------------------------------------------------------------------------------------------
// Fused prefill GEMM: the weight tiles are dequantised in shared memory and fed to tcgen05.mma
// directly, so the fp16 weight is never written to global memory (VPTQ page, "The
// dequantization interface": dequantisation fused with the matrix multiplication, GEMM for
// prefill).  Layers: d = 8, one codebook (no residual stage), no outlier-column block.
//
// Orientation.  The MMA's M side is the weight: a CTA owns 128 weight rows (outputs) and 512
// activation rows, Y^T[128][512] = W_tile[128][K] * X_tile[512][K]^T, as two N = 256
// accumulators that fill the 512 TMEM columns.
//
// Sharing the weight tile.  The CS CTAs of a thread-block cluster (CS = 2 up to 1024 activation
// rows, 4 beyond) own the same 128 weight rows and different 512-row activation groups (a CTA past
// the last activation row still converts and shares its part).  Each converts only its 128 / CS
// rows of every weight K-block into its own slot, and its sparse warps copy them into the same
// slot of each peer (cp.async.bulk shared::cta -> shared::cluster, completing on the peer's slot
// barrier).  So every weight element is gathered and converted once per 512 * CS activation rows.
// A slot is rewritten only when every CTA's MMA has finished with it: the MMA returns a slot with
// one tcgen05.commit multicast to the slot's "cluster free" barrier in every CTA of the cluster.
//
// Warp roles (18 + 128 / (32 CS) warps):
//   warp 0      TMA producer of the activation tiles: 256 rows x 64 k (one 128-byte swizzle row
//               per activation row) into a 5-slot ring of half K-blocks;
//   warp 1      allocates the 512 TMEM columns; one lane issues tcgen05.mma.kind::f16 (M = 128,
//               N = 256, K = 16), four per half K-block, and returns ring slots with
//               tcgen05.commit;
//   sparse warps (one per 32 rows of this CTA's part) the sparse part: once the producers have
//               written a K-block of this CTA's rows, a lane per row writes the row's CSR values
//               and VSR blocks in that K-block over them (REPLACE); then one lane copies the warp's
//               rows to the peers and arrives on the slot's full barrier (the first sparse warp
//               also arms it for the peers' bytes);
//   16 warps    weight producers, then the epilogue.  The 512 lanes cover this CTA's 128 / CS rows
//               x 8 sub-vectors of a K-block (64 columns): a lane owns one sub-vector (CS = 2) or
//               half of one (CS = 4).  Three K-blocks ahead a lane gathers its part of the
//               centroid into registers (index fields loaded three steps before that).  For
//               K-block kb it converts it to the exact fp16 weight fp16(r_i c_j C[k][t]) (C r_i is
//               exact in fp32; the product with c_j is rounded to odd in fp32, so the final fp16
//               rounding is the correctly rounded one, as in the exact dequantisation) while the
//               slot may still be in use; once the slot is free it stores it to its
//               128-byte-swizzled place (chunk s ^ (row % 8) of the row's 128 bytes, the layout a
//               TMA 128B-swizzle load makes) and makes the writes visible to the async proxy
//               (fence.proxy.async).  The weight tile is therefore bit for bit the dequantised W.
// Every mbarrier wait is bounded (1 s); on expiry the kernel records an error code, stops,
// waits (bounded) for its own TMA loads, frees TMEM and returns.  Every thread reaches the
// cluster barriers at start and end.
constexpr int FA_STAGES = 4, FB_STAGES = 5;
constexpr int FA_BYTES = 128 * 64 * 2;             // 16 KB weight slot
constexpr int FB_BYTES = 256 * 64 * 2;             // 32 KB activation half-slot
constexpr int F_PROD_WARPS = 16;
// threads of the kernel for a cluster of cs CTAs: TMA, MMA, 4 / cs sparse warps, the producers
__host__ __device__ constexpr int f_threads(int cs) { return (2 + 4 / cs + F_PROD_WARPS) * 32; }
constexpr int F_ROWS = 128, F_XROWS = 512;
constexpr size_t F_SMEM_BYTES = 1024 + (size_t)FA_STAGES * FA_BYTES + (size_t)FB_STAGES * FB_BYTES + 256;

// fp32 product rounded to odd: toward zero, last bit forced to 1 when inexact (the exact error
// comes from a fused multiply-add).  Rounding that to fp16 gives the correctly rounded product.
__device__ __forceinline__ float rto_mul_f32(float a, float b) {
  float p = __fmul_rz(a, b);
  const float err = fmaf(a, b, -p);
  if (err != 0.f) p = __int_as_float(__float_as_int(p) | 1);
  return p;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// this CTA's shared address as seen in cluster CTA `rank`
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}


// The index field of sub-vector s of one packed row (W = 8, 16, 32: one aligned load; W = 0: any
// width).
template <int W>
__device__ __forceinline__ uint32_t load_field(const uint8_t* row, int s, int w) {
  if constexpr (W == 8) return __ldg(row + s);
  else if constexpr (W == 16) return __ldg(reinterpret_cast<const unsigned short*>(row) + s);
  else if constexpr (W == 32) return __ldg(reinterpret_cast<const uint32_t*>(row) + s);
  else return read_field(row, s, w);
}

template <int W, int CS>
__global__ void __launch_bounds__(f_threads(CS), 1)
    k_gemm_vq(const __grid_constant__ CUtensorMap map_x, const Layer L, int64_t M, void* __restrict__ Y,
              vqlin_dtype yt) {
  static_assert(CS == 2 || CS == 4, "a cluster of 2 or 4 CTAs");
  constexpr int RP = F_ROWS / CS;                    // weight rows this CTA converts
  constexpr int HS = CS / 2;                         // lanes per sub-vector
  constexpr int NW = 4 / HS;                         // 32-bit words (fp16 pairs) per lane
  constexpr int RPW = RP / F_PROD_WARPS;             // rows per producer warp
  constexpr int LPR = 32 / RPW;                      // lanes per row
  constexpr int NSP = RP / 32;                       // sparse warps, a row per lane
  constexpr int PW0 = 2 + NSP;                       // first producer warp
  constexpr uint32_t PART_BYTES = RP * 128;          // this CTA's rows of a slot
  static_assert(LPR == 8 * HS && NSP >= 1, "lane map");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring_a = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring_b = ring_a + (size_t)FA_STAGES * FA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring_b + (size_t)FB_STAGES * FB_BYTES);
  uint64_t* a_full = bars;                          // [FA_STAGES] the sparse warps' arrivals + peers' bytes
  uint64_t* a_free = bars + FA_STAGES;              // [FA_STAGES] the MMA commit of every cluster CTA
  uint64_t* own_full = bars + 2 * FA_STAGES;        // [FA_STAGES] this CTA's producer warps
  uint64_t* b_full = bars + 3 * FA_STAGES;          // [FB_STAGES] TMA transaction bytes
  uint64_t* b_empty = b_full + FB_STAGES;           // [FB_STAGES] one commit
  uint64_t* acc_bar = b_empty + FB_STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.y * F_ROWS;               // weight rows of the cluster
  const int64_t m0 = (int64_t)blockIdx.x * F_XROWS;
  const uint32_t crank = cluster_rank();
  const int K = L.n_in;
  const int num_kb = (K + 63) / 64;
  const int halves = M - m0 > 256 ? 2 : (M - m0 > 0 ? 1 : 0);   // activation half-tiles of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < FA_STAGES; ++s) {
      mbar_init(smem_u32(&a_full[s]), NSP);
      mbar_init(smem_u32(&a_free[s]), CS);
      mbar_init(smem_u32(&own_full[s]), F_PROD_WARPS);
    }
    for (int s = 0; s < FB_STAGES; ++s) {
      mbar_init(smem_u32(&b_full[s]), 1);
      mbar_init(smem_u32(&b_empty[s]), 1);
    }
    mbar_init(smem_u32(acc_bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  cluster_sync();                                  // every peer's barriers exist before any remote use
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_holder;
  const int total_h = num_kb * halves;
  int issued_b = 0;

  if (warp == 0 && lane == 0) {
    // ---------------- activation tiles (TMA)
    for (int hk = 0; hk < total_h; ++hk) {
      const int s = hk % FB_STAGES;
      const uint32_t ph = (uint32_t)(hk / FB_STAGES) & 1u;
      if (*abort_flag || !mbar_wait(smem_u32(&b_empty[s]), ph ^ 1u, 1)) { *abort_flag = 1; break; }
      const uint32_t full = smem_u32(&b_full[s]);
      mbar_expect_tx(full, FB_BYTES);
      const int kb = hk / halves, h = hk - kb * halves;
      tma_load_2d(smem_u32(ring_b + (size_t)s * FB_BYTES), &map_x, full, kb * 64, (int)(m0 + h * 256));
      issued_b = hk + 1;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer (a CTA without activation rows still returns every slot)
    constexpr uint32_t idesc = idesc_f16(128, 256);
    int hk = 0;
    for (int kb = 0; kb < num_kb && !*abort_flag; ++kb) {
      const int sa = kb % FA_STAGES;
      if (!mbar_wait(smem_u32(&a_full[sa]), (uint32_t)(kb / FA_STAGES) & 1u, 2)) { *abort_flag = 1; break; }
      const uint64_t da = desc_sw128(smem_u32(ring_a + (size_t)sa * FA_BYTES));
      for (int h = 0; h < halves; ++h, ++hk) {
        const int sb = hk % FB_STAGES;
        if (!mbar_wait(smem_u32(&b_full[sb]), (uint32_t)(hk / FB_STAGES) & 1u, 2)) { *abort_flag = 1; break; }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint64_t db = desc_sw128(smem_u32(ring_b + (size_t)sb * FB_BYTES));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_f16(tmem + (uint32_t)(h * 256), da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc, (kb | k) != 0);
        mma_commit(smem_u32(&b_empty[sb]));
      }
      if (*abort_flag) break;
      // the slot is free here once this MMA group completes: tell every CTA of the cluster
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
          ::"r"(smem_u32(&a_free[sa])), "h"((uint16_t)((1u << CS) - 1u)) : "memory");
    }
    mma_commit(smem_u32(acc_bar));
  } else if (warp >= 2 && warp < PW0) {
    // ---------------- sparse part and copies: lane l of sparse warp sw owns row
    // crank * RP + 32 sw + l of the tile.  The row's CSR entries come by K-block: the start and end
    // of K-block x four steps ahead, up to four of its entries (column in the block, value) two
    // steps ahead, so the K-block's work is a few stores; more than four entries in one row and
    // K-block (rare) are loaded on the spot.  The VSR blocks come two ahead.
    const int sw = warp - 2;
    const int rt = (int)crank * RP + sw * 32 + lane;
    const int64_t row = (int64_t)n0 + rt;
    const bool row_ok = row < L.n_out;
    const bool has_csr = L.nnz > 0 && row_ok;
    const int32_t* kbs = has_csr ? L.kb_start + row * (num_kb + 1) : nullptr;
    const uint32_t* kbe = L.kb_entry;
    const uint32_t slot_row = (uint32_t)rt * 128u, rsw = (uint32_t)(rt & 7);
    int vb = 0, vb_end = 0;                          // VSR cursor, two blocks ahead
    if (L.vsr_nb > 0 && row_ok) { vb = L.vsr_rp[row]; vb_end = L.vsr_rp[row + 1]; }
    const uint4* vsr4 = reinterpret_cast<const uint4*>(L.vsr_val);
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    int s0 = vb < vb_end ? L.vsr_pos[vb] : 0x7FFFFFFF;
    uint4 b0 = vb < vb_end ? __ldg(vsr4 + vb) : z4;
    ++vb;
    int s1 = vb < vb_end ? L.vsr_pos[vb] : 0x7FFFFFFF;
    uint4 b1 = vb < vb_end ? __ldg(vsr4 + vb) : z4;
    ++vb;
    struct Ent { uint32_t e[4]; int s, n; };
    auto load_t = [&](int x, int2& t) {
      if (has_csr) { x = min(x, num_kb - 1); t.x = __ldg(kbs + x); t.y = __ldg(kbs + x + 1); }
      else t = make_int2(0, 0);
    };
    auto load_e = [&](const int2& t, Ent& en) {
      en.s = t.x;
      en.n = t.y - t.x;
      if (en.n > 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) en.e[i] = __ldg(kbe + t.x + i);   // inside the 16 bytes of padding
      }
    };
    auto put = [&](uint32_t slot, uint32_t ent) {
      const uint32_t k = ent >> 16;                   // column inside the K-block
      const uint32_t adr = slot + ((((k >> 3) ^ rsw) << 4) | ((k & 7u) << 1));
      asm volatile("st.shared.u16 [%0], %1;" ::"r"(adr), "h"((uint16_t)(ent & 0xFFFFu)) : "memory");
    };
    bool ok = true;
    // K-block kb: the stores once the producers are done, then the copies; T and E rotate as in
    // the producers (array i holds K-blocks congruent to i mod 4)
    auto sstep = [&](int kb, int2& t_load, const int2& t_use, Ent& e_load, const Ent& e_cur) {
      const int sa = kb % FA_STAGES;
      const bool mine = !*abort_flag && mbar_wait(smem_u32(&own_full[sa]), (uint32_t)(kb / FA_STAGES) & 1u, 6);
      if (!__all_sync(0xffffffffu, mine)) { *abort_flag = 1; ok = false; return; }
      const uint32_t slot0 = smem_u32(ring_a + (size_t)sa * FA_BYTES);
      const uint32_t slot = slot0 + slot_row;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i < e_cur.n) put(slot, e_cur.e[i]);
      for (int i = 4; i < e_cur.n; ++i) put(slot, __ldg(kbe + e_cur.s + i));
      while (s0 < (kb + 1) * 8) {
        const uint32_t adr = slot + (((uint32_t)(s0 - kb * 8) ^ rsw) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(adr), "r"(b0.x), "r"(b0.y), "r"(b0.z),
                     "r"(b0.w)
                     : "memory");
        s0 = s1;
        b0 = b1;
        s1 = vb < vb_end ? L.vsr_pos[vb] : 0x7FFFFFFF;
        b1 = vb < vb_end ? __ldg(vsr4 + vb) : z4;
        ++vb;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        // the warp's rows of the K-block are complete: copy them into every peer's slot
        const uint32_t full = smem_u32(&a_full[sa]);
        const uint32_t part = slot0 + (uint32_t)(crank * RP + sw * 32) * 128u;
#pragma unroll
        for (int q = 1; q < CS; ++q) {
          const uint32_t peer = (crank + (uint32_t)q) % CS;
          asm volatile(
              "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
              ::"r"(peer_addr(part, peer)), "r"(part), "r"(32u * 128u), "r"(peer_addr(full, peer))
              : "memory");
        }
        if (sw == 0) mbar_expect_tx(full, (CS - 1) * PART_BYTES);   // the peers' rows are due
        else asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(full) : "memory");
      }
      load_e(t_use, e_load);
      load_t(kb + 4, t_load);
    };
    int2 T0, T1, T2, T3;
    Ent E0, E1, E2, E3;
    load_t(0, T0); load_t(1, T1); load_t(2, T2); load_t(3, T3);
    load_e(T0, E0); load_e(T1, E1);
    E2.n = E3.n = 0;
    for (int kb = 0; kb < num_kb && ok; kb += 4) {
      sstep(kb, T0, T2, E2, E0);
      if (!ok || kb + 1 >= num_kb) break;
      sstep(kb + 1, T1, T3, E3, E1);
      if (!ok || kb + 2 >= num_kb) break;
      sstep(kb + 2, T2, T0, E0, E2);
      if (!ok || kb + 3 >= num_kb) break;
      sstep(kb + 3, T3, T1, E1, E3);
    }
  } else if (warp >= PW0) {
    // ---------------- weight producers
    const int pw = warp - PW0;
    const int it = lane % LPR;                        // item of the row: sub-vector it / HS, part it % HS
    const int svl = it / HS, hp = it % HS;
    const int r = (int)crank * RP + pw * RPW + lane / LPR;   // row inside the 128-row tile
    const int64_t row = (int64_t)n0 + r;
    const bool row_ok = row < L.n_out;
    const uint8_t* codes_row = L.codes + (row_ok ? row : 0) * L.stride;
    const uint32_t m1 = (1u << L.bits1) - 1u;
    const float rsc = (L.rs && row_ok) ? __half2float(L.rs[row]) : 1.f;
    const bool has_cs = L.cs != nullptr;
    const uint32_t rsw = (uint32_t)(r & 7);
    const uint32_t* cb1w = reinterpret_cast<const uint32_t*>(L.cb1);
    const int last_kb = num_kb - 1;
    // Every global load is issued ahead of its use and unconditionally (K-block indices past the
    // last are clamped; values for sub-vectors past the last are never used): index fields three
    // steps before their gathers, centroids and column scales three K-blocks before their
    // conversion.
    auto load_f = [&](int kb) -> uint32_t {
      return load_field<W>(codes_row, min(min(kb, last_kb) * 8 + svl, L.n_sub - 1), L.w);
    };
    auto load_cs = [&](int kb, uint32_t* c) {
      // the 8 / HS column scales of the lane's part (clamped into the vector: unused past n_in)
      const int col = min(min(kb, last_kb) * 64 + svl * 8 + hp * (8 / HS), K - 8 / HS);
      if constexpr (NW == 4) {
        const uint4 t = has_cs ? __ldg(reinterpret_cast<const uint4*>(L.cs + col)) : make_uint4(0, 0, 0, 0);
        c[0] = t.x; c[1] = t.y; c[2] = t.z; c[3] = t.w;
      } else {
        const uint2 t = has_cs ? __ldg(reinterpret_cast<const uint2*>(L.cs + col)) : make_uint2(0, 0);
        c[0] = t.x; c[1] = t.y;
      }
    };
    auto gather = [&](int kb, uint32_t f, uint32_t* g) {
      const int sv = min(min(kb, last_kb) * 8 + svl, L.n_sub - 1);
      const uint32_t* p = cb1w + ((size_t)((uint32_t)group_of(L, sv) * (uint32_t)L.k1 + (f & m1)) * 4 + hp * NW);
      if constexpr (NW == 4) {
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(g[0]), "=r"(g[1]), "=r"(g[2]), "=r"(g[3]) : "l"(p));
      } else {
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(g[0]), "=r"(g[1]) : "l"(p));
      }
    };
    bool ok = true;
    // One pipeline step for K-block kb: the loads for later K-blocks; the conversion of kb into
    // registers; then, once every CTA's MMA is done with kb's slot, the store and the arrival for
    // the sparse warp.  The callers rotate fixed register arrays through the roles, so no value in
    // flight is ever copied.
    auto step = [&](int kb, const uint32_t* g_cur, uint32_t* g_next, uint32_t f_next, uint32_t& f_load,
                    const uint32_t* c_cur, uint32_t* c_load) {
      f_load = load_f(kb + 6);
      load_cs(kb + 3, c_load);
      gather(kb + 3, f_next, g_next);
      uint32_t w[NW];
      const bool valid = row_ok && kb * 8 + svl < L.n_sub;
#pragma unroll
      for (int q = 0; q < NW; ++q) {
        const __half2 h2 = *reinterpret_cast<const __half2*>(&g_cur[q]);
        float a0 = __low2float(h2) * rsc, a1 = __high2float(h2) * rsc;   // exact
        if (has_cs) {
          const __half2 c2 = *reinterpret_cast<const __half2*>(&c_cur[q]);
          a0 = rto_mul_f32(a0, __low2float(c2));
          a1 = rto_mul_f32(a1, __high2float(c2));
        }
        const __half2 o = __floats2half2_rn(a0, a1);
        w[q] = valid ? *reinterpret_cast<const uint32_t*>(&o) : 0u;
      }
      // the slot is free once every CTA's MMA is done with its previous K-block
      const int sa = kb % FA_STAGES;
      const bool mine = !*abort_flag && mbar_wait(smem_u32(&a_free[sa]), ((uint32_t)(kb / FA_STAGES) & 1u) ^ 1u, 3);
      if (!__all_sync(0xffffffffu, mine)) { *abort_flag = 1; ok = false; return; }
      const uint32_t adr = smem_u32(ring_a + (size_t)sa * FA_BYTES) + (uint32_t)r * 128u +
                           ((((uint32_t)svl ^ rsw) << 4) | (uint32_t)(hp * 8));
      if constexpr (NW == 4)
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(adr), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                     "r"(w[3])
                     : "memory");
      else
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(adr), "r"(w[0]), "r"(w[1]) : "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&own_full[sa])) : "memory");
    };
    // Array X_i holds the values of K-blocks congruent to i mod 4.
    uint32_t G0[NW], G1[NW], G2[NW], G3[NW];          // centroid parts in flight
    uint32_t F0, F1, F2, F3;                           // index fields
    uint32_t C0[NW], C1[NW], C2[NW], C3[NW];          // column scales
    F0 = load_f(0); F1 = load_f(1); F2 = load_f(2); F3 = load_f(3);
    gather(0, F0, G0); gather(1, F1, G1); gather(2, F2, G2);
    F0 = load_f(4); F1 = load_f(5);
    load_cs(0, C0); load_cs(1, C1); load_cs(2, C2);
    for (int kb = 0; kb < num_kb && ok; kb += 4) {
      step(kb, G0, G3, F3, F2, C0, C3);
      if (!ok || kb + 1 >= num_kb) break;
      step(kb + 1, G1, G0, F0, F3, C1, C0);
      if (!ok || kb + 2 >= num_kb) break;
      step(kb + 2, G2, G1, F1, F0, C2, C1);
      if (!ok || kb + 3 >= num_kb) break;
      step(kb + 3, G3, G2, F2, F1, C3, C2);
    }
    // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31; the four warps of
    // group (w - PW0) / 4 read 128 columns of accumulator ((w - PW0) / 4) / 2
    const int q = warp & 3, part = (warp - PW0) >> 2, half = part >> 1, c0 = (part & 1) * 128;
    const bool done = mbar_wait(smem_u32(acc_bar), 0, 4);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // the decision is the same for all 16 producer warps (tcgen05.ld is warp-wide, and the
    // 16-bit path below has a barrier among them)
    uint32_t go;
    asm volatile(
        "{\n .reg .pred p, r;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred r, 1, %2, p;\n selp.u32 %0, 1, 0, r;\n}"
        : "=r"(go) : "r"((uint32_t)(done && !*abort_flag)), "n"(F_PROD_WARPS * 32) : "memory");
    if (go && yt == VQLIN_F32) {
      if (half < halves) {
        const int64_t i = (int64_t)n0 + q * 32 + lane;
        const bool i_ok = i < L.n_out;
#pragma unroll 1
        for (int c = c0; c < c0 + 128; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 256 + c), v);
          const int64_t mb = m0 + half * 256 + c;
          if (!i_ok) continue;
#pragma unroll
          for (int jx = 0; jx < 32; ++jx) {
            const int64_t m = mb + jx;
            if (m < M) reinterpret_cast<float*>(Y)[m * L.n_out + i] = __uint_as_float(v[jx]);
          }
        }
      }
    } else if (go) {
      // 16-bit outputs: stage the CTA's 512 x 128 tile of Y in the activation ring (every MMA has
      // completed, so it is free), Y-major, then write whole 256-byte row segments of Y
      static_assert((size_t)FB_STAGES * FB_BYTES >= 512 * 128 * 2, "the output tile fits the activation ring");
      unsigned short* stage = reinterpret_cast<unsigned short*>(ring_b);   // [512][128]
      const bool f16 = yt == VQLIN_F16;
      if (half < halves) {
#pragma unroll 1
        for (int c = c0; c < c0 + 128; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 256 + c), v);
          unsigned short* sp = stage + (size_t)(half * 256 + c) * 128 + q * 32 + lane;
#pragma unroll
          for (int jx = 0; jx < 32; ++jx) {
            const float f = __uint_as_float(v[jx]);
            sp[jx * 128] = f16 ? __half_as_ushort(__float2half_rn(f)) : __bfloat16_as_ushort(__float2bfloat16_rn(f));
          }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(F_PROD_WARPS * 32) : "memory");
      const int p = pw * 32 + lane, ch = p & 15;       // 16 threads per row of the tile, 8 columns each
      const int64_t i0 = (int64_t)n0 + ch * 8;
      const bool vec = i0 + 8 <= L.n_out && (L.n_out & 7) == 0 && (reinterpret_cast<uintptr_t>(Y) & 15) == 0;
#pragma unroll 4
      for (int ml = p >> 4; ml < 512; ml += 32) {
        const int64_t m = m0 + ml;
        if (m >= M) break;
        const unsigned short* sp = stage + (size_t)ml * 128 + ch * 8;
        unsigned short* yp = reinterpret_cast<unsigned short*>(Y) + m * L.n_out + i0;
        if (vec) {
          *reinterpret_cast<uint4*>(yp) = *reinterpret_cast<const uint4*>(sp);
        } else {
          for (int t = 0; t < 8; ++t)
            if (i0 + t < L.n_out) yp[t] = sp[t];
        }
      }
    }
  }
  // ---------------- teardown
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int hk = (issued_b > FB_STAGES ? issued_b - FB_STAGES : 0); hk < issued_b; ++hk)
      mbar_wait(smem_u32(&b_full[hk % FB_STAGES]), (uint32_t)(hk / FB_STAGES) & 1u, 4);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(smem_u32(acc_bar), 0, 5);
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
  }
  // Every copy and slot release into this CTA was issued before its sender reached this barrier.
  // On the normal path each copy has landed (this CTA's MMA consumed every K-block); after an
  // abort give the ones still in flight (a few KB, microseconds) time to land before the CTA exits.
  __syncwarp();
  cluster_sync();
  if (*abort_flag) {
    const uint64_t t0 = now_ns();
    while (now_ns() - t0 < 100000ull) __nanosleep(1000);
  }
}

}  // namespace tc

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major [rows][cols] fp16 matrix as a 2-D tensor map with a box of
// box_rows x 64 columns, 128-byte swizzle, zero fill out of bounds.
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm_f16(const __half* A, const __half* W, int64_t M, int N, int K, void* Y, vqlin_dtype yt,
                            cudaStream_t s) {
  // TMA needs 16-byte aligned bases and row strides (K % 8 == 0, checked by the caller)
  if ((reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(W) & 15) || (K % 8) || M > 0x7FFFFFFF)
    return cudaErrorInvalidValue;
  CUtensorMap ma, mw;
  if (!make_map(&ma, A, (uint64_t)M, (uint64_t)K, tc::BM) || !make_map(&mw, W, (uint64_t)N, (uint64_t)K, tc::BN))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(tc::k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((N + tc::BN - 1) / tc::BN, (unsigned)((M + tc::BM - 1) / tc::BM));
  note_launches(1);
  tc::k_gemm_tc<<<grid, tc::THREADS, tc::SMEM_BYTES, s>>>(ma, mw, M, N, K, Y, yt);
  return cudaGetLastError();
}

bool gemm_fused_supported(const Layer& L) {
  return L.d == 8 && L.k2 == 0 && L.n_ocols == 0 && L.n_sub > 0 && (L.n_in % 8) == 0 && L.w <= 32;
}

template <int CS>
static cudaError_t launch_vq_cs(const Layer& L, const CUtensorMap& mx, int64_t M, void* Y, vqlin_dtype yt,
                                cudaStream_t s) {
  auto k = L.w == 8 ? tc::k_gemm_vq<8, CS> : L.w == 16 ? tc::k_gemm_vq<16, CS> : L.w == 32 ? tc::k_gemm_vq<32, CS>
                                                                                           : tc::k_gemm_vq<0, CS>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::F_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // activation groups on x (rounded up to whole clusters: a CTA past M only gathers and shares
  // its rows), weight tiles on y
  const int64_t groups = (M + tc::F_XROWS - 1) / tc::F_XROWS;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)((groups + CS - 1) / CS * CS), (unsigned)((L.n_out + tc::F_ROWS - 1) / tc::F_ROWS));
  cfg.blockDim = dim3(tc::f_threads(CS));
  cfg.dynamicSmemBytes = tc::F_SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launches(1);
  return cudaLaunchKernelEx(&cfg, k, mx, L, M, Y, yt);
}

cudaError_t launch_gemm_vq(const Layer& L, const __half* X, int64_t M, void* Y, vqlin_dtype yt, cudaStream_t s) {
  if (!gemm_fused_supported(L) || (reinterpret_cast<uintptr_t>(X) & 15) || M < 1 || M > 0x7FFFFFFF)
    return cudaErrorInvalidValue;
  CUtensorMap mx;
  if (!make_map(&mx, X, (uint64_t)M, (uint64_t)L.n_in, 256)) return cudaErrorInvalidValue;
  // A cluster shares each weight tile over four 512-row activation groups, or two up to 1024
  // activation rows (a CTA past the last row still converts and shares its part of the tile).
  const int64_t groups = (M + tc::F_XROWS - 1) / tc::F_XROWS;
  cudaError_t e = groups > 2 ? launch_vq_cs<4>(L, mx, M, Y, yt, s) : launch_vq_cs<2>(L, mx, M, Y, yt, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int read_and_clear_device_error() {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return -1;
  if (v) cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
  return v;
}

}  // namespace vqlin
