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
// accumulators that fill the 512 TMEM columns.  Each weight row is then gathered once per 512
// activation rows (the TMEM limit), not once per activation tile of a conventional tiling.
//
// Warp roles (10 warps):
//   warp 0      TMA producer of the activation tiles: 256 rows x 64 k (one 128-byte swizzle row
//               per activation row) into a 5-slot ring of half K-blocks;
//   warp 1      allocates the 512 TMEM columns; one lane issues tcgen05.mma.kind::f16 (M = 128,
//               N = 256, K = 16), four per half K-block, and returns ring slots with
//               tcgen05.commit;
//   warps 2-9   weight producers, then the epilogue.  Thread p owns weight row p % 128 and the
//               sub-vectors 4 (p / 128) .. +3 of every K-block (64 columns = 8 sub-vectors).
//               For K-block kb it reads its four index fields, copies the four centroids with
//               cp.async straight to their 128-byte-swizzled places in the weight slot (chunk
//               s ^ (row % 8) of the row's 128 bytes, the layout a TMA 128B-swizzle load makes),
//               and, once they have landed, converts them in place to the exact fp16 weight
//               fp16(r_i c_j C[k][t]) (C r_i is exact in fp32; the product with c_j is rounded to
//               odd in fp32, so the final fp16 rounding is the correctly rounded one, as in the
//               exact dequantisation), writes the CSR values of its columns over them (REPLACE),
//               makes the writes visible to the tensor core (fence.proxy.async) and arrives on
//               the slot's barrier.  The weight tile is therefore bit for bit the dequantised W.
// Every mbarrier wait is bounded (1 s); on expiry the kernel records an error code, stops,
// waits (bounded) for its own copies, frees TMEM and returns.
constexpr int FA_STAGES = 4, FB_STAGES = 5;
constexpr int FA_BYTES = 128 * 64 * 2;             // 16 KB weight slot
constexpr int FB_BYTES = 256 * 64 * 2;             // 32 KB activation half-slot
constexpr int F_PROD_WARPS = 8;
constexpr int F_THREADS = (2 + F_PROD_WARPS) * 32;
constexpr int F_LOOKAHEAD = FA_STAGES - 1;         // K-blocks of gathers in flight per thread
constexpr int F_ROWS = 128, F_XROWS = 512;
constexpr size_t F_SMEM_BYTES = 1024 + (size_t)FA_STAGES * FA_BYTES + (size_t)FB_STAGES * FB_BYTES + 256;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// fp32 product rounded to odd: toward zero, last bit forced to 1 when inexact (the exact error
// comes from a fused multiply-add).  Rounding that to fp16 gives the correctly rounded product.
__device__ __forceinline__ float rto_mul_f32(float a, float b) {
  float p = __fmul_rz(a, b);
  const float err = fmaf(a, b, -p);
  if (err != 0.f) p = __int_as_float(__float_as_int(p) | 1);
  return p;
}

// The four index fields of sub-vectors kb*8 + 4*hs .. +3 of one packed row: they occupy the w/2
// bytes at byte kb*w + hs*w/2 (eight fields of a K-block are w bytes).  One vector load for
// W = 8, 16, 32; three 32-bit loads of the K-block's w bytes for W = 12, 24; field by field
// otherwise (W = 0: any width).
template <int W>
__device__ __forceinline__ void load_fields4(const uint8_t* row, int kb, int hs, int w, uint32_t* f) {
  if constexpr (W == 8) {
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(row + kb * 8 + hs * 4));
#pragma unroll
    for (int u = 0; u < 4; ++u) f[u] = (v >> (8 * u)) & 0xFFu;
  } else if constexpr (W == 16) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(row + kb * 16 + hs * 8));
    f[0] = v.x & 0xFFFFu; f[1] = v.x >> 16; f[2] = v.y & 0xFFFFu; f[3] = v.y >> 16;
  } else if constexpr (W == 32) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + kb * 32 + hs * 16));
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  } else if constexpr (W == 12 || W == 24) {
    // W = 12: the K-block's 12 bytes (fields at bits 12 (4 hs + u)); W = 24: this half's 12 bytes
    // (fields at bits 24 u); either way three 4-byte-aligned words
    const uint32_t* p = reinterpret_cast<const uint32_t*>(row + kb * W + (W == 24 ? hs * 12 : 0));
    const uint32_t a = __ldg(p), b = __ldg(p + 1), c = __ldg(p + 2);
    const unsigned long long lo = (unsigned long long)a | ((unsigned long long)b << 32);
    const unsigned long long hi = (unsigned long long)b | ((unsigned long long)c << 32);
    constexpr uint32_t mask = (1u << W) - 1u;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int bit = (W == 12 ? 4 * hs + u : u) * W;
      f[u] = (uint32_t)((bit <= 64 - W ? (lo >> bit) : (hi >> (bit - 32))) & mask);
    }
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) f[u] = read_field(row, (int64_t)kb * 8 + 4 * hs + u, w);
  }
}

template <int W>
__global__ void __launch_bounds__(F_THREADS, 1)
    k_gemm_vq(const __grid_constant__ CUtensorMap map_x, const Layer L, int64_t M, void* __restrict__ Y,
              vqlin_dtype yt) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring_a = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring_b = ring_a + (size_t)FA_STAGES * FA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring_b + (size_t)FB_STAGES * FB_BYTES);
  uint64_t* a_full = bars;                          // [FA_STAGES], 8 producer-warp arrivals
  uint64_t* a_empty = bars + FA_STAGES;             // [FA_STAGES], one commit
  uint64_t* b_full = bars + 2 * FA_STAGES;          // [FB_STAGES], TMA transaction bytes
  uint64_t* b_empty = b_full + FB_STAGES;           // [FB_STAGES], one commit
  uint64_t* acc_bar = b_empty + FB_STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * F_ROWS;
  const int64_t m0 = (int64_t)blockIdx.y * F_XROWS;
  const int K = L.n_in;
  const int num_kb = (K + 63) / 64;
  const int halves = (M - m0) > 256 ? 2 : 1;        // activation half-tiles of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < FA_STAGES; ++s) {
      mbar_init(smem_u32(&a_full[s]), F_PROD_WARPS);
      mbar_init(smem_u32(&a_empty[s]), 1);
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
    // ---------------- MMA issuer
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
      mma_commit(smem_u32(&a_empty[sa]));
    }
    mma_commit(smem_u32(acc_bar));
  } else if (warp >= 2) {
    // ---------------- weight producers
    const int p = threadIdx.x - 64;
    const int r = p & (F_ROWS - 1), hs = p >> 7;
    const int64_t row = (int64_t)n0 + r;
    const bool row_ok = row < L.n_out;
    const uint8_t* codes_row = L.codes + (row_ok ? row : 0) * L.stride;
    const uint32_t m1 = (1u << L.bits1) - 1u;
    const float rsc = (L.rs && row_ok) ? __half2float(L.rs[row]) : 1.f;
    const bool has_cs = L.cs != nullptr;
    int e = 0, e_end = 0;                              // this row's CSR entries not yet placed
    if (L.nnz > 0 && row_ok) { e = L.row_ptr[row]; e_end = L.row_ptr[row + 1]; }
    const uint32_t rsw = (uint32_t)(r & 7);
    int next_j = e < e_end ? L.col[e] : 0x7FFFFFFF;     // column of the next CSR entry (prefetched)
    int vb = 0, vb_end = 0;                             // this row's VSR blocks not yet placed
    if (L.vsr_nb > 0 && row_ok) { vb = L.vsr_rp[row]; vb_end = L.vsr_rp[row + 1]; }
    int next_s = vb < vb_end ? L.vsr_pos[vb] : 0x7FFFFFFF;   // sub-vector of the next VSR block
    // issue the gathers of K-block kb into its slot (the slot must have been released by the MMA);
    // false if the wait gave up (the whole warp then leaves together)
    auto issue = [&](int kb) -> bool {
      const int sa = kb % FA_STAGES;
      const bool mine = !*abort_flag && mbar_wait(smem_u32(&a_empty[sa]), ((uint32_t)(kb / FA_STAGES) & 1u) ^ 1u, 3);
      if (!__all_sync(0xffffffffu, mine)) { *abort_flag = 1; return false; }
      const uint32_t slot = smem_u32(ring_a + (size_t)sa * FA_BYTES) + (uint32_t)r * 128u;
      uint32_t fl[4];
      if (row_ok) load_fields4<W>(codes_row, kb, hs, L.w, fl);   // the row's stride pads it past the last field
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int sl = 4 * hs + u, sv = kb * 8 + sl;
        const uint32_t dst = slot + (((uint32_t)sl ^ rsw) << 4);
        if (row_ok && sv < L.n_sub) {
          const uint32_t f = (uint32_t)group_of(L, sv) * (uint32_t)L.k1 + (fl[u] & m1);
          cp_async16(dst, reinterpret_cast<const uint4*>(L.cb1) + f);
        } else {
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
        }
      }
      return true;
    };
    bool ok = true;
    // K-blocks 0 .. F_LOOKAHEAD - 1 first: their slots are free from the start
    for (int kb = 0; kb < F_LOOKAHEAD; ++kb) {
      if (ok && kb < num_kb) ok = issue(kb);
      cp_async_commit();                                  // one group per K-block (possibly empty)
    }
    for (int kb = 0; kb < num_kb && ok; ++kb) {
      // convert K-block kb in place as soon as this thread's copies have landed, so the MMA can
      // take it while the gathers of the next K-blocks are still in flight
      cp_async_wait<F_LOOKAHEAD - 1>();
      const int sa = kb % FA_STAGES;
      const uint32_t slot = smem_u32(ring_a + (size_t)sa * FA_BYTES) + (uint32_t)r * 128u;
      const int col0 = kb * 64 + hs * 32;                 // first column of this thread's 4 sub-vectors
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int sl = 4 * hs + u, sv = kb * 8 + sl;
        if (!row_ok || sv >= L.n_sub) continue;
        const uint32_t adr = slot + (((uint32_t)sl ^ rsw) << 4);
        uint32_t w4[4];
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3]) : "r"(adr));
        float cj[8];
        if (has_cs) {
          const uint4 cu = __ldg(reinterpret_cast<const uint4*>(L.cs + col0 + u * 8));
          const __half* ch = reinterpret_cast<const __half*>(&cu);
#pragma unroll
          for (int t = 0; t < 8; ++t) cj[t] = __half2float(ch[t]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __half2 h2 = *reinterpret_cast<const __half2*>(&w4[q]);
          float a0 = __low2float(h2) * rsc, a1 = __high2float(h2) * rsc;   // exact
          if (has_cs) { a0 = rto_mul_f32(a0, cj[2 * q]); a1 = rto_mul_f32(a1, cj[2 * q + 1]); }
          w4[q] = (uint32_t)__half_as_ushort(__float2half_rn(a0)) |
                  ((uint32_t)__half_as_ushort(__float2half_rn(a1)) << 16);
        }
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(adr), "r"(w4[0]), "r"(w4[1]), "r"(w4[2]),
                     "r"(w4[3])
                     : "memory");
      }
      // sparse positions of this row inside the thread's 32 columns take the stored value
      while (next_j < col0 + 32) {
        if (next_j >= col0) {
          const int k = next_j - kb * 64;                 // column inside the K-block
          const uint32_t adr = slot + ((((uint32_t)k >> 3) ^ rsw) << 4) + (((uint32_t)k & 7u) << 1);
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(adr), "h"(L.val[e]) : "memory");
        }
        ++e;
        next_j = e < e_end ? L.col[e] : 0x7FFFFFFF;
      }
      // VSR blocks of this row among the thread's 4 sub-vectors replace them whole (16 bytes)
      while (next_s < kb * 8 + 4 * hs + 4) {
        if (next_s >= kb * 8 + 4 * hs) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(L.vsr_val) + vb);
          const uint32_t adr = slot + (((uint32_t)(next_s - kb * 8) ^ rsw) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(adr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                       : "memory");
        }
        ++vb;
        next_s = vb < vb_end ? L.vsr_pos[vb] : 0x7FFFFFFF;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&a_full[sa])) : "memory");
      // then refill: the gathers of K-block kb + F_LOOKAHEAD go to the slot of K-block kb - 1
      if (kb + F_LOOKAHEAD < num_kb) ok = issue(kb + F_LOOKAHEAD);
      cp_async_commit();
    }
    cp_async_wait<0>();                                   // nothing of ours may land after exit
    // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31, accumulator (w - 2) / 4
    const int q = warp & 3, half = (warp - 2) >> 2;
    const bool done = mbar_wait(smem_u32(acc_bar), 0, 4);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // tcgen05.ld is warp-wide: the whole warp reads, or none of it
    if (__all_sync(0xffffffffu, done && !*abort_flag) && half < halves) {
      const int64_t i = (int64_t)n0 + q * 32 + lane;
      const bool i_ok = i < L.n_out;
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 256 + c), v);
        const int64_t mb = m0 + half * 256 + c;
        if (!i_ok) continue;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int64_t m = mb + j;
          if (m < M) store_from_float(Y, yt, m * L.n_out + i, __uint_as_float(v[j]));
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

cudaError_t launch_gemm_vq(const Layer& L, const __half* X, int64_t M, void* Y, vqlin_dtype yt, cudaStream_t s) {
  if (!gemm_fused_supported(L) || (reinterpret_cast<uintptr_t>(X) & 15) || M < 1 || M > 0x7FFFFFFF)
    return cudaErrorInvalidValue;
  CUtensorMap mx;
  if (!make_map(&mx, X, (uint64_t)M, (uint64_t)L.n_in, 256)) return cudaErrorInvalidValue;
  auto k = L.w == 8 ? tc::k_gemm_vq<8> : L.w == 12 ? tc::k_gemm_vq<12> : L.w == 16 ? tc::k_gemm_vq<16>
         : L.w == 24 ? tc::k_gemm_vq<24> : L.w == 32 ? tc::k_gemm_vq<32> : tc::k_gemm_vq<0>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::F_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((L.n_out + tc::F_ROWS - 1) / tc::F_ROWS, (unsigned)((M + tc::F_XROWS - 1) / tc::F_XROWS));
  note_launches(1);
  k<<<grid, tc::F_THREADS, tc::F_SMEM_BYTES, s>>>(mx, L, M, Y, yt);
  return cudaGetLastError();
}

int read_and_clear_device_error() {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return -1;
  if (v) cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
  return v;
}

}  // namespace vqlin
