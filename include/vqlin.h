/*
 * vqlin.h — C ABI of libvqlin, a linear layer that runs directly on
 * vector-quantised (VQ) weights with a sparse outlier correction, for
 * NVIDIA B200 (sm_100a).
 *
 * What one layer computes
 * -----------------------
 * The weight W is n_out x n_in (row = output feature, the usual Linear
 * layout).  It is never stored densely.  Instead:
 *
 *   - the columns of W are split into the "main" columns and an optional,
 *     caller-chosen set of "outlier columns" (VPTQ: Extreme Low-bit Vector
 *     Post-Training Quantization for Large Language Models, section
 *     "Outlier Elimination": a separate codebook for a few percent of the
 *     columns, decoded through a static branch);
 *   - each row's main columns, taken in increasing column order, are cut into
 *     sub-vectors of d consecutive elements; sub-vector s of row i is the
 *     codebook entry C1[i1] (plus C2[i2] when a residual codebook is given:
 *     VPTQ page, section "Residual Vector Quantization", "Decoding process");
 *   - each row's outlier columns, in increasing column order, are cut the same
 *     way and decoded with their own codebook Co;
 *   - every element is multiplied by a row scale r[i] and a column scale c[j]
 *     (SCVQ: Sparse-Compensated Vector Quantization for Large Language Models,
 *     summary, step 1 "bi-normalized across rows and columns"; the stored
 *     scales are multipliers at decode time);
 *   - a sparse CSR matrix S gives exact values for chosen positions:
 *     W[i,j] = v_ij for (i,j) in S (HAS-VQ: Hessian-Adaptive Sparse Vector
 *     Quantization for High-Fidelity LLM Compression, abstract: the sparse
 *     feedback makes outliers reconstruct exactly; SCVQ summary, step 4: one
 *     sparse correction matrix).  Positions in S take precedence over the
 *     outlier block, which takes precedence over the main body.
 *
 *   So, for (i,j) not in S:
 *     W[i,j] = r[i] * c[j] * Co[io(i, p/d)][p % d]                 if j is the p-th outlier column
 *     W[i,j] = r[i] * c[j] * (C1[i1(i,q/d)] + C2[i2(i,q/d)])[q % d] if j is the q-th main column
 *   (no residual codebook: the C2 term is absent, not +0; no scale: factor 1).
 *
 * The layer then computes y[b,:] = W x[b,:] (decode, batch 1..16) or
 * Y = X W^T (prefill).  Both fuse the dequantisation into the product, so the
 * fp16 weight is never written to global memory (VPTQ page, "The dequantization
 * interface": dequantisation fused into the GEMV for decoding and the GEMM for
 * prefill): the prefill dequantises each weight tile in shared memory and feeds
 * it to the tcgen05 tensor cores.  (Layers with a residual codebook, an outlier
 * block or d != 8 take a two-phase prefill instead: exact dequantisation into the
 * caller's workspace, then the tensor-core GEMM.)
 *
 * Packed index format
 * -------------------
 * A field is w = bits1 + bits2 bits wide (bits2 = 0 without a residual
 * codebook).  Row i of the code matrix starts at byte i * row_stride_bytes.
 * Field s of a row occupies bits [s*w, s*w + w) of that row's byte string,
 * least significant bit first, bytes in increasing address order (so byte b
 * holds bits 8b..8b+7, bit 0 = its LSB).  Within a field, i1 is the low bits1
 * bits and i2 the next bits2 bits.  Example: w = 12+12, i1 = 0xABC,
 * i2 = 0x123 -> bytes BC 3A 12.  Bits after the row's last field are ignored.
 * The outlier block uses the same scheme with bits_o-bit fields.
 * (The VPTQ page gives only "ceil(log2 k) bits per index"; the bit order and
 * the per-row layout are this library's choice.)
 *
 * Sub-vectors per row: n_sub = ceil(n_main / d), n_main = n_in - n_ocols;
 * n_sub_o = ceil(n_ocols / d).  The last sub-vector of a row may cover fewer
 * than d real columns; its remaining elements are ignored.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - fp16/bf16 arrays are passed as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Every call returns a vqlin_status; nothing is thrown across the ABI and
 *    no kernel traps.  A failed call leaves its outputs unspecified.
 *    vqlin_last_error() gives a thread-local, human-readable detail string.
 *  - Kernels run asynchronously on `stream`; a launch failure is reported as
 *    VQLIN_ERR_CUDA.  The handle is immutable after vqlin_create, so calls on
 *    different streams may run concurrently.
 */
#ifndef VQLIN_H
#define VQLIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VQLIN_ABI_VERSION 1
#define VQLIN_MAX_BATCH 16

typedef enum {
  VQLIN_OK = 0,
  VQLIN_ERR_INVALID_ARG = 1,  /* NULL pointer, bad size, bad stride or alignment   */
  VQLIN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d not in {4,6,8,12}) */
  VQLIN_ERR_INVALID_DATA = 3, /* index >= k, malformed CSR, non-finite value        */
  VQLIN_ERR_OOM = 4,          /* device or host allocation failed                   */
  VQLIN_ERR_CUDA = 5,         /* a CUDA call or kernel launch failed                */
  VQLIN_ERR_WORKSPACE = 6     /* workspace NULL, too small or misaligned            */
} vqlin_status;

typedef enum { VQLIN_F32 = 0, VQLIN_F16 = 1, VQLIN_BF16 = 2 } vqlin_dtype;

typedef struct vqlin_handle vqlin_handle;

/*
 * Layer description.  Pointers are borrowed for the duration of vqlin_create
 * only; they are device pointers unless src_on_host is non-zero, in which
 * case they are host pointers.
 */
typedef struct {
  int32_t n_out, n_in;        /* W is n_out x n_in; both >= 1                         */
  int32_t d;                  /* sub-vector length: 4, 6, 8 or 12 (VPTQ's vector
                                 lengths); the tensor-core and codebook-stationary
                                 decode paths are d = 8, the others run CUDA cores    */
  int32_t src_on_host;        /* 0: pointers below are device pointers; 1: host        */

  /* main body */
  int32_t k1, bits1;          /* entries of C1 (1 <= k1 <= 2^bits1), 1 <= bits1 <= 16  */
  int32_t k2, bits2;          /* residual C2: k2 = bits2 = 0 for none; else k2 <= 2^bits2,
                                 1 <= bits2 <= 16 and bits1 + bits2 <= 32              */
  const void* codes;          /* n_out rows of packed fields (format above)           */
  int64_t row_stride_bytes;   /* >= ceil(n_sub * (bits1+bits2) / 8)                    */
  const uint16_t* codebook1;  /* fp16 [k1][d], row-major                              */
  const uint16_t* codebook2;  /* fp16 [k2][d] or NULL when k2 == 0                    */

  /* scales (SCVQ bi-normalisation); NULL means all ones */
  const uint16_t* row_scale;  /* fp16 [n_out]                                          */
  const uint16_t* col_scale;  /* fp16 [n_in]                                           */

  /* outlier-column block (VPTQ "Outlier Elimination"); n_ocols = 0 for none */
  int32_t n_ocols;            /* 0 <= n_ocols <= n_in                                  */
  const int32_t* ocols;       /* strictly increasing column ids in [0, n_in)           */
  int32_t ko, bits_o;         /* entries of Co (ko <= 2^bits_o), 1 <= bits_o <= 16     */
  const uint16_t* codebook_o; /* fp16 [ko][d] (the block uses the layer's d)           */
  const void* codes_o;        /* n_out rows of packed bits_o-bit fields                */
  int64_t o_row_stride_bytes; /* >= ceil(n_sub_o * bits_o / 8)                         */

  /* sparse correction, CSR, REPLACE semantics: W[i,j] = values[e] exactly */
  int64_t nnz;                /* 0 <= nnz; nnz = 0 allows NULL arrays                 */
  const int32_t* row_ptr;     /* [n_out + 1], row_ptr[0] = 0, non-decreasing, = nnz at end */
  const int32_t* col_idx;     /* [nnz], strictly increasing within a row, in [0, n_in) */
  const uint16_t* values;     /* fp16 [nnz], finite                                    */

  /* VSR: a structured sparse correction by whole sub-vectors (SCVQ summary: the important
     weights sit contiguously within rows, in line with VQ's sub-vector grouping, and are kept
     in a structured sparse format, "VSR").  The pages give no layout; this library's reading is
     a row-compressed format whose unit is one main-column sub-vector: block b of row i covers
     sub-vector s = vsr_pos[b], i.e. the main columns q = s*d .. s*d + d - 1, and REPLACES every
     one of its elements: W[i, main column q] = vsr_values[b*d + q - s*d] (a tail sub-vector's
     values past the last main column are ignored).  A block may not share an element with the
     CSR matrix (INVALID_DATA).  Per block: one 4-byte position and d fp16 values, instead of d
     (value, column) pairs. */
  int64_t vsr_nblocks;        /* 0 <= vsr_nblocks; 0 allows NULL arrays                 */
  const int32_t* vsr_row_ptr; /* [n_out + 1] over blocks, [0] = 0, non-decreasing, = vsr_nblocks at end */
  const int32_t* vsr_pos;     /* [vsr_nblocks], strictly increasing within a row, in [0, n_sub) */
  const uint16_t* vsr_values; /* fp16 [vsr_nblocks][d], finite                           */

  /* Codebook groups (VPTQ page, "Outlier Elimination", on group partitioning: the non-outlier
     weights split into group_num groups with independent codebooks).  The pages do not say how
     groups are formed; this library's reading: the main sub-vector positions of every row form
     n_groups contiguous ranges of g = ceil(n_sub / n_groups) positions, position s decodes with
     codebook s / g, and codebook1 (and codebook2) hold the n_groups codebooks back to back,
     [n_groups][k][d].  0 or 1: one codebook.  1 <= n_groups <= n_sub. */
  int32_t n_groups;

  /* Symmetric codebook (SCVQ summary: symmetry constraints shrink the codebook, to a quarter of
     its size).  The pages do not name the symmetry; this library's reading: each codebook1 stores
     k1 / 4 base entries, and entry t * (k1 / 4) + b of the k1 addressed by the indices is base
     entry b under sign pattern t: t = 0 all +, t = 1 all -, t = 2 odd elements negated, t = 3 even
     elements negated (a group of four sign patterns; negation is exact in fp16).  0: none;
     1: this symmetry (needs k1 % 4 == 0; the residual and outlier codebooks stay plain). */
  int32_t cb_symmetry;
} vqlin_desc;

/* Sizes and bit accounting of a created layer. */
typedef struct {
  int32_t n_out, n_in, d, n_sub, n_sub_o, n_ocols;
  int64_t nnz;
  int64_t index_bytes;        /* packed main + outlier fields, rows packed without padding */
  int64_t codebook_bytes;     /* stored codebooks: 2 * d * (n_groups * (k1s + k2) + ko), k1s =
                                 k1 / 4 with a symmetric codebook, else k1                */
  int64_t scale_bytes;        /* 2 * (n_out if row scales) + 2 * (n_in if column scales) */
  int64_t sparse_bytes;       /* CSR: nnz * (2 value + 4 column) + 4 * (n_out + 1)      */
  /* VPTQ page, "Compression ratio calculation": original fp16 bits divided by
     (codebook bits + index bits); equivalent bit width = 16 / ratio.  These two
     use exactly that formula over the main codebooks as stored (n_groups * k1s
     entries) and the main indices only. */
  double vptq_compression_ratio;
  double vptq_bits_per_weight;
  /* everything the layer stores (indices, all codebooks, scales, CSR, VSR), in bits per weight */
  double total_bits_per_weight;
  int64_t vsr_bytes;          /* VSR: 4 * (n_out + 1) + vsr_nblocks * (4 + 2 d), 0 without VSR */
} vqlin_info;

/*
 * Validate `desc`, copy and repack everything into device memory owned by the
 * returned handle, and synchronise `stream` before returning.
 * Checks: shapes and bit widths; CSR structure, column range, ordering and
 * finiteness; codebook and scale finiteness; ocols ordering; every decoded
 * index < its k.  Errors: INVALID_ARG, UNSUPPORTED, INVALID_DATA, OOM, CUDA.
 * On error *out is set to NULL.
 */
vqlin_status vqlin_create(const vqlin_desc* desc, void* stream, vqlin_handle** out);

/* Free the handle's device memory.  NULL is accepted.  The caller must make sure
   no call using the handle is still running. */
vqlin_status vqlin_destroy(vqlin_handle* h);

vqlin_status vqlin_get_info(const vqlin_handle* h, vqlin_info* info);

/*
 * Dense fp16 weight: W[i*ldw + j] for 0 <= i < n_out, 0 <= j < n_in, written
 * on `stream` (device pointer, ldw >= n_in).  Each element is the IEEE fp16
 * value nearest (ties to even; overflow to +-inf) to the exact real value of
 * the formula above; at CSR positions it is v_ij bit for bit.  Zero results
 * carry the sign IEEE arithmetic gives r*c*(C1 + C2) (C1 alone without C2).
 * (VPTQ page, "The dequantization interface": W = C[indices] and
 * C[indices1] + Cres[indices2].)
 */
vqlin_status vqlin_dequant(const vqlin_handle* h, uint16_t* W, int64_t ldw, void* stream);

/*
 * Decode (VPTQ page: "QGemv", dequantisation fused into the GEMV):
 *   y[b*n_out + i] = sum_j W[i,j] * x[b*n_in + j],  0 <= b < batch <= 16.
 * x: device [batch][n_in] of xt (F16, BF16 or F32); y: device [batch][n_out]
 * of yt.  Products and sums are fp32 (W's unrounded value r*c*C enters through
 * fp32 arithmetic, not through an fp16 weight; with d = 8 the tensor-core path
 * carries x' = c*x as two fp16 parts, so |c_j x_j| must stay below 65504).
 * x and y must be 16-byte aligned and must not overlap.  Summation order is
 * unspecified.
 */
vqlin_status vqlin_gemv(const vqlin_handle* h, const void* x, vqlin_dtype xt, int32_t batch,
                        void* y, vqlin_dtype yt, void* stream);

/*
 * The same product with a caller-owned scratch buffer (>= vqlin_gemv_workspace_size(h,
 * batch) bytes, 256-byte aligned, device memory, not used by another call at the same
 * time; its contents need not be initialised and are unspecified afterwards).  The
 * scratch enables the faster kernels:
 *   - layers with a large single-stage codebook (k1 > 10240, d = 8) and batch <= 4 run
 *     the codebook-stationary decode, whose blocks each own a slice of the codebook
 *     and write per-block partial sums here (deterministic: fixed-point row sums);
 *   - layers too wide for one pass of the tensor-core decode sum column chunks here
 *     in fp32 and convert to yt at the end (vqlin_gemv instead has each block loop
 *     over the chunks itself).
 * Results agree with vqlin_gemv within the GEMV tolerance (summation order differs).
 * Errors additionally: WORKSPACE.
 */
vqlin_status vqlin_gemv_ws(const vqlin_handle* h, const void* x, vqlin_dtype xt, int32_t batch,
                           void* y, vqlin_dtype yt, void* workspace, size_t ws_bytes, void* stream);
size_t vqlin_gemv_workspace_size(const vqlin_handle* h, int32_t batch);

/*
 * The decode GEMV for callers that cannot allocate device memory at call time
 * (a serving loop whose pool already owns the GPU's memory, a path where
 * cudaMalloc's implicit device synchronisation is not allowed, a plug-in that
 * may only touch the buffers it is handed).  It computes what vqlin_gemv_ws
 * computes, with a scratch array built into the library (8 MiB per device, held
 * until the process exits) in place of a caller buffer, and it allocates
 * nothing.  The array holds the codebook-stationary partial sums of a 4096-row
 * layer with a 65536-entry codebook up to batch 4 and the column-split fp32
 * accumulator of any layer with batch * n_out <= 2097152; a plan that needs more
 * runs the kernels that need no scratch (as vqlin_gemv does).  Limit: batch *
 * n_out <= 2097152, else VQLIN_ERR_UNSUPPORTED.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) and caches it: make
 * that first call outside stream capture.  All calls share the array: calls
 * whose kernels overlap on the GPU race on it, so the caller must serialise
 * them.  What must start at zero is cleared on the call's stream before each
 * use.  (No counterpart on the pages: this is an interface convenience.)
 */
vqlin_status vqlin_gemv_noalloc(const vqlin_handle* h, const void* x, vqlin_dtype xt, int32_t batch,
                                void* y, vqlin_dtype yt, void* stream);

/*
 * Prefill: Y[m*n_out + i] = sum_j W[i,j] * X[m*n_in + j] for 0 <= m < M.
 * X: device [M][n_in] of xt (F16 or BF16; BF16 is converted to fp16, exact for
 * 2^-14 <= |x| <= 65504), Y: device [M][n_out] of yt.  The weight enters the
 * tensor-core product as its fp16 dequantised value (bit for bit what
 * vqlin_dequant writes); accumulation is fp32.  For d = 8 layers with one
 * codebook and no outlier block the weight tiles are dequantised in shared
 * memory inside the GEMM, and the workspace only holds BF16 activations
 * converted to fp16 (M * n_in * 2 bytes; unused for F16); other layers
 * dequantise the whole weight into the workspace first.
 * workspace: device memory of at least vqlin_gemm_workspace_size(h, M) bytes,
 * 256-byte aligned, owned by the caller, not used concurrently by another call.
 * Errors additionally: WORKSPACE, UNSUPPORTED (M < 1 or n_in % 8 != 0).
 */
vqlin_status vqlin_gemm(const vqlin_handle* h, const void* X, vqlin_dtype xt, int64_t M,
                        void* Y, vqlin_dtype yt, void* workspace, size_t ws_bytes, void* stream);
size_t vqlin_gemm_workspace_size(const vqlin_handle* h, int64_t M);

/*
 * Test hook: decoded fields.  which = 0: main body, out[i*n_sub + s] =
 * i1 | (i2 << bits1); which = 1: outlier block, out[i*n_sub_o + s].
 * `out` is a device uint32 array.
 */
vqlin_status vqlin_unpack_indices(const vqlin_handle* h, int32_t which, uint32_t* out, void* stream);

/*
 * Device-side failure detection.  Kernels that wait on hardware barriers bound
 * every wait (1 s); when one gives up it records a code, skips its remaining
 * work and returns, so the context stays usable.  This call synchronises the
 * current device, returns the recorded code in *code (0 = none; 1-5 = the
 * GEMM pipeline wait that expired; 6 = the decode entry-stream wait; 7 = the
 * self-test below) and clears it.  No counterpart on the pages.
 */
vqlin_status vqlin_device_error(int32_t* code);

/*
 * Nearest-centroid assignment, the encoding step that produces the indices the layer
 * stores (VPTQ page, "Step 3": Q_V(v) = argmin_i ||v - C_i||^2, plain Euclidean distance;
 * "Residual Vector Quantization": i1 = Q_1(v), i2 = argmin_j ||(v - C1[i1]) - C2_j||^2).
 *   V    device fp16 [n][d] sub-vectors (d in {4, 6, 8, 12}), finite values
 *   C1   device fp16 [k1][d] codebook, k1 >= 1
 *   C2   device fp16 [k2][d] residual codebook, or NULL with k2 = 0
 *   idx1 device uint32 [n]; idx2 device uint32 [n] when k2 > 0 (else ignored)
 * Distances are taken in binary32: each difference is one rounded subtraction and the running
 * sum one fused multiply-add per element, elements in order, centroids from index 0 up; ties keep
 * the lowest index; the residual is the binary32 difference v - C1[i1].  So idx1 is a nearest
 * centroid up to rounding: its exact squared distance D satisfies D (1 - e) <= Dmin (1 + e) with
 * e = (d + 3) 2^-24 and Dmin the exact minimum (idx1 is the exact argmin wherever that minimum
 * is unique beyond the slack; an exact hit, distance 0, returns its lowest index); idx2 is the
 * same for v - C1[idx1], up to the additional rounding of that residual.  n = 0 does nothing.
 * Runs on `stream`; the caller owns every buffer.  No counterpart of this signature on the pages.
 */
vqlin_status vqlin_assign(const uint16_t* V, int64_t n, int32_t d, const uint16_t* C1, int32_t k1,
                          const uint16_t* C2, int32_t k2, uint32_t* idx1, uint32_t* idx2, void* stream);

/*
 * Failure-detection self-test.  Launches on `stream` one thread that waits on a
 * shared-memory mbarrier nothing completes, bounded by `limit_us` microseconds
 * (1..1,000,000) of %globaltimer, exactly like the decode kernel's entry-stream
 * wait.  When the limit passes the kernel records code 7 and returns, so a
 * following vqlin_device_error() reports 7 and the context stays usable.  No
 * counterpart on the pages.
 */
vqlin_status vqlin_selftest_wait_timeout(int32_t limit_us, void* stream);

/*
 * Number of kernels this library has enqueued in this process so far, over
 * every device, stream and thread (a launch recorded into a CUDA graph counts
 * once, when it is recorded).  Library copies and memsets are not counted.
 * Take the difference around a call to learn how many kernels it launched.
 * No counterpart on the pages.
 */
uint64_t vqlin_kernel_launches(void);

const char* vqlin_status_string(vqlin_status s);
const char* vqlin_last_error(void);
int32_t vqlin_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* VQLIN_H */
