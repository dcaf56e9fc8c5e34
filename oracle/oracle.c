/*
 * oracle.c — plain, slow, single-threaded CPU reference for the VQ + sparse
 * linear layer.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call it; the library never does.  It shares
 * no code, header or constant with the CUDA library.
 *
 * What it computes (each function cites the page and section it follows):
 *
 *   W[i,j] = v_ij                                           (i,j) in the sparse set
 *          = r_i c_j Co[io(i, p/d)][p mod d]                j = p-th outlier column
 *          = r_i c_j (C1[i1(i,q/d)] + C2[i2(i,q/d)])[q mod d]  j = q-th main column
 *
 *   - HAS-VQ: Hessian-Adaptive Sparse Vector Quantization for High-Fidelity LLM
 *     Compression, abstract: the residual sparse feedback reconstructs the
 *     outliers exactly, so sparse positions take the stored value itself.
 *   - SCVQ: Sparse-Compensated Vector Quantization for Large Language Models,
 *     summary: bi-normalisation by row and column scales (applied here as
 *     multipliers) and a single sparse correction matrix.
 *   - VPTQ: Extreme Low-bit Vector Post-Training Quantization for Large
 *     Language Models: "The dequantization interface" (index matrix of
 *     ceil(log2 k)-bit integers, codebooks [k, V], W = C[indices]),
 *     "Residual Vector Quantization" (decoding adds C[index1] + Cres[index2]),
 *     "Outlier Elimination" (a separate codebook for a set of columns, chosen by
 *     a static branch), "Compression ratio calculation" (bit accounting).
 *
 * Readings where the pages are silent (listed with the rest in the design
 * notes): sub-vectors run along the input columns of a row; fields are packed
 * LSB-first per row; i1 sits in the low bits of a residual field; scales
 * multiply; sparse entries replace; the outlier block ignores the residual
 * codebook; rounding to fp16 is round-to-nearest-even with overflow to inf.
 *
 * Exactness: oracle_dequant_exact() evaluates r*c*(C1+C2) as an exact integer
 * times a power of two (__int128) and rounds it to fp16 by integer arithmetic.
 * oracle_dequant_f64() evaluates the same expression in IEEE double (the sum
 * and the first product are exact, the second product rounds once).
 * oracle_gemv_f64() is the dense product with those double weights.
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fPIC -shared oracle.c -o liboracle.so
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

typedef __int128 i128;
typedef unsigned __int128 u128;

/* ------------------------------------------------------------------ */
/* IEEE binary16 / bfloat16 decoding                                    */
/* ------------------------------------------------------------------ */

/* Exact decomposition of a finite fp16: value = (-1)^sign * mant * 2^exp2,
   0 <= mant < 2048.  Returns 0 for inf/NaN (which the layer format forbids). */
static int f16_split(uint16_t h, int* sign, int64_t* mant, int* exp2) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, f = h & 0x3FF;
  if (e == 31) return 0;
  *sign = s;
  if (e == 0) { *mant = f; *exp2 = -24; }          /* subnormal: f * 2^-24   */
  else { *mant = 1024 + f; *exp2 = e - 25; }        /* (1024+f) * 2^(e-15-10) */
  return 1;
}

double oracle_f16_to_f64(uint16_t h) {
  int s, e; int64_t m;
  if (!f16_split(h, &s, &m, &e)) {
    if ((h & 0x3FF) != 0) return NAN;
    return (h >> 15) ? -INFINITY : INFINITY;
  }
  double v = ldexp((double)m, e);
  return s ? -v : v;
}

double oracle_bf16_to_f64(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 7) & 0xFF, f = h & 0x7F;
  double v;
  if (e == 255) return f ? NAN : (s ? -INFINITY : INFINITY);
  if (e == 0) v = ldexp((double)f, -133);           /* f * 2^(-126-7) */
  else v = ldexp((double)(128 + f), e - 134);       /* (128+f) * 2^(e-127-7) */
  return s ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Round (-1)^sign * M * 2^E to the nearest fp16, ties to even.         */
/* ------------------------------------------------------------------ */
static int bitlen128(u128 x) {
  int n = 0;
  while (x) { ++n; x >>= 1; }
  return n;
}

uint16_t oracle_round_f16(int sign, u128 M, int E) {
  uint16_t sbit = sign ? 0x8000 : 0;
  if (M == 0) return sbit;
  int nb = bitlen128(M);
  int top = nb - 1 + E;                 /* 2^top <= value < 2^(top+1)        */
  int e = top < -14 ? -14 : top;        /* binade, clamped at the subnormals */
  int qe = e - 10;                      /* weight of the last kept bit       */
  int shift = qe - E;
  u128 N;
  if (shift <= 0) {
    N = M << (-shift);                  /* exact, nothing dropped            */
  } else if (shift > nb) {
    N = 0;                              /* below half of the last kept bit   */
  } else {
    N = (shift >= 128) ? 0 : (M >> shift);
    u128 rem = M - (N << shift);
    u128 half = (u128)1 << (shift - 1);
    if (rem > half || (rem == half && (N & 1))) N += 1;
  }
  if (N == 0) return sbit;
  if (N >= 2048) { N >>= 1; qe += 1; }  /* carried into the next binade (N was 2048) */
  if (qe == -24 && N < 1024) return (uint16_t)(sbit | (uint16_t)N);   /* subnormal */
  int ef = qe + 25;                     /* biased exponent field             */
  if (ef >= 31) return (uint16_t)(sbit | 0x7C00);                     /* overflow  */
  return (uint16_t)(sbit | (uint16_t)(ef << 10) | (uint16_t)(N - 1024));
}

/* Python-callable form with the 128-bit magnitude split in two halves. */
uint16_t oracle_round_f16_parts(int sign, uint64_t m_hi, uint64_t m_lo, int E) {
  return oracle_round_f16(sign, ((u128)m_hi << 64) | m_lo, E);
}

/* ------------------------------------------------------------------ */
/* Packed fields: bits [s*w, s*w+w) of a row, least significant first.  */
/* (VPTQ page, "The dequantization interface": ceil(log2 k)-bit indices; */
/*  the bit order is this format's reading.)                             */
/* ------------------------------------------------------------------ */
uint32_t oracle_field(const uint8_t* row, int64_t s, int w) {
  uint32_t v = 0;
  for (int t = 0; t < w; ++t) {
    int64_t bit = s * (int64_t)w + t;
    uint32_t b = (row[bit >> 3] >> (bit & 7)) & 1u;
    v |= b << t;
  }
  return v;
}

void oracle_unpack(const uint8_t* codes, int64_t stride, int32_t n_rows, int32_t n_fields, int w,
                   uint32_t* out) {
  for (int32_t i = 0; i < n_rows; ++i)
    for (int32_t s = 0; s < n_fields; ++s)
      out[(int64_t)i * n_fields + s] = oracle_field(codes + (int64_t)i * stride, s, w);
}

/* ------------------------------------------------------------------ */
/* Layer                                                               */
/* ------------------------------------------------------------------ */
typedef struct {
  int32_t n_out, n_in, d;
  int32_t k1, bits1, k2, bits2;
  const uint8_t* codes; int64_t stride;
  const uint16_t* cb1; const uint16_t* cb2;
  const uint16_t* rs; const uint16_t* cs;
  int32_t n_ocols; const int32_t* ocols;
  int32_t ko, bits_o; const uint16_t* cbo; const uint8_t* codes_o; int64_t stride_o;
  int64_t nnz; const int32_t* row_ptr; const int32_t* col_idx; const uint16_t* values;
  int64_t vsr_nb; const int32_t* vsr_row_ptr; const int32_t* vsr_pos; const uint16_t* vsr_values;
  int32_t n_groups; int32_t cb_symmetry;
} oracle_layer;

enum { ORACLE_OK = 0, ORACLE_BAD_INDEX = 1, ORACLE_BAD_VALUE = 2, ORACLE_BAD_CSR = 3, ORACLE_OOM = 4 };

/* For every column j: is_out[j] = 1 for an outlier column; rank[j] = its
   position among the outlier columns (p) or among the main columns (q). */
static int column_ranks(const oracle_layer* L, uint8_t* is_out, int32_t* rank) {
  memset(is_out, 0, (size_t)L->n_in);
  for (int32_t t = 0; t < L->n_ocols; ++t) {
    int32_t j = L->ocols[t];
    if (j < 0 || j >= L->n_in || (t > 0 && L->ocols[t - 1] >= j)) return ORACLE_BAD_INDEX;
    is_out[j] = 1;
  }
  int32_t p = 0, q = 0;
  for (int32_t j = 0; j < L->n_in; ++j) rank[j] = is_out[j] ? p++ : q++;
  return ORACLE_OK;
}

static int32_t n_main_cols(const oracle_layer* L) { return L->n_in - L->n_ocols; }
static int32_t n_main_sub(const oracle_layer* L) { return (n_main_cols(L) + L->d - 1) / L->d; }
static int32_t n_groups_of(const oracle_layer* L) { return L->n_groups > 1 ? L->n_groups : 1; }

/* Codebook group of main sub-vector s (VPTQ page, "Outlier Elimination", on group partitioning:
   independent codebooks per group; reading: contiguous ranges of ceil(n_sub / n_groups)
   positions). */
static int32_t group_of(const oracle_layer* L, int32_t s) {
  const int32_t G = n_groups_of(L), n_sub = n_main_sub(L);
  if (G == 1) return 0;
  const int32_t size = (n_sub + G - 1) / G;
  return s / size;
}

/* Element e (0..d-1) of entry i1 of group g's main codebook.  A symmetric codebook (SCVQ
   summary: symmetry constraints shrink the codebook to a quarter) stores k1/4 base entries;
   entry t*(k1/4) + b is base entry b under sign pattern t: 0 none, 1 all negated, 2 odd
   elements negated, 3 even elements negated (fp16 negation flips the sign bit, exactly). */
static uint16_t main_entry(const oracle_layer* L, int32_t g, uint32_t i1, int32_t e) {
  const int32_t d = L->d;
  if (!L->cb_symmetry) return L->cb1[((int64_t)g * L->k1 + i1) * d + e];
  const uint32_t k1s = (uint32_t)L->k1 / 4u;
  const uint32_t t = i1 / k1s, b = i1 % k1s;
  const uint16_t v = L->cb1[((int64_t)g * k1s + b) * d + e];
  const int neg = (t == 1) || (t == 2 && (e & 1)) || (t == 3 && !(e & 1));
  return neg ? (uint16_t)(v ^ 0x8000u) : v;
}

/* Decoded codebook values of one weight element (i, j) that is not in the sparse set: the fp16
   bits of the first-stage (or outlier-block) element in *h1, and a pointer to the residual
   element in *e2 (NULL when there is none). */
static int element_codes(const oracle_layer* L, const uint8_t* is_out, const int32_t* rank, int32_t i,
                         int32_t j, uint16_t* h1, const uint16_t** e2) {
  int32_t d = L->d;
  if (is_out[j]) {
    int32_t p = rank[j];
    uint32_t io = oracle_field(L->codes_o + (int64_t)i * L->stride_o, p / d, L->bits_o);
    if (io >= (uint32_t)L->ko) return ORACLE_BAD_INDEX;
    *h1 = *(L->cbo + (int64_t)io * d + (p % d));
    *e2 = NULL;                        /* the residual codebook does not apply */
  } else {
    int32_t q = rank[j];
    uint32_t f = oracle_field(L->codes + (int64_t)i * L->stride, q / d, L->bits1 + L->bits2);
    uint32_t i1 = L->bits1 >= 32 ? f : (f & ((1u << L->bits1) - 1u));
    uint32_t i2 = L->bits2 ? (f >> L->bits1) : 0;
    if (i1 >= (uint32_t)L->k1) return ORACLE_BAD_INDEX;
    const int32_t g = group_of(L, q / d);
    *h1 = main_entry(L, g, i1, q % d);
    if (L->k2 > 0) {
      if (i2 >= (uint32_t)L->k2) return ORACLE_BAD_INDEX;
      *e2 = L->cb2 + ((int64_t)g * L->k2 + i2) * d + (q % d);
    } else {
      *e2 = NULL;
    }
  }
  return ORACLE_OK;
}

/* Main-column ids in order (main_col[q] = the q-th column that is not an outlier column). */
static void main_columns(const oracle_layer* L, const uint8_t* is_out, int32_t* main_col) {
  int32_t q = 0;
  for (int32_t j = 0; j < L->n_in; ++j) if (!is_out[j]) main_col[q++] = j;
}

/* VSR blocks (SCVQ summary: a structured sparse format for salient weights that sit
   contiguously within rows; reading: whole main-column sub-vectors, REPLACE): structure,
   finiteness, and no element shared with the CSR matrix. */
static int check_vsr(const oracle_layer* L, const uint8_t* is_out, const int32_t* rank) {
  if (L->vsr_nb == 0) return ORACLE_OK;
  const int32_t d = L->d, n_sub = n_main_sub(L);
  if (L->vsr_row_ptr[0] != 0 || L->vsr_row_ptr[L->n_out] != L->vsr_nb) return ORACLE_BAD_CSR;
  for (int32_t i = 0; i < L->n_out; ++i) {
    if (L->vsr_row_ptr[i + 1] < L->vsr_row_ptr[i]) return ORACLE_BAD_CSR;
    for (int32_t b = L->vsr_row_ptr[i]; b < L->vsr_row_ptr[i + 1]; ++b) {
      const int32_t s = L->vsr_pos[b];
      if (s < 0 || s >= n_sub || (b > L->vsr_row_ptr[i] && L->vsr_pos[b - 1] >= s)) return ORACLE_BAD_CSR;
      for (int32_t t = 0; t < d; ++t)
        if (((L->vsr_values[(int64_t)b * d + t] >> 10) & 0x1F) == 31) return ORACLE_BAD_VALUE;
    }
    if (L->nnz > 0)
      for (int32_t e = L->row_ptr[i]; e < L->row_ptr[i + 1]; ++e) {
        const int32_t j = L->col_idx[e];
        if (is_out[j]) continue;
        for (int32_t b = L->vsr_row_ptr[i]; b < L->vsr_row_ptr[i + 1]; ++b)
          if (L->vsr_pos[b] == rank[j] / d) return ORACLE_BAD_CSR;   /* element in both */
      }
  }
  return ORACLE_OK;
}

static int check_shape(const oracle_layer* L) {
  const int32_t n_sub = n_main_sub(L);
  if (L->n_groups < 0 || (n_sub > 0 && n_groups_of(L) > n_sub)) return ORACLE_BAD_VALUE;
  if (L->cb_symmetry && (L->cb_symmetry != 1 || L->k1 % 4 != 0)) return ORACLE_BAD_VALUE;
  return ORACLE_OK;
}

/* Exact fp16 of r*c*(C1 + C2) (C1 alone without a residual; factors of 1
   when a scale is absent), zero signs as IEEE arithmetic gives them. */
static int exact_body_f16(uint16_t h1, const uint16_t* h2, const uint16_t* hr, const uint16_t* hc,
                          uint16_t* out) {
  int s1, e1; int64_t m1;
  if (!f16_split(h1, &s1, &m1, &e1)) return ORACLE_BAD_VALUE;
  i128 S; int eS, sS;
  if (h2) {
    int s2, e2; int64_t m2;
    if (!f16_split(*h2, &s2, &m2, &e2)) return ORACLE_BAD_VALUE;
    int emin = e1 < e2 ? e1 : e2;
    i128 a = (i128)m1 << (e1 - emin), b = (i128)m2 << (e2 - emin);
    S = (s1 ? -a : a) + (s2 ? -b : b);
    eS = emin;
    if (S != 0) sS = S < 0;
    else sS = (s1 && s2);              /* x + (-x) = +0; (-0) + (-0) = -0 */
    if (S < 0) S = -S;
  } else {
    S = m1; eS = e1; sS = s1;
  }
  u128 M = (u128)S;
  int E = eS, sign = sS;
  const uint16_t* fs[2] = {hr, hc};
  for (int t = 0; t < 2; ++t) {
    if (!fs[t]) continue;
    int sf, ef; int64_t mf;
    if (!f16_split(*fs[t], &sf, &mf, &ef)) return ORACLE_BAD_VALUE;
    M *= (u128)mf; E += ef; sign ^= sf;
  }
  *out = oracle_round_f16(sign, M, E);
  return ORACLE_OK;
}

/* Python-callable single-element form (NULL pointers = absent term). */
int oracle_body_f16(uint16_t c1, const uint16_t* c2, const uint16_t* r, const uint16_t* c, uint16_t* out) {
  return exact_body_f16(c1, c2, r, c, out);
}

static int check_csr(const oracle_layer* L) {
  if (L->nnz == 0) return ORACLE_OK;
  if (L->row_ptr[0] != 0 || L->row_ptr[L->n_out] != L->nnz) return ORACLE_BAD_CSR;
  for (int32_t i = 0; i < L->n_out; ++i) {
    if (L->row_ptr[i + 1] < L->row_ptr[i]) return ORACLE_BAD_CSR;
    for (int32_t e = L->row_ptr[i]; e < L->row_ptr[i + 1]; ++e) {
      int32_t j = L->col_idx[e];
      if (j < 0 || j >= L->n_in) return ORACLE_BAD_CSR;
      if (e > L->row_ptr[i] && L->col_idx[e - 1] >= j) return ORACLE_BAD_CSR;
      uint16_t v = L->values[e];
      if (((v >> 10) & 0x1F) == 31) return ORACLE_BAD_VALUE;
    }
  }
  return ORACLE_OK;
}

/* vqlin_dequant's definition, bit-exact: W[i*ldw + j] as fp16 bits. */
int oracle_dequant_exact(const oracle_layer* L, uint16_t* W, int64_t ldw) {
  uint8_t* is_out = (uint8_t*)malloc((size_t)L->n_in);
  int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * (size_t)L->n_in);
  int32_t* main_col = (int32_t*)malloc(sizeof(int32_t) * (size_t)L->n_in);
  int rc = (is_out && rank && main_col) ? ORACLE_OK : ORACLE_OOM;
  if (rc == ORACLE_OK) rc = check_shape(L);
  if (rc == ORACLE_OK) rc = column_ranks(L, is_out, rank);
  if (rc == ORACLE_OK) rc = check_csr(L);
  if (rc == ORACLE_OK) rc = check_vsr(L, is_out, rank);
  if (rc == ORACLE_OK) main_columns(L, is_out, main_col);
  for (int32_t i = 0; rc == ORACLE_OK && i < L->n_out; ++i) {
    const uint16_t* hr = L->rs ? &L->rs[i] : NULL;
    for (int32_t j = 0; rc == ORACLE_OK && j < L->n_in; ++j) {
      uint16_t h1;
      const uint16_t* e2;
      rc = element_codes(L, is_out, rank, i, j, &h1, &e2);
      if (rc != ORACLE_OK) break;
      rc = exact_body_f16(h1, e2, hr, L->cs ? &L->cs[j] : NULL, &W[(int64_t)i * ldw + j]);
    }
    if (rc == ORACLE_OK && L->nnz > 0)
      for (int32_t e = L->row_ptr[i]; e < L->row_ptr[i + 1]; ++e)
        W[(int64_t)i * ldw + L->col_idx[e]] = L->values[e];   /* REPLACE: exact outliers */
    if (rc == ORACLE_OK && L->vsr_nb > 0)
      for (int32_t b = L->vsr_row_ptr[i]; b < L->vsr_row_ptr[i + 1]; ++b)
        for (int32_t t = 0; t < L->d; ++t) {
          const int32_t q = L->vsr_pos[b] * L->d + t;
          if (q < n_main_cols(L)) W[(int64_t)i * ldw + main_col[q]] = L->vsr_values[(int64_t)b * L->d + t];
        }
  }
  free(is_out); free(rank); free(main_col);
  return rc;
}

/* Double-precision weights of the selected rows: W[t*n_in + j] for row rows[t]. */
int oracle_dequant_f64_rows(const oracle_layer* L, const int32_t* rows, int32_t n_rows, double* W) {
  uint8_t* is_out = (uint8_t*)malloc((size_t)L->n_in);
  int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * (size_t)L->n_in);
  int32_t* main_col = (int32_t*)malloc(sizeof(int32_t) * (size_t)L->n_in);
  int rc = (is_out && rank && main_col) ? ORACLE_OK : ORACLE_OOM;
  if (rc == ORACLE_OK) rc = check_shape(L);
  if (rc == ORACLE_OK) rc = column_ranks(L, is_out, rank);
  if (rc == ORACLE_OK) rc = check_csr(L);
  if (rc == ORACLE_OK) rc = check_vsr(L, is_out, rank);
  if (rc == ORACLE_OK) main_columns(L, is_out, main_col);
  for (int32_t t = 0; rc == ORACLE_OK && t < n_rows; ++t) {
    int32_t i = rows[t];
    double r = L->rs ? oracle_f16_to_f64(L->rs[i]) : 1.0;
    for (int32_t j = 0; j < L->n_in; ++j) {
      uint16_t h1;
      const uint16_t* e2;
      rc = element_codes(L, is_out, rank, i, j, &h1, &e2);
      if (rc != ORACLE_OK) break;
      double v = oracle_f16_to_f64(h1);
      if (e2) v = v + oracle_f16_to_f64(*e2);
      v = v * r;
      if (L->cs) v = v * oracle_f16_to_f64(L->cs[j]);
      W[(int64_t)t * L->n_in + j] = v;
    }
    if (rc == ORACLE_OK && L->nnz > 0)
      for (int32_t e = L->row_ptr[i]; e < L->row_ptr[i + 1]; ++e)
        W[(int64_t)t * L->n_in + L->col_idx[e]] = oracle_f16_to_f64(L->values[e]);
    if (rc == ORACLE_OK && L->vsr_nb > 0)
      for (int32_t b = L->vsr_row_ptr[i]; b < L->vsr_row_ptr[i + 1]; ++b)
        for (int32_t u = 0; u < L->d; ++u) {
          const int32_t q = L->vsr_pos[b] * L->d + u;
          if (q < n_main_cols(L)) W[(int64_t)t * L->n_in + main_col[q]] = oracle_f16_to_f64(L->vsr_values[(int64_t)b * L->d + u]);
        }
  }
  free(is_out); free(rank); free(main_col);
  return rc;
}

/* Y[m*n_rows + t] = sum_j W(rows[t], j) * X[m*n_in + j], all in double,
   one row of weights at a time (VPTQ page: QGemv = dequantise + GEMV). */
int oracle_gemv_f64_rows(const oracle_layer* L, const int32_t* rows, int32_t n_rows, const double* X,
                         int64_t m, double* Y) {
  double* w = (double*)malloc(sizeof(double) * (size_t)L->n_in);
  if (!w) return ORACLE_OOM;
  int rc = ORACLE_OK;
  for (int32_t t = 0; t < n_rows && rc == ORACLE_OK; ++t) {
    rc = oracle_dequant_f64_rows(L, rows + t, 1, w);
    if (rc != ORACLE_OK) break;
    for (int64_t b = 0; b < m; ++b) {
      const double* x = X + b * L->n_in;
      double acc = 0.0;
      for (int32_t j = 0; j < L->n_in; ++j) acc += w[j] * x[j];
      Y[b * n_rows + t] = acc;
    }
  }
  free(w);
  return rc;
}

/* VPTQ page, "Compression ratio calculation": original fp16 bits over
   (codebook bits V*k*16 + index bits M*ceil(log2 k)/V). */
double oracle_vptq_compression_ratio(int64_t n_elems, int32_t V, int64_t k) {
  int bits = 0;
  while (((int64_t)1 << bits) < k) ++bits;           /* ceil(log2 k) */
  double original = 16.0 * (double)n_elems;
  double codebook = (double)V * (double)k * 16.0;
  double index = (double)n_elems * (double)bits / (double)V;
  return original / (codebook + index);
}

/* ---------------------------------------------------------------- nearest-centroid assignment
   VPTQ page, "Step 3: Vector quantization of column n": Q_V(v) = argmin_i ||v - C_i||^2, the
   plain Euclidean nearest centroid; "Residual Vector Quantization": i1 = Q_1(v), then the
   residual v - C[i1] is quantised with the residual codebook, i2 = argmin_j ||(v - C[i1]) -
   Cres_j||^2.  The pages fix no precision, so this computes the definition exactly: every
   finite fp16 value is an integer multiple of 2^-24, so a difference of two is an exact integer
   in those units (at most 42 bits with sign, also for a residual) and a squared distance an exact
   integer in units of 2^-48 (at most 2^88 for d <= 12, inside __int128).  Centroids are scanned
   from index 0 up and a later one wins only when strictly closer, so ties keep the lowest index
   (the pages give no tie rule; this is the reading taken). */

/* A finite fp16 value as an exact integer count of 2^-24. */
static int64_t f16_units(uint16_t h) {
  int s = 0, e = 0; int64_t m = 0;
  if (!f16_split(h, &s, &m, &e)) return 0;   /* callers reject inf/NaN first */
  /* value = m * 2^e with e >= -24 */
  int64_t v = m << (e + 24);
  return s ? -v : v;
}

/* ||v - c||^2 in units of 2^-48, v given in units of 2^-24, c as fp16. */
static i128 sqdist_units(const int64_t* v, const uint16_t* c, int32_t d) {
  i128 acc = 0;
  for (int32_t t = 0; t < d; ++t) {
    i128 diff = (i128)v[t] - (i128)f16_units(c[t]);
    acc += diff * diff;
  }
  return acc;
}

static uint32_t nearest_exact(const int64_t* v, int32_t d, const uint16_t* C, int32_t k) {
  uint32_t best = 0;
  i128 best_d = 0;
  for (int32_t i = 0; i < k; ++i) {
    i128 D = sqdist_units(v, C + (int64_t)i * d, d);
    if (i == 0 || D < best_d) { best = (uint32_t)i; best_d = D; }
  }
  return best;
}

static int all_finite(const uint16_t* a, int64_t n) {
  for (int64_t e = 0; e < n; ++e) if (((a[e] >> 10) & 0x1F) == 31) return 0;
  return 1;
}

/* idx1[s] = Q_1(V[s]); with a residual codebook also idx2[s] = argmin_j ||(V[s] - C1[idx1[s]]) -
   C2_j||^2.  V [n][d], C1 [k1][d], C2 [k2][d] as fp16 bits; 1 <= d <= 64. */
int oracle_assign_exact(const uint16_t* V, int64_t n, int32_t d, const uint16_t* C1, int32_t k1,
                        const uint16_t* C2, int32_t k2, uint32_t* idx1, uint32_t* idx2) {
  int64_t v[64];
  if (d < 1 || d > 64 || k1 < 1 || k2 < 0 || (k2 > 0 && !C2)) return ORACLE_BAD_VALUE;
  if (!all_finite(V, n * d) || !all_finite(C1, (int64_t)k1 * d) || !all_finite(C2, (int64_t)k2 * d))
    return ORACLE_BAD_VALUE;
  for (int64_t s = 0; s < n; ++s) {
    for (int32_t t = 0; t < d; ++t) v[t] = f16_units(V[s * d + t]);
    const uint32_t i1 = nearest_exact(v, d, C1, k1);
    idx1[s] = i1;
    if (k2 > 0) {
      for (int32_t t = 0; t < d; ++t) v[t] -= f16_units(C1[(int64_t)i1 * d + t]);
      idx2[s] = nearest_exact(v, d, C2, k2);
    }
  }
  return ORACLE_OK;
}

/* The residual stage alone, for a given first-stage choice idx1 (each < k1): idx2[s] = argmin_j
   ||(V[s] - C1[idx1[s]]) - C2_j||^2, exactly. */
int oracle_residual_assign_exact(const uint16_t* V, int64_t n, int32_t d, const uint16_t* C1, int32_t k1,
                                 const uint32_t* idx1, const uint16_t* C2, int32_t k2, uint32_t* idx2) {
  int64_t v[64];
  if (d < 1 || d > 64 || k1 < 1 || k2 < 1 || !C2) return ORACLE_BAD_VALUE;
  if (!all_finite(V, n * d) || !all_finite(C1, (int64_t)k1 * d) || !all_finite(C2, (int64_t)k2 * d))
    return ORACLE_BAD_VALUE;
  for (int64_t s = 0; s < n; ++s) {
    if (idx1[s] >= (uint32_t)k1) return ORACLE_BAD_INDEX;
    for (int32_t t = 0; t < d; ++t) v[t] = f16_units(V[s * d + t]) - f16_units(C1[(int64_t)idx1[s] * d + t]);
    idx2[s] = nearest_exact(v, d, C2, k2);
  }
  return ORACLE_OK;
}

/* Exact ||v - base - c||^2 in units of 2^-48 as a 128-bit integer split into two halves
   (base may be NULL for zero); v, base and c are fp16 [d]. */
int oracle_sqdist_exact(const uint16_t* v, const uint16_t* base, const uint16_t* c, int32_t d, uint64_t* hi,
                        uint64_t* lo) {
  int64_t w[64];
  if (d < 1 || d > 64 || !all_finite(v, d) || !all_finite(c, d) || (base && !all_finite(base, d)))
    return ORACLE_BAD_VALUE;
  for (int32_t t = 0; t < d; ++t) w[t] = f16_units(v[t]) - (base ? f16_units(base[t]) : 0);
  u128 D = (u128)sqdist_units(w, c, d);
  *hi = (uint64_t)(D >> 64);
  *lo = (uint64_t)D;
  return ORACLE_OK;
}
