// Host side of the libvqlin C ABI: validation, repacking, device upload,
// bit accounting, errors and dispatch.  The arithmetic of every call runs in
// the kernels of k_*.cu; create-time preparation runs here.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "vqlin_internal.cuh"

namespace vqlin {

static thread_local std::string g_err;
static std::atomic<uint64_t> g_kernel_launches{0};

void note_launches(int n) { g_kernel_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
}

vqlin_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return VQLIN_OK;
  set_error("%s: %s", what, cudaGetErrorString(e));
  return e == cudaErrorMemoryAllocation ? VQLIN_ERR_OOM : VQLIN_ERR_CUDA;
}

namespace {

// fp16 bits -> double (exact); false for inf/NaN.
bool f16_finite(uint16_t h) { return ((h >> 10) & 0x1F) != 31; }
double f16_val(uint16_t h) { return (double)__half2float(__ushort_as_half(h)); }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

uint32_t host_field(const uint8_t* row, int64_t s, int w) {
  int64_t bit = s * (int64_t)w;
  uint64_t v = 0;
  int nbytes = (int)(((bit & 7) + w + 7) >> 3);
  for (int t = 0; t < nbytes; ++t) v |= (uint64_t)row[(bit >> 3) + t] << (8 * t);
  v >>= (bit & 7);
  return w >= 32 ? (uint32_t)v : (uint32_t)(v & ((1ull << w) - 1ull));
}

void host_put_field(uint8_t* row, int64_t k, int w, uint32_t v) {
  int64_t bit = k * (int64_t)w;
  for (int b = 0; b < w; ++b, ++bit)
    if ((v >> b) & 1u) row[bit >> 3] |= (uint8_t)(1u << (bit & 7));
}

// Copy `bytes` from a caller buffer (device or host) into a host vector.
vqlin_status fetch(const void* src, size_t bytes, bool on_host, std::vector<uint8_t>& dst, const char* what) {
  dst.resize(bytes);
  if (bytes == 0) return VQLIN_OK;
  if (!src) {
    set_error("%s is NULL", what);
    return VQLIN_ERR_INVALID_ARG;
  }
  if (on_host) {
    memcpy(dst.data(), src, bytes);
    return VQLIN_OK;
  }
  return cuda_status(cudaMemcpy(dst.data(), src, bytes, cudaMemcpyDeviceToHost), what);
}

template <class T>
const T* as(const std::vector<uint8_t>& v) { return reinterpret_cast<const T*>(v.data()); }

struct Uploader {
  vqlin_handle* h;
  vqlin_status st = VQLIN_OK;
  template <class T>
  T* put(const void* src, size_t bytes, size_t pad = 16) {
    if (st != VQLIN_OK || bytes == 0) return nullptr;
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, bytes + pad);
    if (e != cudaSuccess) { st = cuda_status(e, "cudaMalloc"); return nullptr; }
    h->allocs[h->n_allocs++] = p;
    e = cudaMemset(p, 0, bytes + pad);
    if (e == cudaSuccess && src) e = cudaMemcpy(p, src, bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { st = cuda_status(e, "upload"); return nullptr; }
    return reinterpret_cast<T*>(p);
  }
};

}  // namespace
}  // namespace vqlin

using namespace vqlin;

extern "C" {

const char* vqlin_status_string(vqlin_status s) {
  switch (s) {
    case VQLIN_OK: return "ok";
    case VQLIN_ERR_INVALID_ARG: return "invalid argument";
    case VQLIN_ERR_UNSUPPORTED: return "unsupported";
    case VQLIN_ERR_INVALID_DATA: return "invalid data";
    case VQLIN_ERR_OOM: return "out of memory";
    case VQLIN_ERR_CUDA: return "CUDA error";
    case VQLIN_ERR_WORKSPACE: return "bad workspace";
  }
  return "unknown status";
}

const char* vqlin_last_error(void) { return g_err.c_str(); }

vqlin_status vqlin_device_error(int32_t* code) {
  if (!code) { set_error("code is NULL"); return VQLIN_ERR_INVALID_ARG; }
  vqlin_status st = cuda_status(cudaDeviceSynchronize(), "device synchronize");
  if (st) return st;
  int v = read_and_clear_device_error();
  int w = read_and_clear_cs_error();
  if (v < 0 || w < 0) { set_error("cannot read the device error words"); return VQLIN_ERR_CUDA; }
  *code = v ? v : w;
  return VQLIN_OK;
}
int32_t vqlin_abi_version(void) { return VQLIN_ABI_VERSION; }

uint64_t vqlin_kernel_launches(void) { return vqlin::g_kernel_launches.load(std::memory_order_relaxed); }

vqlin_status vqlin_destroy(vqlin_handle* h) {
  if (!h) return VQLIN_OK;
  int dev = -1;
  cudaGetDevice(&dev);
  cudaSetDevice(h->device);
  for (int i = 0; i < h->n_allocs; ++i) cudaFree(h->allocs[i]);
  if (dev >= 0) cudaSetDevice(dev);
  delete h;
  return VQLIN_OK;
}

vqlin_status vqlin_create(const vqlin_desc* D, void* stream, vqlin_handle** out) {
  if (out) *out = nullptr;
  if (!D || !out) { set_error("desc and out must not be NULL"); return VQLIN_ERR_INVALID_ARG; }
  const bool host = D->src_on_host != 0;
  // ---- shape checks
  if (D->n_out < 1 || D->n_in < 1) { set_error("n_out and n_in must be >= 1"); return VQLIN_ERR_INVALID_ARG; }
  if (D->d < 1 || D->d > 64) { set_error("d = %d out of range", D->d); return VQLIN_ERR_INVALID_ARG; }
  if (D->d != 4 && D->d != 6 && D->d != 8 && D->d != 12) {
    set_error("d = %d: kernels support d in {4, 6, 8, 12}", D->d);
    return VQLIN_ERR_UNSUPPORTED;
  }
  if (D->bits1 < 1 || D->bits1 > 16 || D->k1 < 1 || (int64_t)D->k1 > (1ll << D->bits1)) {
    set_error("need 1 <= bits1 <= 16 and 1 <= k1 <= 2^bits1 (k1 = %d, bits1 = %d)", D->k1, D->bits1);
    return VQLIN_ERR_INVALID_ARG;
  }
  if (D->k2 < 0 || D->bits2 < 0 || (D->k2 == 0) != (D->bits2 == 0) ||
      (D->k2 > 0 && (D->bits2 > 16 || (int64_t)D->k2 > (1ll << D->bits2)))) {
    set_error("residual codebook: need k2 = bits2 = 0, or 1 <= bits2 <= 16 and 1 <= k2 <= 2^bits2");
    return VQLIN_ERR_INVALID_ARG;
  }
  if (D->n_ocols < 0 || D->n_ocols > D->n_in) { set_error("n_ocols out of range"); return VQLIN_ERR_INVALID_ARG; }
  if (D->n_ocols > 0 && (D->bits_o < 1 || D->bits_o > 16 || D->ko < 1 || (int64_t)D->ko > (1ll << D->bits_o))) {
    set_error("outlier block: need 1 <= bits_o <= 16 and 1 <= ko <= 2^bits_o");
    return VQLIN_ERR_INVALID_ARG;
  }
  if (D->nnz < 0 || D->nnz > (int64_t)D->n_out * D->n_in || D->nnz > 0x7FFFFFFFll) {
    set_error("nnz out of range");
    return VQLIN_ERR_INVALID_ARG;
  }
  if (D->n_in == D->n_ocols && D->n_ocols > 0) { /* all columns in the outlier block: fine */ }
  const int d = D->d, w = D->bits1 + D->bits2;
  const int32_t n_main = D->n_in - D->n_ocols;
  const int32_t n_sub = (int32_t)ceil_div(n_main, d);
  // codebook groups and the symmetric codebook
  const int32_t G = D->n_groups > 1 ? D->n_groups : 1;
  if (D->n_groups < 0 || (G > 1 && G > n_sub)) {
    set_error("n_groups = %d: need 0 or 1 <= n_groups <= n_sub = %d", D->n_groups, n_sub);
    return VQLIN_ERR_INVALID_ARG;
  }
  if (D->cb_symmetry != 0 && (D->cb_symmetry != 1 || D->k1 % 4 != 0)) {
    set_error("cb_symmetry must be 0, or 1 with k1 %% 4 == 0 (k1 = %d)", D->k1);
    return VQLIN_ERR_INVALID_ARG;
  }
  const int32_t k1s = D->cb_symmetry ? D->k1 / 4 : D->k1;   // stored entries per group
  const int32_t g_size = G > 1 ? (int32_t)ceil_div(n_sub, G) : (n_sub > 0 ? n_sub : 1);
  if (D->vsr_nblocks < 0 || D->vsr_nblocks > (int64_t)D->n_out * n_sub || D->vsr_nblocks > 0x7FFFFFFFll) {
    set_error("vsr_nblocks out of range");
    return VQLIN_ERR_INVALID_ARG;
  }
  const int32_t n_sub_o = (int32_t)ceil_div(D->n_ocols, d);
  const int64_t row_bytes = ceil_div((int64_t)n_sub * w, 8);
  const int64_t row_bytes_o = ceil_div((int64_t)n_sub_o * D->bits_o, 8);
  if (n_sub > 0 && D->row_stride_bytes < row_bytes) {
    set_error("row_stride_bytes = %lld < %lld", (long long)D->row_stride_bytes, (long long)row_bytes);
    return VQLIN_ERR_INVALID_ARG;
  }
  if (n_sub_o > 0 && D->o_row_stride_bytes < row_bytes_o) {
    set_error("o_row_stride_bytes too small");
    return VQLIN_ERR_INVALID_ARG;
  }

  int prev_dev = 0;
  cudaGetDevice(&prev_dev);
  // ---- bring everything to the host
  std::vector<uint8_t> codes, cb1, cb2, cbo, codes_o, rs, cs, ocols, rp, ci, vals, vrp, vpos, vvals;
  vqlin_status st = VQLIN_OK;
  if (n_sub > 0) st = fetch(D->codes, (size_t)D->row_stride_bytes * D->n_out, host, codes, "codes");
  if (!st) st = fetch(D->codebook1, (size_t)G * k1s * d * 2, host, cb1, "codebook1");
  if (!st && D->k2) st = fetch(D->codebook2, (size_t)G * D->k2 * d * 2, host, cb2, "codebook2");
  if (!st && D->row_scale) st = fetch(D->row_scale, (size_t)D->n_out * 2, host, rs, "row_scale");
  if (!st && D->col_scale) st = fetch(D->col_scale, (size_t)D->n_in * 2, host, cs, "col_scale");
  if (!st && D->n_ocols) {
    st = fetch(D->ocols, (size_t)D->n_ocols * 4, host, ocols, "ocols");
    if (!st) st = fetch(D->codebook_o, (size_t)D->ko * d * 2, host, cbo, "codebook_o");
    if (!st) st = fetch(D->codes_o, (size_t)D->o_row_stride_bytes * D->n_out, host, codes_o, "codes_o");
  }
  if (!st && D->nnz) {
    st = fetch(D->row_ptr, (size_t)(D->n_out + 1) * 4, host, rp, "row_ptr");
    if (!st) st = fetch(D->col_idx, (size_t)D->nnz * 4, host, ci, "col_idx");
    if (!st) st = fetch(D->values, (size_t)D->nnz * 2, host, vals, "values");
  }
  if (!st && D->vsr_nblocks) {
    st = fetch(D->vsr_row_ptr, (size_t)(D->n_out + 1) * 4, host, vrp, "vsr_row_ptr");
    if (!st) st = fetch(D->vsr_pos, (size_t)D->vsr_nblocks * 4, host, vpos, "vsr_pos");
    if (!st) st = fetch(D->vsr_values, (size_t)D->vsr_nblocks * d * 2, host, vvals, "vsr_values");
  }
  if (st) return st;

  // ---- validate values
  auto finite_all = [](const std::vector<uint8_t>& v) {
    const uint16_t* p = as<uint16_t>(v);
    for (size_t i = 0; i < v.size() / 2; ++i) if (!f16_finite(p[i])) return false;
    return true;
  };
  if (!finite_all(cb1) || !finite_all(cb2) || !finite_all(cbo) || !finite_all(rs) || !finite_all(cs) ||
      !finite_all(vvals)) {
    set_error("a codebook, scale or VSR entry is inf or NaN");
    return VQLIN_ERR_INVALID_DATA;
  }
  // A symmetric codebook holds k1/4 base entries per group; entry t * (k1/4) + b of the k1 that
  // the indices address is base entry b under sign pattern t (0 none, 1 all elements negated, 2
  // odd elements negated, 3 even elements negated).  Negating fp16 flips its sign bit, so the
  // expansion is exact; every kernel then reads k1 entries per group.
  if (D->cb_symmetry) {
    std::vector<uint8_t> full((size_t)G * D->k1 * d * 2);
    const uint16_t* base = as<uint16_t>(cb1);
    uint16_t* out16 = reinterpret_cast<uint16_t*>(full.data());
    for (int32_t g = 0; g < G; ++g)
      for (int32_t t = 0; t < 4; ++t)
        for (int32_t b = 0; b < k1s; ++b)
          for (int e = 0; e < d; ++e) {
            const bool neg = t == 1 || (t == 2 && (e & 1)) || (t == 3 && !(e & 1));
            const uint16_t v = base[((size_t)g * k1s + b) * d + e];
            out16[(((size_t)g * D->k1) + (size_t)t * k1s + b) * d + e] = neg ? (uint16_t)(v ^ 0x8000u) : v;
          }
    cb1.swap(full);
  }
  // column classification
  std::vector<int32_t> colmap;   // main ids then outlier ids
  std::vector<int32_t> rank(D->n_in), is_out(D->n_in, 0);
  if (D->n_ocols) {
    const int32_t* oc = as<int32_t>(ocols);
    for (int32_t t = 0; t < D->n_ocols; ++t) {
      if (oc[t] < 0 || oc[t] >= D->n_in || (t > 0 && oc[t - 1] >= oc[t])) {
        set_error("ocols must be strictly increasing and in [0, n_in)");
        return VQLIN_ERR_INVALID_DATA;
      }
      is_out[oc[t]] = 1;
    }
    colmap.reserve(D->n_in);
    for (int32_t j = 0; j < D->n_in; ++j) if (!is_out[j]) colmap.push_back(j);
    for (int32_t t = 0; t < D->n_ocols; ++t) colmap.push_back(oc[t]);
  }
  {
    int32_t p = 0, q = 0;
    for (int32_t j = 0; j < D->n_in; ++j) rank[j] = is_out[j] ? p++ : q++;
  }
  // indices in range (and repack rows to a 16-byte stride)
  const int64_t stride = round_up(std::max<int64_t>(row_bytes, 1), 16);
  const int64_t stride_o = round_up(std::max<int64_t>(row_bytes_o, 1), 16);
  std::vector<uint8_t> codes_r((size_t)stride * D->n_out, 0), codes_o_r;
  const uint32_t m1 = (1u << D->bits1) - 1u;
  for (int32_t i = 0; i < D->n_out && n_sub > 0; ++i) {
    const uint8_t* row = codes.data() + (size_t)i * D->row_stride_bytes;
    memcpy(codes_r.data() + (size_t)i * stride, row, (size_t)row_bytes);
    // clear the bits past the last field so the repacked rows are canonical
    int64_t used_bits = (int64_t)n_sub * w;
    if (used_bits & 7) codes_r[(size_t)i * stride + (used_bits >> 3)] &= (uint8_t)((1u << (used_bits & 7)) - 1u);
    for (int32_t s = 0; s < n_sub; ++s) {
      uint32_t f = host_field(row, s, w);
      uint32_t i1 = f & m1, i2 = D->bits2 ? (f >> D->bits1) : 0;
      if (i1 >= (uint32_t)D->k1 || (D->k2 && i2 >= (uint32_t)D->k2)) {
        set_error("row %d sub-vector %d: index (%u, %u) out of range", i, s, i1, i2);
        return VQLIN_ERR_INVALID_DATA;
      }
    }
  }
  if (D->n_ocols) {
    codes_o_r.assign((size_t)stride_o * D->n_out, 0);
    for (int32_t i = 0; i < D->n_out; ++i) {
      const uint8_t* row = codes_o.data() + (size_t)i * D->o_row_stride_bytes;
      memcpy(codes_o_r.data() + (size_t)i * stride_o, row, (size_t)row_bytes_o);
      int64_t used_bits = (int64_t)n_sub_o * D->bits_o;
      if (used_bits & 7) codes_o_r[(size_t)i * stride_o + (used_bits >> 3)] &= (uint8_t)((1u << (used_bits & 7)) - 1u);
      for (int32_t s = 0; s < n_sub_o; ++s)
        if (host_field(row, s, D->bits_o) >= (uint32_t)D->ko) {
          set_error("row %d outlier sub-vector %d: index out of range", i, s);
          return VQLIN_ERR_INVALID_DATA;
        }
    }
  }
  // CSR structure and the fused correction delta = v - body (double, stored fp32)
  std::vector<float> delta((size_t)D->nnz);
  std::vector<uint16_t> col16;
  if (D->nnz) {
    const int32_t* r = as<int32_t>(rp);
    const int32_t* c = as<int32_t>(ci);
    const uint16_t* v = as<uint16_t>(vals);
    if (r[0] != 0 || r[D->n_out] != D->nnz) { set_error("row_ptr must start at 0 and end at nnz"); return VQLIN_ERR_INVALID_DATA; }
    const uint16_t* C1 = as<uint16_t>(cb1);
    const uint16_t* C2 = D->k2 ? as<uint16_t>(cb2) : nullptr;
    const uint16_t* CO = D->n_ocols ? as<uint16_t>(cbo) : nullptr;
    for (int32_t i = 0; i < D->n_out; ++i) {
      if (r[i + 1] < r[i]) { set_error("row_ptr decreases at row %d", i); return VQLIN_ERR_INVALID_DATA; }
      double ri = D->row_scale ? f16_val(as<uint16_t>(rs)[i]) : 1.0;
      for (int32_t e = r[i]; e < r[i + 1]; ++e) {
        int32_t j = c[e];
        if (j < 0 || j >= D->n_in || (e > r[i] && c[e - 1] >= j)) {
          set_error("row %d: CSR columns must be strictly increasing and in [0, n_in)", i);
          return VQLIN_ERR_INVALID_DATA;
        }
        if (!f16_finite(v[e])) { set_error("CSR value %d is inf or NaN", e); return VQLIN_ERR_INVALID_DATA; }
        double body;
        if (is_out[j]) {
          int32_t p = rank[j];
          uint32_t io = host_field(codes_o.data() + (size_t)i * D->o_row_stride_bytes, p / d, D->bits_o);
          body = f16_val(CO[(size_t)io * d + p % d]);
        } else {
          int32_t q = rank[j];
          uint32_t f = host_field(codes.data() + (size_t)i * D->row_stride_bytes, q / d, w);
          const size_t g = (size_t)((q / d) / g_size);
          body = f16_val(C1[(g * D->k1 + (f & m1)) * d + q % d]);
          if (C2) body += f16_val(C2[(g * D->k2 + (f >> D->bits1)) * d + q % d]);
        }
        body *= ri;
        if (D->col_scale) body *= f16_val(as<uint16_t>(cs)[j]);
        delta[e] = (float)(f16_val(v[e]) - body);
      }
    }
    if (D->n_in <= 65536) {
      col16.resize((size_t)D->nnz);
      for (int64_t e = 0; e < D->nnz; ++e) col16[e] = (uint16_t)c[e];
    }
  }

  // VSR blocks: structure, no element shared with the CSR matrix, and the fused-product form
  // delta = v - body per element (double, stored fp32; 0 past the last main column)
  std::vector<float> vdelta((size_t)D->vsr_nblocks * d, 0.f);
  if (D->vsr_nblocks) {
    const int32_t* r = as<int32_t>(vrp);
    const int32_t* ps = as<int32_t>(vpos);
    const uint16_t* vv = as<uint16_t>(vvals);
    const uint16_t* C1 = as<uint16_t>(cb1);
    const uint16_t* C2 = D->k2 ? as<uint16_t>(cb2) : nullptr;
    if (r[0] != 0 || r[D->n_out] != D->vsr_nblocks) { set_error("vsr_row_ptr must start at 0 and end at vsr_nblocks"); return VQLIN_ERR_INVALID_DATA; }
    std::vector<int32_t> main_col(n_main);
    for (int32_t j = 0; j < D->n_in; ++j) if (!is_out[j]) main_col[rank[j]] = j;
    const int32_t* cr = D->nnz ? as<int32_t>(rp) : nullptr;
    const int32_t* cc = D->nnz ? as<int32_t>(ci) : nullptr;
    for (int32_t i = 0; i < D->n_out; ++i) {
      if (r[i + 1] < r[i]) { set_error("vsr_row_ptr decreases at row %d", i); return VQLIN_ERR_INVALID_DATA; }
      const double ri = D->row_scale ? f16_val(as<uint16_t>(rs)[i]) : 1.0;
      int32_t e = cr ? cr[i] : 0;
      const int32_t e_end = cr ? cr[i + 1] : 0;
      for (int32_t b = r[i]; b < r[i + 1]; ++b) {
        const int32_t sv = ps[b];
        if (sv < 0 || sv >= n_sub || (b > r[i] && ps[b - 1] >= sv)) {
          set_error("row %d: VSR positions must be strictly increasing and in [0, n_sub)", i);
          return VQLIN_ERR_INVALID_DATA;
        }
        const uint32_t f = host_field(codes.data() + (size_t)i * D->row_stride_bytes, sv, w);
        const size_t g = (size_t)(sv / g_size);
        for (int t = 0; t < d; ++t) {
          const int32_t q = sv * d + t;
          if (q >= n_main) break;
          const int32_t j = main_col[q];
          while (e < e_end && cc[e] < j) ++e;           // CSR columns of the row, increasing
          if (e < e_end && cc[e] == j) {
            set_error("row %d column %d is in both the CSR matrix and a VSR block", i, j);
            return VQLIN_ERR_INVALID_DATA;
          }
          double body = f16_val(C1[(g * D->k1 + (f & m1)) * d + t]);
          if (C2) body += f16_val(C2[(g * D->k2 + (f >> D->bits1)) * d + t]);
          body *= ri;
          if (D->col_scale) body *= f16_val(as<uint16_t>(cs)[j]);
          vdelta[(size_t)b * d + t] = (float)(f16_val(vv[(size_t)b * d + t]) - body);
        }
      }
    }
  }

  // tensor-core decode layout (see vqlin_internal.cuh).  Its kernels work on 8-wide parts: for
  // d != 8 every sub-vector becomes V = ceil(d / 8) parts, zero-padded, each with its own entry of
  // a padded codebook (entry k, part h at k * V + h); x' is then staged through a map from the
  // layout's columns to the layer's (padding to none).  With codebook groups (or parts) the fields
  // hold (g * k1 + i1) * V + h | ((g * k2 + i2) * V + h) << tc_b1, widened to the next width the
  // kernels take.  Outlier-column blocks are decoded there only at d = 8.
  std::vector<uint8_t> tcodes;
  std::vector<uint16_t> tcb1, tcb2;                 // padded codebooks (d != 8 only)
  std::vector<int32_t> tcmap;                       // layout column -> layer column or -1 (d != 8)
  int32_t n_ls = 0;
  int64_t tstride = 0;
  const int V = (d + 7) / 8;
  const int32_t tc_nsub = n_sub * V;
  int tc_b1 = D->bits1, tc_w = w;
  if (G > 1 || V > 1) {
    auto bits_for = [](int64_t n) { int b = 1; while ((1ll << b) < n) ++b; return b; };
    tc_b1 = bits_for((int64_t)G * D->k1 * V);
    const int need = tc_b1 + (D->k2 ? bits_for((int64_t)G * D->k2 * V) : 0);
    tc_w = need <= 8 ? 8 : need <= 12 ? 12 : need <= 16 ? 16 : need <= 24 ? 24 : need <= 32 ? 32 : 0;
  }
  const bool tc_geom = d == 8 || D->n_ocols == 0;
  if (tc_geom && n_sub > 0 && (tc_w == 8 || tc_w == 12 || tc_w == 16 || tc_w == 24 || tc_w == 32)) {
    n_ls = (int32_t)ceil_div(tc_nsub, 64);
    tstride = (int64_t)n_ls * 8 * tc_w;
    const int64_t rows_pad = round_up(D->n_out, 16);
    tcodes.assign((size_t)(rows_pad * tstride), 0);
    for (int32_t i = 0; i < D->n_out; ++i) {
      const uint8_t* row = codes.data() + (size_t)i * D->row_stride_bytes;
      uint8_t* dst = tcodes.data() + (size_t)i * tstride;
      for (int32_t ls = 0; ls < n_ls; ++ls)
        for (int t = 0; t < 4; ++t)
          for (int ps = 0; ps < 16; ++ps) {
            const int32_t vsv = 64 * ls + 4 * ps + t;          // part index in the layout
            if (vsv >= tc_nsub) continue;   // padding fields stay 0 (a valid index; x' is 0 there)
            const int32_t sv = vsv / V, h = vsv - sv * V;
            uint32_t f = host_field(row, sv, w);
            if (G > 1 || V > 1) {
              const uint32_t g = (uint32_t)(sv / g_size);
              f = ((g * (uint32_t)D->k1 + (f & m1)) * (uint32_t)V + (uint32_t)h) |
                  ((D->k2 ? (g * (uint32_t)D->k2 + (f >> D->bits1)) * (uint32_t)V + (uint32_t)h : 0u) << tc_b1);
            }
            host_put_field(dst, (int64_t)ls * 64 + t * 16 + ps, tc_w, f);
          }
    }
    if (d != 8) {
      auto pad = [&](const std::vector<uint8_t>& cb, int64_t entries, std::vector<uint16_t>& out) {
        const uint16_t* c = as<uint16_t>(cb);
        out.assign((size_t)entries * V * 8, 0);
        for (int64_t k = 0; k < entries; ++k)
          for (int h = 0; h < V; ++h)
            for (int e = 0; e < 8 && 8 * h + e < d; ++e) out[((size_t)k * V + h) * 8 + e] = c[(size_t)k * d + 8 * h + e];
      };
      pad(cb1, (int64_t)G * D->k1, tcb1);
      if (D->k2) pad(cb2, (int64_t)G * D->k2, tcb2);
      tcmap.assign((size_t)tc_nsub * 8, -1);
      for (int32_t c = 0; c < tc_nsub * 8; ++c) {
        const int32_t vsv = c / 8, k = c % 8, sv = vsv / V, h = vsv - sv * V, e = 8 * h + k, q = sv * d + e;
        if (e < d && q < n_main) tcmap[c] = q;      // no outlier block here, so main column q is column q
      }
    }
  }

  // codebook-stationary layout for large single-stage codebooks (see vqlin_internal.cuh)
  std::vector<uint64_t> cs_words;
  std::vector<int64_t> cs_start;
  std::vector<uint16_t> cs_wpos;
  std::vector<float> cs_bound;
  int32_t cs_P = 0, cs_H = 0, cs_E = 0, cs_rpp = 0, cs_lbits = 0, cs_ebits = 0, cs_epw = 0;
  // the codebook-stationary layout indexes the virtual codebook of all groups, g * k1 + i1
  const int64_t kv = (int64_t)G * D->k1;
  if (d == 8 && D->k2 == 0 && kv > 10240 && kv <= (1 << 24) && n_sub > 0 && n_sub <= 65536) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    auto bitlen = [](int64_t v) { int b = 0; while ((1ll << b) <= v) ++b; return b < 1 ? 1 : b; };
    const int H = D->n_out >= 2048 ? 2 : 1;
    int P = (int)std::max<int64_t>(ceil_div(kv, 1023), std::max(1, sms / H));
    P = (int)std::min<int64_t>(P, kv);
    const int E = (int)ceil_div(kv, P);
    P = (int)ceil_div(kv, E);
    const int rpp = (int)ceil_div(D->n_out, H);
    const int lb = bitlen(E), rb = bitlen(rpp - 1), eb = lb + rb;   // local indices 0..E (E = null entry)
    const int epw = eb <= 21 ? 3 : (eb <= 32 ? 2 : 0);
    if (epw && rpp <= 65535) {
      const int ncta = P * H;
      const int slot = epw == 3 ? 21 : 32;
      const uint32_t null_entry = (uint32_t)E;                  // row 0, zero centroid
      std::vector<std::vector<uint64_t>> bw(ncta);              // words of every block
      std::vector<std::vector<uint16_t>> bp(ncta);              // their positions
      std::vector<int> fill(ncta, 0);                           // entries in the block's open word
      std::vector<int32_t> per_row((size_t)ncta * rpp, 0);      // entries of every (block, row)
      auto put = [&](int cc, uint32_t ent, int32_t sv) {
        if (fill[cc] == 0) { bw[cc].push_back(0); bp[cc].push_back((uint16_t)sv); }
        bw[cc].back() |= (uint64_t)ent << (fill[cc] * slot);
        fill[cc] = (fill[cc] + 1) % epw;
      };
      for (int32_t sv = 0; sv < n_sub; ++sv) {
        for (int32_t i = 0; i < D->n_out; ++i) {
          uint32_t idx = (uint32_t)((sv / g_size) * D->k1) + (host_field(codes.data() + (size_t)i * D->row_stride_bytes, sv, w) & m1);
          const int pp = (int)(idx / (uint32_t)E), hh = i / rpp, cc = pp * H + hh;
          put(cc, ((uint32_t)(i - hh * rpp) << lb) | (idx - (uint32_t)pp * E), sv);
          per_row[(size_t)cc * rpp + (i - hh * rpp)] += 1;
        }
        for (int cc = 0; cc < ncta; ++cc)   // close the run of position sv
          while (fill[cc] != 0) put(cc, null_entry, sv);
      }
      // Fixed-point bound of every block: (most entries of one row in the block) * (largest l1
      // norm of a centroid of its slice).  Every product satisfies |c . x'| <= l1(c) * max|x'|,
      // so a row's partial sum in the block stays below bound * max|x'|.
      const uint16_t* C1 = as<uint16_t>(cb1);
      std::vector<double> l1(P, 0.0);
      for (int32_t k = 0; k < (int32_t)kv; ++k) {
        double a1 = 0;
        for (int t = 0; t < 8; ++t) a1 += std::fabs(f16_val(C1[(size_t)k * 8 + t]));
        l1[k / E] = std::max(l1[k / E], a1);
      }
      std::vector<float> bound(ncta, 0.f);
      int64_t max_cnt = 0;
      for (int cc = 0; cc < ncta; ++cc) {
        int32_t m = 0;
        for (int r = 0; r < rpp; ++r) m = std::max(m, per_row[(size_t)cc * rpp + r]);
        max_cnt = std::max<int64_t>(max_cnt, m);
        bound[cc] = std::nextafter((float)((double)m * l1[cc / H]), INFINITY);
      }
      // A row's fixed-point rounding error is at most n_sub * max_cnt * 2^-31 times the
      // largest possible single product (k_gemv_cs.cu); past 2^20 the layout is not used.
      if ((int64_t)n_sub * max_cnt <= (1ll << 20)) {
        cs_P = P; cs_H = H; cs_E = E; cs_rpp = rpp; cs_lbits = lb; cs_ebits = eb; cs_epw = epw;
        uint64_t null_word = 0;
        for (int u = 0; u < epw; ++u) null_word |= (uint64_t)null_entry << (u * slot);
        const uint64_t emask = (1ull << eb) - 1ull;
        cs_start.assign(ncta + 1, 0);
        for (int cc = 0; cc < ncta; ++cc) {
          // whole groups of 32 words (one warp instruction covers one group)
          while (bw[cc].size() % 32) { bw[cc].push_back(null_word); bp[cc].push_back(0); }
          cs_start[cc + 1] = cs_start[cc] + (int64_t)bw[cc].size();
          // Inside a group, deal the entries of every position run to the slots so that the
          // rows that one slot column sends to the shared-memory accumulator fall in different
          // banks (row mod 32): greedy, each entry to the open slot whose column holds the
          // fewest rows of its bank so far.
          for (size_t g0 = 0; g0 < bw[cc].size(); g0 += 32) {
            int cnt[3][32] = {};
            size_t w = g0;
            while (w < g0 + 32) {
              size_t w1 = w + 1;
              while (w1 < g0 + 32 && bp[cc][w1] == bp[cc][w]) ++w1;
              const int m = (int)(w1 - w);
              std::vector<uint32_t> ents;
              for (size_t q = w; q < w1; ++q)
                for (int u = 0; u < epw; ++u) {
                  const uint32_t e = (uint32_t)((bw[cc][q] >> (u * slot)) & emask);
                  if ((e & ((1u << lb) - 1u)) != null_entry) ents.push_back(e);
                }
              std::vector<std::vector<uint32_t>> col(epw);
              for (uint32_t e : ents) {
                const int bank = (int)((e >> lb) & 31u);
                int best = -1;
                for (int u = 0; u < epw; ++u) {
                  if ((int)col[u].size() >= m) continue;
                  if (best < 0 || cnt[u][bank] < cnt[best][bank] ||
                      (cnt[u][bank] == cnt[best][bank] && col[u].size() < col[best].size()))
                    best = u;
                }
                col[best].push_back(e);
                cnt[best][bank] += 1;
              }
              for (int j = 0; j < m; ++j) {
                uint64_t word = 0;
                for (int u = 0; u < epw; ++u)
                  word |= (uint64_t)(j < (int)col[u].size() ? col[u][j] : null_entry) << (u * slot);
                bw[cc][w + j] = word;
              }
              w = w1;
            }
          }
        }
        cs_words.assign((size_t)cs_start[ncta], null_word);
        cs_wpos.assign(cs_words.size(), 0);
        for (int cc = 0; cc < ncta; ++cc) {
          std::copy(bw[cc].begin(), bw[cc].end(), cs_words.begin() + cs_start[cc]);
          std::copy(bp[cc].begin(), bp[cc].end(), cs_wpos.begin() + cs_start[cc]);
        }
        cs_bound = std::move(bound);
      }
    }
  }

  // ---- upload
  vqlin_handle* h = new vqlin_handle();
  memset(h, 0, sizeof *h);
  cudaGetDevice(&h->device);
  Uploader up{h};
  Layer& L = h->L;
  L.n_out = D->n_out; L.n_in = D->n_in; L.d = d;
  L.k1 = D->k1; L.bits1 = D->bits1; L.k2 = D->k2; L.bits2 = D->bits2; L.w = w;
  L.n_main = n_main; L.n_sub = n_sub;
  L.n_ocols = D->n_ocols; L.n_sub_o = n_sub_o; L.ko = D->n_ocols ? D->ko : 0; L.bits_o = D->n_ocols ? D->bits_o : 0;
  L.stride = stride; L.stride_o = D->n_ocols ? stride_o : 0;
  L.codes = up.put<uint8_t>(codes_r.data(), codes_r.size());
  L.codes_o = D->n_ocols ? up.put<uint8_t>(codes_o_r.data(), codes_o_r.size()) : nullptr;
  L.n_groups = G;
  L.g_size = g_size;
  L.g_magic = g_size > 1 ? (uint32_t)(((1ull << 32) + (uint64_t)g_size - 1) / (uint64_t)g_size) : 0u;
  L.cb1 = up.put<__half>(cb1.data(), cb1.size());
  L.cb2 = D->k2 ? up.put<__half>(cb2.data(), cb2.size()) : nullptr;
  L.cbo = D->n_ocols ? up.put<__half>(cbo.data(), cbo.size()) : nullptr;
  L.rs = D->row_scale ? up.put<__half>(rs.data(), rs.size()) : nullptr;
  L.cs = D->col_scale ? up.put<__half>(cs.data(), cs.size()) : nullptr;
  L.colmap = D->n_ocols ? up.put<int32_t>(colmap.data(), colmap.size() * 4) : nullptr;
  L.nnz = D->nnz;
  if (D->nnz) {
    L.row_ptr = up.put<int32_t>(rp.data(), rp.size());
    L.col = up.put<int32_t>(ci.data(), ci.size());
    L.val = up.put<uint16_t>(vals.data(), vals.size());
    L.delta = up.put<float>(delta.data(), delta.size() * 4);
    L.col16 = col16.empty() ? nullptr : up.put<uint16_t>(col16.data(), col16.size() * 2);
  }
  L.vsr_nb = D->vsr_nblocks;
  if (D->vsr_nblocks) {
    L.vsr_rp = up.put<int32_t>(vrp.data(), vrp.size());
    L.vsr_pos = up.put<int32_t>(vpos.data(), vpos.size());
    L.vsr_val = up.put<uint16_t>(vvals.data(), vvals.size());
    L.vsr_delta = up.put<float>(vdelta.data(), vdelta.size() * 4);
  }
  if (D->nnz && gemm_fused_supported(L)) {
    // the CSR entries by 64-column K-block for the fused prefill GEMM
    const int32_t nkb = (D->n_in + 63) / 64;
    std::vector<int32_t> kbs((size_t)D->n_out * (nkb + 1));
    std::vector<uint32_t> kbe((size_t)D->nnz);
    const int32_t* r = as<int32_t>(rp);
    const int32_t* c = as<int32_t>(ci);
    const uint16_t* v = as<uint16_t>(vals);
    for (int32_t i = 0; i < D->n_out; ++i) {
      int32_t e = r[i];
      for (int32_t kb = 0; kb <= nkb; ++kb) {
        while (e < r[i + 1] && c[e] < kb * 64) ++e;
        kbs[(size_t)i * (nkb + 1) + kb] = e;
      }
    }
    for (int64_t e = 0; e < D->nnz; ++e) kbe[e] = ((uint32_t)(c[e] & 63) << 16) | v[e];
    L.kb_start = up.put<int32_t>(kbs.data(), kbs.size() * 4);
    L.kb_entry = up.put<uint32_t>(kbe.data(), kbe.size() * 4);
  }
  L.tcodes = tcodes.empty() ? nullptr : up.put<uint8_t>(tcodes.data(), tcodes.size());
  if (!cs_words.empty()) {
    L.cs_words = up.put<uint64_t>(cs_words.data(), cs_words.size() * 8);
    L.cs_start = up.put<int64_t>(cs_start.data(), cs_start.size() * 8);
    L.cs_wpos = up.put<uint16_t>(cs_wpos.data(), cs_wpos.size() * 2);
    L.cs_bound = up.put<float>(cs_bound.data(), cs_bound.size() * 4);
    L.cs_P = cs_P; L.cs_H = cs_H; L.cs_E = cs_E; L.cs_rpp = cs_rpp;
    L.cs_local_bits = cs_lbits; L.cs_ebits = cs_ebits; L.cs_epw = cs_epw;
    L.cs_max_words = 0;
    for (size_t cc = 0; cc + 1 < cs_start.size(); ++cc)
      L.cs_max_words = std::max<int64_t>(L.cs_max_words, cs_start[cc + 1] - cs_start[cc]);
  }
  L.n_ls = n_ls;
  L.tstride = tstride;
  L.tc_w = tcodes.empty() ? 0 : tc_w;
  L.tc_bits1 = tc_b1;
  L.tc_nsub = tcodes.empty() ? 0 : tc_nsub;
  L.tc_k1 = G * D->k1 * V;
  L.tc_k2 = G * D->k2 * V;
  L.tc_cb1 = tcb1.empty() ? L.cb1 : up.put<__half>(tcb1.data(), tcb1.size() * 2);
  L.tc_cb2 = tcb2.empty() ? L.cb2 : up.put<__half>(tcb2.data(), tcb2.size() * 2);
  L.tc_colmap = tcmap.empty() ? nullptr : up.put<int32_t>(tcmap.data(), tcmap.size() * 4);
  L.tcodes_rows = tcodes.empty() ? 0 : (int32_t)round_up(D->n_out, 16);
  if (up.st == VQLIN_OK) up.st = cuda_status(cudaStreamSynchronize((cudaStream_t)stream), "create sync");
  if (up.st != VQLIN_OK) {
    vqlin_status s = up.st;
    vqlin_destroy(h);
    return s;
  }
  // ---- info
  vqlin_info& I = h->info;
  I.n_out = D->n_out; I.n_in = D->n_in; I.d = d; I.n_sub = n_sub; I.n_sub_o = n_sub_o; I.n_ocols = D->n_ocols;
  I.nnz = D->nnz;
  I.index_bytes = row_bytes * D->n_out + (D->n_ocols ? row_bytes_o * D->n_out : 0);
  I.codebook_bytes = 2ll * d * ((int64_t)G * (k1s + D->k2) + (D->n_ocols ? D->ko : 0));
  I.scale_bytes = (D->row_scale ? 2ll * D->n_out : 0) + (D->col_scale ? 2ll * D->n_in : 0);
  I.sparse_bytes = D->nnz ? D->nnz * 6 + 4ll * (D->n_out + 1) : 0;
  I.vsr_bytes = D->vsr_nblocks ? D->vsr_nblocks * (4 + 2ll * d) + 4ll * (D->n_out + 1) : 0;
  {
    // VPTQ "Compression ratio calculation": 16*M / (V*k*16 + M*ceil(log2 k)/V), with the main
    // codebooks counted as stored (n_groups of k1s entries)
    double M = (double)D->n_out * D->n_in;
    int lb = 0;
    while ((1ll << lb) < D->k1) ++lb;
    double ratio = 16.0 * M / ((double)d * G * k1s * 16.0 + M * lb / d);
    I.vptq_compression_ratio = ratio;
    I.vptq_bits_per_weight = 16.0 / ratio;
    double total_bits = 8.0 * (I.index_bytes + I.codebook_bytes + I.scale_bytes + I.sparse_bytes + I.vsr_bytes +
                               4ll * D->n_ocols);
    I.total_bits_per_weight = total_bits / M;
  }
  cudaSetDevice(prev_dev);
  *out = h;
  return VQLIN_OK;
}

vqlin_status vqlin_get_info(const vqlin_handle* h, vqlin_info* info) {
  if (!h || !info) { set_error("NULL argument"); return VQLIN_ERR_INVALID_ARG; }
  *info = h->info;
  return VQLIN_OK;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

vqlin_status vqlin_unpack_indices(const vqlin_handle* h, int32_t which, uint32_t* out, void* stream) {
  if (!h || !out || (which != 0 && which != 1)) { set_error("bad argument"); return VQLIN_ERR_INVALID_ARG; }
  if (which == 1 && h->L.n_ocols == 0) return VQLIN_OK;
  return cuda_status(launch_unpack(h->L, which, out, (cudaStream_t)stream), "unpack launch");
}

vqlin_status vqlin_dequant(const vqlin_handle* h, uint16_t* W, int64_t ldw, void* stream) {
  if (!h || !W || ldw < h->L.n_in) { set_error("bad argument (W NULL or ldw < n_in)"); return VQLIN_ERR_INVALID_ARG; }
  if (!aligned(W, 2)) { set_error("W must be 2-byte aligned"); return VQLIN_ERR_INVALID_ARG; }
  return cuda_status(launch_dequant(h->L, reinterpret_cast<__half*>(W), ldw, (cudaStream_t)stream), "dequant launch");
}

static bool dtype_ok(vqlin_dtype t) { return t == VQLIN_F32 || t == VQLIN_F16 || t == VQLIN_BF16; }

vqlin_status vqlin_gemv(const vqlin_handle* h, const void* x, vqlin_dtype xt, int32_t batch, void* y,
                        vqlin_dtype yt, void* stream) {
  if (!h || !x || !y) { set_error("NULL argument"); return VQLIN_ERR_INVALID_ARG; }
  if (!dtype_ok(xt) || !dtype_ok(yt)) { set_error("bad dtype"); return VQLIN_ERR_INVALID_ARG; }
  if (batch < 1 || batch > VQLIN_MAX_BATCH) { set_error("batch = %d: must be 1..16", batch); return VQLIN_ERR_UNSUPPORTED; }
  if (!aligned(x, 16) || !aligned(y, 16)) { set_error("x and y must be 16-byte aligned"); return VQLIN_ERR_INVALID_ARG; }
  return cuda_status(launch_gemv(h->L, x, xt, batch, y, yt, nullptr, 0, (cudaStream_t)stream), "gemv launch");
}

size_t vqlin_gemv_workspace_size(const vqlin_handle* h, int32_t batch) {
  if (!h || batch < 1 || batch > VQLIN_MAX_BATCH) return 0;
  return gemv_workspace_bytes(h->L, batch);
}

vqlin_status vqlin_gemv_ws(const vqlin_handle* h, const void* x, vqlin_dtype xt, int32_t batch, void* y,
                           vqlin_dtype yt, void* workspace, size_t ws_bytes, void* stream) {
  if (!h || !x || !y) { set_error("NULL argument"); return VQLIN_ERR_INVALID_ARG; }
  if (!dtype_ok(xt) || !dtype_ok(yt)) { set_error("bad dtype"); return VQLIN_ERR_INVALID_ARG; }
  if (batch < 1 || batch > VQLIN_MAX_BATCH) { set_error("batch = %d: must be 1..16", batch); return VQLIN_ERR_UNSUPPORTED; }
  if (!aligned(x, 16) || !aligned(y, 16)) { set_error("x and y must be 16-byte aligned"); return VQLIN_ERR_INVALID_ARG; }
  if (!workspace || ws_bytes < gemv_workspace_bytes(h->L, batch) || !aligned(workspace, 256)) {
    set_error("workspace must be >= %zu bytes and 256-byte aligned", gemv_workspace_bytes(h->L, batch));
    return VQLIN_ERR_WORKSPACE;
  }
  return cuda_status(launch_gemv(h->L, x, xt, batch, y, yt, workspace, ws_bytes, (cudaStream_t)stream),
                     "gemv launch");
}

static size_t ws_align(size_t b) { return (b + 255) & ~size_t(255); }

size_t vqlin_gemm_workspace_size(const vqlin_handle* h, int64_t M) {
  if (!h || M < 1) return 0;
  // the fused path needs room only for bf16 activations converted to fp16; the two-phase path
  // also holds the dequantised fp16 weight
  size_t w = gemm_fused_supported(h->L) ? 0 : ws_align((size_t)h->L.n_out * h->L.n_in * 2);
  size_t x = ws_align((size_t)M * h->L.n_in * 2);
  return w + x;
}

vqlin_status vqlin_gemm(const vqlin_handle* h, const void* X, vqlin_dtype xt, int64_t M, void* Y, vqlin_dtype yt,
                        void* workspace, size_t ws_bytes, void* stream) {
  if (!h || !X || !Y) { set_error("NULL argument"); return VQLIN_ERR_INVALID_ARG; }
  if (M < 1) { set_error("M must be >= 1"); return VQLIN_ERR_UNSUPPORTED; }
  if (xt != VQLIN_F16 && xt != VQLIN_BF16) { set_error("X must be F16 or BF16"); return VQLIN_ERR_UNSUPPORTED; }
  if (!dtype_ok(yt)) { set_error("bad Y dtype"); return VQLIN_ERR_INVALID_ARG; }
  if (h->L.n_in % 8 != 0) { set_error("gemm needs n_in %% 8 == 0"); return VQLIN_ERR_UNSUPPORTED; }
  if (!aligned(X, 16) || !aligned(Y, 16)) { set_error("X and Y must be 16-byte aligned"); return VQLIN_ERR_INVALID_ARG; }
  size_t need = vqlin_gemm_workspace_size(h, M);
  if (!workspace || ws_bytes < need || !aligned(workspace, 256)) {
    set_error("workspace must be >= %zu bytes and 256-byte aligned", need);
    return VQLIN_ERR_WORKSPACE;
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (gemm_fused_supported(h->L)) {
    // weight tiles dequantised in shared memory inside the GEMM; bf16 activations are first
    // converted to fp16 in the workspace (exact in the precondition's range)
    const __half* A = reinterpret_cast<const __half*>(X);
    if (xt == VQLIN_BF16) {
      __half* X16 = reinterpret_cast<__half*>(workspace);
      vqlin_status st = cuda_status(launch_convert_to_f16(X, xt, M * h->L.n_in, X16, s), "gemm convert launch");
      if (st) return st;
      A = X16;
    }
    return cuda_status(launch_gemm_vq(h->L, A, M, Y, yt, s), "gemm launch");
  }
  __half* W = reinterpret_cast<__half*>(workspace);
  __half* X16 = reinterpret_cast<__half*>(reinterpret_cast<char*>(workspace) + ws_align((size_t)h->L.n_out * h->L.n_in * 2));
  vqlin_status st = cuda_status(launch_dequant(h->L, W, h->L.n_in, s), "gemm dequant launch");
  if (st) return st;
  const __half* A = reinterpret_cast<const __half*>(X);
  if (xt == VQLIN_BF16) {
    st = cuda_status(launch_convert_to_f16(X, xt, M * h->L.n_in, X16, s), "gemm convert launch");
    if (st) return st;
    A = X16;
  }
  return cuda_status(launch_gemm_f16(A, W, M, h->L.n_out, h->L.n_in, Y, yt, s), "gemm launch");
}

}  // extern "C"
