// vqlin_gemv_noalloc: the decode GEMV for callers that cannot allocate device
// memory at call time.
//
// Some callers must not call cudaMalloc once they are running: a serving loop
// whose memory pool already owns every byte of the GPU (weights, KV cache,
// activations), a latency-critical path where cudaMalloc's implicit device
// synchronisation is not allowed, or a plug-in inside another framework that
// may only touch buffers it is handed.  vqlin_gemv_ws needs a caller-supplied
// scratch buffer; this entry point instead uses a fixed-size scratch array
// compiled into the library, so the caller passes only x and y.
//
// The scratch is a file-scope __device__ array of kScratchBytes (8 MiB).  Every
// GPU that loads the library holds it until the process exits.  It is sized so
// that the kernels vqlin_gemv_ws would pick also run here for the layers this
// library targets: the codebook-stationary decode of a 4096-row layer with a
// 65536-entry codebook keeps 74 fp32 partial-sum planes per batch row (4.6 MiB at
// batch 4), and the column-split decode keeps one fp32 accumulator of
// batch * n_out floats.  A layer whose plan needs more than the array holds
// falls back to the kernels that need no scratch, as vqlin_gemv does; a layer
// with batch * n_out above kScratchBytes / 4 is refused with UNSUPPORTED.
//
// Host code cannot use the array's name as a device address, so the first call
// on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it; make that first call outside any stream
// capture.  All calls share the one array: calls whose kernels overlap on the
// GPU (for example on two streams) race on it and must be serialised by the
// caller.  Whatever part must start at zero is cleared on the call's stream
// before every use, so what a previous call left there does not leak into the
// result.
#include <mutex>

#include "vqlin_internal.cuh"

namespace vqlin {

constexpr size_t kScratchBytes = 8u << 20;               // 8 MiB
constexpr size_t kScratchFloats = kScratchBytes / sizeof(float);
static __device__ __align__(256) float g_gemv_scratch[kScratchFloats];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};
}  // namespace

// Device address of the scratch array on the current device (looked up once per device).
static vqlin_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device ordinal %d is beyond the %d devices this library tracks", dev, kMaxDevices);
    return VQLIN_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gemv_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(scratch)");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return VQLIN_OK;
}

}  // namespace vqlin

using namespace vqlin;

extern "C" vqlin_status vqlin_gemv_noalloc(const vqlin_handle* h, const void* x, vqlin_dtype xt, int32_t batch,
                                           void* y, vqlin_dtype yt, void* stream) {
  if (!h || !x || !y) { set_error("NULL argument"); return VQLIN_ERR_INVALID_ARG; }
  if (!(xt == VQLIN_F32 || xt == VQLIN_F16 || xt == VQLIN_BF16) || !(yt == VQLIN_F32 || yt == VQLIN_F16 || yt == VQLIN_BF16)) {
    set_error("bad dtype");
    return VQLIN_ERR_INVALID_ARG;
  }
  if (batch < 1 || batch > VQLIN_MAX_BATCH) { set_error("batch = %d: must be 1..16", batch); return VQLIN_ERR_UNSUPPORTED; }
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15)) {
    set_error("x and y must be 16-byte aligned");
    return VQLIN_ERR_INVALID_ARG;
  }
  const size_t need = (size_t)batch * h->L.n_out;
  if (need > kScratchFloats) {
    set_error("batch * n_out = %zu exceeds the built-in scratch of %zu floats; use vqlin_gemv_ws", need,
              kScratchFloats);
    return VQLIN_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  vqlin_status st = scratch_address(&scratch);
  if (st) return st;
  return cuda_status(launch_gemv(h->L, x, xt, batch, y, yt, scratch, kScratchBytes, (cudaStream_t)stream),
                     "gemv (no-alloc) launch");
}
