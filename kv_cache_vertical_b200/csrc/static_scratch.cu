// static_scratch.cu -- hq_decode_attn_static: decode attention whose scratch is
// a fixed, file-scope device array instead of a caller-allocated workspace.
//
// For callers that cannot allocate device memory when they call: code that
// runs while someone else is capturing the stream into a CUDA graph (a
// cudaMalloc there would break the capture), serving runtimes that fix their
// device memory at start-up, and hosts that forbid allocation after
// initialization.  The kernels and results are those of hq_decode_attn.
//
// The array lives in every GPU that loads the library, until the process
// exits.  In host code its name only stands for it (a host-side shadow): the
// device address is looked up with cudaGetSymbolAddress, with the device
// current, on the first call made in a CUDA context, and cached for that
// context.  Every call shares the array: it first clears the part that must
// start at zero (status word and the split counters); calls that overlap on the
// GPU race on it.  The first 4 bytes are the device status word of the last
// call (hq_read_static_status).
#include <cuda.h>

#include <mutex>

#include "hq_internal.cuh"

namespace {

__device__ __align__(256) uint8_t g_static_scratch[HQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
  CUcontext ctx;   // the context the address belongs to
  void *addr;
};
ScratchAddr g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// The current CUDA context (driver entry point, looked up once), or nullptr.
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext *);
  static Fn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (Fn) nullptr;
    return reinterpret_cast<Fn>(p);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_static_scratch in the current device's context
// (nullptr on error).  Looked up again whenever the context differs from the
// one the cached address came from (a reset device gets a new context, and
// the module, with the array, is loaded again at a possibly new address).
void *scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr &e = g_scratch[dev];
  if (ctx && e.addr && e.ctx == ctx) return e.addr;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return nullptr;
  ctx = current_context();             // the lookup makes the device's context current if none was
  if (!ctx) return nullptr;
  e.ctx = ctx;
  e.addr = p;
  return p;
}

}  // namespace

extern "C" hq_status hq_decode_attn_static(const void *q, const hq_kv_cache *cache, int B,
                                           int Hq, int Hkv, int D, float softmax_scale,
                                           float *out, float *lse_out, void *stream) {
  const hq_status st = hq::check_decode_args(q, cache, B, Hq, Hkv, D, out);
  if (st != HQ_OK) return st;
  const size_t need = hq::decode_ws_bytes(B, Hq, Hkv, D, cache->n_lo, cache->n_hi, cache->bits);
  if (need > HQ_STATIC_SCRATCH_BYTES) return HQ_ERR_SCRATCH_LIMIT;
  uint8_t *ws = static_cast<uint8_t *>(scratch_address());
  if (!ws) return HQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t zero = hq::decode_ws_zero_bytes(B, Hq, Hkv, D, cache->n_lo, cache->n_hi, cache->bits);
  if (cudaMemsetAsync(ws, 0, zero, s) != cudaSuccess) return HQ_ERR_CUDA;
  const cudaError_t e =
      hq::launch_decode(static_cast<const __nv_bfloat16 *>(q), *cache, B, Hq, Hkv, D,
                        hq::resolve_softmax_scale(softmax_scale, D), out, lse_out, ws,
                        reinterpret_cast<uint32_t *>(ws), s);
  return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

extern "C" hq_status hq_read_static_status(int clear, uint32_t *status_out, void *stream) {
  if (!status_out) return HQ_ERR_INVALID_ARG;
  uint8_t *ws = static_cast<uint8_t *>(scratch_address());
  if (!ws) return HQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess) return HQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HQ_ERR_CUDA;
  if (clear && cudaMemsetAsync(ws, 0, sizeof v, s) != cudaSuccess) return HQ_ERR_CUDA;
  *status_out = v;
  return HQ_OK;
}
