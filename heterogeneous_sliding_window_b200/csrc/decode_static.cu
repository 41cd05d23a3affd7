// moa_decode_static_ws: decode attention for callers that cannot allocate
// device memory.
//
// moa_decode needs a caller-provided workspace for its split partials and
// per-(sequence, head) tickets.  Some callers have no way to provide one: a
// plugin or operator that the host framework hands only its input and output
// pointers, a runtime whose device memory is fully reserved up front by
// another allocator, or code that must not call cudaMalloc because that call
// synchronises the device.  This entry point serves them from a fixed-size
// scratch array that lives in the library's own device image instead.
//
// Cost of that convenience:
//  * every GPU that loads libmoa holds kStaticScratchBytes of device memory
//    for this array until the process exits;
//  * all calls on a device share the one array, which keeps the contents of
//    the last call; two calls whose kernels overlap on the GPU (different
//    streams, or different threads without ordering) race on it and may
//    produce wrong outputs;
//  * requests whose workspace would exceed the array are rejected with
//    MOA_ERR_WORKSPACE before anything is launched.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // 8 MiB per GPU

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch, looked up once per device.  In host
// code the name g_decode_scratch is only a host-side stand-in for the symbol;
// handing it to a kernel would read the wrong memory.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

moa_status scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return moa::cuda_fail(e, "static scratch: current device");
  if (dev < 0 || dev >= kMaxDevices) return MOA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return moa::cuda_fail(e, "static scratch symbol");
    if (p == nullptr) return moa::cuda_fail(cudaErrorInvalidSymbol, "static scratch symbol");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOA_OK;
}

}  // namespace

extern "C" moa_status moa_decode_static_ws(moa_kv_cache* c, const void* q, void* o, int32_t Hq,
                                           const int32_t* spans, float scale, void* stream) {
  if (!c || !q || !o || !spans) return MOA_ERR_INVALID_ARG;
  if (!moa::aligned16(q) || !moa::aligned16(o)) return MOA_ERR_INVALID_ARG;
  if (Hq < 1 || Hq > MOA_MAX_HEADS || Hq % c->Hkv != 0) return MOA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale <= 0.f || scale > 1e30f) return MOA_ERR_INVALID_ARG;
  const int32_t G = Hq / c->Hkv;
  for (int32_t h = 0; h < Hq; ++h) {
    if (spans[h] < 1) return MOA_ERR_INVALID_ARG;
    if (spans[h] > c->cap[h / G]) return MOA_ERR_CAPACITY;
  }
  const size_t need = moa::decode_workspace_bytes(c->B, Hq, c->d, spans);
  if (need > kStaticScratchBytes) return MOA_ERR_WORKSPACE;
  void* scratch = nullptr;
  moa_status st = moa::guarded([&] { return scratch_for_current_device(&scratch); });
  if (st != MOA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // The header and the per-(b, h) tickets must start at zero; the partials
  // are fully rewritten by every call.
  const size_t zero_bytes = 256 + (size_t)c->B * Hq * sizeof(uint32_t);
  const cudaError_t e = cudaMemsetAsync(scratch, 0, zero_bytes, s);
  if (e != cudaSuccess) return moa::cuda_fail(e, "static scratch memset");
  return moa::guarded([&] { return moa::launch_decode(c, q, o, Hq, spans, scale, scratch, kStaticScratchBytes, s); });
}
