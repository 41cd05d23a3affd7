// C ABI front end of libmoa: argument validation and dispatch to the kernels.
// Every check that can fail does so here, on the host, before anything is
// enqueued; the kernels assume validated arguments.
#include <algorithm>
#include <mutex>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "internal.h"

namespace moa {

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned long long* done) {
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
  std::lock_guard<std::mutex> lock(mu);
  if (bit != 0 && (*done & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) *done |= bit;
  return e;
}

moa_status cuda_fail(cudaError_t e, const char* where) {
  static const bool verbose = std::getenv("MOA_VERBOSE") != nullptr;
  if (verbose) std::fprintf(stderr, "libmoa: %s: %s\n", where, cudaGetErrorString(e));
  // Clear the runtime's record of a non-sticky error here, so that a later
  // launch check does not report it against an unrelated kernel.
  (void)cudaGetLastError();
  return MOA_ERR_CUDA;
}

}  // namespace moa

using namespace moa;

static bool valid_d(int32_t d) { return d == 64 || d == 128; }
static bool valid_dtype(moa_dtype t) { return t == MOA_F32 || t == MOA_BF16; }

extern "C" const char* moa_status_string(moa_status s) {
  switch (s) {
    case MOA_OK: return "MOA_OK";
    case MOA_ERR_INVALID_ARG: return "MOA_ERR_INVALID_ARG";
    case MOA_ERR_CAPACITY: return "MOA_ERR_CAPACITY";
    case MOA_ERR_WORKSPACE: return "MOA_ERR_WORKSPACE";
    case MOA_ERR_UNSUPPORTED: return "MOA_ERR_UNSUPPORTED";
    case MOA_ERR_CUDA: return "MOA_ERR_CUDA";
    case MOA_ERR_TIMEOUT: return "MOA_ERR_TIMEOUT";
    case MOA_ERR_HOST: return "MOA_ERR_HOST";
  }
  return "MOA_ERR_UNKNOWN";
}

extern "C" moa_status moa_kv_header_bytes(int32_t B, size_t* bytes_out) {
  if (B < 1 || !bytes_out) return MOA_ERR_INVALID_ARG;
  *bytes_out = header_bytes(B);
  return MOA_OK;
}

extern "C" moa_status moa_kv_bytes_sink(int32_t B, int32_t Hkv, int32_t d, moa_dtype dtype,
                                        const int32_t* capacity, const int32_t* sink_capacity,
                                        size_t* bytes_out) {
  if (B < 1 || Hkv < 1 || Hkv > MOA_MAX_HEADS || !valid_d(d) || !valid_dtype(dtype) ||
      !capacity || !bytes_out)
    return MOA_ERR_INVALID_ARG;
  int64_t sum = 0, sum_sink = 0;
  for (int32_t g = 0; g < Hkv; ++g) {
    if (capacity[g] < 1) return MOA_ERR_INVALID_ARG;
    sum += capacity[g];
    if (sink_capacity) {
      if (sink_capacity[g] < 0) return MOA_ERR_INVALID_ARG;
      sum_sink += sink_capacity[g];
    }
  }
  if (sum_sink > INT32_MAX) return MOA_ERR_INVALID_ARG;
  *bytes_out = header_bytes(B) + (size_t)B * (size_t)(sum + sum_sink) * 2 * (size_t)d * elem_bytes(dtype);
  return MOA_OK;
}

extern "C" moa_status moa_kv_bytes(int32_t B, int32_t Hkv, int32_t d, moa_dtype dtype,
                                   const int32_t* capacity, size_t* bytes_out) {
  return moa_kv_bytes_sink(B, Hkv, d, dtype, capacity, nullptr, bytes_out);
}

extern "C" moa_status moa_kv_alloc(void* dev_buf, size_t bytes, int32_t B, int32_t Hkv, int32_t d,
                                   moa_dtype dtype, const int32_t* capacity, void* stream,
                                   moa_kv_cache** out) {
  return moa_kv_alloc_sink(dev_buf, bytes, B, Hkv, d, dtype, capacity, nullptr, stream, out);
}

extern "C" moa_status moa_kv_alloc_sink(void* dev_buf, size_t bytes, int32_t B, int32_t Hkv, int32_t d,
                                        moa_dtype dtype, const int32_t* capacity,
                                        const int32_t* sink_capacity, void* stream, moa_kv_cache** out) {
  if (!out) return MOA_ERR_INVALID_ARG;
  *out = nullptr;
  size_t need = 0;
  moa_status st = moa_kv_bytes_sink(B, Hkv, d, dtype, capacity, sink_capacity, &need);
  if (st != MOA_OK) return st;
  if (!dev_buf || ((uintptr_t)dev_buf & 255u) != 0) return MOA_ERR_INVALID_ARG;
  if (bytes < need) return MOA_ERR_CAPACITY;
  moa_kv_cache* c = new (std::nothrow) moa_kv_cache();
  if (!c) return MOA_ERR_INVALID_ARG;
  c->buf = (char*)dev_buf;
  c->bytes = need;
  c->B = B;
  c->Hkv = Hkv;
  c->d = d;
  c->dtype = dtype;
  c->header = header_bytes(B);
  c->cap.assign(capacity, capacity + Hkv);
  c->goff.assign(Hkv + 1, 0);
  for (int32_t g = 0; g < Hkv; ++g) c->goff[g + 1] = c->goff[g] + capacity[g];
  c->scap.assign(Hkv, 0);
  if (sink_capacity) c->scap.assign(sink_capacity, sink_capacity + Hkv);
  c->soff.assign(Hkv + 1, 0);
  for (int32_t g = 0; g < Hkv; ++g) c->soff[g + 1] = c->soff[g] + c->scap[g];
  c->sink_off = (size_t)B * (size_t)c->goff[Hkv] * 2 * (size_t)d * elem_bytes(dtype);
  if (cudaMemsetAsync(dev_buf, 0, need, (cudaStream_t)stream) != cudaSuccess) {
    delete c;
    return MOA_ERR_CUDA;
  }
  *out = c;
  return MOA_OK;
}

extern "C" moa_status moa_kv_free(moa_kv_cache* cache) {
  delete cache;
  return MOA_OK;
}

extern "C" moa_status moa_kv_layout(const moa_kv_cache* c, void** data_out, int64_t* goff) {
  if (!c || !data_out) return MOA_ERR_INVALID_ARG;
  *data_out = c->buf + c->header;
  if (goff)
    for (int32_t g = 0; g <= c->Hkv; ++g) goff[g] = c->goff[g];
  return MOA_OK;
}

extern "C" moa_status moa_kv_append(moa_kv_cache* c, const void* k, const void* v, int32_t n_tok,
                                    void* stream) {
  if (!c || !k || !v || n_tok < 1) return MOA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return MOA_ERR_INVALID_ARG;
  return launch_append(c, k, v, n_tok, (cudaStream_t)stream);
}

extern "C" moa_status moa_kv_positions(const moa_kv_cache* c, int64_t* t_host, void* stream) {
  if (!c || !t_host) return MOA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t err = 0;
  if (cudaMemcpyAsync(&err, c->buf + kHdrErr, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOA_ERR_CUDA;
  if (cudaMemcpyAsync(t_host, c->buf + kHdrT, 8 * (size_t)c->B, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return MOA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOA_ERR_CUDA;
  if (err & kErrTimeout) return MOA_ERR_TIMEOUT;
  return err ? MOA_ERR_INVALID_ARG : MOA_OK;
}

extern "C" moa_status moa_kv_set_positions(moa_kv_cache* c, const int64_t* t_host, void* stream) {
  if (!c || !t_host) return MOA_ERR_INVALID_ARG;
  for (int32_t b = 0; b < c->B; ++b)
    if (t_host[b] < 0) return MOA_ERR_INVALID_ARG;
  // Pageable source: the runtime stages it before returning, so t_host may be
  // reused as soon as this call returns.
  if (cudaMemcpyAsync(c->buf + kHdrT, t_host, 8 * (size_t)c->B, cudaMemcpyHostToDevice,
                      (cudaStream_t)stream) != cudaSuccess)
    return MOA_ERR_CUDA;
  return MOA_OK;
}

extern "C" moa_status moa_workspace_bytes(moa_op op, int32_t B, int32_t Hq, int64_t N, int32_t d,
                                          const int32_t* spans, size_t* bytes_out) {
  if (!bytes_out || B < 1 || Hq < 1 || Hq > MOA_MAX_HEADS || !valid_d(d)) return MOA_ERR_INVALID_ARG;
  if (op == MOA_OP_PREFILL) {
    if (N < 1 || N > INT32_MAX) return MOA_ERR_INVALID_ARG;
    *bytes_out = prefill_workspace_bytes(B, Hq, N);
    return MOA_OK;
  }
  if (op == MOA_OP_DECODE) {
    if (!spans) return MOA_ERR_INVALID_ARG;
    for (int32_t h = 0; h < Hq; ++h)
      if (spans[h] < 1) return MOA_ERR_INVALID_ARG;
    *bytes_out = decode_workspace_bytes(B, Hq, d, spans);
    return MOA_OK;
  }
  return MOA_ERR_INVALID_ARG;
}

extern "C" moa_status moa_workspace_bytes_sink(moa_op op, int32_t B, int32_t Hq, int64_t N, int32_t d,
                                               const int32_t* spans, const int32_t* sinks, size_t* bytes_out) {
  if (!sinks) return MOA_ERR_INVALID_ARG;
  if (Hq >= 1 && Hq <= MOA_MAX_HEADS)
    for (int32_t h = 0; h < Hq; ++h)
      if (sinks[h] < 0) return MOA_ERR_INVALID_ARG;
  const moa_status st = moa_workspace_bytes(op, B, Hq, N, d, spans, bytes_out);
  if (st != MOA_OK || op != MOA_OP_DECODE) return st;
  *bytes_out = decode_workspace_bytes(B, Hq, d, spans, sinks);
  return MOA_OK;
}

extern "C" moa_status moa_workspace_init(void* ws, size_t bytes, void* stream) {
  if (!ws || bytes == 0) return MOA_ERR_INVALID_ARG;
  return cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream) == cudaSuccess ? MOA_OK : MOA_ERR_CUDA;
}

extern "C" moa_status moa_workspace_check(const void* ws, void* stream) {
  if (!ws) return MOA_ERR_INVALID_ARG;
  uint32_t err = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&err, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOA_ERR_CUDA;
  return err ? MOA_ERR_TIMEOUT : MOA_OK;
}

extern "C" moa_status moa_stream_read(const void* buf, size_t bytes, void* out, void* stream) {
  if (!buf || !out || bytes % 16 != 0 || reinterpret_cast<uintptr_t>(buf) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(out) % 8 != 0)
    return MOA_ERR_INVALID_ARG;
  return launch_stream_read(buf, bytes, out, (cudaStream_t)stream);
}

extern "C" moa_status moa_prefill_stall_test(const void* q, const void* k, const void* v, void* o, void* ws,
                                             size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !o) return MOA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return MOA_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws & 255u) != 0 || ws_bytes < prefill_workspace_bytes(1, 1, 128)) return MOA_ERR_WORKSPACE;
  return guarded([&] { return launch_prefill_stall_test(q, k, v, o, ws, ws_bytes, (cudaStream_t)stream); });
}

extern "C" moa_status moa_prefill_schedule(int32_t B, int32_t Hq, int64_t N, const int32_t* spans,
                                           int32_t n_ctas, int32_t* rows_out, int64_t cap,
                                           int64_t* n_rows_out) {
  if (B < 1 || Hq < 1 || Hq > MOA_MAX_HEADS || N < 1 || N > INT32_MAX || !spans || !n_rows_out ||
      n_ctas < 1 || n_ctas > kPrefillMaxCtas || cap < 0 || (cap > 0 && !rows_out))
    return MOA_ERR_INVALID_ARG;
  for (int32_t h = 0; h < Hq; ++h)
    if (spans[h] < 1) return MOA_ERR_INVALID_ARG;
  return guarded([&] {
    const std::vector<int32_t> rows = prefill_schedule_rows(B, Hq, (int32_t)N, spans, n_ctas);
    const int64_t n = (int64_t)rows.size() / 7;
    std::copy(rows.begin(), rows.begin() + 7 * std::min(n, cap), rows_out);
    *n_rows_out = n;
    return MOA_OK;
  });
}

static moa_status prefill_common(const void* q, const void* k, const void* v, void* o, int32_t B,
                                 int32_t Hq, int32_t Hkv, int64_t N, int32_t d, moa_dtype dtype,
                                 const int32_t* spans, const int32_t* sinks, float scale, void* ws,
                                 size_t ws_bytes, moa_kv_cache* fill, void* stream);

extern "C" moa_status moa_prefill(const void* q, const void* k, const void* v, void* o, int32_t B,
                                  int32_t Hq, int32_t Hkv, int64_t N, int32_t d, moa_dtype dtype,
                                  const int32_t* spans, float scale, void* ws, size_t ws_bytes,
                                  moa_kv_cache* fill, void* stream) {
  return guarded([&] {
    return prefill_common(q, k, v, o, B, Hq, Hkv, N, d, dtype, spans, nullptr, scale, ws, ws_bytes, fill, stream);
  });
}

extern "C" moa_status moa_prefill_sink(const void* q, const void* k, const void* v, void* o, int32_t B,
                                       int32_t Hq, int32_t Hkv, int64_t N, int32_t d, moa_dtype dtype,
                                       const int32_t* spans, const int32_t* sinks, float scale, void* ws,
                                       size_t ws_bytes, moa_kv_cache* fill, void* stream) {
  if (!sinks) return MOA_ERR_INVALID_ARG;
  return guarded([&] {
    return prefill_common(q, k, v, o, B, Hq, Hkv, N, d, dtype, spans, sinks, scale, ws, ws_bytes, fill, stream);
  });
}

static moa_status prefill_common(const void* q, const void* k, const void* v, void* o, int32_t B,
                                 int32_t Hq, int32_t Hkv, int64_t N, int32_t d, moa_dtype dtype,
                                 const int32_t* spans, const int32_t* sinks, float scale, void* ws,
                                 size_t ws_bytes, moa_kv_cache* fill, void* stream) {
  if (!q || !k || !v || !o || !spans) return MOA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return MOA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq > MOA_MAX_HEADS || Hkv > MOA_MAX_HEADS || Hq % Hkv != 0)
    return MOA_ERR_INVALID_ARG;
  if (N < 1 || N > INT32_MAX || !valid_d(d) || !valid_dtype(dtype)) return MOA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale <= 0.f || scale > 1e30f) return MOA_ERR_INVALID_ARG;
  for (int32_t h = 0; h < Hq; ++h) {
    if (spans[h] < 1) return MOA_ERR_INVALID_ARG;
    if (sinks && sinks[h] < 0) return MOA_ERR_INVALID_ARG;
  }
  const int32_t G = Hq / Hkv;
  if (fill) {
    if (fill->B != B || fill->Hkv != Hkv || fill->d != d || fill->dtype != dtype)
      return MOA_ERR_INVALID_ARG;
    for (int32_t h = 0; h < Hq; ++h) {
      if (spans[h] > fill->cap[h / G]) return MOA_ERR_CAPACITY;
      if (sinks && sinks[h] > fill->scap[h / G]) return MOA_ERR_CAPACITY;
    }
  }
  // global-token counts above N behave as N (and keep the kernels' arithmetic in range)
  int32_t sk[MOA_MAX_HEADS];
  bool any_sink = false;
  if (sinks)
    for (int32_t h = 0; h < Hq; ++h) {
      sk[h] = (int32_t)std::min<int64_t>(sinks[h], N);
      any_sink = any_sink || sk[h] > 0;
    }
  const int32_t* sinks_or_null = any_sink ? sk : nullptr;
  cudaStream_t s = (cudaStream_t)stream;
  moa_status st;
  if (dtype == MOA_F32) {
    st = launch_prefill_f32((const float*)q, (const float*)k, (const float*)v, (float*)o, B, Hq, Hkv,
                            (int32_t)N, d, spans, scale, s, sinks_or_null);
  } else {
    if (d != 128) return MOA_ERR_UNSUPPORTED;
    if (!ws || ((uintptr_t)ws & 255u) != 0) return MOA_ERR_WORKSPACE;
    if (ws_bytes < prefill_workspace_bytes(B, Hq, N)) return MOA_ERR_WORKSPACE;
    // the kernel writes the cache itself
    return launch_prefill_bf16(q, k, v, o, B, Hq, Hkv, (int32_t)N, spans, scale, ws, ws_bytes, s, fill,
                               sinks_or_null);
  }
  if (st != MOA_OK || !fill) return st;
  return launch_append(fill, k, v, (int32_t)N, s);
}

// Shared checks of the chunk entry points; MOA_OK when the call is well formed.
static moa_status chunk_args(const moa_kv_cache* c, int32_t Hq, int32_t n, const int32_t* spans) {
  if (!c || !spans) return MOA_ERR_INVALID_ARG;
  if (Hq < 1 || Hq > MOA_MAX_HEADS || Hq % c->Hkv != 0 || n < 1) return MOA_ERR_INVALID_ARG;
  const int32_t G = Hq / c->Hkv;
  int32_t max_s = 1;
  for (int32_t h = 0; h < Hq; ++h) {
    if (spans[h] < 1) return MOA_ERR_INVALID_ARG;
    if (spans[h] > c->cap[h / G]) return MOA_ERR_CAPACITY;
    max_s = std::max(max_s, spans[h]);
  }
  if ((int64_t)n + max_s + 128 > INT32_MAX) return MOA_ERR_INVALID_ARG;
  if (c->dtype != MOA_BF16 || c->d != 128) return MOA_ERR_UNSUPPORTED;
  return MOA_OK;
}

extern "C" moa_status moa_chunk_workspace_bytes(const moa_kv_cache* c, int32_t Hq, int32_t n,
                                                const int32_t* spans, size_t* bytes_out) {
  if (!bytes_out) return MOA_ERR_INVALID_ARG;
  const moa_status st = chunk_args(c, Hq, n, spans);
  if (st != MOA_OK) return st;
  *bytes_out = prefill_chunk_workspace_bytes(c->B, Hq, c->Hkv, n, spans);
  return MOA_OK;
}

extern "C" moa_status moa_prefill_chunk(moa_kv_cache* c, const void* q, const void* k, const void* v,
                                        void* o, int32_t Hq, int32_t n, const int32_t* spans, float scale,
                                        void* ws, size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !o) return MOA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return MOA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale <= 0.f || scale > 1e30f) return MOA_ERR_INVALID_ARG;
  const moa_status st = chunk_args(c, Hq, n, spans);
  if (st != MOA_OK) return st;
  if (!ws || ((uintptr_t)ws & 255u) != 0) return MOA_ERR_WORKSPACE;
  if (ws_bytes < prefill_chunk_workspace_bytes(c->B, Hq, c->Hkv, n, spans)) return MOA_ERR_WORKSPACE;
  return guarded([&] {
    return launch_prefill_chunk(c, q, k, v, o, Hq, n, spans, scale, ws, ws_bytes, (cudaStream_t)stream);
  });
}

// Shared checks and dispatch of the decode entry points (k, v: the fused
// append's new token, or both null; sinks: global tokens per query head, or
// null).
static moa_status decode_common(moa_kv_cache* c, const void* q, const void* k, const void* v, void* o,
                                int32_t Hq, const int32_t* spans, const int32_t* sinks, float scale,
                                void* ws, size_t ws_bytes, void* stream) {
  if (!c || !q || !o || !spans) return MOA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o)) return MOA_ERR_INVALID_ARG;
  if ((k == nullptr) != (v == nullptr)) return MOA_ERR_INVALID_ARG;
  if (k && (!aligned16(k) || !aligned16(v))) return MOA_ERR_INVALID_ARG;
  if (Hq < 1 || Hq > MOA_MAX_HEADS || Hq % c->Hkv != 0) return MOA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale <= 0.f || scale > 1e30f) return MOA_ERR_INVALID_ARG;
  const int32_t G = Hq / c->Hkv;
  bool any_sink = false;
  for (int32_t h = 0; h < Hq; ++h) {
    if (spans[h] < 1) return MOA_ERR_INVALID_ARG;
    if (spans[h] > c->cap[h / G]) return MOA_ERR_CAPACITY;
    if (sinks) {
      if (sinks[h] < 0) return MOA_ERR_INVALID_ARG;
      if (sinks[h] > c->scap[h / G]) return MOA_ERR_CAPACITY;
      any_sink = any_sink || sinks[h] > 0;
    }
  }
  const int32_t* sk = any_sink ? sinks : nullptr;
  if (!ws || ((uintptr_t)ws & 255u) != 0) return MOA_ERR_WORKSPACE;
  if (ws_bytes < decode_workspace_bytes(c->B, Hq, c->d, spans, sk)) return MOA_ERR_WORKSPACE;
  return launch_decode(c, q, o, Hq, spans, scale, ws, ws_bytes, (cudaStream_t)stream, k, v, sk);
}

extern "C" moa_status moa_decode_append(moa_kv_cache* c, const void* q, const void* k, const void* v,
                                        void* o, int32_t Hq, const int32_t* spans, float scale, void* ws,
                                        size_t ws_bytes, void* stream) {
  if (!k || !v) return MOA_ERR_INVALID_ARG;
  return guarded([&] { return decode_common(c, q, k, v, o, Hq, spans, nullptr, scale, ws, ws_bytes, stream); });
}

extern "C" moa_status moa_decode_append_sink(moa_kv_cache* c, const void* q, const void* k, const void* v,
                                             void* o, int32_t Hq, const int32_t* spans, const int32_t* sinks,
                                             float scale, void* ws, size_t ws_bytes, void* stream) {
  if (!k || !v || !sinks) return MOA_ERR_INVALID_ARG;
  return guarded([&] { return decode_common(c, q, k, v, o, Hq, spans, sinks, scale, ws, ws_bytes, stream); });
}

extern "C" moa_status moa_decode_sink(moa_kv_cache* c, const void* q, void* o, int32_t Hq,
                                      const int32_t* spans, const int32_t* sinks, float scale, void* ws,
                                      size_t ws_bytes, void* stream) {
  if (!sinks) return MOA_ERR_INVALID_ARG;
  return guarded([&] { return decode_common(c, q, nullptr, nullptr, o, Hq, spans, sinks, scale, ws, ws_bytes, stream); });
}

extern "C" moa_status moa_decode(moa_kv_cache* c, const void* q, void* o, int32_t Hq,
                                 const int32_t* spans, float scale, void* ws, size_t ws_bytes,
                                 void* stream) {
  return guarded([&] { return decode_common(c, q, nullptr, nullptr, o, Hq, spans, nullptr, scale, ws, ws_bytes, stream); });
}
