// Internal declarations shared by the translation units of libmoa.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include <vector>

#include "moa.h"

#define MOA_MAX_HEADS 128

struct moa_kv_cache {
  char* buf = nullptr;           // caller-owned device buffer
  size_t bytes = 0;
  int32_t B = 0, Hkv = 0, d = 0;
  moa_dtype dtype = MOA_BF16;
  size_t header = 0;             // bytes before the data region
  std::vector<int32_t> cap;      // C_g
  std::vector<int64_t> goff;     // prefix sums of C_g, size Hkv + 1
  // global-token rows: K_g per key/value head (all 0: none), their prefix
  // sums, and the region's byte offset from the start of the data region
  std::vector<int32_t> scap;
  std::vector<int64_t> soff;
  size_t sink_off = 0;
  bool has_sinks() const { return soff.empty() ? false : soff.back() > 0; }
};

namespace moa {

inline size_t elem_bytes(moa_dtype t) { return t == MOA_F32 ? 4 : 2; }
inline size_t header_bytes(int64_t B) { return (size_t)(((16 + 8 * B) + 255) / 256 * 256); }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Header field offsets (bytes) inside a cache buffer.
constexpr size_t kHdrErr = 0;
constexpr size_t kHdrAppendCtr = 4;
constexpr size_t kHdrT = 16;

// Device error bits (cache and workspace error words).
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrEmpty = 2u;

int sm_count();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per device (the attribute does not carry over between
// devices); `done` is the caller's per-kernel record of devices already set.
cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned long long* done);

// MOA_ERR_CUDA with the CUDA error reported on stderr when the environment
// variable MOA_VERBOSE is set (the status alone cannot carry the reason);
// clears the runtime's pending error.
moa_status cuda_fail(cudaError_t e, const char* where);
// Runs an entry point's host-side work.  A C++ exception (a schedule's
// vectors that cannot be allocated, a lock that cannot be taken) becomes
// MOA_ERR_HOST instead of crossing the C boundary; the throwing paths run
// before any launch.
template <class F>
moa_status guarded(F&& f) noexcept {
  try {
    return f();
  } catch (...) {
    return MOA_ERR_HOST;
  }
}
inline moa_status check_launch(const char* where) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOA_OK : cuda_fail(e, where);
}

// Global-token region of a cache (nullptr when it keeps none) and, per key/value
// head, its row count and row offset as the kernels take them.
inline char* sink_region(const moa_kv_cache* c) {
  return c->has_sinks() ? c->buf + c->header + c->sink_off : nullptr;
}

// kv.cu
// Reads `bytes` (a multiple of 16) at 16-byte-aligned `buf` into a checksum
// at `out` (one uint64 on the device).
moa_status launch_stream_read(const void* buf, size_t bytes, void* out, cudaStream_t stream);
moa_status launch_append(moa_kv_cache* c, const void* k, const void* v, int32_t n_tok,
                         cudaStream_t s);

// decode.cu.  sinks: global tokens per query head, or nullptr for none.
size_t decode_workspace_bytes(int32_t B, int32_t Hq, int32_t d, const int32_t* spans,
                              const int32_t* sinks = nullptr);
moa_status launch_decode(moa_kv_cache* c, const void* q, void* o, int32_t Hq,
                         const int32_t* spans, float scale, void* ws, size_t ws_bytes,
                         cudaStream_t s, const void* k_new = nullptr, const void* v_new = nullptr,
                         const int32_t* sinks = nullptr);

// prefill_simt.cu (fp32)
moa_status launch_prefill_f32(const float* q, const float* k, const float* v, float* o,
                              int32_t B, int32_t Hq, int32_t Hkv, int32_t N, int32_t d,
                              const int32_t* spans, float scale, cudaStream_t s,
                              const int32_t* sinks = nullptr);

// prefill_sm100.cu (bf16, tcgen05)
constexpr int kTileM = 128;   // query rows per query tile (a work unit holds two)
constexpr int kTileN = 128;   // keys per key/value tile
constexpr int kPrefillMaxCtas = 1024;   // persistent grid bound (one CTA per SM)
// Work units (b, h, first query tile m, first key tile of m), dealt to n_ctas
// per-CTA lists: CTA c runs units[off[c] .. off[c+1]) in order.
struct PrefillSchedule {
  int32_t n_ctas;
  std::vector<int32_t> off;     // n_ctas + 1
  std::vector<int32_t> units;   // 4 int32 per unit
};
// sinks (nullable): global tokens per head; a query tile also visits the key
// tiles below its band that hold them.
PrefillSchedule prefill_schedule(int32_t B, int32_t Hq, int32_t N, const int32_t* spans, int32_t n_ctas,
                                 int32_t m0 = 0, const int32_t* sinks = nullptr);
// Rows (CTA, unit, b, h, query tile, first key tile, last key tile), one per query tile.
std::vector<int32_t> prefill_schedule_rows(int32_t B, int32_t Hq, int32_t N, const int32_t* spans,
                                           int32_t n_ctas);

size_t prefill_workspace_bytes(int32_t B, int32_t Hq, int64_t N);
// fill != nullptr: the kernel also appends the N key/value rows to that cache
// (the bytes and positions of launch_append(fill, k, v, N)).
moa_status launch_prefill_bf16(const void* q, const void* k, const void* v, void* o,
                               int32_t B, int32_t Hq, int32_t Hkv, int32_t N,
                               const int32_t* spans, float scale, void* ws, size_t ws_bytes,
                               cudaStream_t s, moa_kv_cache* fill = nullptr,
                               const int32_t* sinks = nullptr);

// Self-test of the prefill kernel's bounded waits (prefill_sm100.cu): one CTA
// on a 1 x 1 x 128 x 128 problem whose unit records are never published.
moa_status launch_prefill_stall_test(const void* q, const void* k, const void* v, void* o, void* ws,
                                     size_t ws_bytes, cudaStream_t s);

// Chunked prefill (prefill_sm100.cu): the n new tokens of every sequence
// attend to the cache's window plus themselves, then are appended.
size_t prefill_chunk_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t n, const int32_t* spans);
moa_status launch_prefill_chunk(moa_kv_cache* c, const void* q, const void* k, const void* v, void* o,
                                int32_t Hq, int32_t n, const int32_t* spans, float scale, void* ws,
                                size_t ws_bytes, cudaStream_t s);
// kv.cu: key/value rows of positions t_b - W .. t_b - 1 of every (b, g) into
// sk, sv [B, Hkv, W, d], read through the ring (zeros where the position is
// negative or no longer held).  Only rows W - C_g + 1 - 127 and up, rounded
// down to a tile, are written: no query of the group's heads reaches below.
moa_status launch_gather_window(const moa_kv_cache* c, int32_t W, void* sk, void* sv, cudaStream_t s);

}  // namespace moa
