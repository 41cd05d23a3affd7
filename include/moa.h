/*
 * moa.h -- C ABI of libmoa: heterogeneous sliding-window attention (MoA) on B200.
 *
 * The method ("Mixture of Attention" project page, section "Key findings /
 * Finding two: windows change with input length") gives every attention head
 * h its own causal sliding window whose length follows a linear rule in the
 * input length N, S_h = alpha_h + beta_h * N.  Query row i of head h attends
 * only to keys j with i - S_h < j <= i.  Deployment ("Demo", step 03, same
 * page) serves decoding from a fixed-size KV cache whose size differs per
 * head; the blog walkthrough "MoA: Mixture of Sparse Attention for Automatic
 * Large Language Model Compression", section 5, implements the static KV
 * cache, the mask and the attention aggregation in a CUDA kernel.
 *
 * Conventions for every entry point
 *  - Device pointers are plain CUDA device addresses owned by the caller; the
 *    library never allocates or frees device memory.  Host pointers are read
 *    (or written) before the call returns unless stated otherwise.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Device work is enqueued asynchronously on it; the caller keeps every
 *    buffer alive until that work has completed.
 *  - Argument errors are detected on the host, return a status and launch
 *    nothing.  Launch failures return MOA_ERR_CUDA.  Host memory that a
 *    launch's plan needs (the prefill's work schedule) and cannot get returns
 *    MOA_ERR_HOST, with nothing launched.  Nothing calls exit/abort, and no
 *    C++ exception leaves the library.
 *  - Tensors are dense, row-major, 16-byte aligned:
 *      q, o : [B, Hq,  N, d]     k, v : [B, Hkv, N, d]     (prefill)
 *      q, o : [B, Hq,  d]        k, v : [B, Hkv, n_tok, d] (decode / append)
 *    with grouped-query attention: query head h reads key/value head h / (Hq/Hkv).
 *  - Supported: d in {64, 128}; dtype MOA_F32 for d 64/128 (SIMT, fp32
 *    throughout); dtype MOA_BF16 for d 128 (tensor cores, fp32 accumulate).
 *    Hq <= 128, Hkv <= 128, Hq % Hkv == 0, 1 <= N < 2^31, B >= 1.
 */
#ifndef MOA_H
#define MOA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOA_OK = 0,
  MOA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or shape, NaN rule */
  MOA_ERR_CAPACITY = 2,     /* a span exceeds its key/value head's cache capacity  */
  MOA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than moa_workspace_bytes */
  MOA_ERR_UNSUPPORTED = 4,  /* valid request the library does not implement (e.g. bf16 d=64) */
  MOA_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed */
  MOA_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up (error word set) */
  MOA_ERR_HOST = 7          /* host-side memory for a launch's plan could not be had (nothing launched) */
} moa_status;

typedef enum { MOA_F32 = 0, MOA_BF16 = 1 } moa_dtype;

typedef enum { MOA_OP_PREFILL = 0, MOA_OP_DECODE = 1 } moa_op;

/* Opaque host-side handle describing a caller-owned cache buffer. */
typedef struct moa_kv_cache moa_kv_cache;

/* Human-readable name of a status code (static string, never NULL). */
const char* moa_status_string(moa_status s);

/* ---------------------------------------------------------------------------
 * Span rule.  "Mixture of Attention" project page, "Finding two" (S = alpha +
 * beta * N), "Method design / Elastic search space" (spans respect the
 * kernel's block size) and the heads A/B/C panel (span clamped to N).
 *   x = alpha[h] + beta[h] * (double)N      (binary64, two separate roundings)
 *   S = block * floor(x / block + 0.5)      (nearest multiple, ties up)
 *   spans_out[h] = min(N, max(block, S))
 * Host only; no CUDA call.  alpha/beta must be finite and >= 0, N >= 1,
 * 1 <= block, n_heads >= 1.  Writes n_heads int32 values.  Spans above
 * INT32_MAX cannot occur because N < 2^31 is required.
 * ------------------------------------------------------------------------- */
moa_status moa_rules_eval(const double* alpha, const double* beta, int32_t n_heads,
                          int64_t N, int32_t block, int32_t* spans_out);

/* ---------------------------------------------------------------------------
 * Per-head ring-buffer KV cache ("Demo" step 03: fixed-size per-head cache).
 * Key/value head g of each sequence owns C_g = capacity[g] slots; token
 * position p lives in slot p mod C_g, so the ring always holds the last C_g
 * tokens, which serve every query head of the group whose span is <= C_g.
 *
 * Buffer layout (caller-owned device memory, size from moa_kv_bytes):
 *   header, H = round_up(16 + 8*B, 256) bytes:
 *     bytes 0..3   uint32 error word (0 = ok; bit 0 = bounded wait timed out,
 *                  bit 1 = decode found an empty sequence)
 *     bytes 4..7   uint32 append-completion counter (internal, returns to 0)
 *     bytes 8..15  reserved, zero
 *     bytes 16..   int64 t[B]: tokens appended so far, per sequence
 *   data at byte H: for b in [0,B), for g in [0,Hkv): K block [C_g][d], then
 *     V block [C_g][d], elements of the cache dtype.  The K block of (b, g)
 *     starts at element (b * sum_g C_g + sum_{g'<g} C_g') * 2 * d.
 * ------------------------------------------------------------------------- */

/* Bytes of the buffer for the layout above.  capacity: host int32[Hkv], >= 1. */
moa_status moa_kv_bytes(int32_t B, int32_t Hkv, int32_t d, moa_dtype dtype,
                        const int32_t* capacity, size_t* bytes_out);

/* Size of the header region (the data region starts at this byte offset). */
moa_status moa_kv_header_bytes(int32_t B, size_t* bytes_out);

/* Bind a caller-owned device buffer of at least moa_kv_bytes bytes (256-byte
 * aligned) as an empty cache: zeroes the whole buffer on `stream` and returns a
 * new host handle in *out.  The handle copies `capacity`; it never owns
 * dev_buf.  Release the handle with moa_kv_free. */
moa_status moa_kv_alloc(void* dev_buf, size_t bytes, int32_t B, int32_t Hkv, int32_t d,
                        moa_dtype dtype, const int32_t* capacity, void* stream,
                        moa_kv_cache** out);

/* Free the host handle (not the device buffer).  NULL is accepted. */
moa_status moa_kv_free(moa_kv_cache* cache);

/* Append n_tok >= 1 tokens per sequence.  k, v: device [B, Hkv, n_tok, d] in
 * the cache dtype.  Token r of sequence b gets position t_b + r and is stored
 * in slot (t_b + r) mod C_g; only the last min(n_tok, C_g) rows are copied,
 * the rest would be overwritten.  Then t_b += n_tok (on the device, in the
 * same launch).  Calls on one cache must be ordered on one stream. */
moa_status moa_kv_append(moa_kv_cache* cache, const void* k, const void* v,
                         int32_t n_tok, void* stream);

/* Read t[B] into host memory t_host and check the error word.  Synchronises
 * `stream`.  Returns MOA_ERR_TIMEOUT if error bit 0 is set, MOA_ERR_INVALID_ARG
 * if only bit 1 is (a decode ran on a sequence with no cached token), else
 * MOA_OK.  The error word is sticky: clear it by re-binding the buffer. */
moa_status moa_kv_positions(const moa_kv_cache* cache, int64_t* t_host, void* stream);

/* Overwrite t[B] from host memory (e.g. restoring a cache whose data bytes the
 * caller saved and copied back).  Enqueued on `stream`; t_host is consumed
 * before return.  Every t_host[b] must be >= 0. */
moa_status moa_kv_set_positions(moa_kv_cache* cache, const int64_t* t_host, void* stream);

/* Device address of the data region and the slot offset of each key/value
 * head: group_row_offset[g] = sum_{g'<g} C_g' for g in [0, Hkv], so
 * group_row_offset[Hkv] = sum_g C_g.  group_row_offset may be NULL. */
moa_status moa_kv_layout(const moa_kv_cache* cache, void** data_out, int64_t* group_row_offset);

/* ---------------------------------------------------------------------------
 * Workspace.  Caller-owned device scratch, 256-byte aligned.  A decode
 * workspace must be zeroed once before its first use (moa_workspace_init or a
 * memset); moa_decode leaves its counters at zero again.  A prefill workspace
 * needs no initialisation.  Word 0 of every workspace is an error word.
 * `spans` is host int32[Hq]; N is ignored for MOA_OP_DECODE.
 * ------------------------------------------------------------------------- */
moa_status moa_workspace_bytes(moa_op op, int32_t B, int32_t Hq, int64_t N, int32_t d,
                               const int32_t* spans, size_t* bytes_out);

/* Zero `bytes` bytes of workspace on `stream`. */
moa_status moa_workspace_init(void* workspace, size_t bytes, void* stream);

/* Synchronise `stream` and read the workspace error word: MOA_ERR_TIMEOUT if a
 * bounded wait in the last prefill using it gave up, else MOA_OK. */
moa_status moa_workspace_check(const void* workspace, void* stream);

/* Self-test of the failure path of the prefill kernel.  Every wait of the
 * kernel on an mbarrier gives up after 2 s of wall time, records
 * MOA_ERR_TIMEOUT in the workspace error word, lets the other roles leave,
 * waits for its in-flight copies, frees its tensor memory and returns, so a
 * lost arrival ends as a status instead of a hung GPU.  This call launches the
 * kernel on a 1 x 1 x 128 x 128 bf16 problem (q, k, v, o: device, 16-byte
 * aligned, 32 KB each) with its work-unit records withheld, so that path runs:
 * after about 2 s moa_workspace_check(workspace) returns MOA_ERR_TIMEOUT and
 * the context stays usable.  workspace: at least
 * moa_workspace_bytes(MOA_OP_PREFILL, 1, 1, 128, 128, {128}) bytes, 256-byte
 * aligned.  Not part of the attention path. */
moa_status moa_prefill_stall_test(const void* q, const void* k, const void* v, void* o, void* workspace,
                                  size_t ws_bytes, void* stream);

/* Read-only bandwidth probe for the decode roofline.  Decode attention
 * reads each head's window of K/V rows once per token and writes almost
 * nothing, so its bandwidth ceiling is a plain read stream.  Reads `bytes`
 * of device memory at `buf` once with the decode kernel's access width
 * (16-byte loads, every SM) and writes their checksum to `out` (device
 * uint64): with the buffer seen as little-endian uint32 words, the XOR of
 * the even-indexed words in the high half and of the odd-indexed words in
 * the low half.  buf must be 16-byte aligned, bytes a multiple of 16, out
 * 8-byte aligned (else MOA_ERR_INVALID_ARG, nothing launched).  Enqueued on
 * `stream`; the caller owns both buffers. */
moa_status moa_stream_read(const void* buf, size_t bytes, void* out, void* stream);

/* ---------------------------------------------------------------------------
 * Prefill: windowed causal attention over a whole prompt ("Finding two" and
 * its N x N causal-band figure; blog section 2.1).  For every (b, h, i):
 *   o[b,h,i,:] = softmax_j(scale * q[b,h,i,:] . k[b,g,j,:]) v[b,g,j,:]
 * over j in (i - S_h, i], g = h / (Hq/Hkv).  spans: host int32[Hq], each >= 1
 * (a span above N behaves as N).  MOA_BF16 runs the tensor-core kernel (d must
 * be 128) and needs a workspace of moa_workspace_bytes(MOA_OP_PREFILL, ...)
 * bytes; MOA_F32 may pass workspace NULL.  The schedule of work units is
 * uploaded into the workspace from host memory on every call.
 * fill_or_null: if non-NULL, a cache with B, Hkv, d and dtype equal to this
 * call's, spans[h] <= C_{h/(Hq/Hkv)}; the prompt's K/V are appended to it
 * exactly as moa_kv_append(cache, k, v, N) would (same bytes and positions).
 * MOA_BF16 writes the cache inside the prefill kernel (one launch in all);
 * MOA_F32 appends with a second launch.
 * ------------------------------------------------------------------------- */
moa_status moa_prefill(const void* q, const void* k, const void* v, void* o,
                       int32_t B, int32_t Hq, int32_t Hkv, int64_t N, int32_t d,
                       moa_dtype dtype, const int32_t* spans, float scale,
                       void* workspace, size_t ws_bytes, moa_kv_cache* fill_or_null,
                       void* stream);

/* Host view of the prefill schedule.  The kernel's work unit is two
 * consecutive query tiles of 128 rows (m, m+1) of one (sequence, head),
 * sharing one stream of key/value tiles (a head with an odd number of query
 * tiles ends with a one-tile unit).  Units are sorted longest first and dealt
 * to n_ctas per-CTA lists (1 <= n_ctas <= 1024; moa_prefill uses the number
 * of SMs, or fewer when there are fewer units) by the greedy
 * longest-processing-time rule.  One row of 7 int32 per query tile, a unit's
 * rows adjacent, each CTA's units in the order it runs them:
 * (cta, unit, b, h, m, lo, hi) -- query rows [128m, 128m+127] visit key tiles
 * lo..hi of 128 keys (hi = m, the diagonal tile).  Writes min(cap, n) rows,
 * *n_rows_out = n.  Host only. */
moa_status moa_prefill_schedule(int32_t B, int32_t Hq, int64_t N, const int32_t* spans,
                                int32_t n_ctas, int32_t* rows_out, int64_t cap,
                                int64_t* n_rows_out);

/* ---------------------------------------------------------------------------
 * Chunked prefill: a prompt that arrives in pieces, served from the same
 * fixed-size per-head cache as decode ("Mixture of Attention" project page,
 * "Demo" step 03; the windowed attention of "Finding two" at an offset).
 * Sequence b holds t_b tokens in `cache`; q, k, v hold its next n tokens
 * (positions t_b .. t_b+n-1).  Query i of head h attends to positions
 * j in (t_b + i - S_h, t_b + i], j >= 0: the older ones read through the
 * ring, the chunk's own from k, v.  Then the chunk is appended (the cache
 * ends as after moa_kv_append(cache, k, v, n)).  With t_b = 0 this is
 * moa_prefill of the chunk with fill.
 *   q, o: device [B, Hq, n, d]; k, v: device [B, Hkv, n, d]; all 16-byte
 *   aligned, bf16, d = 128 (other caches: MOA_ERR_UNSUPPORTED).
 *   spans: host int32[Hq], 1 <= spans[h] <= C_{h/(Hq/Hkv)}, else
 *   MOA_ERR_CAPACITY.
 *   workspace: moa_chunk_workspace_bytes(...) bytes, 256-byte aligned, no
 *   initialisation needed; it holds the work-unit schedule and the window's
 *   key/value rows gathered from the ring, [B, Hkv, W, d] with
 *   W = max_h S_h - 1 rounded up to 128.
 * Two launches on `stream` (one when every span is 1): the window gather,
 * then the tensor-core prefill kernel (key tiles below W from the gathered
 * rows, the chunk's own straight from k, v; rows of negative positions
 * masked), which also appends the chunk to the ring.  Errors as
 * moa_prefill. */
moa_status moa_chunk_workspace_bytes(const moa_kv_cache* cache, int32_t Hq, int32_t n,
                                     const int32_t* spans, size_t* bytes_out);
moa_status moa_prefill_chunk(moa_kv_cache* cache, const void* q, const void* k, const void* v,
                             void* o, int32_t Hq, int32_t n, const int32_t* spans, float scale,
                             void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Decode: one new query token per sequence against the ring cache.  Call
 * moa_kv_append for the token's k, v first; then query head h of sequence b
 * (at position t_b - 1) attends to positions j in (t_b - 1 - S_h, t_b - 1],
 * read from slots j mod C_g.  q, o: device [B, Hq, d] in the cache dtype.
 * spans: host int32[Hq], 1 <= spans[h] <= C_{h/(Hq/Hkv)}, else MOA_ERR_CAPACITY.
 * workspace: moa_workspace_bytes(MOA_OP_DECODE, ...) bytes, zeroed before
 * first use.  One kernel launch: split-KV partials with the log-sum-exp
 * combine done by the last split of each (b, h).
 * ------------------------------------------------------------------------- */
moa_status moa_decode(moa_kv_cache* cache, const void* q, void* o, int32_t Hq,
                      const int32_t* spans, float scale, void* workspace, size_t ws_bytes,
                      void* stream);

/* One decode step in one launch: the same result, cache bytes and positions as
 * moa_kv_append(cache, k, v, 1) followed by moa_decode(cache, q, o, ...)
 * ("Mixture of Attention" project page, "Demo" step 03: the fixed-size
 * per-head cache is written at slot t mod C_g and each head attends to its
 * last S_h positions).  k, v: [B, Hkv, 1, d] device, 16-byte aligned.  The
 * window entry of the new token is taken from k, v directly; one CTA per
 * (sequence, kv head) writes it to its slot, and the last CTA of each
 * sequence to have read t_b advances it.  Workspace and errors as moa_decode. */
moa_status moa_decode_append(moa_kv_cache* cache, const void* q, const void* k, const void* v,
                             void* o, int32_t Hq, const int32_t* spans, float scale,
                             void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Band plus global ("sink") tokens.  The codewithpapers page for arXiv
 * 2406.14909 lists, from the official repository, a global-pattern generator
 * (gen_global_pattern) beside the band pattern and StreamingLLM density
 * counters; the project page's Table 4 compares with StreamingLLM.  The pages
 * give no formula; the reading taken: query head h keeps its band and, in
 * addition, attends to the first k_h positions of the sequence (those that
 * are causal), each key once:
 *   keys(i) = { j : i - S_h < j <= i }  union  { j : 0 <= j < k_h, j <= i }.
 * k_h = 0 for every head gives exactly the plain entry points above.
 *
 * A cache that serves such heads keeps, besides the ring, the first K_g
 * positions of every sequence for good: sink_capacity[g] = K_g >= the k_h of
 * every query head of key/value head g.  Layout: the plain layout above
 * (header, ring region), then the global-token region: for b in [0,B), for g
 * in [0,Hkv): K rows [K_g][d], then V rows [K_g][d]; position p < K_g at row
 * p.  Its block for (b, g) starts at element
 * (b * sum_g K_g + sum_{g'<g} K_g') * 2 * d of the region, which starts at
 * byte H + B * sum_g C_g * 2 * d * elem_size.  Every append (moa_kv_append,
 * the prefill fill, the fused decode append, the chunked prefill) also writes
 * positions below K_g there.  sum_g K_g <= 2^31 - 1.
 * ------------------------------------------------------------------------- */

/* moa_kv_bytes / moa_kv_alloc for a cache with global-token rows.
 * sink_capacity: host int32[Hkv], each >= 0 (NULL = all 0, the plain cache). */
moa_status moa_kv_bytes_sink(int32_t B, int32_t Hkv, int32_t d, moa_dtype dtype,
                             const int32_t* capacity, const int32_t* sink_capacity,
                             size_t* bytes_out);
moa_status moa_kv_alloc_sink(void* dev_buf, size_t bytes, int32_t B, int32_t Hkv, int32_t d,
                             moa_dtype dtype, const int32_t* capacity,
                             const int32_t* sink_capacity, void* stream, moa_kv_cache** out);

/* moa_prefill with global tokens: sinks is host int32[Hq], each >= 0 (values
 * above N behave as N).  With fill_or_null, sinks[h] <= K_{h/(Hq/Hkv)} of the
 * cache (else MOA_ERR_CAPACITY).  Same kernels, launches, workspace and errors
 * as moa_prefill: the tensor-core kernel adds to each query tile's band the
 * key tiles that hold its global tokens. */
moa_status moa_prefill_sink(const void* q, const void* k, const void* v, void* o,
                            int32_t B, int32_t Hq, int32_t Hkv, int64_t N, int32_t d,
                            moa_dtype dtype, const int32_t* spans, const int32_t* sinks,
                            float scale, void* workspace, size_t ws_bytes,
                            moa_kv_cache* fill_or_null, void* stream);

/* Decode workspace size with global tokens (sinks: host int32[Hq], >= 0);
 * for MOA_OP_PREFILL it equals moa_workspace_bytes. */
moa_status moa_workspace_bytes_sink(moa_op op, int32_t B, int32_t Hq, int64_t N, int32_t d,
                                    const int32_t* spans, const int32_t* sinks,
                                    size_t* bytes_out);

/* moa_decode / moa_decode_append with global tokens: the query at position
 * t = t_b - 1 of head h attends to keys(t) above, its band through the ring
 * and the global tokens below the band from the global-token rows.
 * sinks: host int32[Hq], 0 <= sinks[h] <= K_{h/(Hq/Hkv)} (else
 * MOA_ERR_CAPACITY).  workspace: moa_workspace_bytes_sink(MOA_OP_DECODE, ...)
 * bytes, zeroed before first use.  One launch: the split-KV kernel with more
 * splits over the global-token rows (per head, or for bf16 d = 128 with 2, 4
 * or 8 query heads per key/value head per group, the group's rows read once
 * for all its heads).  Errors as moa_decode. */
moa_status moa_decode_sink(moa_kv_cache* cache, const void* q, void* o, int32_t Hq,
                           const int32_t* spans, const int32_t* sinks, float scale,
                           void* workspace, size_t ws_bytes, void* stream);
moa_status moa_decode_append_sink(moa_kv_cache* cache, const void* q, const void* k,
                                  const void* v, void* o, int32_t Hq, const int32_t* spans,
                                  const int32_t* sinks, float scale, void* workspace,
                                  size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Decode without a caller workspace.  The paper has no counterpart: this is
 * a deployment convenience of this library.
 *
 * Same computation, arguments and errors as moa_decode, minus the workspace
 * (one more error below).
 * It is for callers that cannot allocate device memory -- e.g. an operator
 * plugin that its host framework gives only input and output pointers, a
 * runtime whose device memory is entirely owned by another allocator, or code
 * that must not call cudaMalloc because that call synchronises the device.
 * The split partials and tickets live instead in one fixed 8 MiB scratch
 * array inside libmoa's device image, which every GPU that loads the library
 * keeps until the process exits.  The caller still passes q, o and the cache.
 *  - Requests whose decode workspace (moa_workspace_bytes(MOA_OP_DECODE, ...))
 *    exceeds 8 MiB return MOA_ERR_WORKSPACE and launch nothing.
 *  - The first call on each device looks up the array's device address with
 *    that device current (cudaGetSymbolAddress); make that first call before
 *    any stream capture.
 *  - Each call clears the array's tickets on `stream`, then launches the
 *    decode kernel; the array keeps the last call's partials.  All calls on a
 *    device share the array, so calls whose work overlaps on the GPU (other
 *    streams, unordered threads) race and may return wrong outputs.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *  - Errors beyond moa_decode's: MOA_ERR_UNSUPPORTED when the current device
 *    index is 64 or more (the per-device address table holds 64 devices).
 * ------------------------------------------------------------------------- */
moa_status moa_decode_static_ws(moa_kv_cache* cache, const void* q, void* o, int32_t Hq,
                                const int32_t* spans, float scale, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOA_H */
