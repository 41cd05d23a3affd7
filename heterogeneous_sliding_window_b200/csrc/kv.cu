// Per-head ring-buffer KV cache: append kernel.
//
// "Mixture of Attention" project page, "Demo" step 03: decoding is served
// from a fixed-size KV cache sized per head.  Token position p of a sequence
// is kept in slot p mod C_g of its key/value head g, so the buffer always
// holds the last C_g tokens -- all that a head with span S_h <= C_g reads.
// A cache that serves heads with global tokens also keeps positions p < K_g
// for good, at row p of its global-token region.
#include <algorithm>

#include "internal.h"

namespace moa {
namespace {

constexpr int kAppendRows = 64;      // rows per block and per key/value head
constexpr int kAppendThreads = 256;

struct AppendParams {
  char* data;                 // data region of the cache buffer
  uint32_t* ctr;              // header: completion counter
  int64_t* t;                 // header: tokens per sequence
  const char* k;
  const char* v;
  int32_t Hkv, n_tok, row_bytes;
  int64_t sumC;
  int32_t cap[MOA_MAX_HEADS];
  int64_t goff[MOA_MAX_HEADS];
  // global-token rows (sink == nullptr: none); blocks x >= ring_blocks copy them
  char* sink;
  int64_t sumK;
  int32_t ring_blocks;
  int32_t scap[MOA_MAX_HEADS];
  int64_t soff[MOA_MAX_HEADS];
};

__global__ void __launch_bounds__(kAppendThreads) append_kernel(const __grid_constant__ AppendParams p) {
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int C = p.cap[g];
  const int nrows = p.n_tok < C ? p.n_tok : C;   // only the last C rows survive
  const int64_t t0 = p.t[b];
  if ((int)blockIdx.x >= p.ring_blocks) {
    // global-token rows: token r at position t0 + r < K_g goes to row t0 + r
    const int r0 = ((int)blockIdx.x - p.ring_blocks) * kAppendRows;
    const int64_t lim = min((int64_t)p.n_tok, (int64_t)p.scap[g] - t0);
    if (p.sink != nullptr && r0 < lim) {
      const int rows = (int)min((int64_t)kAppendRows, lim - r0);
      const int vpr = p.row_bytes / 16;
      char* kdst = p.sink + (size_t)((int64_t)b * p.sumK + p.soff[g]) * 2 * p.row_bytes;
      char* vdst = kdst + (size_t)p.scap[g] * p.row_bytes;
      const size_t src_base = ((size_t)b * p.Hkv + g) * (size_t)p.n_tok;
      for (int idx = threadIdx.x; idx < rows * vpr; idx += kAppendThreads) {
        const int rr = idx / vpr;
        const int vv = idx - rr * vpr;
        const int r = r0 + rr;
        const size_t src = (src_base + r) * p.row_bytes + (size_t)vv * 16;
        const size_t dst = (size_t)(t0 + r) * p.row_bytes + (size_t)vv * 16;
        *reinterpret_cast<int4*>(kdst + dst) = __ldg(reinterpret_cast<const int4*>(p.k + src));
        *reinterpret_cast<int4*>(vdst + dst) = __ldg(reinterpret_cast<const int4*>(p.v + src));
      }
    }
  } else if (blockIdx.x * kAppendRows < nrows) {
    const int r0 = blockIdx.x * kAppendRows;
    const int rows = min(kAppendRows, nrows - r0);
    const int vpr = p.row_bytes / 16;
    const int first = p.n_tok - nrows;          // source row of the first survivor
    char* kdst = p.data + (size_t)((int64_t)b * p.sumC + p.goff[g]) * 2 * p.row_bytes;
    char* vdst = kdst + (size_t)C * p.row_bytes;
    const size_t src_base = ((size_t)b * p.Hkv + g) * (size_t)p.n_tok;
    for (int idx = threadIdx.x; idx < rows * vpr; idx += kAppendThreads) {
      const int rr = idx / vpr;
      const int vv = idx - rr * vpr;
      const int r = first + r0 + rr;
      const int64_t slot = (t0 + r) % C;
      const size_t src = (src_base + r) * p.row_bytes + (size_t)vv * 16;
      const size_t dst = (size_t)slot * p.row_bytes + (size_t)vv * 16;
      const int4 kv = __ldg(reinterpret_cast<const int4*>(p.k + src));
      const int4 vv4 = __ldg(reinterpret_cast<const int4*>(p.v + src));
      *reinterpret_cast<int4*>(kdst + dst) = kv;
      *reinterpret_cast<int4*>(vdst + dst) = vv4;
    }
  }
  // The last block to finish advances every sequence's position.  All blocks
  // read t[b] above, before they take a ticket, so none sees the new value.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned total = gridDim.x * gridDim.y * gridDim.z;
    const unsigned prev = atomicAdd(p.ctr, 1u);
    if (prev == total - 1) {
      const int B = gridDim.z;
      for (int bb = 0; bb < B; ++bb) p.t[bb] += p.n_tok;
      *p.ctr = 0u;
      __threadfence();
    }
  }
}

// Window gather for a chunk: row r of (b, g) is position t_b - W + r, read
// through the ring (zeros for positions below 0 or older than the ring
// holds).  Rows below R_g = 128 * floor((W - C_g + 1) / 128) are never in a
// visited key tile of the group's heads (every span is <= C_g), so they are
// skipped.
constexpr int kGatherRows = 64;

struct GatherParams {
  const char* data;           // data region of the cache buffer
  const int64_t* t;           // header: tokens per sequence
  char* sk;                   // [B, Hkv, W, d]
  char* sv;
  int32_t Hkv, W, row_bytes;
  int64_t sumC;
  int32_t cap[MOA_MAX_HEADS];
  int64_t goff[MOA_MAX_HEADS];
};

__global__ void __launch_bounds__(kAppendThreads) gather_window_kernel(const __grid_constant__ GatherParams p) {
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int C = p.cap[g];
  const int lowest = p.W - C + 1 > 0 ? (p.W - C + 1) / 128 * 128 : 0;
  const int r0 = lowest + blockIdx.x * kGatherRows;
  if (r0 >= p.W) return;
  const int rows = min(kGatherRows, p.W - r0);
  const int vpr = p.row_bytes / 16;
  const int64_t t0 = p.t[b];
  const char* kring = p.data + (size_t)((int64_t)b * p.sumC + p.goff[g]) * 2 * p.row_bytes;
  const char* vring = kring + (size_t)C * p.row_bytes;
  const size_t zrow = ((size_t)b * p.Hkv + g) * (size_t)p.W;
  for (int idx = threadIdx.x; idx < rows * vpr; idx += kAppendThreads) {
    const int rr = idx / vpr;
    const int vv = idx - rr * vpr;
    const int r = r0 + rr;
    int4 kx = make_int4(0, 0, 0, 0), vx = make_int4(0, 0, 0, 0);
    const int64_t pos = t0 - p.W + r;
    if (pos >= 0 && pos >= t0 - C) {
      const size_t src = (size_t)(pos % C) * p.row_bytes + (size_t)vv * 16;
      kx = __ldg(reinterpret_cast<const int4*>(kring + src));
      vx = __ldg(reinterpret_cast<const int4*>(vring + src));
    }
    const size_t dst = (zrow + r) * p.row_bytes + (size_t)vv * 16;
    *reinterpret_cast<int4*>(p.sk + dst) = kx;
    *reinterpret_cast<int4*>(p.sv + dst) = vx;
  }
}

}  // namespace

moa_status launch_gather_window(const moa_kv_cache* c, int32_t W, void* sk, void* sv, cudaStream_t s) {
  GatherParams p;
  p.data = c->buf + c->header;
  p.t = reinterpret_cast<const int64_t*>(c->buf + kHdrT);
  p.sk = (char*)sk;
  p.sv = (char*)sv;
  p.Hkv = c->Hkv;
  p.W = W;
  p.row_bytes = c->d * (int)elem_bytes(c->dtype);
  p.sumC = c->goff[c->Hkv];
  int max_rows = 0;
  for (int g = 0; g < c->Hkv; ++g) {
    p.cap[g] = c->cap[g];
    p.goff[g] = c->goff[g];
    const int lowest = W - c->cap[g] + 1 > 0 ? (W - c->cap[g] + 1) / 128 * 128 : 0;
    max_rows = std::max(max_rows, W - lowest);
  }
  dim3 grid((max_rows + kGatherRows - 1) / kGatherRows, c->Hkv, c->B);
  gather_window_kernel<<<grid, kAppendThreads, 0, s>>>(p);
  return check_launch("window gather launch");
}

moa_status launch_append(moa_kv_cache* c, const void* k, const void* v, int32_t n_tok,
                         cudaStream_t s) {
  AppendParams p;
  p.data = c->buf + c->header;
  p.ctr = reinterpret_cast<uint32_t*>(c->buf + kHdrAppendCtr);
  p.t = reinterpret_cast<int64_t*>(c->buf + kHdrT);
  p.k = (const char*)k;
  p.v = (const char*)v;
  p.Hkv = c->Hkv;
  p.n_tok = n_tok;
  p.row_bytes = c->d * (int)elem_bytes(c->dtype);
  p.sumC = c->goff[c->Hkv];
  int maxrows = 0, maxsink = 0;
  for (int g = 0; g < c->Hkv; ++g) {
    p.cap[g] = c->cap[g];
    p.goff[g] = c->goff[g];
    p.scap[g] = c->scap[g];
    p.soff[g] = c->soff[g];
    const int r = n_tok < c->cap[g] ? n_tok : c->cap[g];
    if (r > maxrows) maxrows = r;
    maxsink = std::max(maxsink, std::min(n_tok, c->scap[g]));
  }
  p.sink = sink_region(c);
  p.sumK = c->soff[c->Hkv];
  p.ring_blocks = (maxrows + kAppendRows - 1) / kAppendRows;
  // the global-token blocks cover the first min(n_tok, K_g) tokens; which of
  // them land (positions below K_g) is decided on the device from t_b
  const int sink_blocks = p.sink ? (maxsink + kAppendRows - 1) / kAppendRows : 0;
  dim3 grid(p.ring_blocks + sink_blocks, c->Hkv, c->B);
  append_kernel<<<grid, kAppendThreads, 0, s>>>(p);
  return check_launch("append launch");
}

}  // namespace moa
