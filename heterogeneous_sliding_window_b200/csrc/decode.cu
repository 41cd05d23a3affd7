// Decode attention against the per-head ring-buffer cache (split-KV).
//
// One new query token per sequence.  Query head h attends to its last S_h
// cached positions ("Mixture of Attention" project page, "Finding two": the
// per-head window; "Demo" step 03: fixed-size per-head KV cache).  The work is
// HBM-bound: every cached key and value of the window is read once.
//
// Grid: one CTA per (sequence b, head h, split s) where split s covers window
// entries [s*kChunk, (s+1)*kChunk).  A CTA
//   1. streams its K rows with 16-byte loads (a row is spread over LPR lanes),
//      forms q.k in fp32 and reduces each dot product with xor-shuffles;
//   2. takes the chunk max m and p_j = 2^(s_j - m), l = sum p_j;
//   3. streams its V rows and accumulates sum p_j v_j in fp32;
//   4. single split: writes o = acc / l.  Otherwise writes (m, l, acc) to the
//      workspace; the last split of (b, h) to finish (atomic ticket) merges all
//      partials with the log-sum-exp rule and writes o, then rearms its ticket.
#include <cuda_bf16.h>

#include "internal.h"

namespace moa {
namespace {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kChunk = 256;          // window entries per split
constexpr int kUnroll = 4;           // independent 16-byte loads in flight per thread

struct DecodeParams {
  const char* data;                  // cache data region
  const int64_t* t;                  // cache header: tokens per sequence
  uint32_t* err;                     // cache header: error word
  const void* q;
  void* o;
  float* part_o;                     // [B * items_per_b, D]
  float* part_ml;                    // [B * items_per_b, 2]
  uint32_t* ctr;                     // [B * Hq] tickets
  int32_t Hq, G, items_per_b;
  float scale_log2;
  int64_t sumC;
  int32_t span[MOA_MAX_HEADS];
  int32_t split_pre[MOA_MAX_HEADS + 1];
  int32_t cap[MOA_MAX_HEADS];
  int64_t goff[MOA_MAX_HEADS];
};

template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void cvt(const int4 r, float* f) {
    f[0] = __int_as_float(r.x); f[1] = __int_as_float(r.y);
    f[2] = __int_as_float(r.z); f[3] = __int_as_float(r.w);
  }
  __device__ static void store(float* dst, float x) { *dst = x; }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void cvt(const int4 r, float* f) {
    const uint32_t w[4] = {(uint32_t)r.x, (uint32_t)r.y, (uint32_t)r.z, (uint32_t)r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static void store(__nv_bfloat16* dst, float x) { *dst = __float2bfloat16_rn(x); }
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int VE = Vec16<T>::N;     // elements per 16-byte vector
  constexpr int LPR = D / VE;         // lanes per cached row
  constexpr int RPW = 32 / LPR;       // rows per warp per step
  constexpr int RPS = RPW * kDecWarps;
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row must map onto a warp");

  __shared__ float sc[kChunk];
  __shared__ float red[RPS][D];
  __shared__ float wred[kDecWarps];
  __shared__ int last_flag;

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR, li = lane % LPR;

  const int item = blockIdx.x;
  const int b = item / p.items_per_b;
  const int r = item - b * p.items_per_b;
  int lo = 0, hi = p.Hq - 1;          // head h: last h with split_pre[h] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.split_pre[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const int h = lo;
  const int s = r - p.split_pre[h];
  const int nsplit = p.split_pre[h + 1] - p.split_pre[h];
  const int g = h / p.G;
  const int C = p.cap[g];
  const int64_t tb = p.t[b];
  const int Seff = (int)(tb < (int64_t)p.span[h] ? tb : (int64_t)p.span[h]);
  const int w0 = s * kChunk;
  const int nrows = max(0, min(kChunk, Seff - w0));
  const int64_t pos0 = tb - Seff + w0;                 // first window position of this split
  const int slot0 = nrows > 0 ? (int)(pos0 % C) : 0;

  const T* Kb = reinterpret_cast<const T*>(p.data) + (size_t)((int64_t)b * p.sumC + p.goff[g]) * 2 * D;
  const T* Vb = Kb + (size_t)C * D;

  float qf[VE];
  {
    const int4 raw = __ldg(reinterpret_cast<const int4*>(
        reinterpret_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * D + li * VE));
    Vec16<T>::cvt(raw, qf);
#pragma unroll
    for (int e = 0; e < VE; ++e) qf[e] *= p.scale_log2;
  }

  // Phase 1: scores (log2 domain).
  for (int base = 0; base < nrows; base += RPS * kUnroll) {
    int4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int row = base + u * RPS + warp * RPW + sub;
      if (row < nrows) {
        int slot = slot0 + row;
        if (slot >= C) slot -= C;
        raw[u] = __ldcs(reinterpret_cast<const int4*>(Kb + (size_t)slot * D + li * VE));
      } else {
        raw[u] = make_int4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float kf[VE];
      Vec16<T>::cvt(raw[u], kf);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < VE; ++e) dot = fmaf(qf[e], kf[e], dot);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const int row = base + u * RPS + warp * RPW + sub;
      if (li == 0 && row < nrows) sc[row] = dot;
    }
  }
  __syncthreads();

  // Phase 2: chunk max and exponentials.
  float m = -INFINITY;
  for (int i = tid; i < nrows; i += kDecThreads) m = fmaxf(m, sc[i]);
  m = warp_max(m);
  if (lane == 0) wred[warp] = m;
  __syncthreads();
  m = wred[0];
#pragma unroll
  for (int w = 1; w < kDecWarps; ++w) m = fmaxf(m, wred[w]);
  __syncthreads();
  float l = 0.f;
  for (int i = tid; i < nrows; i += kDecThreads) {
    const float e = exp2f(sc[i] - m);
    sc[i] = e;
    l += e;
  }
  l = warp_sum(l);
  if (lane == 0) wred[warp] = l;
  __syncthreads();
  l = 0.f;
#pragma unroll
  for (int w = 0; w < kDecWarps; ++w) l += wred[w];

  // Phase 3: weighted sum of values.
  float acc[VE];
#pragma unroll
  for (int e = 0; e < VE; ++e) acc[e] = 0.f;
  for (int base = 0; base < nrows; base += RPS * kUnroll) {
    int4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int row = base + u * RPS + warp * RPW + sub;
      if (row < nrows) {
        int slot = slot0 + row;
        if (slot >= C) slot -= C;
        raw[u] = __ldcs(reinterpret_cast<const int4*>(Vb + (size_t)slot * D + li * VE));
      } else {
        raw[u] = make_int4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int row = base + u * RPS + warp * RPW + sub;
      const float pr = row < nrows ? sc[row] : 0.f;
      float vf[VE];
      Vec16<T>::cvt(raw[u], vf);
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = fmaf(pr, vf[e], acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < VE; ++e) red[warp * RPW + sub][li * VE + e] = acc[e];
  __syncthreads();
  float od = 0.f;
  if (tid < D) {
#pragma unroll
    for (int rr = 0; rr < RPS; ++rr) od += red[rr][tid];
  }

  T* out = reinterpret_cast<T*>(p.o) + ((size_t)b * p.Hq + h) * D;
  if (nsplit == 1) {
    if (tid < D) Vec16<T>::store(out + tid, l > 0.f ? od / l : 0.f);
    if (tid == 0 && Seff == 0) atomicOr(p.err, kErrEmpty);
    return;
  }
  const size_t idx = (size_t)b * p.items_per_b + r;
  if (tid < D) p.part_o[idx * D + tid] = od;
  if (tid == 0) {
    p.part_ml[2 * idx] = m;
    p.part_ml[2 * idx + 1] = l;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(&p.ctr[(size_t)b * p.Hq + h], 1u);
    last_flag = (prev == (unsigned)(nsplit - 1));
  }
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  const size_t first = (size_t)b * p.items_per_b + p.split_pre[h];
  float M = -INFINITY;
  for (int ss = 0; ss < nsplit; ++ss) M = fmaxf(M, __ldcg(&p.part_ml[2 * (first + ss)]));
  float L = 0.f, A = 0.f;
  if (M != -INFINITY) {
    for (int ss = 0; ss < nsplit; ++ss) {
      const float ms = __ldcg(&p.part_ml[2 * (first + ss)]);
      const float w = exp2f(ms - M);              // 0 for empty splits (ms = -inf)
      L = fmaf(w, __ldcg(&p.part_ml[2 * (first + ss) + 1]), L);
      if (tid < D) A = fmaf(w, __ldcg(&p.part_o[(first + ss) * D + tid]), A);
    }
  }
  if (tid < D) Vec16<T>::store(out + tid, L > 0.f ? A / L : 0.f);
  if (tid == 0) {
    p.ctr[(size_t)b * p.Hq + h] = 0u;
    if (Seff == 0) atomicOr(p.err, kErrEmpty);
  }
}

struct DecodeLayout {
  int items_per_b;
  size_t ctr_off, ml_off, o_off, total;
};

DecodeLayout decode_layout(int32_t B, int32_t Hq, int32_t d, const int32_t* spans) {
  DecodeLayout L;
  int items = 0;
  for (int h = 0; h < Hq; ++h) items += (spans[h] + kChunk - 1) / kChunk;
  L.items_per_b = items;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  L.ctr_off = 256;
  L.ml_off = L.ctr_off + up((size_t)B * Hq * 4);
  L.o_off = L.ml_off + up((size_t)B * items * 2 * 4);
  L.total = L.o_off + up((size_t)B * items * d * 4);
  return L;
}

}  // namespace

size_t decode_workspace_bytes(int32_t B, int32_t Hq, int32_t d, const int32_t* spans) {
  return decode_layout(B, Hq, d, spans).total;
}

moa_status launch_decode(moa_kv_cache* c, const void* q, void* o, int32_t Hq, const int32_t* spans,
                         float scale, void* ws, size_t ws_bytes, cudaStream_t s) {
  const DecodeLayout L = decode_layout(c->B, Hq, c->d, spans);
  if (ws_bytes < L.total) return MOA_ERR_WORKSPACE;
  DecodeParams p;
  p.data = c->buf + c->header;
  p.t = reinterpret_cast<const int64_t*>(c->buf + kHdrT);
  p.err = reinterpret_cast<uint32_t*>(c->buf + kHdrErr);
  p.q = q;
  p.o = o;
  char* w = (char*)ws;
  p.ctr = reinterpret_cast<uint32_t*>(w + L.ctr_off);
  p.part_ml = reinterpret_cast<float*>(w + L.ml_off);
  p.part_o = reinterpret_cast<float*>(w + L.o_off);
  p.Hq = Hq;
  p.G = Hq / c->Hkv;
  p.items_per_b = L.items_per_b;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.sumC = c->goff[c->Hkv];
  p.split_pre[0] = 0;
  for (int h = 0; h < Hq; ++h) {
    p.span[h] = spans[h];
    p.split_pre[h + 1] = p.split_pre[h] + (spans[h] + kChunk - 1) / kChunk;
  }
  for (int g = 0; g < c->Hkv; ++g) {
    p.cap[g] = c->cap[g];
    p.goff[g] = c->goff[g];
  }
  const long long grid = (long long)c->B * L.items_per_b;
  if (grid > 0x7fffffffLL) return MOA_ERR_UNSUPPORTED;
  if (c->dtype == MOA_BF16) {
    if (c->d == 128) decode_kernel<__nv_bfloat16, 128><<<(unsigned)grid, kDecThreads, 0, s>>>(p);
    else decode_kernel<__nv_bfloat16, 64><<<(unsigned)grid, kDecThreads, 0, s>>>(p);
  } else {
    if (c->d == 128) decode_kernel<float, 128><<<(unsigned)grid, kDecThreads, 0, s>>>(p);
    else decode_kernel<float, 64><<<(unsigned)grid, kDecThreads, 0, s>>>(p);
  }
  return check_launch("decode launch");
}

}  // namespace moa
