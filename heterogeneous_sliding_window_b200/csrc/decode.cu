// Decode attention against the per-head ring-buffer cache (split-KV).
//
// One new query token per sequence.  Query head h attends to its last S_h
// cached positions ("Mixture of Attention" project page, "Finding two": the
// per-head window; "Demo" step 03: fixed-size per-head KV cache).  The work is
// HBM-bound: every cached key and value of the window is read once.
//
// Grid: one CTA per (sequence b, head h, split s) where split s covers window
// entries [s*CH, (s+1)*CH).  The split size is chosen per launch (see
// head_chunk): kChunk when the launch has enough splits to fill the GPU,
// half of it at small batch.  The CTA's 128 threads form row groups of
// LPR lanes (one 16-byte vector of a cached row per lane); each group walks
// its share of the chunk in batches of kUnroll rows, issuing the K and V loads
// of a whole batch together (2*kUnroll 16-byte loads in flight per thread),
// and keeps an online softmax (running max m, sum l, fp32 accumulator) over
// its rows:
//   s_j = scale * q.k_j (xor-shuffle reduction over the group's lanes)
//   m' = max(m, s_j over the batch), acc = acc * 2^(m - m') + sum p_j v_j
// The groups then merge in shared memory with the log-sum-exp rule.  A single
// split writes o = acc / l; otherwise the CTA writes (m, l, acc) to the
// workspace and the last split of (b, h) to finish (atomic ticket) merges all
// partials the same way, writes o, and rearms its ticket.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace moa {
namespace {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
#ifndef MOA_DECODE_CHUNK
#define MOA_DECODE_CHUNK 512
#endif
constexpr int kChunk = MOA_DECODE_CHUNK;   // window entries per split (per-head kernel)
// Group-window entries per split of the group kernels.  1024 measured best on
// Llama3-8B-shaped layers (B=32, context 8192, 50 %: 0.166 ms against 0.174 ms
// at 512 and 0.181 ms at 2048; B=8, context 32768, 25 %: 0.113 ms against
// 0.134 ms at 512): half the splits, half the per-split merges and partials.
#ifndef MOA_GQA_CHUNK
#define MOA_GQA_CHUNK 1024
#endif
constexpr int kGroupChunk = MOA_GQA_CHUNK;
// Number of splits of x entries, chunk at a time (64-bit, so spans up to
// INT32_MAX do not wrap).
__host__ __device__ __forceinline__ int splits_of(int x, int chunk) { return (int)(((long long)x + chunk - 1) / chunk); }
static_assert(kGroupChunk >= kChunk, "group split size (the workspace holds the per-head kernel's slots)");
// Per-head split size at small batch.  A launch with fewer than about one
// wave of CTAs (7 per SM) leaves SMs idle while each CTA streams its long
// split, so such a launch takes splits of kMinChunk = kChunk / 2 entries
// instead.  On one Vicuna-7B-shaped layer (32 heads, context 4096, 50 %) a
// layer took 15.7-15.9 us at batch 1 against 19.0-19.7, 18.3 at batch 2
// against 22.6 and 24.6 at batch 4 against 26.7; 128- and 64-entry splits
// were no better.  Larger launches keep kChunk, which measured best there.
constexpr int kMinChunk = kChunk / 2;
constexpr long long kHeadItems = 1024;
constexpr int kUnroll = 4;           // rows per batch: 2*kUnroll 16-byte loads in flight
// Batches whose rows are contiguous in the ring load from one base pointer at
// constant offsets (1).  Besides the address arithmetic this frees registers
// (71 against 78: seven CTAs per SM instead of six); on the Vicuna-7B-shaped
// step the decode went from 0.939 to 0.955-0.957 of the measured copy.
#ifndef MOA_DECODE_BATCH_FAST
#define MOA_DECODE_BATCH_FAST 1
#endif
constexpr bool kDecodeBatchFast = MOA_DECODE_BATCH_FAST != 0;   // contiguous batches from one base pointer
#ifndef MOA_GROUP_MMA
#define MOA_GROUP_MMA 1
#endif
constexpr bool kGroupMma = MOA_GROUP_MMA != 0;   // tensor-core group kernel for bf16, d = 128
#ifndef MOA_GROUP_MMA2
#define MOA_GROUP_MMA2 1
#endif
constexpr bool kGroupMma2 = MOA_GROUP_MMA2 != 0; // ... also for two query heads per KV head

struct DecodeParams {
  char* data;                        // cache data region
  int64_t* t;                        // cache header: tokens per sequence
  const void* k_new;                 // fused append: the step's k, v [B, Hkv, 1, D]; null otherwise
  const void* v_new;
  uint32_t* bctr;                    // fused append: CTAs of sequence b that have read t[b]
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
  int32_t split_pre[MOA_MAX_HEADS + 1];   // per query head (per KV group in the group kernel)
  int32_t hslot_pre[MOA_MAX_HEADS + 1];   // group kernel: first partial slot of each query head
  int32_t cap[MOA_MAX_HEADS];
  int64_t goff[MOA_MAX_HEADS];
  // Global tokens (per-head kernel only; sink_data == nullptr: none).  Head h
  // has ceil(span/chunk) window splits, then ceil(sink[h]/chunk) splits over
  // the global-token rows of its KV head (K_g = scap[g] rows at soff[g]).
  char* sink_data;
  int64_t sumK;
  int32_t sink[MOA_MAX_HEADS];
  int32_t scap[MOA_MAX_HEADS];
  int64_t soff[MOA_MAX_HEADS];
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

// Fused append: every CTA of sequence b counts itself once all its threads
// have read t[b]; the last of the items_per_b CTAs sets t[b] to t0 + 1 (no
// CTA of this launch reads t[b] after that) and rearms the counter.
__device__ __forceinline__ void step_counted(const DecodeParams& p, int b, int64_t t0) {
  (void)t0;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&p.bctr[b], 1u);
    if (prev == (unsigned)(p.items_per_b - 1)) {
      p.bctr[b] = 0u;
      p.t[b] = t0 + 1;
    }
  }
}

template <typename T, int D, int CH>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int VE = Vec16<T>::N;     // elements per 16-byte vector
  constexpr int LPR = D / VE;         // lanes per cached row
  constexpr int RPW = 32 / LPR;       // row groups per warp
  constexpr int NG = RPW * kDecWarps; // row groups per CTA
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row must map onto a warp");

  __shared__ float g_acc[NG][D];
  __shared__ float g_m[NG], g_l[NG];
  __shared__ int last_flag;

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR, li = lane % LPR;
  const int grp = warp * RPW + sub;

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
  const bool fused = p.k_new != nullptr;
  const int64_t t0 = p.t[b];
  if (fused) step_counted(p, b, t0);
  const int64_t tb = fused ? t0 + 1 : t0;              // tokens attended
  const int Seff = (int)(tb < (int64_t)p.span[h] ? tb : (int64_t)p.span[h]);
  const int nwin = splits_of(p.span[h], CH);           // window splits of head h
  // Splits s >= nwin read the global tokens below the window: positions
  // 0 .. min(k_h, tb - Seff) - 1, at rows of the same index.
  const bool gsplit = s >= nwin;
  const int w0 = (gsplit ? s - nwin : s) * CH;
  const int nent = gsplit ? (int)min((int64_t)p.sink[h], tb - Seff) : Seff;
  const int nrows = max(0, min(CH, nent - w0));
  const int64_t pos0 = tb - Seff + w0;                 // first window position of this split
  const int slot0 = gsplit ? w0 : nrows > 0 ? (int)(pos0 % C) : 0;

  T* Kb = reinterpret_cast<T*>(p.data) + (size_t)((int64_t)b * p.sumC + p.goff[g]) * 2 * D;
  T* Vb = Kb + (size_t)C * D;
  if (gsplit) {
    Kb = reinterpret_cast<T*>(p.sink_data) + (size_t)((int64_t)b * p.sumK + p.soff[g]) * 2 * D;
    Vb = Kb + (size_t)p.scap[g] * D;
  }
  const int Cw = gsplit ? 0x7fffffff : C;              // global-token rows do not wrap
  // fused append: the newest window entry comes from the step's k, v, and the
  // group's first head writes it to its slot (and to its global-token row
  // when its position is below K_g)
  const int e_new = fused && !gsplit ? Seff - 1 : -1;
  const bool writer = fused && h == g * p.G;
  const T* kn = fused ? reinterpret_cast<const T*>(p.k_new) + ((size_t)b * (p.Hq / p.G) + g) * D : nullptr;
  const T* vn = fused ? reinterpret_cast<const T*>(p.v_new) + ((size_t)b * (p.Hq / p.G) + g) * D : nullptr;

  float qf[VE];
  {
    const int4 raw = __ldg(reinterpret_cast<const int4*>(
        reinterpret_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * D + li * VE));
    Vec16<T>::cvt(raw, qf);
#pragma unroll
    for (int e = 0; e < VE; ++e) qf[e] *= p.scale_log2;
  }

  float m = -INFINITY, l = 0.f;
  float acc[VE];
#pragma unroll
  for (int e = 0; e < VE; ++e) acc[e] = 0.f;

  // The trip count is uniform across the CTA (every lane takes part in the
  // shuffles below); rows past the chunk are masked instead.
  for (int base = 0; base < nrows; base += NG * kUnroll) {
    int4 kr[kUnroll], vr[kUnroll];
    // Common case (uniform across the CTA): every row of the batch inside the
    // split, their slots contiguous, none the fused append's new entry: one
    // base pointer per lane and constant offsets.
    int bslot = slot0 + base;
    if (bslot >= Cw) bslot -= Cw;
    if (kDecodeBatchFast && base + NG * kUnroll <= nrows && bslot + NG * kUnroll <= Cw &&
        !(e_new >= w0 + base && e_new < w0 + base + NG * kUnroll)) {
      const T* kp = Kb + (size_t)(bslot + grp) * D + li * VE;
      const T* vp = Vb + (size_t)(bslot + grp) * D + li * VE;
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        kr[u] = __ldcs(reinterpret_cast<const int4*>(kp + (size_t)u * NG * D));
        vr[u] = __ldcs(reinterpret_cast<const int4*>(vp + (size_t)u * NG * D));
      }
    } else
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int row = base + u * NG + grp;
      if (row < nrows) {
        int slot = slot0 + row;
        if (slot >= Cw) slot -= Cw;
        if (w0 + row == e_new) {
          kr[u] = __ldg(reinterpret_cast<const int4*>(kn + li * VE));
          vr[u] = __ldg(reinterpret_cast<const int4*>(vn + li * VE));
          if (writer) {
            *reinterpret_cast<int4*>(Kb + (size_t)slot * D + li * VE) = kr[u];
            *reinterpret_cast<int4*>(Vb + (size_t)slot * D + li * VE) = vr[u];
            if (p.sink_data != nullptr && t0 < (int64_t)p.scap[g]) {
              T* ks = reinterpret_cast<T*>(p.sink_data) + (size_t)((int64_t)b * p.sumK + p.soff[g]) * 2 * D +
                      (size_t)t0 * D;
              *reinterpret_cast<int4*>(ks + li * VE) = kr[u];
              *reinterpret_cast<int4*>(ks + (size_t)p.scap[g] * D + li * VE) = vr[u];
            }
          }
        } else {
          kr[u] = __ldcs(reinterpret_cast<const int4*>(Kb + (size_t)slot * D + li * VE));
          vr[u] = __ldcs(reinterpret_cast<const int4*>(Vb + (size_t)slot * D + li * VE));
        }
      } else {
        kr[u] = make_int4(0, 0, 0, 0);
        vr[u] = make_int4(0, 0, 0, 0);
      }
    }
    float sv[kUnroll];
    float bmax = m;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float kf[VE];
      Vec16<T>::cvt(kr[u], kf);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < VE; ++e) dot = fmaf(qf[e], kf[e], dot);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      sv[u] = (base + u * NG + grp < nrows) ? dot : -INFINITY;
      bmax = fmaxf(bmax, sv[u]);
    }
    if (bmax > m) {                                   // uniform across the group's lanes
      const float corr = exp2f(m - bmax);             // 0 when m = -inf
      l *= corr;
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] *= corr;
      m = bmax;
    }
    // A group that has seen no row yet keeps m = -inf; its masked scores must
    // still give p = 0, not 2^(-inf - -inf) = NaN.
    const float mref = m == -INFINITY ? 0.f : m;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const float pu = exp2f(sv[u] - mref);           // 0 for rows past the chunk
      l += pu;
      float vf[VE];
      Vec16<T>::cvt(vr[u], vf);
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = fmaf(pu, vf[e], acc[e]);
    }
  }

  // merge the row groups (log-sum-exp)
#pragma unroll
  for (int e = 0; e < VE; ++e) g_acc[grp][li * VE + e] = acc[e];
  if (li == 0) {
    g_m[grp] = m;
    g_l[grp] = l;
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < NG; ++k) M = fmaxf(M, g_m[k]);
  float L = 0.f, od = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      const float w = exp2f(g_m[k] - M);
      L = fmaf(w, g_l[k], L);
      if (tid < D) od = fmaf(w, g_acc[k][tid], od);
    }
  }

  T* out = reinterpret_cast<T*>(p.o) + ((size_t)b * p.Hq + h) * D;
  if (nsplit == 1) {
    if (tid < D) Vec16<T>::store(out + tid, L > 0.f ? od / L : 0.f);
    if (tid == 0 && Seff == 0) atomicOr(p.err, kErrEmpty);
    return;
  }
  const size_t idx = (size_t)b * p.items_per_b + r;
  if (tid < D) p.part_o[idx * D + tid] = od;
  if (tid == 0) {
    p.part_ml[2 * idx] = M;
    p.part_ml[2 * idx + 1] = L;
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
  // Merge of the splits' partials by the whole CTA: the maximum and the
  // denominator are reduced over the threads, and each output column sums
  // its splits in four independent chains, so the loads overlap.  A serial
  // walk over the splits would put one L2 round trip per split on the tail
  // of the launch, which at small batch is its critical path.
  __shared__ float w_sh[kDecThreads];
  __shared__ float red[kDecWarps];
  float mx = -INFINITY;
  for (int ss = tid; ss < nsplit; ss += kDecThreads) mx = fmaxf(mx, __ldcg(&p.part_ml[2 * (first + ss)]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  float MM = red[0];
#pragma unroll
  for (int k = 1; k < kDecWarps; ++k) MM = fmaxf(MM, red[k]);
  __syncthreads();                                 // red is reused for the denominator
  float ll = 0.f, A0 = 0.f, A1 = 0.f, A2 = 0.f, A3 = 0.f;
  if (MM != -INFINITY) {
    for (int base = 0; base < nsplit; base += kDecThreads) {
      const int ss = base + tid;
      float w = 0.f;
      if (ss < nsplit) {
        w = exp2f(__ldcg(&p.part_ml[2 * (first + ss)]) - MM);   // 0 for empty splits (m = -inf)
        ll = fmaf(w, __ldcg(&p.part_ml[2 * (first + ss) + 1]), ll);
      }
      w_sh[tid] = w;
      __syncthreads();
      const int n = min(kDecThreads, nsplit - base);
      if (tid < D) {
        const float* po = p.part_o + (first + base) * D + tid;
        int k = 0;
        for (; k + 3 < n; k += 4) {
          A0 = fmaf(w_sh[k], __ldcg(po + (size_t)k * D), A0);
          A1 = fmaf(w_sh[k + 1], __ldcg(po + (size_t)(k + 1) * D), A1);
          A2 = fmaf(w_sh[k + 2], __ldcg(po + (size_t)(k + 2) * D), A2);
          A3 = fmaf(w_sh[k + 3], __ldcg(po + (size_t)(k + 3) * D), A3);
        }
        for (; k < n; ++k) A0 = fmaf(w_sh[k], __ldcg(po + (size_t)k * D), A0);
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ll += __shfl_xor_sync(0xffffffffu, ll, o);
  if ((tid & 31) == 0) red[tid >> 5] = ll;
  __syncthreads();
  float LL = 0.f;
#pragma unroll
  for (int k = 0; k < kDecWarps; ++k) LL += red[k];
  const float A = (A0 + A1) + (A2 + A3);
  if (tid < D) Vec16<T>::store(out + tid, LL > 0.f ? A / LL : 0.f);
  if (tid == 0) {
    p.ctr[(size_t)b * p.Hq + h] = 0u;
    if (Seff == 0) atomicOr(p.err, kErrEmpty);
  }
}

// ---------------------------------------------------------------------------
// Decode for grouped-query attention with the K/V reads shared by the group.
//
// The G query heads of KV group g read windows that all end at the newest
// position and differ only in length, so every cached row of the group's
// longest window is loaded once and applied to each head whose window covers
// it.  Grid: one CTA per (sequence b, group g, split s of the group's window
// of W = min(t_b, C_g) entries); the row groups and batches are those of
// decode_kernel, with G online softmaxes per row group instead of one.  The
// last split of (b, g) to finish merges the partials of all G heads.  Bytes
// read per step drop from the sum of the heads' windows to the group's
// longest window.
// ---------------------------------------------------------------------------
template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecThreads) decode_group_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int VE = Vec16<T>::N;
  constexpr int LPR = D / VE;
  constexpr int RPW = 32 / LPR;
  constexpr int NG = RPW * kDecWarps;
  constexpr int U = G >= 8 ? 4 : 6;   // rows per batch (registers: G q and accumulator vectors)
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row must map onto a warp");

  __shared__ float g_acc[NG][D];
  __shared__ float g_m[NG], g_l[NG];
  __shared__ int last_flag;

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR, li = lane % LPR;
  const int grp = warp * RPW + sub;

  const int item = blockIdx.x;
  const int b = item / p.items_per_b;
  const int r = item - b * p.items_per_b;
  const int Hkv = p.Hq / G;
  int lo = 0, hi = Hkv - 1;           // group g: last g with split_pre[g] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.split_pre[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int s = r - p.split_pre[g];
  const int nsplit = p.split_pre[g + 1] - p.split_pre[g];
  const int C = p.cap[g];
  const bool fused = p.k_new != nullptr;
  const int64_t t0 = p.t[b];
  if (fused) step_counted(p, b, t0);
  const int64_t tb = fused ? t0 + 1 : t0;              // tokens attended
  const int W = (int)(tb < (int64_t)C ? tb : (int64_t)C);   // the group's longest window
  const int w0 = s * kGroupChunk;
  const int nrows = max(0, min(kGroupChunk, W - w0));
  const int64_t pos0 = tb - W + w0;
  const int slot0 = nrows > 0 ? (int)(pos0 % C) : 0;

  T* Kb = reinterpret_cast<T*>(p.data) + (size_t)((int64_t)b * p.sumC + p.goff[g]) * 2 * D;
  T* Vb = Kb + (size_t)C * D;
  // fused append: the newest window entry comes from the step's k, v, which
  // this CTA (the group's only reader of that entry) writes to its slot
  const int e_new = fused ? W - 1 : -1;
  const T* kn = fused ? reinterpret_cast<const T*>(p.k_new) + ((size_t)b * Hkv + g) * D : nullptr;
  const T* vn = fused ? reinterpret_cast<const T*>(p.v_new) + ((size_t)b * Hkv + g) * D : nullptr;

  // head j of the group sees window entries e >= e0[j] (e counts from the
  // oldest entry of the group's window).  q is held as f32 pairs.
  using sm100::f2_pack;
  using sm100::f2_unpack;
  using sm100::f2_fma;
  using sm100::f2_add;
  uint64_t q2[G][VE / 2];
  int e0[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const int h = g * G + j;
    const int Sh = (int)(tb < (int64_t)p.span[h] ? tb : (int64_t)p.span[h]);
    e0[j] = W - Sh;
    const int4 raw = __ldg(reinterpret_cast<const int4*>(
        reinterpret_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * D + li * VE));
    float qf[VE];
    Vec16<T>::cvt(raw, qf);
#pragma unroll
    for (int e = 0; e < VE / 2; ++e) q2[j][e] = f2_pack(qf[2 * e] * p.scale_log2, qf[2 * e + 1] * p.scale_log2);
  }
  // After the transposing reduction below, lane li of a row group holds the
  // full score of head hj = li >> kShift (LPR / G lanes per head).
  constexpr int kLogG = G == 8 ? 3 : G == 4 ? 2 : G == 2 ? 1 : 0;
  static_assert((1 << kLogG) == G && G <= LPR, "group size");
  constexpr int kLogL = LPR == 32 ? 5 : LPR == 16 ? 4 : LPR == 8 ? 3 : LPR == 4 ? 2 : LPR == 2 ? 1 : 0;
  static_assert((1 << kLogL) == LPR, "lanes per row");
  constexpr int kShift = kLogL - kLogG;
  const int hj = li >> kShift;
  const int e0_own = [&] {
    int v = 0;
#pragma unroll
    for (int j = 0; j < G; ++j) if (j == hj) v = e0[j];
    return v;
  }();
  const int lane0 = sub * LPR;                          // first lane of this row group

  // running max and sum of head hj (this lane's), accumulators of every head
  float m_own = -INFINITY, l_own = 0.f;
  uint64_t acc2[G][VE / 2];
#pragma unroll
  for (int j = 0; j < G; ++j)
#pragma unroll
    for (int e = 0; e < VE / 2; ++e) acc2[j][e] = 0;

  // The trip count is uniform across the CTA (every lane takes part in the
  // shuffles below); rows past the chunk are masked instead.
  for (int base = 0; base < nrows; base += NG * U) {
    int4 kr[U], vr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * NG + grp;
      if (row < nrows) {
        int slot = slot0 + row;
        if (slot >= C) slot -= C;
        if (w0 + row == e_new) {
          kr[u] = __ldg(reinterpret_cast<const int4*>(kn + li * VE));
          vr[u] = __ldg(reinterpret_cast<const int4*>(vn + li * VE));
          *reinterpret_cast<int4*>(Kb + (size_t)slot * D + li * VE) = kr[u];
          *reinterpret_cast<int4*>(Vb + (size_t)slot * D + li * VE) = vr[u];
        } else {
          kr[u] = __ldcs(reinterpret_cast<const int4*>(Kb + (size_t)slot * D + li * VE));
          vr[u] = __ldcs(reinterpret_cast<const int4*>(Vb + (size_t)slot * D + li * VE));
        }
      } else {
        kr[u] = make_int4(0, 0, 0, 0);
        vr[u] = make_int4(0, 0, 0, 0);
      }
    }
    // scores: G partial dot products per lane, then a reduction over the row
    // group's lanes that halves the number of values at each of the first
    // kLogG levels, so each lane ends with one head's full sum
    float s_own[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kf[VE];
      Vec16<T>::cvt(kr[u], kf);
      float d[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        uint64_t a2 = 0;
#pragma unroll
        for (int e = 0; e < VE / 2; ++e) a2 = f2_fma(q2[j][e], f2_pack(kf[2 * e], kf[2 * e + 1]), a2);
        float x0, x1;
        f2_unpack(a2, x0, x1);
        d[j] = x0 + x1;
      }
      int n = G;
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) {
        if (n > 1) {
          const bool up = (li & off) != 0;
#pragma unroll
          for (int k = 0; k < n / 2; ++k) {
            const float send = up ? d[k] : d[k + n / 2];
            const float keep = up ? d[k + n / 2] : d[k];
            d[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
          n >>= 1;
        } else {
          d[0] += __shfl_xor_sync(0xffffffffu, d[0], off);
        }
      }
      const int row = base + u * NG + grp;
      s_own[u] = (row < nrows && w0 + row >= e0_own) ? d[0] : -INFINITY;
    }
    // online softmax of head hj over the batch
    float bmax = m_own;
#pragma unroll
    for (int u = 0; u < U; ++u) bmax = fmaxf(bmax, s_own[u]);
    // 0 when the max moves up from -inf, 1 when unchanged (also while still -inf)
    const float corr_own = bmax == m_own ? 1.f : exp2f(m_own - bmax);
    m_own = bmax;
    // a head that has seen no row yet keeps m = -inf: p = 0, not NaN
    const float mref = m_own == -INFINITY ? 0.f : m_own;
    float p_own[U];
    l_own *= corr_own;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      p_own[u] = exp2f(s_own[u] - mref);
      l_own += p_own[u];
    }
    // every lane updates the accumulators of every head: correction factors
    // and weights come from the lanes that own each head
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const float cj = __shfl_sync(0xffffffffu, corr_own, lane0 + (j << kShift));
      const uint64_t c2 = f2_pack(cj, cj);
#pragma unroll
      for (int e = 0; e < VE / 2; ++e) acc2[j][e] = f2_fma(acc2[j][e], c2, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float vf[VE];
      Vec16<T>::cvt(vr[u], vf);
      uint64_t v2[VE / 2];
#pragma unroll
      for (int e = 0; e < VE / 2; ++e) v2[e] = f2_pack(vf[2 * e], vf[2 * e + 1]);
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p_own[u], lane0 + (j << kShift));
        const uint64_t p2 = f2_pack(pj, pj);
#pragma unroll
        for (int e = 0; e < VE / 2; ++e) acc2[j][e] = f2_fma(p2, v2[e], acc2[j][e]);
      }
    }
  }

  // per head: merge the row groups (log-sum-exp) and write the split's partial
#pragma unroll
  for (int j = 0; j < G; ++j) {
#pragma unroll
    for (int e = 0; e < VE / 2; ++e) f2_unpack(acc2[j][e], g_acc[grp][li * VE + 2 * e], g_acc[grp][li * VE + 2 * e + 1]);
    if (li == (j << kShift)) {
      g_m[grp] = m_own;
      g_l[grp] = l_own;
    }
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < NG; ++k) M = fmaxf(M, g_m[k]);
    float L = 0.f, od = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        const float w = exp2f(g_m[k] - M);
        L = fmaf(w, g_l[k], L);
        if (tid < D) od = fmaf(w, g_acc[k][tid], od);
      }
    }
    const int h = g * G + j;
    if (nsplit == 1) {
      if (tid < D)
        Vec16<T>::store(reinterpret_cast<T*>(p.o) + ((size_t)b * p.Hq + h) * D + tid, L > 0.f ? od / L : 0.f);
    } else {
      const size_t idx = (size_t)b * p.hslot_pre[p.Hq] + p.hslot_pre[h] + s;
      if (tid < D) p.part_o[idx * D + tid] = od;
      if (tid == 0) {
        p.part_ml[2 * idx] = M;
        p.part_ml[2 * idx + 1] = L;
      }
    }
    __syncthreads();                                   // g_acc is reused by the next head
  }
  if (nsplit == 1) {
    if (tid == 0 && W == 0) atomicOr(p.err, kErrEmpty);
    return;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(&p.ctr[(size_t)b * p.Hq + g], 1u);
    last_flag = (prev == (unsigned)(nsplit - 1));
  }
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
#pragma unroll 1
  for (int j = 0; j < G; ++j) {
    const int h = g * G + j;
    const size_t first = (size_t)b * p.hslot_pre[p.Hq] + p.hslot_pre[h];
    float MM = -INFINITY;
    for (int ss = 0; ss < nsplit; ++ss) MM = fmaxf(MM, __ldcg(&p.part_ml[2 * (first + ss)]));
    float LL = 0.f, A = 0.f;
    if (MM != -INFINITY) {
      for (int ss = 0; ss < nsplit; ++ss) {
        const float ms = __ldcg(&p.part_ml[2 * (first + ss)]);
        const float w = exp2f(ms - MM);              // 0 for splits outside this head's window
        LL = fmaf(w, __ldcg(&p.part_ml[2 * (first + ss) + 1]), LL);
        if (tid < D) A = fmaf(w, __ldcg(&p.part_o[(first + ss) * D + tid]), A);
      }
    }
    if (tid < D) Vec16<T>::store(reinterpret_cast<T*>(p.o) + ((size_t)b * p.Hq + h) * D + tid, LL > 0.f ? A / LL : 0.f);
  }
  if (tid == 0) {
    p.ctr[(size_t)b * p.Hq + g] = 0u;
    if (W == 0) atomicOr(p.err, kErrEmpty);
  }
}

// ---------------------------------------------------------------------------
// Grouped-query decode on the tensor cores (bf16, d = 128).
//
// Same work item, window geometry and partial layout as decode_group_kernel:
// one CTA per (b, KV group g, split of kGroupChunk group-window entries).  Warp w
// takes entries [128w, 128w + 128) of the split in tiles of 16 cached rows:
//   * cp.async copies the tile's K and V rows (16 x 256 bytes each) into a
//     two-stage per-warp buffer, 16-byte chunks XOR-swizzled by row so that
//     ldmatrix reads them without bank conflicts;
//   * S^T[16 rows x 8 heads] = K_tile . Q_g^T with mma.m16n8k16 (A = K from
//     ldmatrix, B = the group's q held in registers; heads past G are zero);
//   * per head an online softmax over the rows (each lane holds heads
//     2(lane%4), 2(lane%4)+1 for rows lane/4 and lane/4 + 8);
//   * P goes through a 256-byte per-warp scratch into the B-operand layout,
//     and O^T[128 dims x 8 heads] += V_tile^T . P^T (A = V from ldmatrix.trans).
// The four warps then merge by log-sum-exp in shared memory and the split's
// partial (m, l, o) per head is written or, with one split, o itself.
// A tile whose 16 slots are contiguous and inside the split is copied from one
// base pointer at constant offsets; others walk the ring row by row.  Splits
// past a group's window read its global-token rows (each head masks its own
// count).
constexpr int kMmaRows = 16;                      // cached rows per tile
constexpr int kMmaTileBytes = kMmaRows * 128 * 2; // one 16 x 128 bf16 tile
#ifndef MOA_MMA_STAGES
#define MOA_MMA_STAGES 2
#endif
constexpr int kMmaStages = MOA_MMA_STAGES;        // K/V tiles in flight per warp + 1
constexpr uint32_t kMmaWarpBytes = kMmaStages * 2 * kMmaTileBytes + 256;   // stages + P scratch
constexpr int kMmaWarpRows = kGroupChunk / kDecWarps;  // entries per warp and split
constexpr size_t kMmaSmem = (size_t)kDecWarps * kMmaWarpBytes;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// d[0..3] += A[16x16] . B[16x8], bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// byte offset of 16-byte chunk c of row r in a swizzled 16 x 256-byte tile
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4)); }

template <int G>
__global__ void __launch_bounds__(kDecThreads) decode_group_mma_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int D = 128;
  static_assert(G == 2 || G == 4 || G == 8, "group size");
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ int last_flag;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int g4 = lane >> 2, c4 = lane & 3;

  const int item = blockIdx.x;
  const int b = item / p.items_per_b;
  const int r = item - b * p.items_per_b;
  const int Hkv = p.Hq / G;
  int lo = 0, hi = Hkv - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.split_pre[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int s = r - p.split_pre[g];
  const int nsplit = p.split_pre[g + 1] - p.split_pre[g];
  const int C = p.cap[g];
  const bool fused = p.k_new != nullptr;
  const int64_t t0 = p.t[b];
  if (fused) step_counted(p, b, t0);
  const int64_t tb = fused ? t0 + 1 : t0;
  const int W = (int)(tb < (int64_t)C ? tb : (int64_t)C);
  // Splits s >= nwin cover the group's global tokens below its heads' windows:
  // positions 0 .. GW - 1 (the union over the group's heads), rows of the
  // global-token region, which do not wrap.
  const int nwin = splits_of(C, kGroupChunk);
  const bool gsplit = s >= nwin;
  int GW = 0;
  if (gsplit) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const int64_t Sj = tb < (int64_t)p.span[g * G + j] ? tb : (int64_t)p.span[g * G + j];
      GW = max(GW, (int)min((int64_t)p.sink[g * G + j], tb - Sj));
    }
  }
  const int w0 = (gsplit ? s - nwin : s) * kGroupChunk;
  const int nrows = max(0, min(kGroupChunk, (gsplit ? GW : W) - w0));
  const int64_t pos0 = tb - W + w0;
  const int slot0 = gsplit ? w0 : nrows > 0 ? (int)(pos0 % C) : 0;
  const int Cw = gsplit ? (1 << 30) : C;           // global-token rows do not wrap
  const __nv_bfloat16* Kb = reinterpret_cast<const __nv_bfloat16*>(p.data) + (size_t)((int64_t)b * p.sumC + p.goff[g]) * 2 * D;
  const __nv_bfloat16* Vb = Kb + (size_t)C * D;
  if (gsplit) {
    Kb = reinterpret_cast<const __nv_bfloat16*>(p.sink_data) + (size_t)((int64_t)b * p.sumK + p.soff[g]) * 2 * D;
    Vb = Kb + (size_t)p.scap[g] * D;
  }
  const int e_new = fused && !gsplit ? W - 1 : -1;
  // the fused append also keeps the new token's global-token row
  __nv_bfloat16* ks_new = nullptr;
  if (fused && !gsplit && p.sink_data != nullptr && t0 < (int64_t)p.scap[g])
    ks_new = reinterpret_cast<__nv_bfloat16*>(p.sink_data) + (size_t)((int64_t)b * p.sumK + p.soff[g]) * 2 * D +
             (size_t)t0 * D;
  const __nv_bfloat16* kn = fused ? reinterpret_cast<const __nv_bfloat16*>(p.k_new) + ((size_t)b * Hkv + g) * D : nullptr;
  const __nv_bfloat16* vn = fused ? reinterpret_cast<const __nv_bfloat16*>(p.v_new) + ((size_t)b * Hkv + g) * D : nullptr;

  // B operand of S^T: q of head n = lane/4 (zero past G), dims 16kk + 2(lane%4) + {0,1} and + {8,9}
  uint32_t qb[8][2];
  {
    const bool hv = g4 < G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + g * G + (hv ? g4 : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qb[kk][0] = hv ? __ldg(qrow + 8 * kk + c4) : 0u;
      qb[kk][1] = hv ? __ldg(qrow + 8 * kk + c4 + 4) : 0u;
    }
  }
  // heads this lane owns in the accumulator layouts, and the entries [e0, e1)
  // of this split's range each head sees (window splits: from where its window
  // starts; global splits: below the end of its global tokens)
  const int h0 = 2 * c4, h1 = 2 * c4 + 1;
  int e0a = 1 << 30, e0b = 1 << 30;              // past every entry: heads beyond G see no row
  int e1a = 1 << 30, e1b = 1 << 30;
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const int Sh = (int)(tb < (int64_t)p.span[g * G + j] ? tb : (int64_t)p.span[g * G + j]);
    const int lo_j = gsplit ? 0 : W - Sh;
    const int hi_j = gsplit ? (int)min((int64_t)p.sink[g * G + j], tb - Sh) : (1 << 30);
    if (j == h0) { e0a = lo_j; e1a = hi_j; }
    if (j == h1) { e0b = lo_j; e1b = hi_j; }
  }

  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(dsm) + (uint32_t)warp * kMmaWarpBytes;
  const uint32_t sP = sbase + kMmaStages * 2 * kMmaTileBytes;    // [8 heads][16 rows] bf16
  uint16_t* sPg = reinterpret_cast<uint16_t*>(dsm + (size_t)warp * kMmaWarpBytes + kMmaStages * 2 * kMmaTileBytes);
  const int wrow0 = warp * kMmaWarpRows;                          // first split entry of this warp
  const int wrows = max(0, min(kMmaWarpRows, nrows - wrow0));
  const int ntiles = (wrows + kMmaRows - 1) / kMmaRows;

  // issue the copies of tile ti into stage st (rows past the split are zero-filled)
  // Lane `lane` copies chunk cc = lane & 15 of tile rows rr0 + 2q, q = 0..7
  // (rr0 = lane >> 4): its slot advances by 2 per row with one wrap test, and
  // its swizzled destinations repeat every four rows (row residues mod 8 are
  // rr0 + 2(q & 3)), so they are computed once.
  const int cc = lane & 15, rr0 = lane >> 4;
  uint32_t soff[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) soff[u] = swz(rr0 + 2 * u, cc);
  const size_t vofs = (size_t)(Vb - Kb);                       // V block after the K block
  auto load_tile = [&](int ti, int st) {
    const uint32_t dK = sbase + (uint32_t)st * 2 * kMmaTileBytes, dV = dK + kMmaTileBytes;
    const int trow = wrow0 + ti * kMmaRows;                      // the tile's first split entry
    int tslot = slot0 + trow;
    if (tslot >= Cw) tslot -= Cw;
    // Common case: all 16 rows inside the split, their slots contiguous (no
    // wrap), none the fused append's new entry: one base pointer per lane and
    // constant offsets (two rows, 512 bytes, apart per copy).
    if (trow + kMmaRows <= nrows && tslot + kMmaRows <= Cw &&
        !(e_new >= w0 + trow && e_new < w0 + trow + kMmaRows)) {
      const __nv_bfloat16* pk = Kb + (size_t)(tslot + rr0) * D + cc * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t off = (uint32_t)(q >> 2) * 2048u + soff[q & 3];
        cp_async16(dK + off, pk + (size_t)q * 2 * D, 16u);
        cp_async16(dV + off, pk + vofs + (size_t)q * 2 * D, 16u);
      }
      return;
    }
    int row = trow + rr0;                                        // split entry of q = 0
    int slot = slot0 + row;
    if (slot >= Cw) slot -= Cw;                                  // exact while row < nrows <= C
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const bool ok = row < nrows;
      const __nv_bfloat16* srcK = ok ? Kb + (size_t)slot * D + cc * 8 : Kb;
      const __nv_bfloat16* srcV = ok ? Vb + (size_t)slot * D + cc * 8 : Vb;
      if (ok && w0 + row == e_new) {
        // this CTA is the group's only reader of the newest entry: write it to its slot
        const int4 kx = __ldg(reinterpret_cast<const int4*>(kn + cc * 8));
        const int4 vx = __ldg(reinterpret_cast<const int4*>(vn + cc * 8));
        *reinterpret_cast<int4*>(const_cast<__nv_bfloat16*>(srcK)) = kx;
        *reinterpret_cast<int4*>(const_cast<__nv_bfloat16*>(srcV)) = vx;
        if (ks_new != nullptr) {
          *reinterpret_cast<int4*>(ks_new + cc * 8) = kx;
          *reinterpret_cast<int4*>(ks_new + (size_t)p.scap[g] * D + cc * 8) = vx;
        }
        srcK = kn + cc * 8;
        srcV = vn + cc * 8;
      }
      const uint32_t off = (uint32_t)(q >> 2) * 2048u + soff[q & 3];
      cp_async16(dK + off, srcK, ok ? 16u : 0u);
      cp_async16(dV + off, srcV, ok ? 16u : 0u);
      row += 2;
      slot += 2;
      if (slot >= Cw) slot -= Cw;
    }
  };

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads h0, h1
  float oacc[8][4];
#pragma unroll
  for (int mb = 0; mb < 8; ++mb)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[mb][e] = 0.f;

  // prologue: the first kMmaStages - 1 tiles in flight (one commit group each)
#pragma unroll
  for (int k = 0; k < kMmaStages - 1; ++k) {
    if (k < ntiles) load_tile(k, k);
    cp_async_commit();
  }
  for (int ti = 0; ti < ntiles; ++ti) {
    const int nx = ti + kMmaStages - 1;
    if (nx < ntiles) load_tile(nx, nx % kMmaStages);
    cp_async_commit();
    cp_async_wait<kMmaStages - 1>();                    // tile ti has landed
    __syncwarp();
    const uint32_t tK = sbase + (uint32_t)(ti % kMmaStages) * 2 * kMmaTileBytes, tV = tK + kMmaTileBytes;
    // S^T = K . Q^T
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int ar = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t a[4];
        ldsm_x4(tK + swz(ar, 2 * kk + (lane >> 4)), a);
        mma16816(sacc, a, qb[kk][0], qb[kk][1]);
      }
    }
    // mask and scale: rows g4 and g4 + 8 of the tile, heads h0 and h1
    const int ra = wrow0 + ti * kMmaRows + g4, rb = ra + 8;
    const float sc = p.scale_log2;
    const float s0 = (ra < nrows && w0 + ra >= e0a && w0 + ra < e1a) ? sacc[0] * sc : -INFINITY;
    const float s1 = (ra < nrows && w0 + ra >= e0b && w0 + ra < e1b) ? sacc[1] * sc : -INFINITY;
    const float s2 = (rb < nrows && w0 + rb >= e0a && w0 + rb < e1a) ? sacc[2] * sc : -INFINITY;
    const float s3 = (rb < nrows && w0 + rb >= e0b && w0 + rb < e1b) ? sacc[3] * sc : -INFINITY;
    float t0m = fmaxf(s0, s2), t1m = fmaxf(s1, s3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      t0m = fmaxf(t0m, __shfl_xor_sync(0xffffffffu, t0m, off));
      t1m = fmaxf(t1m, __shfl_xor_sync(0xffffffffu, t1m, off));
    }
    const float n0 = fmaxf(m0, t0m), n1 = fmaxf(m1, t1m);
    const float cr0 = n0 == m0 ? 1.f : exp2f(m0 - n0);        // 0 when m was -inf
    const float cr1 = n1 == m1 ? 1.f : exp2f(m1 - n1);
    m0 = n0;
    m1 = n1;
    const float r0 = m0 == -INFINITY ? 0.f : m0, r1 = m1 == -INFINITY ? 0.f : m1;
    const float p0 = exp2f(s0 - r0), p1 = exp2f(s1 - r1), p2 = exp2f(s2 - r0), p3 = exp2f(s3 - r1);
    l0 = l0 * cr0 + p0 + p2;
    l1 = l1 * cr1 + p1 + p3;
#pragma unroll
    for (int mb = 0; mb < 8; ++mb) {
      oacc[mb][0] *= cr0;
      oacc[mb][1] *= cr1;
      oacc[mb][2] *= cr0;
      oacc[mb][3] *= cr1;
    }
    // P^T into the B-operand layout through the scratch [head][row]
    sPg[h0 * 16 + g4] = __bfloat16_as_ushort(__float2bfloat16_rn(p0));
    sPg[h1 * 16 + g4] = __bfloat16_as_ushort(__float2bfloat16_rn(p1));
    sPg[h0 * 16 + g4 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(p2));
    sPg[h1 * 16 + g4 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(p3));
    __syncwarp();
    uint32_t pb0, pb1;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(pb0) : "r"(sP + (uint32_t)(g4 * 32 + c4 * 4)));
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(pb1) : "r"(sP + (uint32_t)(g4 * 32 + c4 * 4 + 16)));
    // O^T += V^T . P^T
    {
      const int vr = (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
      for (int mb = 0; mb < 8; ++mb) {
        uint32_t a[4];
        ldsm_x4_t(tV + swz(vr, 2 * mb + ((lane >> 3) & 1)), a);
        mma16816(oacc[mb], a, pb0, pb1);
      }
    }
    __syncwarp();                                       // stage and scratch are rewritten next
  }
  cp_async_wait<0>();
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }

  // merge the four warps: per warp m, l [8 heads] and o [8 heads][128] in fp32
  __syncthreads();
  float* mw = reinterpret_cast<float*>(dsm);                  // [4][8]
  float* lw = mw + kDecWarps * 8;                             // [4][8]
  float* ow = lw + kDecWarps * 8;                             // [4][8][128]
  if (g4 == 0) {
    mw[warp * 8 + h0] = m0;
    mw[warp * 8 + h1] = m1;
    lw[warp * 8 + h0] = l0;
    lw[warp * 8 + h1] = l1;
  }
#pragma unroll
  for (int mb = 0; mb < 8; ++mb) {
    float* o = ow + warp * 8 * D;
    o[h0 * D + 16 * mb + g4] = oacc[mb][0];
    o[h1 * D + 16 * mb + g4] = oacc[mb][1];
    o[h0 * D + 16 * mb + g4 + 8] = oacc[mb][2];
    o[h1 * D + 16 * mb + g4 + 8] = oacc[mb][3];
  }
  __syncthreads();
#pragma unroll 1
  for (int j = 0; j < G; ++j) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, mw[w * 8 + j]);
    float L = 0.f, od = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float wt = exp2f(mw[w * 8 + j] - M);
        L = fmaf(wt, lw[w * 8 + j], L);
        od = fmaf(wt, ow[(w * 8 + j) * D + tid], od);
      }
    }
    const int h = g * G + j;
    if (nsplit == 1) {
      reinterpret_cast<__nv_bfloat16*>(p.o)[((size_t)b * p.Hq + h) * D + tid] = __float2bfloat16_rn(L > 0.f ? od / L : 0.f);
    } else {
      const size_t idx = (size_t)b * p.hslot_pre[p.Hq] + p.hslot_pre[h] + s;
      p.part_o[idx * D + tid] = od;
      if (tid == 0) {
        p.part_ml[2 * idx] = M;
        p.part_ml[2 * idx + 1] = L;
      }
    }
  }
  if (nsplit == 1) {
    if (tid == 0 && W == 0) atomicOr(p.err, kErrEmpty);
    return;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(&p.ctr[(size_t)b * p.Hq + g], 1u);
    last_flag = (prev == (unsigned)(nsplit - 1));
  }
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
#pragma unroll 1
  for (int j = 0; j < G; ++j) {
    const int h = g * G + j;
    const size_t first = (size_t)b * p.hslot_pre[p.Hq] + p.hslot_pre[h];
    float MM = -INFINITY;
    for (int ss = 0; ss < nsplit; ++ss) MM = fmaxf(MM, __ldcg(&p.part_ml[2 * (first + ss)]));
    float LL = 0.f, A = 0.f;
    if (MM != -INFINITY) {
      for (int ss = 0; ss < nsplit; ++ss) {
        const float ms = __ldcg(&p.part_ml[2 * (first + ss)]);
        const float wt = exp2f(ms - MM);
        LL = fmaf(wt, __ldcg(&p.part_ml[2 * (first + ss) + 1]), LL);
        A = fmaf(wt, __ldcg(&p.part_o[(first + ss) * D + tid]), A);
      }
    }
    reinterpret_cast<__nv_bfloat16*>(p.o)[((size_t)b * p.Hq + h) * D + tid] = __float2bfloat16_rn(LL > 0.f ? A / LL : 0.f);
  }
  if (tid == 0) {
    p.ctr[(size_t)b * p.Hq + g] = 0u;
    if (W == 0) atomicOr(p.err, kErrEmpty);
  }
}

template <int G>
cudaError_t launch_group_mma(const DecodeParams& p, unsigned grid, cudaStream_t s) {
  static unsigned long long attr_done = 0;
  const cudaError_t attr =
      ensure_smem_attr(reinterpret_cast<const void*>(decode_group_mma_kernel<G>), (int)kMmaSmem, &attr_done);
  if (attr != cudaSuccess) return attr;
  decode_group_mma_kernel<G><<<grid, kDecThreads, kMmaSmem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int D, int G>
cudaError_t launch_group(const DecodeParams& p, unsigned grid, cudaStream_t s) {
  decode_group_kernel<T, D, G><<<grid, kDecThreads, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_group_g(const DecodeParams& p, int G, unsigned grid, cudaStream_t s) {
  return G == 4 ? launch_group<T, D, 4>(p, grid, s) : launch_group<T, D, 8>(p, grid, s);
}

template <typename T, int D>
cudaError_t launch_one(const DecodeParams& p, int chunk, unsigned grid, cudaStream_t s) {
  if (chunk == kChunk)
    decode_kernel<T, D, kChunk><<<grid, kDecThreads, 0, s>>>(p);
  else
    decode_kernel<T, D, kMinChunk><<<grid, kDecThreads, 0, s>>>(p);
  return cudaGetLastError();
}

struct DecodeLayout {
  int chunk;                         // per-head split size
  int items_per_b;
  size_t ctr_off, bctr_off, ml_off, o_off, total;
};

// Per-head splits of one sequence at split size c (window, then global tokens).
long long head_items(int32_t Hq, const int32_t* spans, const int32_t* sinks, int c) {
  long long items = 0;
  for (int h = 0; h < Hq; ++h) items += splits_of(spans[h], c) + (sinks ? splits_of(sinks[h], c) : 0);
  return items;
}

// The per-head split size of a launch: kChunk, or kMinChunk when the launch
// would have fewer than kHeadItems splits.  A function of the shapes alone,
// so the workspace size and the launch agree.
int head_chunk(int32_t B, int32_t Hq, const int32_t* spans, const int32_t* sinks) {
  return (long long)B * head_items(Hq, spans, sinks, kChunk) < kHeadItems ? kMinChunk : kChunk;
}

// Partial slots per sequence: the per-head kernel uses sum_h ceil(S_h / chunk),
// the group kernel sum_h ceil(C_g(h) / chunk); both are at most
// Hq * ceil(max_h S_h / chunk), which sizes the workspace without knowing the
// number of KV heads.
DecodeLayout decode_layout(int32_t B, int32_t Hq, int32_t d, const int32_t* spans, const int32_t* sinks) {
  DecodeLayout L;
  L.chunk = head_chunk(B, Hq, spans, sinks);
  int max_s = 0, max_k = 0;
  for (int h = 0; h < Hq; ++h) {
    max_s = max_s > spans[h] ? max_s : spans[h];
    if (sinks) max_k = max_k > sinks[h] ? max_k : sinks[h];
  }
  L.items_per_b = (int)head_items(Hq, spans, sinks, L.chunk);
  // The group kernels split more coarsely (kGroupChunk >= chunk), so these
  // slots hold their partials too.
  const size_t slots = (size_t)Hq * ((size_t)splits_of(max_s, L.chunk) + (size_t)splits_of(max_k, L.chunk));
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  L.ctr_off = 256;
  L.bctr_off = L.ctr_off + up((size_t)B * Hq * 4);
  L.ml_off = L.bctr_off + up((size_t)B * 4);
  L.o_off = L.ml_off + up((size_t)B * slots * 2 * 4);
  L.total = L.o_off + up((size_t)B * slots * d * 4);
  return L;
}

}  // namespace

size_t decode_workspace_bytes(int32_t B, int32_t Hq, int32_t d, const int32_t* spans, const int32_t* sinks) {
  return decode_layout(B, Hq, d, spans, sinks).total;
}

moa_status launch_decode(moa_kv_cache* c, const void* q, void* o, int32_t Hq, const int32_t* spans,
                         float scale, void* ws, size_t ws_bytes, cudaStream_t s, const void* k_new,
                         const void* v_new, const int32_t* sinks) {
  const DecodeLayout L = decode_layout(c->B, Hq, c->d, spans, sinks);
  if (ws_bytes < L.total) return MOA_ERR_WORKSPACE;
  DecodeParams p;
  p.data = c->buf + c->header;
  p.t = reinterpret_cast<int64_t*>(c->buf + kHdrT);
  p.k_new = k_new;
  p.v_new = v_new;
  p.err = reinterpret_cast<uint32_t*>(c->buf + kHdrErr);
  p.q = q;
  p.o = o;
  char* w = (char*)ws;
  p.ctr = reinterpret_cast<uint32_t*>(w + L.ctr_off);
  p.bctr = reinterpret_cast<uint32_t*>(w + L.bctr_off);
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
    p.sink[h] = sinks ? sinks[h] : 0;
    p.split_pre[h + 1] = p.split_pre[h] + splits_of(spans[h], L.chunk) + splits_of(p.sink[h], L.chunk);
  }
  for (int g = 0; g < c->Hkv; ++g) {
    p.cap[g] = c->cap[g];
    p.goff[g] = c->goff[g];
    p.scap[g] = c->scap[g];
    p.soff[g] = c->soff[g];
  }
  // the cache's global-token rows are written by every fused append, also
  // when this call attends to none of them
  p.sink_data = sink_region(c);
  p.sumK = c->soff[c->Hkv];
  // The group kernels read each cached row once for all G heads; the
  // per-head kernel reads overlapping windows once per head and L2 serves
  // most of the repeats.  bf16 with d = 128 and G = 2, 4 or 8 always takes
  // the tensor-core group kernel: on Llama3-8B-shaped layers (B=32, context
  // 8192) it beat the per-head kernel at every overlap tried, down to heads'
  // windows summing to 1.8x the group windows.  The SIMT group kernel (other
  // types and sizes) does G dot products per row on the CUDA cores: it was
  // 5 % faster than the per-head kernel at 2.24x and 8 % slower at 2.0x, so
  // it is taken above 2.2x.
  const int G = Hq / c->Hkv;
  int64_t head_rows = 0, group_rows = 0;
  for (int h = 0; h < Hq; ++h) head_rows += spans[h];
  for (int g = 0; g < c->Hkv; ++g) group_rows += c->cap[g];
  // The tensor-core group kernel also serves global tokens (splits over the
  // group's global-token rows) and keeps the rows of caches that hold them.
  // The SIMT group kernel does neither: such calls take the per-head kernel.
  const bool plain = p.sink_data == nullptr;
  const bool mma_group = kGroupMma && c->dtype == MOA_BF16 && c->d == 128 &&
                         (G == 4 || G == 8 || (kGroupMma2 && G == 2));
  if (mma_group || (plain && (G == 4 || G == 8) && head_rows * 10 > group_rows * 22)) {
    // group kernel: splits per KV group over its capacity (then over its
    // heads' largest global-token count), G partial slots each.  Its split
    // size stays kGroupChunk at every batch: smaller group splits measured
    // slower even at batch 1 (0.038 against 0.021 ms on a Llama3-8B-shaped
    // layer), as each warp then gets only a tile or two and the last split
    // merges many more partials.
    int items = 0;
    p.split_pre[0] = 0;
    p.hslot_pre[0] = 0;
    for (int g = 0; g < c->Hkv; ++g) {
      int kmax = 0;
      for (int j = 0; j < G; ++j) kmax = max(kmax, p.sink[g * G + j]);
      const int ns = splits_of(c->cap[g], kGroupChunk) + splits_of(kmax, kGroupChunk);
      p.split_pre[g + 1] = p.split_pre[g] + ns;
      for (int j = 0; j < G; ++j) p.hslot_pre[g * G + j + 1] = p.hslot_pre[g * G + j] + ns;
      items += ns;
    }
    p.items_per_b = items;
    const long long grid = (long long)c->B * items;
    if (grid > 0x7fffffffLL) return MOA_ERR_UNSUPPORTED;
    cudaError_t e;
    if (mma_group)
      e = G == 2 ? launch_group_mma<2>(p, (unsigned)grid, s)
                 : G == 4 ? launch_group_mma<4>(p, (unsigned)grid, s) : launch_group_mma<8>(p, (unsigned)grid, s);
    else if (c->dtype == MOA_BF16)
      e = c->d == 128 ? launch_group_g<__nv_bfloat16, 128>(p, G, (unsigned)grid, s)
                      : launch_group_g<__nv_bfloat16, 64>(p, G, (unsigned)grid, s);
    else
      e = c->d == 128 ? launch_group_g<float, 128>(p, G, (unsigned)grid, s)
                      : launch_group_g<float, 64>(p, G, (unsigned)grid, s);
    return e == cudaSuccess ? MOA_OK : cuda_fail(e, "decode launch");
  }
  const long long grid = (long long)c->B * L.items_per_b;
  if (grid > 0x7fffffffLL) return MOA_ERR_UNSUPPORTED;
  cudaError_t e;
  if (c->dtype == MOA_BF16)
    e = c->d == 128 ? launch_one<__nv_bfloat16, 128>(p, L.chunk, (unsigned)grid, s)
                    : launch_one<__nv_bfloat16, 64>(p, L.chunk, (unsigned)grid, s);
  else
    e = c->d == 128 ? launch_one<float, 128>(p, L.chunk, (unsigned)grid, s)
                    : launch_one<float, 64>(p, L.chunk, (unsigned)grid, s);
  return e == cudaSuccess ? MOA_OK : cuda_fail(e, "decode launch");
}

}  // namespace moa
