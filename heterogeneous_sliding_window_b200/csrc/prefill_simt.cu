// fp32 prefill for heterogeneous sliding windows (SIMT, fp32 throughout).
//
// "Mixture of Attention" project page, "Finding two" and its N x N causal
// figure: query row i of head h sees keys j with i - S_h < j <= i, and, for a
// head with global tokens, also the keys j < sink[h] (j <= i).  This path
// keeps every operation in fp32 (no tensor cores, no TF32) for the small
// fp32 configuration; one warp owns one query row and walks its window with
// an online softmax: lanes split the head dimension, a dot product is reduced
// with xor-shuffles, and the running (max, sum, accumulator) are rescaled as
// the max grows.
#include "internal.h"

namespace moa {
namespace {

constexpr int kRowsPerBlock = 4;

struct SimtParams {
  const float* q;
  const float* k;
  const float* v;
  float* o;
  int32_t Hq, Hkv, G, N;
  float scale_log2;
  int32_t span[MOA_MAX_HEADS];
  int32_t sink[MOA_MAX_HEADS];   // global tokens per head: keys j < sink[h] are kept too
};

template <int D>
__global__ void __launch_bounds__(32 * kRowsPerBlock) prefill_f32_kernel(const __grid_constant__ SimtParams p) {
  constexpr int E = D / 32;                      // head-dim elements per lane
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  if (i >= p.N) return;                          // whole warp leaves together
  const int h = blockIdx.y, b = blockIdx.z, g = h / p.G;
  const int S = p.span[h];
  const int lo = max(0, i - S + 1);
  const int gs = min(p.sink[h], lo);             // global tokens below the band: keys [0, gs)
  const float* qr = p.q + (((size_t)b * p.Hq + h) * p.N + i) * D;
  const float* kb = p.k + ((size_t)b * p.Hkv + g) * (size_t)p.N * D;
  const float* vb = p.v + ((size_t)b * p.Hkv + g) * (size_t)p.N * D;
  float qv[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = qr[lane + 32 * e] * p.scale_log2;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = gs > 0 ? 0 : lo; j <= i; j = j + 1 == gs ? lo : j + 1) {
    const float* kr = kb + (size_t)j * D;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) s = fmaf(qv[e], kr[lane + 32 * e], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(m, s);
    const float corr = exp2f(m - mn);            // 0 on the first key (m = -inf)
    const float pj = exp2f(s - mn);
    l = l * corr + pj;
    const float* vr = vb + (size_t)j * D;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(pj, vr[lane + 32 * e], acc[e] * corr);
    m = mn;
  }
  float* orow = p.o + (((size_t)b * p.Hq + h) * p.N + i) * D;
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < E; ++e) orow[lane + 32 * e] = acc[e] * inv;
}

}  // namespace

moa_status launch_prefill_f32(const float* q, const float* k, const float* v, float* o, int32_t B,
                              int32_t Hq, int32_t Hkv, int32_t N, int32_t d, const int32_t* spans,
                              float scale, cudaStream_t s, const int32_t* sinks) {
  SimtParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.N = N;
  p.scale_log2 = scale * 1.4426950408889634f;
  for (int h = 0; h < Hq; ++h) {
    p.span[h] = spans[h];
    p.sink[h] = sinks ? sinks[h] : 0;
  }
  if (B > 65535) return MOA_ERR_UNSUPPORTED;
  dim3 grid((N + kRowsPerBlock - 1) / kRowsPerBlock, Hq, B);
  if (d == 128) prefill_f32_kernel<128><<<grid, 32 * kRowsPerBlock, 0, s>>>(p);
  else prefill_f32_kernel<64><<<grid, 32 * kRowsPerBlock, 0, s>>>(p);
  return check_launch("prefill_f32 launch");
}

}  // namespace moa
