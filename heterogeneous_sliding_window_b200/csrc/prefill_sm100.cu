// bf16 prefill for heterogeneous sliding windows on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes ("Mixture of Attention" project page, "Finding two" and
// the N x N causal-band figure; blog walkthrough section 2.1): for query row
// i of head h, softmax(scale * q_i . k_j) over the keys i - S_h < j <= i,
// applied to v_j.  Heads differ only in S_h.
//
// How (B200 design, not the pages' A100 kernel):
//  * Work unit = (b, h, m): query rows [128m, 128m+127] of one head.  Because
//    the window is a band, the unit needs exactly the key tiles lo..m with
//    lo = floor(max(0, 128m - S_h + 1) / 128); every other tile is skipped.
//  * Units are sorted longest-first on the host and taken by a persistent
//    grid (one CTA per SM) through an atomic counter, so heads with very
//    different spans still balance across the 148 SMs.
//  * Per unit: TMA brings Q (once) and K/V tiles (double-buffered, separate
//    K and V rings) into 128-byte-swizzled shared memory.  One thread issues
//    tcgen05.mma (M=128, N=128, K=16 steps) for S = Q K^T into tensor memory;
//    128 threads (one per query row) read S from TMEM, mask only where the
//    tile crosses the diagonal or the window's lower edge, run the online
//    softmax in the exp2 domain with a lazy rescale (the running max used for
//    the exponentials only moves when it would grow by more than 2^8), write
//    P as bf16 into swizzled shared memory, and the MMA thread accumulates
//    O += P V into tensor memory (V read MN-major straight from its TMA tile).
//    S of the next tile is issued as soon as the current S has been read, so
//    the tensor core overlaps the exponentials.
//  * Epilogue: O / l in fp32 -> bf16 (round to nearest even), staged through
//    shared memory and stored with coalesced 16-byte writes; rows >= N are
//    dropped, out-of-range TMA rows read as zeros.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace moa {
namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr int kD = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;   // one 128 x 128 bf16 tile
constexpr uint32_t kHalfBytes = 128 * 64 * 2;    // one 128-row x 128-byte swizzled half
// Shared memory carve-up (offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_P = OFF_Q + kTileBytes;
constexpr uint32_t OFF_K = OFF_P + kTileBytes;        // 2 stages
constexpr uint32_t OFF_V = OFF_K + 2 * kTileBytes;    // 2 stages
constexpr uint32_t OFF_BAR = OFF_V + 2 * kTileBytes;
constexpr uint32_t kStageRowBytes = 272;              // epilogue staging row (256 + 16 pad)
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024; // + barriers + alignment slack
static_assert(128 * kStageRowBytes <= OFF_K, "epilogue staging must fit in Q and P");

constexpr uint32_t kTmemCols = 256;                   // S: [0,128), O: [128,256)
constexpr uint32_t kColS = 0, kColO = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;        // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;             // log2 of the largest tolerated growth

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);

struct PrefillParams {
  uint32_t* hdr;                 // [0] error word, [1] unit counter
  const int4* units;             // (b, h, m, lo), longest first
  void* o;
  int32_t n_units, N, Hq, Hkv, G;
  float scale_log2;
  int32_t span[MOA_MAX_HEADS];
};

struct Bars {                    // mbarrier addresses (shared::cta)
  uint32_t q, k[2], v[2], s, o;
};

// K-major operand (Q, K or P) of one 16-wide K step kk (0..7): the 128-wide
// K extent is stored as two 64-column swizzled halves of 16 KB.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int kk) {
  return smem_desc_sw128(base + (uint32_t)(kk >> 2) * kHalfBytes + (uint32_t)(kk & 3) * 32u, 16u,
                         1024u);
}
// MN-major V operand of K step kk (keys 16kk..16kk+15): 8-key groups are
// 1024 B apart (SBO), the two 64-wide head-dim halves 16 KB apart (LBO).
__device__ __forceinline__ uint64_t desc_v(uint32_t base, int kk) {
  return smem_desc_sw128(base + (uint32_t)kk * 2048u, kHalfBytes, 1024u);
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bar_mem = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 64);
  volatile int* s_unit = reinterpret_cast<volatile int*>(smem + OFF_BAR + 68);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  Bars bars;
  bars.q = smem_addr(bar_mem + 0);
  bars.k[0] = smem_addr(bar_mem + 1);
  bars.k[1] = smem_addr(bar_mem + 2);
  bars.v[0] = smem_addr(bar_mem + 3);
  bars.v[1] = smem_addr(bar_mem + 4);
  bars.s = smem_addr(bar_mem + 5);
  bars.o = smem_addr(bar_mem + 6);

  if (tid == 0) {
    for (int i = 0; i < 7; ++i) mbar_init(smem_addr(bar_mem + i), 1);
    mbar_fence_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 0) tmem_alloc(smem_addr((const void*)tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;   // this warp's TMEM lane quarter
  const uint32_t tS = tmem + lane_base + kColS;
  const uint32_t tO = tmem + lane_base + kColO;

  const uint32_t sQ = sbase + OFF_Q, sP = sbase + OFF_P;
  const uint32_t sK[2] = {sbase + OFF_K, sbase + OFF_K + kTileBytes};
  const uint32_t sV[2] = {sbase + OFF_V, sbase + OFF_V + kTileBytes};

  // Thread 0's bookkeeping of issued / consumed barrier phases (for the
  // parities and for draining after a timeout).
  uint32_t ik[2] = {0, 0}, wk[2] = {0, 0}, iv[2] = {0, 0}, wv[2] = {0, 0};
  uint32_t iq = 0, wq = 0, is_ = 0, io = 0;
  uint32_t gt = 0;                // tiles processed by this CTA (bar_s / bar_o parity)
  bool ok = true;                 // this thread's waits all succeeded
  bool aborted = false;           // block-uniform: some thread's wait gave up

  auto fail = [&]() {
    ok = false;
    atomicOr(p.hdr, kErrTimeout);
  };

  for (;;) {
    if (tid == 0) *s_unit = (int)atomicAdd(p.hdr + 1, 1u);
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    const int u = *s_unit;
    if (u >= p.n_units) break;
    const int4 U = p.units[u];
    const int b = U.x, h = U.y, m = U.z, lo = U.w;
    const int nt = m - lo + 1;
    const int S = p.span[h];
    const int zq = b * p.Hq + h;
    const int zk = b * p.Hkv + h / p.G;

    if (tid == 0) {
      mbar_expect_tx(bars.q, kTileBytes);
      tma_load_3d(sQ, &tmQ, bars.q, 0, m * 128, zq);
      tma_load_3d(sQ + kHalfBytes, &tmQ, bars.q, 64, m * 128, zq);
      ++iq;
      for (int i = 0; i < 2 && i < nt; ++i) {
        const int st = (gt + i) & 1;
        mbar_expect_tx(bars.k[st], kTileBytes);
        tma_load_3d(sK[st], &tmK, bars.k[st], 0, (lo + i) * 128, zk);
        tma_load_3d(sK[st] + kHalfBytes, &tmK, bars.k[st], 64, (lo + i) * 128, zk);
        ++ik[st];
        mbar_expect_tx(bars.v[st], kTileBytes);
        tma_load_3d(sV[st], &tmV, bars.v[st], 0, (lo + i) * 128, zk);
        tma_load_3d(sV[st] + kHalfBytes, &tmV, bars.v[st], 64, (lo + i) * 128, zk);
        ++iv[st];
      }
      const int st0 = gt & 1;
      if (mbar_wait(bars.q, wq & 1, kTimeoutNs)) ++wq; else fail();
      if (ok) { if (mbar_wait(bars.k[st0], wk[st0] & 1, kTimeoutNs)) ++wk[st0]; else fail(); }
      if (ok) {
        tc_fence_after();
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tS - lane_base, desc_kmajor(sQ, kk), desc_kmajor(sK[st0], kk), IDESC_QK, kk > 0);
        mma_commit(bars.s);
        ++is_;
      }
    }

    float m_run = -INFINITY;      // running max used for the exponentials (log2 domain)
    float l_run = 0.f;
    const int i_row = m * 128 + tid;   // this thread's query row

    for (int it = 0; it < nt; ++it) {
      const uint32_t g = gt + it;
      const int st = g & 1;
      const int kt = lo + it;
      if (ok && !mbar_wait(bars.s, g & 1, kTimeoutNs)) fail();
      tc_fence_after();
      __syncwarp();
      float s[128];
      {
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      }
      tc_fence_before();
      if (__syncthreads_or(!ok)) { aborted = true; break; }   // S has been read by every row
      if (tid == 0) {
        tc_fence_after();
        if (it + 2 < nt) {                              // K stage st is free again
          mbar_expect_tx(bars.k[st], kTileBytes);
          tma_load_3d(sK[st], &tmK, bars.k[st], 0, (kt + 2) * 128, zk);
          tma_load_3d(sK[st] + kHalfBytes, &tmK, bars.k[st], 64, (kt + 2) * 128, zk);
          ++ik[st];
        }
        if (it + 1 < nt) {                              // next S overlaps this softmax
          const int sn = (g + 1) & 1;
          if (mbar_wait(bars.k[sn], wk[sn] & 1, kTimeoutNs)) {
            ++wk[sn];
            tc_fence_after();
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16_ss(tS - lane_base, desc_kmajor(sQ, kk), desc_kmajor(sK[sn], kk), IDESC_QK, kk > 0);
            mma_commit(bars.s);
            ++is_;
          } else {
            fail();
          }
        }
      }

      // ---- mask (only tiles crossing the diagonal or the window's lower edge)
      const int hi_c = i_row - kt * 128;               // keys c <= hi_c are causal
      const int lo_c = i_row - S - kt * 128;           // keys c >  lo_c are inside the window
      if (hi_c < 127 || lo_c >= 0) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > hi_c || c <= lo_c) s[c] = -INFINITY;
      }
      float tmax = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) tmax = fmaxf(tmax, s[c]);
      const float mt = tmax * p.scale_log2;
      const float m_old = m_run;
      bool rescale = mt > m_run + kRescaleThreshold;
      float alpha = 1.f;
      if (rescale) {
        alpha = ex2_approx(m_old - mt);                // 0 when m_old = -inf
        m_run = mt;
        l_run *= alpha;
      }
      const float neg = (m_run == -INFINITY) ? 0.f : -m_run;
      const bool o_rescale = rescale && (m_old != -INFINITY) && it > 0;

      // PV of the previous tile must be done before O and P are touched.
      if (it > 0) {
        if (ok && !mbar_wait(bars.o, (g - 1) & 1, kTimeoutNs)) fail();
        tc_fence_after();
        if (tid == 0 && ok && it + 1 < nt) {            // V stage of tile it-1 is free
          const int sn = (g + 1) & 1;
          mbar_expect_tx(bars.v[sn], kTileBytes);
          tma_load_3d(sV[sn], &tmV, bars.v[sn], 0, (kt + 1) * 128, zk);
          tma_load_3d(sV[sn] + kHalfBytes, &tmV, bars.v[sn], 64, (kt + 1) * 128, zk);
          ++iv[sn];
        }
      }
      __syncwarp();
      if (__any_sync(0xffffffffu, o_rescale)) {
        const float a = o_rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a);
          tmem_st32(tO + c * 32, r);
        }
        tmem_st_wait();
      }

      // ---- exponentials, row sum, P (bf16) into swizzled shared memory
      float lsum = 0.f;
      const uint32_t row_off = (uint32_t)tid * 128u;
      const uint32_t sw = (uint32_t)(tid & 7);
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {               // 16-byte chunks of 8 keys
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2_approx(fmaf(s[ch * 8 + 2 * e], p.scale_log2, neg));
          const float p1 = ex2_approx(fmaf(s[ch * 8 + 2 * e + 1], p.scale_log2, neg));
          lsum += p0 + p1;
          w[e] = pack_bf16x2(p0, p1);
        }
        const uint32_t half = (uint32_t)(ch >> 3);
        const uint32_t cc = (uint32_t)(ch & 7);
        const uint32_t addr = sP + half * kHalfBytes + row_off + ((cc ^ sw) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]),
                     "r"(w[2]), "r"(w[3])
                     : "memory");
      }
      l_run += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      if (__syncthreads_or(!ok)) { aborted = true; break; }   // P written, O rescaled
      if (tid == 0) {
        tc_fence_after();
        if (mbar_wait(bars.v[st], wv[st] & 1, kTimeoutNs)) {
          ++wv[st];
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tO - lane_base, desc_kmajor(sP, kk), desc_v(sV[st], kk), IDESC_PV,
                        (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bars.o);
          ++io;
        } else {
          fail();
        }
      }
    }
    if (aborted) break;

    // ---- epilogue: O / l -> bf16, staged in shared memory, coalesced store
    if (ok && !mbar_wait(bars.o, (gt + nt - 1) & 1, kTimeoutNs)) fail();
    tc_fence_after();
    __syncwarp();
    {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint8_t* stage = smem + OFF_Q;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(r[8 * j + 0]) * inv, __uint_as_float(r[8 * j + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(r[8 * j + 2]) * inv, __uint_as_float(r[8 * j + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(r[8 * j + 4]) * inv, __uint_as_float(r[8 * j + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(r[8 * j + 6]) * inv, __uint_as_float(r[8 * j + 7]) * inv);
          *reinterpret_cast<uint4*>(stage + tid * kStageRowBytes + (c * 4 + j) * 16) = w;
        }
      }
    }
    tc_fence_before();
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    {
      const uint8_t* stage = smem + OFF_Q;
      __nv_bfloat16* obase = reinterpret_cast<__nv_bfloat16*>(p.o) + ((size_t)zq * p.N + (size_t)m * 128) * kD;
      const int rows = min(128, p.N - m * 128);
#pragma unroll 4
      for (int k = 0; k < 16; ++k) {
        const int lin = k * kThreads + tid;            // 16-byte chunk index in the tile
        const int row = lin >> 4, ch = lin & 15;
        if (row < rows) {
          const uint4 w = *reinterpret_cast<const uint4*>(stage + row * kStageRowBytes + ch * 16);
          *reinterpret_cast<uint4*>(obase + (size_t)row * kD + ch * 8) = w;
        }
      }
    }
    fence_proxy_async_smem();                           // staging reads before the next TMA writes
    __syncthreads();                                    // staging (Q / P area) free again
    gt += nt;
  }

  // ---- teardown: after a timeout, drain what thread 0 still has in flight
  __syncthreads();
  if (tid == 0 && aborted) {
    const uint64_t drain = 200000000ull;               // 0.2 s per outstanding phase
    while (wq < iq && mbar_wait(bars.q, wq & 1, drain)) ++wq;
    for (int st = 0; st < 2; ++st) {
      while (wk[st] < ik[st] && mbar_wait(bars.k[st], wk[st] & 1, drain)) ++wk[st];
      while (wv[st] < iv[st] && mbar_wait(bars.v[st], wv[st] & 1, drain)) ++wv[st];
    }
    // MMAs: one commit covers all earlier MMAs of this thread.
    if (is_ > 0) mbar_wait(bars.s, (is_ - 1) & 1, drain);
    if (io > 0) mbar_wait(bars.o, (io - 1) & 1, drain);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool make_map(CUtensorMap* map, const void* ptr, int32_t N, int64_t heads) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)N * kD * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr size_t kUnitsOffset = 256;

}  // namespace

std::vector<int32_t> prefill_units(int32_t B, int32_t Hq, int32_t N, const int32_t* spans) {
  const int32_t M = (N + kTileM - 1) / kTileM;
  struct U { int32_t b, h, m, lo, cost; };
  std::vector<U> v;
  v.reserve((size_t)B * Hq * M);
  for (int32_t b = 0; b < B; ++b)
    for (int32_t h = 0; h < Hq; ++h)
      for (int32_t m = 0; m < M; ++m) {
        const int64_t first_key = std::max<int64_t>(0, (int64_t)m * kTileM - spans[h] + 1);
        const int32_t lo = (int32_t)(first_key / kTileN);
        v.push_back({b, h, m, lo, m - lo + 1});
      }
  std::stable_sort(v.begin(), v.end(), [](const U& a, const U& c) { return a.cost > c.cost; });
  std::vector<int32_t> out(v.size() * 4);
  for (size_t i = 0; i < v.size(); ++i) {
    out[4 * i + 0] = v[i].b;
    out[4 * i + 1] = v[i].h;
    out[4 * i + 2] = v[i].m;
    out[4 * i + 3] = v[i].lo;
  }
  return out;
}

size_t prefill_workspace_bytes(int32_t B, int32_t Hq, int64_t N) {
  const int64_t M = (N + kTileM - 1) / kTileM;
  return kUnitsOffset + (size_t)B * Hq * M * 16;
}

moa_status launch_prefill_bf16(const void* q, const void* k, const void* v, void* o, int32_t B,
                               int32_t Hq, int32_t Hkv, int32_t N, const int32_t* spans, float scale,
                               void* ws, size_t ws_bytes, cudaStream_t s) {
  if (ws_bytes < prefill_workspace_bytes(B, Hq, N)) return MOA_ERR_WORKSPACE;
  if ((int64_t)B * Hq > INT32_MAX || (int64_t)B * Hkv > INT32_MAX) return MOA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, N, (int64_t)B * Hq) || !make_map(&mk, k, N, (int64_t)B * Hkv) ||
      !make_map(&mv, v, N, (int64_t)B * Hkv))
    return MOA_ERR_CUDA;
  // Header (error word, unit counter, zeroed) and the longest-first unit list,
  // uploaded in one copy.  The pageable source is staged by the runtime
  // before cudaMemcpyAsync returns.
  std::vector<int32_t> units = prefill_units(B, Hq, N, spans);
  const size_t n_units = units.size() / 4;
  std::vector<int32_t> blob(kUnitsOffset / 4 + units.size(), 0);
  std::copy(units.begin(), units.end(), blob.begin() + kUnitsOffset / 4);
  if (cudaMemcpyAsync(ws, blob.data(), blob.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOA_ERR_CUDA;

  PrefillParams p;
  p.hdr = reinterpret_cast<uint32_t*>(ws);
  p.units = reinterpret_cast<const int4*>((char*)ws + kUnitsOffset);
  p.o = o;
  p.n_units = (int32_t)n_units;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  for (int h = 0; h < Hq; ++h) p.span[h] = spans[h];

  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(prefill_bf16_sm100_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return MOA_ERR_CUDA;
  const int grid = (int)std::min<size_t>(n_units, (size_t)sm_count());
  prefill_bf16_sm100_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? MOA_OK : MOA_ERR_CUDA;
}

}  // namespace moa
