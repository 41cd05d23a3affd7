// bf16 prefill for heterogeneous sliding windows on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes ("Mixture of Attention" project page, "Finding two" and
// the N x N causal-band figure; blog walkthrough section 2.1): for query row
// i of head h, softmax(scale * q_i . k_j) over the keys i - S_h < j <= i,
// applied to v_j.  Heads differ only in S_h.
//
// How (B200 design, not the pages' A100 kernel):
//  * Work unit = (b, h, mp): two query tiles A = rows [256mp, 256mp+128) and
//    B = rows [256mp+128, 256mp+256) of one head.  Because the window is a
//    band, tile X needs exactly the key tiles loX..hiX (hiX its diagonal tile,
//    loX = floor(max(0, 128*tileX - S_h + 1) / 128)); every other key tile is
//    skipped.  The two query tiles share every K/V tile they both need.
//  * Units are sorted longest-first on the host and handed out by a
//    persistent grid (one CTA per SM): a producer thread takes the next unit
//    from an atomic counter and publishes it through a two-slot ring in
//    shared memory, so heads with very different spans balance across SMs.
//  * Warp roles (384 threads; warps 2-3 idle):
//      warp 0      TMA producer: Q_A, Q_B once per unit; K and V tiles through
//                  two-stage rings (128-byte swizzle).
//      warp 1      MMA issuer (one thread): S_X = Q_X K^T and O_X += P_X V with
//                  tcgen05.mma (M=128, N=128, K=16 steps), fp32 accumulators
//                  in tensor memory: S_A, S_B, O_A, O_B = 4 x 128 columns.
//      warps 4-7   softmax for tile A, warps 8-11 for tile B: one thread per
//                  query row reads its S row from TMEM, masks only tiles that
//                  cross the diagonal or the window's lower edge, runs the
//                  online softmax in the exp2 domain with a lazy rescale (the
//                  running max used for the exponentials moves only when it
//                  would grow by more than 2^8), and writes P as bf16 back into
//                  tensor memory over S; the PV MMA reads P from there (A
//                  operand in TMEM) and V straight from its TMA tile (MN-major).
//    The MMA thread alternates A and B, so the tensor core works on one query
//    tile while the other tile's exponentials run.
//  * Epilogue: each softmax thread normalises its O row (fp32 -> bf16,
//    round to nearest even) and stores it; rows >= N are dropped, and
//    out-of-range TMA rows read as zeros.
//  * Every mbarrier wait is bounded (2 s of globaltimer, or earlier if another
//    role gave up); on a timeout the kernel sets the workspace error word,
//    lets every role leave, waits for its in-flight copies, frees TMEM and
//    returns.
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

constexpr int kThreads = 384;                    // 3 warpgroups
// Register split (setmaxnreg): the block launches with 384 x 168 registers;
// warpgroup 0 (producer, MMA issuer, two idle warps) drops to 104 and the two
// softmax warpgroups rise to 200: 128*104 + 256*200 = 64512 = 384*168.
constexpr uint32_t kRegsLaunch = 168, kRegsControl = 104, kRegsSoftmax = 200;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr int kD = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;   // one 128 x 128 bf16 tile
constexpr uint32_t kHalfBytes = 128 * 64 * 2;    // one 128-row x 128-byte swizzled half
// Shared memory carve-up (offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_QA = 0;
constexpr uint32_t OFF_QB = OFF_QA + kTileBytes;
constexpr uint32_t kKStages = 2, kVStages = 2;        // K and V ring depths
constexpr uint32_t OFF_K = OFF_QB + kTileBytes;
constexpr uint32_t OFF_V = OFF_K + kKStages * kTileBytes;
constexpr uint32_t OFF_BAR = OFF_V + kVStages * kTileBytes;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024; // + barriers + alignment slack

constexpr uint32_t kTmemCols = 512;   // S_A [0,128) S_B [128,256) O_A [256,384) O_B [384,512)
constexpr uint64_t kTimeoutNs = 2000000000ull;        // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;             // log2 of the largest tolerated growth

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);

// mbarrier slots (8 bytes each) at OFF_BAR
enum {
  B_QFULL = 0, B_QEMPTY, B_SFULL_A, B_SFULL_B, B_PFULL_A, B_PFULL_B, B_OFULL_A, B_OFULL_B,
  B_OEMPTY_A, B_OEMPTY_B, B_UFULL0, B_UFULL1, B_UEMPTY0, B_UEMPTY1,
  B_KFULL0, B_KEMPTY0 = B_KFULL0 + 4, B_VFULL0 = B_KEMPTY0 + 4, B_VEMPTY0 = B_VFULL0 + 4,
  B_COUNT = B_VEMPTY0 + 4
};
static_assert(kKStages <= 4 && kVStages <= 4, "ring depth");

// Position in a ring of `n` stages: stage index and mbarrier phase parity.
struct Ring {
  uint32_t stage = 0, phase = 0;
  __device__ void next(uint32_t n) {
    if (++stage == n) { stage = 0; phase ^= 1u; }
  }
};
constexpr uint32_t OFF_TMEM_SLOT = OFF_BAR + 8 * B_COUNT;        // uint32
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;                // int
constexpr uint32_t OFF_UNIT = OFF_ABORT + 4;                     // int[2]
static_assert(OFF_UNIT + 8 <= OFF_BAR + 512, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct PrefillParams {
  uint32_t* hdr;                 // [0] error word, [1] unit counter
  const int4* units;             // (b, h, mp, unused), longest first
  void* o;
  int32_t n_units, N, Hq, Hkv, G, n_qtiles;
  float scale_log2;
  int32_t span[MOA_MAX_HEADS];
};

// K-major operand (Q or K) of one 16-wide K step kk (0..7): the 128-wide
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

struct Ctx {
  uint32_t bar0;                       // address of barrier 0
  volatile int* abort;
  volatile int* ring;                  // published unit indices, 2 slots
  uint32_t* hdr;
  __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
  // Bounded wait that also gives up when another role has already failed.
  __device__ bool wait(int i, uint32_t parity) const {
    const uint32_t b = bar(i);
    if (mbar_try(b, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
      if (mbar_try(b, parity)) return true;
      if (*abort) return false;
      if (globaltimer() - t0 > kTimeoutNs) {
        *abort = 1;
        atomicOr(hdr, kErrTimeout);
        return false;
      }
    }
  }
};

// First key tile needed by query tile `qt` under span S.
__device__ __forceinline__ int first_key_tile(int qt, int S) {
  const int first_key = max(0, qt * 128 - S + 1);
  return first_key >> 7;
}

struct UnitInfo {
  int S, zq, zk;
  int loA, hiA, loB, hiB;
  bool actB;
};

__device__ __forceinline__ UnitInfo decode_unit(const PrefillParams& p, int u) {
  UnitInfo x;
  const int4 U = p.units[u];
  const int b = U.x, h = U.y, mp = U.z;
  x.S = p.span[h];
  x.zq = b * p.Hq + h;
  x.zk = b * p.Hkv + h / p.G;
  x.hiA = 2 * mp;
  x.loA = first_key_tile(x.hiA, x.S);
  x.hiB = x.hiA + 1;
  x.loB = first_key_tile(x.hiB, x.S);
  x.actB = x.hiB < p.n_qtiles;
  return x;
}

// ---------------------------------------------------------------------------
// Softmax role: 128 threads own the 128 rows of query tile X.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void softmax_role(const PrefillParams& p, const Ctx& c, uint32_t tmem,
                                             int X, int warp, int lane) {
  const int quarter = warp & 3;                      // TMEM lane quarter this warp may access
  const int r = quarter * 32 + lane;                 // row within the query tile
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_base + (uint32_t)(X * 128);
  const uint32_t tO = tmem + lane_base + 256u + (uint32_t)(X * 128);
  uint32_t s_cnt = 0, o_cnt = 0;
  for (uint32_t i = 0;; ++i) {
    if (!c.wait(B_UFULL0 + (i & 1), (i >> 1) & 1)) return;
    const int u = c.ring[i & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(c.bar(B_UEMPTY0 + (i & 1)));
    if (u >= p.n_units) return;
    const UnitInfo x = decode_unit(p, u);
    if (X == 1 && !x.actB) continue;
    const int qt = X == 0 ? x.hiA : x.hiB;
    const int lo = X == 0 ? x.loA : x.loB;
    const int i_row = qt * 128 + r;

    float m_run = -INFINITY, l_run = 0.f;
    for (int kt = lo; kt <= qt; ++kt) {
      if (!c.wait(B_SFULL_A + X, s_cnt & 1)) return;
      ++s_cnt;
      tc_fence_after();
      __syncwarp();
      float s[128];
      {
        uint32_t sr[128];
        tmem_ld128(tS, sr);
#pragma unroll
        for (int cc = 0; cc < 128; ++cc) s[cc] = __uint_as_float(sr[cc]);
      }
      // mask: only tiles crossing the diagonal or the window's lower edge
      const int hi_c = i_row - kt * 128;             // keys c <= hi_c are causal
      const int lo_c = i_row - x.S - kt * 128;       // keys c >  lo_c are inside the window
      if (hi_c < 127 || lo_c >= 0) {
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          if (cc > hi_c || cc <= lo_c) s[cc] = -INFINITY;
      }
      float mx[8];                                   // 8 independent max chains
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
      for (int cc = 16; cc < 128; cc += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], s[cc + 2 * k], s[cc + 2 * k + 1]);
      const float tmax = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      const float mt = tmax * p.scale_log2;
      const float m_old = m_run;
      const bool rescale = mt > m_run + kRescaleThreshold;
      float alpha = 1.f;
      if (rescale) {
        alpha = ex2_approx(m_old - mt);              // 0 when m_old = -inf
        m_run = mt;
        l_run *= alpha;
      }
      const float neg = (m_run == -INFINITY) ? 0.f : -m_run;
      // O_X is stable here: PV_X(kt-1) completed before S_X(kt) (in-order MMAs).
      const bool o_rescale = rescale && (m_old != -INFINITY) && kt > lo;
      if (__any_sync(0xffffffffu, o_rescale)) {
        const float a = o_rescale ? alpha : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t rr[32];
          tmem_ld32(tO + cc * 32, rr);
#pragma unroll
          for (int j = 0; j < 32; ++j) rr[j] = __float_as_uint(__uint_as_float(rr[j]) * a);
          tmem_st32(tO + cc * 32, rr);
        }
      }
      // exponentials (MUFU ex2), row sum in 8 independent chains, P (bf16
      // pairs) into TMEM over S
      float ls[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) ls[k] = 0.f;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {               // 2 x 32 columns = 128 keys
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x0 = fmaf(s[cc * 64 + 2 * j], p.scale_log2, neg);
          const float x1 = fmaf(s[cc * 64 + 2 * j + 1], p.scale_log2, neg);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          ls[j & 7] += p0 + p1;
          w[j] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + cc * 32, w);
      }
      l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(c.bar(B_PFULL_A + X));
    }

    // epilogue: O / l -> bf16 -> global
    if (!c.wait(B_OFULL_A + X, o_cnt & 1)) return;
    ++o_cnt;
    tc_fence_after();
    __syncwarp();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + ((size_t)x.zq * p.N + (size_t)i_row) * kD;
    const bool store = i_row < p.N;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t rr[32];
      tmem_ld32(tO + cc * 32, rr);
      if (store) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(rr[8 * j + 0]) * inv, __uint_as_float(rr[8 * j + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(rr[8 * j + 2]) * inv, __uint_as_float(rr[8 * j + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(rr[8 * j + 4]) * inv, __uint_as_float(rr[8 * j + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(rr[8 * j + 6]) * inv, __uint_as_float(rr[8 * j + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + cc * 32 + j * 8) = w;
        }
      }
    }
    tc_fence_before();
    mbar_arrive(c.bar(B_OEMPTY_A + X));
  }
}

// ---------------------------------------------------------------------------
// MMA role: one thread.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void issue_pv(uint32_t tO, uint32_t tP, uint32_t sV, bool first) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_bf16_ts(tO, tP + (uint32_t)kk * 8u, desc_v(sV, kk), IDESC_PV, (!first || kk > 0) ? 1u : 0u);
}

__device__ __forceinline__ void mma_role(const PrefillParams& p, const Ctx& c, uint32_t tmem,
                                         uint32_t sQ0, uint32_t sK0, uint32_t sV0) {
  Ring kr, vr;                              // K and V ring positions
  uint32_t qc = 0;                          // units consumed
  uint32_t pc[2] = {0, 0}, oe[2] = {0, 0};  // P tiles consumed, units started per X
  for (uint32_t i = 0;; ++i) {
    if (!c.wait(B_UFULL0 + (i & 1), (i >> 1) & 1)) return;
    const int u = c.ring[i & 1];
    mbar_arrive(c.bar(B_UEMPTY0 + (i & 1)));
    if (u >= p.n_units) return;
    const UnitInfo x = decode_unit(p, u);
    const int lo = x.loA;
    const int hi = x.actB ? x.hiB : x.hiA;
    if (!c.wait(B_QFULL, qc & 1)) return;
    ++qc;
    tc_fence_after();
    bool first_pv[2] = {true, true};
    uint32_t v_prev = 0;                   // V stage of key tile kt-1
    for (int kt = lo; kt <= hi; ++kt) {
      const uint32_t ks = kr.stage;
      if (!c.wait(B_KFULL0 + ks, kr.phase)) return;
      kr.next(kKStages);
      tc_fence_after();
      if (kt > lo) {                       // V(kt-1) feeds this step's PVs
        v_prev = vr.stage;
        if (!c.wait(B_VFULL0 + v_prev, vr.phase)) return;
        vr.next(kVStages);
        tc_fence_after();
      }
#pragma unroll
      for (int X = 0; X < 2; ++X) {
        const bool act = X == 0 || x.actB;
        const int loX = X == 0 ? x.loA : x.loB;
        const int hiX = X == 0 ? x.hiA : x.hiB;
        if (!act) continue;
        if (kt - 1 >= loX && kt - 1 <= hiX) {                // O_X += P_X(kt-1) V(kt-1)
          if (!c.wait(B_PFULL_A + X, pc[X] & 1)) return;
          ++pc[X];
          if (first_pv[X]) {
            if (!c.wait(B_OEMPTY_A + X, (oe[X] & 1) ^ 1)) return;
            ++oe[X];
          }
          tc_fence_after();
          issue_pv(tmem + 256u + 128u * X, tmem + 128u * X, sV0 + v_prev * kTileBytes, first_pv[X]);
          first_pv[X] = false;
        }
        if (kt >= loX && kt <= hiX) {                        // S_X = Q_X K(kt)^T
          const uint32_t sK = sK0 + ks * kTileBytes;
          const uint32_t sQ = sQ0 + (uint32_t)X * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + 128u * X, desc_kmajor(sQ, kk), desc_kmajor(sK, kk), IDESC_QK,
                        kk > 0 ? 1u : 0u);
          mma_commit(c.bar(B_SFULL_A + X));
        }
      }
      mma_commit(c.bar(B_KEMPTY0 + ks));
      if (kt > lo) mma_commit(c.bar(B_VEMPTY0 + v_prev));
    }
    mma_commit(c.bar(B_QEMPTY));           // every S of the unit is issued
    // tail: PVs of the last key tile
    v_prev = vr.stage;
    if (!c.wait(B_VFULL0 + v_prev, vr.phase)) return;
    vr.next(kVStages);
    tc_fence_after();
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      const bool act = X == 0 || x.actB;
      const int loX = X == 0 ? x.loA : x.loB;
      const int hiX = X == 0 ? x.hiA : x.hiB;
      if (!act || hi < loX || hi > hiX) continue;
      if (!c.wait(B_PFULL_A + X, pc[X] & 1)) return;
      ++pc[X];
      if (first_pv[X]) {
        if (!c.wait(B_OEMPTY_A + X, (oe[X] & 1) ^ 1)) return;
        ++oe[X];
      }
      tc_fence_after();
      issue_pv(tmem + 256u + 128u * X, tmem + 128u * X, sV0 + v_prev * kTileBytes, first_pv[X]);
      first_pv[X] = false;
    }
    mma_commit(c.bar(B_VEMPTY0 + v_prev));
    mma_commit(c.bar(B_OFULL_A));
    if (x.actB) mma_commit(c.bar(B_OFULL_B));
  }
}

// ---------------------------------------------------------------------------
// Producer role: one thread (unit fetch + TMA).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void producer_role(const PrefillParams& p, const Ctx& c,
                                              const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                              const CUtensorMap* tmV, uint32_t sQ0, uint32_t sK0,
                                              uint32_t sV0) {
  Ring kr, vr;
  uint32_t qc = 0;
  for (uint32_t i = 0;; ++i) {
    if (!c.wait(B_UEMPTY0 + (i & 1), ((i >> 1) & 1) ^ 1)) return;
    const int u = (int)atomicAdd(p.hdr + 1, 1u);
    c.ring[i & 1] = u;
    mbar_arrive(c.bar(B_UFULL0 + (i & 1)));
    if (u >= p.n_units) return;
    const UnitInfo x = decode_unit(p, u);
    const int lo = x.loA;
    const int hi = x.actB ? x.hiB : x.hiA;
    if (!c.wait(B_QEMPTY, (qc & 1) ^ 1)) return;
    ++qc;
    mbar_expect_tx(c.bar(B_QFULL), x.actB ? 2 * kTileBytes : kTileBytes);
    tma_load_3d(sQ0, tmQ, c.bar(B_QFULL), 0, x.hiA * 128, x.zq);
    tma_load_3d(sQ0 + kHalfBytes, tmQ, c.bar(B_QFULL), 64, x.hiA * 128, x.zq);
    if (x.actB) {
      tma_load_3d(sQ0 + kTileBytes, tmQ, c.bar(B_QFULL), 0, x.hiB * 128, x.zq);
      tma_load_3d(sQ0 + kTileBytes + kHalfBytes, tmQ, c.bar(B_QFULL), 64, x.hiB * 128, x.zq);
    }
    for (int kt = lo; kt <= hi; ++kt) {
      const uint32_t ks = kr.stage;
      if (!c.wait(B_KEMPTY0 + ks, kr.phase ^ 1)) return;
      kr.next(kKStages);
      mbar_expect_tx(c.bar(B_KFULL0 + ks), kTileBytes);
      tma_load_3d(sK0 + ks * kTileBytes, tmK, c.bar(B_KFULL0 + ks), 0, kt * 128, x.zk);
      tma_load_3d(sK0 + ks * kTileBytes + kHalfBytes, tmK, c.bar(B_KFULL0 + ks), 64, kt * 128, x.zk);
      const uint32_t vs = vr.stage;
      if (!c.wait(B_VEMPTY0 + vs, vr.phase ^ 1)) return;
      vr.next(kVStages);
      mbar_expect_tx(c.bar(B_VFULL0 + vs), kTileBytes);
      tma_load_3d(sV0 + vs * kTileBytes, tmV, c.bar(B_VFULL0 + vs), 0, kt * 128, x.zk);
      tma_load_3d(sV0 + vs * kTileBytes + kHalfBytes, tmV, c.bar(B_VFULL0 + vs), 64, kt * 128, x.zk);
    }
  }
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
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  Ctx c;
  c.bar0 = sbase + OFF_BAR;
  c.abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  c.ring = reinterpret_cast<volatile int*>(smem + OFF_UNIT);
  c.hdr = p.hdr;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == B_PFULL_A || i == B_PFULL_B || i == B_OEMPTY_A || i == B_OEMPTY_B) cnt = 128;
      if (i == B_UEMPTY0 || i == B_UEMPTY1) cnt = 9;   // MMA thread + 8 softmax warps
      mbar_init(c.bar(i), cnt);
    }
    *c.abort = 0;
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

  if (warp < 4) {
    regs_dec<kRegsControl>();
    if (warp == 0 && lane == 0)
      producer_role(p, c, &tmQ, &tmK, &tmV, sbase + OFF_QA, sbase + OFF_K, sbase + OFF_V);
    else if (warp == 1 && lane == 0)
      mma_role(p, c, tmem, sbase + OFF_QA, sbase + OFF_K, sbase + OFF_V);
  } else {
    regs_inc<kRegsSoftmax>();
    softmax_role(p, c, tmem, warp < 8 ? 0 : 1, warp, lane);
  }

  // teardown: after a timeout give in-flight copies and MMAs time to land
  __syncthreads();
  if (*c.abort && tid == 0) {
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 20000000ull) __nanosleep(100000);
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

int64_t first_tile_host(int64_t qt, int32_t S) {
  return std::max<int64_t>(0, qt * kTileM - S + 1) / kTileN;
}

}  // namespace

// Units of two query tiles (256 rows); a unit's cost is the number of
// (query tile, key tile) pairs it visits.
std::vector<int32_t> prefill_units(int32_t B, int32_t Hq, int32_t N, const int32_t* spans) {
  const int64_t M = (N + kTileM - 1) / kTileM;      // query tiles
  const int64_t MP = (M + 1) / 2;                   // units per head
  struct U { int32_t b, h, mp; int64_t cost; };
  std::vector<U> v;
  v.reserve((size_t)B * Hq * MP);
  for (int32_t b = 0; b < B; ++b)
    for (int32_t h = 0; h < Hq; ++h)
      for (int64_t mp = 0; mp < MP; ++mp) {
        const int64_t qa = 2 * mp, qb = 2 * mp + 1;
        int64_t cost = qa - first_tile_host(qa, spans[h]) + 1;
        if (qb < M) cost += qb - first_tile_host(qb, spans[h]) + 1;
        v.push_back({b, h, (int32_t)mp, cost});
      }
  std::stable_sort(v.begin(), v.end(), [](const U& a, const U& c) { return a.cost > c.cost; });
  std::vector<int32_t> out(v.size() * 4);
  for (size_t i = 0; i < v.size(); ++i) {
    out[4 * i + 0] = v[i].b;
    out[4 * i + 1] = v[i].h;
    out[4 * i + 2] = v[i].mp;
    out[4 * i + 3] = 0;
  }
  return out;
}

void prefill_unit_tiles(int32_t N, int32_t S, int32_t mp, int32_t tiles[4]) {
  const int64_t M = (N + kTileM - 1) / kTileM;
  const int64_t qa = 2 * (int64_t)mp, qb = qa + 1;
  tiles[0] = (int32_t)first_tile_host(qa, S);
  tiles[1] = (int32_t)qa;
  tiles[2] = qb < M ? (int32_t)first_tile_host(qb, S) : -1;
  tiles[3] = qb < M ? (int32_t)qb : -1;
}

size_t prefill_workspace_bytes(int32_t B, int32_t Hq, int64_t N) {
  const int64_t M = (N + kTileM - 1) / kTileM;
  const int64_t MP = (M + 1) / 2;
  return kUnitsOffset + (size_t)B * Hq * MP * 16;
}

moa_status launch_prefill_bf16(const void* q, const void* k, const void* v, void* o, int32_t B,
                               int32_t Hq, int32_t Hkv, int32_t N, const int32_t* spans, float scale,
                               void* ws, size_t ws_bytes, cudaStream_t s) {
  if (ws_bytes < prefill_workspace_bytes(B, Hq, N)) return MOA_ERR_WORKSPACE;
  if ((int64_t)B * Hq > INT32_MAX || (int64_t)B * Hkv > INT32_MAX) return MOA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, N, (int64_t)B * Hq) || !make_map(&mk, k, N, (int64_t)B * Hkv) ||
      !make_map(&mv, v, N, (int64_t)B * Hkv))
    return cuda_fail(cudaErrorInvalidValue, "tensor map encode");
  // Header (error word, unit counter, zeroed) and the longest-first unit list,
  // uploaded in one copy.  The pageable source is staged by the runtime
  // before cudaMemcpyAsync returns.
  std::vector<int32_t> units = prefill_units(B, Hq, N, spans);
  const size_t n_units = units.size() / 4;
  std::vector<int32_t> blob(kUnitsOffset / 4 + units.size(), 0);
  std::copy(units.begin(), units.end(), blob.begin() + kUnitsOffset / 4);
  cudaError_t e = cudaMemcpyAsync(ws, blob.data(), blob.size() * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill unit upload");

  PrefillParams p;
  p.hdr = reinterpret_cast<uint32_t*>(ws);
  p.units = reinterpret_cast<const int4*>((char*)ws + kUnitsOffset);
  p.o = o;
  p.n_units = (int32_t)n_units;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = (N + kTileM - 1) / kTileM;
  p.scale_log2 = scale * 1.4426950408889634f;
  for (int h = 0; h < Hq; ++h) p.span[h] = spans[h];

  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(prefill_bf16_sm100_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "prefill smem attribute");
  const int grid = (int)std::min<size_t>(n_units, (size_t)sm_count());
  prefill_bf16_sm100_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, p);
  return check_launch("prefill_bf16 launch");
}

}  // namespace moa
