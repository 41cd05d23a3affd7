// bf16 prefill for heterogeneous sliding windows on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes ("Mixture of Attention" project page, "Finding two" and
// the N x N causal-band figure; blog walkthrough section 2.1): for query row
// i of head h, softmax(scale * q_i . k_j) over the keys i - S_h < j <= i,
// applied to v_j.  Heads differ only in S_h.
//
// How (B200 design, not the pages' A100 kernel):
//  * Work unit = (b, h, m): query rows [128m, 128m+128) of one head.  Because
//    the window is a band, the unit needs exactly the key tiles lo..m
//    (lo = floor(max(0, 128m - S_h + 1) / 128)); every other key tile is
//    skipped.
//  * Units are sorted longest-first on the host and handed out by a
//    persistent grid (one CTA per SM): a producer thread takes the next unit
//    from an atomic counter and publishes it through a two-slot ring in
//    shared memory, so heads with very different spans balance across SMs.
//  * Warp roles (384 threads, setmaxnreg split 144 / 216 / 144):
//      warp 0       TMA producer: Q once per unit into one of two buffers
//                   (the next unit's Q loads while this unit runs), K and V
//                   tiles through two-stage rings (128-byte swizzle).
//      warp 1       MMA issuer (one thread), tcgen05.mma M=128, N=128, K=16:
//                   S(k) = Q K(k)^T into one of two S buffers in tensor memory,
//                   O += P(k-1) V(k-1) with P read from tensor memory.  S(k+1)
//                   is issued right after PV(k-1), without waiting for the
//                   softmax of tile k, so the tensor core works on the next
//                   tile while the current tile's exponentials run.
//      warps 4-7    softmax: one thread per query row reads its S row, masks
//                   only tiles that cross the diagonal or the window's lower
//                   edge, takes exponentials against the row's running maximum
//                   (exact tile maxima only when needed, see softmax_role),
//                   and writes P as bf16 pairs back over its S buffer.
//      warps 8-11   epilogue: O / l -> bf16 (round to nearest even) -> global,
//                   from one of two O buffers, so the next unit's PVs proceed
//                   while the previous unit is written out.
//    Tensor memory: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
//  * Rows >= N are dropped at the store; out-of-range TMA rows read as zeros.
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
// warpgroup 0 (producer, MMA issuer, two idle warps) and the epilogue
// warpgroup drop to 144, the softmax warpgroup rises to 216.
constexpr uint32_t kRegsLaunch = 168, kRegsControl = 144, kRegsSoftmax = 216, kRegsEpilogue = 144;
static_assert(128 * (kRegsControl + kRegsSoftmax + kRegsEpilogue) <= kThreads * kRegsLaunch,
              "register split");
constexpr int kD = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;   // one 128 x 128 bf16 tile
constexpr uint32_t kHalfBytes = 128 * 64 * 2;    // one 128-row x 128-byte swizzled half
// Shared memory carve-up (offsets from a 1024-byte aligned base).
constexpr uint32_t kKStages = 2, kVStages = 2;        // K and V ring depths
constexpr uint32_t OFF_Q = 0;                         // two Q buffers (units alternate)
constexpr uint32_t OFF_K = OFF_Q + 2 * kTileBytes;
constexpr uint32_t OFF_V = OFF_K + kKStages * kTileBytes;
constexpr uint32_t OFF_INVL = OFF_V + kVStages * kTileBytes;   // float[2][128]
constexpr uint32_t OFF_BAR = OFF_INVL + 2 * 128 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;          // + barriers + alignment slack

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;        // 2 s per wait

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);

// mbarrier slots (8 bytes each) at OFF_BAR
enum {
  B_QFULL0 = 0, B_QFULL1, B_QEMPTY0, B_QEMPTY1, B_SFULL0, B_SFULL1, B_PFULL0, B_PFULL1, B_PVDONE,
  B_OFULL0, B_OFULL1,
  B_LFULL0, B_LFULL1, B_OEMPTY0, B_OEMPTY1, B_UFULL0, B_UFULL1, B_UEMPTY0, B_UEMPTY1,
  B_KFULL0, B_KEMPTY0 = B_KFULL0 + 4, B_VFULL0 = B_KEMPTY0 + 4, B_VEMPTY0 = B_VFULL0 + 4,
  B_COUNT = B_VEMPTY0 + 4
};
static_assert(kKStages <= 4 && kVStages <= 4, "ring depth");
constexpr uint32_t OFF_TMEM_SLOT = OFF_BAR + 8 * B_COUNT;        // uint32
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;                // int
constexpr uint32_t OFF_UNIT = OFF_ABORT + 4;                     // int[2]
static_assert(OFF_UNIT + 8 <= OFF_BAR + 512, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// Position in a ring of `n` stages: stage index and mbarrier phase parity.
struct Ring {
  uint32_t stage = 0, phase = 0;
  __device__ void next(uint32_t n) {
    if (++stage == n) { stage = 0; phase ^= 1u; }
  }
};

struct PrefillParams {
  uint32_t* hdr;                 // [0] error word, [1] unit counter
  const int4* units;             // (b, h, m, lo), longest first
  void* o;
  int32_t n_units, N, Hq, Hkv, G;
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
  // Warp-wide roles: every lane waits, then the warp agrees on the outcome
  // (all lanes are present), so no lane leaves while the others go on to a
  // warp-collective tcgen05 instruction.
  __device__ bool wait_warp(int i, uint32_t parity) const {
    const bool ok = wait(i, parity);
    return !__any_sync(0xffffffffu, !ok);
  }
  // Next unit index from the ring.  Single-thread roles (warp_wide = false)
  // release the slot themselves; warp-wide roles release it from lane 0 after
  // every lane has read it.
  __device__ bool next_unit(uint32_t i, int lane, bool warp_wide, int* u) const {
    if (warp_wide) {
      if (!wait_warp(B_UFULL0 + (i & 1), (i >> 1) & 1)) return false;
      *u = ring[i & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_UEMPTY0 + (i & 1)));
    } else {
      if (!wait(B_UFULL0 + (i & 1), (i >> 1) & 1)) return false;
      *u = ring[i & 1];
      mbar_arrive(bar(B_UEMPTY0 + (i & 1)));
    }
    return true;
  }
};

struct UnitInfo {
  int S, zq, zk, m, lo;
};

__device__ __forceinline__ UnitInfo decode_unit(const PrefillParams& p, int u) {
  UnitInfo x;
  const int4 U = p.units[u];
  x.S = p.span[U.y];
  x.zq = U.x * p.Hq + U.y;
  x.zk = U.x * p.Hkv + U.y / p.G;
  x.m = U.z;
  x.lo = U.w;
  return x;
}

// ---------------------------------------------------------------------------
// Softmax role: 128 threads own the 128 rows of the unit's query tile.
//
// Exponentials are taken against the running maximum m of the row (log2
// domain) without first reducing the tile: a tile whose largest score exceeds
// m by more than 15 makes the tile's sum of 2^(s - m) reach 2^15, and only
// then (rarely after the first tile) is the tile's exact maximum computed, m
// raised, the row sum and O rescaled, and the tile redone.  Every exponential
// is therefore at most 2^15, far inside fp32 and bf16 range, and O / l is
// exact whichever m was used.  A row with no maximum yet (first tile with
// in-window keys) takes the exact maximum directly.
// ---------------------------------------------------------------------------
constexpr float kTileSumLimit = 32768.f;             // 2^15

// Row maximum of 128 scores, 8 independent chains.
__device__ __forceinline__ float row_max128(const float* s) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
  for (int cc = 16; cc < 128; cc += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], s[cc + 2 * k], s[cc + 2 * k + 1]);
  return max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// p = 2^(s * c - m) for 128 scores as bf16 pairs w[64] (MUFU ex2); returns
// the fp32 sum.
__device__ __forceinline__ float exp_tile(const float* s, float c, float neg, uint32_t* w) {
  const uint64_t c2 = f2_pack(c, c), n2 = f2_pack(neg, neg);
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const uint64_t x2 = f2_fma(f2_pack(s[2 * j], s[2 * j + 1]), c2, n2);
    float x0, x1;
    f2_unpack(x2, x0, x1);
    const uint64_t p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
    acc[j & 3] = f2_add(acc[j & 3], p2);
    float p0, p1;
    f2_unpack(p2, p0, p1);
    w[j] = pack_bf16x2(p0, p1);
  }
  const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float a, b;
  f2_unpack(t, a, b);
  return a + b;
}

__device__ __forceinline__ void mask_tile(float* s, int hi_c, int lo_c) {
  if (hi_c < 127 || lo_c >= 0) {
#pragma unroll
    for (int cc = 0; cc < 128; ++cc)
      if (cc > hi_c || cc <= lo_c) s[cc] = -INFINITY;
  }
}

__device__ __forceinline__ void softmax_role(const PrefillParams& p, const Ctx& c, uint32_t tmem,
                                             float* inv_l, int warp, int lane) {
  const int quarter = warp & 3;                      // TMEM lane quarter this warp may access
  const int r = quarter * 32 + lane;                 // row within the query tile
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  const float sc = p.scale_log2;
  uint32_t tcount = 0, uc = 0;
  for (uint32_t i = 0;; ++i) {
    int u;
    if (!c.next_unit(i, lane, true, &u)) return;
    if (u >= p.n_units) return;
    const UnitInfo x = decode_unit(p, u);
    const uint32_t tO = tmem + lane_base + kColO + 128u * (uc & 1);
    const int i_row = x.m * 128 + r;
    float m_run = -INFINITY, l_run = 0.f;
    for (int kt = x.lo; kt <= x.m; ++kt, ++tcount) {
      const uint32_t sb = tcount & 1;
      const uint32_t tS = tmem + lane_base + kColS + 128u * sb;
      if (!c.wait_warp(B_SFULL0 + sb, (tcount >> 1) & 1)) return;
      tc_fence_after();
      const int hi_c = i_row - kt * 128;             // keys c <= hi_c are causal
      const int lo_c = i_row - x.S - kt * 128;       // keys c >  lo_c are inside the window
      float s[128];
      {
        uint32_t sr[128];
        tmem_ld128(tS, sr);
#pragma unroll
        for (int cc = 0; cc < 128; ++cc) s[cc] = __uint_as_float(sr[cc]);
      }
      mask_tile(s, hi_c, lo_c);
      // rows without a maximum yet take this tile's exact maximum
      const bool need_max = m_run == -INFINITY;
      if (__any_sync(0xffffffffu, need_max)) {
        const float tmax = row_max128(s);
        if (need_max) m_run = tmax * sc;            // stays -inf if every key is masked
      }
      uint32_t w[64];
      float l_tile = exp_tile(s, sc, m_run == -INFINITY ? 0.f : -m_run, w);
      const bool redo = !(l_tile < kTileSumLimit);
      if (__any_sync(0xffffffffu, redo)) {
        // Rare: a score far above the running maximum.  Take the tile's exact
        // maximum, rescale the row, and recompute the tile.
        const float mt = row_max128(s) * sc;
        float alpha = 1.f;
        if (redo) {
          alpha = ex2_approx(m_run - mt);
          m_run = mt;
          l_run *= alpha;
        }
        if (__any_sync(0xffffffffu, redo && kt > x.lo)) {
          // O must hold every PV up to tile kt-1: wait for that PV's completion.
          if (!c.wait_warp(B_PVDONE, (tcount - 1) & 1)) return;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t rr[32];
            tmem_ld32(tO + cc * 32, rr);
#pragma unroll
            for (int j = 0; j < 32; ++j) rr[j] = __float_as_uint(__uint_as_float(rr[j]) * alpha);
            tmem_st32(tO + cc * 32, rr);
          }
        }
        l_tile = exp_tile(s, sc, m_run == -INFINITY ? 0.f : -m_run, w);
      }
      l_run += l_tile;
      tmem_st32(tS, w);
      tmem_st32(tS + 32, w + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(c.bar(B_PFULL0 + sb));
    }
    // Hand the row's normaliser to the epilogue warpgroup.  The slot was last
    // used by unit uc-2: wait until the epilogue has released it (a unit of
    // one or two key tiles can otherwise get here before that epilogue ran).
    if (!c.wait_warp(B_OEMPTY0 + (uc & 1), ((uc >> 1) & 1) ^ 1)) return;
    inv_l[128 * (uc & 1) + r] = l_run > 0.f ? 1.f / l_run : 0.f;
    mbar_arrive(c.bar(B_LFULL0 + (uc & 1)));
    ++uc;
  }
}

// ---------------------------------------------------------------------------
// Epilogue role: 128 threads write the unit's 128 output rows.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void epilogue_role(const PrefillParams& p, const Ctx& c, uint32_t tmem,
                                              const float* inv_l, int warp, int lane) {
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  uint32_t uc = 0;
  for (uint32_t i = 0;; ++i) {
    int u;
    if (!c.next_unit(i, lane, true, &u)) return;
    if (u >= p.n_units) return;
    const UnitInfo x = decode_unit(p, u);
    const uint32_t ob = uc & 1;
    if (!c.wait_warp(B_OFULL0 + ob, (uc >> 1) & 1)) return;
    if (!c.wait_warp(B_LFULL0 + ob, (uc >> 1) & 1)) return;
    tc_fence_after();
    const uint32_t tO = tmem + lane_base + kColO + 128u * ob;
    const float inv = inv_l[128 * ob + r];
    const int i_row = x.m * 128 + r;
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
    mbar_arrive(c.bar(B_OEMPTY0 + ob));
    ++uc;
  }
}

// ---------------------------------------------------------------------------
// MMA role: one thread.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_role(const PrefillParams& p, const Ctx& c, uint32_t tmem,
                                         uint32_t sQ0, uint32_t sK0, uint32_t sV0) {
  Ring kr, vr;                      // K and V ring positions
  uint32_t tc = 0, tp = 0, uc = 0;  // S tiles issued, PV tiles issued, units
  for (uint32_t i = 0;; ++i) {
    int u;
    if (!c.next_unit(i, 0, false, &u)) return;
    if (u >= p.n_units) return;
    const UnitInfo x = decode_unit(p, u);
    const uint32_t ob = uc & 1;
    const uint32_t tO = tmem + kColO + 128u * ob;
    const uint32_t sQ = sQ0 + ob * kTileBytes;
    if (!c.wait(B_QFULL0 + ob, (uc >> 1) & 1)) return;
    tc_fence_after();
    // PV of the unit's tile jj (P in the S buffer that tile used).
    auto pv = [&](bool first) -> bool {
      if (!c.wait(B_PFULL0 + (tp & 1), (tp >> 1) & 1)) return false;
      if (!c.wait(B_VFULL0 + vr.stage, vr.phase)) return false;
      if (first && !c.wait(B_OEMPTY0 + ob, ((uc >> 1) & 1) ^ 1)) return false;
      tc_fence_after();
      const uint32_t tP = tmem + kColS + 128u * (tp & 1);
      const uint32_t sV = sV0 + vr.stage * kTileBytes;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ts(tO, tP + (uint32_t)kk * 8u, desc_v(sV, kk), IDESC_PV, (!first || kk > 0) ? 1u : 0u);
      mma_commit(c.bar(B_PVDONE));
      mma_commit(c.bar(B_VEMPTY0 + vr.stage));
      vr.next(kVStages);
      ++tp;
      return true;
    };
    for (int kt = x.lo; kt <= x.m; ++kt) {
      // S(kt) = Q K(kt)^T into S buffer tc & 1
      if (!c.wait(B_KFULL0 + kr.stage, kr.phase)) return;
      tc_fence_after();
      const uint32_t sK = sK0 + kr.stage * kTileBytes;
      const uint32_t tS = tmem + kColS + 128u * (tc & 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tS, desc_kmajor(sQ, kk), desc_kmajor(sK, kk), IDESC_QK, kk > 0 ? 1u : 0u);
      mma_commit(c.bar(B_SFULL0 + (tc & 1)));
      mma_commit(c.bar(B_KEMPTY0 + kr.stage));
      kr.next(kKStages);
      ++tc;
      if (kt == x.m) mma_commit(c.bar(B_QEMPTY0 + ob));   // every S of the unit issued
      // O += P(kt-1) V(kt-1)
      if (kt > x.lo && !pv(kt - 1 == x.lo)) return;
    }
    if (!pv(x.m == x.lo)) return;                   // last tile's PV
    mma_commit(c.bar(B_OFULL0 + ob));
    ++uc;
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
    const uint32_t qb = qc & 1;
    if (!c.wait(B_QEMPTY0 + qb, ((qc >> 1) & 1) ^ 1)) return;
    ++qc;
    const uint32_t sQ = sQ0 + qb * kTileBytes;
    mbar_expect_tx(c.bar(B_QFULL0 + qb), kTileBytes);
    tma_load_3d(sQ, tmQ, c.bar(B_QFULL0 + qb), 0, x.m * 128, x.zq);
    tma_load_3d(sQ + kHalfBytes, tmQ, c.bar(B_QFULL0 + qb), 64, x.m * 128, x.zq);
    for (int kt = x.lo; kt <= x.m; ++kt) {
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
  float* inv_l = reinterpret_cast<float*>(smem + OFF_INVL);

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == B_PFULL0 || i == B_PFULL1 || i == B_LFULL0 || i == B_LFULL1 || i == B_OEMPTY0 ||
          i == B_OEMPTY1)
        cnt = 128;
      if (i == B_UEMPTY0 || i == B_UEMPTY1) cnt = 9;   // MMA thread + 4 softmax + 4 epilogue warps
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
      producer_role(p, c, &tmQ, &tmK, &tmV, sbase + OFF_Q, sbase + OFF_K, sbase + OFF_V);
    else if (warp == 1 && lane == 0)
      mma_role(p, c, tmem, sbase + OFF_Q, sbase + OFF_K, sbase + OFF_V);
  } else if (warp < 8) {
    regs_inc<kRegsSoftmax>();
    softmax_role(p, c, tmem, inv_l, warp, lane);
  } else {
    regs_dec<kRegsEpilogue>();
    epilogue_role(p, c, tmem, inv_l, warp, lane);
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

// Units of one 128-row query tile; a unit's cost is its number of key tiles.
std::vector<int32_t> prefill_units(int32_t B, int32_t Hq, int32_t N, const int32_t* spans) {
  const int64_t M = (N + kTileM - 1) / kTileM;      // query tiles
  struct U { int32_t b, h, m, lo; int64_t cost; };
  std::vector<U> v;
  v.reserve((size_t)B * Hq * M);
  for (int32_t b = 0; b < B; ++b)
    for (int32_t h = 0; h < Hq; ++h)
      for (int64_t m = 0; m < M; ++m) {
        const int64_t lo = first_tile_host(m, spans[h]);
        v.push_back({b, h, (int32_t)m, (int32_t)lo, m - lo + 1});
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
