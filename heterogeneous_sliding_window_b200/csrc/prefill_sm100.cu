// bf16 prefill for heterogeneous sliding windows on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes ("Mixture of Attention" project page, "Finding two" and
// the N x N causal-band figure; blog walkthrough section 2.1): for query row
// i of head h, softmax(scale * q_i . k_j) over the keys i - S_h < j <= i,
// applied to v_j.  Heads differ only in S_h.
//
// How (B200 design, not the pages' A100 kernel):
//  * Work unit = (b, h, m): query tiles A = m and B = m + 1 (128 rows each)
//    of one head.  Because the window is a band, tile A needs exactly the
//    key tiles loA..m and tile B the tiles loB..m+1
//    (lo = floor(max(0, 128t - S_h + 1) / 128) for query tile t); every other
//    key tile is skipped, and the two tiles share one stream of K and V tiles
//    loA..m+1.  A head with an odd number of query tiles ends with a unit
//    that has tile A only.
//  * Units are dealt on the host to one list per CTA of the persistent grid
//    (one CTA per SM), longest first, each to the list with the least work
//    so far, so heads with very different spans balance across SMs without
//    atomics and every CTA can read its next units ahead of time.
//  * Warp roles (384 threads, setmaxnreg split 120 / 192 / 192):
//      warp 0       TMA producer: the unit's two Q tiles into two rotating
//                   Q slots (the next unit's Q_A loads once this unit's A is
//                   done), K tiles through a three-stage ring and V tiles
//                   through a two-stage ring (128-byte swizzle).
//      warp 1       MMA issuer (one thread), tcgen05.mma M=128, N=128, K=16.
//                   Per key tile j:  O_A += P_A(j) V(j),  S_A(j+1) = Q_A K(j+1)^T,
//                   O_B += P_B(j) V(j),  S_B(j+1) = Q_B K(j+1)^T.
//                   The tensor core works on one tile's PV and next S while
//                   the other tile's softmax runs (ping-pong).  Each S-ready
//                   commit also covers that tile's previous PV.  In a unit's
//                   last key tile, where only tile B is left, the next unit's
//                   first S_A is issued, so tile A's softmax starts the next
//                   unit while tile B finishes this one.
//      warp 2       unit fetcher: this CTA's unit records into a four-slot
//                   ring in shared memory.
//      warp 3       cache writer (when the call fills a KV cache): copies the
//                   surviving key/value rows of its units into the ring
//                   cache, so the fill needs no launch of its own.
//      warps 4-7    softmax of tile A, warps 8-11 softmax of tile B: one
//                   thread per query row reads its S row in two 64-column
//                   halves, masks only tiles that cross the diagonal or the
//                   window's lower edge, takes exponentials against a
//                   per-row reference (see softmax_role), and writes P as
//                   bf16 pairs back over S; after the unit's last tile it
//                   reads O, releases the O buffer, and writes O / l as bf16
//                   (round to nearest even).
//    Tensor memory: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
//  * Rows >= N are dropped at the store; out-of-range TMA rows read as zeros.
//  * Every mbarrier wait is bounded (2 s of globaltimer, or earlier if another
//    role gave up); on a timeout the kernel sets the workspace error word,
//    lets every role leave, waits for its in-flight copies, frees TMEM and
//    returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <functional>
#include <memory>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace moa {
namespace {

using namespace sm100;

constexpr int kThreads = 384;                    // 3 warpgroups
// Register split (setmaxnreg): the block launches with 384 x 168 registers;
// warpgroup 0 (producer, MMA issuer, unit fetcher, cache writer) drops to
// 120, the two softmax warpgroups rise to 192.
constexpr uint32_t kRegsLaunch = 168, kRegsControl = 120, kRegsSoftmax = 192;
static_assert(128 * (kRegsControl + 2 * kRegsSoftmax) <= kThreads * kRegsLaunch, "register split");
constexpr int kD = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;   // one 128 x 128 bf16 tile
constexpr uint32_t kHalfBytes = 128 * 64 * 2;    // one 128-row x 128-byte swizzled half
// Shared memory carve-up (offsets from a 1024-byte aligned base).
// Ring depths (compile-time choices; shared memory holds seven 32 KB tiles).
// Two Q slots and three K stages measured best on the Vicuna-7B-shaped prompt
// (25 % density, with the early first S of tile B: 885 against 857 TFLOP/s
// back to back for three Q slots and two K stages, 839-846 against 772-826
// after an L2 flush).
#ifndef MOA_PREFILL_Q_SLOTS
#define MOA_PREFILL_Q_SLOTS 2
#endif
#ifndef MOA_PREFILL_K_STAGES
#define MOA_PREFILL_K_STAGES 3
#endif
#ifndef MOA_PREFILL_V_STAGES
#define MOA_PREFILL_V_STAGES 2
#endif
#ifndef MOA_PREFILL_EARLY_SB
#define MOA_PREFILL_EARLY_SB 1
#endif
constexpr bool kEarlySB = MOA_PREFILL_EARLY_SB != 0;   // tile B's first S issued in the unit's prologue
constexpr uint32_t kQSlots = MOA_PREFILL_Q_SLOTS;     // rotating Q tiles (two per unit)
constexpr uint32_t kKStages = MOA_PREFILL_K_STAGES, kVStages = MOA_PREFILL_V_STAGES;   // K and V ring depths
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + kQSlots * kTileBytes;
constexpr uint32_t OFF_V = OFF_K + kKStages * kTileBytes;
constexpr uint32_t OFF_BAR = OFF_V + kVStages * kTileBytes;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;          // + barriers + alignment slack

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;        // 2 s per wait

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);

// mbarrier slots (8 bytes each) at OFF_BAR; "X" slots come as (A, B) pairs.
enum {
  B_QFULL0 = 0, B_QEMPTY0 = B_QFULL0 + 3,
  B_SFULL0 = B_QEMPTY0 + 3, B_PFULL0 = B_SFULL0 + 2, B_OFULL0 = B_PFULL0 + 2,
  B_OEMPTY0 = B_OFULL0 + 2,
  B_UFULL0 = B_OEMPTY0 + 2, B_UEMPTY0 = B_UFULL0 + 4,
  B_KFULL0 = B_UEMPTY0 + 4, B_KEMPTY0 = B_KFULL0 + 4, B_VFULL0 = B_KEMPTY0 + 4, B_VEMPTY0 = B_VFULL0 + 4,
  B_COUNT = B_VEMPTY0 + 4
};
static_assert(kQSlots >= 2 && kQSlots <= 3 && kKStages >= 2 && kKStages <= 4 && kVStages >= 2 && kVStages <= 4,
              "ring depth");
constexpr uint32_t OFF_TMEM_SLOT = OFF_BAR + 8 * B_COUNT;        // uint32
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 4;                // int
constexpr uint32_t kUnitSlots = 4;                                // unit record ring depth
constexpr uint32_t OFF_UNIT = (OFF_ABORT + 4 + 15) / 16 * 16;    // int4[kUnitSlots] unit records
constexpr uint32_t OFF_KMIN = OFF_UNIT + 16 * kUnitSlots;         // int[kUnitSlots]: first valid key row
static_assert(OFF_KMIN + 4 * kUnitSlots <= OFF_BAR + 512, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// Position in a ring of `n` stages: stage index and mbarrier phase parity.
struct Ring {
  uint32_t stage = 0, phase = 0;
  __device__ void next(uint32_t n) {
    if (++stage == n) { stage = 0; phase ^= 1u; }
  }
};

struct PrefillParams {
  uint32_t* hdr;                 // [0] error word
  const int32_t* cta_off;        // units of CTA c: units[cta_off[c] .. cta_off[c+1])
  const int4* units;             // (b, h, m, loA), grouped by CTA, longest first within a CTA
  void* o;
  // Key rows 0 .. N-1; query row r is key position q_off + r (q_off a
  // multiple of 128), r < Nq.  A prompt has q_off = 0 and Nq = N.  A chunk
  // continuing sequence b (t != nullptr) sees key rows below q_off - t[b] as
  // positions before the sequence's start: they are masked.  Key rows below
  // q_off come from the window maps, rows q_off.. from the K/V maps at row
  // (key row - q_off).
  int32_t N, Nq, q_off;
  const int64_t* t;
  int32_t Hq, Hkv, G;
  int32_t stall;                 // self-test of the bounded waits: the fetcher publishes nothing
  int32_t o_wide;                // o is 32-byte aligned: output rows go out in 32-byte stores
  float scale_log2;
  int32_t span[MOA_MAX_HEADS];
  int32_t sink[MOA_MAX_HEADS];   // global tokens per head (keys j < sink[h] are kept too), 0: none
  // Cache fill (fill_data == nullptr: none).  Row r of k_rows / v_rows
  // [B, Hkv, Nq, d] is position t_b + r of sequence b; the last min(Nq, C_g)
  // rows go to ring slot (t_b + r) mod C_g of KV head g, and the last CTA to
  // finish advances every t_b by Nq.
  char* fill_data;               // cache data region
  uint32_t* fill_ctr;            // cache header: completion counter
  int64_t* fill_t;               // cache header: tokens per sequence
  const char* k_rows;
  const char* v_rows;
  int64_t fill_sumC;             // sum of the capacities (row pairs per sequence)
  int32_t B;
  int32_t fill_cap[MOA_MAX_HEADS];
  int64_t fill_goff[MOA_MAX_HEADS];
  // Global-token rows of the cache (fill_sink == nullptr: none): positions
  // below fill_scap[g] also go to row p of (b, g)'s block in this region.
  char* fill_sink;
  int64_t fill_sumK;             // sum of the global-token row counts
  int32_t fill_scap[MOA_MAX_HEADS];
};
// The five tensor maps (128 bytes each) and the parameters share the kernel
// parameter space (32764 bytes on sm_70 and later since CUDA 12.1).
static_assert(sizeof(PrefillParams) + 5 * 128 <= 32764, "kernel parameters");

struct Ctx {
  uint32_t bar0;                       // address of barrier 0
  volatile int* abort;
  volatile int4* ring;                 // published unit records, kUnitSlots slots (x < 0: no more units)
  volatile int* ring_kmin;             // per slot: the unit's first valid key row
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
  // One arrival per warp: every lane's prior accesses are ordered before
  // lane 0's arrive by __syncwarp.
  __device__ void arrive_warp(int i) const {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar(i));
  }
  // Next unit record from the ring.  Single-thread roles (warp_wide = false)
  // release the slot themselves; warp-wide roles release it from lane 0 after
  // every lane has read it.
  __device__ bool next_unit(uint32_t i, int lane, bool warp_wide, int4* u, int* kmin) const {
    const uint32_t slot = i % kUnitSlots, par = (i / kUnitSlots) & 1;
    if (warp_wide) {
      if (!wait_warp(B_UFULL0 + slot, par)) return false;
      *u = const_cast<const int4&>(ring[slot]);
      *kmin = ring_kmin[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_UEMPTY0 + slot));
    } else {
      if (!wait(B_UFULL0 + slot, par)) return false;
      *u = const_cast<const int4&>(ring[slot]);
      *kmin = ring_kmin[slot];
      mbar_arrive(bar(B_UEMPTY0 + slot));
    }
    return true;
  }
};

__device__ __forceinline__ int first_key_tile(int t, int S) {
  const long long f = (long long)t * 128 - S + 1;
  return f > 0 ? (int)(f / 128) : 0;
}

// The unit's two query tiles: X = 0 (A, tile m) and X = 1 (B, tile m + 1).
// Query tile X visits the key tiles [0, min(ks, lo[X])) that hold global
// tokens below its band, then its band [lo[X], m[X]].  The two tiles share
// one stream of key tiles: the global prefix [0, P) with P = min(ks, lo[B]),
// then [Lb, R] with Lb = max(lo[A], P).  Without global tokens (ks = 0) the
// stream is lo[A] .. R.  Every stream tile up to m[A] belongs to tile A;
// tile B skips the band tiles of A below lo[B].
struct UnitInfo {
  int S, k, zq, zk, kmin;
  int m[2], lo[2];
  bool hasB;
  int ks;                              // key tiles t < ks hold global tokens
  int P, Lb, R;                        // the shared key-tile stream (see above)
  int start;                           // its first key tile
  int first[2];                        // first key tile of each query tile
  __device__ bool in(int X, int j) const {
    return (X == 0 || hasB) && (j < ks || j >= lo[X]) && j <= m[X];
  }
  __device__ int next(int j) const { return j + 1 == P ? Lb : j + 1; }
};

__device__ __forceinline__ UnitInfo decode_unit(const PrefillParams& p, const int4 U, int kmin) {
  UnitInfo x;
  x.S = p.span[U.y];
  x.k = p.sink[U.y];
  x.zq = U.x * p.Hq + U.y;
  x.zk = U.x * p.Hkv + U.y / p.G;
  x.kmin = kmin;
  x.m[0] = U.z;
  x.lo[0] = max(U.w, kmin >> 7);
  x.m[1] = U.z + 1;
  x.hasB = (long long)x.m[1] * 128 < (long long)p.N;
  x.lo[1] = max(first_key_tile(x.m[1], x.S), kmin >> 7);
  x.R = x.hasB ? x.m[1] : x.m[0];
  x.ks = (int)(((long long)x.k + 127) >> 7);
  x.P = min(x.ks, x.hasB ? x.lo[1] : x.lo[0]);
  x.Lb = max(x.lo[0], x.P);
  x.first[0] = x.ks > 0 ? 0 : x.lo[0];
  x.first[1] = x.ks > 0 ? 0 : x.lo[1];
  x.start = x.first[0];
  return x;
}

// ---------------------------------------------------------------------------
// Softmax role: 128 threads own the 128 rows of query tile X of each unit.
//
// Each S tile is handled in two halves of 64 keys.  Exponentials are taken
// against a per-row reference m (log2 domain) without reducing the half
// first: the row's first half with in-window keys uses m = 0, later halves
// the current m.  Only when a half's sum of 2^(s - m) leaves [2^-15, 2^15)
// (a score more than 15 above m, or, for the first reference, every score far
// below 0) is the half's exact maximum taken, m moved there, the row sum, O
// and the first half's P rescaled, and the half redone.  Every exponential
// thus stays within 2^15 and the sum never underflows, and O / l does not
// depend on which m was used.  P of the whole tile is written over S only
// after both halves are done.
// ---------------------------------------------------------------------------
constexpr float kSumHi = 32768.f;                    // 2^15
constexpr float kSumLo = 1.f / 32768.f;              // 2^-15

// 64 scores of half hh (columns 64hh .. 64hh+63) from tensor memory, masked.
// Kept columns: lo_c < col <= hi_c (the band) and col < min(k_c, hi_c + 1)
// (global tokens).  Returns whether the half keeps any column.
__device__ __forceinline__ bool load_half(uint32_t tS, int hh, int hi_c, int lo_c, int k_c, bool edge,
                                          float* s) {
  uint32_t sr[64];
  tmem_ld64(tS + 64u * (uint32_t)hh, sr);
#pragma unroll
  for (int cc = 0; cc < 64; ++cc) s[cc] = __uint_as_float(sr[cc]);
  if (!edge) return true;
  // Bits of a 64-bit word built once per half, so each score costs one bit
  // test and one select rather than compares and a select (integer compares
  // and selects issue at half the rate of the FMA pipe).
  const int a = max(lo_c + 1 - 64 * hh, 0), b = min(hi_c - 64 * hh, 63);
  unsigned long long keep = a > b ? 0ull : ((~0ull) >> (63 - max(b, 0))) & ((~0ull) << min(a, 63));
  const int gb = min(min(k_c, hi_c + 1) - 1 - 64 * hh, 63);     // last global column of the half
  if (gb >= 0) keep |= (~0ull) >> (63 - gb);
  const uint32_t k0 = (uint32_t)keep, k1 = (uint32_t)(keep >> 32);
#pragma unroll
  for (int cc = 0; cc < 64; ++cc)
    if (!(((cc < 32 ? k0 : k1) >> (cc & 31)) & 1u)) s[cc] = -INFINITY;
  return keep != 0ull;
}

__device__ __forceinline__ float max64(const float* s) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
  for (int cc = 16; cc < 64; cc += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], s[cc + 2 * k], s[cc + 2 * k + 1]);
  return max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// Pairs of exponentials that may be taken by the cubic on the FMA pipe
// (exp2_poly2) rather than by MUFU ex2: one in kPolyEvery, none when 0.
// MUFU issues 16 ex2 per clock per SM, the tensor core's pace at d = 128, and
// with three Q slots and two-stage rings one pair in eight on the cubic paid.
// With two Q slots, a three-stage K ring and tile B's first S in the prologue
// the fewer the better: none measured 936 TFLOP/s against 922 for one pair in
// 32, 909 for two in 32 and 890 for four (25 % density, back to back), and
// 1004-1035 against 988-1000 for two in 32 at 50 %.
#ifndef MOA_PREFILL_POLY_EVERY
#define MOA_PREFILL_POLY_EVERY 0
#endif
constexpr int kPolyEvery = MOA_PREFILL_POLY_EVERY;
constexpr int kPolyMod = kPolyEvery > 0 ? kPolyEvery : 1;   // the modulus of the test below, never 0

// p = 2^(s * c - m) for 64 scores as bf16 pairs w[32]; returns the fp32 sum.
__device__ __forceinline__ float exp_half(const float* s, float c, float neg, uint32_t* w) {
  const uint64_t c2 = f2_pack(c, c), n2 = f2_pack(neg, neg);
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint64_t x2 = f2_fma(f2_pack(s[2 * j], s[2 * j + 1]), c2, n2);
    uint64_t p2;
    if (kPolyEvery > 0 && j % kPolyMod == kPolyMod - 1) {
      p2 = exp2_poly2(x2);
    } else {
      float x0, x1;
      f2_unpack(x2, x0, x1);
      p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
    }
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

// Output rows of one finished query tile (its uc-th): O / l -> bf16 (round to
// nearest even) -> global.  The O buffer is released as soon as it is in
// registers, so the next unit's PVs of this tile stream can start while the
// stores go out.  False when the wait for O gave up.
__device__ __forceinline__ bool write_o(const PrefillParams& p, const Ctx& c, uint32_t tO, int X, uint32_t uc,
                                        int zq, int i_row, float l_run) {
  if (!c.wait_warp(B_OFULL0 + X, uc & 1)) return false;
  tc_fence_after();
  const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
  uint32_t pk[64];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t rr[32];
    tmem_ld32(tO + cc * 32, rr);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      pk[16 * cc + j] = pack_bf16x2(__uint_as_float(rr[2 * j]) * inv, __uint_as_float(rr[2 * j + 1]) * inv);
  }
  tc_fence_before();
  c.arrive_warp(B_OEMPTY0 + X);
  const int o_row = i_row - p.q_off;
  if (o_row < p.Nq) {
    // Each thread writes its own 256-byte row, so one store instruction
    // touches 32 rows; 32-byte stores halve the instructions and write whole
    // sectors.
    __nv_bfloat16* orow_p = reinterpret_cast<__nv_bfloat16*>(p.o) + ((size_t)zq * p.Nq + (size_t)o_row) * kD;
    if (p.o_wide) {
#pragma unroll
      for (int j = 0; j < 8; ++j) st_global_v8(orow_p + 16 * j, pk + 8 * j);
    } else {
      uint4* orow = reinterpret_cast<uint4*>(orow_p);
#pragma unroll
      for (int j = 0; j < 16; ++j) orow[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    }
  }
  return true;
}

__device__ __forceinline__ void softmax_role(const PrefillParams& p, const Ctx& c, uint32_t tmem,
                                             int X, int warp, int lane) {
  const int quarter = warp & 3;                      // TMEM lane quarter this warp may access
  const int r = quarter * 32 + lane;                 // row within the query tile
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_base + kColS + 128u * (uint32_t)X;
  const uint32_t tO = tmem + lane_base + kColO + 128u * (uint32_t)X;
  const float sc = p.scale_log2;
  uint32_t tcount = 0, uc = 0;
  for (uint32_t i = 0;; ++i) {
    int4 U;
    int kmin;
    if (!c.next_unit(i, lane, true, &U, &kmin)) return;
    if (U.x < 0) return;
    const UnitInfo x = decode_unit(p, U, kmin);
    if (X == 1 && !x.hasB) continue;
    // this warpgroup's query tile and first key tile, selected rather than
    // indexed so the unit record stays in registers
    const int m_x = X ? x.m[1] : x.m[0];
    const int lo_x = X ? x.lo[1] : x.lo[0];
    const int s_x = min(x.ks, lo_x);                  // global tiles below the band: [0, s_x)
    const int first_x = s_x > 0 ? 0 : lo_x;
    const int i_row = m_x * 128 + r;
    float m_run = -INFINITY, l_run = 0.f;            // m_run = -inf: no reference yet
    for (int kt = first_x; kt <= m_x; kt = kt + 1 == s_x ? lo_x : kt + 1, ++tcount) {
      if (!c.wait_warp(B_SFULL0 + X, tcount & 1)) return;
      tc_fence_after();
      const int hi_c = i_row - kt * 128;             // keys c <= hi_c are causal
      const int lo_c = max(i_row - x.S, x.kmin - 1) - kt * 128;   // keys c > lo_c are inside the window
      const int k_c = x.k - kt * 128;                // keys c < k_c are global tokens
      // every column kept: causal, and band and global tokens cover the tile
      const bool full = hi_c >= 127 && (lo_c < 0 || k_c > lo_c || k_c >= 128);
      const bool edge = !full;
      uint32_t w[64];                                // P of the tile, bf16 pairs
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float s[64];
        const bool any_key = load_half(tS, hh, hi_c, lo_c, k_c, edge, s);
        const bool est = m_run != -INFINITY;
        float l_h = exp_half(s, sc, est ? -m_run : 0.f, w + 32 * hh);
        const bool bad = any_key && (!(l_h < kSumHi) || (!est && l_h < kSumLo));
        if (__any_sync(0xffffffffu, bad)) {
          // Rare: move the reference to this half's exact maximum.
          const float mt = max64(s) * sc;
          float alpha = 1.f;
          if (bad) {
            alpha = ex2_approx(m_run - mt);          // 0 when there was no reference
            m_run = mt;
            l_run *= alpha;
          }
          if (kt != first_x) {
            // O holds every PV of the earlier tiles (the S-ready commit of
            // this tile covered them).
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t rr[32];
              tmem_ld32(tO + cc * 32, rr);
#pragma unroll
              for (int j = 0; j < 32; ++j) rr[j] = __float_as_uint(__uint_as_float(rr[j]) * alpha);
              tmem_st32(tO + cc * 32, rr);
            }
          }
          if (hh == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j)             // P of the first half, still in registers
              w[j] = pack_bf16x2(__uint_as_float(w[j] << 16) * alpha,
                                 __uint_as_float(w[j] & 0xffff0000u) * alpha);
          }
          l_h = exp_half(s, sc, m_run == -INFINITY ? 0.f : -m_run, w + 32 * hh);
        }
        if (!est && any_key && !bad) m_run = 0.f;   // the first reference
        l_run += l_h;
      }
      tmem_st32(tS, w);
      tmem_st32(tS + 32, w + 32);
      tmem_st_wait();
      tc_fence_before();
      c.arrive_warp(B_PFULL0 + X);
    }
    if (!write_o(p, c, tO, X, uc++, x.zq, i_row, l_run)) return;
  }
}

// ---------------------------------------------------------------------------
// MMA role: one thread.  tcgen05.mma issue blocks for about the length of the
// MMA, so the tensor core idles whenever this thread is not issuing: the code
// between MMA groups is kept to scalar bookkeeping, descriptors are built from
// templates by adding the tile's address, and all per-stream state is scalar.
// ---------------------------------------------------------------------------
// Descriptor words (128-byte swizzle, 8-row groups 1024 B apart): K-major Q
// and K tiles (two 64-column halves 16 KB apart, K step = 32 B) and the
// MN-major V tile (8-key groups 1024 B apart, head-dim halves 16 KB apart).
constexpr uint32_t kDescHi = sw128_hi(1024u);
__device__ __forceinline__ uint32_t desc_qk_lo(uint32_t saddr) { return sw128_lo(saddr, 16u); }
__device__ __forceinline__ uint32_t desc_v_lo(uint32_t saddr) { return sw128_lo(saddr, kHalfBytes); }

// S = Q K^T for one 128-row query tile and one 128-key tile (8 K-steps of 16).
__device__ __forceinline__ void mma_qk(uint32_t tS, uint32_t q_lo, uint32_t k_lo, uint32_t hi) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((uint32_t)(kk >> 2) * kHalfBytes + (uint32_t)(kk & 3) * 32u) >> 4;
    mma_bf16_ss_lo(tS, q_lo + off, k_lo + off, hi, IDESC_QK, kk > 0 ? 1u : 0u);
  }
}
// O (+)= P V with P (bf16 pairs) in tensor memory, V MN-major in shared memory.
__device__ __forceinline__ void mma_pv(uint32_t tO, uint32_t tP, uint32_t v_lo, uint32_t hi, bool first) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_bf16_ts_lo(tO, tP + (uint32_t)kk * 8u, v_lo + (uint32_t)kk * (2048u >> 4), hi, IDESC_PV,
                   (!first || kk > 0) ? 1u : 0u);
}

// Q slots of a unit's two tiles (A then B), in the producer's order of loads.
struct QSlots {
  uint32_t sA, pA, sB, pB;
};
__device__ __forceinline__ QSlots take_q(const UnitInfo& x, uint32_t& nq) {
  QSlots q;
  q.sA = nq % kQSlots;
  q.pA = (nq / kQSlots) & 1;
  ++nq;
  q.sB = 0;
  q.pB = 0;
  if (x.hasB) {
    q.sB = nq % kQSlots;
    q.pB = (nq / kQSlots) & 1;
    ++nq;
  }
  return q;
}

__device__ __forceinline__ void mma_role(const PrefillParams& p, const Ctx& c, uint32_t tmem,
                                         uint32_t sQ0, uint32_t sK0, uint32_t sV0) {
  const uint32_t hi = kDescHi;
  const uint32_t tSA = tmem + kColS, tSB = tmem + kColS + 128u;
  const uint32_t tOA = tmem + kColO, tOB = tmem + kColO + 128u;
  uint32_t kst = 0, kph = 0, vst = 0, vph = 0;       // K and V ring positions
  uint32_t nq = 0;                                   // Q tiles used so far (slot nq % kQSlots)
  uint32_t tpA = 0, tpB = 0, ucA = 0, ucB = 0;       // PV tiles and units per stream
  uint32_t ui = 0;                                   // unit records read
  int4 U;
  int kmin;
  if (!c.next_unit(ui++, 0, false, &U, &kmin)) return;
  if (U.x < 0) return;
  UnitInfo x = decode_unit(p, U, kmin);
  QSlots q = take_q(x, nq);
  bool started_A = false;                            // S_A(start) of x already issued
  while (true) {
    bool qrB = false;
    // prologue: the S tiles of the stream's first key tile (tile A always
    // starts there; its S may have been issued during the previous unit's
    // last step)
    if (!c.wait(B_KFULL0 + kst, kph)) return;
    {
      const uint32_t dk = desc_qk_lo(sK0 + kst * kTileBytes);
      if (!started_A) {
        if (!c.wait(B_QFULL0 + q.sA, q.pA)) return;
        tc_fence_after();
        mma_qk(tSA, desc_qk_lo(sQ0 + q.sA * kTileBytes), dk, hi);
        mma_commit(c.bar(B_SFULL0));
        if (x.start == x.m[0]) mma_commit(c.bar(B_QEMPTY0 + q.sA));
      }
      if (x.in(1, x.start)) {
        if (!c.wait(B_QFULL0 + q.sB, q.pB)) return;
        qrB = true;
        tc_fence_after();
        mma_qk(tSB, desc_qk_lo(sQ0 + q.sB * kTileBytes), dk, hi);
        mma_commit(c.bar(B_SFULL0 + 1));
      }
    }
    mma_commit(c.bar(B_KEMPTY0 + kst));
    if (++kst == kKStages) { kst = 0; kph ^= 1u; }
    // When tile B starts one stream tile after tile A, its first S goes to
    // the tensor core now rather than after PV_A of the first tile, so B's
    // softmax can work while A's finishes the previous unit's epilogue.  The
    // ring's next K slot holds that tile; it is released in the loop as usual.
    bool sB_early = false;
    if (kEarlySB && x.hasB && x.start < x.R && !x.in(1, x.start) && x.first[1] == x.next(x.start)) {
      if (!c.wait(B_KFULL0 + kst, kph)) return;
      if (!c.wait(B_QFULL0 + q.sB, q.pB)) return;
      qrB = true;
      tc_fence_after();
      mma_qk(tSB, desc_qk_lo(sQ0 + q.sB * kTileBytes), desc_qk_lo(sK0 + kst * kTileBytes), hi);
      mma_commit(c.bar(B_SFULL0 + 1));
      if (x.first[1] == x.m[1]) mma_commit(c.bar(B_QEMPTY0 + q.sB));
      sB_early = true;
    }
    // next unit, when its tile A could start during this unit's last step
    bool have_next = false, ended = false;
    int4 Uy = make_int4(0, 0, 0, 0);
    int ykmin = 0;
    uint32_t ysA = 0, ypA = 0;
    for (int j = x.start;; ) {
      const bool more = j < x.R;
      const int jn = x.next(j);                      // the stream's next key tile, when more
      if (!c.wait(B_VFULL0 + vst, vph)) return;
      const uint32_t dv = desc_v_lo(sV0 + vst * kTileBytes);
      const uint32_t dk = desc_qk_lo(sK0 + kst * kTileBytes);   // K(jn) when more
      if (more && !c.wait(B_KFULL0 + kst, kph)) return;
      // stream A: O_A += P_A(j) V(j), then S_A(jn)
      if (j <= x.m[0]) {
        if (!c.wait(B_PFULL0, tpA & 1)) return;
        const bool first = j == x.first[0];
        if (first && !c.wait(B_OEMPTY0, (ucA & 1) ^ 1)) return;
        tc_fence_after();
        mma_pv(tOA, tSA, dv, hi, first);
        ++tpA;
        if (j == x.m[0]) {
          mma_commit(c.bar(B_OFULL0));
          ++ucA;
        } else {
          mma_qk(tSA, desc_qk_lo(sQ0 + q.sA * kTileBytes), dk, hi);   // jn <= m_A, so more
          mma_commit(c.bar(B_SFULL0));               // also covers PV_A(j)
          if (jn == x.m[0]) mma_commit(c.bar(B_QEMPTY0 + q.sA));
        }
      } else if (!more) {
        // Last step, tile B only: S_A of the next unit's first key tile (the
        // next K in the ring) goes to the tensor core now, so tile A's
        // softmax starts the next unit while tile B finishes this one.
        if (!c.next_unit(ui++, 0, false, &Uy, &ykmin)) return;
        if (Uy.x < 0) {
          ended = true;
        } else {
          // tile A of the next unit: query tile Uy.z, first key tile
          // max(Uy.w, ykmin / 128); its Q slot is the next in the rotation
          ysA = nq % kQSlots;
          ypA = (nq / kQSlots) & 1;
          if (!c.wait(B_KFULL0 + kst, kph)) return;
          if (!c.wait(B_QFULL0 + ysA, ypA)) return;
          tc_fence_after();
          mma_qk(tSA, desc_qk_lo(sQ0 + ysA * kTileBytes), desc_qk_lo(sK0 + kst * kTileBytes), hi);
          mma_commit(c.bar(B_SFULL0));
          const UnitInfo y = decode_unit(p, Uy, ykmin);
          if (y.start == y.m[0]) mma_commit(c.bar(B_QEMPTY0 + ysA));
          have_next = true;
        }
      }
      // stream B: O_B += P_B(j) V(j), then S_B(jn)
      if (x.hasB) {
        if (x.in(1, j)) {
          if (!c.wait(B_PFULL0 + 1, tpB & 1)) return;
          const bool first = j == x.first[1];
          if (first && !c.wait(B_OEMPTY0 + 1, (ucB & 1) ^ 1)) return;
          tc_fence_after();
          mma_pv(tOB, tSB, dv, hi, first);
          ++tpB;
          if (j == x.m[1]) {
            mma_commit(c.bar(B_OFULL0 + 1));
            ++ucB;
          }
        }
        if (more && x.in(1, jn) && !(sB_early && j == x.start)) {
          if (!qrB) {
            if (!c.wait(B_QFULL0 + q.sB, q.pB)) return;
            qrB = true;
            tc_fence_after();
          }
          mma_qk(tSB, desc_qk_lo(sQ0 + q.sB * kTileBytes), dk, hi);
          mma_commit(c.bar(B_SFULL0 + 1));
          if (jn == x.m[1]) mma_commit(c.bar(B_QEMPTY0 + q.sB));
        }
      }
      mma_commit(c.bar(B_VEMPTY0 + vst));
      if (++vst == kVStages) { vst = 0; vph ^= 1u; }
      if (!more) break;
      mma_commit(c.bar(B_KEMPTY0 + kst));
      if (++kst == kKStages) { kst = 0; kph ^= 1u; }
      j = jn;
    }
    if (ended) return;
    if (have_next) {
      x = decode_unit(p, Uy, ykmin);
      q = take_q(x, nq);                             // slot of tile A = ysA
      started_A = true;
      continue;
    }
    if (!c.next_unit(ui++, 0, false, &U, &kmin)) return;
    if (U.x < 0) return;
    x = decode_unit(p, U, kmin);
    q = take_q(x, nq);
    started_A = false;
  }
}

// ---------------------------------------------------------------------------
// Producer role: one thread (unit fetch + TMA).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void producer_role(const PrefillParams& p, const Ctx& c,
                                              const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                              const CUtensorMap* tmV, const CUtensorMap* tmKw,
                                              const CUtensorMap* tmVw, uint32_t sQ0, uint32_t sK0,
                                              uint32_t sV0) {
  Ring kr, vr;
  uint32_t nq = 0;
  auto load_q = [&](int m, int zq) -> bool {
    const uint32_t slot = nq % kQSlots, par = (nq / kQSlots) & 1;
    ++nq;
    if (!c.wait(B_QEMPTY0 + slot, par ^ 1)) return false;
    const uint32_t sQ = sQ0 + slot * kTileBytes;
    mbar_expect_tx(c.bar(B_QFULL0 + slot), kTileBytes);
    tma_load_3d(sQ, tmQ, c.bar(B_QFULL0 + slot), 0, m * 128 - p.q_off, zq);
    tma_load_3d(sQ + kHalfBytes, tmQ, c.bar(B_QFULL0 + slot), 64, m * 128 - p.q_off, zq);
    return true;
  };
  auto load_k = [&](int kt, int zk) -> bool {
    const uint32_t ks = kr.stage;
    if (!c.wait(B_KEMPTY0 + ks, kr.phase ^ 1)) return false;
    kr.next(kKStages);
    mbar_expect_tx(c.bar(B_KFULL0 + ks), kTileBytes);
    const bool win = kt * 128 < p.q_off;
    const CUtensorMap* mk = win ? tmKw : tmK;
    const int row = win ? kt * 128 : kt * 128 - p.q_off;
    tma_load_3d(sK0 + ks * kTileBytes, mk, c.bar(B_KFULL0 + ks), 0, row, zk);
    tma_load_3d(sK0 + ks * kTileBytes + kHalfBytes, mk, c.bar(B_KFULL0 + ks), 64, row, zk);
    return true;
  };
  auto load_v = [&](int kt, int zk) -> bool {
    const uint32_t vs = vr.stage;
    if (!c.wait(B_VEMPTY0 + vs, vr.phase ^ 1)) return false;
    vr.next(kVStages);
    mbar_expect_tx(c.bar(B_VFULL0 + vs), kTileBytes);
    const bool win = kt * 128 < p.q_off;
    const CUtensorMap* mv = win ? tmVw : tmV;
    const int row = win ? kt * 128 : kt * 128 - p.q_off;
    tma_load_3d(sV0 + vs * kTileBytes, mv, c.bar(B_VFULL0 + vs), 0, row, zk);
    tma_load_3d(sV0 + vs * kTileBytes + kHalfBytes, mv, c.bar(B_VFULL0 + vs), 64, row, zk);
    return true;
  };
  for (uint32_t i = 0;; ++i) {
    int4 U;
    int kmin;
    if (!c.next_unit(i, 0, false, &U, &kmin)) return;
    if (U.x < 0) return;
    const UnitInfo x = decode_unit(p, U, kmin);
    // Loads in the MMA's order of use: Q_A, K(start), then per key tile j
    // of the stream: V(j), K(next); Q_B right before the first K tile that
    // tile B uses.
    if (!load_q(x.m[0], x.zq)) return;
    if (!load_k(x.start, x.zk)) return;
    if (x.hasB && x.first[1] == x.start && !load_q(x.m[1], x.zq)) return;
    for (int j = x.start;; j = x.next(j)) {
      if (!load_v(j, x.zk)) return;
      if (j >= x.R) break;
      const int jn = x.next(j);
      if (x.hasB && x.first[1] == jn && !load_q(x.m[1], x.zq)) return;
      if (!load_k(jn, x.zk)) return;
    }
  }
}

// ---------------------------------------------------------------------------
// Unit fetcher: one thread publishes the records of this CTA's units (a
// balanced list built on the host) up to kUnitSlots ahead of the slowest
// consumer, then a record with x < 0; no role waits on a global load.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fetcher_role(const PrefillParams& p, const Ctx& c) {
  if (p.stall) return;           // every other role's first wait runs out
  const int first = p.cta_off[blockIdx.x], last = p.cta_off[blockIdx.x + 1];
  for (uint32_t i = 0;; ++i) {
    const uint32_t slot = i % kUnitSlots;
    if (!c.wait(B_UEMPTY0 + slot, ((i / kUnitSlots) & 1) ^ 1)) return;
    const int u = first + (int)i;
    const int4 U = u < last ? p.units[u] : make_int4(-1, 0, 0, 0);
    int kmin = 0;
    if (p.t != nullptr && U.x >= 0) {
      const long long f = (long long)p.q_off - p.t[U.x];
      kmin = f > 0 ? (int)f : 0;
    }
    const_cast<int4&>(c.ring[slot]) = U;
    c.ring_kmin[slot] = kmin;
    mbar_arrive(c.bar(B_UFULL0 + slot));
    if (U.x < 0) return;
  }
}

// ---------------------------------------------------------------------------
// Cache writer (warp 3, all lanes): for each unit of this CTA whose head is
// the first of its KV group, copies the surviving key and value rows of the
// unit's query tiles from k_rows / v_rows into the ring.  Each KV group's rows
// are thus written exactly once.  The attention never reads the ring (its
// keys come from k, v and the gathered window), so the copies need no
// ordering with the other roles; only the position update waits for the
// whole grid (see the end of the kernel).  Rows are 256 bytes (d = 128,
// bf16): 16 lanes per row, two rows per load, eight rows per pass.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fill_role(const PrefillParams& p, int lane) {
  constexpr int kRowBytes = kD * 2;
  const int first = p.cta_off[blockIdx.x], last = p.cta_off[blockIdx.x + 1];
  const int half = lane >> 4;                        // which of two rows
  const size_t col = (size_t)(lane & 15) * 16;       // byte offset within the row
  for (int u = first; u < last; ++u) {
    const int4 U = p.units[u];
    if (U.y % p.G != 0) continue;
    const int g = U.y / p.G;
    const int C = p.fill_cap[g];
    const int q0 = U.z * 128 - p.q_off;              // the unit's first query row
    if (p.fill_sink != nullptr && p.fill_scap[g] > 0) {
      // global-token rows: positions t_b + r below K_g, at row t_b + r of (b, g)'s block
      const int64_t tb = p.fill_t[U.x];
      const int Kg = p.fill_scap[g];
      const int g_end = (int)min((int64_t)min(q0 + 256, p.Nq), (int64_t)Kg - tb);
      int64_t soff = 0;
      for (int gg = 0; gg < g; ++gg) soff += p.fill_scap[gg];
      char* ks = p.fill_sink + (size_t)((int64_t)U.x * p.fill_sumK + soff) * 2 * kRowBytes;
      char* vs = ks + (size_t)Kg * kRowBytes;
      const size_t src0 = ((size_t)U.x * p.Hkv + g) * (size_t)p.Nq;
      for (int r = q0 + half; r < g_end; r += 2) {
        const size_t src = (src0 + r) * kRowBytes + col;
        const size_t dst = (size_t)(tb + r) * kRowBytes + col;
        *reinterpret_cast<int4*>(ks + dst) = __ldg(reinterpret_cast<const int4*>(p.k_rows + src));
        *reinterpret_cast<int4*>(vs + dst) = __ldg(reinterpret_cast<const int4*>(p.v_rows + src));
      }
    }
    const int r_first = max(q0, p.Nq - C);           // rows below Nq - C are overwritten later
    const int r_end = min(q0 + 256, p.Nq);
    if (r_first >= r_end) continue;
    // r_end - r_first <= C, so slot0 + (r - r_first) wraps at most once
    const int slot0 = (int)((p.fill_t[U.x] + r_first) % C);
    char* kring = p.fill_data + (size_t)((int64_t)U.x * p.fill_sumC + p.fill_goff[g]) * 2 * kRowBytes;
    char* vring = kring + (size_t)C * kRowBytes;
    const size_t src0 = ((size_t)U.x * p.Hkv + g) * (size_t)p.Nq;
    for (int r0 = r_first; r0 < r_end; r0 += 8) {
      int4 kx[4], vx[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + 2 * j + half;
        if (r < r_end) {
          const size_t src = (src0 + r) * kRowBytes + col;
          kx[j] = __ldg(reinterpret_cast<const int4*>(p.k_rows + src));
          vx[j] = __ldg(reinterpret_cast<const int4*>(p.v_rows + src));
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + 2 * j + half;
        if (r < r_end) {
          int slot = slot0 + (r - r_first);
          if (slot >= C) slot -= C;
          const size_t dst = (size_t)slot * kRowBytes + col;
          *reinterpret_cast<int4*>(kring + dst) = kx[j];
          *reinterpret_cast<int4*>(vring + dst) = vx[j];
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmKw,
                          const __grid_constant__ CUtensorMap tmVw,
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
  c.ring = reinterpret_cast<volatile int4*>(smem + OFF_UNIT);
  c.ring_kmin = reinterpret_cast<volatile int*>(smem + OFF_KMIN);
  c.hdr = p.hdr;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if ((i >= B_PFULL0 && i < B_PFULL0 + 2) || (i >= B_OEMPTY0 && i < B_OEMPTY0 + 2))
        cnt = 4;                                        // one arrival per warp of a warpgroup
      if (i >= B_UEMPTY0 && i < B_UEMPTY0 + (int)kUnitSlots) cnt = 10;   // producer, MMA, 2 x 4 softmax warps
      mbar_init(c.bar(i), cnt);
    }
    *c.abort = 0;
    mbar_fence_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (p.q_off > 0) {
      prefetch_tmap(&tmKw);
      prefetch_tmap(&tmVw);
    }
  }
  if (warp == 0) tmem_alloc(smem_addr((const void*)tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    if constexpr (kRegsControl < kRegsLaunch) regs_dec<kRegsControl>();
    if (warp == 0 && lane == 0)
      producer_role(p, c, &tmQ, &tmK, &tmV, &tmKw, &tmVw, sbase + OFF_Q, sbase + OFF_K, sbase + OFF_V);
    else if (warp == 2 && lane == 0)
      fetcher_role(p, c);
    else if (warp == 1 && lane == 0)
      mma_role(p, c, tmem, sbase + OFF_Q, sbase + OFF_K, sbase + OFF_V);
    else if (warp == 3 && p.fill_data != nullptr)
      fill_role(p, lane);
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
  // Cache fill: the last CTA to finish advances the positions.  Every CTA's
  // fetcher and cache writer read t before the barrier above, so none of
  // them can see the new value.
  if (p.fill_data != nullptr && tid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(p.fill_ctr, 1u);
    if (prev == gridDim.x - 1) {
      for (int b = 0; b < p.B; ++b) p.fill_t[b] += p.Nq;
      *p.fill_ctr = 0u;
      __threadfence();
    }
  }
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

constexpr size_t kOffsOffset = 256;                          // int32 cta_off[kMaxCtas + 1]
constexpr size_t kUnitsOffset = kOffsOffset + (4 * (kPrefillMaxCtas + 1) + 15) / 16 * 16;
constexpr int64_t kUnitOverheadTiles = 4;     // per-unit pipeline fill/drain, in tile steps

int64_t first_tile_host(int64_t qt, int32_t S) {
  return std::max<int64_t>(0, qt * kTileM - S + 1) / kTileN;
}

}  // namespace

// Units of two consecutive 128-row query tiles (m, m + 1) of one head, sorted
// longest first and dealt to n_ctas lists by the greedy longest-processing-
// time rule (each unit to the list with the least work so far); a unit's work
// is its (query tile, key tile) pairs plus a fixed per-unit overhead.
PrefillSchedule prefill_schedule(int32_t B, int32_t Hq, int32_t N, const int32_t* spans, int32_t n_ctas,
                                 int32_t m0, const int32_t* sinks) {
  const int64_t M = ((int64_t)N + kTileM - 1) / kTileM;   // key tiles; query tiles are m0 .. M-1
  const int64_t per_head = std::max<int64_t>(0, (M - m0 + 1) / 2);
  const int64_t n_units = (int64_t)B * Hq * per_head;
  // unit u = (b * Hq + h) * per_head + k covers query tiles m0 + 2k and m0 + 2k + 1
  std::vector<int32_t> lo((size_t)n_units), cost((size_t)n_units);
  int32_t max_cost = 0;
  for (int32_t h = 0; h < Hq; ++h)
    for (int64_t k = 0; k < per_head; ++k) {
      const int64_t m = m0 + 2 * k;
      const int64_t l = first_tile_host(m, spans[h]);
      // key tiles below the band that hold global tokens
      const int64_t ks = sinks ? ((int64_t)sinks[h] + kTileN - 1) / kTileN : 0;
      int64_t c = m - l + 1 + std::min(ks, l) + kUnitOverheadTiles;
      if (m + 1 < M) {
        const int64_t lb = first_tile_host(m + 1, spans[h]);
        c += m + 1 - lb + 1 + std::min(ks, lb);
      }
      for (int32_t b = 0; b < B; ++b) {
        const size_t u = (size_t)(((int64_t)b * Hq + h) * per_head + k);
        lo[u] = (int32_t)l;
        cost[u] = (int32_t)c;
      }
      max_cost = std::max(max_cost, (int32_t)c);
    }
  // Longest first, equal costs in unit order: a stable counting sort.
  std::vector<int32_t> start((size_t)max_cost + 2, 0);
  for (int64_t u = 0; u < n_units; ++u) ++start[(size_t)(max_cost - cost[u]) + 1];
  for (size_t i = 1; i < start.size(); ++i) start[i] += start[i - 1];
  std::vector<int32_t> order((size_t)n_units);
  for (int64_t u = 0; u < n_units; ++u) order[(size_t)start[(size_t)(max_cost - cost[u])]++] = (int32_t)u;
  // Greedy LPT: each unit to the list with the least work so far (ties: the
  // lowest list).  A binary min-heap of keys work * 2^11 + list: keys are
  // distinct, so the minimum, and with it the schedule, does not depend on
  // how the heap is arranged.  The chosen list's work only grows, so its key
  // is sifted down from the root.
  static_assert(kPrefillMaxCtas <= 2048, "list index field");
  const int32_t n = (int32_t)std::max<int64_t>(1, std::min<int64_t>(n_ctas, n_units));
  std::vector<uint64_t> heap((size_t)n);
  for (int32_t c = 0; c < n; ++c) heap[(size_t)c] = (uint64_t)c;   // work 0, ascending lists: a heap
  std::vector<int32_t> list_of((size_t)n_units);
  PrefillSchedule out;
  out.n_ctas = n;
  out.off.assign((size_t)n + 1, 0);
  for (int64_t i = 0; i < n_units; ++i) {
    const uint64_t top = heap[0];
    const int32_t list = (int32_t)(top & 2047u);
    list_of[(size_t)i] = list;
    ++out.off[(size_t)list + 1];
    const uint64_t key = top + ((uint64_t)cost[(size_t)order[(size_t)i]] << 11);
    size_t pos = 0;
    for (;;) {
      size_t child = 2 * pos + 1;
      if (child >= (size_t)n) break;
      if (child + 1 < (size_t)n && heap[child + 1] < heap[child]) ++child;
      if (heap[child] >= key) break;
      heap[pos] = heap[child];
      pos = child;
    }
    heap[pos] = key;
  }
  for (int32_t c = 0; c < n; ++c) out.off[(size_t)c + 1] += out.off[(size_t)c];
  // Each list in the order its units were dealt (longest first).
  out.units.assign((size_t)n_units * 4, 0);
  std::vector<int32_t> fill(out.off.begin(), out.off.end() - 1);
  for (int64_t i = 0; i < n_units; ++i) {
    const int32_t u = order[(size_t)i];
    const int32_t bh = (int32_t)(u / per_head), k = (int32_t)(u % per_head);
    int32_t* dst = &out.units[(size_t)fill[(size_t)list_of[(size_t)i]]++ * 4];
    dst[0] = bh / Hq;
    dst[1] = bh % Hq;
    dst[2] = m0 + 2 * k;
    dst[3] = lo[(size_t)u];
  }
  return out;
}

// One row (CTA, unit, b, h, query tile, first key tile, last key tile) per
// query tile, in the order each CTA takes its units.
std::vector<int32_t> prefill_schedule_rows(int32_t B, int32_t Hq, int32_t N, const int32_t* spans,
                                           int32_t n_ctas) {
  const int64_t M = ((int64_t)N + kTileM - 1) / kTileM;
  const PrefillSchedule sch = prefill_schedule(B, Hq, N, spans, n_ctas);
  std::vector<int32_t> rows;
  rows.reserve((size_t)B * Hq * M * 7);
  for (int32_t c = 0; c < sch.n_ctas; ++c)
    for (int32_t i = sch.off[c]; i < sch.off[c + 1]; ++i) {
      const int32_t b = sch.units[4 * i], h = sch.units[4 * i + 1], m = sch.units[4 * i + 2];
      for (int32_t t = m; t <= m + 1 && t < M; ++t) {
        const int32_t row[7] = {c, i, b, h, t, (int32_t)first_tile_host(t, spans[h]), t};
        rows.insert(rows.end(), row, row + 7);
      }
    }
  return rows;
}

size_t prefill_workspace_bytes(int32_t B, int32_t Hq, int64_t N) {
  const int64_t M = ((int64_t)N + kTileM - 1) / kTileM;
  return kUnitsOffset + (size_t)B * Hq * M * 16;
}

namespace {

// The workspace image of a schedule: zeroed header, per-CTA list offsets and
// the units, uploaded in one copy.  The schedule depends only on the shapes,
// the spans and the grid, so the last few images are kept and a call with the
// same arguments (every layer of a model, every step of a server) reuses one
// instead of rebuilding it.
struct UnitBlob {
  int32_t n_ctas = 0;
  std::vector<int32_t> words;
};

struct BlobKey {
  int32_t B, Hq, N, grid, m0;
  std::vector<int32_t> spans, sinks;
  bool operator==(const BlobKey& o) const {
    return B == o.B && Hq == o.Hq && N == o.N && grid == o.grid && m0 == o.m0 && spans == o.spans &&
           sinks == o.sinks;
  }
};

std::shared_ptr<const UnitBlob> unit_blob(int32_t B, int32_t Hq, int32_t N, const int32_t* spans, int32_t grid,
                                          int32_t m0, const int32_t* sinks) {
  constexpr size_t kKept = 8;
  static std::mutex mu;
  static std::vector<std::pair<BlobKey, std::shared_ptr<const UnitBlob>>> kept;   // most recent first
  BlobKey key{B, Hq, N, grid, m0, std::vector<int32_t>(spans, spans + Hq),
              sinks ? std::vector<int32_t>(sinks, sinks + Hq) : std::vector<int32_t>()};
  {
    std::lock_guard<std::mutex> lock(mu);
    for (size_t i = 0; i < kept.size(); ++i)
      if (kept[i].first == key) {
        std::rotate(kept.begin(), kept.begin() + (long)i, kept.begin() + (long)i + 1);
        return kept[0].second;
      }
  }
  const PrefillSchedule sch = prefill_schedule(B, Hq, N, spans, grid, m0, sinks);
  auto blob = std::make_shared<UnitBlob>();
  blob->n_ctas = sch.n_ctas;
  blob->words.assign(kUnitsOffset / 4 + sch.units.size(), 0);
  std::copy(sch.off.begin(), sch.off.end(), blob->words.begin() + kOffsOffset / 4);
  std::copy(sch.units.begin(), sch.units.end(), blob->words.begin() + kUnitsOffset / 4);
  std::lock_guard<std::mutex> lock(mu);
  kept.insert(kept.begin(), {std::move(key), blob});
  if (kept.size() > kKept) kept.pop_back();
  return blob;
}

// Query rows 0 .. Nq-1 are key positions q_off .. q_off+Nq-1 (q_off a
// multiple of 128).  Key rows q_off .. q_off+Nq-1 are k, v [B, Hkv, Nq, d];
// rows 0 .. q_off-1 are kw, vw [B, Hkv, q_off, d].  t: per-sequence token
// counts of a chunk (rows below q_off - t[b] masked), or nullptr for a prompt
// (q_off = 0).
moa_status launch_prefill_bf16_rows(const void* q, const void* k, const void* v, const void* kw,
                                    const void* vw, void* o, int32_t B, int32_t Hq, int32_t Hkv, int32_t Nq,
                                    int32_t q_off, const int64_t* t, const int32_t* spans, float scale,
                                    void* ws, size_t ws_bytes, cudaStream_t s, moa_kv_cache* fill = nullptr,
                                    bool stall = false,
                                    const std::function<moa_status()>& before = nullptr,
                                    const int32_t* sinks = nullptr) {
  if (ws_bytes < prefill_workspace_bytes(B, Hq, Nq)) return MOA_ERR_WORKSPACE;
  if ((int64_t)B * Hq > INT32_MAX || (int64_t)B * Hkv > INT32_MAX) return MOA_ERR_UNSUPPORTED;
  const int32_t Nk = q_off + Nq;
  CUtensorMap mq, mk, mv, mkw, mvw;
  if (!make_map(&mq, q, Nq, (int64_t)B * Hq) || !make_map(&mk, k, Nq, (int64_t)B * Hkv) ||
      !make_map(&mv, v, Nq, (int64_t)B * Hkv))
    return cuda_fail(cudaErrorInvalidValue, "tensor map encode");
  if (q_off > 0) {
    if (!make_map(&mkw, kw, q_off, (int64_t)B * Hkv) || !make_map(&mvw, vw, q_off, (int64_t)B * Hkv))
      return cuda_fail(cudaErrorInvalidValue, "tensor map encode");
  } else {
    mkw = mk;                                      // never read: no key row lies below q_off
    mvw = mv;
  }
  // Header (error word, zeroed), the per-CTA list offsets and the units,
  // uploaded in one copy.  The pageable source is staged by the runtime
  // before cudaMemcpyAsync returns.
  const int32_t m0 = q_off / kTileM;
  const int64_t Mq = ((int64_t)Nq + kTileM - 1) / kTileM;
  const int64_t n_units = (int64_t)B * Hq * ((Mq + 1) / 2);
  const int32_t grid = (int32_t)std::min<int64_t>({n_units, (int64_t)sm_count(), (int64_t)kPrefillMaxCtas});
  const std::shared_ptr<const UnitBlob> sch = unit_blob(B, Hq, Nk, spans, grid, m0, sinks);
  const std::vector<int32_t>& blob = sch->words;

  PrefillParams p;
  p.hdr = reinterpret_cast<uint32_t*>(ws);
  p.cta_off = reinterpret_cast<const int32_t*>((char*)ws + kOffsOffset);
  p.units = reinterpret_cast<const int4*>((char*)ws + kUnitsOffset);
  p.o = o;
  p.o_wide = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;
  p.N = Nk;
  p.Nq = Nq;
  p.q_off = q_off;
  p.t = t;
  p.stall = stall ? 1 : 0;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  for (int h = 0; h < Hq; ++h) {
    p.span[h] = spans[h];
    p.sink[h] = sinks ? sinks[h] : 0;
  }
  p.B = B;
  p.fill_data = nullptr;
  p.fill_ctr = nullptr;
  p.fill_t = nullptr;
  p.k_rows = static_cast<const char*>(k);
  p.v_rows = static_cast<const char*>(v);
  p.fill_sumC = 0;
  p.fill_sink = nullptr;
  p.fill_sumK = 0;
  if (fill != nullptr) {
    if (fill->B != B || fill->Hkv != Hkv || fill->d != kD || fill->dtype != MOA_BF16) return MOA_ERR_INVALID_ARG;
    p.fill_data = fill->buf + fill->header;
    p.fill_ctr = reinterpret_cast<uint32_t*>(fill->buf + kHdrAppendCtr);
    p.fill_t = reinterpret_cast<int64_t*>(fill->buf + kHdrT);
    p.fill_sumC = fill->goff[Hkv];
    for (int g = 0; g < Hkv; ++g) {
      p.fill_cap[g] = fill->cap[g];
      p.fill_goff[g] = fill->goff[g];
      p.fill_scap[g] = fill->scap[g];
    }
    p.fill_sink = sink_region(fill);
    p.fill_sumK = fill->soff[Hkv];
  }

  static unsigned long long attr_done = 0;
  const cudaError_t attr_err =
      ensure_smem_attr(reinterpret_cast<const void*>(prefill_bf16_sm100_kernel), (int)SMEM_BYTES, &attr_done);
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "prefill smem attribute");
  // All host work is done: whatever must run first on the stream (the chunk's
  // window gather) goes in now, so the kernels follow one another without the
  // device waiting on the host.
  if (before) {
    const moa_status st = before();
    if (st != MOA_OK) return st;
  }
  const cudaError_t e = cudaMemcpyAsync(ws, blob.data(), blob.size() * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill unit upload");
  prefill_bf16_sm100_kernel<<<sch->n_ctas, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, mkw, mvw, p);
  return check_launch("prefill_bf16 launch");
}

// Chunk workspace: the prefill schedule region, then the gathered window
// key and value rows [B, Hkv, W, d] (W = prior keys any query can reach,
// rounded up to a tile).
struct ChunkLayout {
  int32_t W = 0;
  size_t off_k = 0, off_v = 0, bytes = 0;
};

ChunkLayout chunk_layout(int32_t B, int32_t Hq, int32_t Hkv, int32_t n, const int32_t* spans) {
  ChunkLayout L;
  int32_t max_s = 1;
  for (int h = 0; h < Hq; ++h) max_s = std::max(max_s, spans[h]);
  L.W = (max_s - 1 + kTileN - 1) / kTileN * kTileN;
  const size_t rows = (size_t)B * Hkv * (size_t)L.W * kD * 2;
  L.off_k = (prefill_workspace_bytes(B, Hq, n) + 255) / 256 * 256;
  L.off_v = L.off_k + (rows + 255) / 256 * 256;
  L.bytes = L.off_v + rows;
  return L;
}

}  // namespace

moa_status launch_prefill_bf16(const void* q, const void* k, const void* v, void* o, int32_t B,
                               int32_t Hq, int32_t Hkv, int32_t N, const int32_t* spans, float scale,
                               void* ws, size_t ws_bytes, cudaStream_t s, moa_kv_cache* fill,
                               const int32_t* sinks) {
  return launch_prefill_bf16_rows(q, k, v, nullptr, nullptr, o, B, Hq, Hkv, N, 0, nullptr, spans, scale, ws,
                                  ws_bytes, s, fill, false, nullptr, sinks);
}

moa_status launch_prefill_stall_test(const void* q, const void* k, const void* v, void* o, void* ws,
                                     size_t ws_bytes, cudaStream_t s) {
  const int32_t span = 128;
  return launch_prefill_bf16_rows(q, k, v, nullptr, nullptr, o, 1, 1, 1, 128, 0, nullptr, &span, 0.088f, ws,
                                  ws_bytes, s, nullptr, true);
}

size_t prefill_chunk_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t n, const int32_t* spans) {
  return chunk_layout(B, Hq, Hkv, n, spans).bytes;
}

moa_status launch_prefill_chunk(moa_kv_cache* c, const void* q, const void* k, const void* v, void* o,
                                int32_t Hq, int32_t n, const int32_t* spans, float scale, void* ws,
                                size_t ws_bytes, cudaStream_t s) {
  const ChunkLayout L = chunk_layout(c->B, Hq, c->Hkv, n, spans);
  if (ws_bytes < L.bytes) return MOA_ERR_WORKSPACE;
  char* sk = static_cast<char*>(ws) + L.off_k;
  char* sv = static_cast<char*>(ws) + L.off_v;
  const int64_t* t = reinterpret_cast<const int64_t*>(c->buf + kHdrT);
  const int32_t W = L.W;
  // the prefill kernel also appends the chunk to the ring (its keys come from
  // k, v and the gathered rows, never from the ring)
  return launch_prefill_bf16_rows(q, k, v, sk, sv, o, c->B, Hq, c->Hkv, n, W, t, spans, scale, ws, L.off_k, s,
                                  c, false, [&]() -> moa_status {
                                    return W > 0 ? launch_gather_window(c, W, sk, sv, s) : MOA_OK;
                                  });
}

}  // namespace moa
