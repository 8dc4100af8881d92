// attn_fwd_sm100.cu -- fused pair-bias multi-query attention forward, sm_100a.
//
// Computes, for every batch item b, query head h and query position i
// (page "Making Full-Context AlphaGenome Fit on an RTX 3090", section "Why
// stock FlashAttention was not a drop-in replacement", Eq. L_ij):
//   L_ij = cap * tanh((q_i . k_j / sqrt(D) + bias[h, i/16, j/16]) / cap)
//   out_i = softmax_j(L_ij) V,  lse_i = log sum_j exp(L_ij)
// one key tile at a time with the online softmax of section "Online softmax,
// one block at a time"; no L x L tensor exists at any point.
//
// B200 design (not the page's 64 x 64 Pallas tiling, which targeted sm_86):
//  * A query tile is 128 tensor-core rows = 16 consecutive positions x all 8
//    heads.  Every row of the tile shares one 16-position bias row block and
//    all 8 heads consume the same K/V tile (multi-query sharing).
//  * Two SMs work as a pair (a 2-CTA cluster) on a pair of query tiles: each
//    CTA holds one tile, and one thread of the even CTA issues tcgen05.mma
//    with cta_group::2, M = 256 rows over both SMs.  Each CTA stages only half
//    of every K tile (64 of its 128 keys) and half of every V tile (DV/2 of
//    the DV value columns), so each K/V byte crosses from L2 into one SM only
//    and serves the 256 query rows of the pair, and one MMA instruction keeps
//    both tensor cores busy.  DV (value width) is 128 or 192.
//  * One persistent cluster per SM pair takes a contiguous, equal share of all
//    (pair, key tile) steps; a pair whose key range is split between clusters
//    is merged exactly from the pieces' partial results by log-sum-exp (see
//    "Split pairs" below).
//  * Inside each CTA: a producer warp streams its Q tile and a ring of K and V
//    halves with TMA (no multicast); the softmax warpgroups own 32- or 64-key
//    chunks of the key tiles (see "Softmax warpgroups").  In the odd CTA the MMA warp relays
//    "loaded" to the even CTA (a cluster-scope arrive), so each CTA's copies
//    complete on its own barriers and can be drained locally.
//  * Tensor memory (per CTA): two 128-column S buffers (fp32 logits of
//    alternate key tiles) and the DV-column O accumulator.  P is written as
//    bf16 over part of its S buffer and fed to the PV product straight from
//    tensor memory.  With S double-buffered the MMA order per key tile is
//    PV(j), S(j+2): the logits a softmax warp needs next were computed while
//    it worked on the current ones.
//  * Bias: each softmax thread owns one row, so per key tile it needs just
//    the two compact cells of its 32 keys, read from global (L2) one tile
//    ahead and kept in registers; the 16x repeat is never built.
//  * With a finite cap every logit lies in (-cap, cap), so the softmax uses
//    the fixed shift m = cap (exact: softmax is shift invariant) and needs no
//    running max and no rescaling of O.  cap > 40 (where exp(-2 cap) would
//    underflow fp32) and cap = +inf use a running max with lazy rescaling.
//  * Every mbarrier wait is bounded (sm100.cuh); on timeout the kernel records
//    the wait site in the device error word, drains its own copies and MMAs,
//    frees tensor memory and returns.
#include "ag_internal.h"
#include "sm100.cuh"

namespace ag {
namespace attn {

constexpr int kH = 8;
constexpr int kD = 128;
constexpr int kKeys = static_cast<int>(kAttnKeyTile);  // keys per key tile
static_assert(kKeys == 128, "the tile layout below assumes 128-key tiles");
constexpr int kQTileBytes = 128 * kD * 2;     // this CTA's query tile (bf16)
constexpr int kQHalfBytes = kQTileBytes / 2;  // one 64-wide (128-byte) half
// A step load is what one key-tile step needs from this CTA: its half of a
// V tile (128 keys x DV/2 value columns; VLayout below) and its half of the K
// tile two steps ahead (64 keys x 128, two 64-wide halves of 8 KB), or, first in a
// segment, the halves of the segment's first two K tiles.  A ring slot holds
// two consecutive step loads, so the MMA thread waits for data and releases
// it once per two steps (each mbarrier operation costs it about 180 cycles
// while the tensor core is busy, measured).
constexpr int kPartBytes = 16384;            // one K half
constexpr int kKHalfBytes = kPartBytes / 2;  // a K half's 64-wide half
constexpr int kStages = 2;

// This CTA's half of a V tile, 128 keys x DV/2 value columns, MN-major for
// the PV product.  DV = 128: one 128-byte-swizzled 64-column box.  DV = 192
// (the value width of the page's checkpoint, section "Why stock
// FlashAttention was not a drop-in replacement", tensor V): 96 columns, which
// 64-column atoms cannot tile, so three 64-byte-swizzled 32-column boxes
// 8 KB apart.
template <int DV> struct VLayout;
template <> struct VLayout<128> {
  static constexpr int kBoxes = 1, kBoxCols = 64;
  static constexpr int kPartBytes = 128 * 64 * 2;       // 16 KB
  static constexpr uint32_t kDescHi = desc_sw128_hi(1024);
  static constexpr uint32_t kAtomBytes = 16384;         // LBO (one atom: unused)
  static constexpr uint32_t kKStepBytes = 16 * 128;     // 16 keys x 128 B
};
template <> struct VLayout<192> {
  static constexpr int kBoxes = 3, kBoxCols = 32;
  static constexpr int kPartBytes = 128 * 96 * 2;       // 24 KB
  static constexpr uint32_t kDescHi = desc_sw64_hi(512);
  static constexpr uint32_t kAtomBytes = 8192;          // LBO: 32-column atoms
  static constexpr uint32_t kKStepBytes = 16 * 64;      // 16 keys x 64 B
};
// A step load: a K half (part 0) and a V half or a second K half (part 1).
template <int DV> constexpr int step_bytes() { return kPartBytes + VLayout<DV>::kPartBytes; }
template <int DV> constexpr int slot_bytes() { return 2 * step_bytes<DV>(); }
static_assert(step_bytes<128>() >= 2 * kPartBytes && step_bytes<192>() >= 2 * kPartBytes,
              "step load 0 holds two K halves");
constexpr int kWG = 4;                      // softmax warpgroups
constexpr int kSoftThreads = 128 * kWG;
constexpr int kSoftWarps = 4 * kWG;         // per CTA
constexpr int kPairSoftWarps = 2 * kSoftWarps;
constexpr int kNumWarps = 4 * kWG + 4;
constexpr int kThreads = kNumWarps * 32;
constexpr int kWarpLoad = 4 * kWG;          // TMA producer
constexpr int kWarpMma = 4 * kWG + 1;       // MMA issuer (even CTA) / relay (odd)
// Registers per thread: the launch gives every thread kRegsLaunch (the cap
// for this block size, which ptxas allocates when setmaxnreg is present; the
// launcher checks it); the producer warpgroup then drops to kRegsLow (with
// fewer the MMA and relay threads spill).  The softmax keeps the launch count.
constexpr uint32_t kRegsLaunch = 96;
constexpr uint32_t kRegsLow = 88;
static_assert(kSoftThreads * kRegsLaunch + 128 * kRegsLow <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
// Tensor-memory columns: S buffer u at 128 u, O at 256 (DV columns).  P (bf16
// pairs) of chunk c (keys [32c, 32c + 32) of the tile) is written over the
// first 16 columns of that chunk's own S columns, [32c, 32c + 16).
constexpr uint32_t kColO = 256;
constexpr uint32_t kIdescQK = idesc_bf16_f32(256, kKeys, 0);  // K-major B (K)
template <int DV> constexpr uint32_t idesc_pv() { return idesc_bf16_f32(256, DV, 1); }
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Lazy rescale threshold (log2 units) for the running-max modes.
constexpr float kRescaleThreshold = 8.0f;

enum Mode { kStaticCap = 0, kOnlineCap = 1, kNoCap = 2 };

// Wait sites recorded in the device error word.
enum Site : unsigned {
  kSiteProdQ = 1, kSiteProdKV = 2, kSiteMmaQ = 3, kSiteMmaKV = 4,
  kSiteMmaP = 5, kSiteSoftS = 6, kSiteSoftO = 7, kSiteDrain = 8,
  kSiteXchg = 9, kSiteSoftPV = 10, kSiteRelay = 11
};

// Per-CTA barriers.  In the even CTA, q_full and kv_full also count the odd
// CTA's relay (two arrivals: the local producer's, with the byte count, and
// the relay's), so the MMA thread waits once for both halves of a load;
// p_full is used in the even CTA only (the odd CTA's softmax warps arrive on
// it remotely).  q_empty, kv_empty, s_full, pv_done and o_full are signalled
// in both CTAs by the even CTA's MMA commits.
struct __align__(8) Barriers {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  // s_full / p_full by S buffer: a softmax may finish key tile j + 1 before
  // the MMA warp has taken key tile j's arrivals.
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_full;
  uint64_t xm, xd;  // row-max / row-sum exchange between the warpgroups
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int range_begin, range_end;  // this cluster's (pair, key tile) steps
};

// Softmax-side shared memory: row-max (per step, double-buffered by step
// parity) and row-sum (per segment) exchange between the four chunks.
struct Xchg {
  float mpart[2][kWG][128];  // [step parity][chunk][row]
  float dpart[kWG][128];     // [chunk][row]
};

template <int DV> constexpr size_t smem_bytes() {
  return 1024 + static_cast<size_t>(kQTileBytes) +
         kStages * static_cast<size_t>(slot_bytes<DV>()) + sizeof(Barriers) +
         sizeof(Xchg);
}
static_assert(smem_bytes<128>() <= 227 * 1024 && smem_bytes<192>() <= 227 * 1024,
              "shared memory budget");

struct Params {
  const float *bias;
  long long bias_bstride;  // floats between batch items' bias (0: shared)
  float *out;
  float *lse;
  unsigned *err;
  // Split-pair scratch (see "Split pairs"): one slot per cluster.
  float *ws_out;       // [clusters][2][128][DV] partial outputs
  float *ws_lse;       // [clusters][2][128] partial log-sum-exps
  int L, P;
  int nb;          // 16-position query blocks per batch item, ceil(L / 16)
  int pairs;       // query-tile pairs per batch item: ceil(nb / 2)
  int n_items;     // B * pairs
  int n_kt;        // key tiles: ceil(L / 128)
  int last_valid;  // valid keys in the last key tile (1..128)
  int whole;       // 1: cluster ranges hold whole pairs (no split pairs)
  float qk_scale;  // multiplies q.k
  float bias_mul;  // multiplies the compact bias
  float A;         // capped modes: cap * log2(e)
};

// --------------------------------------------------------------------------
// Work split.  The W = n_items * n_kt (pair, key tile) steps are cut into
// one contiguous range per cluster, [W c / G, W (c+1) / G) for cluster c of
// G.  Both CTAs of a cluster walk the range as segments: one pair and a run
// of its key tiles.  A pair covered by more than one cluster is "split".
struct Segment {
  int item, kb, ke;  // pair index and key tiles [kb, ke)
};

__device__ __forceinline__ int num_clusters() { return static_cast<int>(gridDim.x >> 1); }
__device__ __forceinline__ int cluster_index() { return static_cast<int>(blockIdx.x >> 1); }

// W = n_items * n_kt <= 2^30 (checked by the launcher), so steps fit in int;
// only the range bounds need a 64-bit product.  With p.whole the bounds are
// rounded to whole pairs: cluster c gets pairs [n_items c / G, n_items (c+1) / G).
__device__ __forceinline__ int range_start(const Params &p, int c) {
  const long long G = num_clusters();
  if (p.whole)
    return static_cast<int>(static_cast<long long>(p.n_items) * c / G) * p.n_kt;
  return static_cast<int>(static_cast<long long>(p.n_items) * p.n_kt * c / G);
}

__device__ __forceinline__ Segment segment_at(const Params &p, int t, int end) {
  Segment sg;
  sg.item = t / p.n_kt;
  sg.kb = t - sg.item * p.n_kt;
  const int left = end - t;
  sg.ke = left < p.n_kt - sg.kb ? sg.kb + left : p.n_kt;
  return sg;
}

// K/V ring order, shared by the producers, the relay and the MMA warp: for a
// segment with key tiles [kb, ke) (n of them), step load 0 holds K(kb) (part
// 0) and K(kb+1) (part 1); step load i = 1 .. n holds K(kb+i+1) (part 0,
// while it exists) and V(kb+i-1) (part 1).  S runs two key tiles ahead of PV.
// Step loads 2d and 2d+1 share ring slot load d (the last may be alone).
struct StepLoad {
  int k_tile;  // K tile in part 0, or -1
  int second;  // V tile (is_v) or K tile in part 1, or -1
  bool is_v;
};
__device__ __forceinline__ StepLoad step_load(const Segment &sg, int i) {
  const int n = sg.ke - sg.kb;
  if (i == 0) return {sg.kb, n > 1 ? sg.kb + 1 : -1, false};
  return {sg.kb + i + 1 < sg.ke ? sg.kb + i + 1 : -1, sg.kb + i - 1, true};
}
// f(first step load, last step load) for every ring slot load of the segment.
template <typename F>
__device__ __forceinline__ bool for_each_slot_load(const Segment &sg, F &&f) {
  const int n = sg.ke - sg.kb;
  bool ok = true;
  for (int i = 0; i <= n && ok; i += 2) ok = f(i, i + 1 <= n ? i + 1 : i);
  return ok;
}

// --------------------------------------------------------------------------
// MMA issue helpers (single thread of the even CTA).

// Shared-memory descriptors: every operand here has 8-row groups 1 KB apart,
// so all share one high word; the low word (start address and leading
// offset) is built once per tile base and each K step adds a constant to its
// start-address field (addresses stay below 2^18: no carry out of the field).
constexpr uint32_t kDescHi = desc_sw128_hi(1024);

// S[256 x 128] = Q[256 x 128] K^T over the pair: eight K=16 steps over the two
// 64-wide halves of each CTA's Q tile (16 KB apart) and K half (8 KB apart).
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr,
                                         uint32_t k_addr) {
  const uint32_t q_lo = desc_sw128_lo(q_addr, 16), k_lo = desc_sw128_lo(k_addr, 16);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t qo = ((kk >> 2) * kQHalfBytes + (kk & 3) * 32) >> 4;
    const uint32_t ko = ((kk >> 2) * kKHalfBytes + (kk & 3) * 32) >> 4;
    umma2_ss_lo(d_tmem, q_lo + qo, k_lo + ko, kDescHi, kIdescQK, kk > 0 ? 1u : 0u);
  }
}

// O[256 x DV] (+)= P[256 x 128 keys] V[128 keys x DV]: P from each CTA's
// tensor memory (bf16 pairs, 8 columns per 16 keys; keys 32c.. of chunk c
// start at column 32c of the S buffer), V MN-major: each CTA holds DV/2 value
// columns for all 128 keys (VLayout).
template <int DV>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t s_tmem,
                                         uint32_t v_addr, bool accumulate) {
  using VL = VLayout<DV>;
  const uint32_t v_lo = desc_sw128_lo(v_addr, VL::kAtomBytes);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    umma2_ts_lo(d_tmem, s_tmem + 32 * (kk >> 1) + 8 * (kk & 1),
                v_lo + ((kk * VL::kKStepBytes) >> 4), VL::kDescHi, idesc_pv<DV>(),
                (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Bounded wait used while draining: ignores the abort flag, records nothing.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(a, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// The query block this CTA's tile covers in pair item I0 / 2: I0 + rank, or
// (past the end of an odd count) a copy of block I0 whose results are not
// written.
__device__ __forceinline__ int tile_block(const Params &p, int I0, uint32_t rank) {
  const int I = I0 + static_cast<int>(rank);
  return I < p.nb ? I : I0;
}

// --------------------------------------------------------------------------
// Producer warp, lane 0 (each CTA): TMA loads of this CTA's Q tile and of its
// halves of the K and V tiles.
template <int DV>
__device__ __forceinline__ void producer(const CUtensorMap *tm_q,
                                         const CUtensorMap *tm_k,
                                         const CUtensorMap *tm_v, uint8_t *q_s,
                                         uint8_t *kv_s, Barriers *bars,
                                         const Params &p, uint32_t rank,
                                         volatile int *abort) {
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t qcount = 0, kv = 0;
  bool ok = true;
  const int end = bars->range_end;
  for (int t = bars->range_begin; t < end && ok;) {
    const Segment sg = segment_at(p, t, end);
    t += sg.ke - sg.kb;
    const int b = sg.item / p.pairs;
    const int I0 = (sg.item % p.pairs) * 2;
    ok = mbar_wait(&bars->q_empty, (qcount & 1u) ^ 1u, abort, p.err, kSiteProdQ);
    if (!ok) break;
    mbar_arrive_expect_tx(&bars->q_full, kQTileBytes);
    const int qrow = tile_block(p, I0, rank) * 16;
    tma_load_4d(q_s, tm_q, &bars->q_full, 0, qrow, 0, b, pol_q);
    tma_load_4d(q_s + kQHalfBytes, tm_q, &bars->q_full, 64, qrow, 0, b, pol_q);
    ++qcount;
    ok = for_each_slot_load(sg, [&](int i0, int i1) {
      const uint32_t slot = kv % kStages, ph = (kv / kStages) & 1u;
      if (!mbar_wait(&bars->kv_empty[slot], ph ^ 1u, abort, p.err, kSiteProdKV))
        return false;
      uint32_t bytes = 0;
      for (int i = i0; i <= i1; ++i) {
        const StepLoad sl = step_load(sg, i);
        bytes += (sl.k_tile >= 0 ? kPartBytes : 0) +
                 (sl.second < 0 ? 0 : sl.is_v ? VLayout<DV>::kPartBytes : kPartBytes);
      }
      mbar_arrive_expect_tx(&bars->kv_full[slot], bytes);
      // A K half: keys [128 j + 64 rank, +64), all 128 columns.
      auto load_k = [&](uint8_t *to, int j) {
        const int key0 = j * kKeys + 64 * static_cast<int>(rank);
        tma_load_3d(to, tm_k, &bars->kv_full[slot], 0, key0, b, pol_kv);
        tma_load_3d(to + kKHalfBytes, tm_k, &bars->kv_full[slot], 64, key0, b, pol_kv);
      };
      for (int i = i0; i <= i1; ++i) {
        const StepLoad sl = step_load(sg, i);
        uint8_t *dst = kv_s + slot * slot_bytes<DV>() + (i & 1) * step_bytes<DV>();
        if (sl.k_tile >= 0) load_k(dst, sl.k_tile);
        if (sl.is_v) {  // keys [128 j, +128), value columns [DV/2 rank, +DV/2)
#pragma unroll
          for (int a = 0; a < VLayout<DV>::kBoxes; ++a)
            tma_load_3d(dst + kPartBytes + a * VLayout<DV>::kAtomBytes, tm_v,
                        &bars->kv_full[slot],
                        (DV / 2) * static_cast<int>(rank) + a * VLayout<DV>::kBoxCols,
                        sl.second * kKeys, b, pol_kv);
        } else if (sl.second >= 0) {
          load_k(dst + kPartBytes, sl.second);
        }
      }
      ++kv;
      return true;
    });
  }
  // Every copy this thread started must land before the CTA exits.
  if (qcount > 0) drain_wait(&bars->q_full, (qcount - 1) & 1u);
  const uint32_t first = kv > kStages ? kv - kStages : 0;
  for (uint32_t i = first; i < kv; ++i)
    drain_wait(&bars->kv_full[i % kStages], (i / kStages) & 1u);
}

// --------------------------------------------------------------------------
// MMA warp of the odd CTA, lane 0: tells the even CTA's MMA thread, in ring
// order, that this CTA's half of each Q / K / V load has landed.
__device__ __forceinline__ void relay(Barriers *bars, const Params &p,
                                      volatile int *abort) {
  const uint32_t q_leader = cluster_addr(&bars->q_full, 0);
  uint32_t qcount = 0, kv = 0;
  bool ok = true;
  const int end = bars->range_end;
  for (int t = bars->range_begin; t < end && ok;) {
    const Segment sg = segment_at(p, t, end);
    t += sg.ke - sg.kb;
    ok = mbar_wait(&bars->q_full, qcount & 1u, abort, p.err, kSiteRelay);
    ++qcount;
    if (!ok) break;
    mbar_arrive_cluster(q_leader);
    ok = for_each_slot_load(sg, [&](int, int) {
      const uint32_t slot = kv % kStages;
      if (!mbar_wait(&bars->kv_full[slot], (kv / kStages) & 1u, abort, p.err,
                     kSiteRelay))
        return false;
      ++kv;
      mbar_arrive_cluster(cluster_addr(&bars->kv_full[slot], 0));
      return true;
    });
  }
}

// --------------------------------------------------------------------------
// MMA warp of the even CTA, lane 0: tcgen05.mma issuer for the pair.
// kPvDone: also signal pv_done after every PV but the segment's last (the
// running-max modes rescale O and must know when the previous PV finished).
template <bool kPvDone, int DV>
__device__ __forceinline__ void mma_issuer(uint8_t *q_s, uint8_t *kv_s,
                                           Barriers *bars, uint32_t tmem,
                                           const Params &p, volatile int *abort) {
  const uint32_t q_addr = smem_u32(q_s);
  const uint32_t kv_addr = smem_u32(kv_s);
  uint32_t qcount = 0, kv = 0;
  uint32_t pbits = 0;  // bit u: parity of the next p_full[u] phase
  bool ok = true;
  // Both halves of the next ring load: this CTA's copy and the peer's relay
  // (both arrive on this CTA's kv_full).  The odd CTA's arrivals here (relay,
  // softmax) are relaxed (see mbar_arrive_cluster), so these waits acquire at
  // CTA scope: a cluster-scope acquire would order nothing more and costs
  // about 180 cycles per wait on this thread (measured).
  auto wait_kv = [&](uint32_t &slot) {
    slot = kv % kStages;
    const uint32_t ph = (kv / kStages) & 1u;
    ++kv;
    return mbar_wait(&bars->kv_full[slot], ph, abort, p.err, kSiteMmaKV);
  };
  const int end = bars->range_end;
  for (int t = bars->range_begin; t < end && ok;) {
    const Segment sg = segment_at(p, t, end);
    t += sg.ke - sg.kb;
    const int n = sg.ke - sg.kb;
    ok = mbar_wait(&bars->q_full, qcount & 1u, abort, p.err, kSiteMmaQ);
    ++qcount;
    if (!ok) break;
    // Step load 0: S(kb) into buffer 0 and S(kb+1) into buffer 1.
    uint32_t slot;
    ok = wait_kv(slot);
    if (!ok) break;
    tc_fence_after();
    {
      const uint32_t base = kv_addr + slot * slot_bytes<DV>();
      for (int u = 0; u < 2 && u < n; ++u) {
        issue_qk(tmem + 128u * u, q_addr, base + u * kPartBytes);
        umma2_commit_both(&bars->s_full[u]);
        if (u == n - 1) umma2_commit_both(&bars->q_empty);
      }
    }

    // Step load i = j - kb + 1: V(j) in part 1, K(j+2) (while it exists) in
    // part 0; a new ring slot starts at every even i.
    for (int j = sg.kb; j < sg.ke; ++j) {
      const int i = j - sg.kb + 1;
      const uint32_t u = static_cast<uint32_t>(j - sg.kb) & 1u;
      if ((i & 1) == 0) {
        ok = wait_kv(slot);
        if (!ok) break;
      }
      ok = mbar_wait(&bars->p_full[u], (pbits >> u) & 1u, abort, p.err, kSiteMmaP);
      pbits ^= 1u << u;
      if (!ok) break;
      tc_fence_after();
      const uint32_t base = kv_addr + slot * slot_bytes<DV>() + (i & 1) * step_bytes<DV>();
      issue_pv<DV>(tmem + kColO, tmem + 128u * u, base + kPartBytes, j > sg.kb);
      if (j + 1 == sg.ke)
        umma2_commit_both(&bars->o_full);
      else if (kPvDone)
        umma2_commit_both(&bars->pv_done);
      if (j + 2 < sg.ke) {
        // S(j+2) over buffer u: issued after PV(j), which reads P(j) from the
        // same columns (the tensor core runs one thread's MMAs in order).
        issue_qk(tmem + 128u * u, q_addr, base);
        umma2_commit_both(&bars->s_full[u]);
        if (j + 3 == sg.ke) umma2_commit_both(&bars->q_empty);
      }
      if ((i & 1) == 1 || j + 1 == sg.ke) umma2_commit_both(&bars->kv_empty[slot]);
    }
    // A segment of one key tile: its only slot holds step loads 0 and 1 and
    // was released above; otherwise the last slot was released in the loop.
  }
  // All MMAs this thread issued complete before tensor memory is released.
  umma2_commit_self(&bars->drain);
  drain_wait(&bars->drain, 0);
}

// --------------------------------------------------------------------------
// Softmax warpgroups (each CTA, its own query tile).
//
// Thread r of a warpgroup owns tensor-memory lane r, i.e. row r of the tile.
// Static-cap mode: warpgroups 2q and 2q+1 take the key tiles in S buffer q,
// 64 keys each.  Running-max modes: warpgroup g takes keys [32g, 32g + 32) of
// every key tile.  Either way a row's sum is split between four threads and
// combined through shared memory once per work item (and, in the running-max
// modes, its maximum once per key tile).  Each 32-key chunk's P goes over
// the first 16 of its own S columns, so a warpgroup only ever overwrites S
// columns it has already read itself.

// Softmax-side barriers count warps: each warp arrives once, from lane 0,
// after __syncwarp has ordered its lanes' prior work (one arrival per warp
// instead of 32 keeps the mbarrier off the shared-memory pipe).
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
  __syncwarp();
  if (lane_id() == 0) mbar_arrive(bar);
}

// Publish this thread's value, then wait (bounded) until every softmax thread
// of the CTA has published its own.  The warp barrier and the mbarrier's
// arrive/wait order the shared-memory writes before the partners' reads.
__device__ __forceinline__ bool exchange(uint64_t *bar, uint32_t &count,
                                         volatile int *abort, unsigned *err) {
  warp_arrive(bar);
  const bool ok = mbar_wait(bar, count & 1u, abort, err, kSiteXchg);
  ++count;
  return __all_sync(0xffffffffu, ok);
}

// The compact bias cells of chunk g of key tile j (two per 32-key chunk):
// bias[h, I, 8j + 2g + e] (0 past the end: those keys are masked).
__device__ __forceinline__ void load_bias(const float *brow, int j, int g, int P,
                                          float (&bn)[2]) {
  const int J0 = j * 8 + g * 2;
#pragma unroll
  for (int e = 0; e < 2; ++e) bn[e] = (J0 + e < P) ? __ldg(brow + J0 + e) : 0.f;
}

// Column pairs (out of every 8) whose exponential runs on the FMA pipe
// (exp2_poly2) instead of the special-function unit.  The SFU still computes
// every tanh, so it does 1 + (8 - kEmuPairs) / 8 operations per logit.
#ifndef AG_EXP2_EMU_PAIRS
#define AG_EXP2_EMU_PAIRS 6
#endif
constexpr int kEmuPairs = AG_EXP2_EMU_PAIRS;

// Static-shift softmax of one 32-column chunk: p = 2^(A tanh(y) - A) with
// y = s * qk_scale + b / cap, two columns at a time.  Adds the row sum into
// acc and writes 16 bf16 pairs of P.  kMask zeroes columns >= nvalid (only
// the last key tile of a ragged length needs it).
template <bool kMask>
__device__ __forceinline__ void chunk_static(const uint32_t (&s)[32], float b0,
                                             float b1, float2 sc, float2 ap,
                                             float2 an, int col0, int nvalid,
                                             float2 &acc, uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float bb = e < 8 ? b0 : b1;
    const float2 y = __ffma2_rn(
        make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), sc,
        make_float2(bb, bb));
    const float2 t = make_float2(tanh_approx(y.x), tanh_approx(y.y));
    const float2 x = __ffma2_rn(t, ap, an);
    float2 pr;
    if ((e & 7) < kEmuPairs) {
      pr = exp2_poly2(x);
    } else {
      pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    }
    if (kMask) {
      if (col0 + 2 * e >= nvalid) pr.x = 0.f;
      if (col0 + 2 * e + 1 >= nvalid) pr.y = 0.f;
    }
    acc = __fadd2_rn(acc, pr);
    pk[e] = pack_bf16x2(pr.x, pr.y);
  }
}

// One key tile, static shift: S in, P out over the first 16 columns of this
// warpgroup's chunk.  Returns the partial row sum.
template <bool kMask>
__device__ __forceinline__ float tile_static(uint32_t tS, int col0, float b0,
                                             float b1, float2 sc, float2 ap,
                                             float2 an, int nvalid) {
  float2 acc = make_float2(0.f, 0.f);
  uint32_t s[32], pk[16];
  tmem_ld32(tS, s);
  tmem_wait_ld(s);
  chunk_static<kMask>(s, b0, b1, sc, ap, an, col0, nvalid, acc, pk);
  tmem_st16(tS, pk);
  return acc.x + acc.y;
}

// One key tile with a running maximum shared by the four threads of each row
// (exchanged through shared memory).  When the maximum grows past the lazy
// threshold, this warpgroup's DV/4 columns of O are rescaled, after the
// previous PV into O has finished (pv_done).
template <int MODE, int DV>
__device__ __forceinline__ bool tile_online(uint32_t tS, uint32_t tO, int g,
                                            int r, uint32_t par, bool o_live,
                                            uint32_t pv_parity, float b0,
                                            float b1, const Params &p, int nvalid,
                                            Xchg *xc, Barriers *bars,
                                            uint32_t &xcount, volatile int *abort,
                                            float &m, float &d) {
  uint32_t s[32];
  float x[32];
  tmem_ld32(tS, s);
  tmem_wait_ld(s);
  float mt = -INFINITY;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float bb = e < 16 ? b0 : b1;
    const float y = fmaf(__uint_as_float(s[e]), p.qk_scale, bb);
    const float v = (MODE == kOnlineCap) ? p.A * tanh_approx(y) : y;
    x[e] = (32 * g + e < nvalid) ? v : -INFINITY;
    mt = fmaxf(mt, x[e]);
  }
  xc->mpart[par][g][r] = mt;
  if (!exchange(&bars->xm, xcount, abort, p.err)) return false;
#pragma unroll
  for (int q = 0; q < kWG; ++q) mt = fmaxf(mt, xc->mpart[par][q][r]);
  float factor = 1.f;
  if (mt > m + kRescaleThreshold || m == -INFINITY) {
    factor = (m == -INFINITY) ? 0.f : ex2_approx(m - mt);
    m = mt;
    d *= factor;
  }
  if (o_live && __any_sync(0xffffffffu, factor != 1.f)) {
    const bool ok = mbar_wait(&bars->pv_done, pv_parity, abort, p.err, kSiteSoftPV);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    uint32_t o[32];
    tmem_ld32(tO, o);
    tmem_wait_ld(o);
#pragma unroll
    for (int e = 0; e < 32; ++e)
      o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
    tmem_st32(tO, o);
    if constexpr (DV == 192) {  // columns 32 .. 47 of this warpgroup's 48
      uint32_t o2[16];
      tmem_ld16(tO + 32, o2);
      tmem_wait_ld16(o2);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        o2[e] = __float_as_uint(__uint_as_float(o2[e]) * factor);
      tmem_st16(tO + 32, o2);
    }
  }
  float acc = 0.f;
  uint32_t pk[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float p0 = ex2_approx(x[2 * e] - m);
    const float p1 = ex2_approx(x[2 * e + 1] - m);
    acc += p0 + p1;
    pk[e] = pack_bf16x2(p0, p1);
  }
  tmem_st16(tS, pk);
  d += acc;
  return true;
}

// --------------------------------------------------------------------------
// Split pairs.  Every segment of a split pair finishes like a whole pair but
// over its own key range: a normalised partial output and the partial
// log-sum-exp.  The first segment (key tile 0) writes them to out / lse, the
// others to the scratch slot of their cluster (a cluster starts at most one
// segment in the middle of a pair).  attn_merge_kernel, launched right after
// on the same stream, then merges the pieces of every split pair:
//   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) out_s.

// Static-cap mode: the warps split into two groups that take alternate key
// tiles (group q = warpgroups 2q, 2q+1 takes the tiles in S buffer q), each
// warpgroup 64 keys of its group's tiles.  Both S buffers are then in work
// at once, so one group's waits (for its logits, for its tensor-memory
// stores, for its arrival) are covered by the other group's arithmetic.
__device__ __forceinline__ void load_bias4(const float *brow, int j, int hk, int P,
                                           float (&bn)[4]) {
  const int J0 = j * 8 + hk * 4;
#pragma unroll
  for (int e = 0; e < 4; ++e) bn[e] = (J0 + e < P) ? __ldg(brow + J0 + e) : 0.f;
}

__device__ __forceinline__ bool segment_static(const Segment &sg, const float *brow,
                                               uint32_t tmem, uint32_t lane_base,
                                               int g, const Params &p,
                                               Barriers *bars, uint32_t rank,
                                               uint32_t pf_remote, uint32_t &scount,
                                               volatile int *abort, float &d) {
  const int q = g >> 1, hk = g & 1;  // group (S buffer) and key half
  const float2 sc = make_float2(p.qk_scale, p.qk_scale);
  const float2 ap = make_float2(p.A, p.A), an = make_float2(-p.A, -p.A);
  const int j0 = sg.kb + q;
  // Bias cells of this group's next tile.  The cells of tile j + 2 are
  // requested right after tile j's arrival (a load in flight would hold up
  // that arrival); they land while the group waits for tile j + 2's logits.
  float bc[4] = {0.f, 0.f, 0.f, 0.f};
  if (j0 < sg.ke) load_bias4(brow, j0, hk, p.P, bc);
  for (int j = j0; j < sg.ke; j += 2) {
    const int nvalid = (j + 1 == p.n_kt) ? p.last_valid : kKeys;
    bool ok = mbar_wait(&bars->s_full[q], scount & 1u, abort, p.err, kSiteSoftS);
    ++scount;
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + 128u * q + 64 * hk + lane_base;
    const float m = p.bias_mul;
    if (nvalid == kKeys) {
      d += tile_static<false>(tS, 64 * hk, bc[0] * m, bc[1] * m, sc, ap, an, nvalid);
      d += tile_static<false>(tS + 32, 64 * hk + 32, bc[2] * m, bc[3] * m, sc, ap, an,
                              nvalid);
    } else {
      d += tile_static<true>(tS, 64 * hk, bc[0] * m, bc[1] * m, sc, ap, an, nvalid);
      d += tile_static<true>(tS + 32, 64 * hk + 32, bc[2] * m, bc[3] * m, sc, ap, an,
                             nvalid);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane_id() == 0) {
      if (rank == 0)
        mbar_arrive(&bars->p_full[q]);
      else
        mbar_arrive_cluster(pf_remote);
    }
    if (j + 2 < sg.ke) load_bias4(brow, j + 2, hk, p.P, bc);
  }
  return true;
}

// Running-max modes: every warpgroup takes every key tile (32 keys each),
// the four threads of a row sharing its maximum per tile.
template <int MODE, int DV>
__device__ __forceinline__ bool segment_online(const Segment &sg, const float *brow,
                                               uint32_t tmem, uint32_t lane_base,
                                               int g, int r, const Params &p,
                                               Barriers *bars, Xchg *xc,
                                               uint32_t rank, uint32_t pf_remote0,
                                               uint32_t pf_remote1, uint32_t &scount0,
                                               uint32_t &scount1, uint32_t &xmcount,
                                               uint32_t pvd, volatile int *abort,
                                               float &m, float &d) {
  float bc[2], bn[2] = {0.f, 0.f};
  load_bias(brow, sg.kb, g, p.P, bc);
  if (sg.kb + 1 < sg.ke) load_bias(brow, sg.kb + 1, g, p.P, bn);
  for (int j = sg.kb; j < sg.ke; ++j) {
    const uint32_t u = static_cast<uint32_t>(j - sg.kb) & 1u;
    const int nvalid = (j + 1 == p.n_kt) ? p.last_valid : kKeys;
    const float b0 = bc[0] * p.bias_mul, b1 = bc[1] * p.bias_mul;
    const uint32_t sphase = u ? scount1++ : scount0++;
    bool ok = mbar_wait(&bars->s_full[u], sphase & 1u, abort, p.err, kSiteSoftS);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + 128u * u + 32 * g + lane_base;
    const uint32_t tO = tmem + kColO + (DV / 4) * g + lane_base;
    // PV(j-1) is pv_done phase pvd + (j - 1 - kb); PV(j-2) has finished
    // (s_full(j) was committed after it), so that phase is the current or
    // the last completed one and its parity identifies it.
    const uint32_t pv_parity = (pvd + static_cast<uint32_t>(j - 1 - sg.kb)) & 1u;
    if (!tile_online<MODE, DV>(tS, tO, g, r, u, j > sg.kb, pv_parity, b0, b1, p, nvalid,
                           xc, bars, xmcount, abort, m, d))
      return false;
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane_id() == 0) {
      if (rank == 0)
        mbar_arrive(&bars->p_full[u]);
      else
        mbar_arrive_cluster(u ? pf_remote1 : pf_remote0);
    }
    bc[0] = bn[0];
    bc[1] = bn[1];
    if (j + 2 < sg.ke) load_bias(brow, j + 2, g, p.P, bn);
  }
  return true;
}

template <int MODE, int DV>
__device__ __forceinline__ void softmax_role(Barriers *bars, Xchg *xc,
                                             uint32_t tmem, const Params &p,
                                             uint32_t rank, volatile int *abort) {
  const int g = threadIdx.x >> 7;         // warpgroup
  const int r = threadIdx.x & 127;        // tile row == tensor-memory lane
  const int h = r >> 4, il = r & 15;      // head, position inside the block
  const uint32_t lane_base = static_cast<uint32_t>(r >> 5) << 21;  // (32 * quarter) << 16
  const uint32_t pf_remote0 = cluster_addr(&bars->p_full[0], 0);
  const uint32_t pf_remote1 = cluster_addr(&bars->p_full[1], 0);
  uint32_t scount0 = 0, scount1 = 0;  // s_full waits per S buffer
  uint32_t ocount = 0, xmcount = 0, xdcount = 0;
  uint32_t pvd = 0;  // pv_done phases completed before this segment
  bool ok = true;
  const int end = bars->range_end;

  for (int t = bars->range_begin; t < end && ok;) {
    const Segment sg = segment_at(p, t, end);
    t += sg.ke - sg.kb;
    const int b = sg.item / p.pairs;
    const int I0 = (sg.item % p.pairs) * 2;
    const int I = tile_block(p, I0, rank);
    const bool valid = I0 + static_cast<int>(rank) < p.nb;
    const int pos = I * 16 + il;  // this thread's query position
    const float *brow = p.bias + static_cast<long long>(b) * p.bias_bstride +
                        (static_cast<size_t>(h) * p.P + I) * p.P;
    float m = (MODE == kStaticCap) ? p.A : -INFINITY;  // log2 units
    float d = 0.f;
    if constexpr (MODE == kStaticCap) {
      // A thread of group q only ever waits on S buffer q: scount0 counts
      // those waits.
      ok = segment_static(sg, brow, tmem, lane_base, g, p, bars, rank,
                          (g >> 1) ? pf_remote1 : pf_remote0, scount0, abort, d);
    } else {
      ok = segment_online<MODE, DV>(sg, brow, tmem, lane_base, g, r, p, bars, xc, rank,
                                pf_remote0, pf_remote1, scount0, scount1, xmcount,
                                pvd, abort, m, d);
    }
    if (!ok) break;
    pvd += static_cast<uint32_t>(sg.ke - sg.kb - 1);

    // Epilogue: d = sum of the four warpgroups' partial sums; out = O / d
    // over this segment's keys (warpgroup g writes columns [g DV/4, (g+1)
    // DV/4) of the row) and lse, to out / lse or, for a later piece of a
    // split pair, to this cluster's scratch slot.  The copy of block I0 in an
    // odd CTA past the end of an odd block count writes nothing.
    ok = mbar_wait(&bars->o_full, ocount & 1u, abort, p.err, kSiteSoftO);
    ++ocount;
    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
    tc_fence_after();
    xc->dpart[g][r] = d;
    ok = exchange(&bars->xd, xdcount, abort, p.err);
    if (!ok) break;
    float dsum = 0.f;
#pragma unroll
    for (int q = 0; q < kWG; ++q) dsum += xc->dpart[q][r];
    const float inv_d = 1.f / dsum;
    const uint32_t tO = tmem + kColO + (DV / 4) * g + lane_base;
    uint32_t o[32];
    tmem_ld32(tO, o);
    tmem_wait_ld(o);
    uint32_t o2[16];  // columns 32 .. 47 of this warpgroup's 48 (DV = 192)
    if constexpr (DV == 192) {
      tmem_ld16(tO + 32, o2);
      tmem_wait_ld16(o2);
    }
    if (valid && pos < p.L) {  // rows past the end of a partial block: none
      const size_t row = (static_cast<size_t>(b) * kH + h) * p.L +
                         static_cast<size_t>(pos);
      float *orow_base;
      float *lse_dst;
      if (sg.kb == 0) {
        orow_base = p.out + row * DV;
        lse_dst = p.lse + row;
      } else {
        const size_t slot =
            (static_cast<size_t>(cluster_index()) * 2 + rank) * 128 + r;
        orow_base = p.ws_out + slot * DV;
        lse_dst = p.ws_lse + slot;
      }
      float4 *orow = reinterpret_cast<float4 *>(orow_base + (DV / 4) * g);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        orow[e] = make_float4(__uint_as_float(o[4 * e]) * inv_d,
                              __uint_as_float(o[4 * e + 1]) * inv_d,
                              __uint_as_float(o[4 * e + 2]) * inv_d,
                              __uint_as_float(o[4 * e + 3]) * inv_d);
      }
      if constexpr (DV == 192) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          orow[8 + e] = make_float4(__uint_as_float(o2[4 * e]) * inv_d,
                                    __uint_as_float(o2[4 * e + 1]) * inv_d,
                                    __uint_as_float(o2[4 * e + 2]) * inv_d,
                                    __uint_as_float(o2[4 * e + 3]) * inv_d);
        }
      }
      if (g == 0) *lse_dst = (m + lg2_approx(dsum)) * kLn2;
    }
    tc_fence_before();
  }
}

// --------------------------------------------------------------------------
template <int MODE, int DV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *q_s = smem_raw + pad;             // this CTA's query tile
  uint8_t *kv_s = q_s + kQTileBytes;         // K/V ring
  Barriers *bars = reinterpret_cast<Barriers *>(kv_s + kStages * slot_bytes<DV>());
  auto *xc = reinterpret_cast<Xchg *>(reinterpret_cast<uint8_t *>(bars) +
                                      sizeof(Barriers));
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    const uint32_t loads = rank == 0 ? 2 : 1;  // producer (+ relay, even CTA)
    mbar_init(&bars->q_full, loads);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], loads);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bars->s_full[u], 1);
      // Static cap: one warp group per S buffer; otherwise every warp.
      mbar_init(&bars->p_full[u], MODE == kStaticCap ? kPairSoftWarps / 2 : kPairSoftWarps);
    }
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->xm, kSoftWarps);
    mbar_init(&bars->xd, kSoftWarps);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    bars->range_begin = range_start(p, cluster_index());
    bars->range_end = range_start(p, cluster_index() + 1);
    fence_mbar_init();
  }
  if (warp == kWarpLoad && lane_id() == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == kWarpMma) {
    tmem_alloc2(&bars->tmem_base, kTmemCols);
    tmem_relinquish2();
  }
  // Both CTAs' barriers are initialised and their tensor memory allocated
  // before either CTA signals the other.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;

  if (warp >= kWarpLoad) {
    regs_dec<kRegsLow>();
    if (warp == kWarpLoad && lane_id() == 0) {
      producer<DV>(&tm_q, &tm_k, &tm_v, q_s, kv_s, bars, p, rank, abort);
    } else if (warp == kWarpMma && lane_id() == 0) {
      if (rank == 0)
        mma_issuer<MODE != kStaticCap, DV>(q_s, kv_s, bars, tmem, p, abort);
      else
        relay(bars, p, abort);
    }
  } else {
    softmax_role<MODE, DV>(bars, xc, tmem, p, rank, abort);
  }
  __syncwarp();
  // No CTA leaves while the other may still use its shared or tensor memory:
  // the even CTA's MMAs have drained and the odd CTA's remote arrivals are
  // done once every thread of both CTAs is here.
  tc_fence_before();
  cluster_sync();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc2(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------------------
// Split-pair merge.  kMergeBlocksPerBoundary blocks per cluster boundary; only
// the boundary that is the first one inside a pair merges that pair.  One
// warp per output row (query tile row / 128, row % 128): lane l merges the
// 4-column groups l, l + 32, ... of the row's DV columns over the pieces, and
// lane 0 writes the merged lse once every lane has read the first piece's.
constexpr int kMergeThreads = 256;
constexpr int kMergeRowsPerBlock = kMergeThreads / 32;
constexpr int kMergeBlocksPerBoundary = 2 * 128 / kMergeRowsPerBlock;

template <int DV>
__global__ void __launch_bounds__(kMergeThreads)
    attn_merge_kernel(const Params p, int grid) {
  const int c = blockIdx.x / kMergeBlocksPerBoundary + 1;  // boundary between clusters c-1, c
  const int W = p.n_items * p.n_kt;
  auto start = [&](int cc) {
    return static_cast<int>(static_cast<long long>(W) * cc / grid);
  };
  const int tb = start(c);
  if (tb % p.n_kt == 0) return;  // the boundary falls between pairs
  const int item = tb / p.n_kt;
  const int prev = start(c - 1);
  if (c > 1 && prev / p.n_kt == item && prev % p.n_kt != 0) return;  // merged at an earlier boundary
  auto owner = [&](int t) {
    return static_cast<int>(((static_cast<long long>(t) + 1) * grid - 1) / W);
  };
  const int c_first = owner(item * p.n_kt);
  const int n_seg = owner(item * p.n_kt + p.n_kt - 1) - c_first + 1;
  const int b = item / p.pairs;
  const int I0 = (item % p.pairs) * 2;
  const int nX = (I0 + 1 < p.nb) ? 2 : 1;
  const int tr = (blockIdx.x % kMergeBlocksPerBoundary) * kMergeRowsPerBlock +
                 static_cast<int>(threadIdx.x >> 5);  // 0 .. 255
  const int X = tr >> 7, r = tr & 127;
  if (X >= nX) return;
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int h = r >> 4, il = r & 15;
  const int pos = (I0 + X) * 16 + il;
  if (pos >= p.L) return;  // past the end of a partial last block
  const size_t row = (static_cast<size_t>(b) * kH + h) * p.L +
                     static_cast<size_t>(pos);
  auto slot = [&](int s) {
    return (static_cast<size_t>(c_first + s) * 2 + X) * 128 + r;
  };
  float M = -INFINITY;
  for (int s = 0; s < n_seg; ++s)
    M = fmaxf(M, s == 0 ? p.lse[row] : p.ws_lse[slot(s)]);
  float sum = 0.f;
  for (int s = 0; s < n_seg; ++s)
    sum += ex2_approx(((s == 0 ? p.lse[row] : p.ws_lse[slot(s)]) - M) * kLog2e);
  const float lse = M + lg2_approx(sum) * kLn2;
#pragma unroll
  for (int c = lane; c < DV / 4; c += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n_seg; ++s) {
      const float l = s == 0 ? p.lse[row] : p.ws_lse[slot(s)];
      const float wgt = ex2_approx((l - lse) * kLog2e);
      const float4 v = reinterpret_cast<const float4 *>(
          s == 0 ? p.out + row * DV : p.ws_out + slot(s) * DV)[c];
      acc.x = fmaf(wgt, v.x, acc.x);
      acc.y = fmaf(wgt, v.y, acc.y);
      acc.z = fmaf(wgt, v.z, acc.z);
      acc.w = fmaf(wgt, v.w, acc.w);
    }
    reinterpret_cast<float4 *>(p.out + row * DV)[c] = acc;
  }
  __syncwarp();  // every lane has read p.lse[row]
  if (lane == 0) p.lse[row] = lse;
}

}  // namespace attn

// --------------------------------------------------------------------------
// Host launcher.

static bool encode_map(EncodeTiledFn enc, CUtensorMap *map, const void *base,
                       int rank, const cuuint64_t *dims,
                       const cuuint64_t *strides, const cuuint32_t *box,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                   const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One-time per-device setup of a kernel (mode, value width): shared-memory
// opt-in, the register check, and how many 2-CTA clusters can be resident.
template <int MODE, int DV>
static cudaError_t configure_mode(int *max_clusters) {
  static int configured[64] = {0};
  static int clusters[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    // setmaxnreg.dec must lower the count the launch allocated: refuse a
    // build whose allocation is below the launch count the split assumes.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, attn::attn_fwd_kernel<MODE, DV>);
    if (e != cudaSuccess) return e;
    if (static_cast<uint32_t>(fa.numRegs) < attn::kRegsLaunch)
      return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn::attn_fwd_kernel<MODE, DV>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(attn::smem_bytes<DV>()));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(attn::kThreads, 1, 1);
    cfg.dynamicSmemBytes = attn::smem_bytes<DV>();
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, attn::attn_fwd_kernel<MODE, DV>, &cfg);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    clusters[dev] = n;
    configured[dev] = 1;
  }
  *max_clusters = clusters[dev];
  return cudaSuccess;
}

template <int MODE, int DV>
static cudaError_t launch_mode(const CUtensorMap &tq, const CUtensorMap &tk,
                               const CUtensorMap &tv, const attn::Params &p,
                               int clusters, cudaStream_t stream) {
  attn::attn_fwd_kernel<MODE, DV>
      <<<2 * clusters, attn::kThreads, attn::smem_bytes<DV>(), stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int DV>
static cudaError_t configure_any(int mode, int *max_clusters) {
  using namespace attn;
  switch (mode) {
    case kStaticCap: return configure_mode<kStaticCap, DV>(max_clusters);
    case kOnlineCap: return configure_mode<kOnlineCap, DV>(max_clusters);
    default: return configure_mode<kNoCap, DV>(max_clusters);
  }
}

// Grid of a call: one 2-CTA cluster per resident SM pair, never more
// clusters than (pair, key tile) steps or scratch slots.  Whole pairs per
// cluster unless that leaves the grid badly balanced: a split pair costs a
// second pass over its rows (partial results, then the merge), so whole pairs
// win while the busiest cluster's extra work stays below kSplitGain pairs.
static cudaError_t plan_grid(int mode, int dv, int n_items, int n_kt, int num_sms,
                             int scratch_slots, int *clusters_out, int *whole_out) {
  int max_clusters = 0;
  cudaError_t e = dv == 192 ? configure_any<192>(mode, &max_clusters)
                            : configure_any<128>(mode, &max_clusters);
  if (e != cudaSuccess) return e;
  const long long steps = static_cast<long long>(n_items) * n_kt;
  if (steps > (1ll << 30)) return cudaErrorInvalidValue;
  int clusters = num_sms / 2;
  if (max_clusters < clusters) clusters = max_clusters;
  if (scratch_slots < clusters) clusters = scratch_slots;
  if (steps < clusters) clusters = static_cast<int>(steps);
  if (clusters < 1) return cudaErrorInvalidValue;
  constexpr double kSplitGain = 0.5;
  const long long per = (n_items + clusters - 1) / clusters;  // busiest cluster
  const double even = static_cast<double>(n_items) / clusters;
  const int whole = (per - even <= kSplitGain) ? 1 : 0;
  if (whole && n_items < clusters) clusters = n_items;
  *clusters_out = clusters;
  *whole_out = whole;
  return cudaSuccess;
}

static int attn_mode(float cap) {
  using namespace attn;
  if (isinf(cap)) return kNoCap;
  return cap <= 40.0f ? kStaticCap : kOnlineCap;
}

cudaError_t attn_fwd_kernel_count(int64_t B, int64_t L, int64_t Dv, float cap,
                                  int num_sms, int scratch_slots, int *count) {
  using namespace attn;
  if (B == 0 || L == 0) {
    *count = 0;
    return cudaSuccess;
  }
  const int nb = static_cast<int>((L + 15) / 16);
  const int n_items = static_cast<int>(B) * ((nb + 1) / 2);
  const int n_kt = static_cast<int>((L + kKeys - 1) / kKeys);
  int clusters = 0, whole = 0;
  cudaError_t e = plan_grid(attn_mode(cap), static_cast<int>(Dv), n_items, n_kt,
                            num_sms, scratch_slots, &clusters, &whole);
  if (e != cudaSuccess) return e;
  *count = (clusters < 2 || whole) ? 1 : 2;
  return cudaSuccess;
}

cudaError_t launch_attn_fwd(const AttnLaunch &a) {
  using namespace attn;
  const int64_t B = a.B, L = a.L;
  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dims[4] = {kD, static_cast<cuuint64_t>(L), kH,
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {kD * 2, static_cast<cuuint64_t>(L) * kD * 2,
                                   static_cast<cuuint64_t>(L) * kD * 2 * kH};
    const cuuint32_t box[4] = {64, 16, kH, 1};
    if (!encode_map(a.encode, &tq, a.q, 4, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {kD, static_cast<cuuint64_t>(L),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {kD * 2, static_cast<cuuint64_t>(L) * kD * 2};
    const cuuint32_t kbox[3] = {64, kKeys / 2, 1};  // a CTA's 64 keys, one 64-wide half
    if (!encode_map(a.encode, &tk, a.k, 3, dims, strides, kbox))
      return cudaErrorInvalidValue;
    // V [B, L, Dv]: a box is one swizzle atom column of a CTA's value half.
    const cuuint64_t vdims[3] = {static_cast<cuuint64_t>(a.Dv),
                                 static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(B)};
    const cuuint64_t vstrides[2] = {static_cast<cuuint64_t>(a.Dv) * 2,
                                    static_cast<cuuint64_t>(L) * a.Dv * 2};
    const bool dv192 = a.Dv == 192;
    const cuuint32_t vbox[3] = {
        static_cast<cuuint32_t>(dv192 ? VLayout<192>::kBoxCols : VLayout<128>::kBoxCols),
        kKeys, 1};
    if (!encode_map(a.encode, &tv, a.v, 3, vdims, vstrides, vbox,
                    dv192 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  Params p;
  p.bias = a.bias;
  p.out = a.out;
  p.lse = a.lse;
  p.err = a.err;
  p.L = static_cast<int>(L);
  p.P = static_cast<int>((L + 15) / 16);
  p.nb = p.P;
  p.bias_bstride = a.bias_bstride;
  p.pairs = (p.nb + 1) / 2;
  p.n_items = static_cast<int>(B) * p.pairs;
  p.n_kt = static_cast<int>((L + kKeys - 1) / kKeys);
  p.last_valid = static_cast<int>(L - static_cast<int64_t>(p.n_kt - 1) * kKeys);
  const float cap = a.cap;
  const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(kD));
  const int mode = attn_mode(cap);
  if (mode == kNoCap) {
    p.qk_scale = inv_sqrt_d * kLog2e;
    p.bias_mul = kLog2e;
    p.A = 0.f;
  } else {
    p.qk_scale = inv_sqrt_d / cap;
    p.bias_mul = 1.0f / cap;
    p.A = cap * kLog2e;
  }
  if (a.Dv != 128 && a.Dv != 192) return cudaErrorInvalidValue;
  const int dv = static_cast<int>(a.Dv);
  int clusters = 0;
  cudaError_t e = plan_grid(mode, dv, p.n_items, p.n_kt, a.num_sms, a.scratch_slots,
                            &clusters, &p.whole);
  if (e != cudaSuccess) return e;
  if (static_cast<long long>(p.n_items) * p.n_kt != attn_work_steps(B, L))
    return cudaErrorInvalidValue;
  char *base = static_cast<char *>(a.scratch);
  p.ws_out = reinterpret_cast<float *>(base);
  p.ws_lse = reinterpret_cast<float *>(base + a.scratch_slots * kAttnSlotOutBytes);
  if (dv == 192) {
    switch (mode) {
      case kStaticCap: e = launch_mode<kStaticCap, 192>(tq, tk, tv, p, clusters, a.stream); break;
      case kOnlineCap: e = launch_mode<kOnlineCap, 192>(tq, tk, tv, p, clusters, a.stream); break;
      default: e = launch_mode<kNoCap, 192>(tq, tk, tv, p, clusters, a.stream); break;
    }
  } else {
    switch (mode) {
      case kStaticCap: e = launch_mode<kStaticCap, 128>(tq, tk, tv, p, clusters, a.stream); break;
      case kOnlineCap: e = launch_mode<kOnlineCap, 128>(tq, tk, tv, p, clusters, a.stream); break;
      default: e = launch_mode<kNoCap, 128>(tq, tk, tv, p, clusters, a.stream); break;
    }
  }
  if (e != cudaSuccess || clusters < 2 || p.whole) return e;
  const int merge_blocks = (clusters - 1) * kMergeBlocksPerBoundary;
  if (dv == 192)
    attn_merge_kernel<192><<<merge_blocks, kMergeThreads, 0, a.stream>>>(p, clusters);
  else
    attn_merge_kernel<128><<<merge_blocks, kMergeThreads, 0, a.stream>>>(p, clusters);
  return cudaGetLastError();
}

}  // namespace ag
