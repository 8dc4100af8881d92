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
//    heads.  Every row of the tile then shares one 16-position bias row block
//    and all 8 heads consume the same K/V tile (multi-query sharing), so each
//    K/V byte staged in shared memory feeds eight heads.
//  * Work is a pair of query tiles (A and B) against a range of key tiles.
//    One persistent CTA per SM takes a contiguous, equal share of all
//    (pair, key tile) steps, so the grid finishes together; a pair whose key
//    range is split between CTAs is merged exactly from the pieces' partial
//    results by log-sum-exp (see "Split pairs" below).
//  * Inside a CTA the producer warp streams Q tiles and a ring of K and V
//    tiles with TMA; the MMA warp issues every tcgen05.mma from one thread;
//    four softmax warpgroups each own one 32-key chunk of every key tile.
//    The MMA order per key tile j is PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so
//    the softmax warps work on one tile while the tensor core works on the
//    other.
//  * Tensor memory (512 columns): S_A, S_B (fp32 128x128 logits), O_A, O_B
//    (fp32 128x128 accumulators).  P is written as bf16 over part of its S
//    and fed to the PV product straight from tensor memory.
//  * Bias: each softmax thread owns one row, so per 128-key tile it needs
//    just the compact cells of its key chunk, read from global (L2) one tile
//    ahead and kept in registers; the 16x repeat is never built.
//  * With a finite cap every logit lies in (-cap, cap), so the softmax uses
//    the fixed shift m = cap (exact: softmax is shift invariant) and needs no
//    running max and no rescaling of O.  cap > 40 (where exp(-2 cap) would
//    underflow fp32) and cap = +inf use a running max with lazy rescaling.
//  * Every wait is bounded (sm100.cuh); on timeout the kernel records the
//    wait site in the device error word, drains its own copies and MMAs,
//    frees tensor memory and returns.
#include "ag_internal.h"
#include "sm100.cuh"

namespace ag {
namespace attn {

constexpr int kH = 8;
constexpr int kD = 128;
constexpr int kKeys = static_cast<int>(kAttnKeyTile);  // keys per K/V tile
static_assert(kKeys == 128, "the tile layout below assumes 128-key tiles");
constexpr int kStages = 4;                  // K/V ring slots
constexpr int kTileBytes = 128 * 128 * 2;   // one Q, K or V tile (bf16)
constexpr int kHalfBytes = kTileBytes / 2;  // one 64-wide (128-byte) half
// Softmax warpgroups (2 or 4).  Warps 0 .. 4*kWG-1 run the softmax; the next
// warpgroup holds the TMA producer warp, the MMA warp and two idle warps
// (present so that it is whole for the register re-allocation).
#ifndef AG_SOFTMAX_WARPGROUPS
#define AG_SOFTMAX_WARPGROUPS 4
#endif
constexpr int kWG = AG_SOFTMAX_WARPGROUPS;
static_assert(kWG == 2 || kWG == 4, "two or four softmax warpgroups");
constexpr int kChunks = 4 / kWG;             // 32-column chunks per warpgroup
constexpr int kSoftThreads = 128 * kWG;
constexpr int kNumWarps = 4 * kWG + 4;
constexpr int kThreads = kNumWarps * 32;
constexpr int kWarpLoad = 4 * kWG;
constexpr int kWarpMma = 4 * kWG + 1;
// Registers per thread: the launch gives every thread kRegsLaunch (the cap
// for this block size, which ptxas allocates when setmaxnreg is present; the
// launcher checks it).  The producer warpgroup then drops to kRegsLow and,
// where kRegsHigh exceeds the launch count, the softmax warpgroups rise to
// it.  (With four softmax warpgroups the softmax needs no more than the
// launch count, and a producer cap below 80 makes the MMA warp spill.)
constexpr uint32_t kRegsLaunch = kWG == 2 ? 168 : 96;
constexpr uint32_t kRegsLow = kWG == 2 ? 88 : 80;
constexpr uint32_t kRegsHigh = kWG == 2 ? 208 : 96;
static_assert(kSoftThreads * kRegsHigh + 128 * kRegsLow <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
// P (bf16 pairs) of a tile: keys [32c, 32c + 32) of chunk c are written over
// the first 16 columns of that chunk's own S columns, [32c, 32c + 16).
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);  // K-major B (K)
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 1);  // MN-major B (V)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Lazy rescale threshold (log2 units) for the running-max modes.
constexpr float kRescaleThreshold = 8.0f;

enum Mode { kStaticCap = 0, kOnlineCap = 1, kNoCap = 2 };

// Wait sites recorded in the device error word.
enum Site : unsigned {
  kSiteProdQ = 1, kSiteProdKV = 2, kSiteMmaQ = 3, kSiteMmaKV = 4,
  kSiteMmaP = 5, kSiteSoftS = 6, kSiteSoftO = 7, kSiteDrain = 8,
  kSiteXchg = 9
};

struct __align__(8) Barriers {
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t xm[2], xd[2];  // row-max / row-sum exchange between warpgroups
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int range_begin, range_end;  // this CTA's (pair, key tile) steps
};

constexpr size_t kXchgBytes = 2 * 2 * kWG * 128 * sizeof(float);
constexpr size_t kSmemBytes = 1024 + (2 + kStages) * static_cast<size_t>(kTileBytes) +
                              sizeof(Barriers) + kXchgBytes;

struct Params {
  const float *bias;
  float *out;
  float *lse;
  unsigned *err;
  // Split-pair scratch (see "Split pairs"): one slot per CTA.
  float *ws_out;       // [grid][2][128][128] partial outputs
  float *ws_lse;       // [grid][2][128] partial log-sum-exps
  int L, P;
  int nb;          // 16-position query blocks per batch item (L / 16)
  int pairs;       // query-tile pairs per batch item: ceil(nb / 2)
  int n_items;     // B * pairs
  int n_kt;        // key tiles: ceil(L / 128)
  int last_valid;  // valid keys in the last key tile (1..128)
  int whole;       // 1: CTA ranges hold whole pairs (no split pairs)
  float qk_scale;  // multiplies q.k
  float bias_mul;  // multiplies the compact bias
  float A;         // capped modes: cap * log2(e)
};

// --------------------------------------------------------------------------
// Work split.  The W = n_items * n_kt (pair, key tile) steps are cut into
// gridDim.x contiguous ranges [W c / G, W (c+1) / G).  A CTA walks its range
// as segments: one pair and a run of its key tiles.  A pair covered by more
// than one CTA is "split"; its pieces are merged by the last one to finish.
struct Segment {
  int item, kb, ke;  // pair index and key tiles [kb, ke)
};

// W = n_items * n_kt <= 2^30 (checked by the launcher), so steps fit in int;
// only the range bounds need a 64-bit product.  With p.whole the bounds are
// rounded to whole pairs: CTA c gets pairs [n_items c / G, n_items (c+1) / G).
__device__ __forceinline__ int range_start(const Params &p, int c) {
  if (p.whole)
    return static_cast<int>(static_cast<long long>(p.n_items) * c /
                            static_cast<long long>(gridDim.x)) * p.n_kt;
  return static_cast<int>(static_cast<long long>(p.n_items) * p.n_kt * c /
                          static_cast<long long>(gridDim.x));
}

__device__ __forceinline__ Segment segment_at(const Params &p, int t, int end) {
  Segment sg;
  sg.item = t / p.n_kt;
  sg.kb = t - sg.item * p.n_kt;
  const int left = end - t;
  sg.ke = left < p.n_kt - sg.kb ? sg.kb + left : p.n_kt;
  return sg;
}

// --------------------------------------------------------------------------
// MMA issue helpers (single thread).

// Shared-memory descriptors: every operand here has 8-row groups 1 KB apart,
// so all share one high word; the low word (start address and leading
// offset) is built once per tile base and each K step adds a constant to its
// start-address field (addresses stay below 2^18: no carry out of the field).
constexpr uint32_t kDescHi = desc_sw128_hi(1024);

// S[128 x 128] = Q[128 x 128] K^T: eight K=16 steps over two 64-wide halves.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr,
                                         uint32_t k_addr) {
  const uint32_t q_lo = desc_sw128_lo(q_addr, 16), k_lo = desc_sw128_lo(k_addr, 16);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
    umma_ss_lo(d_tmem, q_lo + off, k_lo + off, kDescHi, kIdescQK, kk > 0 ? 1u : 0u);
  }
}

// O[128 x 128] (+)= P[128 x 128 keys] V[128 keys x 128]: P from tensor memory
// (bf16 pairs, 8 columns per 16 keys; keys 32c.. of chunk c start at column
// 32c of the S region), V MN-major in shared memory (the two 64-wide halves
// are 16 KB apart, 8-key row groups 1 KB apart).
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t s_tmem,
                                         uint32_t v_addr, bool accumulate) {
  const uint32_t v_lo = desc_sw128_lo(v_addr, kHalfBytes);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    umma_ts_lo(d_tmem, s_tmem + 32 * (kk >> 1) + 8 * (kk & 1),
               v_lo + ((kk * 2048) >> 4), kDescHi, kIdescPV,
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

// --------------------------------------------------------------------------
// Producer warp, lane 0: TMA loads.
__device__ __forceinline__ void producer(const CUtensorMap *tm_q,
                                         const CUtensorMap *tm_k,
                                         const CUtensorMap *tm_v, uint8_t *q_s,
                                         uint8_t *kv_s, Barriers *bars,
                                         const Params &p, volatile int *abort) {
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  uint32_t qcount[2] = {0, 0};
  uint32_t kv = 0;
  bool ok = true;
  const int end = bars->range_end;
  for (int t = bars->range_begin; t < end && ok;) {
    const Segment sg = segment_at(p, t, end);
    t += sg.ke - sg.kb;
    const int b = sg.item / p.pairs;
    const int I0 = (sg.item % p.pairs) * 2;
    const int nX = (I0 + 1 < p.nb) ? 2 : 1;
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      if (X >= nX) break;
      ok = mbar_wait(&bars->q_empty[X], (qcount[X] & 1u) ^ 1u, abort, p.err,
                     kSiteProdQ);
      if (!ok) break;
      mbar_arrive_expect_tx(&bars->q_full[X], kTileBytes);
      uint8_t *dst = q_s + X * kTileBytes;
      tma_load_4d(dst, tm_q, &bars->q_full[X], 0, (I0 + X) * 16, 0, b, pol_q);
      tma_load_4d(dst + kHalfBytes, tm_q, &bars->q_full[X], 64, (I0 + X) * 16,
                  0, b, pol_q);
      ++qcount[X];
    }
    for (int j = sg.kb; j < sg.ke && ok; ++j) {
#pragma unroll 1
      for (int u = 0; u < 2; ++u) {  // u = 0: K tile j, u = 1: V tile j
        const uint32_t slot = kv % kStages, ph = (kv / kStages) & 1u;
        ok = mbar_wait(&bars->kv_empty[slot], ph ^ 1u, abort, p.err, kSiteProdKV);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->kv_full[slot], kTileBytes);
        uint8_t *dst = kv_s + slot * kTileBytes;
        const CUtensorMap *tm = u == 0 ? tm_k : tm_v;
        tma_load_3d(dst, tm, &bars->kv_full[slot], 0, j * kKeys, b, pol_kv);
        tma_load_3d(dst + kHalfBytes, tm, &bars->kv_full[slot], 64, j * kKeys, b,
                    pol_kv);
        ++kv;
      }
    }
  }
  // Every copy this thread started must land before the CTA exits.
  for (int X = 0; X < 2; ++X)
    if (qcount[X] > 0) drain_wait(&bars->q_full[X], (qcount[X] - 1) & 1u);
  const uint32_t first = kv > kStages ? kv - kStages : 0;
  for (uint32_t i = first; i < kv; ++i)
    drain_wait(&bars->kv_full[i % kStages], (i / kStages) & 1u);
}

// --------------------------------------------------------------------------
// MMA warp, lane 0: tcgen05.mma issuer.
__device__ __forceinline__ void mma_issuer(uint8_t *q_s, uint8_t *kv_s,
                                           Barriers *bars, uint32_t tmem,
                                           const Params &p, volatile int *abort) {
  const uint32_t q_addr = smem_u32(q_s);
  const uint32_t kv_addr = smem_u32(kv_s);
  uint32_t qcount[2] = {0, 0}, pcount[2] = {0, 0};
  uint32_t kv = 0;
  bool ok = true;
  const int end = bars->range_end;
  for (int t = bars->range_begin; t < end && ok;) {
    const Segment sg = segment_at(p, t, end);
    t += sg.ke - sg.kb;
    const int I0 = (sg.item % p.pairs) * 2;
    const int nX = (I0 + 1 < p.nb) ? 2 : 1;
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      if (X >= nX || !ok) break;
      ok = mbar_wait(&bars->q_full[X], qcount[X] & 1u, abort, p.err, kSiteMmaQ);
      ++qcount[X];
    }
    if (!ok) break;
    // First key tile of the segment: S_X(kb) for both query tiles.
    const int n = sg.ke - sg.kb;
    const uint32_t slot_k0 = kv % kStages;
    ok = mbar_wait(&bars->kv_full[slot_k0], (kv / kStages) & 1u, abort, p.err,
                   kSiteMmaKV);
    if (!ok) break;
    ++kv;
    tc_fence_after();
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      if (X >= nX) break;
      issue_qk(tmem + X * 128, q_addr + X * kTileBytes,
               kv_addr + slot_k0 * kTileBytes);
      umma_commit(&bars->s_full[X]);
      if (n == 1) umma_commit(&bars->q_empty[X]);
    }
    umma_commit(&bars->kv_empty[slot_k0]);

    for (int i = 0; i < n && ok; ++i) {
      const uint32_t slot_v = kv % kStages;
      ok = mbar_wait(&bars->kv_full[slot_v], (kv / kStages) & 1u, abort, p.err,
                     kSiteMmaKV);
      if (!ok) break;
      ++kv;
      const bool has_next = i + 1 < n;
      uint32_t slot_k = 0;
      bool k_ready = false;
#pragma unroll
      for (int X = 0; X < 2; ++X) {
        if (X >= nX) break;
        ok = mbar_wait(&bars->p_full[X], pcount[X] & 1u, abort, p.err, kSiteMmaP);
        ++pcount[X];
        if (!ok) break;
        tc_fence_after();
        issue_pv(tmem + 256 + X * 128, tmem + X * 128,
                 kv_addr + slot_v * kTileBytes, i > 0);
        if (!has_next) {
          umma_commit(&bars->o_full[X]);
          continue;
        }
        if (!k_ready) {
          slot_k = kv % kStages;
          ok = mbar_wait(&bars->kv_full[slot_k], (kv / kStages) & 1u, abort,
                         p.err, kSiteMmaKV);
          if (!ok) break;
          ++kv;
          k_ready = true;
          tc_fence_after();
        }
        issue_qk(tmem + X * 128, q_addr + X * kTileBytes,
                 kv_addr + slot_k * kTileBytes);
        umma_commit(&bars->s_full[X]);
        if (i + 2 == n) umma_commit(&bars->q_empty[X]);
      }
      if (!ok) break;
      umma_commit(&bars->kv_empty[slot_v]);
      if (k_ready) umma_commit(&bars->kv_empty[slot_k]);
    }
  }
  // All MMAs this thread issued complete before tensor memory is released.
  umma_commit(&bars->drain);
  drain_wait(&bars->drain, 0);
}

// --------------------------------------------------------------------------
// Softmax warpgroups.
//
// All softmax warps work on query tile A, then all on tile B, then A again:
// warpgroup g takes the kChunks 32-key chunks starting at key 32*kChunks*g of
// every 128-key tile, for all 128 rows (thread r of every warpgroup owns
// tensor-memory lane r).  While the warps run one tile's softmax the tensor
// core runs the other tile's PV and next QK^T, so the two alternate without
// further synchronisation.  A row's sum is split between its kWG threads and
// combined through shared memory once per work item.  Each chunk's P goes over
// the first half of that chunk's own S columns, so a warpgroup only ever
// overwrites S columns it has already read itself.

// Softmax-side shared memory: row-sum and row-max exchange between the kWG
// threads of a row.
struct Xchg {
  float dpart[2][kWG][128];  // [tile][warpgroup][row]
  float mpart[2][kWG][128];
};

// Softmax-side barriers count warps: each warp arrives once, from lane 0,
// after __syncwarp has ordered its lanes' prior work (one arrival per warp
// instead of 32 keeps the mbarrier off the shared-memory pipe).
constexpr uint32_t kSoftWarps = kSoftThreads / 32;

__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
  __syncwarp();
  if (lane_id() == 0) mbar_arrive(bar);
}

// Publish this thread's value, then wait (bounded) until every softmax thread
// has published its own.  The warp barrier and the mbarrier's arrive/wait
// order the shared-memory writes before the partners' reads.
__device__ __forceinline__ bool exchange(uint64_t *bar, uint32_t &count,
                                         volatile int *abort, unsigned *err) {
  warp_arrive(bar);
  const bool ok = mbar_wait(bar, count & 1u, abort, err, kSiteXchg);
  ++count;
  return __all_sync(0xffffffffu, ok);
}

// The compact bias cells of this warpgroup's keys of key tile j (two per
// 32-key chunk): bias[h, I, 8j + 2*kChunks*g + e].
__device__ __forceinline__ void load_bias(const float *brow, int j, int g, int P,
                                          float (&bn)[2 * kChunks]) {
  const int J0 = j * 8 + g * 2 * kChunks;
#pragma unroll
  for (int e = 0; e < 2 * kChunks; ++e)
    bn[e] = (J0 + e < P) ? __ldg(brow + J0 + e) : 0.f;
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
    float2 p;
    if ((e & 7) < kEmuPairs) {
      p = exp2_poly2(x);
    } else {
      p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    }
    if (kMask) {
      if (col0 + 2 * e >= nvalid) p.x = 0.f;
      if (col0 + 2 * e + 1 >= nvalid) p.y = 0.f;
    }
    acc = __fadd2_rn(acc, p);
    pk[e] = pack_bf16x2(p.x, p.y);
  }
}

// This warpgroup's chunks of one tile, static shift: S in, P out over the
// first 16 columns of each chunk.  Returns the partial row sum.
template <bool kMask>
__device__ __forceinline__ float part_tile_static(uint32_t tS, int g,
                                                  const float (&bj)[2 * kChunks],
                                                  float2 sc, float2 ap, float2 an,
                                                  int nvalid) {
  float2 acc = make_float2(0.f, 0.f);
  uint32_t pk[16];
  if constexpr (kChunks == 1) {
    uint32_t sa[32];
    const uint32_t c0 = 32 * g;
    tmem_ld32(tS + c0, sa);
    tmem_wait_ld(sa);
    chunk_static<kMask>(sa, bj[0], bj[1], sc, ap, an, c0, nvalid, acc, pk);
    tmem_st16(tS + c0, pk);
  } else {
    uint32_t sa[32], sb[32];
    const uint32_t c0 = 64 * g;
    tmem_ld32(tS + c0, sa);
    tmem_wait_ld(sa);
    tmem_ld32(tS + c0 + 32, sb);
    chunk_static<kMask>(sa, bj[0], bj[1], sc, ap, an, c0, nvalid, acc, pk);
    tmem_st16(tS + c0, pk);
    tmem_wait_ld(sb);
    chunk_static<kMask>(sb, bj[2], bj[3], sc, ap, an, c0 + 32, nvalid, acc, pk);
    tmem_st16(tS + c0 + 32, pk);
  }
  return acc.x + acc.y;
}

// Log2-domain logits of one chunk for the running-max modes.
template <int MODE>
__device__ __forceinline__ void chunk_logits(const uint32_t (&s)[32], float b0,
                                             float b1, const Params &p, int col0,
                                             int nvalid, float (&x)[32]) {
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const float bb = c < 16 ? b0 : b1;
    const float y = fmaf(__uint_as_float(s[c]), p.qk_scale, bb);
    float v = (MODE == kOnlineCap) ? p.A * tanh_approx(y) : y;
    x[c] = (col0 + c < nvalid) ? v : -INFINITY;
  }
}

// This warpgroup's chunks of one tile with a running maximum shared by the
// kWG threads of each row (exchanged through shared memory).  Rescales this
// warpgroup's columns of O when the maximum grows past the lazy threshold.
template <int MODE>
__device__ __forceinline__ bool part_tile_online(uint32_t tS, uint32_t tO, int g,
                                                 int r, int X, int i,
                                                 const float (&bj)[2 * kChunks],
                                                 const Params &p, int nvalid,
                                                 Xchg *xc, uint64_t *xbar,
                                                 uint32_t &xcount,
                                                 volatile int *abort, float &m,
                                                 float &d) {
  const uint32_t c0 = 32 * kChunks * g;
  float mt = -INFINITY;
#pragma unroll 1
  for (int c = 0; c < kChunks; ++c) {
    uint32_t s[32];
    float x[32];
    tmem_ld32(tS + c0 + c * 32, s);
    tmem_wait_ld(s);
    chunk_logits<MODE>(s, bj[2 * c], bj[2 * c + 1], p, c0 + c * 32, nvalid, x);
#pragma unroll
    for (int e = 0; e < 32; ++e) mt = fmaxf(mt, x[e]);
  }
  xc->mpart[X][g][r] = mt;
  if (!exchange(xbar, xcount, abort, p.err)) return false;
#pragma unroll
  for (int q = 0; q < kWG; ++q) mt = fmaxf(mt, xc->mpart[X][q][r]);
  float factor = 1.f;
  if (mt > m + kRescaleThreshold || m == -INFINITY) {
    factor = (m == -INFINITY) ? 0.f : ex2_approx(m - mt);
    m = mt;
    d *= factor;
  }
  if (i > 0 && __any_sync(0xffffffffu, factor != 1.f)) {
    // The previous tile's PV into O is complete: this tile's s_full was
    // committed after it.  (Before the first tile O holds nothing yet.)
#pragma unroll 1
    for (int c = 0; c < kChunks; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + c0 + c * 32, o);
      tmem_wait_ld(o);
#pragma unroll
      for (int e = 0; e < 32; ++e)
        o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
      tmem_st32(tO + c0 + c * 32, o);
    }
  }
  float acc = 0.f;
#pragma unroll 1
  for (int c = 0; c < kChunks; ++c) {
    uint32_t s[32], pk[16];
    float x[32];
    tmem_ld32(tS + c0 + c * 32, s);
    tmem_wait_ld(s);
    chunk_logits<MODE>(s, bj[2 * c], bj[2 * c + 1], p, c0 + c * 32, nvalid, x);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float p0 = ex2_approx(x[2 * e] - m);
      const float p1 = ex2_approx(x[2 * e + 1] - m);
      acc += p0 + p1;
      pk[e] = pack_bf16x2(p0, p1);
    }
    tmem_st16(tS + c0 + c * 32, pk);
  }
  d += acc;
  return true;
}

// --------------------------------------------------------------------------
// Split pairs.  Every segment of a split pair finishes like a whole pair but
// over its own key range: a normalised partial output and the partial
// log-sum-exp.  The first segment (key tile 0) writes them to out / lse, the
// others to the scratch slot of their CTA (a CTA starts at most one segment in
// the middle of a pair).  attn_merge_kernel, launched right after on the same
// stream, then merges the pieces of every split pair:
//   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) out_s.

template <int MODE>
__device__ __forceinline__ void softmax_role(Barriers *bars, Xchg *xc,
                                             uint32_t tmem, const Params &p,
                                             volatile int *abort) {
  const int g = threadIdx.x >> 7;         // warpgroup: which key chunks
  const int r = threadIdx.x & 127;        // tile row == tensor-memory lane
  const int wq = r >> 5;                  // warp's lane quarter
  const int h = r >> 4, il = r & 15;      // head, position inside the block
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const float2 sc = make_float2(p.qk_scale, p.qk_scale);
  const float2 ap = make_float2(p.A, p.A), an = make_float2(-p.A, -p.A);
  uint32_t scount[2] = {0, 0}, ocount[2] = {0, 0};
  uint32_t xmcount[2] = {0, 0}, xdcount[2] = {0, 0};
  bool ok = true;
  const int end = bars->range_end;

  for (int t = bars->range_begin; t < end && ok;) {
    const Segment sg = segment_at(p, t, end);
    t += sg.ke - sg.kb;
    const int b = sg.item / p.pairs;
    const int I0 = (sg.item % p.pairs) * 2;
    const int nX = (I0 + 1 < p.nb) ? 2 : 1;
    const float *const brow[2] = {
        p.bias + (static_cast<size_t>(h) * p.P + I0) * p.P,
        p.bias + (static_cast<size_t>(h) * p.P + (I0 + (nX > 1 ? 1 : 0))) * p.P};
    float m[2], d[2] = {0.f, 0.f};
    float bn[2][2 * kChunks];
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      m[X] = (MODE == kStaticCap) ? p.A : -INFINITY;  // log2 units
      load_bias(brow[X], sg.kb, g, p.P, bn[X]);
    }
    for (int j = sg.kb, i = 0; j < sg.ke && ok; ++j, ++i) {
      const int nvalid = (j + 1 == p.n_kt) ? p.last_valid : kKeys;
#pragma unroll
      for (int X = 0; X < 2; ++X) {
        if (X >= nX) break;
        float bj[2 * kChunks];
#pragma unroll
        for (int e = 0; e < 2 * kChunks; ++e) bj[e] = bn[X][e] * p.bias_mul;
        if (j + 1 < sg.ke) load_bias(brow[X], j + 1, g, p.P, bn[X]);

        ok = mbar_wait(&bars->s_full[X], scount[X] & 1u, abort, p.err, kSiteSoftS);
        ++scount[X];
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tmem + X * 128 + lane_base;
        if constexpr (MODE == kStaticCap) {
          if (nvalid == kKeys)
            d[X] += part_tile_static<false>(tS, g, bj, sc, ap, an, nvalid);
          else
            d[X] += part_tile_static<true>(tS, g, bj, sc, ap, an, nvalid);
        } else {
          const uint32_t tO = tmem + 256 + X * 128 + lane_base;
          ok = part_tile_online<MODE>(tS, tO, g, r, X, i, bj, p, nvalid, xc,
                                      &bars->xm[X], xmcount[X], abort, m[X], d[X]);
          if (!ok) break;
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(&bars->p_full[X]);
      }
    }
    if (!ok) break;

    // Epilogue: d = sum of the kWG partial sums; out = O / d over this
    // segment's keys (this warpgroup's 32*kChunks columns of the row) and
    // lse, to out / lse or, for a later piece of a split pair, to this CTA's
    // scratch slot.
#pragma unroll
    for (int X = 0; X < 2; ++X) {
      if (X >= nX) break;
      ok = mbar_wait(&bars->o_full[X], ocount[X] & 1u, abort, p.err, kSiteSoftO);
      ++ocount[X];
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      xc->dpart[X][g][r] = d[X];
      ok = exchange(&bars->xd[X], xdcount[X], abort, p.err);
      if (!ok) break;
      float dsum = 0.f;
#pragma unroll
      for (int q = 0; q < kWG; ++q) dsum += xc->dpart[X][q][r];
      const float inv_d = 1.f / dsum;
      const size_t row = (static_cast<size_t>(b) * kH + h) * p.L +
                         static_cast<size_t>(I0 + X) * 16 + il;
      const int c0 = 32 * kChunks * g;
      float *orow_base;
      float *lse_dst;
      if (sg.kb == 0) {
        orow_base = p.out + row * kD;
        lse_dst = p.lse + row;
      } else {
        const size_t slot = (static_cast<size_t>(blockIdx.x) * 2 + X) * 128 + r;
        orow_base = p.ws_out + slot * kD;
        lse_dst = p.ws_lse + slot;
      }
      float4 *orow = reinterpret_cast<float4 *>(orow_base + c0);
      const uint32_t tO = tmem + 256 + X * 128 + lane_base + c0;
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld(o);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          orow[c * 8 + e] = make_float4(__uint_as_float(o[4 * e]) * inv_d,
                                        __uint_as_float(o[4 * e + 1]) * inv_d,
                                        __uint_as_float(o[4 * e + 2]) * inv_d,
                                        __uint_as_float(o[4 * e + 3]) * inv_d);
        }
      }
      if (g == 0) *lse_dst = (m[X] + lg2_approx(dsum)) * kLn2;
      tc_fence_before();
    }
  }
}

// --------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *q_s = smem_raw + pad;                 // 2 query tiles
  uint8_t *kv_s = q_s + 2 * kTileBytes;          // K/V ring
  Barriers *bars = reinterpret_cast<Barriers *>(kv_s + kStages * kTileBytes);
  auto *xc = reinterpret_cast<struct Xchg *>(reinterpret_cast<uint8_t *>(bars) +
                                             sizeof(Barriers));
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int X = 0; X < 2; ++X) {
      mbar_init(&bars->q_full[X], 1);
      mbar_init(&bars->q_empty[X], 1);
      mbar_init(&bars->s_full[X], 1);
      mbar_init(&bars->p_full[X], kSoftWarps);
      mbar_init(&bars->xm[X], kSoftWarps);
      mbar_init(&bars->xd[X], kSoftWarps);
      mbar_init(&bars->o_full[X], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    bars->range_begin = range_start(p, blockIdx.x);
    bars->range_end = range_start(p, blockIdx.x + 1);
    fence_mbar_init();
  }
  if (warp == kWarpLoad && lane_id() == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;

  if (warp >= kWarpLoad) {
    regs_dec<kRegsLow>();
    if (warp == kWarpLoad && lane_id() == 0)
      producer(&tm_q, &tm_k, &tm_v, q_s, kv_s, bars, p, abort);
    else if (warp == kWarpMma && lane_id() == 0)
      mma_issuer(q_s, kv_s, bars, tmem, p, abort);
  } else {
    if constexpr (kRegsHigh > kRegsLaunch) regs_inc<kRegsHigh>();
    softmax_role<MODE>(bars, xc, tmem, p, abort);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------------------
// Split-pair merge.  One block per CTA boundary; the block whose boundary is
// the first one inside a pair merges that pair.  Thread t takes query tile
// t / 128 and row t % 128 and merges the whole 128-column row, so it reads
// the first piece's lse before it overwrites it.
constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
    attn_merge_kernel(const Params p, int grid) {
  const int c = blockIdx.x + 1;  // boundary between CTA c - 1 and CTA c
  const int W = p.n_items * p.n_kt;
  auto start = [&](int cc) {
    return static_cast<int>(static_cast<long long>(W) * cc / grid);
  };
  const int tb = start(c);
  if (tb % p.n_kt == 0) return;  // the boundary falls between pairs
  const int item = tb / p.n_kt;
  const int prev = start(c - 1);
  if (c > 1 && prev / p.n_kt == item && prev % p.n_kt != 0) return;  // merged by an earlier block
  auto owner = [&](int t) {
    return static_cast<int>(((static_cast<long long>(t) + 1) * grid - 1) / W);
  };
  const int c_first = owner(item * p.n_kt);
  const int n_seg = owner(item * p.n_kt + p.n_kt - 1) - c_first + 1;
  const int b = item / p.pairs;
  const int I0 = (item % p.pairs) * 2;
  const int nX = (I0 + 1 < p.nb) ? 2 : 1;
  const int X = threadIdx.x >> 7, r = threadIdx.x & 127;
  if (X >= nX) return;
  const int h = r >> 4, il = r & 15;
  const size_t row = (static_cast<size_t>(b) * kH + h) * p.L +
                     static_cast<size_t>(I0 + X) * 16 + il;
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
  float4 *dst = reinterpret_cast<float4 *>(p.out + row * kD);
#pragma unroll 1
  for (int part = 0; part < kD / 16; ++part) {
    float4 acc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n_seg; ++s) {
      const float l = s == 0 ? p.lse[row] : p.ws_lse[slot(s)];
      const float wgt = ex2_approx((l - lse) * kLog2e);
      const float4 *src = reinterpret_cast<const float4 *>(
          s == 0 ? p.out + row * kD : p.ws_out + slot(s) * kD);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 v = src[part * 4 + e];
        acc[e].x = fmaf(wgt, v.x, acc[e].x);
        acc[e].y = fmaf(wgt, v.y, acc[e].y);
        acc[e].z = fmaf(wgt, v.z, acc[e].z);
        acc[e].w = fmaf(wgt, v.w, acc[e].w);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[part * 4 + e] = acc[e];
  }
  p.lse[row] = lse;
}

}  // namespace attn

// --------------------------------------------------------------------------
// Host launcher.

static bool encode_map(EncodeTiledFn enc, CUtensorMap *map, const void *base,
                       int rank, const cuuint64_t *dims,
                       const cuuint64_t *strides, const cuuint32_t *box) {
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                   const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE>
static cudaError_t launch_mode(const CUtensorMap &tq, const CUtensorMap &tk,
                               const CUtensorMap &tv, const attn::Params &p,
                               int grid, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    // setmaxnreg.inc waits until the registers it asks for are free: refuse
    // to launch a build whose launch allocation cannot cover the split.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, attn::attn_fwd_kernel<MODE>);
    if (e != cudaSuccess) return e;
    if (static_cast<uint32_t>(fa.numRegs) * attn::kThreads <
        attn::kSoftThreads * attn::kRegsHigh + 128 * attn::kRegsLow)
      return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn::attn_fwd_kernel<MODE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(attn::kSmemBytes));
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  attn::attn_fwd_kernel<MODE>
      <<<grid, attn::kThreads, attn::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
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
    const cuuint32_t box[3] = {64, kKeys, 1};
    if (!encode_map(a.encode, &tk, a.k, 3, dims, strides, box))
      return cudaErrorInvalidValue;
    if (!encode_map(a.encode, &tv, a.v, 3, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  Params p;
  p.bias = a.bias;
  p.out = a.out;
  p.lse = a.lse;
  p.err = a.err;
  p.L = static_cast<int>(L);
  p.P = static_cast<int>(L / 16);
  p.nb = static_cast<int>(L / 16);
  p.pairs = (p.nb + 1) / 2;
  p.n_items = static_cast<int>(B) * p.pairs;
  p.n_kt = static_cast<int>((L + kKeys - 1) / kKeys);
  p.last_valid = static_cast<int>(L - static_cast<int64_t>(p.n_kt - 1) * kKeys);
  const float cap = a.cap;
  const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(kD));
  int mode;
  if (isinf(cap)) {
    mode = kNoCap;
    p.qk_scale = inv_sqrt_d * kLog2e;
    p.bias_mul = kLog2e;
    p.A = 0.f;
  } else {
    mode = cap <= 40.0f ? kStaticCap : kOnlineCap;
    p.qk_scale = inv_sqrt_d / cap;
    p.bias_mul = 1.0f / cap;
    p.A = cap * kLog2e;
  }
  // One CTA per SM, never more CTAs than (pair, key tile) steps or scratch
  // slots.  Whole pairs per CTA unless that leaves the grid badly balanced:
  // a split pair costs a second pass over its rows (partial results, then
  // the merge), so whole pairs win while the busiest CTA's extra work stays
  // below kSplitGain pairs.
  const long long steps = static_cast<long long>(p.n_items) * p.n_kt;
  if (steps != attn_work_steps(B, L) || steps > (1ll << 30))
    return cudaErrorInvalidValue;
  int grid = a.num_sms < a.scratch_slots ? a.num_sms : a.scratch_slots;
  if (steps < grid) grid = static_cast<int>(steps);
  if (grid < 1) return cudaErrorInvalidValue;
  {
    constexpr double kSplitGain = 0.5;
    const long long per = (p.n_items + grid - 1) / grid;  // pairs, busiest CTA
    const double even = static_cast<double>(p.n_items) / grid;
    p.whole = (per - even <= kSplitGain) ? 1 : 0;
    if (p.whole && p.n_items < grid) grid = p.n_items;
  }
  char *base = static_cast<char *>(a.scratch);
  p.ws_out = reinterpret_cast<float *>(base);
  p.ws_lse = reinterpret_cast<float *>(base + a.scratch_slots * kAttnSlotOutBytes);
  cudaError_t e;
  switch (mode) {
    case kStaticCap: e = launch_mode<kStaticCap>(tq, tk, tv, p, grid, a.stream); break;
    case kOnlineCap: e = launch_mode<kOnlineCap>(tq, tk, tv, p, grid, a.stream); break;
    default: e = launch_mode<kNoCap>(tq, tk, tv, p, grid, a.stream); break;
  }
  if (e != cudaSuccess || grid < 2 || p.whole) return e;
  attn_merge_kernel<<<grid - 1, kMergeThreads, 0, a.stream>>>(p, grid);
  return cudaGetLastError();
}

}  // namespace ag
