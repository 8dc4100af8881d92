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
//    CTA holds one tile, and tcgen05.mma with cta_group::2 covers M = 256 rows
//    over both SMs.  Each CTA stages only half of every K tile (64 of its 128
//    keys) and half of every V tile (DV/2 value columns), so each K/V byte
//    crosses from L2 into one SM only and serves the 256 query rows of the
//    pair.  DV (value width) is 128 or 192.
//  * Tensor memory (per CTA), fixed-shift mode at value width 128: three
//    128-column step buffers (fp32 logits of key tile t in buffer t % 3, the
//    bf16 probabilities then written over the logits already read) and the
//    128-column O accumulator; the logits of tile t wait only for the PV of
//    tile t - 3.  Running-max modes and value width 192: two S buffers, one
//    or two P buffers of their own and the DV-column O.
//  * Two MMA-issuing warps in the even CTA (an elect.sync-chosen lane
//    issues): one issues every S = Q K^T and one every O += P V, each with its
//    own waits and commits, fed by separate K and V rings (TMA, no
//    multicast).  In the odd CTA two relay threads forward "loaded" to the
//    even CTA (cluster-scope arrives), so each CTA's copies complete on its
//    own barriers and can be drained locally.
//  * Fixed-shift mode at value width 128: the 16 softmax warps form two
//    groups on alternate key tiles, each warpgroup of a group 64 keys of the
//    tile, so one group's waits are covered by the other's arithmetic.
//    Otherwise all four warpgroups work on every key tile, 32 keys each.  The
//    bias of a thread's keys is one compact cell per 16 keys, read from
//    global (L2) a tile ahead and kept in registers: the 16x repeat is never
//    built.
//  * With a finite cap every logit lies in (-cap, cap), so the softmax uses a
//    fixed shift (exact: softmax is shift invariant) and needs no running max
//    and no rescaling of O (cap <= 60: beyond, the probabilities of a row
//    span more than fp32's range).  Larger caps and cap = +inf use a running
//    max with lazy rescaling.
//  * Epilogue at value width 128: each warp stages its 32 x 32 block of out
//    in shared memory and writes it with one bulk tensor store, which drains
//    while the warps go on to the next pair.
//  * Work is cut into segments (a pair of query tiles and a run of its key
//    tiles).  Three schedules: whole pairs per cluster; "two phases", where
//    some pairs are split into a first piece (first launch, result written to
//    out/lse) and a second piece (second launch, programmatic dependent
//    launch, merged with the first piece's result in its epilogue) so that
//    the grid stays balanced without any scratch memory; and contiguous
//    ranges of (pair, key tile) steps whose split pieces go through a
//    caller-provided scratch buffer and a merge kernel.
//  * Every mbarrier wait is bounded (sm100.cuh); on timeout the kernel records
//    the wait site in the device error word, drains its own copies and MMAs,
//    frees tensor memory and returns.
#include <algorithm>
#include <mutex>
#include <vector>

#include "ag_internal.h"
#include "sm100.cuh"

namespace ag {
namespace attn {

constexpr int kH = 8;
constexpr int kD = 128;

// Softmax modes (see the comment before attn_mode for the choice).
//   kStaticCap:   finite cap up to 60, fixed shift (no row maximum needed).
//   kOnlineCap:   cap > 60, running maximum with lazy rescaling.
//   kNoCap:       no soft cap, running maximum.
//   kRowMax:      first pass of the two-pass schedule (value width 128, cap
//                 > 60 or none): each row's largest logit, into lse.
//   kRowShift:    second pass without a cap: the fixed-shift kernel with the
//                 row's own shift ceil(max) read from lse.
//   kRowShiftCap: the same with the soft cap (cap > 60).
enum Mode {
  kStaticCap = 0, kOnlineCap = 1, kNoCap = 2, kRowMax = 3, kRowShift = 4, kRowShiftCap = 5
};
template <int MODE> constexpr bool fixed_shift() {
  return MODE == kStaticCap || MODE == kRowShift || MODE == kRowShiftCap;
}
template <int MODE> constexpr bool row_shift() {
  return MODE == kRowShift || MODE == kRowShiftCap;
}
constexpr int kKeys = static_cast<int>(kAttnKeyTile);  // keys per key tile
static_assert(kKeys == 128, "the tile layout below assumes 128-key tiles");
constexpr int kQTileBytes = 128 * kD * 2;     // this CTA's query tile (bf16)
constexpr int kQHalfBytes = kQTileBytes / 2;  // one 64-wide (128-byte) half
constexpr int kKTileBytes = 64 * kD * 2;      // this CTA's 64 keys of a K tile
constexpr int kKHalfBytes = kKTileBytes / 2;  // one 64-wide half of them
// K ring slots hold two consecutive key tiles, so the S issuer waits for
// data and releases it once per two tiles (each mbarrier operation costs the
// issuing thread about 180 cycles, measured).
constexpr int kStages = 2;
constexpr int kTilesPerSlot = 2;

// This CTA's half of a V tile, 128 keys x DV/2 value columns, MN-major for
// the PV product.  DV = 128: one 128-byte-swizzled 64-column box.  DV = 192
// (the value width of the page's checkpoint, section "Why stock
// FlashAttention was not a drop-in replacement", tensor V): 96 columns, which
// 64-column atoms cannot tile, so three 64-byte-swizzled 32-column boxes
// 8 KB apart.
template <int DV> struct VLayout;
template <> struct VLayout<128> {
  static constexpr int kBoxes = 1, kBoxCols = 64;
  static constexpr int kTileBytes = 128 * 64 * 2;       // 16 KB
  static constexpr uint32_t kDescHi = desc_sw128_hi(1024);
  static constexpr uint32_t kAtomBytes = 16384;         // LBO (one atom: unused)
  static constexpr uint32_t kKStepBytes = 16 * 128;     // 16 keys x 128 B
};
template <> struct VLayout<192> {
  static constexpr int kBoxes = 3, kBoxCols = 32;
  static constexpr int kTileBytes = 128 * 96 * 2;       // 24 KB
  static constexpr uint32_t kDescHi = desc_sw64_hi(512);
  static constexpr uint32_t kAtomBytes = 8192;          // LBO: 32-column atoms
  static constexpr uint32_t kKStepBytes = 16 * 64;      // 16 keys x 64 B
};
constexpr int kKSlotBytes = kTilesPerSlot * kKTileBytes;
// The V ring: value width 128 keeps three one-tile slots (48 KB instead of
// 64 KB, which leaves room for the epilogue's staging of out); value width
// 192 two two-tile slots.  V tiles are needed a few tiles after their K tile
// (PV trails S), so the shallower ring still covers the load latency.
template <int DV> constexpr int v_stages() { return DV == 128 ? 3 : 2; }
template <int DV> constexpr int v_tiles_per_slot() { return DV == 128 ? 1 : 2; }
constexpr int kVStagesMax = 3;
template <int DV> constexpr int v_slot_bytes() {
  return v_tiles_per_slot<DV>() * VLayout<DV>::kTileBytes;
}

// Tensor-memory columns of the running-max modes and of value width 192: S
// buffer u at 128 u; P buffer p (bf16 pairs, 64 columns for 128 keys) at
// 256 + 64 p; O (DV columns) after the P buffers.  DV = 128: 2 S + 2 P + O =
// 512 columns; DV = 192: 2 S + 1 P + O = 512.
template <int DV> struct Tmem {
  static constexpr int kNP = DV == 128 ? 2 : 1;
  static constexpr uint32_t kColP = 256;
  static constexpr uint32_t kColO = 256 + 64 * kNP;
};
// Static cap at value width 128 ("P in place"): three 128-column step
// buffers b = t % 3 at [128 b, 128 b + 128), the softmax writing each 64-key
// half's P (bf16 pairs, 32 columns) over the first columns of that half's
// logits, and O at [384, 512).  S of tile t waits for PV of tile t - 3 (the
// buffer's last reader) instead of for the softmax, so the logits of a warp
// group's next tile are usually ready before the group asks for them.
constexpr uint32_t kIPBufs = 3;
constexpr uint32_t kIPColO = 384;
// The fixed-shift modes at value width 128.
template <int MODE, int DV> constexpr bool p_in_place() {
  return fixed_shift<MODE>() && DV == 128;
}
static_assert(Tmem<128>::kColO + 128 <= 512 && Tmem<192>::kColO + 192 <= 512,
              "tensor memory budget");
constexpr uint32_t kTmemCols = 512;

constexpr int kWG = 4;                      // softmax warpgroups
constexpr int kSoftThreads = 128 * kWG;
constexpr int kSoftWarps = 4 * kWG;         // per CTA
constexpr int kPairSoftWarps = 2 * kSoftWarps;
constexpr int kWarpLoadQK = 4 * kWG;        // TMA: Q and K
constexpr int kWarpIssueS = 4 * kWG + 1;    // even CTA: S issuer; odd: Q/K relay
constexpr int kWarpIssuePV = 4 * kWG + 2;   // even CTA: PV issuer; odd: V relay
constexpr int kWarpLoadV = 4 * kWG + 3;     // TMA: V
constexpr int kNumWarps = 4 * kWG + 4;
constexpr int kThreads = kNumWarps * 32;
// Registers per thread: the launch gives every thread kRegsLaunch (the cap
// for this block size, which ptxas allocates when setmaxnreg is present; the
// launcher refuses a build with fewer); the loader/issuer warpgroup then
// drops to kRegsLow and the four softmax warpgroups rise to kRegsHigh out of
// what it released (ptxas then compiles the softmax without spills).  The
// split must fit the launch allocation, or the increase would wait forever:
// 128 x 56 + 512 x 104 = 60,416 <= 640 x 96 = 61,440.
constexpr uint32_t kRegsLaunch = 96;
constexpr uint32_t kRegsLow = 56;
constexpr uint32_t kRegsHigh = 104;
static_assert(kSoftThreads * kRegsHigh + 128 * kRegsLow <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
static_assert(kRegsLow % 8 == 0 && kRegsHigh % 8 == 0 && kRegsLow >= 24 && kRegsHigh <= 256,
              "setmaxnreg counts are multiples of 8 in [24, 256]");
constexpr uint32_t kIdescQK = idesc_bf16_f32(256, kKeys, 0);  // K-major B (K)
template <int DV> constexpr uint32_t idesc_pv() { return idesc_bf16_f32(256, DV, 1); }
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Lazy rescale threshold (log2 units) for the running-max modes.
constexpr float kRescaleThreshold = 8.0f;

// The capped modes take tanh from the special-function unit (tanh.approx.f32,
// measured on B200 over |y| <= 12: relative error below 1e-5, absolute below
// 8e-6, so the capped logit's error stays below 1e-5 min(cap, |y cap|)).

// Wait sites recorded in the device error word.
enum Site : unsigned {
  kSiteProdQ = 1, kSiteProdK = 2, kSiteIssueQ = 3, kSiteIssueK = 4,
  kSiteIssueP = 5, kSiteSoftS = 6, kSiteSoftO = 7, kSiteDrain = 8,
  kSiteXchg = 9, kSiteSoftPV = 10, kSiteRelay = 11, kSiteProdV = 12,
  kSiteIssueV = 13, kSiteIssueSFree = 14, kSiteIssueOFree = 15
};

// Per-CTA barriers.  In the even CTA, q_full, k_full and v_full also count
// the odd CTA's relay (two arrivals: the local producer's, with the byte
// count, and the relay's), so an issuing thread waits once for both halves
// of a load; s_free and p_full are used in the even CTA only (the odd CTA's
// softmax warps arrive on them remotely).  q_empty, k_empty, v_empty, s_full,
// pv_done and o_full are signalled in both CTAs by the even CTA's commits.
// o_free (even CTA, P in place) counts every softmax warp of the pair once
// per segment, after its last read of O.
struct __align__(8) Barriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kVStagesMax], v_empty[kVStagesMax];  // [v_stages<DV>()] in use
  uint64_t s_full[3], s_free[2];  // s_full: three in use with P in place, else two
  uint64_t p_full[3], pv_done[3];  // three in use with P in place, else [Tmem<DV>::kNP]
  uint64_t o_full, o_free;
  uint64_t xm, xd;  // row-max / row-sum exchange between the warpgroups
  uint64_t drain;   // both issuing threads' MMAs have completed
  uint32_t tmem_base;
  int abort;
};

// Softmax-side shared memory: row-max (per key tile, double-buffered by tile
// parity) and row-sum (per segment) exchange between the four warpgroups.
struct Xchg {
  float mpart[2][kWG][128];  // [tile parity][warpgroup][row]
  float dpart[2][kWG][128];  // [segment parity][warpgroup][row]
};

// Epilogue staging (value width 128): 4 KB per softmax warp, 1024-byte
// aligned.  A segment that writes out directly stages the warp's 32 rows x
// 32 columns of it there in the TMA 128-byte swizzle (row l at 128 l,
// 16-byte chunk c at (c ^ (l & 7)) 16: every 8 lanes of a 16-byte store hit
// all 32 banks) and one lane stores the box with a bulk tensor copy, which
// runs on while the warp goes on to the next segment.  The other segments
// (merge with a first piece, scratch) stage 16 columns at a time in rows
// padded to 20 floats and store them with plain 16-byte stores, 64
// contiguous bytes per row per 4 lanes.  Value width 192 has no room for
// staging and stores directly.
constexpr int kStageRow = 20;
constexpr int kStageWarpFloats = 1024;  // 4 KB
template <int DV> constexpr size_t stage_bytes() {
  return DV == 128 ? static_cast<size_t>(kSoftThreads / 32) * kStageWarpFloats * 4 : 0;
}
static_assert(32 * kStageRow <= kStageWarpFloats, "padded staging fits a warp's slot");
constexpr size_t kBarsXchgBytes = (sizeof(Barriers) + sizeof(Xchg) + 15) & ~static_cast<size_t>(15);
template <int DV> constexpr size_t smem_bytes() {
  return 1024 + static_cast<size_t>(kQTileBytes) + kStages * static_cast<size_t>(kKSlotBytes) +
         v_stages<DV>() * static_cast<size_t>(v_slot_bytes<DV>()) + stage_bytes<DV>() +
         kBarsXchgBytes;
}
static_assert(smem_bytes<128>() <= 227 * 1024 && smem_bytes<192>() <= 227 * 1024,
              "shared memory budget");

// --------------------------------------------------------------------------
// Work schedules.  A segment is one pair of query tiles (an "item": batch
// item b = item / pairs, query blocks 2 (item % pairs) and the next) and a
// run [kb, ke) of its key tiles; every role of a cluster walks the same
// segment sequence.
enum Sched { kSchedRange = 0, kSchedUnits = 1, kSchedTail = 2 };
// Where a segment's normalised result goes: out/lse (a whole pair, or the
// first piece of a split one); this cluster's scratch slot (a later piece of
// a split pair under kSchedRange, merged by attn_merge_kernel); or merged
// into out/lse with the first piece's result (kSchedTail).
enum Dest { kDestOut = 0, kDestScratch = 1, kDestMerge = 2 };

struct Params {
  const float *bias;
  long long bias_bstride;  // floats between batch items' bias (0: shared)
  float *out;
  float *lse;
  unsigned *err;
  float *ws_out;       // kSchedRange scratch: [clusters][2][128][DV] partial outputs
  float *ws_lse;       //                      [clusters][2][128] partial log-sum-exps
  int L;           // keys per batch item
  int Lq;          // query positions per batch item (rows of q, out, lse)
  int P;           // bias cells per bias row, ceil(L / 16)
  int bias_rows;   // bias rows per head in the bias array, ceil(Lq / 16)
  int nb;          // 16-position query blocks per batch item, ceil(Lq / 16)
  int pairs;       // query-tile pairs per batch item: ceil(nb / 2)
  int n_items;     // B * pairs
  int n_kt;        // key tiles: ceil(L / 128)
  int last_valid;  // valid keys in the last key tile (1..128)
  int sched;       // Sched
  int whole;       // kSchedRange: cluster ranges hold whole pairs
  int n_whole;     // kSchedUnits/Tail: items [0, n_whole) run whole; item
                   // n_whole + s is split pair s
  int split_at;    // split pairs: first piece key tiles [0, split_at), second
                   // piece [split_at, n_kt)
  float qk_scale;  // multiplies q.k
  float bias_mul;  // multiplies the compact bias
  float A;         // capped modes: cap * log2(e)
  float shift;     // static modes: the fixed shift (log2 units, an integer; see attn_mode)
  // kSchedUnits: cluster c runs whole items [wb[c], wb[c+1]) and then the
  // first pieces of split pairs [fb[c], fb[c+1]).
  int wb[kAttnMaxClusters + 1];
  int fb[kAttnMaxClusters + 1];
};

struct Segment {
  int item, kb, ke, dest;
};

struct Cursor {
  int a, a_end, f, f_end;
};

__device__ __forceinline__ int num_clusters() { return static_cast<int>(gridDim.x >> 1); }
__device__ __forceinline__ int cluster_index() { return static_cast<int>(blockIdx.x >> 1); }

// kSchedRange: the W = n_items * n_kt (pair, key tile) steps are cut into
// one contiguous range per cluster, [W c / G, W (c+1) / G) for cluster c of G
// (W <= 2^30, checked by the launcher; only the bounds need 64 bits).  With
// p.whole the bounds are rounded to whole pairs.
__device__ __forceinline__ int range_start(const Params &p, int c) {
  const long long G = num_clusters();
  if (p.whole)
    return static_cast<int>(static_cast<long long>(p.n_items) * c / G) * p.n_kt;
  return static_cast<int>(static_cast<long long>(p.n_items) * p.n_kt * c / G);
}

__device__ __forceinline__ Cursor cursor_begin(const Params &p) {
  const int c = cluster_index();
  Cursor cu;
  if (p.sched == kSchedRange) {
    cu.a = range_start(p, c);
    cu.a_end = range_start(p, c + 1);
    cu.f = cu.f_end = 0;
  } else if (p.sched == kSchedUnits) {
    cu.a = p.wb[c];
    cu.a_end = p.wb[c + 1];
    cu.f = p.fb[c];
    cu.f_end = p.fb[c + 1];
  } else {  // kSchedTail: the second piece of split pair c
    cu.a = c;
    cu.a_end = c + 1;
    cu.f = cu.f_end = 0;
  }
  return cu;
}

__device__ __forceinline__ bool next_segment(const Params &p, Cursor &cu, Segment &sg) {
  if (p.sched == kSchedRange) {
    if (cu.a >= cu.a_end) return false;
    sg.item = cu.a / p.n_kt;
    sg.kb = cu.a - sg.item * p.n_kt;
    const int left = cu.a_end - cu.a;
    sg.ke = left < p.n_kt - sg.kb ? sg.kb + left : p.n_kt;
    sg.dest = sg.kb == 0 ? kDestOut : kDestScratch;
    cu.a += sg.ke - sg.kb;
    return true;
  }
  if (p.sched == kSchedUnits) {
    if (cu.a < cu.a_end) {
      sg = {cu.a, 0, p.n_kt, kDestOut};
      ++cu.a;
      return true;
    }
    if (cu.f < cu.f_end) {
      sg = {p.n_whole + cu.f, 0, p.split_at, kDestOut};
      ++cu.f;
      return true;
    }
    return false;
  }
  if (cu.a >= cu.a_end) return false;
  sg = {p.n_whole + cu.a, p.split_at, p.n_kt, kDestMerge};
  ++cu.a;
  return true;
}

// --------------------------------------------------------------------------
// MMA issue helpers (issuing threads of the even CTA).

// Shared-memory descriptors: every operand here has 8-row groups 1 KB apart,
// so all share one high word; the low word (start address and leading
// offset) is built once per tile base and each K step adds a constant to its
// start-address field (addresses stay below 2^18: no carry out of the field).
constexpr uint32_t kDescHi = desc_sw128_hi(1024);

// S[256 x 128] = Q[256 x 128] K^T over the pair: eight K=16 steps over the two
// 64-wide halves of each CTA's Q tile (16 KB apart) and K tile (8 KB apart).
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr,
                                         uint32_t k_addr) {
  const uint32_t q_lo = desc_sw128_lo(q_addr, 16), k_lo = desc_sw128_lo(k_addr, 16);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t qo = ((kk >> 2) * kQHalfBytes + (kk & 3) * 32) >> 4;
    const uint32_t ko = ((kk >> 2) * kKHalfBytes + (kk & 3) * 32) >> 4;
    umma2_ss_w(d_tmem, q_lo + qo, k_lo + ko, kDescHi, kIdescQK, kk > 0 ? 1u : 0u);
  }
}

// O[256 x DV] (+)= P[256 x 128 keys] V[128 keys x DV]: P from each CTA's
// tensor memory (bf16 pairs, 8 columns per 16 keys, keys in column order),
// V MN-major: each CTA holds DV/2 value columns for all 128 keys (VLayout).
template <int DV>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem,
                                         uint32_t v_addr, bool accumulate) {
  using VL = VLayout<DV>;
  const uint32_t v_lo = desc_sw128_lo(v_addr, VL::kAtomBytes);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    umma2_ts_w(d_tmem, p_tmem + 8 * kk, v_lo + ((kk * VL::kKStepBytes) >> 4), VL::kDescHi,
               idesc_pv<DV>(), (accumulate || kk > 0) ? 1u : 0u);
  }
}

// The same for P in place (value width 128): keys 16 kk .. 16 kk + 15 are
// in the half kk / 4 of the step buffer, at its column 64 (kk / 4) + 8 (kk % 4).
__device__ __forceinline__ void issue_pv_in_place(uint32_t d_tmem, uint32_t buf_tmem,
                                                  uint32_t v_addr, bool accumulate) {
  using VL = VLayout<128>;
  const uint32_t v_lo = desc_sw128_lo(v_addr, VL::kAtomBytes);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    umma2_ts_w(d_tmem, buf_tmem + 64 * (kk >> 2) + 8 * (kk & 3),
               v_lo + ((kk * VL::kKStepBytes) >> 4), VL::kDescHi, idesc_pv<128>(),
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
// Producer warps, lane 0 (each CTA): TMA loads of this CTA's Q tile and of
// its halves of the K tiles (producer_qk), and of its halves of the V tiles
// (producer_v).  Key tiles [j0, j0 + 2) of a segment share a ring slot.
__device__ __forceinline__ void producer_qk(const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                            uint8_t *q_s, uint8_t *k_s, Barriers *bars,
                                            const Params &p, uint32_t rank,
                                            volatile int *abort) {
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_k = l2_policy_evict_last();
  uint32_t qc = 0, kl = 0;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    const int b = sg.item / p.pairs;
    const int I0 = (sg.item % p.pairs) * 2;
    ok = mbar_wait(&bars->q_empty, (qc & 1u) ^ 1u, abort, p.err, kSiteProdQ);
    if (!ok) break;
    mbar_arrive_expect_tx(&bars->q_full, kQTileBytes);
    const int qrow = tile_block(p, I0, rank) * 16;
    tma_load_4d(q_s, tm_q, &bars->q_full, 0, qrow, 0, b, pol_q);
    tma_load_4d(q_s + kQHalfBytes, tm_q, &bars->q_full, 64, qrow, 0, b, pol_q);
    ++qc;
    for (int j0 = sg.kb; j0 < sg.ke; j0 += kTilesPerSlot) {
      const uint32_t slot = kl % kStages, ph = (kl / kStages) & 1u;
      ok = mbar_wait(&bars->k_empty[slot], ph ^ 1u, abort, p.err, kSiteProdK);
      if (!ok) break;
      const int nt = sg.ke - j0 < kTilesPerSlot ? sg.ke - j0 : kTilesPerSlot;
      mbar_arrive_expect_tx(&bars->k_full[slot], static_cast<uint32_t>(nt) * kKTileBytes);
      for (int t = 0; t < nt; ++t) {
        // Keys [128 j + 64 rank, +64), all 128 columns, as two 64-wide halves.
        uint8_t *dst = k_s + slot * kKSlotBytes + t * kKTileBytes;
        const int key0 = (j0 + t) * kKeys + 64 * static_cast<int>(rank);
        tma_load_3d(dst, tm_k, &bars->k_full[slot], 0, key0, b, pol_k);
        tma_load_3d(dst + kKHalfBytes, tm_k, &bars->k_full[slot], 64, key0, b, pol_k);
      }
      ++kl;
    }
  }
  // Every copy this thread started must land before the CTA exits.
  if (qc > 0) drain_wait(&bars->q_full, (qc - 1) & 1u);
  for (uint32_t i = kl > kStages ? kl - kStages : 0; i < kl; ++i)
    drain_wait(&bars->k_full[i % kStages], (i / kStages) & 1u);
}

template <int DV>
__device__ __forceinline__ void producer_v(const CUtensorMap *tm_v, uint8_t *v_s,
                                           Barriers *bars, const Params &p, uint32_t rank,
                                           volatile int *abort) {
  using VL = VLayout<DV>;
  constexpr int kVS = v_stages<DV>(), kVT = v_tiles_per_slot<DV>();
  const uint64_t pol_v = l2_policy_evict_last();
  uint32_t vl = 0;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    const int b = sg.item / p.pairs;
    for (int j0 = sg.kb; j0 < sg.ke; j0 += kVT) {
      const uint32_t slot = vl % kVS, ph = (vl / kVS) & 1u;
      ok = mbar_wait(&bars->v_empty[slot], ph ^ 1u, abort, p.err, kSiteProdV);
      if (!ok) break;
      const int nt = sg.ke - j0 < kVT ? sg.ke - j0 : kVT;
      mbar_arrive_expect_tx(&bars->v_full[slot], static_cast<uint32_t>(nt) * VL::kTileBytes);
      for (int t = 0; t < nt; ++t) {
        // Keys [128 j, +128), value columns [DV/2 rank, +DV/2).
        uint8_t *dst = v_s + slot * v_slot_bytes<DV>() + t * VL::kTileBytes;
#pragma unroll
        for (int a = 0; a < VL::kBoxes; ++a)
          tma_load_3d(dst + a * VL::kAtomBytes, tm_v, &bars->v_full[slot],
                      (DV / 2) * static_cast<int>(rank) + a * VL::kBoxCols,
                      (j0 + t) * kKeys, b, pol_v);
      }
      ++vl;
    }
  }
  for (uint32_t i = vl > kVS ? vl - kVS : 0; i < vl; ++i)
    drain_wait(&bars->v_full[i % kVS], (i / kVS) & 1u);
}

// --------------------------------------------------------------------------
// Relays of the odd CTA, lane 0: tell the even CTA's issuing threads, in
// ring order, that this CTA's half of each Q / K load (relay_qk) or V load
// (relay_v) has landed.
__device__ __forceinline__ void relay_qk(Barriers *bars, const Params &p, volatile int *abort) {
  const uint32_t q_leader = cluster_addr(&bars->q_full, 0);
  uint32_t qc = 0, kl = 0;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    ok = mbar_wait(&bars->q_full, qc & 1u, abort, p.err, kSiteRelay);
    ++qc;
    if (!ok) break;
    mbar_arrive_cluster(q_leader);
    for (int j0 = sg.kb; j0 < sg.ke; j0 += kTilesPerSlot) {
      const uint32_t slot = kl % kStages;
      ok = mbar_wait(&bars->k_full[slot], (kl / kStages) & 1u, abort, p.err, kSiteRelay);
      if (!ok) break;
      ++kl;
      mbar_arrive_cluster(cluster_addr(&bars->k_full[slot], 0));
    }
  }
}

template <int DV>
__device__ __forceinline__ void relay_v(Barriers *bars, const Params &p, volatile int *abort) {
  constexpr int kVS = v_stages<DV>(), kVT = v_tiles_per_slot<DV>();
  uint32_t vl = 0;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    for (int j0 = sg.kb; j0 < sg.ke; j0 += kVT) {
      const uint32_t slot = vl % kVS;
      ok = mbar_wait(&bars->v_full[slot], (vl / kVS) & 1u, abort, p.err, kSiteRelay);
      if (!ok) break;
      ++vl;
      mbar_arrive_cluster(cluster_addr(&bars->v_full[slot], 0));
    }
  }
}

// --------------------------------------------------------------------------
// Issuing warps of the even CTA (every lane waits; one elected lane issues).
// The odd CTA's arrivals on their barriers
// (relays, softmax) are relaxed (see mbar_arrive_cluster), so their waits
// acquire at CTA scope: a cluster-scope acquire would order nothing more and
// costs about 180 cycles per wait (measured).

// S = Q K^T for every key tile, into step buffer (use count) % 2, once the
// softmax has read that buffer's previous logits (s_free); with P in place
// into buffer (use count) % 3, once PV has read the P written over that
// buffer's previous logits (pv_done).
template <bool kIP>
__device__ __forceinline__ void issuer_s(uint8_t *q_s, uint8_t *k_s, Barriers *bars,
                                         uint32_t tmem, const Params &p,
                                         volatile int *abort) {
  constexpr uint32_t kBufs = kIP ? kIPBufs : 2;
  const uint32_t q_addr = smem_u32(q_s), k_addr = smem_u32(k_s);
  uint32_t qc = 0, kl = 0, su = 0;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    ok = mbar_wait_warp(&bars->q_full, qc & 1u, abort, p.err, kSiteIssueQ);
    ++qc;
    if (!ok) break;
    uint32_t slot = 0;
    for (int j = sg.kb; j < sg.ke; ++j) {
      const int i = j - sg.kb;
      if ((i & 1) == 0) {
        slot = kl % kStages;
        ok = mbar_wait_warp(&bars->k_full[slot], (kl / kStages) & 1u, abort, p.err, kSiteIssueK);
        ++kl;
        if (!ok) break;
      }
      const uint32_t sb = su % kBufs, sn = su / kBufs;
      if (sn > 0) {
        // The buffer's previous logits are no longer needed: read by the
        // softmax (s_free), or, with P in place, read by PV as P (pv_done).
        ok = mbar_wait_warp(kIP ? &bars->pv_done[sb] : &bars->s_free[sb], (sn - 1) & 1u, abort,
                            p.err, kSiteIssueSFree);
        if (!ok) break;
      }
      tc_fence_after();
      issue_qk(tmem + 128u * sb, q_addr, k_addr + slot * kKSlotBytes + (i & 1) * kKTileBytes);
      umma2_commit_both_w(&bars->s_full[sb]);
      if (j + 1 == sg.ke) umma2_commit_both_w(&bars->q_empty);
      if ((i & 1) == 1 || j + 1 == sg.ke) umma2_commit_both_w(&bars->k_empty[slot]);
      ++su;
    }
  }
  // All MMAs this thread issued complete before tensor memory is released.
  umma2_commit_self_w(&bars->drain);
  drain_wait(&bars->drain, 0);
}

// S for the first pass of the two-pass schedule (kRowMax): a step is one K
// ring slot (two key tiles, or one at the end of a segment), issued into the
// 256-column buffer pair step % 2 and committed once, so the issuing thread
// waits and commits once per two tiles; the softmax releases a pair
// (s_free[pair]) once it has read both tiles' logits.
__device__ __forceinline__ void issuer_rowmax(uint8_t *q_s, uint8_t *k_s, Barriers *bars,
                                              uint32_t tmem, const Params &p,
                                              volatile int *abort) {
  const uint32_t q_addr = smem_u32(q_s), k_addr = smem_u32(k_s);
  uint32_t qc = 0, kl = 0, st = 0;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    ok = mbar_wait_warp(&bars->q_full, qc & 1u, abort, p.err, kSiteIssueQ);
    ++qc;
    if (!ok) break;
    for (int j0 = sg.kb; j0 < sg.ke; j0 += kTilesPerSlot) {
      const int nt = sg.ke - j0 < kTilesPerSlot ? sg.ke - j0 : kTilesPerSlot;
      const uint32_t slot = kl % kStages;
      ok = mbar_wait_warp(&bars->k_full[slot], (kl / kStages) & 1u, abort, p.err, kSiteIssueK);
      ++kl;
      if (!ok) break;
      const uint32_t b = st & 1u, n = st >> 1;
      if (n > 0) {
        ok = mbar_wait_warp(&bars->s_free[b], (n - 1) & 1u, abort, p.err, kSiteIssueSFree);
        if (!ok) break;
      }
      tc_fence_after();
      for (int t = 0; t < nt; ++t)
        issue_qk(tmem + 256u * b + 128u * static_cast<uint32_t>(t), q_addr,
                 k_addr + slot * kKSlotBytes + t * kKTileBytes);
      umma2_commit_both_w(&bars->s_full[b]);
      if (j0 + nt == sg.ke) umma2_commit_both_w(&bars->q_empty);
      umma2_commit_both_w(&bars->k_empty[slot]);
      ++st;
    }
  }
  umma2_commit_self_w(&bars->drain);
  drain_wait(&bars->drain, 0);
}

// O += P V for every key tile, once the softmax has written P (p_full).
template <int DV, bool kIP>
__device__ __forceinline__ void issuer_pv(uint8_t *v_s, Barriers *bars, uint32_t tmem,
                                          const Params &p, volatile int *abort) {
  using T = Tmem<DV>;
  constexpr uint32_t kBufs = kIP ? kIPBufs : T::kNP;
  constexpr int kVS = v_stages<DV>(), kVT = v_tiles_per_slot<DV>();
  const uint32_t v_addr = smem_u32(v_s);
  uint32_t vl = 0, pu = 0, seg = 0;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    uint32_t slot = 0;
    for (int j = sg.kb; j < sg.ke; ++j) {
      const int i = j - sg.kb;
      if (i % kVT == 0) {
        slot = vl % kVS;
        ok = mbar_wait_warp(&bars->v_full[slot], (vl / kVS) & 1u, abort, p.err, kSiteIssueV);
        ++vl;
        if (!ok) break;
      }
      const uint32_t pb = pu % kBufs, pn = pu / kBufs;
      ok = mbar_wait_warp(&bars->p_full[pb], pn & 1u, abort, p.err, kSiteIssueP);
      if (!ok) break;
      if (kIP && i == 0 && seg > 0) {
        // The first PV of a segment overwrites O.  With P in place the two
        // softmax groups take alternate tiles, so the P of this tile does not
        // imply that the other group has read the previous segment's O: wait
        // until every softmax warp of the pair has.
        ok = mbar_wait_warp(&bars->o_free, (seg - 1) & 1u, abort, p.err, kSiteIssueOFree);
        if (!ok) break;
      }
      tc_fence_after();
      const uint32_t va =
          v_addr + slot * v_slot_bytes<DV>() + (i % kVT) * VLayout<DV>::kTileBytes;
      if constexpr (kIP)
        issue_pv_in_place(tmem + kIPColO, tmem + 128u * pb, va, i > 0);
      else
        issue_pv<DV>(tmem + T::kColO, tmem + T::kColP + 64u * pb, va, i > 0);
      umma2_commit_both_w(&bars->pv_done[pb]);
      if (j + 1 == sg.ke) umma2_commit_both_w(&bars->o_full);
      if (i % kVT == kVT - 1 || j + 1 == sg.ke) umma2_commit_both_w(&bars->v_empty[slot]);
      ++pu;
    }
    ++seg;
  }
  umma2_commit_self_w(&bars->drain);
  drain_wait(&bars->drain, 0);
}

// --------------------------------------------------------------------------
// Softmax warpgroups (each CTA, its own query tile).
//
// Thread r of warpgroup g owns tensor-memory lane r, i.e. row r of the tile,
// and keys [32 g, 32 g + 32) of every key tile.  A row's sum is split between
// four threads and combined through shared memory once per segment (and, in
// the running-max modes, its maximum once per key tile).

// Softmax-side barriers count warps: each warp arrives once, from lane 0,
// after __syncwarp has ordered its lanes' prior work.
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
  __syncwarp();
  if (lane_id() == 0) mbar_arrive(bar);
}
// The same on a barrier of the even CTA (local, or remote from the odd CTA).
__device__ __forceinline__ void warp_arrive_leader(uint64_t *bar, uint32_t remote,
                                                   uint32_t rank) {
  __syncwarp();
  if (lane_id() == 0) {
    if (rank == 0)
      mbar_arrive(bar);
    else
      mbar_arrive_cluster(remote);
  }
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

// The compact bias cells of warpgroup g's 32 keys of key tile j:
// bias[h, I, 8j + 2g + e] (0 past the end: those keys are masked).
__device__ __forceinline__ void load_bias(const float *brow, int j, int g, int P,
                                          float (&bn)[2]) {
  const int J0 = j * 8 + g * 2;
#pragma unroll
  for (int e = 0; e < 2; ++e) bn[e] = (J0 + e < P) ? __ldg(brow + J0 + e) : 0.f;
}

// The compact bias cells of warpgroup half hk's 64 keys of key tile j:
// bias[h, I, 8j + 4hk + e] (0 past the end: those keys are masked).
__device__ __forceinline__ void load_bias4(const float *brow, int j, int hk, int P,
                                           float (&bn)[4]) {
  const int J0 = j * 8 + hk * 4;
#pragma unroll
  for (int e = 0; e < 4; ++e) bn[e] = (J0 + e < P) ? __ldg(brow + J0 + e) : 0.f;
}

// Column pairs (out of every 8) whose exponential runs on the FMA pipe
// (exp2_poly2_fma) instead of the special-function unit, in kStaticCap.  The
// SFU still computes every tanh, so it does 1 + (8 - kEmuPairs) / 8
// operations per logit.
#ifndef AG_EXP2_EMU_PAIRS
#define AG_EXP2_EMU_PAIRS 5
#endif
constexpr int kEmuPairs = AG_EXP2_EMU_PAIRS;

// Constants of the static mode, per thread.
struct StaticK {
  float2 sc;     // multiplies s
  float2 a;      // A = cap log2(e) (1 without a cap)
  float2 nsh;    // -shift (for the SFU pairs)
  float2 km;     // 1.5 * 2^23 - shift (exp2_poly2_fma)
  float tmin;    // row shifts: the smallest t for exp2_poly2_fma, (shift - 126) / A
};

// One thread's N keys of a key tile, fixed shift, log2 units:
// t = tanh(y) (or t = y without a cap, MODE kRowShift), p = 2^(A t - shift),
// y = s qk_scale + b / cap.  Adds the row sum into acc and packs N/2 bf16
// pairs of P.  kMask zeroes keys >= nvalid (only the last key tile of a
// ragged length needs it).  With a row's own shift the exponent A t - shift
// has no lower bound, so the FMA-pipe exponential takes t no smaller than
// k.tmin (probabilities below 2^-126, which cannot move a row sum whose
// largest term is at least 1/2, become 2^-126); the special-function unit's
// ex2 flushes them to zero by itself.
template <bool kMask, int N, int MODE = kStaticCap>
__device__ __forceinline__ void chunk_static(const uint32_t (&s)[N], float b0, float b1,
                                             const StaticK &k, int col0, int nvalid,
                                             float2 &acc, uint32_t (&pk)[N / 2]) {
#pragma unroll
  for (int e = 0; e < N / 2; ++e) {
    const float bb = e < 8 ? b0 : b1;
    const float2 y = __ffma2_rn(
        make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), k.sc,
        make_float2(bb, bb));
    const float2 t = MODE == kRowShift ? y : make_float2(tanh_approx(y.x), tanh_approx(y.y));
    float2 pr;
    if ((e & 7) < kEmuPairs) {
      if constexpr (row_shift<MODE>())
        pr = exp2_poly2_fma(make_float2(fmaxf(t.x, k.tmin), fmaxf(t.y, k.tmin)), k.a, k.km);
      else
        pr = exp2_poly2_fma(t, k.a, k.km);
    } else {
      const float2 x = __ffma2_rn(t, k.a, k.nsh);
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

// A running-max mode's capped (or uncapped) logit of one key, log2 units.
template <int MODE>
__device__ __forceinline__ float online_logit(float s, float bb, const Params &p) {
  const float y = fmaf(s, p.qk_scale, bb);
  return (MODE == kOnlineCap) ? p.A * tanh_approx(y) : y;
}

// Per-thread pipeline counters of the softmax role.
struct SoftCounters {
  uint32_t su = 0;  // S buffer uses (key tiles) so far
  uint32_t pu = 0;  // P buffer uses so far
  uint32_t ocount = 0, xmcount = 0, xdcount = 0;
};

// Waits for the S of the next key tile, loads this thread's 32 logits and
// releases the S buffer to the S issuer.
__device__ __forceinline__ bool load_s(Barriers *bars, uint32_t tmem, int g, uint32_t lane_base,
                                       uint32_t rank, const uint32_t (&sf_remote)[2],
                                       SoftCounters &c, const Params &p, volatile int *abort,
                                       uint32_t (&s)[32]) {
  const uint32_t sb = c.su & 1u, sph = (c.su >> 1) & 1u;
  ++c.su;
  const bool ok = mbar_wait(&bars->s_full[sb], sph, abort, p.err, kSiteSoftS);
  if (!__all_sync(0xffffffffu, ok)) return false;
  tc_fence_after();
  tmem_ld32(tmem + 128u * sb + 32u * g + lane_base, s);
  tmem_wait_ld(s);
  tc_fence_before();
  warp_arrive_leader(&bars->s_free[sb], sb ? sf_remote[1] : sf_remote[0], rank);
  return true;
}

// Writes this thread's 16 columns of P into the next P buffer (once the PV
// that last read it has finished) and tells the PV issuer.
template <int DV>
__device__ __forceinline__ bool store_p(Barriers *bars, uint32_t tmem, int g,
                                        uint32_t lane_base, uint32_t rank,
                                        const uint32_t (&pf_remote)[2], SoftCounters &c,
                                        const Params &p, volatile int *abort,
                                        const uint32_t (&pk)[16]) {
  using T = Tmem<DV>;
  const uint32_t pb = c.pu % T::kNP, pn = c.pu / T::kNP;
  ++c.pu;
  if (pn > 0) {
    const bool ok = mbar_wait(&bars->pv_done[pb], (pn - 1) & 1u, abort, p.err, kSiteSoftPV);
    if (!__all_sync(0xffffffffu, ok)) return false;
  }
  tc_fence_after();
  tmem_st16(tmem + T::kColP + 64u * pb + 16u * g + lane_base, pk);
  tmem_wait_st();
  tc_fence_before();
  warp_arrive_leader(&bars->p_full[pb], pb ? pf_remote[1] : pf_remote[0], rank);
  return true;
}

// One 64-key half tile of a grouped static segment (see below): tS and tP
// address this warp's S and P columns, bc holds the four bias cells.
template <bool kMask, int MODE>
__device__ __forceinline__ void tile_grouped(uint32_t tS, const float (&bc)[4], float m,
                                             const StaticK &k, int col0, int nvalid,
                                             float2 &acc) {
  // P piece c (8 columns) goes over columns 8 c .. 8 c + 7 of this half's
  // logits, which pieces 0 .. c have already brought into registers; piece
  // c + 1 (columns 16 c + 16 ..) is being loaded meanwhile.
  uint32_t sa[16], sb[16], pk[8];
  tmem_ld16(tS, sa);
  tmem_wait_ld16(sa);
  tmem_ld16(tS + 16u, sb);
  chunk_static<kMask, 16, MODE>(sa, bc[0] * m, bc[0] * m, k, col0, nvalid, acc, pk);
  tmem_st8(tS, pk);
  tmem_wait_ld16(sb);
  tmem_ld16(tS + 32u, sa);
  chunk_static<kMask, 16, MODE>(sb, bc[1] * m, bc[1] * m, k, col0 + 16, nvalid, acc, pk);
  tmem_st8(tS + 8u, pk);
  tmem_wait_ld16(sa);
  tmem_ld16(tS + 48u, sb);
  chunk_static<kMask, 16, MODE>(sa, bc[2] * m, bc[2] * m, k, col0 + 32, nvalid, acc, pk);
  tmem_st8(tS + 16u, pk);
  tmem_wait_ld16(sb);
  chunk_static<kMask, 16, MODE>(sb, bc[3] * m, bc[3] * m, k, col0 + 48, nvalid, acc, pk);
  tmem_st8(tS + 24u, pk);
}

// Static-shift segment with alternating groups (value width 128, P in
// place): the warps split into two groups that take alternate key tiles,
// group q = warpgroups 2q and 2q + 1, warpgroup hk of it the 64 keys
// [64 hk, 64 hk + 64) of the tile; tile t's logits are in step buffer t % 3
// and its P goes over them.  One group's waits (for its logits, for its
// tensor-memory loads and stores) are covered by the other group's
// arithmetic, so the special-function unit stays busy.  A group waits for
// the s_full phases of its own tiles in order; the phase of the buffer's
// previous tile (the other group's) has completed by then, because the
// logits of the group's own previous tile, issued later, have.
//
// shift: this thread's row's shift (p.shift, or the row's own one in the
// row-shift modes; an integer).
template <int MODE, int DV>
__device__ __forceinline__ bool segment_static_grouped(const Segment &sg, const float *brow,
                                                       uint32_t tmem, uint32_t lane_base, int g,
                                                       const Params &p, Barriers *bars,
                                                       uint32_t rank, SoftCounters &c,
                                                       volatile int *abort, float shift,
                                                       float &d) {
  static_assert(DV == 128, "P in place: value width 128");
  const int q = g >> 1, hk = g & 1;  // group, key half
  StaticK k;
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  const float A = MODE == kRowShift ? 1.f : p.A;
  const float sh = row_shift<MODE>() ? shift : p.shift;
  k.sc = make_float2(p.qk_scale, p.qk_scale);
  k.a = make_float2(A, A);
  k.nsh = make_float2(-sh, -sh);
  k.km = make_float2(kShift - sh, kShift - sh);
  k.tmin = row_shift<MODE>() ? (sh - 126.f) / A : 0.f;
  float2 acc = make_float2(0.f, 0.f);
  const uint32_t pf0 = cluster_addr(&bars->p_full[0], 0);  // the even CTA's p_full
  // Key tile j of the segment is global tile c.su + (j - kb); the group takes
  // the tiles of its parity.
  const int j0 = sg.kb + static_cast<int>((static_cast<uint32_t>(q) - c.su) & 1u);
  float bc[4] = {0.f, 0.f, 0.f, 0.f};
  if (j0 < sg.ke) load_bias4(brow, j0, hk, p.P, bc);
  for (int j = j0; j < sg.ke; j += 2) {
    const uint32_t tile = c.su + static_cast<uint32_t>(j - sg.kb);
    const uint32_t b = tile % kIPBufs, u = tile / kIPBufs;
    const int nvalid = (j + 1 == p.n_kt) ? p.last_valid : kKeys;
    bool ok = mbar_wait(&bars->s_full[b], u & 1u, abort, p.err, kSiteSoftS);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + 128u * b + 64u * hk + lane_base;
    const float m = p.bias_mul;
    // Four pieces of 16 keys (one bias cell each), the tensor-memory load of
    // the next piece in flight while this one is computed.
    if (nvalid == kKeys)
      tile_grouped<false, MODE>(tS, bc, m, k, 64 * hk, nvalid, acc);
    else
      tile_grouped<true, MODE>(tS, bc, m, k, 64 * hk, nvalid, acc);
    if (j + 2 < sg.ke) load_bias4(brow, j + 2, hk, p.P, bc);
    tmem_wait_st();
    tc_fence_before();
    warp_arrive_leader(&bars->p_full[b], pf0 + 8u * b, rank);
  }
  const uint32_t tiles = static_cast<uint32_t>(sg.ke - sg.kb);
  c.su += tiles;
  c.pu += tiles;
  d = acc.x + acc.y;
  return true;
}

// One warpgroup's 32 keys of a key tile in an ungrouped static segment:
// tS and tP address this warp's S and P columns, bc holds the two bias cells.
template <bool kMask>
__device__ __forceinline__ bool tile_split(uint32_t tS, uint32_t tP, const float (&bc)[2],
                                           float m, const StaticK &k, int col0, int nvalid,
                                           uint32_t pn, uint32_t pb, uint32_t sb, uint32_t sfr,
                                           Barriers *bars, uint32_t rank, const Params &p,
                                           volatile int *abort, float2 &acc) {
  uint32_t sa[16], sc[16], pk[8];
  tmem_ld16(tS, sa);
  tmem_wait_ld16(sa);
  tmem_ld16(tS + 16u, sc);
  chunk_static<kMask, 16>(sa, bc[0] * m, bc[0] * m, k, col0, nvalid, acc, pk);
  if (pn > 0) {  // the PV that last read this P buffer
    const bool ok = mbar_wait(&bars->pv_done[pb], (pn - 1) & 1u, abort, p.err, kSiteSoftPV);
    if (!__all_sync(0xffffffffu, ok)) {
      tmem_wait_ld16(sc);
      return false;
    }
  }
  tc_fence_after();
  tmem_st8(tP, pk);
  tmem_wait_ld16(sc);
  tc_fence_before();
  warp_arrive_leader(&bars->s_free[sb], sfr, rank);  // S fully read
  chunk_static<kMask, 16>(sc, bc[1] * m, bc[1] * m, k, col0 + 16, nvalid, acc, pk);
  tmem_st8(tP + 8u, pk);
  return true;
}

// Static-shift segment: every warpgroup takes 32 keys of every key tile
// (value width 192, whose single P buffer both groups would share).
template <int MODE, int DV>
__device__ __forceinline__ bool segment_static(const Segment &sg, const float *brow,
                                               uint32_t tmem, uint32_t lane_base, int g,
                                               const Params &p, Barriers *bars,
                                               uint32_t rank, const uint32_t (&sf_remote)[2],
                                               const uint32_t (&pf_remote)[2],
                                               SoftCounters &c, volatile int *abort,
                                               float &d) {
  using T = Tmem<DV>;
  StaticK k;
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  k.sc = make_float2(p.qk_scale, p.qk_scale);
  k.a = make_float2(p.A, p.A);
  k.nsh = make_float2(-p.shift, -p.shift);
  k.km = make_float2(kShift - p.shift, kShift - p.shift);
  float2 acc = make_float2(0.f, 0.f);
  float bc[2], bn[2] = {0.f, 0.f};
  load_bias(brow, sg.kb, g, p.P, bc);
  for (int j = sg.kb; j < sg.ke; ++j) {
    if (j + 1 < sg.ke) load_bias(brow, j + 1, g, p.P, bn);
    const int nvalid = (j + 1 == p.n_kt) ? p.last_valid : kKeys;
    const uint32_t sb = c.su & 1u, sph = (c.su >> 1) & 1u;
    ++c.su;
    bool ok = mbar_wait(&bars->s_full[sb], sph, abort, p.err, kSiteSoftS);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + 128u * sb + 32u * g + lane_base;
    const uint32_t pb = c.pu % T::kNP, pn = c.pu / T::kNP;
    ++c.pu;
    const uint32_t tP = tmem + T::kColP + 64u * pb + 16u * g + lane_base;
    // Two pieces of 16 keys (one bias cell each), the second piece's
    // tensor-memory load in flight while the first is computed.
    const uint32_t sfr = sb ? sf_remote[1] : sf_remote[0];
    if (nvalid == kKeys)
      ok = tile_split<false>(tS, tP, bc, p.bias_mul, k, 32 * g, nvalid, pn, pb, sb, sfr, bars,
                             rank, p, abort, acc);
    else
      ok = tile_split<true>(tS, tP, bc, p.bias_mul, k, 32 * g, nvalid, pn, pb, sb, sfr, bars,
                            rank, p, abort, acc);
    if (!ok) return false;
    tmem_wait_st();
    tc_fence_before();
    warp_arrive_leader(&bars->p_full[pb], pb ? pf_remote[1] : pf_remote[0], rank);
    bc[0] = bn[0];
    bc[1] = bn[1];
  }
  d = acc.x + acc.y;
  return true;
}

// First pass of the two-pass schedule (kRowMax): the row's largest biased
// score y = s qk_scale + b bias_mul over this segment's keys, every
// warpgroup 32 keys of every key tile, in the steps of issuer_rowmax (the
// buffer pair released once both tiles' logits are in registers).  No P, no
// PV.  c.su counts steps.
__device__ __forceinline__ bool segment_rowmax(const Segment &sg, const float *brow,
                                               uint32_t tmem, uint32_t lane_base, int g,
                                               const Params &p, Barriers *bars, uint32_t rank,
                                               SoftCounters &c, volatile int *abort,
                                               float &ymax) {
  const uint32_t sf0 = cluster_addr(&bars->s_free[0], 0);  // the even CTA's s_free
  for (int j0 = sg.kb; j0 < sg.ke; j0 += kTilesPerSlot) {
    const int nt = sg.ke - j0 < kTilesPerSlot ? sg.ke - j0 : kTilesPerSlot;
    const uint32_t b = c.su & 1u, ph = (c.su >> 1) & 1u;
    ++c.su;
    float bc[kTilesPerSlot][2];
#pragma unroll
    for (int t = 0; t < kTilesPerSlot; ++t)
      if (t < nt) load_bias(brow, j0 + t, g, p.P, bc[t]);
    const bool okw = mbar_wait(&bars->s_full[b], ph, abort, p.err, kSiteSoftS);
    if (!__all_sync(0xffffffffu, okw)) return false;
    tc_fence_after();
    // Both tiles' logits in flight together.
    uint32_t s[kTilesPerSlot][32];
    const uint32_t t0 = tmem + 256u * b + 32u * g + lane_base;
    tmem_ld32(t0, s[0]);
    if (nt > 1) tmem_ld32(t0 + 128u, s[1]);
    tmem_wait_ld(s[0]);
    if (nt > 1) tmem_wait_ld(s[1]);
#pragma unroll
    for (int t = 0; t < kTilesPerSlot; ++t) {
      if (t < nt) {
        const int j = j0 + t;
        const int nvalid = (j + 1 == p.n_kt) ? p.last_valid : kKeys;
        const float b0 = bc[t][0] * p.bias_mul, b1 = bc[t][1] * p.bias_mul;
        if (32 * g + 32 <= nvalid) {
          // qk_scale > 0 and one bias cell per 16 keys: the largest score of
          // a 16-key piece comes from its largest logit.
          float m0 = __uint_as_float(s[t][0]), m1 = __uint_as_float(s[t][16]);
#pragma unroll
          for (int e = 1; e < 16; ++e) {
            m0 = fmaxf(m0, __uint_as_float(s[t][e]));
            m1 = fmaxf(m1, __uint_as_float(s[t][16 + e]));
          }
          ymax = fmaxf(ymax, fmaxf(fmaf(m0, p.qk_scale, b0), fmaf(m1, p.qk_scale, b1)));
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float y = fmaf(__uint_as_float(s[t][e]), p.qk_scale, e < 16 ? b0 : b1);
            if (32 * g + e < nvalid) ymax = fmaxf(ymax, y);
          }
        }
      }
    }
    tc_fence_before();
    warp_arrive_leader(&bars->s_free[b], sf0 + 8u * b, rank);
  }
  return true;
}

// Running-max segment: the four threads of a row share its maximum per key
// tile (through shared memory).  When the maximum grows past the lazy
// threshold, this warpgroup's DV/4 columns of O are rescaled, after the
// previous PV into O has finished.
template <int MODE, int DV>
__device__ __forceinline__ bool segment_online(const Segment &sg, const float *brow,
                                               uint32_t tmem, uint32_t lane_base, int g, int r,
                                               const Params &p, Barriers *bars, Xchg *xc,
                                               uint32_t rank, const uint32_t (&sf_remote)[2],
                                               const uint32_t (&pf_remote)[2],
                                               SoftCounters &c, volatile int *abort,
                                               float &m, float &d) {
  using T = Tmem<DV>;
  float bc[2], bn[2] = {0.f, 0.f};
  load_bias(brow, sg.kb, g, p.P, bc);
  for (int j = sg.kb; j < sg.ke; ++j) {
    if (j + 1 < sg.ke) load_bias(brow, j + 1, g, p.P, bn);
    const int nvalid = (j + 1 == p.n_kt) ? p.last_valid : kKeys;
    const uint32_t par = c.su & 1u;
    uint32_t s[32];
    if (!load_s(bars, tmem, g, lane_base, rank, sf_remote, c, p, abort, s)) return false;
    const float b0 = bc[0] * p.bias_mul, b1 = bc[1] * p.bias_mul;
    float x[32];
    float mt = -INFINITY;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float v = online_logit<MODE>(__uint_as_float(s[e]), e < 16 ? b0 : b1, p);
      x[e] = (32 * g + e < nvalid) ? v : -INFINITY;
      mt = fmaxf(mt, x[e]);
    }
    xc->mpart[par][g][r] = mt;
    if (!exchange(&bars->xm, c.xmcount, abort, p.err)) return false;
#pragma unroll
    for (int q = 0; q < kWG; ++q) mt = fmaxf(mt, xc->mpart[par][q][r]);
    float factor = 1.f;
    if (mt > m + kRescaleThreshold || m == -INFINITY) {
      factor = (m == -INFINITY) ? 0.f : ex2_approx(m - mt);
      m = mt;
      d *= factor;
    }
    if (j > sg.kb && __any_sync(0xffffffffu, factor != 1.f)) {
      // PV(j - 1) used P buffer (pu - 1) % NP; it is that buffer's last phase.
      const uint32_t prev = c.pu - 1;
      const bool ok = mbar_wait(&bars->pv_done[prev % T::kNP], (prev / T::kNP) & 1u, abort,
                                p.err, kSiteSoftPV);
      if (!__all_sync(0xffffffffu, ok)) return false;
      tc_fence_after();
      const uint32_t tO = tmem + T::kColO + (DV / 4) * g + lane_base;
      // This warpgroup's DV/4 columns, 16 at a time.
#pragma unroll 1
      for (int cc = 0; cc < DV / 4; cc += 16) {
        uint32_t o[16];
        tmem_ld16(tO + cc, o);
        tmem_wait_ld16(o);
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
        tmem_st16(tO + cc, o);
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
    d += acc;
    // store_p waits for the stores above (tcgen05.wait::st) before arriving.
    if (!store_p<DV>(bars, tmem, g, lane_base, rank, pf_remote, c, p, abort, pk)) return false;
    bc[0] = bn[0];
    bc[1] = bn[1];
  }
  return true;
}

template <int MODE, int DV>
__device__ __forceinline__ void softmax_role(Barriers *bars, Xchg *xc, float *stage, uint32_t tmem,
                                             const CUtensorMap *tm_o, const Params &p,
                                             uint32_t rank, volatile int *abort) {
  using T = Tmem<DV>;
  const int g = threadIdx.x >> 7;         // warpgroup
  const int r = threadIdx.x & 127;        // tile row == tensor-memory lane
  const int h = r >> 4, il = r & 15;      // head, position inside the block
  const uint32_t lane_base = static_cast<uint32_t>(r >> 5) << 21;  // (32 * quarter) << 16
  const uint32_t sf_remote[2] = {cluster_addr(&bars->s_free[0], 0),
                                 cluster_addr(&bars->s_free[1], 0)};
  const uint32_t pf_remote[2] = {cluster_addr(&bars->p_full[0], 0),
                                 cluster_addr(&bars->p_full[1], 0)};
  constexpr bool kStatic = fixed_shift<MODE>();
  SoftCounters c;
  bool ok = true;
  Cursor cu = cursor_begin(p);
  Segment sg;
  while (ok && next_segment(p, cu, sg)) {
    const int b = sg.item / p.pairs;
    const int I0 = (sg.item % p.pairs) * 2;
    const int I = tile_block(p, I0, rank);
    const bool valid = I0 + static_cast<int>(rank) < p.nb;
    const int pos = I * 16 + il;  // this thread's query position
    const float *brow = p.bias + static_cast<long long>(b) * p.bias_bstride +
                        (static_cast<size_t>(h) * p.bias_rows + I) * p.P;
    if constexpr (MODE == kRowMax) {
      const bool writes = valid && pos < p.Lq;
      const size_t row = (static_cast<size_t>(b) * kH + h) * p.Lq + static_cast<size_t>(pos);
      // First pass: the row's largest logit (log2 units) into lse, for the
      // second pass's shift.  cap tanh is increasing, so the largest capped
      // logit is the cap of the largest biased score.
      float ymax = -INFINITY;
      ok = segment_rowmax(sg, brow, tmem, lane_base, g, p, bars, rank, c, abort, ymax);
      if (!ok) break;
      // Double-buffered by segment parity, like the row sums below.
      float(*mp)[128] = xc->mpart[c.xmcount & 1u];
      mp[g][r] = ymax;
      ok = exchange(&bars->xm, c.xmcount, abort, p.err);
      if (!ok) break;
      float mx = mp[0][r];
#pragma unroll
      for (int q = 1; q < kWG; ++q) mx = fmaxf(mx, mp[q][r]);
      float mrow = p.A > 0.f ? p.A * tanh_approx(mx) : mx;
      if (sg.dest == kDestMerge) {
        // Second piece of a split pair: the first piece's maximum is in lse.
        griddep_wait();
        if (writes) mrow = fmaxf(mrow, p.lse[row]);
      }
      if (writes && g == 0) p.lse[row] = mrow;
      continue;
    }
    // The fixed shift: p.shift, or with row shifts the smallest integer at or
    // above the row's largest logit, which the first pass left in lse.
    float shift = p.shift;
    if constexpr (row_shift<MODE>()) {
      const size_t row = (static_cast<size_t>(b) * kH + h) * p.Lq + static_cast<size_t>(pos);
      shift = (valid && pos < p.Lq) ? ceilf(p.lse[row]) : 0.f;
    }
    float m = kStatic ? shift : -INFINITY;  // log2 units
    float d = 0.f;
    if constexpr (kStatic && DV == 128) {
      ok = segment_static_grouped<MODE, DV>(sg, brow, tmem, lane_base, g, p, bars, rank, c,
                                            abort, shift, d);
    } else if constexpr (kStatic) {
      ok = segment_static<MODE, DV>(sg, brow, tmem, lane_base, g, p, bars, rank, sf_remote,
                                    pf_remote, c, abort, d);
    } else {
      ok = segment_online<MODE, DV>(sg, brow, tmem, lane_base, g, r, p, bars, xc, rank,
                                    sf_remote, pf_remote, c, abort, m, d);
    }
    if (!ok) break;

    // Epilogue: d = sum of the four warpgroups' partial sums; out = O / d
    // over this segment's keys (warpgroup g writes columns [g DV/4, (g+1)
    // DV/4) of the row) and lse.  The copy of block I0 in an odd CTA past the
    // end of an odd block count writes nothing.
    const bool writes = valid && pos < p.Lq;  // rows past the end of a partial block: none
    const size_t row = (static_cast<size_t>(b) * kH + h) * p.Lq + static_cast<size_t>(pos);
    float lse_a = 0.f;
    if (sg.dest == kDestMerge) {
      // The first piece of this pair was written by the previous launch;
      // every thread reads it before warpgroup 0 overwrites lse below (the
      // exchange orders the two).
      griddep_wait();
      if (writes) lse_a = p.lse[row];
    }
    // The partial sums are published before the wait for the last PV, so
    // the exchange has normally completed when O is ready.  Double-buffered
    // by segment parity: a warp writes the buffer of segment n + 2 only after
    // the exchange of segment n + 1, which every warp joins after reading
    // segment n's.
    float(*dp)[128] = xc->dpart[c.xdcount & 1u];
    dp[g][r] = d;
    warp_arrive(&bars->xd);
    ok = mbar_wait(&bars->o_full, c.ocount & 1u, abort, p.err, kSiteSoftO);
    ++c.ocount;
    if (ok) ok = mbar_wait(&bars->xd, c.xdcount & 1u, abort, p.err, kSiteXchg);
    ++c.xdcount;
    if (!__all_sync(0xffffffffu, ok)) {
      ok = false;
      break;
    }
    tc_fence_after();
    float dsum = 0.f;
#pragma unroll
    for (int q = 0; q < kWG; ++q) dsum += dp[q][r];
    const uint32_t tO = tmem + T::kColO + (DV / 4) * g + lane_base;
    const float lse_b = (m + lg2_approx(dsum)) * kLn2;
    float *orow_base;
    float *lse_dst;
    if (sg.dest == kDestScratch) {
      const size_t slot = (static_cast<size_t>(cluster_index()) * 2 + rank) * 128 + r;
      orow_base = p.ws_out + slot * DV;
      lse_dst = p.ws_lse + slot;
    } else {
      orow_base = p.out + row * DV;
      lse_dst = p.lse + row;
    }
    float4 *orow = reinterpret_cast<float4 *>(orow_base + (DV / 4) * g);
    float wb = 1.f / dsum, wa = 0.f, lse_w = lse_b;
    if (sg.dest == kDestMerge) {
      // Log-sum-exp merge with the first piece: lse = log(e^a + e^b),
      // out = e^(a - lse) out_a + e^(b - lse) O_b / d_b.
      const float M = fmaxf(lse_a, lse_b);
      const float ea = ex2_approx((lse_a - M) * kLog2e);
      const float eb = ex2_approx((lse_b - M) * kLog2e);
      const float inv = 1.f / (ea + eb);
      wa = ea * inv;
      wb = eb * inv / dsum;
      lse_w = M + lg2_approx(ea + eb) * kLn2;
    }
    if constexpr (DV == 128) {
      const int lane = static_cast<int>(lane_id());
      float *slot = stage + (threadIdx.x >> 5) * kStageWarpFloats;
      const int r0 = r - lane;  // the warp's first tile row
      // Once this warp's reads of O have completed (tcgen05.wait::ld), the
      // PV issuer may start the next segment's O over it.
      auto release_o = [&] {
        if constexpr (p_in_place<MODE, DV>()) {
          tc_fence_before();
          warp_arrive_leader(&bars->o_free, cluster_addr(&bars->o_free, 0), rank);
        }
      };
      // The bulk store of this warp's previous segment has read the slot.
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      if (sg.dest == kDestOut) {
        // This warpgroup's 32 columns of the warp's 32 rows (heads 2 (warp
        // % 4) and + 1, positions 16 I .. 16 I + 15): scaled into the slot
        // in the 128-byte swizzle, then one bulk tensor store.  Rows past Lq
        // lie outside the tensor and are not written.
        if (valid) {
#pragma unroll
          for (int c16 = 0; c16 < 2; ++c16) {
            uint32_t o[16];
            tmem_ld16(tO + 16u * c16, o);
            tmem_wait_ld16(o);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int chunk = (4 * c16 + e) ^ (lane & 7);
              *reinterpret_cast<float4 *>(slot + 32 * lane + 4 * chunk) = make_float4(
                  __uint_as_float(o[4 * e]) * wb, __uint_as_float(o[4 * e + 1]) * wb,
                  __uint_as_float(o[4 * e + 2]) * wb, __uint_as_float(o[4 * e + 3]) * wb);
            }
          }
        }
        release_o();
        if (valid) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_4d(tm_o, slot, 32 * g, I * 16, 2 * ((threadIdx.x >> 5) & 3), b);
            bulk_commit_group();
          }
        }
      } else {
        // This warpgroup's 32 columns of its warp's 32 rows, 16 columns at a
        // time: scaled into the warp's staging rows, then stored by groups of
        // four lanes, one 64-byte row segment each.
#pragma unroll 1
        for (int c16 = 0; c16 < 2; ++c16) {
          uint32_t o[16];
          tmem_ld16(tO + 16u * c16, o);
          tmem_wait_ld16(o);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<float4 *>(slot + lane * kStageRow + 4 * e) =
                make_float4(__uint_as_float(o[4 * e]) * wb, __uint_as_float(o[4 * e + 1]) * wb,
                            __uint_as_float(o[4 * e + 2]) * wb, __uint_as_float(o[4 * e + 3]) * wb);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int rr = 8 * k + (lane >> 2), cc = lane & 3;  // staging row, float4 column
            float4 val = *reinterpret_cast<const float4 *>(slot + rr * kStageRow + 4 * cc);
            const int rt = r0 + rr;  // tile row
            const int pos_t = I * 16 + (rt & 15);
            const float wa_t = __shfl_sync(0xffffffffu, wa, rr);
            if (valid && pos_t < p.Lq) {
              float *dst_row;
              if (sg.dest == kDestScratch) {
                const size_t slot_row = (static_cast<size_t>(cluster_index()) * 2 + rank) * 128 + rt;
                dst_row = p.ws_out + slot_row * DV;
              } else {
                const size_t row_t = (static_cast<size_t>(b) * kH + (rt >> 4)) * p.Lq +
                                     static_cast<size_t>(pos_t);
                dst_row = p.out + row_t * DV;
              }
              float4 *dst = reinterpret_cast<float4 *>(dst_row + 32 * g + 16 * c16) + cc;
              if (sg.dest == kDestMerge) {
                const float4 av = *dst;
                val.x = fmaf(wa_t, av.x, val.x);
                val.y = fmaf(wa_t, av.y, val.y);
                val.z = fmaf(wa_t, av.z, val.z);
                val.w = fmaf(wa_t, av.w, val.w);
              }
              *dst = val;
            }
          }
          __syncwarp();
        }
        release_o();
      }
    } else {
      // This warpgroup's DV / 4 columns of the row, 16 at a time (every lane
      // loads: tcgen05.ld is warp-wide; rows that do not exist store nothing).
#pragma unroll 1
      for (int c16 = 0; c16 < DV / 4 / 16; ++c16) {
        uint32_t o[16];
        tmem_ld16(tO + 16u * c16, o);
        tmem_wait_ld16(o);
        if (writes) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float4 val =
                make_float4(__uint_as_float(o[4 * e]) * wb, __uint_as_float(o[4 * e + 1]) * wb,
                            __uint_as_float(o[4 * e + 2]) * wb, __uint_as_float(o[4 * e + 3]) * wb);
            if (sg.dest == kDestMerge) {
              const float4 av = orow[4 * c16 + e];
              val.x = fmaf(wa, av.x, val.x);
              val.y = fmaf(wa, av.y, val.y);
              val.z = fmaf(wa, av.z, val.z);
              val.w = fmaf(wa, av.w, val.w);
            }
            orow[4 * c16 + e] = val;
          }
        }
      }
    }
    if (writes) {
      if (g == 0) *lse_dst = lse_w;
    }
    tc_fence_before();
  }
  if constexpr (DV == 128) {
    // Every bulk store this warp started completes before the CTA exits.
    if (lane_id() == 0) bulk_wait_all();
    __syncwarp();
  }
}

// --------------------------------------------------------------------------
template <int MODE, int DV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *q_s = smem_raw + pad;                      // this CTA's query tile
  uint8_t *k_s = q_s + kQTileBytes;                   // K ring
  uint8_t *v_s = k_s + kStages * kKSlotBytes;         // V ring
  float *stage = reinterpret_cast<float *>(v_s + v_stages<DV>() * v_slot_bytes<DV>());
  Barriers *bars = reinterpret_cast<Barriers *>(reinterpret_cast<uint8_t *>(stage) +
                                                stage_bytes<DV>());
  auto *xc = reinterpret_cast<Xchg *>(reinterpret_cast<uint8_t *>(bars) + sizeof(Barriers));
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    // A second launch of a two-phase schedule may start once every CTA of
    // this grid has got here; it only reads this grid's results after
    // griddepcontrol.wait.
    griddep_launch_dependents();
    const uint32_t loads = rank == 0 ? 2 : 1;  // producer (+ relay, even CTA)
    mbar_init(&bars->q_full, loads);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], loads);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < v_stages<DV>(); ++s) {
      mbar_init(&bars->v_full[s], loads);
      mbar_init(&bars->v_empty[s], 1);
    }
    // Static cap at value width 128: one warp group per S and P buffer;
    // otherwise every softmax warp takes part in every key tile.
    constexpr uint32_t kSPArrivals =
        p_in_place<MODE, DV>() ? kPairSoftWarps / 2 : kPairSoftWarps;
    for (int u = 0; u < 3; ++u) {
      mbar_init(&bars->s_full[u], 1);
      if (u < 2) mbar_init(&bars->s_free[u], kSPArrivals);
      mbar_init(&bars->p_full[u], kSPArrivals);
      mbar_init(&bars->pv_done[u], 1);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_free, kPairSoftWarps);
    mbar_init(&bars->xm, kSoftWarps);
    mbar_init(&bars->xd, kSoftWarps);
    mbar_init(&bars->drain, 2);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpLoadQK && lane_id() == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
  }
  if (warp == kWarpLoadV && lane_id() == 0) prefetch_tensormap(&tm_v);
  if (warp == kWarpIssueS) {
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

  if (warp >= kSoftWarps) {  // the four role warps
    regs_dec<kRegsLow>();
    if (rank == 0 && warp == kWarpIssueS) {
      // The whole warp.
      if constexpr (MODE == kRowMax)
        issuer_rowmax(q_s, k_s, bars, tmem, p, abort);
      else
        issuer_s<p_in_place<MODE, DV>()>(q_s, k_s, bars, tmem, p, abort);
    } else if (rank == 0 && warp == kWarpIssuePV) {
      if constexpr (MODE == kRowMax) {
        // No PV in the first pass; the drain still counts this warp.
        umma2_commit_self_w(&bars->drain);
        drain_wait(&bars->drain, 0);
      } else {
        issuer_pv<DV, p_in_place<MODE, DV>()>(v_s, bars, tmem, p, abort);
      }
    } else if (lane_id() == 0) {
      if (warp == kWarpLoadQK) {
        producer_qk(&tm_q, &tm_k, q_s, k_s, bars, p, rank, abort);
      } else if (warp == kWarpLoadV) {
        if constexpr (MODE != kRowMax) producer_v<DV>(&tm_v, v_s, bars, p, rank, abort);
      } else if (warp == kWarpIssueS) {
        relay_qk(bars, p, abort);
      } else if (warp == kWarpIssuePV) {
        if constexpr (MODE != kRowMax) relay_v<DV>(bars, p, abort);
      }
    }
  } else {
    regs_inc<kRegsHigh>();  // covered by the role warpgroup's decrease above
    softmax_role<MODE, DV>(bars, xc, stage, tmem, &tm_o, p, rank, abort);
  }
  __syncwarp();
  // No CTA leaves while the other may still use its shared or tensor memory:
  // the even CTA's MMAs have drained and the odd CTA's remote arrivals are
  // done once every thread of both CTAs is here.
  tc_fence_before();
  cluster_sync();
  if (warp == kWarpIssueS) {
    tc_fence_after();
    tmem_dealloc2(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------------------
// Split-pair merge of kSchedRange.  Every segment of a split pair finishes
// like a whole pair but over its own key range: a normalised partial output
// and the partial log-sum-exp.  The first segment (key tile 0) writes them to
// out / lse, the others to the scratch slot of their cluster (a cluster
// starts at most one segment in the middle of a pair).  This kernel, launched
// right after on the same stream, merges the pieces of every split pair:
//   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) out_s.
// kMergeBlocksPerBoundary blocks per cluster boundary; only the boundary that
// is the first one inside a pair merges that pair.  One warp per output row
// (query tile row / 128, row % 128): lane l merges the 4-column groups l,
// l + 32, ... of the row's DV columns over the pieces, and lane 0 writes the
// merged lse once every lane has read the first piece's.
constexpr int kMergeThreads = 256;
constexpr int kMergeRowsPerBlock = kMergeThreads / 32;
constexpr int kMergeBlocksPerBoundary = 2 * 128 / kMergeRowsPerBlock;

template <int DV>
__global__ void __launch_bounds__(kMergeThreads)
    attn_merge_kernel(const __grid_constant__ Params p, int grid) {
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
  if (pos >= p.Lq) return;  // past the end of a partial last block
  const size_t row = (static_cast<size_t>(b) * kH + h) * p.Lq + static_cast<size_t>(pos);
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
  for (int cc = lane; cc < DV / 4; cc += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n_seg; ++s) {
      const float l = s == 0 ? p.lse[row] : p.ws_lse[slot(s)];
      const float wgt = ex2_approx((l - lse) * kLog2e);
      const float4 v = reinterpret_cast<const float4 *>(
          s == 0 ? p.out + row * DV : p.ws_out + slot(s) * DV)[cc];
      acc.x = fmaf(wgt, v.x, acc.x);
      acc.y = fmaf(wgt, v.y, acc.y);
      acc.z = fmaf(wgt, v.z, acc.z);
      acc.w = fmaf(wgt, v.w, acc.w);
    }
    reinterpret_cast<float4 *>(p.out + row * DV)[cc] = acc;
  }
  __syncwarp();  // every lane has read p.lse[row]
  if (lane == 0) p.lse[row] = lse;
}

}  // namespace attn

// --------------------------------------------------------------------------
// Host side.

static bool encode_map(EncodeTiledFn enc, CUtensorMap *map, const void *base,
                       int rank, const cuuint64_t *dims,
                       const cuuint64_t *strides, const cuuint32_t *box,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B,
                       CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, dtype, rank,
                   const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

// One-time per-device setup of a kernel (mode, value width): shared-memory
// opt-in, the register check, and how many 2-CTA clusters can be resident.
// The per-device table is written under g_cfg_mu, so two host threads making
// their first call on a device at once configure it once.
std::mutex g_cfg_mu;
constexpr int kCfgDevices = 64;

template <int MODE, int DV>
cudaError_t configure_mode(int *max_clusters) {
  static int clusters[kCfgDevices] = {0};  // 0: not configured yet
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kCfgDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_cfg_mu);
  if (clusters[dev] == 0) {
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
  }
  *max_clusters = clusters[dev];
  return cudaSuccess;
}

template <int DV>
cudaError_t configure_any(int mode, int *max_clusters) {
  using namespace attn;
  if constexpr (DV == 128) {
    switch (mode) {
      case kRowMax: return configure_mode<kRowMax, DV>(max_clusters);
      case kRowShift: return configure_mode<kRowShift, DV>(max_clusters);
      case kRowShiftCap: return configure_mode<kRowShiftCap, DV>(max_clusters);
      default: break;
    }
  }
  switch (mode) {
    case kStaticCap: return configure_mode<kStaticCap, DV>(max_clusters);
    case kOnlineCap: return configure_mode<kOnlineCap, DV>(max_clusters);
    default: return configure_mode<kNoCap, DV>(max_clusters);
  }
}

// The fixed shift s (log2 units) puts every probability 2^(A t - s) of a row,
// A = cap log2(e) and t in (-1, 1), in (2^(-A-s), 2^(A-s)).  The smallest
// must stay a normal fp32 number (the row's largest probability may be that
// small, and the exponent insertion of exp2_poly2_fma must not leave the
// exponent field) and the largest, times L and |v|, must not overflow the
// sums.  s = ceil(A) (probabilities up to 1) meets both up to A = 60; above,
// s = 120 - ceil(A) keeps the exponents in [-120, 2 ceil(A) - 120], which
// stays far from overflow up to cap = 60 (A = 86.6, probabilities below
// 2^54).  Larger caps run the running maximum.
int attn_mode(float cap) {
  using namespace attn;
  if (std::isinf(cap)) return kNoCap;
  return cap <= 60.0f ? kStaticCap : kOnlineCap;
}

float attn_static_shift(float A) {
  const float ca = ceilf(A);
  return ca <= 60.0f ? ca : 120.0f - ca;
}

// Value width 128 without scratch runs the caps beyond the fixed shift's
// range (cap > 60, and no cap) in two passes over whole pairs of query
// tiles: kRowMax writes every row's largest logit into lse, then the
// fixed-shift kernel runs with each row's own shift ceil(max) (kRowShift,
// kRowShiftCap), instead of the running maximum, whose exchange of the
// maxima between the four warpgroups on every key tile costs about twice the
// time.  Whole pairs, because a split pair's second piece would need the
// maximum after the first piece has overwritten lse.
bool attn_two_pass(int mode, int dv, bool scratch) {
  return (mode == attn::kOnlineCap || mode == attn::kNoCap) && dv == 128 && !scratch;
}
int attn_second_pass_mode(int mode) {
  return mode == attn::kNoCap ? attn::kRowShift : attn::kRowShiftCap;
}

// --------------------------------------------------------------------------
// Schedules.
struct Plan {
  int sched = attn::kSchedUnits;
  int clusters = 0;       // first (or only) launch
  int tail_clusters = 0;  // second launch of a two-phase schedule (0: none)
  int whole = 1;          // kSchedRange: whole pairs (no merge kernel)
  int n_whole = 0, split_at = 0;
  std::vector<int> wb, fb;
};

// Whole pairs, as evenly as they go: cluster c takes items
// [n c / G, n (c+1) / G).
void plan_whole(int n_items, int G, Plan *pl) {
  const int clusters = std::min(G, n_items);
  pl->sched = attn::kSchedUnits;
  pl->clusters = clusters;
  pl->tail_clusters = 0;
  pl->n_whole = n_items;
  pl->split_at = 0;
  pl->wb.assign(clusters + 1, 0);
  pl->fb.assign(clusters + 1, 0);
  for (int c = 0; c <= clusters; ++c)
    pl->wb[c] = static_cast<int>(static_cast<long long>(n_items) * c / clusters);
}

// Two-phase packing check for a first launch of at most t key-tile steps per
// cluster: nw whole pairs (n_kt steps each) and ns first pieces (a steps
// each, a < n_kt) into G clusters.  Starts from the most whole pairs per
// cluster and trades whole pairs for first pieces where a trade gains the
// most (clusters at one level trade alike, so levels are counted, not
// clusters).  On success gives the per-cluster counts.
bool pack_first_launch(int t, int nw, int ns, int n_kt, int a, int G, std::vector<int> *x,
                       std::vector<int> *y) {
  const int xmax = t / n_kt;
  if (static_cast<long long>(xmax) * G < nw) return false;
  auto firsts = [&](int xx) { return (t - xx * n_kt) / a; };
  std::vector<long long> cnt(xmax + 1, 0);  // clusters holding x whole pairs
  cnt[xmax] = G;
  long long spare = static_cast<long long>(xmax) * G - nw;  // removable wholes
  long long have = static_cast<long long>(G) * firsts(xmax);
  while (have < ns && spare > 0) {
    int best = -1, gain = 0;
    for (int xx = 1; xx <= xmax; ++xx) {
      if (cnt[xx] == 0) continue;
      const int g = firsts(xx - 1) - firsts(xx);
      if (g > gain) {
        gain = g;
        best = xx;
      }
    }
    if (best < 0) break;
    const long long need = (ns - have + gain - 1) / gain;
    const long long k = std::min({cnt[best], spare, need});
    cnt[best] -= k;
    cnt[best - 1] += k;
    have += k * gain;
    spare -= k;
  }
  if (have < ns) return false;
  // Clusters in order of decreasing whole pairs; hand out exactly nw wholes
  // and ns first pieces.
  x->assign(G, 0);
  y->assign(G, 0);
  int c = 0;
  for (int xx = xmax; xx >= 0; --xx)
    for (long long i = 0; i < cnt[xx]; ++i) (*x)[c++] = xx;
  int wl = nw, fl = ns;
  for (int cc = 0; cc < G; ++cc) {
    (*x)[cc] = std::min((*x)[cc], wl);
    wl -= (*x)[cc];
  }
  for (int cc = 0; cc < G; ++cc) {
    (*y)[cc] = std::min(firsts((*x)[cc]), fl);
    fl -= (*y)[cc];
  }
  return wl == 0 && fl == 0;
}

// Extra cost of a second launch, in key-tile steps: its prologue (barriers,
// tensor memory, the Q tile and the first logits) before the softmax runs.
constexpr int kTailCostSteps = 4;
// Extra cost of every segment (a whole pair or a piece), in key-tile steps:
// the drain of its last PV, the epilogue and the restart of the step-buffer
// pipeline, about 7,000-9,000 cycles against 1,790 per steady-state step.
// With it the planner stops cutting a cluster's work into many short first
// pieces (measured at B = 1: L = 4096 89.2 -> 80.0 us, L = 6144 160.8 ->
// 154.8 us, L = 8192 249.8 -> 248.8 us, against a model without it).
constexpr int kSegCostSteps = 5;

// No-scratch schedule: whole pairs, or two phases when that beats them.  A
// plan's cost is its critical path in key-tile steps, every segment counted
// kSegCostSteps longer.
void plan_no_scratch(int n_items, int n_kt, int G, Plan *pl) {
  plan_whole(n_items, G, pl);
  constexpr int c = kSegCostSteps;
  const long long whole_cost = static_cast<long long>((n_items + G - 1) / G) * (n_kt + c);
  if (n_kt < 2 || n_items > 8 * G || n_items <= G) return;
  const int ns = G;  // one second piece per cluster of the second launch
  const int nw = n_items - ns;
  long long best = whole_cost;
  int best_b = 0, best_t = 0;
  for (int b = 1; b < n_kt; ++b) {
    const int a = n_kt - b;
    const long long hi = best - (b + c) - kTailCostSteps - 1;  // t must beat the best so far
    const long long work =
        static_cast<long long>(nw) * (n_kt + c) + static_cast<long long>(ns) * (a + c);
    long long lo = (work + G - 1) / G;
    if (lo > hi) continue;
    std::vector<int> x, y;
    if (!pack_first_launch(static_cast<int>(hi), nw, ns, n_kt + c, a + c, G, &x, &y)) continue;
    long long l = lo, h = hi;  // smallest feasible t in [lo, hi]
    while (l < h) {
      const long long mid = (l + h) / 2;
      if (pack_first_launch(static_cast<int>(mid), nw, ns, n_kt + c, a + c, G, &x, &y))
        h = mid;
      else
        l = mid + 1;
    }
    const long long cost = l + (b + c) + kTailCostSteps;
    if (cost < best) {
      best = cost;
      best_b = b;
      best_t = static_cast<int>(l);
    }
  }
  if (best_b == 0) return;
  std::vector<int> x, y;
  const int a = n_kt - best_b;
  if (!pack_first_launch(best_t, nw, ns, n_kt + c, a + c, G, &x, &y)) return;
  // Drop clusters with no work; ranges stay contiguous per kind.
  std::vector<int> wb(1, 0), fb(1, 0);
  for (int c = 0; c < G; ++c) {
    if (x[c] == 0 && y[c] == 0) continue;
    wb.push_back(wb.back() + x[c]);
    fb.push_back(fb.back() + y[c]);
  }
  pl->sched = attn::kSchedUnits;
  pl->clusters = static_cast<int>(wb.size()) - 1;
  pl->tail_clusters = ns;
  pl->n_whole = nw;
  pl->split_at = a;
  pl->wb = wb;
  pl->fb = fb;
}

// Scratch schedule (kSchedRange): one cluster per SM pair, never more
// clusters than (pair, key tile) steps or scratch slots.  Whole pairs per
// cluster unless that leaves the grid badly balanced: a split pair costs a
// second pass over its rows (partial results, then the merge), so whole pairs
// win while the busiest cluster's extra work stays below kSplitGain pairs.
void plan_range(int n_items, int n_kt, int G, int scratch_slots, Plan *pl) {
  int clusters = std::min(G, scratch_slots);
  const long long steps = static_cast<long long>(n_items) * n_kt;
  if (steps < clusters) clusters = static_cast<int>(steps);
  constexpr double kSplitGain = 0.5;
  const long long per = (n_items + clusters - 1) / clusters;  // busiest cluster
  const double even = static_cast<double>(n_items) / clusters;
  const int whole = (per - even <= kSplitGain) ? 1 : 0;
  if (whole && n_items < clusters) clusters = n_items;
  pl->sched = attn::kSchedRange;
  pl->clusters = clusters;
  pl->tail_clusters = 0;
  pl->whole = whole;
  pl->wb.clear();
  pl->fb.clear();
}

// The schedule for n_items pairs of n_kt key tiles on G clusters: with
// scratch slots, the range schedule; without, whole pairs or two phases.
// Pure host logic (no CUDA call).
Plan plan_for(int n_items, int n_kt, int G, int scratch_slots) {
  Plan pl;
  if (scratch_slots > 0)
    plan_range(n_items, n_kt, G, scratch_slots, &pl);
  else
    plan_no_scratch(n_items, n_kt, std::min(G, kAttnMaxClusters), &pl);
  return pl;
}

// Plans are cached per (items, key tiles, clusters, scratch slots): the
// two-phase search costs more than a launch.
struct PlanKey {
  int n_items, n_kt, G, slots, whole_only;
  bool operator==(const PlanKey &o) const {
    return n_items == o.n_items && n_kt == o.n_kt && G == o.G && slots == o.slots &&
           whole_only == o.whole_only;
  }
};
std::mutex g_plan_mu;
std::vector<std::pair<PlanKey, Plan>> g_plans;

cudaError_t make_plan(int mode, int dv, int n_items, int n_kt, int num_sms, int scratch_slots,
                      Plan *pl) {
  int max_clusters = 0;
  const bool two_pass = attn_two_pass(mode, dv, scratch_slots > 0);
  if (two_pass) {
    int first = 0;
    cudaError_t e1 = configure_any<128>(attn::kRowMax, &first);
    if (e1 != cudaSuccess) return e1;
    mode = attn_second_pass_mode(mode);
  }
  cudaError_t e = dv == 192 ? configure_any<192>(mode, &max_clusters)
                            : configure_any<128>(mode, &max_clusters);
  if (e != cudaSuccess) return e;
  const long long steps = static_cast<long long>(n_items) * n_kt;
  if (steps > (1ll << 30) || steps < 1) return cudaErrorInvalidValue;
  // One cluster per resident SM pair.  The range schedule needs no
  // per-cluster table; the others carry per-cluster ranges in the kernel
  // parameters, sized for kAttnMaxClusters (plan_for clamps them).
  const int G = std::min(num_sms / 2, max_clusters);
  if (G < 1) return cudaErrorInvalidValue;
  const PlanKey key{n_items, n_kt, G, scratch_slots, two_pass ? 1 : 0};
  {
    std::lock_guard<std::mutex> lock(g_plan_mu);
    for (const auto &kv : g_plans)
      if (kv.first == key) {
        *pl = kv.second;
        return cudaSuccess;
      }
  }
  Plan fresh;
  if (two_pass)
    plan_whole(n_items, std::min(G, kAttnMaxClusters), &fresh);
  else
    fresh = plan_for(n_items, n_kt, G, scratch_slots);
  if (fresh.clusters < 1 ||
      (fresh.sched != attn::kSchedRange &&
       (fresh.clusters > kAttnMaxClusters || fresh.tail_clusters > kAttnMaxClusters)))
    return cudaErrorInvalidValue;
  {
    std::lock_guard<std::mutex> lock(g_plan_mu);
    if (g_plans.size() >= 256) g_plans.erase(g_plans.begin());
    g_plans.emplace_back(key, fresh);
  }
  *pl = fresh;
  return cudaSuccess;
}

template <int MODE, int DV>
cudaError_t launch_mode(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                        const CUtensorMap &to, const attn::Params &p, int clusters,
                        bool dependent, cudaStream_t stream) {
  if (!dependent) {
    attn::attn_fwd_kernel<MODE, DV>
        <<<2 * clusters, attn::kThreads, attn::smem_bytes<DV>(), stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError();
  }
  // The second launch of a two-phase schedule: programmatic dependent launch,
  // so its CTAs take the SMs that the first launch's CTAs leave.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(attn::kThreads, 1, 1);
  cfg.dynamicSmemBytes = attn::smem_bytes<DV>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn::attn_fwd_kernel<MODE, DV>, tq, tk, tv, to, p);
}

template <int DV>
cudaError_t launch_dv(int mode, const CUtensorMap &tq, const CUtensorMap &tk,
                      const CUtensorMap &tv, const CUtensorMap &to, const attn::Params &p,
                      int clusters, bool dependent, cudaStream_t stream) {
  using namespace attn;
  if constexpr (DV == 128) {
    switch (mode) {
      case kRowMax:
        return launch_mode<kRowMax, DV>(tq, tk, tv, to, p, clusters, dependent, stream);
      case kRowShift:
        return launch_mode<kRowShift, DV>(tq, tk, tv, to, p, clusters, dependent, stream);
      case kRowShiftCap:
        return launch_mode<kRowShiftCap, DV>(tq, tk, tv, to, p, clusters, dependent, stream);
      default: break;
    }
  }
  switch (mode) {
    case kStaticCap:
      return launch_mode<kStaticCap, DV>(tq, tk, tv, to, p, clusters, dependent, stream);
    case kOnlineCap:
      return launch_mode<kOnlineCap, DV>(tq, tk, tv, to, p, clusters, dependent, stream);
    default: return launch_mode<kNoCap, DV>(tq, tk, tv, to, p, clusters, dependent, stream);
  }
}

}  // namespace

cudaError_t attn_fwd_kernel_count(int64_t B, int64_t Lq, int64_t L, int64_t Dv, float cap,
                                  int num_sms, int scratch_slots, int *count) {
  using namespace attn;
  if (B == 0 || L == 0 || Lq == 0) {
    *count = 0;
    return cudaSuccess;
  }
  const int nb = static_cast<int>((Lq + 15) / 16);
  const int n_items = static_cast<int>(B) * ((nb + 1) / 2);
  const int n_kt = static_cast<int>((L + kKeys - 1) / kKeys);
  Plan pl;
  cudaError_t e = make_plan(attn_mode(cap), static_cast<int>(Dv), n_items, n_kt, num_sms,
                            scratch_slots, &pl);
  if (e != cudaSuccess) return e;
  if (attn_two_pass(attn_mode(cap), static_cast<int>(Dv), scratch_slots > 0)) {
    // The row maxima (one or two launches), then the row-shift kernel.
    Plan p1;
    e = make_plan(kRowMax, static_cast<int>(Dv), n_items, n_kt, num_sms, 0, &p1);
    if (e != cudaSuccess) return e;
    *count = (p1.tail_clusters > 0 ? 2 : 1) + 1;
  } else if (pl.sched == kSchedRange)
    *count = (pl.clusters < 2 || pl.whole) ? 1 : 2;
  else
    *count = pl.tail_clusters > 0 ? 2 : 1;
  return cudaSuccess;
}

cudaError_t attn_fwd_clusters(int64_t B, int64_t L, int64_t Dv, float cap, int num_sms,
                              int scratch_slots, int *clusters) {
  const int nb = static_cast<int>((L + 15) / 16);
  const int n_items = static_cast<int>(B) * ((nb + 1) / 2);
  const int n_kt = static_cast<int>((L + attn::kKeys - 1) / attn::kKeys);
  Plan pl;
  cudaError_t e = make_plan(attn_mode(cap), static_cast<int>(Dv), n_items, n_kt, num_sms,
                            scratch_slots, &pl);
  if (e != cudaSuccess) return e;
  *clusters = pl.clusters;
  return cudaSuccess;
}

void attn_fwd_schedule(int64_t B, int64_t L, int sm_pairs, int scratch_slots, int *sched,
                       int *clusters, int *tail_clusters, int *whole, int *n_whole,
                       int *split_at, int *wb, int *fb) {
  const int nb = static_cast<int>((L + 15) / 16);
  const int n_items = static_cast<int>(B) * ((nb + 1) / 2);
  const int n_kt = static_cast<int>((L + attn::kKeys - 1) / attn::kKeys);
  const Plan pl = plan_for(n_items, n_kt, sm_pairs, scratch_slots);
  *sched = pl.sched;
  *clusters = pl.clusters;
  *tail_clusters = pl.tail_clusters;
  *whole = pl.whole;
  *n_whole = pl.n_whole;
  *split_at = pl.split_at;
  for (int c = 0; c <= kAttnMaxClusters; ++c) {
    wb[c] = c < static_cast<int>(pl.wb.size()) ? pl.wb[c] : 0;
    fb[c] = c < static_cast<int>(pl.fb.size()) ? pl.fb[c] : 0;
  }
}

cudaError_t launch_attn_fwd(const AttnLaunch &a) {
  using namespace attn;
  const int64_t B = a.B, L = a.L, Lq = a.Lq;
  if (a.Dv != 128 && a.Dv != 192) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dims[4] = {kD, static_cast<cuuint64_t>(Lq), kH,
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {kD * 2, static_cast<cuuint64_t>(Lq) * kD * 2,
                                   static_cast<cuuint64_t>(Lq) * kD * 2 * kH};
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
  // out [B, H, Lq, Dv] fp32, stored by the value-width-128 epilogue one box
  // of 32 columns x 16 positions x 2 heads per softmax warp (128-byte rows,
  // 128-byte swizzle).  Value width 192 stores directly and never reads it.
  CUtensorMap to = tq;
  if (a.Dv == 128) {
    const cuuint64_t odims[4] = {128, static_cast<cuuint64_t>(Lq), kH,
                                 static_cast<cuuint64_t>(B)};
    const cuuint64_t ostrides[3] = {128 * 4, static_cast<cuuint64_t>(Lq) * 128 * 4,
                                    static_cast<cuuint64_t>(Lq) * 128 * 4 * kH};
    const cuuint32_t obox[4] = {32, 16, 2, 1};
    if (!encode_map(a.encode, &to, a.out, 4, odims, ostrides, obox, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
      return cudaErrorInvalidValue;
  }
  Params p;
  p.bias = a.bias;
  p.out = a.out;
  p.lse = a.lse;
  p.err = a.err;
  p.ws_out = nullptr;
  p.ws_lse = nullptr;
  p.L = static_cast<int>(L);
  p.Lq = static_cast<int>(Lq);
  p.P = static_cast<int>((L + 15) / 16);
  p.nb = static_cast<int>((Lq + 15) / 16);
  p.bias_rows = p.nb;
  p.bias_bstride = a.bias_bstride;
  p.pairs = (p.nb + 1) / 2;
  p.n_items = static_cast<int>(B) * p.pairs;
  p.n_kt = static_cast<int>((L + kKeys - 1) / kKeys);
  p.last_valid = static_cast<int>(L - static_cast<int64_t>(p.n_kt - 1) * kKeys);
  if (static_cast<long long>(p.n_items) * p.n_kt != attn_work_steps(B, Lq, L))
    return cudaErrorInvalidValue;
  const float cap = a.cap;
  const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(kD));
  const int mode = attn_mode(cap);
  switch (mode) {
    case kNoCap:
      p.qk_scale = inv_sqrt_d * kLog2e;
      p.bias_mul = kLog2e;
      p.A = 0.f;
      p.shift = 0.f;
      break;
    default:
      // y = z / cap, logits A tanh(y) in log2 units.  The static shift is an
      // integer (exp2_poly2_fma folds it into its range reduction): the
      // smallest integer >= A, or 120 - that above A = 60 (attn_mode).
      p.qk_scale = inv_sqrt_d / cap;
      p.bias_mul = 1.0f / cap;
      p.A = cap * kLog2e;
      p.shift = attn_static_shift(p.A);
      break;
  }
  const int dv = static_cast<int>(a.Dv);
  Plan pl;
  cudaError_t e = make_plan(mode, dv, p.n_items, p.n_kt, a.num_sms, a.scratch ? a.scratch_slots : 0,
                            &pl);
  if (e != cudaSuccess) return e;
  p.sched = pl.sched;
  p.whole = pl.whole;
  p.n_whole = pl.n_whole;
  p.split_at = pl.split_at;
  for (int c = 0; c <= kAttnMaxClusters; ++c) {
    p.wb[c] = c < static_cast<int>(pl.wb.size()) ? pl.wb[c] : 0;
    p.fb[c] = c < static_cast<int>(pl.fb.size()) ? pl.fb[c] : 0;
  }
  if (pl.sched == kSchedRange) {
    char *base = static_cast<char *>(a.scratch);
    p.ws_out = reinterpret_cast<float *>(base);
    p.ws_lse = reinterpret_cast<float *>(base + a.scratch_slots * kAttnSlotOutBytes);
  }
  if (attn_two_pass(mode, dv, a.scratch != nullptr)) {
    // The row maxima (on the usual schedule, split pairs merged by maximum),
    // then the row-shift kernel on whole pairs (make_plan's plan for mode).
    Plan p1;
    e = make_plan(kRowMax, dv, p.n_items, p.n_kt, a.num_sms, 0, &p1);
    if (e != cudaSuccess) return e;
    Params q1 = p;
    q1.sched = p1.sched;
    q1.whole = p1.whole;
    q1.n_whole = p1.n_whole;
    q1.split_at = p1.split_at;
    for (int c = 0; c <= kAttnMaxClusters; ++c) {
      q1.wb[c] = c < static_cast<int>(p1.wb.size()) ? p1.wb[c] : 0;
      q1.fb[c] = c < static_cast<int>(p1.fb.size()) ? p1.fb[c] : 0;
    }
    e = launch_dv<128>(kRowMax, tq, tk, tv, to, q1, p1.clusters, false, a.stream);
    if (e != cudaSuccess) return e;
    if (p1.tail_clusters > 0) {
      q1.sched = kSchedTail;
      e = launch_dv<128>(kRowMax, tq, tk, tv, to, q1, p1.tail_clusters, true, a.stream);
      if (e != cudaSuccess) return e;
    }
    return launch_dv<128>(attn_second_pass_mode(mode), tq, tk, tv, to, p, pl.clusters, false,
                          a.stream);
  }
  e = dv == 192 ? launch_dv<192>(mode, tq, tk, tv, to, p, pl.clusters, false, a.stream)
                : launch_dv<128>(mode, tq, tk, tv, to, p, pl.clusters, false, a.stream);
  if (e != cudaSuccess) return e;
  if (pl.sched == kSchedRange) {
    if (pl.clusters < 2 || pl.whole) return cudaSuccess;
    const int merge_blocks = (pl.clusters - 1) * kMergeBlocksPerBoundary;
    if (dv == 192)
      attn_merge_kernel<192><<<merge_blocks, kMergeThreads, 0, a.stream>>>(p, pl.clusters);
    else
      attn_merge_kernel<128><<<merge_blocks, kMergeThreads, 0, a.stream>>>(p, pl.clusters);
    return cudaGetLastError();
  }
  if (pl.tail_clusters == 0) return cudaSuccess;
  p.sched = kSchedTail;
  return dv == 192 ? launch_dv<192>(mode, tq, tk, tv, to, p, pl.tail_clusters, true, a.stream)
                   : launch_dv<128>(mode, tq, tk, tv, to, p, pl.tail_clusters, true, a.stream);
}

}  // namespace ag
