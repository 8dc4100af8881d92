// attn_bwd_sm100.cu -- backward of the pair-bias multi-query attention on the
// tensor cores (sm_100a), value width 128.
//
// The gradients of out for an upstream gradient dout, through Eq. L_ij of the
// page "Making Full-Context AlphaGenome Fit on an RTX 3090" (section "Why
// stock FlashAttention was not a drop-in replacement") and the softmax; the
// page names a backward pass as later work for fine-tuning (section "Where I
// would take it next").  With x_ij = q_i . k_j / sqrt(D) + bias, t = tanh(x /
// cap), p_ij = exp(cap t - lse_i), dp_ij = dout_i . v_j:
//   delta_i = sum_j p_ij dp_ij,   ds_ij = p_ij (dp_ij - delta_i) (1 - t^2)
//   dq_i = sum_j ds_ij k_j / sqrt(D),   dk_j = sum_{h,i} ds_ij q_i / sqrt(D)
//   dv_j = sum_{h,i} p_ij dout_i,       dbias cell = sum of ds over the cell.
//
// Four launches on the caller's stream:
//   bwd_split_kernel   dout (fp32) -> two bf16 planes hi = bf16(dout),
//                      lo = bf16(dout - hi), row-interleaved in the dq buffer
//                      (dq has the same size; it is written last).
//   bwd_query_kernel<1>  per 128-row query tile: S = Q K^T and
//                      dP = dO V^T (dO as hi + lo) on tcgen05, delta.
//   bwd_key_kernel     per 128-key tile, its query range split between the
//                      two CTAs of a cluster: S^T = K Q^T, dP^T = V dO^T,
//                      P^T and dS^T (each as bf16 hi + lo) in tensor memory,
//                      dV += P^T dO and dK += dS^T Q on tcgen05, the compact
//                      dbias cells from dS on the CUDA cores; the odd CTA's
//                      dK, dV partial goes through the dk/dv rows to the even
//                      CTA, which adds it (fixed order: deterministic).
//   bwd_query_kernel<2>  per query tile again: S, dP, dS (hi + lo) and
//                      dQ += dS K on tcgen05; writes dq over the dout planes
//                      of its own rows (which it has already staged).
// Every product that is not of two bf16 inputs (dO, P, dS) is split into a
// bf16 pair whose sum carries 16 significant bits, so the tensor cores add
// no error beyond fp32 accumulation (a single bf16 rounding of these
// operands would move the gradients by about 2e-3 of their size).  No atomics,
// no scratch: every output value is written by one thread in a fixed order.
#include <algorithm>
#include <mutex>

#include "ag_internal.h"
#include "sm100.cuh"

namespace ag {
namespace bwdtc {

constexpr int kH = 8;
constexpr int kD = 128;
constexpr int kQRows = 128;                 // query tile: 16 positions x 8 heads
constexpr int kQTileBytes = kQRows * kD * 2;  // 32 KB, two 64-column halves
constexpr int kQHalf = kQTileBytes / 2;
constexpr int kQKeys = 64;                  // query kernel: keys per step
constexpr int kQKTileBytes = kQKeys * kD * 2;  // 16 KB (K or V)
constexpr int kQKHalf = kQKTileBytes / 2;      // 8 KB
constexpr int kQStages = 3;                 // K/V ring of the query kernel
constexpr int kKKeys = 128;                 // key kernel: keys per CTA
constexpr int kKTileBytes = kKKeys * kD * 2;  // 32 KB (K or V)
constexpr int kKHalf = kKTileBytes / 2;
constexpr int kSubRows = 64;                // key kernel: query rows per step
constexpr int kSubBytes = kSubRows * kD * 2;  // 16 KB (Q, dO hi or dO lo)
constexpr int kSubHalf = kSubBytes / 2;       // 8 KB
constexpr int kKStages = 3;                 // Q/dO ring of the key kernel
constexpr int kSoftWarps = 16;
constexpr int kThreads = 608;               // 16 softmax warps, producer, 2 MMA issuers
constexpr int kWarpLoad = 16, kWarpMma = 17, kWarpMma2 = 18;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

enum Site : unsigned {
  kSiteQ = 40, kSiteKV = 41, kSiteSP = 42, kSiteDS = 43, kSiteEnd = 44, kSiteSoft = 45,
  kSitePeer = 46, kSiteAcc = 47, kSiteXchg = 48, kSiteRing = 49
};

struct Args {
  const float *bias;
  long long bias_bstride;  // floats between items' bias (0: shared)
  const float *lse;
  float *delta;
  float *dq;               // also the dout planes until bwd_query_kernel<2>
  float *dk, *dv, *dbias;
  int B, L, P, nb;         // nb = ceil(L / 16)
  float qk_scale;          // 1 / sqrt(D), or with the cap: 1 / (sqrt(D) cap)
  float bias_mul;          // 1, or 1 / cap
  float inv_sqrt_d;        // 1 / sqrt(D)
  float A;                 // cap log2(e) (0 without a cap)
  int capped;
  unsigned *err;
};

// Descriptors: every tile here is rows of 128 bytes (64 bf16) in 1 KB
// groups of 8 rows with the 128-byte swizzle.
constexpr uint32_t kHi = desc_sw128_hi(1024);
__host__ __device__ constexpr uint32_t idesc(uint32_t N, uint32_t b_mn) {
  return idesc_bf16_f32(128, N, b_mn);
}

// D[128 x N] (+)= A[128 x 128] B: A K-major (two 64-column halves a_half
// bytes apart), B K-major ([N rows x 128], halves b_half apart).
__device__ __forceinline__ void mma_kk(uint32_t d, uint32_t a, uint32_t a_half, uint32_t b,
                                       uint32_t b_half, uint32_t N, bool acc) {
  const uint32_t a_lo = desc_sw128_lo(a, 16), b_lo = desc_sw128_lo(b, 16);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t ao = ((kk >> 2) * a_half + (kk & 3) * 32) >> 4;
    const uint32_t bo = ((kk >> 2) * b_half + (kk & 3) * 32) >> 4;
    umma1_ss_w(d, a_lo + ao, kHi, b_lo + bo, kHi, idesc(N, 0), (acc || kk > 0) ? 1u : 0u);
  }
}

// D[128 x 128] (+)= A[128 x 16 nk] B[16 nk x 128]: A in tensor memory (bf16
// pairs; the 16 K elements of step kk at columns a_col(kk) .. + 8), B
// MN-major ([16 nk rows x 128], two 64-column atoms b_atom bytes apart).
template <typename ACol>
__device__ __forceinline__ void mma_tm(uint32_t d, ACol a_col, int nk, uint32_t b,
                                       uint32_t b_atom, bool acc) {
  const uint32_t b_lo = desc_sw128_lo(b, b_atom);
  for (int kk = 0; kk < nk; ++kk)
    umma1_ts_w(d, a_col(kk), b_lo + ((kk * 16 * 128) >> 4), kHi, idesc(128, 1),
                (acc || kk > 0) ? 1u : 0u);
}

__device__ __forceinline__ void drain(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(a, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
}

__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
  __syncwarp();
  if (lane_id() == 0) mbar_arrive(bar);
}

// A value split into two bf16 whose sum carries 16 significant bits.
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = pack_bf16x2(a - hf.x, b - hf.y);
}

// t = tanh(x / cap) and p = exp(L - lse) (L = cap t, or x without a cap) from
// the raw product s and the cell's bias; log2 units inside.
struct Logit {
  float p, dt;  // probability, dL/dx = 1 - t^2 (1 without a cap)
};
__device__ __forceinline__ Logit logit(float s, float bias, float lse2, const Args &a) {
  const float y = fmaf(s, a.qk_scale, bias * a.bias_mul);
  if (a.capped) {
    const float t = tanh_approx(y);
    return {ex2_approx(fmaf(a.A, t, -lse2)), fmaf(-t, t, 1.f)};
  }
  return {ex2_approx(fmaf(y, kLog2e, -lse2)), 1.f};
}

// The same split by truncation, on the integer and FMA pipes only: hi keeps
// the upper 16 bits of each value, lo the upper 16 bits of the exact
// remainder, so hi + lo is within 2^-14 of the value (relative).  Element a
// goes to the low half of each packed pair.
__device__ __forceinline__ void split2t(float a, float b, uint32_t &hi, uint32_t &lo) {
  const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  const float ra = a - __uint_as_float(ua & 0xffff0000u);
  const float rb = b - __uint_as_float(ub & 0xffff0000u);
  hi = __byte_perm(ua, ub, 0x7632);
  lo = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
}

// 2^x for two values on the FMA pipe (exp2_poly2_fma with a = 1, m = 0),
// x clamped below at -126 so that the result stays a normal number (the
// clamp moves only values under 2^-126, which no gradient here can see).
__device__ __forceinline__ float2 exp2_fma_pair(float x0, float x1) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  return exp2_poly2_fma(make_float2(fmaxf(x0, -126.f), fmaxf(x1, -126.f)),
                        make_float2(1.f, 1.f), make_float2(kShift, kShift));
}

// Probabilities of two logits (raw products s0, s1; lse in log2 units l0,
// l1), with the exponential on the FMA pipe (kEmu) or the special-function
// unit; dt = 1 - t^2 (1 without a cap).
template <bool kCapped, bool kEmu>
__device__ __forceinline__ float2 prob_pair(float s0, float s1, float bias_term, float l0,
                                            float l1, const Args &a, float2 &dt) {
  const float y0 = fmaf(s0, a.qk_scale, bias_term), y1 = fmaf(s1, a.qk_scale, bias_term);
  float x0, x1;
  if (kCapped) {
    const float t0 = tanh_approx(y0), t1 = tanh_approx(y1);
    dt = make_float2(fmaf(-t0, t0, 1.f), fmaf(-t1, t1, 1.f));
    x0 = fmaf(a.A, t0, -l0);
    x1 = fmaf(a.A, t1, -l1);
  } else {
    dt = make_float2(1.f, 1.f);
    x0 = fmaf(y0, kLog2e, -l0);
    x1 = fmaf(y1, kLog2e, -l1);
  }
  if (kEmu) return exp2_fma_pair(x0, x1);
  return make_float2(ex2_approx(x0), ex2_approx(x1));
}

// Exponential pairs (out of the 8 of a 16-logit step) on the FMA pipe, per
// kernel: the delta pass is bound by the special-function unit, the others
// by instruction issue.
#ifndef AG_BWD_EMU_DELTA
#define AG_BWD_EMU_DELTA 3
#endif
#ifndef AG_BWD_EMU_DQ
#define AG_BWD_EMU_DQ 0
#endif
#ifndef AG_BWD_EMU_KEY
#define AG_BWD_EMU_KEY 0
#endif

template <bool kCapped, int kEmu>
__device__ __forceinline__ float2 prob_sel(int pair, float s0, float s1, float bias_term,
                                           float l0, float l1, const Args &a, float2 &dt) {
  if (pair < kEmu) return prob_pair<kCapped, true>(s0, s1, bias_term, l0, l1, a, dt);
  return prob_pair<kCapped, false>(s0, s1, bias_term, l0, l1, a, dt);
}

// Query kernel, pass 1: sum over this thread's 16 keys of p dp for its row
// (keys from nvalid on are past L when kMask).
template <bool kCapped, bool kMask>
__device__ __forceinline__ float delta_part(const uint32_t (&sv)[16], const uint32_t (&pv)[16],
                                            float bias_term, float lse2, int nvalid,
                                            const Args &a) {
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    float2 dt;
    float2 p = prob_sel<kCapped, AG_BWD_EMU_DELTA>(e >> 1, __uint_as_float(sv[e]),
                                                   __uint_as_float(sv[e + 1]), bias_term, lse2,
                                                   lse2, a, dt);
    if (kMask) {
      p.x = e < nvalid ? p.x : 0.f;
      p.y = e + 1 < nvalid ? p.y : 0.f;
    }
    acc0 = fmaf(p.x, __uint_as_float(pv[e]), acc0);
    acc1 = fmaf(p.y, __uint_as_float(pv[e + 1]), acc1);
  }
  return acc0 + acc1;
}

// Query kernel, pass 2: ds = p (dp - delta) dt for this thread's row and 16
// keys, split into bf16 hi and lo pairs.
template <bool kCapped, bool kMask>
__device__ __forceinline__ void ds_row(const uint32_t (&sv)[16], const uint32_t (&pv)[16],
                                       float bias_term, float lse2, float del, int nvalid,
                                       const Args &a, uint32_t (&hi)[8], uint32_t (&lo)[8]) {
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    float2 dt;
    const float2 p = prob_sel<kCapped, AG_BWD_EMU_DQ>(e >> 1, __uint_as_float(sv[e]),
                                                      __uint_as_float(sv[e + 1]), bias_term,
                                                      lse2, lse2, a, dt);
    float d0 = p.x * (__uint_as_float(pv[e]) - del) * dt.x;
    float d1 = p.y * (__uint_as_float(pv[e + 1]) - del) * dt.y;
    if (kMask) {
      d0 = e < nvalid ? d0 : 0.f;
      d1 = e + 1 < nvalid ? d1 : 0.f;
    }
    split2t(d0, d1, hi[e >> 1], lo[e >> 1]);
  }
}

// Key kernel: P and dS of this thread's key for 16 rows (lse2 of row e at
// lr[e], delta at dr[e]: shared memory, the same for every lane), split into
// bf16 hi and lo pairs; returns the sum of ds.
template <bool kCapped>
__device__ __forceinline__ float key_rows(const uint32_t (&sv)[16], const uint32_t (&pv)[16],
                                          const float *lr, const float *dr, float bias_term,
                                          const Args &a, uint32_t (&ph)[8], uint32_t (&pl)[8],
                                          uint32_t (&sh)[8], uint32_t (&sl)[8]) {
  const float4 *l4p = reinterpret_cast<const float4 *>(lr);
  const float4 *d4p = reinterpret_cast<const float4 *>(dr);
  float cell = 0.f;
#pragma unroll
  for (int e4 = 0; e4 < 4; ++e4) {
    const float4 l4 = l4p[e4], d4 = d4p[e4];
    const float la[4] = {l4.x, l4.y, l4.z, l4.w}, da[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int e = 4 * e4 + 2 * h2;
      float2 dt;
      const float2 p = prob_sel<kCapped, AG_BWD_EMU_KEY>(
          e >> 1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), bias_term, la[2 * h2],
          la[2 * h2 + 1], a, dt);
      const float d0 = p.x * (__uint_as_float(pv[e]) - da[2 * h2]) * dt.x;
      const float d1 = p.y * (__uint_as_float(pv[e + 1]) - da[2 * h2 + 1]) * dt.y;
      cell += d0 + d1;
      split2t(p.x, p.y, ph[e >> 1], pl[e >> 1]);
      split2t(d0, d1, sh[e >> 1], sl[e >> 1]);
    }
  }
  return cell;
}

// ---------------------------------------------------------------------------
// dout -> hi, lo planes.  Row r of [B H L] rows (128 values) becomes 256
// bf16 at bytes [512 r, 512 r + 512) of dq: hi first, then lo.
__global__ void __launch_bounds__(256) bwd_split_kernel(const float *__restrict__ dout,
                                                        float *dq, long long n4) {
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n4; i += 256ll * gridDim.x) {
    const float4 x = reinterpret_cast<const float4 *>(dout)[i];
    const long long row = i >> 5, c4 = i & 31;  // 32 float4 per row
    uint32_t h0, l0, h1, l1;
    split2(x.x, x.y, h0, l0);
    split2(x.z, x.w, h1, l1);
    uint2 *base = reinterpret_cast<uint2 *>(reinterpret_cast<char *>(dq) + row * 512);
    base[c4] = make_uint2(h0, h1);        // hi: bytes [0, 256) of the row
    base[32 + c4] = make_uint2(l0, l1);   // lo: bytes [256, 512)
  }
}

// ---------------------------------------------------------------------------
// Query kernel.  Tile t = (item b, 16-position block I): rows h * 16 + il of
// all 8 heads.  PASS 1: delta.  PASS 2: dq (needs delta).
//
// The CTA's steps (64 keys of one of its tiles each) are numbered s = 0, 1,
// ... across its tiles.  K and V come in separate 3-slot rings (slot s % 3):
// V is free as soon as dP has been formed, K only after dQ.  Tensor memory
// holds step buffers b = s % nb (nb = 4 in pass 1, 2 in pass 2), S at
// columns [128 b, 128 b + 64) and dP at [128 b + 64, 128 b + 128); pass 2
// writes dS (bf16 hi, lo) over the S columns it has read, and dQ accumulates
// at [256, 384).
//
// The softmax warps form two groups of two warpgroups: group q takes the
// steps s % 2 == q (so the buffers b % 2 == q), and one group's waits for its
// logits and for tensor-memory traffic are covered by the other group's
// arithmetic.
// Warpgroup hg of a group takes keys [32 hg, 32 hg + 32) of the step (two
// 16-key blocks, one bias cell each); thread r of it owns row r.
//
// The tensor core runs ahead of the softmax warps: pass 1 issues S and dP of
// a step as soon as its buffer has been loaded by the softmax group (up to
// two of each group's steps ahead); pass 2
// issues, per step s, dQ of step s, then dP of step s + 2 (its columns were
// read before dS of step s was written), then S of step s + 2 once dQ of
// step s has read the columns -- a wait covered by the dP products queued.
constexpr int kQBufsMax = 4;
// Step buffers: four in pass 1 (two per softmax group, so the tensor core
// can run two of a group's steps ahead), two in pass 2 (dQ takes the rest).
template <int PASS>
constexpr int q_bufs() { return PASS == 1 ? 4 : 2; }
constexpr int kGroupWarps = kSoftWarps / 2;
struct QBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kQStages], k_empty[kQStages], v_full[kQStages], v_empty[kQStages];
  uint64_t sp_full[kQBufsMax];   // S and dP of the buffer's step are in tensor memory
  uint64_t buf_free[kQBufsMax];  // the buffer's S columns may be overwritten
  uint64_t ds_full[kQBufsMax];   // pass 2: dS of the buffer's step is written
  uint64_t dq_full, dq_free, xd;
  uint64_t drain[2];  // per issuing thread: its last products have completed
  uint32_t tmem;
  int abort;
};

template <int PASS>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_query_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Args a) {
  constexpr int kQBufs = q_bufs<PASS>();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *q_s = smem_raw + pad;                 // Q tile (32 KB)
  uint8_t *dh_s = q_s + kQTileBytes;             // dO hi tile
  uint8_t *dl_s = dh_s + kQTileBytes;            // dO lo tile
  uint8_t *k_ring = dl_s + kQTileBytes;          // K ring, 16 KB a slot
  uint8_t *v_ring = k_ring + kQStages * kQKTileBytes;  // V ring
  QBars *bars = reinterpret_cast<QBars *>(v_ring + kQStages * kQKTileBytes);
  // Row-sum exchange between the warpgroups, double-buffered by tile parity:
  // a thread writes one tile's half only after every thread has passed the
  // previous tile's exchange, i.e. has read the half before.
  float *dpart = reinterpret_cast<float *>(bars + 1);  // [2][4][128]
  const int warp = threadIdx.x >> 5;
  const int n_kt = (a.L + kQKeys - 1) / kQKeys;
  const int tiles = a.B * a.nb;
  // This CTA's tiles are blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_tiles =
      static_cast<int>(blockIdx.x) < tiles
          ? (tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                static_cast<int>(gridDim.x)
          : 0;
  const uint32_t total = static_cast<uint32_t>(my_tiles) * static_cast<uint32_t>(n_kt);

  if (threadIdx.x == 0) {
    // Both issuing threads read the Q/dO tile and write a step's S and dP.
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 2);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int b = 0; b < kQBufs; ++b) {
      mbar_init(&bars->sp_full[b], 2);
      // Pass 1: the buffer's group frees it once it has loaded it; pass 2:
      // issuer 1, once dQ has read the dS written there.
      mbar_init(&bars->buf_free[b], PASS == 1 ? kGroupWarps : 1);
      mbar_init(&bars->ds_full[b], kGroupWarps);
    }
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, kSoftWarps);
    mbar_init(&bars->xd, kSoftWarps);
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc1(&bars->tmem, kTmemCols);
    tmem_relinquish1();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  volatile int *abort = &bars->abort;

  if (warp == kWarpLoad) {
    if (lane_id() == 0) {
      const uint64_t pol_q = l2_policy_evict_first(), pol_k = l2_policy_evict_last();
      uint32_t qc = 0, kl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int b = t / a.nb, I = t - b * a.nb;
        ok = mbar_wait(&bars->q_empty, (qc & 1u) ^ 1u, abort, a.err, kSiteQ);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->q_full, 3 * kQTileBytes);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_4d(q_s + hf * kQHalf, &tm_q, &bars->q_full, 64 * hf, 16 * I, 0, b, pol_q);
          // dO planes: coordinates (column, hi/lo, position, head, item).
          tma_load_5d(dh_s + hf * kQHalf, &tm_do, &bars->q_full, 64 * hf, 0, 16 * I, 0, b,
                      pol_q);
          tma_load_5d(dl_s + hf * kQHalf, &tm_do, &bars->q_full, 64 * hf, 1, 16 * I, 0, b,
                      pol_q);
        }
        ++qc;
        for (int j = 0; j < n_kt && ok; ++j, ++kl) {
          const uint32_t s = kl % kQStages, ph = ((kl / kQStages) & 1u) ^ 1u;
          // V first: its slot is freed earlier than K's.
          ok = mbar_wait(&bars->v_empty[s], ph, abort, a.err, kSiteKV);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->v_full[s], kQKTileBytes);
          uint8_t *vs = v_ring + s * kQKTileBytes;
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(vs + hf * kQKHalf, &tm_v, &bars->v_full[s], 64 * hf, kQKeys * j, b,
                        pol_k);
          ok = mbar_wait(&bars->k_empty[s], ph, abort, a.err, kSiteKV);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->k_full[s], kQKTileBytes);
          uint8_t *ks = k_ring + s * kQKTileBytes;
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(ks + hf * kQKHalf, &tm_k, &bars->k_full[s], 64 * hf, kQKeys * j, b,
                        pol_k);
        }
      }
      if (qc > 0) drain(&bars->q_full, (qc - 1) & 1u);
      for (uint32_t i = kl > kQStages ? kl - kQStages : 0; i < kl; ++i) {
        drain(&bars->v_full[i % kQStages], (i / kQStages) & 1u);
        drain(&bars->k_full[i % kQStages], (i / kQStages) & 1u);
      }
    }
  } else if (warp == kWarpMma || warp == kWarpMma2) {
    // Two issuing threads: issuer 0 forms dP, issuer 1 forms S and (pass 2)
    // dQ from the dS written over S, so the dQ accumulator is fed by one
    // thread in a fixed order.
    const int who = warp - kWarpMma;
    const uint32_t q_a = smem_u32(q_s), dh_a = smem_u32(dh_s), dl_a = smem_u32(dl_s);
    const uint32_t k_a = smem_u32(k_ring), v_a = smem_u32(v_ring);
    const uint32_t tQ = tmem + 256;
    const uint32_t nk = static_cast<uint32_t>(n_kt);
    // Issuer 0: dP = dO V^T (dO as hi + lo) of step s into buffer s % 2,
    // once the softmax warps have read the dP of the buffer's previous
    // step.  Issuer 1: S = Q K^T, once the buffer's previous S (pass 1) or
    // the dS over it (pass 2, read by dQ) is no longer needed.
    auto issue_sp = [&](uint32_t s) -> bool {
      const uint32_t b = s % kQBufs, u = s / kQBufs, st = s % kQStages, j = s % nk;
      const uint32_t rph = (s / kQStages) & 1u;
      if (j == 0 && !mbar_wait_warp(&bars->q_full, (s / nk) & 1u, abort, a.err, kSiteQ))
        return false;
      if (u > 0) {
        uint64_t *prev = (PASS == 1 || who == 1) ? &bars->buf_free[b] : &bars->ds_full[b];
        if (!mbar_wait_warp(prev, (u - 1) & 1u, abort, a.err, kSiteSP)) return false;
      }
      if (who == 0) {
        if (!mbar_wait_warp(&bars->v_full[st], rph, abort, a.err, kSiteKV)) return false;
        tc_fence_after();
        const uint32_t vs = v_a + st * kQKTileBytes, tP = tmem + 128 * b + 64;
        mma_kk(tP, dh_a, kQHalf, vs, kQKHalf, kQKeys, false);  // dP = dO_hi V^T
        mma_kk(tP, dl_a, kQHalf, vs, kQKHalf, kQKeys, true);   //    + dO_lo V^T
        umma1_commit_w(&bars->v_empty[st]);
      } else {
        if (!mbar_wait_warp(&bars->k_full[st], rph, abort, a.err, kSiteKV)) return false;
        tc_fence_after();
        const uint32_t ks = k_a + st * kQKTileBytes, tS = tmem + 128 * b;
        mma_kk(tS, q_a, kQHalf, ks, kQKHalf, kQKeys, false);   // S = Q K^T
        if (PASS == 1) umma1_commit_w(&bars->k_empty[st]);
      }
      umma1_commit_w(&bars->sp_full[b]);
      if (j + 1 == nk) umma1_commit_w(&bars->q_empty);
      return true;
    };
    // Issuer 1, pass 2: dQ += dS K of step s, dS (hi, lo) over the S
    // columns of its buffer.
    auto issue_dq = [&](uint32_t s) -> bool {
      const uint32_t b = s % kQBufs, u = s / kQBufs, st = s % kQStages, j = s % nk;
      if (!mbar_wait_warp(&bars->ds_full[b], u & 1u, abort, a.err, kSiteDS)) return false;
      // The tile's first dQ overwrites the accumulator: every softmax warp
      // must have read the previous tile's.
      const uint32_t tile = s / nk;
      if (j == 0 && tile > 0 &&
          !mbar_wait_warp(&bars->dq_free, (tile - 1) & 1u, abort, a.err, kSiteEnd))
        return false;
      tc_fence_after();
      const uint32_t kp = k_a + st * kQKTileBytes, tS = tmem + 128 * b;
      mma_tm(tQ, [=](int kk) { return tS + 16 * kk; }, 4, kp, kQKHalf, j > 0);
      mma_tm(tQ, [=](int kk) { return tS + 16 * kk + 8; }, 4, kp, kQKHalf, true);
      umma1_commit_w(&bars->buf_free[b]);
      umma1_commit_w(&bars->k_empty[st]);
      if (j + 1 == nk) umma1_commit_w(&bars->dq_full);
      return true;
    };
    if (PASS == 1 || who == 0) {
      for (uint32_t s = 0; s < total; ++s)
        if (!issue_sp(s)) break;
    } else {
      bool ok = true;
      for (uint32_t s = 0; s < 2 && s < total && ok; ++s) ok = issue_sp(s);
      for (uint32_t s = 0; s < total && ok; ++s) {
        ok = issue_dq(s);
        if (ok && s + 2 < total) ok = issue_sp(s + 2);
      }
    }
    umma1_commit_w(&bars->drain[who]);
    drain(&bars->drain[who], 0);
  } else if (warp < kSoftWarps) {
    const int g = threadIdx.x >> 7, r = threadIdx.x & 127;
    const int q = g >> 1, hg = g & 1;  // group (buffer), key half
    const int h = r >> 4, il = r & 15;
    const uint32_t lane_base = static_cast<uint32_t>(r >> 5) << 21;
    uint32_t qc = 0, xc = 0;
    uint32_t s0 = 0;  // the CTA's step number of the tile's first step
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, s0 += static_cast<uint32_t>(n_kt)) {
      const int b = t / a.nb, I = t - b * a.nb;
      const int pos = 16 * I + il;
      const bool row_ok = pos < a.L;
      const size_t row = (static_cast<size_t>(b) * kH + h) * a.L + (row_ok ? pos : 0);
      // A row past L gets lse = +inf: its probabilities are 0 (its dO row,
      // zero-filled, makes its ds 0 too).
      const float lse2 = row_ok ? a.lse[row] * kLog2e : __int_as_float(0x7f800000);
      const float del = (PASS == 2 && row_ok) ? a.delta[row] : 0.f;
      const float *brow = a.bias + static_cast<long long>(b) * a.bias_bstride +
                          (static_cast<size_t>(h) * a.P + I) * a.P;
      float acc = 0.f;
      // This group's steps of the tile: j with (s0 + j) % 2 == q.
      for (int j = static_cast<int>((static_cast<uint32_t>(q) - s0) & 1u); j < n_kt; j += 2) {
        const uint32_t s = s0 + static_cast<uint32_t>(j), u = s / kQBufs;
        const int key0 = kQKeys * j + 32 * hg;  // this thread's 32 keys: two bias cells
        float bt[2];
#pragma unroll
        for (int k = 0; k < 2; ++k)
          bt[k] = (key0 + 16 * k < a.L ? __ldg(brow + key0 / 16 + k) : 0.f) * a.bias_mul;
        const uint32_t bf = s % kQBufs;  // a buffer of this group (bf % 2 == q)
        ok = mbar_wait(&bars->sp_full[bf], u & 1u, abort, a.err, kSiteSoft);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        const uint32_t tS = tmem + 128 * bf + 32 * hg + lane_base;
        if (PASS == 1) {
          uint32_t sv[2][16], pv[2][16];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            tmem_ld16(tS + 16 * k, sv[k]);
            tmem_ld16(tS + 64 + 16 * k, pv[k]);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            tmem_wait_ld16(sv[k]);
            tmem_wait_ld16(pv[k]);
          }
          tc_fence_before();
          warp_arrive(&bars->buf_free[bf]);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int nvalid = a.L - (key0 + 16 * k);  // keys of the 16 before L
            if (nvalid >= 16)
              acc += a.capped ? delta_part<true, false>(sv[k], pv[k], bt[k], lse2, nvalid, a)
                              : delta_part<false, false>(sv[k], pv[k], bt[k], lse2, nvalid, a);
            else
              acc += a.capped ? delta_part<true, true>(sv[k], pv[k], bt[k], lse2, nvalid, a)
                              : delta_part<false, true>(sv[k], pv[k], bt[k], lse2, nvalid, a);
          }
        } else {
          // Both blocks' loads in flight at once; each block's dS is written
          // over its own S columns as soon as it is formed.
          uint32_t sv[2][16], pv[2][16];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            tmem_ld16(tS + 16 * k, sv[k]);
            tmem_ld16(tS + 64 + 16 * k, pv[k]);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            tmem_wait_ld16(sv[k]);
            tmem_wait_ld16(pv[k]);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int nvalid = a.L - (key0 + 16 * k);
            uint32_t hi[8], lo[8];
            if (nvalid >= 16) {
              if (a.capped)
                ds_row<true, false>(sv[k], pv[k], bt[k], lse2, del, nvalid, a, hi, lo);
              else
                ds_row<false, false>(sv[k], pv[k], bt[k], lse2, del, nvalid, a, hi, lo);
            } else {
              if (a.capped)
                ds_row<true, true>(sv[k], pv[k], bt[k], lse2, del, nvalid, a, hi, lo);
              else
                ds_row<false, true>(sv[k], pv[k], bt[k], lse2, del, nvalid, a, hi, lo);
            }
            // In place: this warp's lanes of the S columns it has just read.
            tmem_st8(tS + 16 * k, hi);
            tmem_st8(tS + 16 * k + 8, lo);
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(&bars->ds_full[bf]);
        }
      }
      if (!ok) break;
      if (PASS == 1) {
        float *dp = dpart + (xc & 1u) * 512;
        dp[g * 128 + r] = acc;
        warp_arrive(&bars->xd);
        ok = mbar_wait(&bars->xd, xc & 1u, abort, a.err, kSiteXchg);
        ++xc;
        if (!__all_sync(0xffffffffu, ok)) break;
        if (g == 0 && row_ok) a.delta[row] = dp[r] + dp[128 + r] + dp[256 + r] + dp[384 + r];
      } else {
        // dq row: warpgroup g writes columns [32 g, 32 g + 32).  dq_full also
        // tells that every dS of the tile has been read.
        ok = mbar_wait(&bars->dq_full, qc & 1u, abort, a.err, kSiteEnd);
        ++qc;
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        uint32_t o[32];
        tmem_ld32((tmem + 256) + 32 * g + lane_base, o);
        tmem_wait_ld(o);
        if (row_ok) {
          float4 *dst = reinterpret_cast<float4 *>(a.dq + row * kD + 32 * g);
          const float sc = a.inv_sqrt_d;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]) * sc, __uint_as_float(o[4 * e + 1]) * sc,
                                 __uint_as_float(o[4 * e + 2]) * sc,
                                 __uint_as_float(o[4 * e + 3]) * sc);
        }
        tc_fence_before();
        warp_arrive(&bars->dq_free);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc1(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Key kernel.  Cluster c (2 CTAs) owns key tile c (128 keys) of every item;
// CTA `rank` takes query blocks [nb rank / 2, nb (rank + 1) / 2) of each
// item, each block as two 64-row steps (heads 0-3, then 4-7).  Per item:
// K and V resident, a 3-stage ring of (Q, dO hi, dO lo) steps.
//
// Tensor memory (lane = key): two step buffers b = s % 2 (s counts the
// CTA's steps across items), S^T at [128 b, 128 b + 64) and dP^T at
// [128 b + 64, 128 b + 128); the softmax warps write P^T (bf16 hi, lo) over
// the S^T columns and dS^T (hi, lo) over the dP^T columns they have read.
// dV [256, 384), dK [384, 512).  Warpgroup g takes the step's rows
// [16 g, 16 g + 16): head 4 (step & 1) + g, positions 0..15 of the block;
// thread r owns key r.  The tensor core issues, per step s: dK += dS^T Q
// (then tells that the dS^T columns are read), dV += P^T dO (then the P^T
// columns), and behind them dP^T and S^T of step s + 2 into the same
// buffer, each after the wait for the columns it overwrites, so the waits
// are covered by the products already queued.
struct KBars {
  uint64_t kv_full, kv_free;
  uint64_t ring_full[kKStages], ring_empty[kKStages];
  uint64_t sp_full[2];   // S^T and dP^T of the buffer's step are in tensor memory
  uint64_t pds_full[2];  // P^T and dS^T of the buffer's step are written
  uint64_t ds_read[2];   // dK has read the buffer's dS^T columns
  uint64_t p_read[2];    // dV has read the buffer's P^T columns
  uint64_t acc_full, acc_free;
  uint64_t peer;      // even CTA: the odd CTA's partial of the item is in dk/dv
  uint64_t peer_ack;  // odd CTA: the even CTA has read it
  uint64_t epi;       // every softmax warp of this CTA is through the item's dK, dV
  uint64_t drain[2];  // per issuing thread: its last products have completed
  uint32_t tmem;
  int abort;
};

constexpr size_t kKBarsBytes = (sizeof(KBars) + 15) & ~static_cast<size_t>(15);

__device__ __forceinline__ int block_begin(int nb, uint32_t rank) {
  return static_cast<int>((static_cast<long long>(nb) * rank) / 2);
}

__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort, unsigned *err,
                                                  unsigned site) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      if (err) atomicCAS(err, 0u, (site << 8) | kErrTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void arrive_cluster_release(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   cluster_bar)
               : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    bwd_key_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *k_s = smem_raw + pad;               // K tile (32 KB)
  uint8_t *v_s = k_s + kKTileBytes;            // V tile (32 KB)
  uint8_t *ring = v_s + kKTileBytes;           // stages of Q, dO hi, dO lo (48 KB)
  KBars *bars = reinterpret_cast<KBars *>(ring + kKStages * 3 * kSubBytes);
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();
  const int kt = static_cast<int>(blockIdx.x >> 1);
  const int I0 = block_begin(a.nb, rank), I1 = block_begin(a.nb, rank + 1);
  const int n_sub = 2 * (I1 - I0);  // steps per item

  if (threadIdx.x == 0) {
    // Arrival counts: one commit per issuing thread where both read or
    // write (ring stage, K/V, the step's S^T/dP^T, the accumulators).
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_free, 2);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->ring_full[s], 1);
      mbar_init(&bars->ring_empty[s], 2);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bars->sp_full[q], 2);
      mbar_init(&bars->pds_full[q], kSoftWarps / 2);
      mbar_init(&bars->ds_read[q], 1);
      mbar_init(&bars->p_read[q], 1);
    }
    mbar_init(&bars->acc_full, 2);
    mbar_init(&bars->acc_free, kSoftWarps);
    mbar_init(&bars->peer, 1);
    mbar_init(&bars->peer_ack, 1);
    mbar_init(&bars->epi, kSoftWarps);
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc1(&bars->tmem, kTmemCols);
    tmem_relinquish1();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  volatile int *abort = &bars->abort;

  if (warp == kWarpLoad) {
    if (lane_id() == 0) {
      const uint64_t pol_kv = l2_policy_evict_first(), pol_q = l2_policy_evict_last();
      uint32_t rc = 0;
      bool ok = true;
      for (int b = 0; b < a.B && ok; ++b) {
        ok = mbar_wait(&bars->kv_free, (static_cast<uint32_t>(b) & 1u) ^ 1u, abort, a.err,
                       kSiteKV);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->kv_full, 2 * kKTileBytes);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_3d(k_s + hf * kKHalf, &tm_k, &bars->kv_full, 64 * hf, kKKeys * kt, b, pol_kv);
          tma_load_3d(v_s + hf * kKHalf, &tm_v, &bars->kv_full, 64 * hf, kKKeys * kt, b, pol_kv);
        }
        for (int n = 0; n < n_sub && ok; ++n, ++rc) {
          const uint32_t st = rc % kKStages;
          ok = mbar_wait(&bars->ring_empty[st], ((rc / kKStages) & 1u) ^ 1u, abort, a.err,
                         kSiteRing);
          if (!ok) break;
          const int I = I0 + (n >> 1), h0 = 4 * (n & 1);
          uint8_t *qs = ring + st * 3 * kSubBytes;
          mbar_arrive_expect_tx(&bars->ring_full[st], 3 * kSubBytes);
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(qs + hf * kSubHalf, &tm_q, &bars->ring_full[st], 64 * hf, 16 * I, h0,
                        b, pol_q);
            tma_load_5d(qs + kSubBytes + hf * kSubHalf, &tm_do, &bars->ring_full[st], 64 * hf,
                        0, 16 * I, h0, b, pol_q);
            tma_load_5d(qs + 2 * kSubBytes + hf * kSubHalf, &tm_do, &bars->ring_full[st],
                        64 * hf, 1, 16 * I, h0, b, pol_q);
          }
        }
      }
      if (a.B > 0) drain(&bars->kv_full, static_cast<uint32_t>(a.B - 1) & 1u);
      for (uint32_t i = rc > kKStages ? rc - kKStages : 0; i < rc; ++i)
        drain(&bars->ring_full[i % kKStages], (i / kKStages) & 1u);
    }
  } else if (warp == kWarpMma || warp == kWarpMma2) {
    // Two issuing threads, one per chain of tensor-memory columns: issuer 0
    // forms dP^T and, from the dS^T written over it, dK; issuer 1 forms S^T
    // and, from the P^T written over it, dV.  Each accumulator is fed by one
    // thread in a fixed order.
    const int who = warp - kWarpMma;
    const uint32_t k_a = smem_u32(k_s), v_a = smem_u32(v_s), ring_a = smem_u32(ring);
    const uint32_t tV = tmem + 256, tK = tmem + 384;
    const uint32_t ns = static_cast<uint32_t>(n_sub);
    const uint32_t total = static_cast<uint32_t>(a.B) * ns;
    // Issuer 0: dP^T = V dO^T (dO as hi + lo); issuer 1: S^T = K Q^T; of
    // step s into buffer s % 2, once this issuer's products of step s - 2
    // have read the columns.
    auto issue_sp = [&](uint32_t s) -> bool {
      const uint32_t b = s & 1u, u = s >> 1, st = s % kKStages, n = s % ns, item = s / ns;
      if (n == 0 && !mbar_wait_warp(&bars->kv_full, item & 1u, abort, a.err, kSiteKV)) return false;
      if (!mbar_wait_warp(&bars->ring_full[st], (s / kKStages) & 1u, abort, a.err, kSiteRing))
        return false;
      const uint32_t qs = ring_a + st * 3 * kSubBytes, dh = qs + kSubBytes, dl = dh + kSubBytes;
      const uint32_t tS = tmem + 128 * b, tP = tS + 64;
      if (u > 0 && !mbar_wait_warp(who == 0 ? &bars->ds_read[b] : &bars->p_read[b], (u - 1) & 1u,
                              abort, a.err, kSiteSP))
        return false;
      tc_fence_after();
      if (who == 0) {
        mma_kk(tP, v_a, kKHalf, dh, kSubHalf, kSubRows, false);  // dP^T = V dO_hi^T
        mma_kk(tP, v_a, kKHalf, dl, kSubHalf, kSubRows, true);   //      + V dO_lo^T
      } else {
        mma_kk(tS, k_a, kKHalf, qs, kSubHalf, kSubRows, false);  // S^T = K Q^T
      }
      umma1_commit_w(&bars->sp_full[b]);
      if (n + 1 == ns) umma1_commit_w(&bars->kv_free);
      return true;
    };
    // Issuer 0: dK += dS^T Q; issuer 1: dV += P^T dO (P^T, dS^T and dO as
    // hi + lo) of step s.
    auto issue_g = [&](uint32_t s) -> bool {
      const uint32_t b = s & 1u, u = s >> 1, st = s % kKStages, n = s % ns, item = s / ns;
      if (!mbar_wait_warp(&bars->pds_full[b], u & 1u, abort, a.err, kSiteDS)) return false;
      if (n == 0 && item > 0 &&
          !mbar_wait_warp(&bars->acc_free, (item - 1) & 1u, abort, a.err, kSiteAcc))
        return false;
      tc_fence_after();
      const uint32_t qs = ring_a + st * 3 * kSubBytes, dh = qs + kSubBytes, dl = dh + kSubBytes;
      const uint32_t tS = tmem + 128 * b, tP = tS + 64;
      const bool first = n == 0;
      if (who == 0) {
        mma_tm(tK, [=](int kk) { return tP + 16 * kk; }, 4, qs, kSubHalf, !first);
        mma_tm(tK, [=](int kk) { return tP + 16 * kk + 8; }, 4, qs, kSubHalf, true);
        umma1_commit_w(&bars->ds_read[b]);
      } else {
        mma_tm(tV, [=](int kk) { return tS + 16 * kk; }, 4, dh, kSubHalf, !first);
        mma_tm(tV, [=](int kk) { return tS + 16 * kk; }, 4, dl, kSubHalf, true);
        mma_tm(tV, [=](int kk) { return tS + 16 * kk + 8; }, 4, dh, kSubHalf, true);
        umma1_commit_w(&bars->p_read[b]);
      }
      umma1_commit_w(&bars->ring_empty[st]);
      if (n + 1 == ns) umma1_commit_w(&bars->acc_full);
      return true;
    };
    if (ns == 0) {
      // No query blocks here: zero partials, but the same per-item handshakes.
      for (int b = 0; b < a.B; ++b) {
        if (!mbar_wait_warp(&bars->kv_full, static_cast<uint32_t>(b) & 1u, abort, a.err, kSiteKV))
          break;
        umma1_commit_w(&bars->kv_free);
        if (b > 0 && !mbar_wait_warp(&bars->acc_free, static_cast<uint32_t>(b - 1) & 1u, abort,
                                a.err, kSiteAcc))
          break;
        umma1_commit_w(&bars->acc_full);
      }
    } else {
      bool ok = true;
      for (uint32_t s = 0; s < 2 && s < total && ok; ++s) ok = issue_sp(s);
      for (uint32_t s = 0; s < total && ok; ++s) {
        ok = issue_g(s);
        if (ok && s + 2 < total) ok = issue_sp(s + 2);
      }
    }
    umma1_commit_w(&bars->drain[who]);
    drain(&bars->drain[who], 0);
  } else if (warp < kSoftWarps) {
    const int g = threadIdx.x >> 7, r = threadIdx.x & 127;  // r: key in the tile
    const uint32_t lane_base = static_cast<uint32_t>(r >> 5) << 21;
    const int key = kKKeys * kt + r;
    const bool key_ok = key < a.L;
    const int J = key_ok ? key / 16 : 0;
    const int wq = (r >> 5) & 3;  // this warp's 32 keys: key blocks 8 kt + 2 wq (+1)
    const uint32_t peer_even = cluster_addr(&bars->peer, 0);
    const uint32_t ack_odd = cluster_addr(&bars->peer_ack, 1);
    // Two groups of two warpgroups: group q takes the steps of buffer q
    // (n % 2 == q: heads 4 q .. 4 q + 3), warpgroup hg of it the rows of
    // heads 4 q + 2 hg + k, k = 0, 1 (two 16-row blocks, one bias cell each).
    const int q = g >> 1, hg = g & 1;
    uint32_t uq = 0, acc_count = 0;  // uq: this group's steps so far
    const int lane = static_cast<int>(lane_id());
    // Per warp, two buffers of the step's 32 lse2 then 32 delta values (row
    // 16 k + il: block k, position il).
    float *rows = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + kKBarsBytes) +
                  warp * 128;
    // This lane's row of step n of item b (block lane / 16, position
    // lane % 16): (lse2, delta); a row past L gets lse = +inf (its
    // probabilities are 0) and delta 0.
    auto row_value = [&](int b, int n) -> float2 {
      const int I = I0 + (n >> 1), h = 4 * (n & 1) + 2 * hg + (lane >> 4), il = lane & 15;
      const bool valid = 16 * I + il < a.L;
      const size_t row = (static_cast<size_t>(b) * kH + h) * a.L + 16 * I + (valid ? il : 0);
      return valid ? make_float2(__ldg(a.lse + row) * kLog2e, __ldg(a.delta + row))
                   : make_float2(__int_as_float(0x7f800000), 0.f);
    };
    bool ok = true;
    for (int b = 0; b < a.B && ok; ++b) {
      const float *bias_b = a.bias + static_cast<long long>(b) * a.bias_bstride;
      float *dbias_b = a.dbias + static_cast<long long>(b) * a.bias_bstride;
      const bool add_bias = a.bias_bstride == 0 && b > 0;  // shared bias: sum over items
      float2 rv_next = q < n_sub ? row_value(b, q) : make_float2(0.f, 0.f);
      for (int n = q; n < n_sub; n += 2) {
        const int I = I0 + (n >> 1), h0 = 4 * q + 2 * hg;
        float bt[2];
#pragma unroll
        for (int k = 0; k < 2; ++k)
          bt[k] = __ldg(bias_b + (static_cast<size_t>(h0 + k) * a.P + I) * a.P + J) * a.bias_mul;
        float *rv = rows + 64 * (uq & 1u);
        rv[lane] = rv_next.x;
        rv[32 + lane] = rv_next.y;
        __syncwarp();
        if (n + 2 < n_sub) rv_next = row_value(b, n + 2);
        ok = mbar_wait(&bars->sp_full[q], uq & 1u, abort, a.err, kSiteSoft);
        ++uq;
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
#pragma unroll 1
        for (int k = 0; k < 2; ++k) {
          const uint32_t tS = tmem + 128 * q + 32 * hg + 16 * k + lane_base, tP = tS + 64;
          uint32_t sv[16], pv[16];
          tmem_ld16(tS, sv);
          tmem_ld16(tP, pv);
          tmem_wait_ld16(sv);
          tmem_wait_ld16(pv);
          uint32_t ph[8], pl[8], sh[8], sl[8];
          // Keys past L (zero K rows) get probabilities too; they reach only
          // their own dK, dV rows, which are not stored, and the bias cell
          // sum, which leaves them out.
          const float bterm = k ? bt[1] : bt[0];
          float cell =
              a.capped ? key_rows<true>(sv, pv, rv + 16 * k, rv + 32 + 16 * k, bterm, a, ph, pl,
                                        sh, sl)
                       : key_rows<false>(sv, pv, rv + 16 * k, rv + 32 + 16 * k, bterm, a, ph,
                                         pl, sh, sl);
          if (!key_ok) cell = 0.f;
          // In place: this warp's lanes of the columns it has just read.
          tmem_st8(tS, ph);
          tmem_st8(tS + 8, pl);
          tmem_st8(tP, sh);
          tmem_st8(tP + 8, sl);
          // dbias: sum the cell over its 16 keys (lanes 0-15, 16-31 of the warp).
#pragma unroll
          for (int o = 8; o >= 1; o >>= 1) cell += __shfl_xor_sync(0xffffffffu, cell, o);
          if ((lane & 15) == 0) {
            const int Jc = 8 * kt + 2 * wq + (lane >> 4);
            if (Jc < a.P) {
              float *dst = dbias_b + (static_cast<size_t>(h0 + k) * a.P + I) * a.P + Jc;
              *dst = add_bias ? *dst + cell : cell;
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(&bars->pds_full[q]);
      }
      if (!ok) break;
      // Item epilogue: dK and dV of this CTA's half, then the pair's sum.
      ok = mbar_wait(&bars->acc_full, acc_count & 1u, abort, a.err, kSiteAcc);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t dv_[32], dk_[32];
      tmem_ld32(tmem + 256 + 32 * g + lane_base, dv_);
      tmem_ld32(tmem + 384 + 32 * g + lane_base, dk_);
      tmem_wait_ld(dv_);
      tmem_wait_ld(dk_);
      tc_fence_before();
      warp_arrive(&bars->acc_free);
      float *dvr = a.dv + (static_cast<size_t>(b) * a.L + key) * kD + 32 * g;
      float *dkr = a.dk + (static_cast<size_t>(b) * a.L + key) * kD + 32 * g;
      if (rank == 1) {
        // The odd CTA's partial (zeros if it had no query blocks) goes to the
        // item's rows; the even CTA adds it once it has been told.
        if (key_ok) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            dvr[e] = n_sub > 0 ? __uint_as_float(dv_[e]) : 0.f;
            dkr[e] = n_sub > 0 ? __uint_as_float(dk_[e]) : 0.f;
          }
        }
        __threadfence();
        // Every softmax warp of this CTA has written before thread 0 tells
        // the even CTA (a release at cluster scope after observing them).
        warp_arrive(&bars->epi);
        if (threadIdx.x == 0) {
          ok = mbar_wait(&bars->epi, acc_count & 1u, abort, a.err, kSiteXchg);
          if (ok) arrive_cluster_release(peer_even);
        }
        ok = __all_sync(0xffffffffu, ok);
        // The even CTA acknowledges once all its threads have read the
        // partial, so the two CTAs stay one item apart at most.
        if (ok) ok = mbar_wait(&bars->peer_ack, acc_count & 1u, abort, a.err, kSitePeer);
        if (!__all_sync(0xffffffffu, ok)) break;
      } else {
        ok = mbar_wait_cluster(&bars->peer, acc_count & 1u, abort, a.err, kSitePeer);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (key_ok) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float v0 = n_sub > 0 ? __uint_as_float(dv_[e]) : 0.f;
            const float k0 = n_sub > 0 ? __uint_as_float(dk_[e]) : 0.f;
            dvr[e] = v0 + __ldcg(dvr + e);
            dkr[e] = (k0 + __ldcg(dkr + e)) * a.inv_sqrt_d;
          }
        }
        warp_arrive(&bars->epi);
        if (threadIdx.x == 0) {
          ok = mbar_wait(&bars->epi, acc_count & 1u, abort, a.err, kSiteXchg);
          if (ok) mbar_arrive_cluster(ack_odd);
        }
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      ++acc_count;
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc1(tmem, kTmemCols);
  }
}

constexpr size_t kQuerySmem = 1024 + 3 * kQTileBytes + 2 * kQStages * kQKTileBytes +
                              sizeof(QBars) + 2 * 512 * sizeof(float);
constexpr size_t kKeySmem = 1024 + 2 * kKTileBytes + kKStages * 3 * kSubBytes + kKBarsBytes +
                            kSoftWarps * 128 * sizeof(float);
static_assert(kQuerySmem <= 227 * 1024 && kKeySmem <= 227 * 1024, "shared memory budget");

}  // namespace bwdtc

namespace {

bool encode_bf16(EncodeTiledFn enc, CUtensorMap *map, const void *base, int rank,
                 const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box) {
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::mutex g_bwd_mu;
bool g_bwd_configured[64] = {false};

}  // namespace

bool attn_bwd_tc_supported(const AttnBwdLaunch &x) {
  auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return x.Dv == 128 && x.H == 8 && al(x.q) && al(x.k) && al(x.v) && al(x.dout) && al(x.dq) &&
         x.L <= 65536;
}

cudaError_t launch_attn_bwd_tc(const AttnBwdLaunch &x, int num_sms, unsigned *err,
                               EncodeTiledFn enc) {
  using namespace bwdtc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(g_bwd_mu);
    if (!g_bwd_configured[dev]) {
      e = cudaFuncSetAttribute(bwd_query_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kQuerySmem));
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_query_kernel<2>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kQuerySmem));
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_key_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kKeySmem));
      if (e != cudaSuccess) return e;
      g_bwd_configured[dev] = true;
    }
  }
  const cuuint64_t B = static_cast<cuuint64_t>(x.B), L = static_cast<cuuint64_t>(x.L);
  CUtensorMap tq_q, tq_k, tdo_q, tdo_k, tk_q, tk_k, tv_q, tv_k;
  {  // q [B, H, L, D]: 128-row tiles (query kernel) and 64-row steps (key kernel)
    const cuuint64_t dims[4] = {kD, L, kH, B};
    const cuuint64_t strides[3] = {kD * 2, L * kD * 2, L * kD * 2 * kH};
    const cuuint32_t box_q[4] = {64, 16, 8, 1}, box_k[4] = {64, 16, 4, 1};
    if (!encode_bf16(enc, &tq_q, x.q, 4, dims, strides, box_q) ||
        !encode_bf16(enc, &tq_k, x.q, 4, dims, strides, box_k))
      return cudaErrorInvalidValue;
  }
  {  // the dout planes in dq: bf16 [B, H, L, 2 (hi, lo), 128]
    const cuuint64_t dims[5] = {kD, 2, L, kH, B};
    const cuuint64_t strides[4] = {kD * 2, kD * 4, L * kD * 4, L * kD * 4 * kH};
    const cuuint32_t box_q[5] = {64, 1, 16, 8, 1}, box_k[5] = {64, 1, 16, 4, 1};
    if (!encode_bf16(enc, &tdo_q, x.dq, 5, dims, strides, box_q) ||
        !encode_bf16(enc, &tdo_k, x.dq, 5, dims, strides, box_k))
      return cudaErrorInvalidValue;
  }
  {  // k, v [B, L, 128]: 64-key tiles (query kernel) and 128-key tiles (key kernel)
    const cuuint64_t dims[3] = {kD, L, B};
    const cuuint64_t strides[2] = {kD * 2, L * kD * 2};
    const cuuint32_t box_q[3] = {64, kQKeys, 1}, box_k[3] = {64, kKKeys, 1};
    if (!encode_bf16(enc, &tk_q, x.k, 3, dims, strides, box_q) ||
        !encode_bf16(enc, &tk_k, x.k, 3, dims, strides, box_k) ||
        !encode_bf16(enc, &tv_q, x.v, 3, dims, strides, box_q) ||
        !encode_bf16(enc, &tv_k, x.v, 3, dims, strides, box_k))
      return cudaErrorInvalidValue;
  }
  Args a;
  a.bias = x.bias;
  a.bias_bstride = x.bias_bstride;
  a.lse = x.lse;
  a.delta = x.delta;
  a.dq = x.dq;
  a.dk = x.dk;
  a.dv = x.dv;
  a.dbias = x.dbias;
  a.B = static_cast<int>(x.B);
  a.L = static_cast<int>(x.L);
  a.P = static_cast<int>((x.L + 15) / 16);
  a.nb = a.P;
  a.inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(kD));
  a.capped = std::isinf(x.cap) ? 0 : 1;
  a.qk_scale = a.capped ? a.inv_sqrt_d / x.cap : a.inv_sqrt_d;
  a.bias_mul = a.capped ? 1.0f / x.cap : 1.0f;
  a.A = a.capped ? x.cap * kLog2e : 0.0f;
  a.err = err;
  const long long n4 = static_cast<long long>(x.B) * kH * x.L * kD / 4;
  const long long split_grid = std::min<long long>((n4 + 255) / 256, 8ll * num_sms);
  bwd_split_kernel<<<static_cast<unsigned>(split_grid), 256, 0, x.stream>>>(x.dout, x.dq, n4);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int tiles = a.B * a.nb;
  const unsigned q_grid = static_cast<unsigned>(std::min(num_sms, tiles));
  bwd_query_kernel<1><<<q_grid, kThreads, kQuerySmem, x.stream>>>(tq_q, tdo_q, tk_q, tv_q, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned k_grid = static_cast<unsigned>(2 * ((x.L + kKKeys - 1) / kKKeys));
  bwd_key_kernel<<<k_grid, kThreads, kKeySmem, x.stream>>>(tq_k, tdo_k, tk_k, tv_k, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_query_kernel<2><<<q_grid, kThreads, kQuerySmem, x.stream>>>(tq_q, tdo_q, tk_q, tv_q, a);
  return cudaGetLastError();
}

}  // namespace ag
