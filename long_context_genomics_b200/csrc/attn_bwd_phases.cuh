// attn_bwd_phases.cuh -- the per-thread phases of the attention backward.
//
// Each phase is what one thread of a 256-thread CTA does between two
// barriers, written as a __host__ __device__ function of the thread index
// and the CTA's shared-memory tiles; the kernels in attn_bwd.cu call them
// in order with __syncthreads() between.
//
// What is computed (the chain rule through Eq. L_ij of the page "Making
// Full-Context AlphaGenome Fit on an RTX 3090", section "Why stock
// FlashAttention was not a drop-in replacement"; the page lists a backward
// pass as later work for fine-tuning, section "Where I would take it next"):
//   x_ij    = q_i . k_j / sqrt(D) + bias[h, i/16, j/16]
//   L_ij    = cap * tanh(x_ij / cap)              (no cap: L_ij = x_ij)
//   p_ij    = exp(L_ij - lse_i)                   (lse from the forward)
//   dp_ij   = dout_i . v_j
//   delta_i = sum_j p_ij dp_ij
//   ds_ij   = p_ij (dp_ij - delta_i) (1 - tanh^2(x_ij / cap))
//   dq_i    = sum_j ds_ij k_j / sqrt(D)
//   dk_j    = sum_{h,i} ds_ij q_i / sqrt(D),  dv_j = sum_{h,i} p_ij dout_i
//   dbias[h, I, J] = sum over the 16 x 16 cell of ds_ij (and over the
//                    batch items that share the bias).
// All arithmetic is fp32 on the CUDA cores from the bf16 q, k, v.
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stddef.h>

namespace agbwd {

constexpr int kD = 128;        // query / key width
constexpr int kCh = 32;        // query rows per chunk, keys per tile
constexpr int kThreads = 256;  // threads per CTA
constexpr int kBlk = 16;       // positions per compact bias cell

struct BwdArgs {
  const __nv_bfloat16 *q;  // [B, H, L, D]
  const __nv_bfloat16 *k;  // [B, L, D]
  const __nv_bfloat16 *v;  // [B, L, Dv]
  const float *bias;       // [H, P, P] per item at bias + b * bias_bstride
  long long bias_bstride;  // floats; 0 = one bias shared by every item
  const float *lse;        // [B, H, L] from the forward
  const float *dout;       // [B, H, L, Dv]
  float *delta;            // [B, H, L]   written by the query kernel
  float *dq;               // [B, H, L, D]
  float *dk;               // [B, L, D]
  float *dv;               // [B, L, Dv]
  float *dbias;            // layout of bias
  int B, H, L, P;
  int capped;              // 0: no soft cap
  float cap;
  float inv_sqrt_d;
};

// Shared-memory tiles, in floats.  Rows are padded by one float so that
// threads reading one column of different rows hit different banks.
template <int DV>
struct Tiles {
  static constexpr int kQs = kD + 1, kOs = DV + 1, kPs = kCh + 1;
  static constexpr int kQ = 0;                     // q chunk     [32][D+1]
  static constexpr int kK = kQ + kCh * kQs;        // k tile      [32][D+1]
  static constexpr int kO = kK + kCh * kQs;        // dout chunk  [32][Dv+1]
  static constexpr int kV = kO + kCh * kOs;        // v tile      [32][Dv+1]
  static constexpr int kP = kV + kCh * kOs;        // p (or p dp) [32][33]
  static constexpr int kS = kP + kCh * kPs;        // ds          [32][33]
  static constexpr int kLse = kS + kCh * kPs;      // lse of the chunk's rows
  static constexpr int kDelta = kLse + kCh;        // delta of the chunk's rows
  static constexpr int kRed = kDelta + kCh;        // dbias partial sums [128]
  static constexpr int kFloats = kRed + 128;
  static constexpr size_t kBytes = sizeof(float) * kFloats;
  static constexpr int kAccV = 8 * DV / 64;        // dv accumulators per thread
};

// Rows [r0, r0 + 32) of a row-major [n, W] matrix into a [32][W + 1] tile,
// widened to fp32; rows at or past n are zero.
__host__ __device__ inline void load_rows_bf16(int t, float *dst,
                                               const __nv_bfloat16 *src, int W,
                                               int r0, int n) {
  for (int e = t; e < kCh * W; e += kThreads) {
    const int r = e / W, c = e - r * W;
    dst[r * (W + 1) + c] =
        (r0 + r < n) ? __bfloat162float(src[static_cast<size_t>(r0 + r) * W + c]) : 0.0f;
  }
}

__host__ __device__ inline void load_rows_f32(int t, float *dst, const float *src,
                                              int W, int r0, int n) {
  for (int e = t; e < kCh * W; e += kThreads) {
    const int r = e / W, c = e - r * W;
    dst[r * (W + 1) + c] = (r0 + r < n) ? src[static_cast<size_t>(r0 + r) * W + c] : 0.0f;
  }
}

// Scores of the 32 x 32 (query, key) block at rows i0.., keys j0.. of item b,
// head h.  Thread t takes rows {t/16, t/16 + 16} x keys {t%16, t%16 + 16}.
// kDeltaPass: write p_ij * dp_ij into the p tile (for delta) and no ds.
// Otherwise: write p_ij into the p tile and ds_ij into the ds tile.  Pairs
// past the end of the sequence get 0.
template <int DV, bool kDeltaPass>
__host__ __device__ inline void phase_scores(int t, float *sm, const BwdArgs &a,
                                             int b, int h, int i0, int j0) {
  using T = Tiles<DV>;
  const float *Q = sm + T::kQ, *K = sm + T::kK, *O = sm + T::kO, *V = sm + T::kV;
  const float *lse = sm + T::kLse, *delta = sm + T::kDelta;
  float *Pt = sm + T::kP, *St = sm + T::kS;
  const int ti = t >> 4, tj = t & 15;
  float s[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
  float dp[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
  for (int d = 0; d < kD; ++d) {
    const float q0 = Q[ti * T::kQs + d], q1 = Q[(ti + 16) * T::kQs + d];
    const float k0 = K[tj * T::kQs + d], k1 = K[(tj + 16) * T::kQs + d];
    s[0][0] = fmaf(q0, k0, s[0][0]);
    s[0][1] = fmaf(q0, k1, s[0][1]);
    s[1][0] = fmaf(q1, k0, s[1][0]);
    s[1][1] = fmaf(q1, k1, s[1][1]);
  }
  for (int c = 0; c < DV; ++c) {
    const float g0 = O[ti * T::kOs + c], g1 = O[(ti + 16) * T::kOs + c];
    const float v0 = V[tj * T::kOs + c], v1 = V[(tj + 16) * T::kOs + c];
    dp[0][0] = fmaf(g0, v0, dp[0][0]);
    dp[0][1] = fmaf(g0, v1, dp[0][1]);
    dp[1][0] = fmaf(g1, v0, dp[1][0]);
    dp[1][1] = fmaf(g1, v1, dp[1][1]);
  }
  const float *bias_bh = a.bias + static_cast<long long>(b) * a.bias_bstride +
                         static_cast<size_t>(h) * a.P * a.P;
  for (int x = 0; x < 2; ++x) {
    for (int y = 0; y < 2; ++y) {
      const int i = ti + 16 * x, j = tj + 16 * y;
      const int gi = i0 + i, gj = j0 + j;
      float p = 0.0f, ds = 0.0f;
      if (gi < a.L && gj < a.L) {
        const float z = fmaf(s[x][y], a.inv_sqrt_d,
                             bias_bh[static_cast<size_t>(gi / kBlk) * a.P + gj / kBlk]);
        float l = z, g = 1.0f;
        if (a.capped) {
          const float th = tanhf(z / a.cap);
          l = a.cap * th;
          g = 1.0f - th * th;
        }
        p = expf(l - lse[i]);
        ds = p * (dp[x][y] - delta[i]) * g;
      }
      if (kDeltaPass) {
        Pt[i * T::kPs + j] = p * dp[x][y];
      } else {
        Pt[i * T::kPs + j] = p;
        St[i * T::kPs + j] = ds;
      }
    }
  }
}

// Delta pass: row t (t < 32) adds its 32 values of p * dp.
template <int DV>
__host__ __device__ inline void phase_delta_add(int t, float *sm) {
  using T = Tiles<DV>;
  if (t >= kCh) return;
  const float *Pt = sm + T::kP;
  float acc = 0.0f;
  for (int j = 0; j < kCh; ++j) acc += Pt[t * T::kPs + j];
  sm[T::kDelta + t] += acc;
}

// dq accumulation over one key tile: thread t owns rows t/64 + 4e (e < 8)
// and columns t%64 + 64m (m < 2): acc[2e + m] += sum_j ds[i][j] * k[j][d].
template <int DV>
__host__ __device__ inline void phase_dq(int t, const float *sm, float (&acc)[16]) {
  using T = Tiles<DV>;
  const float *K = sm + T::kK, *St = sm + T::kS;
  const int ig = t >> 6, cl = t & 63;
  for (int j = 0; j < kCh; ++j) {
    const float k0 = K[j * T::kQs + cl], k1 = K[j * T::kQs + cl + 64];
    for (int e = 0; e < 8; ++e) {
      const float ds = St[(ig + 4 * e) * T::kPs + j];
      acc[2 * e] = fmaf(ds, k0, acc[2 * e]);
      acc[2 * e + 1] = fmaf(ds, k1, acc[2 * e + 1]);
    }
  }
}

// dk, dv accumulation over one query chunk: thread t owns keys t/64 + 4e
// (e < 8), dk columns t%64 + 64m (m < 2) and dv columns t%64 + 64m
// (m < Dv/64): dk[2e + m] += sum_i ds[i][j] q[i][d],
// dv[(Dv/64)e + m] += sum_i p[i][j] dout[i][c].
template <int DV>
__host__ __device__ inline void phase_kv(int t, const float *sm, float (&dk)[16],
                                         float (&dv)[Tiles<DV>::kAccV]) {
  using T = Tiles<DV>;
  constexpr int kMv = DV / 64;
  const float *Q = sm + T::kQ, *O = sm + T::kO, *Pt = sm + T::kP, *St = sm + T::kS;
  const int jg = t >> 6, cl = t & 63;
  for (int i = 0; i < kCh; ++i) {
    const float q0 = Q[i * T::kQs + cl], q1 = Q[i * T::kQs + cl + 64];
    float g[kMv];
    for (int m = 0; m < kMv; ++m) g[m] = O[i * T::kOs + cl + 64 * m];
    for (int e = 0; e < 8; ++e) {
      const int j = jg + 4 * e;
      const float ds = St[i * T::kPs + j], p = Pt[i * T::kPs + j];
      dk[2 * e] = fmaf(ds, q0, dk[2 * e]);
      dk[2 * e + 1] = fmaf(ds, q1, dk[2 * e + 1]);
      for (int m = 0; m < kMv; ++m) dv[kMv * e + m] = fmaf(p, g[m], dv[kMv * e + m]);
    }
  }
}

// dbias, first half: the chunk's 32 x 32 ds block holds 2 x 2 compact cells.
// Thread t < 128 sums 8 values of cell t/32 (query half (t/32)/2, key half
// (t/32)%2): row 16*qh + (t%32)/2, keys 16*kh + 8*(t%2) .. + 8.
template <int DV>
__host__ __device__ inline void phase_dbias_partial(int t, float *sm) {
  using T = Tiles<DV>;
  if (t >= 128) return;
  const float *St = sm + T::kS;
  const int cell = t >> 5, lane = t & 31;
  const int i = 16 * (cell >> 1) + (lane >> 1);
  const int jb = 16 * (cell & 1) + 8 * (lane & 1);
  float acc = 0.0f;
  for (int j = jb; j < jb + 8; ++j) acc += St[i * T::kPs + j];
  sm[T::kRed + t] = acc;
}

// dbias, second half: thread t < 4 adds the 32 partials of cell t and
// stores it (the first item, or one bias per item) or adds it (later items
// sharing the bias).  Each cell of item b's bias belongs to exactly one
// chunk of one key tile, so one thread of one CTA writes it.
template <int DV>
__host__ __device__ inline void phase_dbias_store(int t, const float *sm,
                                                  const BwdArgs &a, int b, int h,
                                                  int i0, int j0) {
  using T = Tiles<DV>;
  if (t >= 4) return;
  float acc = 0.0f;
  for (int r = 0; r < 32; ++r) acc += sm[T::kRed + 32 * t + r];
  const int I = i0 / kBlk + (t >> 1), J = j0 / kBlk + (t & 1);
  if (I >= a.P || J >= a.P) return;
  float *cell = a.dbias + static_cast<long long>(b) * a.bias_bstride +
                (static_cast<size_t>(h) * a.P + I) * a.P + J;
  if (a.bias_bstride == 0 && b > 0)
    *cell += acc;
  else
    *cell = acc;
}

}  // namespace agbwd
