// attn_bwd.cu -- backward of the pair-bias multi-query attention.
//
// Two kernels on the caller's stream, each built from the phases in
// attn_bwd_phases.cuh with a barrier between phases:
//
//   attn_bwd_q_kernel   one CTA per (32 query rows, head, item).  Pass 1
//                       runs over every key tile and forms
//                       delta_i = sum_j p_ij dp_ij from its definition;
//                       pass 2 runs over them again and accumulates
//                       dq_i = sum_j ds_ij k_j / sqrt(D).  Writes delta, dq.
//   attn_bwd_kv_kernel  one CTA per tile of 32 keys.  For every item, head
//                       and 32-row query chunk it forms ds and p for its
//                       keys and accumulates dk, dv (summed over the heads
//                       that share K and V) and the 2 x 2 compact bias cells
//                       the block covers.  Reads delta from the first kernel.
//
// Every output value is written by one thread of one CTA, in a fixed order,
// so the results are deterministic and need no atomics; a bias shared by the
// batch items gets its cells summed over the items in item order.
//
// This is a first, CUDA-core fp32 implementation: every product runs on the
// FMA pipe from shared-memory tiles.  Its arithmetic count per call is
// 2 (D + Dv) B H L^2 for the delta pass, 2 (2 D + Dv) B H L^2 for dq and
// 4 (D + Dv) B H L^2 for dk and dv.
#include <cuda_runtime.h>

#include "ag_internal.h"
#include "attn_bwd_phases.cuh"

namespace agbwd {

template <int DV>
__global__ void __launch_bounds__(kThreads, 2) attn_bwd_q_kernel(BwdArgs a) {
  using T = Tiles<DV>;
  extern __shared__ float sm[];
  const int t = threadIdx.x;
  const int n_chunks = (a.L + kCh - 1) / kCh;
  const int b = blockIdx.x / n_chunks;
  const int i0 = (blockIdx.x - b * n_chunks) * kCh;
  const int h = blockIdx.y;
  const size_t row0 = (static_cast<size_t>(b) * a.H + h) * a.L;  // row (b, h, 0)
  const __nv_bfloat16 *kb = a.k + static_cast<size_t>(b) * a.L * kD;
  const __nv_bfloat16 *vb = a.v + static_cast<size_t>(b) * a.L * DV;

  load_rows_bf16(t, sm + T::kQ, a.q + row0 * kD, kD, i0, a.L);
  load_rows_f32(t, sm + T::kO, a.dout + row0 * DV, DV, i0, a.L);
  if (t < kCh) {
    sm[T::kLse + t] = (i0 + t < a.L) ? a.lse[row0 + i0 + t] : 0.0f;
    sm[T::kDelta + t] = 0.0f;
  }
  // Pass 1: delta.
  for (int j0 = 0; j0 < a.L; j0 += kCh) {
    load_rows_bf16(t, sm + T::kK, kb, kD, j0, a.L);
    load_rows_bf16(t, sm + T::kV, vb, DV, j0, a.L);
    __syncthreads();
    phase_scores<DV, true>(t, sm, a, b, h, i0, j0);
    __syncthreads();
    phase_delta_add<DV>(t, sm);
  }
  __syncthreads();
  if (t < kCh && i0 + t < a.L) a.delta[row0 + i0 + t] = sm[T::kDelta + t];
  // Pass 2: dq.
  float acc[16];
  for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
  for (int j0 = 0; j0 < a.L; j0 += kCh) {
    load_rows_bf16(t, sm + T::kK, kb, kD, j0, a.L);
    load_rows_bf16(t, sm + T::kV, vb, DV, j0, a.L);
    __syncthreads();
    phase_scores<DV, false>(t, sm, a, b, h, i0, j0);
    __syncthreads();
    phase_dq<DV>(t, sm, acc);
    __syncthreads();
  }
  const int ig = t >> 6, cl = t & 63;
  for (int e = 0; e < 8; ++e) {
    const int i = i0 + ig + 4 * e;
    if (i >= a.L) continue;
    float *dst = a.dq + (row0 + i) * kD;
    dst[cl] = acc[2 * e] * a.inv_sqrt_d;
    dst[cl + 64] = acc[2 * e + 1] * a.inv_sqrt_d;
  }
}

template <int DV>
__global__ void __launch_bounds__(kThreads, 2) attn_bwd_kv_kernel(BwdArgs a) {
  using T = Tiles<DV>;
  constexpr int kMv = DV / 64;
  extern __shared__ float sm[];
  const int t = threadIdx.x;
  const int j0 = blockIdx.x * kCh;
  const int jg = t >> 6, cl = t & 63;
  for (int b = 0; b < a.B; ++b) {
    float dk[16], dv[T::kAccV];
    for (int e = 0; e < 16; ++e) dk[e] = 0.0f;
    for (int e = 0; e < T::kAccV; ++e) dv[e] = 0.0f;
    load_rows_bf16(t, sm + T::kK, a.k + static_cast<size_t>(b) * a.L * kD, kD, j0, a.L);
    load_rows_bf16(t, sm + T::kV, a.v + static_cast<size_t>(b) * a.L * DV, DV, j0, a.L);
    for (int h = 0; h < a.H; ++h) {
      const size_t row0 = (static_cast<size_t>(b) * a.H + h) * a.L;
      for (int i0 = 0; i0 < a.L; i0 += kCh) {
        load_rows_bf16(t, sm + T::kQ, a.q + row0 * kD, kD, i0, a.L);
        load_rows_f32(t, sm + T::kO, a.dout + row0 * DV, DV, i0, a.L);
        if (t < kCh) {
          const bool in = i0 + t < a.L;
          sm[T::kLse + t] = in ? a.lse[row0 + i0 + t] : 0.0f;
          sm[T::kDelta + t] = in ? a.delta[row0 + i0 + t] : 0.0f;
        }
        __syncthreads();
        phase_scores<DV, false>(t, sm, a, b, h, i0, j0);
        __syncthreads();
        phase_kv<DV>(t, sm, dk, dv);
        phase_dbias_partial<DV>(t, sm);
        __syncthreads();
        phase_dbias_store<DV>(t, sm, a, b, h, i0, j0);
      }
    }
    for (int e = 0; e < 8; ++e) {
      const int j = j0 + jg + 4 * e;
      if (j >= a.L) continue;
      float *dkj = a.dk + (static_cast<size_t>(b) * a.L + j) * kD;
      dkj[cl] = dk[2 * e] * a.inv_sqrt_d;
      dkj[cl + 64] = dk[2 * e + 1] * a.inv_sqrt_d;
      float *dvj = a.dv + (static_cast<size_t>(b) * a.L + j) * DV;
      for (int m = 0; m < kMv; ++m) dvj[cl + 64 * m] = dv[kMv * e + m];
    }
  }
}

template <int DV>
static cudaError_t launch_dv(const BwdArgs &a, cudaStream_t stream) {
  using T = Tiles<DV>;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_q_kernel<DV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(T::kBytes));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_kv_kernel<DV>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(T::kBytes));
  if (e != cudaSuccess) return e;
  const unsigned n_chunks = static_cast<unsigned>((a.L + kCh - 1) / kCh);
  const dim3 grid_q(n_chunks * static_cast<unsigned>(a.B), static_cast<unsigned>(a.H));
  attn_bwd_q_kernel<DV><<<grid_q, kThreads, T::kBytes, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_kv_kernel<DV><<<n_chunks, kThreads, T::kBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace agbwd

namespace ag {

cudaError_t launch_attn_bwd(const AttnBwdLaunch &x) {
  agbwd::BwdArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(x.q);
  a.k = static_cast<const __nv_bfloat16 *>(x.k);
  a.v = static_cast<const __nv_bfloat16 *>(x.v);
  a.bias = x.bias;
  a.bias_bstride = x.bias_bstride;
  a.lse = x.lse;
  a.dout = x.dout;
  a.delta = x.delta;
  a.dq = x.dq;
  a.dk = x.dk;
  a.dv = x.dv;
  a.dbias = x.dbias;
  a.B = static_cast<int>(x.B);
  a.H = static_cast<int>(x.H);
  a.L = static_cast<int>(x.L);
  a.P = static_cast<int>((x.L + agbwd::kBlk - 1) / agbwd::kBlk);
  a.capped = isinf(x.cap) ? 0 : 1;
  a.cap = x.cap;
  a.inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(agbwd::kD));
  if (x.Dv == 192) return agbwd::launch_dv<192>(a, x.stream);
  return agbwd::launch_dv<128>(a, x.stream);
}

int attn_bwd_kernel_count() { return 2; }

}  // namespace ag
