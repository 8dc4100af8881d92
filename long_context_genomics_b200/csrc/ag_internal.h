// ag_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/ag.h"

namespace ag {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType,
                                   cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

// Scratch of the attention kernel's range schedule (ag_attn_fwd_noalloc) for
// pairs of query tiles whose key range is split between clusters: per slot a
// partial output [2][128][Dv] fp32 (sized for the widest Dv, 192) and a
// partial log-sum-exp [2][128] fp32.  Nothing in it must be initialised.
constexpr size_t kAttnSlotOutBytes = 2 * 128 * 192 * sizeof(float);
constexpr size_t kAttnSlotLseBytes = 2 * 128 * sizeof(float);
inline size_t attn_scratch_bytes(int slots) {
  return static_cast<size_t>(slots) * (kAttnSlotOutBytes + kAttnSlotLseBytes);
}

// Keys per K/V tile of the attention kernel, and its work steps: pairs of
// 128-row query tiles (16 positions x 8 heads each) times key tiles.  The
// kernel indexes steps with int, so callers keep this at or below 2^30.
constexpr int64_t kAttnKeyTile = 128;
// Most 2-CTA clusters an attention launch uses (one per SM pair up to 256 SMs).
constexpr int kAttnMaxClusters = 128;
inline int64_t attn_work_steps(int64_t B, int64_t Lq, int64_t L) {
  const int64_t blocks = (Lq + 15) / 16;  // the last may be partial
  return B * ((blocks + 1) / 2) * ((L + kAttnKeyTile - 1) / kAttnKeyTile);
}
inline int64_t attn_work_steps(int64_t B, int64_t L) { return attn_work_steps(B, L, L); }

struct AttnLaunch {
  const void *q, *k, *v;
  const float *bias;
  int64_t bias_bstride;  // floats between batch items' bias (0: shared)
  float *out, *lse;
  int64_t B, L;         // batch items, keys per item
  int64_t Lq;           // query positions per item (rows of q, out and lse)
  int64_t Dv;           // value width: 128 or 192
  float cap;
  unsigned *err;        // device error word
  int num_sms;
  void *scratch;        // NULL: schedules that need no scratch (whole pairs or
                        // two launches); else attn_scratch_bytes(scratch_slots)
                        // bytes, 256-aligned, for the range schedule
  int scratch_slots;    // clusters the range schedule may use (>= 1)
  EncodeTiledFn encode;
  cudaStream_t stream;
};

// Returns cudaSuccess or the first CUDA error; CUDA_ERROR_* from tensor-map
// encoding is reported as cudaErrorInvalidValue.
cudaError_t launch_attn_fwd(const AttnLaunch &a);

// How many kernels launch_attn_fwd launches for these sizes on the current
// device (0 for an empty call, 1, or 2 when split pairs need the merge kernel
// or a second launch); scratch_slots 0 for the schedules without scratch.
cudaError_t attn_fwd_kernel_count(int64_t B, int64_t Lq, int64_t L, int64_t Dv, float cap,
                                  int num_sms, int scratch_slots, int *count);
// The schedule launch_attn_fwd uses for these sizes with sm_pairs resident
// 2-CTA clusters (pure host logic): wb and fb hold kAttnMaxClusters + 1 ints.
void attn_fwd_schedule(int64_t B, int64_t L, int sm_pairs, int scratch_slots, int *sched,
                       int *clusters, int *tail_clusters, int *whole, int *n_whole,
                       int *split_at, int *wb, int *fb);
// How many 2-CTA clusters the first launch of such a call uses.
cudaError_t attn_fwd_clusters(int64_t B, int64_t L, int64_t Dv, float cap, int num_sms,
                              int scratch_slots, int *clusters);

// Backward of the attention (attn_bwd.cu): two kernels, the query kernel
// (delta, dq) then the key kernel (dk, dv, dbias), on `stream`.
struct AttnBwdLaunch {
  const void *q, *k, *v;  // bf16 [B,H,L,128], [B,L,128], [B,L,Dv]
  const float *bias;
  int64_t bias_bstride;   // floats between batch items' bias (0: shared)
  const float *lse, *dout;
  float *delta, *dq, *dk, *dv, *dbias;
  int64_t B, H, L, Dv;
  float cap;              // > 0, +inf for no cap
  cudaStream_t stream;
};
cudaError_t launch_attn_bwd(const AttnBwdLaunch &a);
int attn_bwd_kernel_count();
// Tensor-core backward (attn_bwd_sm100.cu): value width 128, q, k, v, dout
// and dq 16-byte aligned; four launches (dout split, query pass 1, key pass,
// query pass 2).  Uses dq as the staging place of dout's bf16 halves.
bool attn_bwd_tc_supported(const AttnBwdLaunch &a);
cudaError_t launch_attn_bwd_tc(const AttnBwdLaunch &a, int num_sms, unsigned *err,
                               EncodeTiledFn encode);

// Projects `cells` consecutive cells of 128 channels into 8 head planes of
// `cells` floats each.
cudaError_t launch_pair_bias_project(const float *pair, const float *W,
                                     float *bias, int64_t cells, int num_sms,
                                     unsigned *err, EncodeTiledFn encode,
                                     cudaStream_t stream);

cudaError_t launch_wait_timeout_probe(uint64_t timeout_ns, unsigned *err,
                                      cudaStream_t stream);

// Shared by the entry points (ag_api.cu).
struct DeviceInfo {
  bool ready = false;
  bool sm100 = false;
  int num_sms = 0;
  unsigned *err = nullptr;  // device address of the device error word
};
// Per-device set-up of the current device, done once; AG_ERR_UNSUPPORTED on
// anything but sm_100.
ag_status device_info(DeviceInfo **out);
ag_status get_encoder(EncodeTiledFn *fn);
ag_status check_attn_sizes(int64_t B, int64_t H, int64_t L, int64_t D, int64_t block,
                           float cap);
bool aligned(const void *p, uintptr_t a);
bool overlap(const void *a, uint64_t na, const void *b, uint64_t nb);
ag_status from_cuda(cudaError_t e);

}  // namespace ag
