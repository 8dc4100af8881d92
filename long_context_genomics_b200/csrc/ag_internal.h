// ag_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ag {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType,
                                   cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

struct AttnLaunch {
  const void *q, *k, *v;
  const float *bias;
  float *out, *lse;
  int64_t B, L;
  float cap;
  unsigned *err;        // device error word
  int num_sms;
  EncodeTiledFn encode;
  cudaStream_t stream;
};

// Returns cudaSuccess or the first CUDA error; CUDA_ERROR_* from tensor-map
// encoding is reported as cudaErrorInvalidValue.
cudaError_t launch_attn_fwd(const AttnLaunch &a);

cudaError_t launch_pair_bias_project(const float *pair, const float *W,
                                     float *bias, int64_t P, int num_sms,
                                     cudaStream_t stream);

cudaError_t launch_wait_timeout_probe(uint64_t timeout_ns, unsigned *err,
                                      cudaStream_t stream);

}  // namespace ag
