// pair_bias_project.cu -- compact pair representation -> per-head bias.
//
//   bias[h, p, q] = sum_c pair[p, q, c] * W[c, h]      (Cp = 128, H = 8)
//
// Page "Making Full-Context AlphaGenome Fit on an RTX 3090", section
// "Profiling pointed at one very large object": the dense path projects a
// compact pair representation into the attention bias (and then repeats it;
// the attention kernel reads the compact result directly instead).
//
// Bound by HBM: 512 bytes of pair data per cell against 8 outputs.  One warp
// handles 8 consecutive cells per step.  Lane l reads channels 4l..4l+3 of
// every cell (each load instruction moves one whole 512-byte cell, fully
// coalesced) and keeps W[4l..4l+3, 0..7] in registers.  The 64 partial sums
// (8 heads x 8 cells) are then reduced across the warp by a butterfly
// reduce-scatter (offsets 16, 8, 4, 2, 1), after which lane l holds the two
// finished values of head l/4 for cells 2(l%4) and 2(l%4)+1: a float2 store,
// eight consecutive cells per head across the warp.
#include "ag_internal.h"

namespace ag {
namespace proj {

constexpr int kCp = 128;
constexpr int kH = 8;
constexpr int kCells = 8;  // cells per warp step
constexpr int kThreads = 256;

// One reduce-scatter level: lanes with bit `o` set keep the upper half of
// the first 2*n values, the others the lower half; each adds its partner's.
template <int n>
__device__ __forceinline__ void rs_level(float (&a)[64], int o, bool upper) {
#pragma unroll
  for (int j = 0; j < n; ++j) {
    const float keep = upper ? a[j + n] : a[j];
    const float send = upper ? a[j] : a[j + n];
    a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}

__global__ void __launch_bounds__(kThreads)
    pair_bias_project_kernel(const float4 *__restrict__ pair,
                             const float *__restrict__ W,
                             float *__restrict__ bias, long long n_cells,
                             int vec_store) {
  const int lane = threadIdx.x & 31;
  float w[4][kH];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < kH; ++h) w[i][h] = __ldg(W + (4 * lane + i) * kH + h);

  const long long n_groups = (n_cells + kCells - 1) / kCells;
  const long long warp0 =
      (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int h_out = lane >> 2;              // head this lane finishes
  const int n_out = 2 * (lane & 3);         // first of its two cells

  for (long long g = warp0; g < n_groups; g += n_warps) {
    const long long c0 = g * kCells;
    float4 x[kCells];
#pragma unroll
    for (int n = 0; n < kCells; ++n) {
      const long long cell = c0 + n;
      x[n] = cell < n_cells ? __ldcs(pair + cell * (kCp / 4) + lane)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float a[64];  // a[h * 8 + n]
#pragma unroll
    for (int h = 0; h < kH; ++h)
#pragma unroll
      for (int n = 0; n < kCells; ++n)
        a[h * kCells + n] =
            fmaf(x[n].w, w[3][h],
                 fmaf(x[n].z, w[2][h], fmaf(x[n].y, w[1][h], x[n].x * w[0][h])));
    rs_level<32>(a, 16, lane & 16);
    rs_level<16>(a, 8, lane & 8);
    rs_level<8>(a, 4, lane & 4);
    rs_level<4>(a, 2, lane & 2);
    rs_level<2>(a, 1, lane & 1);
    // a[0], a[1]: head h_out, cells c0 + n_out and c0 + n_out + 1.
    float *dst = bias + static_cast<long long>(h_out) * n_cells + c0 + n_out;
    const long long cell = c0 + n_out;
    if (vec_store && cell + 1 < n_cells) {
      __stcs(reinterpret_cast<float2 *>(dst), make_float2(a[0], a[1]));
    } else {
      if (cell < n_cells) dst[0] = a[0];
      if (cell + 1 < n_cells) dst[1] = a[1];
    }
  }
}

}  // namespace proj

cudaError_t launch_pair_bias_project(const float *pair, const float *W,
                                     float *bias, int64_t P, int num_sms,
                                     cudaStream_t stream) {
  using namespace proj;
  const long long n_cells = static_cast<long long>(P) * P;
  const long long n_groups = (n_cells + kCells - 1) / kCells;
  const long long warps_per_block = kThreads / 32;
  long long blocks = (n_groups + warps_per_block - 1) / warps_per_block;
  const long long max_blocks = static_cast<long long>(num_sms) * 8;
  if (blocks > max_blocks) blocks = max_blocks;
  if (blocks < 1) blocks = 1;
  // float2 stores need an even cell count (then every head's plane starts
  // 8-byte aligned, as does every even cell inside it).
  const int vec_store = (n_cells % 2 == 0) ? 1 : 0;
  pair_bias_project_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      reinterpret_cast<const float4 *>(pair), W, bias, n_cells, vec_store);
  return cudaGetLastError();
}

}  // namespace ag
