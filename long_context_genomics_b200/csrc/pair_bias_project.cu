// pair_bias_project.cu -- compact pair representation -> per-head bias.
//
//   bias[h, p, q] = sum_c pair[p, q, c] * W[c, h]      (Cp = 128, H = 8)
//
// Page "Making Full-Context AlphaGenome Fit on an RTX 3090", section
// "Profiling pointed at one very large object": the dense path projects a
// compact pair representation into the attention bias (and then repeats it;
// the attention kernel reads the compact result directly instead).
//
// Bound by HBM: 512 bytes of pair data per cell against 8 outputs.  A
// persistent CTA per SM streams chunks of 32 consecutive cells (16 KB) into a
// 12-stage shared-memory ring with TMA (one producer lane; the pair tensor is
// seen as [cells, 128] fp32 rows, four 32-channel boxes per chunk with the
// 128-byte swizzle), so up to 192 KB per SM are in flight.  Each of twelve
// consumer warps takes whole chunks (chunk n of the CTA goes to warp n % 12,
// so warp w always uses ring slot w and waits for its phases in order; a
// slot shared by warps would let a warp wait for a phase one ahead of the
// slot's current one, which a parity wait cannot tell from the phase
// before).  Lane l owns cell l of the chunk and sums
// its 128 channels for all 8 heads in registers (packed fp32x2 products, two
// heads per instruction).  The swizzle puts the 16-byte channel group g of
// cell l at group slot g ^ (l % 8) of its 128-byte row, so the eight lanes of
// a shared-memory phase read eight different bank groups; W sits in shared
// memory and every lane reads the same W row (a broadcast).  No cross-lane
// reduction is needed, and lane l stores cell l of each head plane: 32
// consecutive floats per store instruction.
#include <mutex>

#include "ag_internal.h"
#include "sm100.cuh"

namespace ag {
namespace proj {

constexpr int kCp = 128;
constexpr int kH = 8;
constexpr int kCellBytes = kCp * 4;                  // 512
constexpr int kChunkCells = 32;                      // one cell per lane
constexpr int kChunkBytes = kChunkCells * kCellBytes;  // 16 KB
constexpr int kBoxBytes = kChunkCells * 128;         // 32 cells x 32 channels
// Measured on B200 at P = 512 (134 MB): 12 stages of 16 KB per SM reach the
// same time as 6 of 32 KB; fewer bytes in flight are slower, and two or three
// CTAs per SM with the same bytes in flight are slower too.
constexpr int kStages = 12;
constexpr int kConsumerWarps = 12;
static_assert(kStages % kConsumerWarps == 0, "each ring slot belongs to one consumer warp");
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + producer warp
constexpr int kWBytes = kCp * kH * 4;                // 4 KB
constexpr size_t kSmemBytes = 1024 + kStages * kChunkBytes + kWBytes + 2 * kStages * 8 + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

enum Site : unsigned { kSiteFull = 20, kSiteEmpty = 21 };


__global__ void __launch_bounds__(kThreads, 1)
    pair_bias_project_kernel(const __grid_constant__ CUtensorMap tm_pair,
                             const float *__restrict__ W, float *__restrict__ bias,
                             long long n_cells, unsigned *err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *ring = smem_raw + pad;
  float *w_s = reinterpret_cast<float *>(ring + kStages * kChunkBytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(w_s + kCp * kH);
  uint64_t *empty = full + kStages;
  int *abort_flag = reinterpret_cast<int *>(empty + kStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < kCp * kH; i += kThreads) w_s[i] = __ldg(W + i);
  __syncthreads();
  volatile int *abort = abort_flag;
  const long long n_chunks = (n_cells + kChunkCells - 1) / kChunkCells;

  if (warp == kConsumerWarps) {
    // Producer: one lane issues four 32-channel boxes per chunk.  Rows past
    // the last cell are filled with zeros and their results never stored.
    if (lane == 0) {
      prefetch_tensormap(&tm_pair);
      const uint64_t pol = l2_policy_evict_first();
      uint32_t it = 0;
      for (long long ch = blockIdx.x; ch < n_chunks; ch += gridDim.x, ++it) {
        const uint32_t slot = it % kStages, ph = (it / kStages) & 1u;
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort, err, kSiteEmpty)) break;
        mbar_arrive_expect_tx(&full[slot], kChunkBytes);
        const int row = static_cast<int>(ch * kChunkCells);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_load_2d(ring + slot * kChunkBytes + q * kBoxBytes, &tm_pair, &full[slot], 32 * q,
                      row, pol);
      }
      // Every copy this thread started must land before the CTA exits.
      const uint32_t first = it > kStages ? it - kStages : 0;
      for (uint32_t i = first; i < it; ++i) {
        const uint32_t a = smem_u32(&full[i % kStages]);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_test(a, (i / kStages) & 1u))
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    }
  } else {
    // Consumer warp `warp` takes the CTA's chunks it = warp, warp + 12, ...
    const float4 *w4 = reinterpret_cast<const float4 *>(w_s);  // W[c][0..3], W[c][4..7]
    const uint32_t swz = static_cast<uint32_t>(lane & 7);
    for (uint32_t it = warp;; it += kConsumerWarps) {
      const long long ch = blockIdx.x + static_cast<long long>(it) * gridDim.x;
      if (ch >= n_chunks) break;
      const uint32_t slot = it % kStages, ph = (it / kStages) & 1u;
      const bool ok = mbar_wait(&full[slot], ph, abort, err, kSiteFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t *base = ring + slot * kChunkBytes + lane * 128;
      float2 acc[kH / 2];
#pragma unroll
      for (int hp = 0; hp < kH / 2; ++hp) acc[hp] = make_float2(0.f, 0.f);
      // Channel group g (channels 4g .. 4g+3): box g / 8, 16-byte slot
      // (g % 8) ^ (lane % 8) of this lane's 128-byte row.
#pragma unroll 8
      for (int g = 0; g < kCp / 4; ++g) {
        const float4 x = *reinterpret_cast<const float4 *>(
            base + (g >> 3) * kBoxBytes + ((static_cast<uint32_t>(g & 7) ^ swz) << 4));
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 wa = w4[(4 * g + k) * 2], wb = w4[(4 * g + k) * 2 + 1];
          const float2 xx = make_float2(xs[k], xs[k]);
          acc[0] = __ffma2_rn(xx, make_float2(wa.x, wa.y), acc[0]);
          acc[1] = __ffma2_rn(xx, make_float2(wa.z, wa.w), acc[1]);
          acc[2] = __ffma2_rn(xx, make_float2(wb.x, wb.y), acc[2]);
          acc[3] = __ffma2_rn(xx, make_float2(wb.z, wb.w), acc[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
      const long long cell = ch * kChunkCells + lane;
      if (cell < n_cells) {
#pragma unroll
        for (int hp = 0; hp < kH / 2; ++hp) {
          __stcs(bias + (2 * hp) * n_cells + cell, acc[hp].x);
          __stcs(bias + (2 * hp + 1) * n_cells + cell, acc[hp].y);
        }
      }
    }
  }
  __syncthreads();
}

}  // namespace proj

cudaError_t launch_pair_bias_project(const float *pair, const float *W, float *bias,
                                     int64_t cells, int num_sms, unsigned *err,
                                     EncodeTiledFn encode, cudaStream_t stream) {
  using namespace proj;
  static std::once_flag once[64];
  static cudaError_t once_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    once_err[dev] = cudaFuncSetAttribute(pair_bias_project_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
  });
  if (once_err[dev] != cudaSuccess) return once_err[dev];
  const long long n_cells = cells;
  // pair as a 2-D tensor: n_cells rows of 128 fp32 channels (512-byte rows).
  CUtensorMap tm;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kCp), static_cast<cuuint64_t>(n_cells)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kCellBytes)};
  const cuuint32_t box[2] = {32, kChunkCells};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(pair), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const long long n_chunks = (n_cells + kChunkCells - 1) / kChunkCells;
  const long long grid = n_chunks < num_sms ? n_chunks : num_sms;
  pair_bias_project_kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(
      tm, W, bias, n_cells, err);
  return cudaGetLastError();
}

}  // namespace ag
