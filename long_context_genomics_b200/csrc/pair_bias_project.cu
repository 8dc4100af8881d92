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
// persistent CTA per SM streams chunks of 64 consecutive cells (32 KB) into a
// 4-stage shared-memory ring with untiled bulk copies issued by one producer
// lane, so 128 KB per SM are in flight.  Eight consumer warps take 8 cells
// each per chunk.  Lane l reads channels 4l..4l+3 of a cell (one conflict-free
// 16-byte shared load per cell) and keeps W[4l..4l+3, 0..7] in registers
// (products for two heads per packed fp32x2 instruction); the
// 64 partial sums (8 heads x 8 cells) are reduced across the warp by a
// butterfly reduce-scatter (offsets 16, 8, 4, 2, 1), after which lane l holds
// the two finished values of head l/4 for cells 2(l%4) and 2(l%4)+1: a float2
// store, eight consecutive cells per head across the warp.
#include "ag_internal.h"
#include "sm100.cuh"

namespace ag {
namespace proj {

constexpr int kCp = 128;
constexpr int kH = 8;
constexpr int kCellBytes = kCp * 4;                  // 512
constexpr int kChunkCells = 64;
constexpr int kChunkBytes = kChunkCells * kCellBytes;  // 32 KB
constexpr int kStages = 4;
constexpr int kConsumerWarps = 8;                    // 8 cells each per chunk
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + producer warp
constexpr size_t kSmemBytes = 1024 + kStages * kChunkBytes + 2 * kStages * 8 + 16;

enum Site : unsigned { kSiteFull = 20, kSiteEmpty = 21 };

// One reduce-scatter level: lanes with bit `o` set keep the upper half of
// the first 2*n values, the others the lower half; each adds its partner's
// (two values per packed add).
template <int n>
__device__ __forceinline__ void rs_level(float (&a)[64], int o, bool upper) {
#pragma unroll
  for (int j = 0; j < n; j += 2) {
    const float2 keep = upper ? make_float2(a[j + n], a[j + n + 1])
                              : make_float2(a[j], a[j + 1]);
    const float2 send = upper ? make_float2(a[j], a[j + 1])
                              : make_float2(a[j + n], a[j + n + 1]);
    const float2 recv = make_float2(__shfl_xor_sync(0xffffffffu, send.x, o),
                                    __shfl_xor_sync(0xffffffffu, send.y, o));
    const float2 sum = __fadd2_rn(keep, recv);
    a[j] = sum.x;
    a[j + 1] = sum.y;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    pair_bias_project_kernel(const float *__restrict__ pair,
                             const float *__restrict__ W, float *__restrict__ bias,
                             long long n_cells, int vec_store, unsigned *err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *ring = smem_raw + pad;
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + kStages * kChunkBytes);
  uint64_t *empty = full + kStages;
  int *abort_flag = reinterpret_cast<int *>(empty + kStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int *abort = abort_flag;
  const long long n_chunks = (n_cells + kChunkCells - 1) / kChunkCells;

  if (warp == kConsumerWarps) {
    // Producer: one lane issues the bulk copies.
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      uint32_t it = 0;
      for (long long ch = blockIdx.x; ch < n_chunks; ch += gridDim.x, ++it) {
        const uint32_t slot = it % kStages, ph = (it / kStages) & 1u;
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort, err, kSiteEmpty)) break;
        const long long c0 = ch * kChunkCells;
        const long long nc = n_cells - c0 < kChunkCells ? n_cells - c0 : kChunkCells;
        const uint32_t bytes = static_cast<uint32_t>(nc) * kCellBytes;
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_load(ring + slot * kChunkBytes, pair + c0 * kCp, bytes, &full[slot], pol);
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
    // W[4l + i, h] for heads in pairs (2p, 2p + 1).
    float2 w[4][kH / 2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int hp = 0; hp < kH / 2; ++hp)
        w[i][hp] = make_float2(__ldg(W + (4 * lane + i) * kH + 2 * hp),
                               __ldg(W + (4 * lane + i) * kH + 2 * hp + 1));
    const int h_out = lane >> 2;       // head this lane finishes
    const int n_out = 2 * (lane & 3);  // first of its two cells
    uint32_t it = 0;
    for (long long ch = blockIdx.x; ch < n_chunks; ch += gridDim.x, ++it) {
      const uint32_t slot = it % kStages, ph = (it / kStages) & 1u;
      const bool ok = mbar_wait(&full[slot], ph, abort, err, kSiteFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      const long long c0 = ch * kChunkCells + warp * 8;  // this warp's 8 cells
      const float4 *cells = reinterpret_cast<const float4 *>(
          ring + slot * kChunkBytes + warp * 8 * kCellBytes);
      float4 x[8];
#pragma unroll
      for (int n = 0; n < 8; ++n)
        x[n] = (c0 + n < n_cells) ? cells[n * (kCp / 4) + lane]
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
      if (c0 >= n_cells) continue;
      float a[64];  // a[h * 8 + n]: the same products and order as
                    // fmaf(x.w, w3, fmaf(x.z, w2, fmaf(x.y, w1, x.x * w0))),
                    // two heads per packed instruction
#pragma unroll
      for (int hp = 0; hp < kH / 2; ++hp)
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          float2 v = __fmul2_rn(make_float2(x[n].x, x[n].x), w[0][hp]);
          v = __ffma2_rn(make_float2(x[n].y, x[n].y), w[1][hp], v);
          v = __ffma2_rn(make_float2(x[n].z, x[n].z), w[2][hp], v);
          v = __ffma2_rn(make_float2(x[n].w, x[n].w), w[3][hp], v);
          a[(2 * hp) * 8 + n] = v.x;
          a[(2 * hp + 1) * 8 + n] = v.y;
        }
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
  __syncthreads();
}

}  // namespace proj

cudaError_t launch_pair_bias_project(const float *pair, const float *W,
                                     float *bias, int64_t P, int num_sms,
                                     unsigned *err, cudaStream_t stream) {
  using namespace proj;
  static int configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(pair_bias_project_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  const long long n_cells = static_cast<long long>(P) * P;
  const long long n_chunks = (n_cells + kChunkCells - 1) / kChunkCells;
  const long long grid = n_chunks < num_sms ? n_chunks : num_sms;
  // float2 stores need an even cell count (then every head's plane starts
  // 8-byte aligned, as does every even cell inside it).
  const int vec_store = (n_cells % 2 == 0) ? 1 : 0;
  pair_bias_project_kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes,
                             stream>>>(pair, W, bias, n_cells, vec_store, err);
  return cudaGetLastError();
}

}  // namespace ag
