// attn_noalloc.cu -- ag_attn_fwd_noalloc: the attention forward for callers
// that cannot allocate device memory.
//
// Its range schedule (contiguous runs of (pair, key tile) steps per SM pair,
// split pairs merged by a second kernel) needs scratch for the split pieces.
// Here that scratch is a file-scope device array compiled into the library,
// kept in a translation unit of its own so that the array is loaded (under
// CUDA's lazy module loading) only by processes that call this entry point.
#include <mutex>

#include "ag_internal.h"

namespace ag {
namespace {

// 148 slots of the split-pair scratch layout (kAttnSlotOutBytes +
// kAttnSlotLseBytes each): one per 2-CTA cluster of a 296-SM device.
constexpr int kStaticScratchSlots = 148;
constexpr size_t kStaticScratchBytes =
    kStaticScratchSlots * (kAttnSlotOutBytes + kAttnSlotLseBytes);
__device__ __align__(256) unsigned char g_static_attn_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {nullptr};

// Device address of g_static_attn_scratch on the current device, looked up
// once per device with that device current (host code may not use the
// symbol itself as an address: in host code it names a host-side stand-in).
ag_status static_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_attn_scratch) != cudaSuccess || !p)
      return AG_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return AG_OK;
}

}  // namespace
}  // namespace ag

extern "C" ag_status ag_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                         const float *bias, int64_t B, int64_t H, int64_t L,
                                         int64_t D, int64_t block, float cap, float *out,
                                         float *lse, void *stream) {
  // The same checks, in the same order, as ag_attn_fwd.
  const ag_status vs = ag::check_attn_sizes(B, H, L, D, block, cap);
  if (vs != AG_OK) return vs;
  if (B == 0 || L == 0) return AG_OK;
  if (!q || !k || !v || !bias || !out || !lse) return AG_ERR_NULL;
  if (!ag::aligned(q, 16) || !ag::aligned(k, 16) || !ag::aligned(v, 16) ||
      !ag::aligned(bias, 4) || !ag::aligned(out, 16) || !ag::aligned(lse, 4))
    return AG_ERR_ALIGN;
  const uint64_t P = static_cast<uint64_t>((L + block - 1) / block);
  const uint64_t qb = static_cast<uint64_t>(B) * H * L * D * 2;
  const uint64_t kb = static_cast<uint64_t>(B) * L * D * 2;
  const uint64_t bb = static_cast<uint64_t>(H) * P * P * 4;
  const uint64_t ob = static_cast<uint64_t>(B) * H * L * D * 4;
  const uint64_t lb = static_cast<uint64_t>(B) * H * L * 4;
  const void *ins[4] = {q, k, v, bias};
  const uint64_t insz[4] = {qb, kb, kb, bb};
  for (int t = 0; t < 4; ++t)
    if (ag::overlap(out, ob, ins[t], insz[t]) || ag::overlap(lse, lb, ins[t], insz[t]))
      return AG_ERR_ALIAS;
  if (ag::overlap(out, ob, lse, lb)) return AG_ERR_ALIAS;
  ag::DeviceInfo *dev = nullptr;
  ag_status st = ag::device_info(&dev);
  if (st != AG_OK) return st;
  // One scratch slot per cluster of the launch.  The grid comes from the
  // launcher's own plan for this device (one 2-CTA cluster per SM pair at
  // most, fewer for small problems); a call whose plan needs more clusters
  // than the array has slots is refused rather than given another grid.
  int clusters = 0;
  st = ag::from_cuda(ag::attn_fwd_clusters(B, L, D, cap, dev->num_sms,
                                           ag::kStaticScratchSlots + 1, &clusters));
  if (st != AG_OK) return st;
  if (clusters > ag::kStaticScratchSlots) return AG_ERR_SCRATCH;
  ag::EncodeTiledFn enc = nullptr;
  st = ag::get_encoder(&enc);
  if (st != AG_OK) return st;
  void *scratch = nullptr;
  st = ag::static_scratch(&scratch);
  if (st != AG_OK) return st;
  ag::AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.bias = bias;
  a.bias_bstride = 0;
  a.out = out;
  a.lse = lse;
  a.B = B;
  a.L = L;
  a.Lq = L;
  a.Dv = D;
  a.cap = cap;
  a.err = dev->err;
  a.num_sms = dev->num_sms;
  a.scratch = scratch;
  a.scratch_slots = ag::kStaticScratchSlots;
  a.encode = enc;
  a.stream = static_cast<cudaStream_t>(stream);
  return ag::from_cuda(ag::launch_attn_fwd(a));
}
