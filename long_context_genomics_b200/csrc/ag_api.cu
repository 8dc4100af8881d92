// ag_api.cu -- the extern "C" entry points declared in include/ag.h.
//
// Validation happens on the host before anything is launched; a failed
// check returns its status and writes nothing.  The compute itself is in
// attn_fwd_sm100.cu and pair_bias_project.cu.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/ag.h"
#include "ag_internal.h"
#include "sm100.cuh"

namespace ag {

// One error word per device (each device that loads the library holds its
// own copy of this variable).
__device__ unsigned g_device_error_word;

namespace {

constexpr int kMaxDevices = 64;

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

}  // namespace

// Per-device set-up, done once with that device current.
ag_status device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess)
      return AG_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.num_sms = sms;
    if (d.sm100) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess)
        return AG_ERR_CUDA;
      d.err = static_cast<unsigned *>(p);
    }
    d.ready = true;
  }
  if (!d.sm100) return AG_ERR_UNSUPPORTED;
  *out = &d;
  return AG_OK;
}

ag_status get_encoder(EncodeTiledFn *fn) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_encode) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return AG_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = g_encode;
  return AG_OK;
}

bool aligned(const void *p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// [a, a + na) and [b, b + nb) overlap (byte ranges).
bool overlap(const void *a, uint64_t na, const void *b, uint64_t nb) {
  if (na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a);
  const uintptr_t y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// A failure from an earlier asynchronous launch is sticky; it is reported
// here rather than attributed to the next call.
ag_status from_cuda(cudaError_t e) { return e == cudaSuccess ? AG_OK : AG_ERR_CUDA; }

namespace {

__global__ void wait_timeout_probe_kernel(uint64_t timeout_ns, unsigned *err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing arrives on `bar`: the wait must run out and report site 255.
    (void)mbar_wait(&bar, 0, &abort_flag, err, 255u, timeout_ns);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout_probe(uint64_t timeout_ns, unsigned *err,
                                      cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(timeout_ns, err);
  return cudaGetLastError();
}

}  // namespace ag

extern "C" {

const char *ag_status_string(int s) {
  switch (s) {
    case AG_OK: return "AG_OK";
    case AG_ERR_NULL: return "AG_ERR_NULL: a required pointer is NULL";
    case AG_ERR_SHAPE: return "AG_ERR_SHAPE: negative or inconsistent size";
    case AG_ERR_ALIGN: return "AG_ERR_ALIGN: pointer not aligned as required";
    case AG_ERR_UNSUPPORTED:
      return "AG_ERR_UNSUPPORTED: sizes or device not supported by the kernels";
    case AG_ERR_VALUE: return "AG_ERR_VALUE: scalar argument out of range";
    case AG_ERR_CUDA: return "AG_ERR_CUDA: a CUDA call failed";
    case AG_ERR_ALIAS: return "AG_ERR_ALIAS: an output overlaps an input";
    case AG_ERR_DEVICE: return "AG_ERR_DEVICE: the device error word is set";
    case AG_ERR_SCRATCH:
      return "AG_ERR_SCRATCH: the call needs more scratch than the static buffer holds";
    default: return "unknown ag_status";
  }
}

int ag_version(void) { return 10000 * 0 + 100 * 1 + 0; }

ag_status ag_pair_bias_project(const float *pair, const float *W, float *bias,
                               int64_t P, int64_t Cp, int64_t H, void *stream) {
  return ag_pair_bias_project_rows(pair, W, bias, P, P, Cp, H, stream);
}

ag_status ag_pair_bias_project_rows(const float *pair, const float *W, float *bias,
                                    int64_t R, int64_t P, int64_t Cp, int64_t H,
                                    void *stream) {
  if (R < 0 || P < 0 || Cp <= 0 || H <= 0) return AG_ERR_SHAPE;
  if (Cp != 128 || H != 8 || P > 4096 || R > 4096) return AG_ERR_UNSUPPORTED;
  if (P == 0 || R == 0) return AG_OK;
  if (!pair || !W || !bias) return AG_ERR_NULL;
  if (!ag::aligned(pair, 16) || !ag::aligned(W, 4) || !ag::aligned(bias, 8))
    return AG_ERR_ALIGN;
  const uint64_t cells = static_cast<uint64_t>(R) * P;
  const uint64_t bias_bytes = cells * H * 4;
  if (ag::overlap(bias, bias_bytes, pair, cells * Cp * 4) ||
      ag::overlap(bias, bias_bytes, W, static_cast<uint64_t>(Cp) * H * 4))
    return AG_ERR_ALIAS;
  ag::DeviceInfo *dev = nullptr;
  ag_status st = ag::device_info(&dev);
  if (st != AG_OK) return st;
  ag::EncodeTiledFn enc = nullptr;
  st = ag::get_encoder(&enc);
  if (st != AG_OK) return st;
  return ag::from_cuda(ag::launch_pair_bias_project(
      pair, W, bias, static_cast<int64_t>(cells), dev->num_sms, dev->err, enc,
      static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace ag {
// Size and value checks shared by the attention entry points, in order:
// shapes, then cap, then what the kernels support (including the work-step
// bound: pairs of query tiles x key tiles must stay below 2^30).
ag_status check_attn_sizes(int64_t B, int64_t H, int64_t L, int64_t D, int64_t block,
                           float cap) {
  if (B < 0 || H <= 0 || L < 0 || D <= 0 || block <= 0) return AG_ERR_SHAPE;
  if (std::isnan(cap) || !(cap > 0.0f)) return AG_ERR_VALUE;
  if (H != 8 || D != 128 || block != 16 || L > 65536) return AG_ERR_UNSUPPORTED;
  if (B > 0 && L > 0 && B * L > (int64_t(1) << 28)) return AG_ERR_UNSUPPORTED;
  if (B > 0 && L > 0 && attn_work_steps(B, L) > (int64_t(1) << 30))
    return AG_ERR_UNSUPPORTED;
  return AG_OK;
}

// The value width and the per-item bias stride (after check_attn_sizes), for
// a bias of `rows` rows of P cells per head.
static ag_status check_value_width_and_bias_stride(int64_t B, int64_t H, int64_t rows,
                                                   int64_t P, int64_t Dv,
                                                   int64_t bias_batch_stride) {
  if (Dv <= 0) return AG_ERR_SHAPE;
  if (Dv != 128 && Dv != 192) return AG_ERR_UNSUPPORTED;
  const int64_t per_item = H * rows * P;
  if (bias_batch_stride < 0 || (bias_batch_stride > 0 && bias_batch_stride < per_item))
    return AG_ERR_SHAPE;
  // The items' bias span, (B - 1) * stride + H * rows * P floats, must stay far
  // below 2^63 bytes so that the alias check and the kernel's offsets are exact.
  constexpr int64_t kMaxBiasSpan = int64_t(1) << 56;
  if (B > 1 && bias_batch_stride > (kMaxBiasSpan - per_item) / (B - 1))
    return AG_ERR_SHAPE;
  return AG_OK;
}
}  // namespace ag

extern "C" {

ag_status ag_attn_fwd(const void *q, const void *k, const void *v,
                      const float *bias, int64_t B, int64_t H, int64_t L,
                      int64_t D, int64_t block, float cap, float *out,
                      float *lse, void *stream) {
  return ag_attn_fwd_strided_bias(q, k, v, bias, 0, B, H, L, D, block, cap, out,
                                  lse, stream);
}

ag_status ag_attn_fwd_strided_bias(const void *q, const void *k, const void *v,
                                   const float *bias, int64_t bias_batch_stride,
                                   int64_t B, int64_t H, int64_t L, int64_t D,
                                   int64_t block, float cap, float *out,
                                   float *lse, void *stream) {
  return ag_attn_fwd_ex(q, k, v, bias, bias_batch_stride, B, H, L, D, D, block, cap,
                        out, lse, stream);
}

ag_status ag_attn_fwd_ex(const void *q, const void *k, const void *v,
                         const float *bias, int64_t bias_batch_stride, int64_t B,
                         int64_t H, int64_t L, int64_t D, int64_t Dv, int64_t block,
                         float cap, float *out, float *lse, void *stream) {
  return ag_attn_fwd_query_slab(q, k, v, bias, bias_batch_stride, B, H, L, L, D, Dv, block,
                                cap, out, lse, stream);
}

ag_status ag_attn_fwd_query_slab(const void *q, const void *k, const void *v,
                                 const float *bias, int64_t bias_batch_stride, int64_t B,
                                 int64_t H, int64_t Lq, int64_t L, int64_t D, int64_t Dv,
                                 int64_t block, float cap, float *out, float *lse,
                                 void *stream) {
  const ag_status vs = ag::check_attn_sizes(B, H, L, D, block, cap);
  if (vs != AG_OK) return vs;
  if (Lq < 0) return AG_ERR_SHAPE;
  if (Lq > 65536 || (B > 0 && Lq > 0 && B * Lq > (int64_t(1) << 28)) ||
      (B > 0 && Lq > 0 && L > 0 && ag::attn_work_steps(B, Lq, L) > (int64_t(1) << 30)))
    return AG_ERR_UNSUPPORTED;
  const int64_t P = (L + block - 1) / block;
  const int64_t rows = (Lq + block - 1) / block;
  const ag_status ws =
      ag::check_value_width_and_bias_stride(B, H, rows, P, Dv, bias_batch_stride);
  if (ws != AG_OK) return ws;
  if (B == 0 || L == 0 || Lq == 0) return AG_OK;
  if (!q || !k || !v || !bias || !out || !lse) return AG_ERR_NULL;
  if (!ag::aligned(q, 16) || !ag::aligned(k, 16) || !ag::aligned(v, 16) ||
      !ag::aligned(bias, 4) || !ag::aligned(out, 16) || !ag::aligned(lse, 4))
    return AG_ERR_ALIGN;
  const uint64_t qb = static_cast<uint64_t>(B) * H * Lq * D * 2;
  const uint64_t kb = static_cast<uint64_t>(B) * L * D * 2;
  const uint64_t vb = static_cast<uint64_t>(B) * L * Dv * 2;
  const uint64_t bb = (static_cast<uint64_t>(B - 1) * bias_batch_stride +
                       static_cast<uint64_t>(H) * rows * P) * 4;
  const uint64_t ob = static_cast<uint64_t>(B) * H * Lq * Dv * 4;
  const uint64_t lb = static_cast<uint64_t>(B) * H * Lq * 4;
  const void *ins[4] = {q, k, v, bias};
  const uint64_t insz[4] = {qb, kb, vb, bb};
  for (int t = 0; t < 4; ++t)
    if (ag::overlap(out, ob, ins[t], insz[t]) || ag::overlap(lse, lb, ins[t], insz[t]))
      return AG_ERR_ALIAS;
  if (ag::overlap(out, ob, lse, lb)) return AG_ERR_ALIAS;
  ag::DeviceInfo *dev = nullptr;
  ag_status st = ag::device_info(&dev);
  if (st != AG_OK) return st;
  ag::EncodeTiledFn enc = nullptr;
  st = ag::get_encoder(&enc);
  if (st != AG_OK) return st;
  ag::AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.bias = bias;
  a.bias_bstride = bias_batch_stride;
  a.out = out;
  a.lse = lse;
  a.B = B;
  a.L = L;
  a.Lq = Lq;
  a.Dv = Dv;
  a.cap = cap;
  a.err = dev->err;
  a.num_sms = dev->num_sms;
  a.scratch = nullptr;  // whole pairs or two launches: no scratch
  a.scratch_slots = 0;
  a.encode = enc;
  a.stream = static_cast<cudaStream_t>(stream);
  return ag::from_cuda(ag::launch_attn_fwd(a));
}

ag_status ag_attn_fwd_launch_count(int64_t B, int64_t H, int64_t L, int64_t D,
                                   int64_t block, float cap, int *count) {
  if (!count) return AG_ERR_NULL;
  const ag_status vs = ag::check_attn_sizes(B, H, L, D, block, cap);
  if (vs != AG_OK) return vs;
  if (B == 0 || L == 0) {
    *count = 0;
    return AG_OK;
  }
  ag::DeviceInfo *dev = nullptr;
  ag_status st = ag::device_info(&dev);
  if (st != AG_OK) return st;
  int n = 0;
  st = ag::from_cuda(ag::attn_fwd_kernel_count(B, L, L, D, cap, dev->num_sms, 0, &n));
  if (st != AG_OK) return st;
  *count = n;
  return AG_OK;
}

ag_status ag_attn_fwd_schedule(int64_t B, int64_t L, int sm_pairs, int with_scratch,
                               int *sched, int *clusters, int *tail_clusters, int *whole,
                               int *n_whole, int *split_at, int *wb, int *fb) {
  if (!sched || !clusters || !tail_clusters || !whole || !n_whole || !split_at || !wb || !fb)
    return AG_ERR_NULL;
  const ag_status vs = ag::check_attn_sizes(B, 8, L, 128, 16, 5.0f);
  if (vs != AG_OK) return vs;
  if (B == 0 || L == 0 || sm_pairs < 1) return AG_ERR_SHAPE;
  ag::attn_fwd_schedule(B, L, sm_pairs, with_scratch ? sm_pairs : 0, sched, clusters,
                        tail_clusters, whole, n_whole, split_at, wb, fb);
  return AG_OK;
}

ag_status ag_attn_bwd(const void *q, const void *k, const void *v, const float *bias,
                      int64_t bias_batch_stride, const float *lse, const float *dout,
                      int64_t B, int64_t H, int64_t L, int64_t D, int64_t Dv,
                      int64_t block, float cap, float *dq, float *dk, float *dv,
                      float *dbias, float *delta, void *stream) {
  ag_status st = ag::check_attn_sizes(B, H, L, D, block, cap);
  if (st != AG_OK) return st;
  const int64_t Pc = (L + block - 1) / block;
  st = ag::check_value_width_and_bias_stride(B, H, Pc, Pc, Dv, bias_batch_stride);
  if (st != AG_OK) return st;
  if (B == 0 || L == 0) return AG_OK;
  if (!q || !k || !v || !bias || !lse || !dout || !dq || !dk || !dv || !dbias || !delta)
    return AG_ERR_NULL;
  if (!ag::aligned(q, 2) || !ag::aligned(k, 2) || !ag::aligned(v, 2) ||
      !ag::aligned(bias, 4) || !ag::aligned(lse, 4) || !ag::aligned(dout, 4) ||
      !ag::aligned(dq, 4) || !ag::aligned(dk, 4) || !ag::aligned(dv, 4) ||
      !ag::aligned(dbias, 4) || !ag::aligned(delta, 4))
    return AG_ERR_ALIGN;
  const uint64_t P = static_cast<uint64_t>((L + block - 1) / block);
  const uint64_t rows = static_cast<uint64_t>(B) * H * L;
  const uint64_t bias_bytes =
      (static_cast<uint64_t>(B - 1) * bias_batch_stride + H * P * P) * 4;
  const uint64_t bias_span = bias_batch_stride ? bias_bytes : H * P * P * 4;
  const void *ins[6] = {q, k, v, bias, lse, dout};
  const uint64_t insz[6] = {rows * D * 2, static_cast<uint64_t>(B) * L * D * 2,
                            static_cast<uint64_t>(B) * L * Dv * 2, bias_span, rows * 4,
                            rows * Dv * 4};
  const void *outs[5] = {dq, dk, dv, dbias, delta};
  const uint64_t outsz[5] = {rows * D * 4, static_cast<uint64_t>(B) * L * D * 4,
                             static_cast<uint64_t>(B) * L * Dv * 4, bias_span, rows * 4};
  for (int o = 0; o < 5; ++o) {
    for (int t = 0; t < 6; ++t)
      if (ag::overlap(outs[o], outsz[o], ins[t], insz[t])) return AG_ERR_ALIAS;
    for (int u = o + 1; u < 5; ++u)
      if (ag::overlap(outs[o], outsz[o], outs[u], outsz[u])) return AG_ERR_ALIAS;
  }
  // The tensor-core path (value width 128) reads q, k, v, dout and dq's
  // staging planes with TMA or 16-byte vectors.
  if (Dv == 128 && (!ag::aligned(q, 16) || !ag::aligned(k, 16) || !ag::aligned(v, 16) ||
                    !ag::aligned(dout, 16) || !ag::aligned(dq, 16)))
    return AG_ERR_ALIGN;
  ag::DeviceInfo *dev = nullptr;
  st = ag::device_info(&dev);
  if (st != AG_OK) return st;
  ag::AttnBwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.bias = bias;
  a.bias_bstride = bias_batch_stride;
  a.lse = lse;
  a.dout = dout;
  a.delta = delta;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dbias = dbias;
  a.B = B;
  a.H = H;
  a.L = L;
  a.Dv = Dv;
  a.cap = cap;
  a.stream = static_cast<cudaStream_t>(stream);
  if (ag::attn_bwd_tc_supported(a)) {
    ag::EncodeTiledFn enc = nullptr;
    st = ag::get_encoder(&enc);
    if (st != AG_OK) return st;
    return ag::from_cuda(ag::launch_attn_bwd_tc(a, dev->num_sms, dev->err, enc));
  }
  return ag::from_cuda(ag::launch_attn_bwd(a));
}

ag_status ag_attn_bwd_launch_count(int64_t Dv, int *count) {
  if (!count) return AG_ERR_NULL;
  if (Dv <= 0) return AG_ERR_SHAPE;
  if (Dv != 128 && Dv != 192) return AG_ERR_UNSUPPORTED;
  *count = Dv == 128 ? 4 : ag::attn_bwd_kernel_count();
  return AG_OK;
}

ag_status ag_device_error(int device, int *code, int clear) {
  if (!code) return AG_ERR_NULL;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return AG_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return AG_ERR_CUDA;
  ag::DeviceInfo *dev = nullptr;
  ag_status st = ag::device_info(&dev);
  unsigned word = 0;
  if (st == AG_OK) {
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(&word, dev->err, sizeof(word), cudaMemcpyDeviceToHost) !=
            cudaSuccess) {
      st = AG_ERR_CUDA;
    } else if (clear && word != 0) {
      const unsigned zero = 0;
      if (cudaMemcpy(dev->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) !=
          cudaSuccess)
        st = AG_ERR_CUDA;
    }
  }
  cudaSetDevice(prev);
  if (st != AG_OK) return st;
  *code = static_cast<int>(word);
  return word ? AG_ERR_DEVICE : AG_OK;
}

ag_status ag_debug_wait_timeout(uint64_t timeout_ns, void *stream) {
  if (timeout_ns < 1000000ull || timeout_ns > 10000000000ull) return AG_ERR_VALUE;
  ag::DeviceInfo *dev = nullptr;
  ag_status st = ag::device_info(&dev);
  if (st != AG_OK) return st;
  return ag::from_cuda(ag::launch_wait_timeout_probe(
      timeout_ns, dev->err, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
