// zo_probe_losses_static: the fp32 probe-loss path without a context and
// without device allocation.  Its scratch - the per-row loss sums that the
// forward kernel writes and the reduction reads, plus the error word the
// kernels latch into - is a file-scope device array.  Host code cannot use
// the array's name as a device address, so its address is resolved here, once
// per device, with cudaGetSymbolAddress while that device is current.
#include <math.h>

#include <mutex>

#include "zo_internal.h"

namespace {

constexpr int kMaxDevices = 64;

// [0, ZO_STATIC_SCRATCH_FLOATS): per-row loss sums; then one error word.
static __device__ __align__(256) float g_static_scratch[ZO_STATIC_SCRATCH_FLOATS + 64];

std::mutex g_mu;
float* g_scratch_dev[kMaxDevices] = {};
int g_major[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

// Resolve the scratch address and device properties for the current device.
int resolve(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_dev[dev]) return ZO_OK;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ZO_ERR_NO_DEVICE;
  g_major[dev] = prop.major;
  g_sms[dev] = prop.multiProcessorCount;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return ZO_ERR_CUDA;
  }
  g_scratch_dev[dev] = static_cast<float*>(p);
  return ZO_OK;
}

}  // namespace

extern "C" int zo_probe_losses_static(const zo_model_spec* spec, const float* theta,
                                      uint64_t seed, int32_t n_pert, float eps,
                                      const int32_t* tokens, const int32_t* targets,
                                      int32_t batch, int32_t seq, float* loss_plus,
                                      float* loss_minus, void* stream) {
  if (!spec || !theta || !tokens || !targets || !loss_plus || !loss_minus)
    return ZO_ERR_INVALID_ARG;
  const zo_model_spec s0 = *spec;
  if (s0.vocab < 2 || s0.embed < 1 || s0.hidden < 1 || s0.layers < 1 ||
      s0.layers > zo::kMaxLayersHost || s0.dtype != ZO_DTYPE_FP32)
    return ZO_ERR_INVALID_ARG;
  if (n_pert < 1 || batch < 1 || seq < 1 || !(eps > 0.f) || !isfinite(eps))
    return ZO_ERR_INVALID_ARG;
  if ((int64_t)2 * n_pert * batch > ZO_STATIC_SCRATCH_FLOATS) return ZO_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZO_ERR_NO_DEVICE;
  const int rc = resolve(dev);
  if (rc != ZO_OK) return rc;
  if (g_major[dev] != 10) return ZO_ERR_NO_DEVICE;

  // a context on the stack that points at the static scratch
  zo_ctx c;
  c.spec = s0;
  c.spec.max_batch = batch;
  c.spec.max_seq = seq;
  c.spec.chunk = n_pert;
  c.device = dev;
  c.sm_count = g_sms[dev];
  zo::layout_of(c.spec, c.seg);
  int bb = 8;
  while (bb > 1 && (bb / 2 >= batch || zo::fp32_smem_bytes(c.spec, bb, c.seg.d_pad) > 200 * 1024))
    bb /= 2;
  if (zo::fp32_smem_bytes(c.spec, bb, c.seg.d_pad) > 200 * 1024) return ZO_ERR_UNSUPPORTED;
  c.fp32_bb = bb;
  c.fp32_smem = zo::fp32_smem_bytes(c.spec, bb, c.seg.d_pad);
  c.chunk = n_pert;
  c.rowloss = g_scratch_dev[dev];
  c.err = reinterpret_cast<unsigned*>(g_scratch_dev[dev] + ZO_STATIC_SCRATCH_FLOATS);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // every row sum is written by the forward before the reduction reads it,
  // so nothing in the array needs clearing between calls
  if (zo::launch_fp32_forward(&c, theta, seed, 0, n_pert, eps, tokens, targets, batch, seq, st) !=
      cudaSuccess)
    return ZO_ERR_CUDA;
  if (zo::launch_reduce_losses(&c, targets, batch, seq, 0, n_pert, loss_plus, loss_minus, nullptr,
                               st) != cudaSuccess)
    return ZO_ERR_CUDA;
  return ZO_OK;
}
