// sla_classify_noalloc: classification for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc at the point where they classify: code
// running while a CUDA graph is being captured, allocator-less embedded or
// real-time runtimes, and host frameworks whose memory is owned by a pool
// they may not grow.  sla_classify needs a caller-provided workspace for its
// pooled Q and K; this variant keeps that scratch in a fixed array compiled
// into the library instead, so the caller passes only the inputs and the
// mask outputs.
//
// The scratch array lives in device global memory of every GPU that loads
// the library, for the life of the process.  Host code cannot use the
// array's name as a device address (in host code it names a host-side
// stand-in), so the device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device, and kept for the life of the process (it is stale after a
// cudaDeviceReset() of that device).  All calls share the one array: calls
// whose work overlaps on the GPU (different streams, or different host
// threads) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "sla.h"
#include "sla_internal.h"

namespace {

// Pooled Q then pooled K, fp32 [B*H, T, d] each: 16 MiB in total, enough for
// B*H*T*d <= 2M (e.g. 12 heads x 1182 blocks x d=128).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_classify_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device (set up on the
// first call for that device).
sla_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SLA_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_classify_scratch) != cudaSuccess || !p) return SLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SLA_OK;
}

}  // namespace

using namespace sla;

extern "C" sla_status sla_classify_noalloc(const sla_shape* shape, const void* q, const void* k,
                                           const sla_mask* mask, void* stream) {
  if (!shape || !q || !k || !mask) return SLA_ERR_INVALID_ARG;
  sla_sizes sz;
  sla_status st = sla_query_sizes(shape, &sz);
  if (st != SLA_OK) return st;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(k) & 15u))
    return SLA_ERR_INVALID_ARG;
  if (!mask->cls || !mask->marg_bits || !mask->crit_col_ptr ||
      (sz.n_crit > 0 && (!mask->crit_idx || !mask->crit_col_idx)))
    return SLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(mask->marg_bits) & 15u) ||
      (mask->crit_idx && (reinterpret_cast<uintptr_t>(mask->crit_idx) & 15u)))
    return SLA_ERR_INVALID_ARG;
  const size_t bh = size_t(shape->B) * size_t(shape->H);
  const size_t pooled = bh * size_t(sz.T) * size_t(shape->d) * sizeof(float);
  if (2 * pooled > kNoAllocScratchBytes) return SLA_ERR_WORKSPACE;  // beyond the fixed scratch

  void* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != SLA_OK) return st;
  float* qbar = static_cast<float*>(scratch);
  float* kbar = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + pooled);

  Problem p;
  p.B = shape->B;
  p.H = shape->H;
  p.BH = int(bh);
  p.N = shape->N;
  p.d = shape->d;
  p.T = sz.T;
  p.Tp = pad128(sz.T);
  p.nv = shape->n_valid != 0 ? shape->n_valid : shape->N;  // validated by sla_query_sizes
  p.n_crit = sz.n_crit;
  p.n_negl = sz.n_negl;
  p.scale = shape->softmax_scale > 0.f ? shape->softmax_scale : 1.0f / sqrtf(float(shape->d));
  p.scale_log2 = p.scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Every scratch element the classifier reads is written by the pooling
  // kernel first, so nothing needs clearing between calls.
  // the same named launches as sla_classify, so the opt-in profiler counts
  // them and a failed launch is attributed to its kernel
  if (launch_named("pool", s, [&] { return launch_pool(p, q, k, qbar, kbar, s); }) != cudaSuccess)
    return SLA_ERR_CUDA;
  if (launch_named("classify", s, [&] {
        return launch_classify(p, qbar, kbar, nullptr, mask->pooled_logits, mask->cls,
                               mask->crit_idx, mask->marg_bits, s);
      }) != cudaSuccess)
    return SLA_ERR_CUDA;
  if (launch_named("crit_csr", s, [&] {
        return launch_crit_csr(p, mask->cls, mask->crit_col_ptr, mask->crit_col_idx, s);
      }) != cudaSuccess)
    return SLA_ERR_CUDA;
  return SLA_OK;
}
