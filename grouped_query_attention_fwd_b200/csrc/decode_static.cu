// Decode entry point that allocates nothing: its scratch is a static device
// array instead of a caller-provided workspace.
//
// Who needs it: callers that are handed device buffers for q, k, v and out by
// a host framework and have no allocator of their own to obtain a workspace
// (plugin-style interfaces), and callers that must not call cudaMalloc in a
// steady-state loop because it can synchronise the device.  Everything else
// should use gqa_forward, which also reports kernel wait timeouts.
//
// The array below belongs to the library for the life of the process on every
// GPU that loads it.  All calls share it: each call clears the part that must
// start at zero (error word and split-merge counters) on its own stream before
// its kernel runs, the partial-result area keeps whatever the last call left,
// and calls that overlap on the GPU race on it.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "gqa.h"
#include "kernels.h"

namespace gqa {
namespace {

static_assert(GQA_STATIC_SCRATCH_BYTES % 256 == 0, "scratch size must be a multiple of 256");

__device__ __align__(256) uint8_t g_decode_scratch[GQA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];
std::mutex g_setup_mu;

// Device address of g_decode_scratch on the current device.  In host code
// the symbol's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_DEVICE;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return GQA_ERR_CUDA;
      }
      g_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return GQA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace gqa

using namespace gqa;

extern "C" GQA_API int gqa_forward_decode_noalloc(const gqa_problem* p, const void* q,
                                                  const void* k, const void* v,
                                                  const uint8_t* mask, void* out,
                                                  void* stream_ptr) {
  gqa_plan plan;
  const int rc = gqa_query(p, 0, &plan);  // validates, plans for the current device
  if (rc != GQA_OK) return rc;
  if (plan.kernel == GQA_KERNEL_NONE) return GQA_OK;
  if (plan.kernel != GQA_KERNEL_DECODE) return GQA_ERR_UNSUPPORTED;
  if (plan.workspace_bytes > static_cast<int64_t>(GQA_STATIC_SCRATCH_BYTES))
    return GQA_ERR_SCRATCH_LIMIT;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return GQA_ERR_NULL;
  if (p->has_mask && mask == nullptr) return GQA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GQA_ERR_LAYOUT;

  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  void* scratch = nullptr;
  const int src = scratch_address(dev, &scratch);
  if (src != GQA_OK) return src;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

  const DecodeShape s = plan_decode(*p, sms);
  // Error word and ticket counters must start at zero; partials need not.
  // Nothing reports a wait that gave up here, so the counters are zeroed on
  // every call instead of trusting the last one to have left them zero.
  const int64_t zero_end = s.counters_offset + s.groups * 4;
  if (cudaMemsetAsync(ws, 0, static_cast<size_t>(zero_end), stream) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  CUtensorMap tmk, tmv;
  int erc = encode_decode_kv_map(&tmk, k, *p, p->k_stride);
  if (erc != GQA_OK) return erc;
  erc = encode_decode_kv_map(&tmv, v, *p, p->v_stride);
  if (erc != GQA_OK) return erc;

  const DecodeArgs a = make_decode_args(*p, s, q, mask, out, ws);
  return launch_decode(*p, s, a, tmk, tmv, stream);
}
