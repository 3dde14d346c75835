// Decode entry point that allocates nothing: its scratch is a static device
// array instead of a caller-provided workspace.
//
// Who needs it: callers that are handed device buffers for q, k, v and out by
// a host framework and have no allocator of their own to obtain a workspace
// (plugin-style interfaces), and callers that must not call cudaMalloc in a
// steady-state loop because it can synchronise the device.  Everything else
// should use gqa_forward, which also reports kernel wait timeouts and
// out-of-range lengths or page indices (gqa_device_status).
//
// It takes every problem that gqa_forward sends to the decode kernel (bf16 or
// fp16; seq_q == 1 or (heads_q / heads_kv) * seq_q <= 16; mask, causal offset,
// window, per-sequence lengths and paged caches), and fills the output as
// gqa_forward does when seq_k == 0 (zeros) or no key is visible (NaN).
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
// (with that device current) and cached per device.  Outside stream capture
// it is looked up again on every call, so that a module reloaded after a
// device reset is followed; during capture the cached address is used (the
// first call on a device must therefore come before any capture).
int scratch_address(int dev, cudaStream_t stream, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_DEVICE;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
    cudaGetLastError();
    cs = cudaStreamCaptureStatusActive;  // unknown: do not call into the module
  }
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (cs == cudaStreamCaptureStatusNone || p == nullptr) {
    if (cs != cudaStreamCaptureStatusNone) return GQA_ERR_CUDA;  // first call inside a capture
    std::lock_guard<std::mutex> lock(g_setup_mu);
    void* fresh = nullptr;
    if (cudaGetSymbolAddress(&fresh, g_decode_scratch) != cudaSuccess || fresh == nullptr) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    g_scratch_addr[dev].store(fresh, std::memory_order_release);
    p = fresh;
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
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  // No key at all, or none visible: the output is filled as gqa_forward
  // fills it (zeros, or NaN), which needs no scratch.
  if (plan.kernel == GQA_KERNEL_ZERO || plan.kernel == GQA_KERNEL_NAN) {
    if (out == nullptr) return GQA_ERR_NULL;
    return launch_zero(*p, out, stream, plan.kernel == GQA_KERNEL_NAN);
  }
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
  const int src = scratch_address(dev, stream, &scratch);
  if (src != GQA_OK) return src;
  uint8_t* ws = static_cast<uint8_t*>(scratch);

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
