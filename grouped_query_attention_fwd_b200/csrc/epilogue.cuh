// Shared mask / scale / fp32-accumulation epilogue of every kernel.
//
// Scores are kept in the base-2 domain: t = (q.k) * scale * log2(e), so that
// exp(s - m) = exp2(t - m2).  Hidden keys get t = -inf.  The running maximum
// used as the exponent reference is replaced by 0 while it is still -inf (no
// visible key yet), so that exp2(-inf - ref) = 0 instead of NaN; a row that
// never sees a visible key ends with l = 0 and output 0/0 = NaN, the softmax
// of an all -inf row ("28. Grouped-Query Attention (GQA)", "Reference
// solution": masked_fill with -inf, then softmax).
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

namespace gqa {

constexpr float kLog2e = 1.4426950408889634f;

// Key j visible from query i under the optional bool mask (causal and window
// limits are applied by each kernel as a key range).
__device__ __forceinline__ bool mask_allows(const uint8_t* mask_row, int64_t j) {
  return mask_row == nullptr || mask_row[j] != 0;
}

// Exponent reference for a running maximum that may still be -inf.
__device__ __forceinline__ float exp_ref(float m) { return m == -INFINITY ? 0.0f : m; }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

}  // namespace gqa
