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
#include <string.h>

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

// 2^x evaluated on the FMA pipe instead of the MUFU unit, to share the
// exponentials of a softmax tile between the two pipes.
// Method: x = n + f with n = round-to-nearest(x) (taken from the low mantissa
// bits of x + 1.5 * 2^23) and f in [-1/2, 1/2] (Cody-Waite argument
// reduction); 2^f from the degree-3 polynomial that minimises the maximum
// relative error on [-1/2, 1/2] (Remez exchange; the coefficients and the
// bound 7.5e-5 are produced by csrc/exp2_poly_fit.py); 2^n by adding n to the
// exponent field.  Inputs below -126 (hidden keys are -inf) give exactly 0,
// as ex2.approx.ftz does, so a hidden key never carries weight; inputs must
// stay below 127.
__host__ __device__ __forceinline__ float exp2_poly(float x_in) {
  const float x = fmaxf(x_in, -126.0f);
  const float kShifter = 12582912.0f;  // 1.5 * 2^23
  const float t = x + kShifter;
  const float nf = t - kShifter;
  const float f = x - nf;
  int n;
  float p;
#if defined(__CUDA_ARCH__)
  n = __float_as_int(t) - __float_as_int(kShifter);
  p = fmaf(fmaf(fmaf(5.517166853e-02f, f, 2.426111251e-01f), f, 6.932609677e-01f), f,
           9.999280572e-01f);
  const float r = __int_as_float(__float_as_int(p) + static_cast<int>(static_cast<uint32_t>(n) << 23));
  return x_in < -126.0f ? 0.0f : r;
#else
  uint32_t tb, sb, pb;
  const float sh = kShifter;
  memcpy(&tb, &t, 4);
  memcpy(&sb, &sh, 4);
  n = static_cast<int>(tb) - static_cast<int>(sb);
  p = fmaf(fmaf(fmaf(5.517166853e-02f, f, 2.426111251e-01f), f, 6.932609677e-01f), f,
           9.999280572e-01f);
  memcpy(&pb, &p, 4);
  pb = pb + (static_cast<uint32_t>(n) << 23);
  float r;
  memcpy(&r, &pb, 4);
  return x_in < -126.0f ? 0.0f : r;
#endif
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

}  // namespace gqa
