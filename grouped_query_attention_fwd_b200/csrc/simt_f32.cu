// fp32 path on the CUDA cores, plus the zero fill used when seq_k == 0.
//
// The tensor cores have no fp32-operand mode with fp32 accuracy (tf32 keeps
// 10 mantissa bits), so single precision runs here: one warp per output row
// (b, h, i), lanes split the head dimension, online softmax in fp32 over the
// keys of kv head h / g.  This path exists for exact-precision callers and the
// small fp32 problems; the bf16 kernels carry the throughput.
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int kMaxDPerLane = 8;  // head_dim <= 256

__global__ void __launch_bounds__(256)
    gqa_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                   const float* __restrict__ v, const uint8_t* __restrict__ mask,
                   float* __restrict__ out, int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq,
                   int64_t Sk, int64_t D, int64_t qs0, int64_t qs1, int64_t qs2, int64_t ks0,
                   int64_t ks1, int64_t ks2, int64_t vs0, int64_t vs1, int64_t vs2, int64_t os0,
                   int64_t os1, int64_t os2, int64_t ms0, int64_t ms1, int causal,
                   int64_t causal_offset, int64_t window, const int32_t* __restrict__ lens,
                   const int32_t* __restrict__ bt, int64_t bt_stride, int64_t page_size,
                   int64_t num_pages, uint32_t* __restrict__ err, float scale_log2) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= B * Hq * Sq) return;
  const int64_t i = row % Sq;
  const int64_t h = (row / Sq) % Hq;
  const int64_t b = row / (Sq * Hq);
  const int64_t g = Hq / Hkv;
  const int64_t kv = h / g;

  const float* qr = q + b * qs0 + h * qs1 + i * qs2;
  // Contiguous: key j of entry b at b * s0 + kv * s1 + j * s2.  Paged: at
  // page * s0 + kv * s1 + (j % page_size) * s2, page from the block table.
  const float* kb = k + (bt ? 0 : b * ks0) + kv * ks1;
  const float* vb = v + (bt ? 0 : b * vs0) + kv * vs1;
  const uint8_t* mrow = mask ? mask + b * ms0 + i * ms1 : nullptr;

  float qv[kMaxDPerLane], acc[kMaxDPerLane];
#pragma unroll
  for (int e = 0; e < kMaxDPerLane; ++e) {
    const int64_t d = lane + 32 * e;
    qv[e] = d < D ? qr[d] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  // Entry b holds len keys; its diagonal sits at i + off.
  int64_t len = Sk;
  if (lens != nullptr) {
    len = lens[b];
    if (len < 0 || len > Sk) {
      if (h == 0 && i == 0 && lane == 0) atomicOr(err, kErrKvLength);
      len = len < 0 ? 0 : Sk;
    }
  }
  const int64_t off = causal_offset + (len - Sk);
  // Keys [jbeg, jend) pass the length, causal and window rules; the mask is per key.
  int64_t jend = len, jbeg = 0;
  if (causal) {
    jend = i + off + 1 < len ? i + off + 1 : len;
    if (window > 0 && i + off - window + 1 > 0) jbeg = i + off - window + 1;
  }
  for (int64_t j = jbeg; j < jend; ++j) {
    if (mrow != nullptr && mrow[j] == 0) continue;
    int64_t koff = j * ks2, voff = j * vs2;
    if (bt != nullptr) {
      const int64_t page = bt[b * bt_stride + j / page_size];
      if (page < 0 || page >= num_pages) {
        if (lane == 0) atomicOr(err, kErrPage);
        continue;  // the result is undefined once this is reported; skip the key
      }
      koff = page * ks0 + (j % page_size) * ks2;
      voff = page * vs0 + (j % page_size) * vs2;
    }
    const float* kr = kb + koff;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxDPerLane; ++e) {
      const int64_t d = lane + 32 * e;
      if (d < D) dot = fmaf(qv[e], kr[d], dot);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float t = dot * scale_log2;
    const float m_new = fmaxf(m, t);
    const float alpha = exp2f(m - m_new);
    const float p = exp2f(t - m_new);
    l = l * alpha + p;
    const float* vr = vb + voff;
#pragma unroll
    for (int e = 0; e < kMaxDPerLane; ++e) {
      const int64_t d = lane + 32 * e;
      if (d < D) acc[e] = fmaf(p, vr[d], acc[e] * alpha);
    }
    m = m_new;
  }
  float* orow = out + b * os0 + h * os1 + i * os2;
#pragma unroll
  for (int e = 0; e < kMaxDPerLane; ++e) {
    const int64_t d = lane + 32 * e;
    if (d < D) orow[d] = acc[e] / l;  // l == 0 (no visible key): NaN
  }
}

// Fills out with zeros (no keys at all: an empty weighted sum) or with NaN
// (keys exist but causal / window leave none to any query: the softmax of an
// all -inf row).
__global__ void gqa_fill_kernel(uint8_t* out, int64_t B, int64_t Hq, int64_t Sq, int64_t D,
                                int64_t os0, int64_t os1, int64_t os2, int elem_bytes, int nan) {
  const int64_t n = B * Hq * Sq * D;
  for (int64_t x = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; x < n;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t d = x % D, i = (x / D) % Sq, h = (x / (D * Sq)) % Hq, b = x / (D * Sq * Hq);
    uint8_t* dst = out + (b * os0 + h * os1 + i * os2 + d) * elem_bytes;
    if (elem_bytes == 4)
      *reinterpret_cast<uint32_t*>(dst) = nan ? 0x7FC00000u : 0u;
    else
      *reinterpret_cast<uint16_t*>(dst) = nan ? static_cast<uint16_t>(0x7FC0u) : static_cast<uint16_t>(0u);
  }
}

}  // namespace

int launch_f32(const gqa_problem& p, const float* q, const float* k, const float* v,
               const uint8_t* mask, float* out, uint32_t* err, cudaStream_t stream) {
  const int64_t rows = p.batch * p.heads_q * p.seq_q;
  const int warps_per_block = 8;
  const int64_t blocks = (rows + warps_per_block - 1) / warps_per_block;
  if (blocks > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  const float scale_log2 = static_cast<float>(static_cast<double>(p.scale) * 1.4426950408889634);
  gqa_f32_kernel<<<static_cast<unsigned>(blocks), warps_per_block * 32, 0, stream>>>(
      q, k, v, p.has_mask ? mask : nullptr, out, p.batch, p.heads_q, p.heads_kv, p.seq_q,
      p.seq_k, p.head_dim, p.q_stride[0], p.q_stride[1], p.q_stride[2], p.k_stride[0],
      p.k_stride[1], p.k_stride[2], p.v_stride[0], p.v_stride[1], p.v_stride[2], p.o_stride[0],
      p.o_stride[1], p.o_stride[2], p.mask_stride[0], p.mask_stride[1], p.causal,
      p.causal_offset, p.window, p.kv_lens, p.block_table, p.block_table_stride, p.page_size,
      p.num_pages, err, scale_log2);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int launch_zero(const gqa_problem& p, void* out, cudaStream_t stream, bool nan) {
  const int elem = p.dtype == GQA_DTYPE_F32 ? 4 : 2;
  gqa_fill_kernel<<<592, 256, 0, stream>>>(static_cast<uint8_t*>(out), p.batch, p.heads_q,
                                           p.seq_q, p.head_dim, p.o_stride[0], p.o_stride[1],
                                           p.o_stride[2], elem, nan ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace gqa
