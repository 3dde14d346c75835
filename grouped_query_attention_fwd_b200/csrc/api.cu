// C-ABI layer: validation, planning, TMA descriptor encoding and dispatch.
// Every entry point returns a status code; nothing throws across the ABI.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "gqa.h"
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int64_t kErrWordBytes = kWorkspaceHeadBytes;  // error word, append ticket

// bf16 and fp16 share the tensor-core paths.
bool half_paths(const gqa_problem& p) {
  return p.dtype == GQA_DTYPE_BF16 || p.dtype == GQA_DTYPE_F16;
}

int validate(const gqa_problem* pp) {
  if (pp == nullptr) return GQA_ERR_NULL;
  const gqa_problem& p = *pp;
  if (p.dtype != GQA_DTYPE_BF16 && p.dtype != GQA_DTYPE_F32 && p.dtype != GQA_DTYPE_F16)
    return GQA_ERR_ARG;
  if (!std::isfinite(p.scale)) return GQA_ERR_ARG;
  if (p.batch < 0 || p.seq_q < 0 || p.seq_k < 0) return GQA_ERR_SHAPE;
  if (p.heads_q <= 0 || p.heads_kv <= 0 || p.head_dim <= 0) return GQA_ERR_SHAPE;
  if (p.heads_q % p.heads_kv != 0) return GQA_ERR_SHAPE;
  // Sizes must fit the kernels' 32-bit coordinates.
  const int64_t lim = int64_t(1) << 31;
  if (p.batch >= lim || p.heads_q >= lim || p.seq_q >= lim || p.seq_k >= lim) return GQA_ERR_SHAPE;
  if (p.q_stride[3] != 1 || p.k_stride[3] != 1 || p.v_stride[3] != 1 || p.o_stride[3] != 1)
    return GQA_ERR_LAYOUT;
  if (p.has_mask && p.mask_stride[2] != 1) return GQA_ERR_LAYOUT;
  for (int d = 0; d < 3; ++d)
    if (p.q_stride[d] < 0 || p.k_stride[d] < 0 || p.v_stride[d] < 0 || p.o_stride[d] < 0 ||
        (p.has_mask && p.mask_stride[d] < 0))
      return GQA_ERR_LAYOUT;
  if (p.window < 0 || (p.window > 0 && !p.causal)) return GQA_ERR_ARG;
  if (p.causal_offset <= -lim || p.causal_offset >= lim || p.window >= lim) return GQA_ERR_ARG;
  if (half_paths(p)) {
    // Multiples of 8 up to 128: the kernels run at 64 or 128 wide, TMA
    // filling the columns past head_dim with zeros.
    if (p.head_dim % 8 != 0 || p.head_dim > 128) return GQA_ERR_UNSUPPORTED;
    // 16-byte rule of the TMA unit for every stride of a dimension longer than 1.
    // A paged k / v runs over (page, kv head, key in page).
    const int64_t qsz[3] = {p.batch, p.heads_q, p.seq_q};
    const int64_t ksz[3] = {p.block_table ? p.num_pages : p.batch, p.heads_kv,
                            p.block_table ? p.page_size : p.seq_k};
    for (int d = 0; d < 3; ++d) {
      if (qsz[d] > 1 && (p.q_stride[d] % 8 != 0 || p.o_stride[d] % 8 != 0)) return GQA_ERR_LAYOUT;
      if (ksz[d] > 1 && (p.k_stride[d] % 8 != 0 || p.v_stride[d] % 8 != 0)) return GQA_ERR_LAYOUT;
    }
    if (p.seq_q > 1) {
      const int64_t g = p.heads_q / p.heads_kv;
      if (g > 128) return GQA_ERR_UNSUPPORTED;  // one query position per 128-row tile at most
    }
  } else {
    if (p.head_dim > 256) return GQA_ERR_UNSUPPORTED;
  }
  if (p.block_table != nullptr) {
    // Pages hold whole 64-key halves of the decode kernel's 128-key tiles.
    if (p.page_size < 64 || p.page_size % 64 != 0 || p.page_size >= lim) return GQA_ERR_SHAPE;
    if (p.block_table_stride < 1 || p.block_table_stride >= lim) return GQA_ERR_SHAPE;
    if (p.num_pages < 1 || p.num_pages >= lim) return GQA_ERR_SHAPE;
    if (p.seq_k > p.block_table_stride * p.page_size) return GQA_ERR_SHAPE;
  }
  if (p.kv_lens != nullptr) {
    // The decode kernel keeps the lengths and their prefix sums in shared
    // memory and counts tiles in 32 bits.
    if (p.batch > kMaxRaggedBatch) return GQA_ERR_UNSUPPORTED;
    const int64_t tiles = (p.seq_k + kDecodeKeysPerTile - 1) / kDecodeKeysPerTile;
    if (p.batch * p.heads_kv * ((p.heads_q / p.heads_kv) * p.seq_q + 7) / 8 * tiles >= lim)
      return GQA_ERR_UNSUPPORTED;
  }
  return GQA_OK;
}

// No key is visible to any query under causal / window.
bool nothing_visible(const gqa_problem& p) {
  if (!p.causal) return false;
  // Query i sees keys [i + off - window + 1, i + off] (window > 0) or [0, i + off].
  const int64_t top = p.seq_q - 1 + p.causal_offset;  // largest upper bound
  if (top < 0) return true;
  if (p.window > 0 && p.causal_offset - p.window + 1 > p.seq_k - 1) return true;
  return false;
}

int pick_kernel(const gqa_problem& p) {
  if (p.batch == 0 || p.seq_q == 0) return GQA_KERNEL_NONE;
  if (p.seq_k == 0) return GQA_KERNEL_ZERO;
  if (nothing_visible(p)) return GQA_KERNEL_NAN;
  if (p.dtype == GQA_DTYPE_F32) return GQA_KERNEL_F32;
  // Decode streams K/V once per pass of at most 16 (head, query) rows: one
  // pass covers every query position when g * seq_q <= 16 (single-token and
  // short multi-token decode); larger query blocks go to the prefill tiles.
  const int64_t g = p.heads_q / p.heads_kv;
  if (p.seq_q == 1 || g * p.seq_q <= kDecodeMaxRowsPerPass) return GQA_KERNEL_DECODE;
  return GQA_KERNEL_PREFILL;
}

int device_sm_count(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  int sms = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  if (major != 10) return GQA_ERR_DEVICE;
  *out = sms;
  return GQA_OK;
}

int64_t elem_bytes(const gqa_problem& p) { return p.dtype == GQA_DTYPE_F32 ? 4 : 2; }

int fill_plan(const gqa_problem& p, int sm_count, gqa_plan* plan) {
  std::memset(plan, 0, sizeof(*plan));
  const int64_t eb = elem_bytes(p);
  const int64_t qo = p.batch * p.heads_q * p.seq_q * p.head_dim * eb;
  const int64_t kv = p.batch * p.heads_kv * p.seq_k * p.head_dim * eb;
  plan->algorithmic_bytes = 2 * qo + 2 * kv + (p.has_mask ? p.batch * p.seq_q * p.seq_k : 0);
  double flops = 4.0 * double(p.batch) * double(p.heads_q) * double(p.seq_q) * double(p.seq_k) *
                 double(p.head_dim);
  if (p.causal) flops *= 0.5;
  plan->algorithmic_flops = flops;
  plan->workspace_bytes = kErrWordBytes;
  plan->kernel = pick_kernel(p);
  switch (plan->kernel) {
    case GQA_KERNEL_NONE:
      break;
    case GQA_KERNEL_ZERO:
    case GQA_KERNEL_NAN:
      plan->grid = 592;
      plan->block = 256;
      plan->launches = 1;
      break;
    case GQA_KERNEL_F32: {
      const int64_t rows = p.batch * p.heads_q * p.seq_q;
      plan->grid = static_cast<int32_t>((rows + 7) / 8);
      plan->block = 256;
      plan->launches = 1;
      plan->work_units = static_cast<int32_t>(rows);
      break;
    }
    case GQA_KERNEL_DECODE: {
      const DecodeShape s = plan_decode(p, sm_count);
      if (s.units >= (int64_t(1) << 31)) return GQA_ERR_UNSUPPORTED;  // 32-bit unit indices
      plan->grid = s.grid;
      plan->block = kDecodeThreads;
      plan->smem_bytes = s.smem_bytes;
      plan->launches = s.zero_counters ? 2 : 1;  // (+ a counter memset for huge problems)
      plan->work_units = static_cast<int32_t>(s.units);
      plan->workspace_bytes = s.workspace_end;
      break;
    }
    case GQA_KERNEL_PREFILL: {
      const PrefillShape s = plan_prefill(p, sm_count);
      plan->grid = s.grid;
      plan->block = kPrefillThreads;
      plan->smem_bytes = s.smem_bytes;
      // (+ the mask summary pre-pass, and the sort of the items by cost)
      plan->launches = 1 + (p.has_mask ? 1 : 0) + (s.order_offset >= 0 ? 1 : 0);
      plan->work_units = static_cast<int32_t>(s.work);
      plan->workspace_bytes = s.workspace_end;
      break;
    }
  }
  plan->workspace_bytes = (plan->workspace_bytes + 255) / 256 * 256;
  return GQA_OK;
}

// ------------------------------------------------------------ TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 4-D bf16 map over (d, s, h, b) of a tensor with element strides st[0..2]
// for (b, h, s); box {64, box_s, box_h, 1} with 128-byte swizzle.
int encode_half_map(CUtensorMap* map, const void* base, int64_t B, int64_t H, int64_t S,
                    int64_t D, const int64_t st[4], uint32_t box_s, uint32_t box_h, bool f16) {
  auto enc = get_encoder();
  if (enc == nullptr) return GQA_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  // Strides of length-1 dimensions are never stepped; give them a legal value.
  int64_t sb = st[2] * 2, hb = st[1] * 2, bb = st[0] * 2;
  if (S <= 1) sb = D * 2 < 16 ? 16 : ((D * 2 + 15) / 16) * 16;
  if (H <= 1) hb = sb * (S > 0 ? S : 1);
  if (B <= 1) bb = hb * (H > 0 ? H : 1);
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(sb), static_cast<cuuint64_t>(hb),
                           static_cast<cuuint64_t>(bb)};
  cuuint32_t box[4] = {64, box_s, box_h, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   4, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_LAYOUT;
}

bool aligned(const void* ptr, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0;
}

}  // namespace
}  // namespace gqa

namespace gqa {
namespace {
// Diagnostic trace buffer of the decode kernel (gqa_debug_decode_trace).
std::mutex g_trace_mu;
uint64_t* g_trace_buf = nullptr;
int64_t g_trace_bytes = 0;
uint64_t g_trace_next = 0;
}  // namespace

int g_withhold_unit = -1;  // one-shot test settings (gqa_debug_decode_withhold)
uint64_t g_wait_ns = kWaitLimitNs;

void decode_test_settings(int* withhold_unit, uint64_t* wait_ns) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  *withhold_unit = g_withhold_unit;
  *wait_ns = g_wait_ns;
  g_withhold_unit = -1;
  g_wait_ns = kWaitLimitNs;
}

uint64_t* decode_trace_slot(int grid) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  if (g_trace_buf == nullptr || grid <= 0) return nullptr;
  const int64_t words = static_cast<int64_t>(grid) * kDecodeTraceWords;
  const int64_t slots = g_trace_bytes / (words * 8);
  if (slots <= 0) return nullptr;
  const int64_t slot = static_cast<int64_t>(g_trace_next++ % static_cast<uint64_t>(slots));
  return g_trace_buf + slot * words;
}

// K/V tensor map for the decode tile shape, shared with the static-scratch
// decode entry point.
int encode_decode_kv_map(CUtensorMap* map, const void* base, const gqa_problem& p,
                         const int64_t st[4]) {
  const bool f16 = p.dtype == GQA_DTYPE_F16;
  if (p.block_table != nullptr)  // (d, key in page, kv head, page), 64-key boxes
    return encode_half_map(map, base, p.num_pages, p.heads_kv, p.page_size, p.head_dim, st,
                           kDecodePageBox, 1, f16);
  return encode_half_map(map, base, p.batch, p.heads_kv, p.seq_k, p.head_dim, st,
                         kDecodeKeysPerTile, 1, f16);
}
}  // namespace gqa

using namespace gqa;

extern "C" {

GQA_API int gqa_version(void) { return 10300; }

GQA_API const char* gqa_status_string(int status) {
  switch (status) {
    case GQA_OK: return "ok";
    case GQA_ERR_NULL: return "a required pointer is NULL";
    case GQA_ERR_SHAPE: return "inconsistent or invalid sizes (heads_q must be a multiple of heads_kv)";
    case GQA_ERR_LAYOUT: return "unsupported memory layout (innermost stride must be 1; bf16 bases and strides must be multiples of 16 bytes)";
    case GQA_ERR_UNSUPPORTED: return "unsupported combination (bf16/fp16 need head_dim a multiple of 8, at most 128)";
    case GQA_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case GQA_ERR_CUDA: return "a CUDA runtime call failed";
    case GQA_ERR_TIMEOUT: return "a kernel gave up on an internal wait; outputs are undefined";
    case GQA_ERR_ARG: return "invalid scalar argument (finite scale, known dtype, window >= 0 and only with causal)";
    case GQA_ERR_DEVICE: return "no usable sm_100 CUDA device";
    case GQA_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the library's static array holds";
    case GQA_ERR_KV_LENGTH: return "a kv length was outside [0, capacity], or an append did not fit the cache";
    case GQA_ERR_PAGE: return "a block-table entry in use was outside [0, num_pages)";
    default: return "unknown status";
  }
}

GQA_API int gqa_query(const gqa_problem* p, int sm_count, gqa_plan* plan) {
  if (plan == nullptr) return GQA_ERR_NULL;
  const int rc = validate(p);
  if (rc != GQA_OK) return rc;
  if (sm_count <= 0) {
    const int drc = device_sm_count(&sm_count);
    if (drc != GQA_OK) return drc;
  }
  return fill_plan(*p, sm_count, plan);
}

GQA_API int gqa_forward(const gqa_problem* pp, const void* q, const void* k, const void* v,
                        const uint8_t* mask, void* out, void* workspace, size_t workspace_bytes,
                        void* stream_ptr) {
  const int rc = validate(pp);
  if (rc != GQA_OK) return rc;
  const gqa_problem& p = *pp;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  gqa_plan plan;
  int sms = 0;
  {
    const int drc = device_sm_count(&sms);
    if (drc != GQA_OK) return drc;
  }
  const int prc = fill_plan(p, sms, &plan);
  if (prc != GQA_OK) return prc;
  if (plan.kernel == GQA_KERNEL_NONE) return GQA_OK;
  if (out == nullptr) return GQA_ERR_NULL;
  if (plan.kernel == GQA_KERNEL_ZERO) return launch_zero(p, out, stream, false);
  if (plan.kernel == GQA_KERNEL_NAN) return launch_zero(p, out, stream, true);
  if (q == nullptr || k == nullptr || v == nullptr) return GQA_ERR_NULL;
  if (p.has_mask && mask == nullptr) return GQA_ERR_NULL;
  if (workspace == nullptr) return GQA_ERR_WORKSPACE;
  if (!aligned(workspace, 256) || workspace_bytes < static_cast<size_t>(plan.workspace_bytes))
    return GQA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);

  if (plan.kernel == GQA_KERNEL_F32) {
    if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(out, 4))
      return GQA_ERR_LAYOUT;
    return launch_f32(p, static_cast<const float*>(q), static_cast<const float*>(k),
                      static_cast<const float*>(v), mask, static_cast<float*>(out), err, stream);
  }

  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return GQA_ERR_LAYOUT;
  const float scale_log2 =
      static_cast<float>(static_cast<double>(p.scale) * 1.4426950408889634073599);
  const int64_t g = p.heads_q / p.heads_kv;

  if (plan.kernel == GQA_KERNEL_DECODE) {
    const DecodeShape s = plan_decode(p, sms);
    CUtensorMap tmk, tmv;
    int erc = encode_decode_kv_map(&tmk, k, p, p.k_stride);
    if (erc != GQA_OK) return erc;
    erc = encode_decode_kv_map(&tmv, v, p, p.v_stride);
    if (erc != GQA_OK) return erc;
    const DecodeArgs a = make_decode_args(p, s, q, mask, out, ws);
    // The ticket counters must start at zero; other calls sharing this
    // workspace (a prefill's tile classes, a larger problem's partials) may
    // have left bytes there.
    if (s.zero_counters &&
        cudaMemsetAsync(a.counters, 0, static_cast<size_t>(s.groups) * 4, stream) != cudaSuccess)
      return GQA_ERR_CUDA;
    return launch_decode(p, s, a, tmk, tmv, stream);
  }

  // Prefill.
  const PrefillShape s = plan_prefill(p, sms);
  CUtensorMap tmq, tmk, tmv;
  const bool f16 = p.dtype == GQA_DTYPE_F16;
  int erc = encode_half_map(&tmq, q, p.batch, p.heads_q, p.seq_q, p.head_dim, p.q_stride,
                            static_cast<uint32_t>(s.qpt), static_cast<uint32_t>(g), f16);
  if (erc != GQA_OK) return erc;
  if (p.block_table != nullptr) {  // paged: 64-key boxes, one page each
    erc = encode_decode_kv_map(&tmk, k, p, p.k_stride);
    if (erc != GQA_OK) return erc;
    erc = encode_decode_kv_map(&tmv, v, p, p.v_stride);
    if (erc != GQA_OK) return erc;
  } else {
    erc = encode_half_map(&tmk, k, p.batch, p.heads_kv, p.seq_k, p.head_dim, p.k_stride, 128,
                          1, f16);
    if (erc != GQA_OK) return erc;
    erc = encode_half_map(&tmv, v, p.batch, p.heads_kv, p.seq_k, p.head_dim, p.v_stride, 128,
                          1, f16);
    if (erc != GQA_OK) return erc;
  }
  PrefillArgs a{};
  a.mask = p.has_mask ? mask : nullptr;
  for (int d = 0; d < 3; ++d) a.ms[d] = p.mask_stride[d];
  a.out = static_cast<uint16_t*>(out);
  for (int d = 0; d < 4; ++d) a.os[d] = p.o_stride[d];
  a.summary = ws + s.summary_offset;
  a.order = s.order_offset >= 0 ? reinterpret_cast<int32_t*>(ws + s.order_offset) : nullptr;
  a.bounds = s.bounds_offset >= 0 ? reinterpret_cast<int32_t*>(ws + s.bounds_offset) : nullptr;
  a.err = err;
  a.B = static_cast<int>(p.batch);
  a.Hq = static_cast<int>(p.heads_q);
  a.Hkv = static_cast<int>(p.heads_kv);
  a.Sq = static_cast<int>(p.seq_q);
  a.Sk = static_cast<int>(p.seq_k);
  a.g = static_cast<int>(g);
  a.causal = p.causal;
  a.causal_offset = p.causal_offset;
  a.window = p.window;
  a.has_mask = p.has_mask;
  a.lens = p.kv_lens;
  a.Dv = static_cast<int>(p.head_dim);
  a.scale_log2 = scale_log2;
  if (s.pp) return launch_prefill_pp(p, s, a, tmq, tmk, tmv, stream);
  return launch_prefill(p, s, a, tmq, tmk, tmv, stream);
}

GQA_API int gqa_kv_append(const gqa_kv_append_desc* d, void* cache_k, void* cache_v,
                          const void* k_new, const void* v_new, int32_t* kv_lens,
                          void* workspace, size_t workspace_bytes, void* stream_ptr) {
  if (d == nullptr) return GQA_ERR_NULL;
  if (d->dtype != GQA_DTYPE_BF16 && d->dtype != GQA_DTYPE_F32 && d->dtype != GQA_DTYPE_F16)
    return GQA_ERR_ARG;
  if (d->reserved != 0) return GQA_ERR_ARG;
  const int64_t lim = int64_t(1) << 31;
  if (d->batch < 0 || d->heads_kv <= 0 || d->capacity < 0 || d->head_dim <= 0 || d->n_new < 0 ||
      d->batch >= lim || d->heads_kv >= lim || d->capacity >= lim || d->head_dim > 4096)
    return GQA_ERR_SHAPE;
  if (d->n_new > d->capacity) return GQA_ERR_SHAPE;
  if (d->block_table != nullptr &&
      (d->page_size < 1 || d->block_table_stride < 1 || d->num_pages < 1 ||
       d->capacity > d->block_table_stride * d->page_size))
    return GQA_ERR_SHAPE;
  const int64_t* st[4] = {d->cache_k_stride, d->cache_v_stride, d->k_new_stride, d->v_new_stride};
  for (const int64_t* x : st) {
    if (x[3] != 1) return GQA_ERR_LAYOUT;
    if (x[0] < 0 || x[1] < 0 || x[2] < 0) return GQA_ERR_LAYOUT;
  }
  if (d->batch == 0 || d->n_new == 0) return GQA_OK;
  if (cache_k == nullptr || cache_v == nullptr || k_new == nullptr || v_new == nullptr ||
      kv_lens == nullptr)
    return GQA_ERR_NULL;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < 256)
    return GQA_ERR_WORKSPACE;
  const int eb = d->dtype == GQA_DTYPE_F32 ? 4 : 2;
  if (!aligned(cache_k, eb) || !aligned(cache_v, eb) || !aligned(k_new, eb) ||
      !aligned(v_new, eb) || !aligned(kv_lens, 4))
    return GQA_ERR_LAYOUT;
  AppendArgs a{};
  a.ck = static_cast<uint8_t*>(cache_k);
  a.cv = static_cast<uint8_t*>(cache_v);
  a.kn = static_cast<const uint8_t*>(k_new);
  a.vn = static_cast<const uint8_t*>(v_new);
  a.lens = kv_lens;
  a.err = static_cast<uint32_t*>(workspace);
  a.ticket = static_cast<uint32_t*>(workspace) + 1;
  for (int i = 0; i < 3; ++i) {
    a.cks[i] = d->cache_k_stride[i] * eb;
    a.cvs[i] = d->cache_v_stride[i] * eb;
    a.kns[i] = d->k_new_stride[i] * eb;
    a.vns[i] = d->v_new_stride[i] * eb;
  }
  a.B = static_cast<int>(d->batch);
  a.H = static_cast<int>(d->heads_kv);
  a.cap = d->capacity;
  a.n_new = d->n_new;
  a.row_bytes = static_cast<int>(d->head_dim * eb);
  // 16-byte pieces when every row start is 16-byte aligned, else elements.
  bool v16 = a.row_bytes % 16 == 0 && aligned(cache_k, 16) && aligned(cache_v, 16) &&
             aligned(k_new, 16) && aligned(v_new, 16);
  for (int i = 0; i < 3 && v16; ++i)
    v16 = a.cks[i] % 16 == 0 && a.cvs[i] % 16 == 0 && a.kns[i] % 16 == 0 && a.vns[i] % 16 == 0;
  a.vec = v16 ? 16 : eb;
  a.bt = d->block_table;
  a.bt_stride = d->block_table_stride;
  a.page_size = d->page_size;
  a.num_pages = d->num_pages;
  return launch_kv_append(a, static_cast<cudaStream_t>(stream_ptr));
}

GQA_API int gqa_debug_decode_trace(void* device_buffer, int64_t bytes) {
  if (device_buffer != nullptr && bytes < 0) return GQA_ERR_ARG;
  if (device_buffer != nullptr && (reinterpret_cast<uintptr_t>(device_buffer) & 7u) != 0)
    return GQA_ERR_LAYOUT;
  std::lock_guard<std::mutex> lock(g_trace_mu);
  g_trace_buf = static_cast<uint64_t*>(device_buffer);
  g_trace_bytes = device_buffer != nullptr ? bytes : 0;
  g_trace_next = 0;
  return GQA_OK;
}

GQA_API int gqa_debug_decode_withhold(int64_t unit, int64_t wait_limit_ns) {
  if (unit < -1 || unit >= (int64_t(1) << 31)) return GQA_ERR_ARG;
  if (wait_limit_ns < 1000 || wait_limit_ns > static_cast<int64_t>(kWaitLimitNs))
    return GQA_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_trace_mu);
  g_withhold_unit = static_cast<int>(unit);
  g_wait_ns = static_cast<uint64_t>(wait_limit_ns);
  return GQA_OK;
}

GQA_API int gqa_device_status(void* workspace, size_t workspace_bytes, void* stream_ptr) {
  if (workspace == nullptr) return GQA_ERR_NULL;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  uint32_t word[4] = {0, 0, 0, 0};
  if (cudaMemcpyAsync(word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  if (word[0] != 0 && (word[0] & ~(kErrKvLength | kErrPage)) == 0) {
    // Only a length or a page index was out of range: the kernels finished.
    const int status = (word[0] & kErrKvLength) ? GQA_ERR_KV_LENGTH : GQA_ERR_PAGE;
    const uint32_t zero = 0;
    if (cudaMemcpyAsync(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    return status;
  }
  if (word[0] != 0) {
    // A kernel gave up part-way: its split counters may be off.  Return the
    // whole workspace to the all-zero state that the next call expects.
    const size_t n = workspace_bytes > sizeof(word) ? workspace_bytes : sizeof(word);
    if (cudaMemsetAsync(workspace, 0, n, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    return GQA_ERR_TIMEOUT;
  }
  return GQA_OK;
}

}  // extern "C"
