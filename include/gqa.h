/*
 * gqa.h -- C ABI of the B200 (sm_100a) grouped-query attention forward.
 *
 * Operation (page "28. Grouped-Query Attention (GQA)", sections "Step-by-Step
 * Approach" and "Reference solution"; causal form from "Grouped-Query Attention
 * Explained Simply", "Minimal implementation"; bool attention mask from
 * "Multi-Query Attention", "Implementation"):
 *
 *   g            = heads_q / heads_kv                 (must divide exactly)
 *   s[b,h,i,j]   = scale * sum_d q[b,h,i,d] * k[b,h/g,j,d]
 *                  -inf where has_mask and mask[b,i,j] == 0
 *                  -inf where causal and j > i
 *   out[b,h,i,:] = sum_j softmax_j(s[b,h,i,:]) * v[b,h/g,j,:]
 *
 * Query head h reads kv head h / g (the contiguous "repeat_interleave"
 * grouping); the kv head is never expanded in memory -- each K/V tile is read
 * once and serves all g query heads of its group ("Multi-Query Attention",
 * remark under "Implementation": a zero stride over the head dimension).
 *
 * Conventions
 *  - Tensors are described by sizes and element strides; the innermost
 *    (head_dim) stride must be 1.  q and out are [batch, heads_q, seq_q,
 *    head_dim]; k and v are [batch, heads_kv, seq_k, head_dim]; the optional
 *    mask is uint8 [batch, seq_q, seq_k], nonzero = attend, shared by every
 *    head.  Any other strides are allowed (e.g. a [B, S, H, D] buffer viewed as
 *    [B, H, S, D]), subject to the 16-byte rules below on the bf16 paths.
 *  - dtype: GQA_DTYPE_BF16 or GQA_DTYPE_F16 (16-bit in/out, fp32 accumulation
 *    and softmax, head_dim a multiple of 8 up to 128) or GQA_DTYPE_F32 (fp32
 *    throughout, head_dim 1..256).
 *  - causal: key j is visible to query i iff j <= i + causal_offset.  The
 *    pages' causal attention (seq_q == seq_k) is causal_offset = 0 (top-left);
 *    decoding after a KV cache, bottom-right alignment, is causal_offset =
 *    seq_k - seq_q.  window > 0 (causal only) also hides keys
 *    j <= i + causal_offset - window: a sliding window of `window` keys ending
 *    at the diagonal (the sliding-window attention that "28. Grouped-Query
 *    Attention (GQA)", "Problem", names for Mistral).  With has_mask as well,
 *    a key must pass every rule.
 *  - kv_lens (optional, device int32 [batch]): a KV cache of capacity seq_k
 *    whose entry b holds kv_lens[b] valid keys.  Keys j >= kv_lens[b] are
 *    hidden, and the causal diagonal moves with the length: entry b uses
 *    causal_offset + kv_lens[b] - seq_k, so the offset is given for a full
 *    cache (bottom-right: seq_k - seq_q).  This is the GQA cache of shape
 *    (B, num_kv_groups, T, head_dim) that "Grouped-Query Attention vs
 *    Multi-Head Attention: Understanding GQA Implementation", "Memory
 *    Footprint and KV-Cache Optimization", describes, with a per-sequence T.
 *    A length outside [0, seq_k] is clamped and reported by gqa_device_status
 *    as GQA_ERR_KV_LENGTH.  Cache rows past a length never reach the result,
 *    whatever they hold (NaN included): the decode path masks them, and the
 *    prefill path zeroes the V rows of the last key tile in shared memory.
 *  - Paged cache (block_table != NULL; every path): k and v point
 *    to a pool of num_pages pages, each [heads_kv, page_size, head_dim],
 *    described by k_stride / v_stride over (page, h_kv, key in page, d).  Key
 *    j of batch entry b lives in page block_table[b * block_table_stride +
 *    j / page_size], row j % page_size.  page_size is a multiple of 64;
 *    seq_k <= block_table_stride * page_size is the capacity of a sequence.
 *    Pages past a sequence's length are never read, so their table entries
 *    may hold anything; a page index outside [0, num_pages) for a key below
 *    the length reads zeros and is reported as GQA_ERR_PAGE.
 *  - A row whose keys are all hidden yields NaN (the softmax of an all -inf
 *    row).  seq_k == 0 yields zeros (an empty weighted sum).  batch == 0 or
 *    seq_q == 0 is a no-op.
 *  - Memory: every pointer passed to gqa_forward is DEVICE memory of the
 *    current CUDA device, owned by the caller, and must stay valid until the
 *    work queued on `stream` has finished.  The library allocates nothing and
 *    keeps no state between calls.
 *  - Execution: gqa_forward only validates, plans and enqueues kernels on
 *    `stream` (a cudaStream_t; NULL = the legacy default stream); it returns
 *    before the work is done.  Errors in the arguments are returned at once;
 *    a kernel that gives up on an internal wait records it in the workspace's
 *    error word, read by gqa_device_status.
 *  - No function throws across this boundary; every function returns a status
 *    code (or a string / number as documented).
 */
#ifndef GQA_B200_GQA_H
#define GQA_B200_GQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

/* Status codes. */
#define GQA_OK 0
#define GQA_ERR_NULL 1        /* a required pointer is NULL */
#define GQA_ERR_SHAPE 2       /* sizes inconsistent, negative, or heads_q % heads_kv != 0 */
#define GQA_ERR_LAYOUT 3      /* innermost stride != 1, or a base/stride the TMA unit cannot
                                 address (bf16 paths: base and non-innermost strides must be
                                 multiples of 16 bytes) */
#define GQA_ERR_UNSUPPORTED 4 /* dtype / head_dim combination the kernels do not cover */
#define GQA_ERR_WORKSPACE 5   /* workspace NULL, too small, or not 256-byte aligned */
#define GQA_ERR_CUDA 6        /* a CUDA runtime call failed (launch, attribute, encode) */
#define GQA_ERR_TIMEOUT 7     /* a kernel's bounded internal wait ran out (gqa_device_status) */
#define GQA_ERR_ARG 8         /* scale not finite, unknown dtype, or a window without causal */
#define GQA_ERR_DEVICE 9      /* no usable CUDA device, or not an sm_100 device */
#define GQA_ERR_SCRATCH_LIMIT 10 /* gqa_forward_decode_noalloc: the problem needs more scratch
                                    than GQA_STATIC_SCRATCH_BYTES */
#define GQA_ERR_KV_LENGTH 11  /* gqa_device_status: a kv_lens entry was outside [0, seq_k], or an
                                 append did not fit the cache (that entry was left unchanged) */
#define GQA_ERR_PAGE 12       /* gqa_device_status: a block-table entry used for a key below
                                 the length was outside [0, num_pages) */

#define GQA_DTYPE_BF16 0
#define GQA_DTYPE_F32 1
#define GQA_DTYPE_F16 2

#define GQA_KERNEL_NONE 0     /* nothing to launch (empty problem) */
#define GQA_KERNEL_DECODE 1   /* bf16 / fp16, seq_q == 1 or (heads_q/heads_kv) * seq_q <= 16:
                                 split-K stream over the KV cache, one launch */
#define GQA_KERNEL_PREFILL 2  /* bf16 / fp16, longer query blocks: tcgen05 / tensor-memory tiles */
#define GQA_KERNEL_F32 3      /* fp32 CUDA-core path */
#define GQA_KERNEL_ZERO 4     /* seq_k == 0: the output is filled with zeros */
#define GQA_KERNEL_NAN 5      /* causal / window leave no key to any query: NaN (see above) */

/* One attention problem.  Strides are in elements. */
typedef struct gqa_problem {
  int32_t dtype;          /* GQA_DTYPE_BF16, GQA_DTYPE_F16 or GQA_DTYPE_F32, for q, k, v, out */
  int32_t causal;         /* nonzero: key j hidden from query i when j > i */
  int32_t has_mask;       /* nonzero: a mask pointer is passed to gqa_forward */
  float scale;            /* multiplies q.k; 1/sqrt(head_dim) reproduces the pages */
  int64_t batch, heads_q, heads_kv, seq_q, seq_k, head_dim;
  int64_t q_stride[4];    /* over (b, h, i, d) */
  int64_t k_stride[4];    /* over (b, h_kv, j, d) */
  int64_t v_stride[4];    /* over (b, h_kv, j, d) */
  int64_t o_stride[4];    /* over (b, h, i, d) */
  int64_t mask_stride[3]; /* over (b, i, j); the j stride must be 1 */
  int64_t causal_offset;  /* with causal: key j visible to query i iff j <= i + causal_offset */
  int64_t window;         /* with causal, > 0: keys j <= i + causal_offset - window hidden too */
  const int32_t* kv_lens; /* NULL, or device [batch]: valid keys per entry (see above) */
  const int32_t* block_table; /* NULL (contiguous k / v), or device [batch, block_table_stride] */
  int64_t block_table_stride; /* entries per batch row of block_table */
  int64_t page_size;          /* keys per page, a multiple of 64 */
  int64_t num_pages;          /* pages in the k / v pools */
} gqa_problem;

/* What gqa_forward will do for a problem on a device. */
typedef struct gqa_plan {
  int32_t kernel;            /* GQA_KERNEL_* */
  int32_t grid;              /* CTAs of the main kernel */
  int32_t block;             /* threads per CTA of the main kernel */
  int32_t smem_bytes;        /* dynamic shared memory per CTA of the main kernel */
  int32_t launches;          /* kernels enqueued per call */
  int32_t work_units;        /* decode: 128-key tiles streamed; prefill: 128-row tiles */
  int64_t workspace_bytes;   /* bytes of device scratch gqa_forward needs (>= 256) */
  int64_t algorithmic_bytes; /* bytes of q, k, v, out (and mask) the call must move once */
  double algorithmic_flops;  /* 4*B*Hq*Sq*Sk*D, halved when causal */
} gqa_plan;

/*
 * gqa_query -- validate `p` and describe the plan.
 *   sm_count: number of SMs to plan for; <= 0 asks the current CUDA device.
 * Returns GQA_OK, an argument error (checked before any device query), or
 * GQA_ERR_DEVICE when sm_count <= 0 and no device is usable.  Pure host code;
 * enqueues nothing.
 */
GQA_API int gqa_query(const gqa_problem* p, int sm_count, gqa_plan* plan);

/*
 * gqa_forward -- enqueue out = GQA(q, k, v, mask) on `stream`.
 *   q, k, v, out: device pointers described by `p` (dtype, sizes, strides).
 *   mask:         device uint8 pointer if p->has_mask, else ignored (may be NULL).
 *   workspace:    device scratch of at least plan.workspace_bytes, 256-byte
 *                 aligned, owned by the caller, ZERO-FILLED before its first
 *                 use.  Its head holds the error word and the decode ticket
 *                 counters (bytes [256, 256 + 64 KiB)); every call leaves that
 *                 head as it found it, so one workspace serves any sequence
 *                 of calls of any shapes without being cleared again.  After
 *                 an error gqa_device_status re-zeroes it.  Calls that share a
 *                 workspace must be ordered on one stream; calls that overlap
 *                 on the GPU race.
 *   stream:       cudaStream_t.
 * Returns GQA_OK once the kernels are enqueued, or an error code with nothing
 * enqueued.  Does not synchronise.
 */
GQA_API int gqa_forward(const gqa_problem* p, const void* q, const void* k, const void* v,
                        const uint8_t* mask, void* out, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * gqa_device_status -- synchronise `stream` and read the workspace's error
 * word.  Returns GQA_OK; or GQA_ERR_TIMEOUT if a kernel gave up on a wait (its
 * outputs are then undefined), in which case the first `workspace_bytes` of
 * the workspace are zeroed; or GQA_ERR_KV_LENGTH if a length was out of range
 * (the error word is cleared); or GQA_ERR_CUDA if the stream reports a CUDA
 * error.
 */
GQA_API int gqa_device_status(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Size of the library's static device scratch array used by
 * gqa_forward_decode_noalloc: 8 MiB, held on every GPU that loads the library
 * until the process exits.
 */
#define GQA_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)

/*
 * gqa_forward_decode_noalloc -- gqa_forward for the decode path without a
 * caller workspace.  The pages have no counterpart: this is a deployment
 * variant for callers that cannot allocate device memory -- code that is only
 * handed the q/k/v/out buffers by a host framework and has no allocator of its
 * own, or a steady-state loop that must not call cudaMalloc because it can
 * synchronise the device.
 *   p, q, k, v, mask, out, stream: as for gqa_forward (device pointers).
 * Accepts what gqa_forward sends to the decode kernel (GQA_KERNEL_DECODE):
 * bf16 or fp16, seq_q == 1 or (heads_q / heads_kv) * seq_q <= 16, with any of
 * mask, causal_offset, window, kv_lens and a paged cache.  seq_k == 0 fills
 * `out` with zeros and a problem in which no query sees a key fills it with
 * NaN, as gqa_forward does.  Longer query blocks (GQA_KERNEL_PREFILL) and
 * fp32 return GQA_ERR_UNSUPPORTED.
 * Scratch: a file-scope static device array of GQA_STATIC_SCRATCH_BYTES inside
 * the library.  The call looks up that array's device address on the current
 * device (cudaGetSymbolAddress) and caches it; during a stream capture only
 * the cached address is used, so make the first call on each device before
 * any capture.  The call allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine).  Every call on a device shares the one array:
 * each call zeroes the part that must start at zero (with cudaMemsetAsync on
 * `stream`) and leaves the rest as the last call left it, so calls that
 * overlap on the GPU race -- order them on one stream.
 * Returns GQA_OK once enqueued; GQA_ERR_UNSUPPORTED as above;
 * GQA_ERR_SCRATCH_LIMIT when the problem's scratch (the workspace_bytes
 * gqa_query reports) exceeds GQA_STATIC_SCRATCH_BYTES; the argument errors of
 * gqa_forward otherwise.  Errors found by the kernel are NOT reported: a wait
 * that runs out, a kv_lens entry outside [0, seq_k] (clamped) and a block-table
 * entry outside [0, num_pages) (read as zeros) are recorded only in the static
 * array, which the next call clears.  Use gqa_forward with gqa_device_status
 * where those must be detected.
 */
GQA_API int gqa_forward_decode_noalloc(const gqa_problem* p, const void* q, const void* k,
                                       const void* v, const uint8_t* mask, void* out,
                                       void* stream);

/*
 * KV-cache append: the step before each decode or prefill chunk, writing the
 * new tokens' keys and values after the ones a sequence already holds (the
 * cache_k / cache_v buffers of "Grouped-Query Attention vs Multi-Head
 * Attention: Understanding GQA Implementation", "GroupedQueryAttention Class
 * Structure", grown in place per sequence instead of concatenated).
 */
typedef struct gqa_kv_append_desc {
  int32_t dtype;                /* GQA_DTYPE_BF16, F16 or F32 (cache and new rows alike) */
  int32_t reserved;             /* must be 0 */
  int64_t batch, heads_kv, capacity, head_dim, n_new;
  int64_t cache_k_stride[4];    /* over (b, h_kv, j, d), j < capacity; d stride 1 */
  int64_t cache_v_stride[4];
  int64_t k_new_stride[4];      /* over (b, h_kv, t, d), t < n_new; d stride 1 */
  int64_t v_new_stride[4];
  /* Paged cache (block_table != NULL): cache_k / cache_v are page pools and
   * their strides run over (page, h_kv, key in page, d), as for gqa_forward;
   * capacity is then the largest length a sequence may reach. */
  const int32_t* block_table;
  int64_t block_table_stride, page_size, num_pages;
} gqa_kv_append_desc;

/*
 * gqa_kv_append -- for every entry b with L = kv_lens[b] and
 * 0 <= L <= capacity - n_new: cache_k[b, :, L + t, :] = k_new[b, :, t, :] and
 * the same for v, for t < n_new, then kv_lens[b] = L + n_new.  An entry that
 * does not fit is left unchanged (cache and length) and gqa_device_status
 * then returns GQA_ERR_KV_LENGTH.  With a block table, row L + t of entry b is
 * row (L + t) % page_size of page block_table[b * stride + (L + t) /
 * page_size]; an entry whose new rows would use a page index outside
 * [0, num_pages) is left unchanged and reported as GQA_ERR_PAGE.
 *   cache_k, cache_v, k_new, v_new: device pointers described by `d`; the new
 *                 rows must not overlap the cache.
 *   kv_lens:      device int32 [batch], read and updated in place.
 *   workspace:    a gqa_forward workspace (zero-filled before its first use,
 *                 256-byte aligned, at least 256 bytes); the append uses only
 *                 its first 16 bytes and leaves them as it found them.  One
 *                 launch, no cross-CTA wait.
 * Returns GQA_OK once enqueued, or an argument error with nothing enqueued.
 * The pages have no counterpart for the in-place length update: the pages
 * concatenate along the sequence and keep one length for the whole batch.
 */
GQA_API int gqa_kv_append(const gqa_kv_append_desc* d, void* cache_k, void* cache_v,
                          const void* k_new, const void* v_new, int32_t* kv_lens,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqa_debug_decode_trace -- diagnostics: record per-CTA phase timestamps of
 * the decode kernel.  Not part of the operation (the pages have no
 * counterpart); used to account for the time of a launch that is not spent
 * streaming K/V.
 *   device_buffer: device memory of `bytes` bytes, 8-byte aligned, owned by
 *                  the caller, or NULL to stop recording.
 * While set, every decode launch (gqa_forward, gqa_forward_decode_noalloc)
 * writes, per CTA, 16 unsigned 64-bit words (%globaltimer nanoseconds and
 * counts; layout: kDecodeTraceWords / DecodeTraceWord in the library's
 * csrc/kernels.h) into the next slot of grid * 128 bytes; launch k uses slot
 * k mod (bytes / slot size).  The setting is process-wide and is captured
 * into CUDA graphs with the launch.  Returns GQA_OK, GQA_ERR_ARG for a
 * negative size or GQA_ERR_LAYOUT for a misaligned buffer.
 */
GQA_API int gqa_debug_decode_trace(void* device_buffer, int64_t bytes);

/*
 * gqa_debug_decode_withhold -- test of the kernels' bounded waits (failure
 * detection without a GPU fault; the pages have no counterpart).  The NEXT
 * decode launch of the process (gqa_forward or gqa_forward_decode_noalloc)
 * uses `wait_limit_ns` (1000 .. 1e9) as the limit of every internal wait and,
 * if `unit` >= 0, its producer never issues the copies of that 128-key unit
 * (index in launch order) and issues nothing after it: the consumers' wait
 * for the unit runs out, the CTA unwinds (every copy already issued lands
 * first), the output is undefined and gqa_device_status then returns
 * GQA_ERR_TIMEOUT and re-zeroes the workspace.  The setting is consumed by
 * that one launch.  Returns GQA_OK or GQA_ERR_ARG.
 */
GQA_API int gqa_debug_decode_withhold(int64_t unit, int64_t wait_limit_ns);

/* Static English description of a status code (never NULL). */
GQA_API const char* gqa_status_string(int status);

/* ABI version of this library (major * 10000 + minor * 100 + patch). */
GQA_API int gqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_B200_GQA_H */
