// KV-cache append: copy the new tokens' K and V rows of every batch entry to
// the rows after the ones it already holds, then advance its length.
//
// The copy is a plain HBM-bound gather/scatter: consecutive threads take
// consecutive 16-byte pieces of a row (then rows, then heads), so both sides
// are read and written in full sectors.  Each entry's length is read before
// its rows are written; the lengths are advanced by the last CTA to finish
// (a ticket counter), which by then has seen every other CTA's reads
// complete -- one launch, and no CTA waits for another.
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

template <typename V>
__global__ void __launch_bounds__(256) gqa_kv_append_kernel(const AppendArgs a) {
  // A decode launched after this one as a programmatic dependent may start its
  // prologue now; it waits for this launch to complete before reading the
  // lengths and rows written here.
  griddep_launch_dependents();
  const int per_row = a.row_bytes / static_cast<int>(sizeof(V));
  const int64_t per_tensor = static_cast<int64_t>(a.B) * a.H * a.n_new * per_row;
  const int64_t total = 2 * per_tensor;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool is_v = x >= per_tensor;
    int64_t y = is_v ? x - per_tensor : x;
    const int c = static_cast<int>(y % per_row);
    y /= per_row;
    const int64_t t = y % a.n_new;
    y /= a.n_new;
    const int h = static_cast<int>(y % a.H);
    const int b = static_cast<int>(y / a.H);
    const int64_t len = a.lens[b];
    if (len < 0 || len > a.cap - a.n_new) {
      if (!is_v && t == 0 && h == 0 && c == 0) atomicOr(a.err, kErrKvLength);
      continue;
    }
    const int64_t* ns = is_v ? a.vns : a.kns;
    const int64_t* cs = is_v ? a.cvs : a.cks;
    const uint8_t* src = (is_v ? a.vn : a.kn) + b * ns[0] + h * ns[1] + t * ns[2] +
                         static_cast<int64_t>(c) * sizeof(V);
    int64_t row_off = b * cs[0] + (len + t) * cs[2];
    if (a.bt != nullptr) {  // paged: row len + t of entry b lives in a page of the pool
      const int64_t page = a.bt[b * a.bt_stride + (len + t) / a.page_size];
      if (page < 0 || page >= a.num_pages) {
        if (!is_v && h == 0 && c == 0) atomicOr(a.err, kErrPage);
        continue;
      }
      row_off = page * cs[0] + ((len + t) % a.page_size) * cs[2];
    }
    uint8_t* dst = (is_v ? a.cv : a.ck) + row_off + h * cs[1] + static_cast<int64_t>(c) * sizeof(V);
    *reinterpret_cast<V*>(dst) = *reinterpret_cast<const V*>(src);
  }

  __shared__ int last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(a.ticket, 1u) == gridDim.x - 1 ? 1 : 0;
  }
  __syncthreads();
  if (last) {
    // Every CTA has read the lengths it needed: advance them.
    __threadfence();
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
      const int64_t len = a.lens[b];
      if (len < 0 || len > a.cap - a.n_new) continue;
      bool pages_ok = true;  // every page the new rows went to was in the pool
      if (a.bt != nullptr) {
        for (int64_t pg = len / a.page_size; pg <= (len + a.n_new - 1) / a.page_size; ++pg) {
          const int64_t page = a.bt[b * a.bt_stride + pg];
          pages_ok = pages_ok && page >= 0 && page < a.num_pages;
        }
      }
      if (pages_ok) a.lens[b] = static_cast<int32_t>(len + a.n_new);
    }
    if (threadIdx.x == 0) atomicExch(a.ticket, 0u);
  }
}

}  // namespace

int launch_kv_append(const AppendArgs& a, cudaStream_t stream) {
  const int64_t vecs = 2 * static_cast<int64_t>(a.B) * a.H * a.n_new * (a.row_bytes / a.vec);
  int64_t blocks = (vecs + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  const unsigned grid = static_cast<unsigned>(blocks);
  if (a.vec == 16)
    gqa_kv_append_kernel<uint4><<<grid, 256, 0, stream>>>(a);
  else if (a.vec == 4)
    gqa_kv_append_kernel<uint32_t><<<grid, 256, 0, stream>>>(a);
  else
    gqa_kv_append_kernel<uint16_t><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace gqa
