// Pieces shared by the two prefill kernels (one query tile per SM, and two
// query tiles per SM): the geometry of a query tile's visible
// keys, the classification of key tiles, per-key visibility bits, the
// shared-memory matrix descriptors and the packing of P.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace prefill {

constexpr int BM = 128;  // rows per tile = TMEM lanes
constexpr int BN = 128;  // keys per K/V tile
constexpr float kRescaleLog2 = 8.0f;  // lazy rescale: the reference may trail the maximum by 2^8

// P as a 16-bit pair, `lo` in the low half.  For bf16, P being finite and
// non-negative, rounding to nearest (ties away from zero) is an integer add
// of half a unit in the last place and a byte permute.
template <bool F16>
__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
  if (F16) return pack2<F16>(lo, hi);
  return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
}

__device__ __forceinline__ int64_t imin64(int64_t x, int64_t y) { return x < y ? x : y; }
__device__ __forceinline__ int64_t imax64(int64_t x, int64_t y) { return x > y ? x : y; }

// Paged K / V cache: a pool of num_pages pages, each [Hkv, page_size, D];
// key j of entry b is row j % page_size of page bt[b * bt_stride + j /
// page_size].  bt == nullptr: contiguous caches.
struct PagedKV {
  const int32_t* bt;
  int64_t bt_stride;
  int page_size, num_pages;
};

// Work item: one query tile of one (batch, kv head).
struct Pair {
  int b, kv, mt0, nt_beg, nt_end;
  int len;  // cache length of entry b (seq_k without per-sequence lengths)
};

// Causal offset of the item's entry: the diagonal moves with its length.
__device__ __forceinline__ int64_t pair_off(const PrefillArgs& a, const Pair& pr) {
  return a.causal_offset + (static_cast<int64_t>(pr.len) - a.Sk);
}

struct Slot {  // the item's query tile
  int mt, q0, q_last;
  bool live;
  int64_t key_lo, key_hi;  // keys some row of the tile can see (causal / window)
};

__device__ __forceinline__ Slot slot_of(const Pair& pr, const PrefillArgs& a, int qpt) {
  Slot sl;
  sl.mt = pr.mt0;
  sl.live = true;
  sl.q0 = sl.mt * qpt;
  sl.q_last = min(sl.q0 + qpt, a.Sq) - 1;
  sl.key_lo = 0;
  sl.key_hi = pr.len;
  if (a.causal) {
    const int64_t off = pair_off(a, pr);
    sl.key_hi = imin64(pr.len, static_cast<int64_t>(sl.q_last) + off + 1);
    if (a.window > 0) sl.key_lo = imax64(0, static_cast<int64_t>(sl.q0) + off - a.window + 1);
  }
  if (sl.key_hi <= sl.key_lo) sl.key_lo = sl.key_hi = 0;
  return sl;
}

// Class of key tile nt for the item's query tile: 0 every key hidden from
// every row (skip), 1 mixed (mask per element), 2 every key visible to every row.
__device__ __forceinline__ int tile_class(const PrefillArgs& a, const Pair& pr, const Slot& sl,
                                          int nt, int m_tiles, int n_tiles) {
  if (!sl.live) return 0;
  const int64_t j0 = static_cast<int64_t>(nt) * BN, j1 = j0 + BN - 1;
  if (j1 < sl.key_lo || j0 >= sl.key_hi) return 0;
  int cls = 2;
  if (j1 >= pr.len) cls = 1;
  if (a.causal) {
    // Every row sees the whole tile iff the first row's upper limit and the
    // last row's lower limit (window) both enclose it.
    const int64_t off = pair_off(a, pr);
    if (j1 > static_cast<int64_t>(sl.q0) + off) cls = 1;
    if (a.window > 0 && j0 <= static_cast<int64_t>(sl.q_last) + off - a.window) cls = 1;
  }
  if (a.has_mask) {
    const int c = a.summary[(static_cast<int64_t>(pr.b) * m_tiles + sl.mt) * n_tiles + nt];
    if (c == 0) return 0;
    if (c == 1) cls = 1;
  }
  return cls;
}

// Visibility of keys j0 .. j0 + 32 NW - 1 for query q, one bit per key: inside the
// entry's cache (j < len), within the causal limit (j <= q + off) and the
// window (j > q + off - window), and allowed by the mask row (nonzero byte),
// which is read as 16-byte vectors when aligned.
template <int NW>
__device__ __forceinline__ void visible_bits(uint32_t (&vb)[NW], const uint8_t* mrow, int j0,
                                             const PrefillArgs& a, const Pair& pr, int q,
                                             bool vec) {
  constexpr int W = 32 * NW;
  int64_t hi = pr.len, lo = 0;  // keys [lo, hi) pass the length, causal and window rules
  if (a.causal) {
    const int64_t off = pair_off(a, pr);
    hi = imin64(hi, static_cast<int64_t>(q) + off + 1);
    if (a.window > 0) lo = static_cast<int64_t>(q) + off - a.window + 1;
  }
  const int n = static_cast<int>(imax64(0, imin64(W, hi - j0)));
  const int n0 = static_cast<int>(imax64(0, imin64(n, lo - j0)));
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int k = n - 32 * w;
    const int k0 = n0 - 32 * w;
    const uint32_t below_hi = k >= 32 ? ~0u : (k <= 0 ? 0u : ((1u << k) - 1u));
    const uint32_t below_lo = k0 >= 32 ? ~0u : (k0 <= 0 ? 0u : ((1u << k0) - 1u));
    vb[w] = below_hi & ~below_lo;
  }
  if (mrow == nullptr) return;
  const uint8_t* m = mrow + j0;
  if (vec && n == W) {
#pragma unroll
    for (int v = 0; v < 2 * NW; ++v) {
      const uint4 x = *reinterpret_cast<const uint4*>(m + 16 * v);
      const uint32_t wds[4] = {x.x, x.y, x.z, x.w};
      uint32_t bits = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // one bit per nonzero byte: 0xff per nonzero byte, then gather the MSBs
        const uint32_t ne = __vcmpne4(wds[e], 0u);
        const uint32_t msb = (ne >> 7) & 0x01010101u;
        bits |= ((msb * 0x01020408u) >> 24) << (4 * e);  // byte k -> bit k
      }
      vb[v >> 1] &= (v & 1) ? ((bits << 16) | 0xFFFFu) : (bits | 0xFFFF0000u);
    }
  } else {
    for (int c = 0; c < n; ++c)
      if (m[c] == 0) vb[c >> 5] &= ~(1u << (c & 31));
  }
}

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) {
  // K-major, 128-byte swizzle: 8-row groups 1024 bytes apart; LBO unused (1).
  return smem_desc_sw128(saddr, 16, 1024);
}

__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t saddr, uint32_t chunk_bytes) {
  // MN-major, 128-byte swizzle: 64-element MN chunks `chunk_bytes` apart (LBO),
  // 8-row K groups 1024 bytes apart (SBO).
  return smem_desc_sw128(saddr, chunk_bytes, 1024);
}


// Position in the heavy-first list of the r-th item taken by CTA c: rounds
// alternate direction (c, then P-1-c, ...) so that every CTA's total causal
// work comes out nearly equal.
__device__ __forceinline__ int64_t snake(int64_t r, int64_t c, int64_t P) {
  return r * P + ((r & 1) ? (P - 1 - c) : c);
}

}  // namespace prefill
}  // namespace gqa
