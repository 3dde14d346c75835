// Prefill kernel (seq_q >= 2) on the 5th-generation tensor cores.
//
// The g query heads that share a kv head are packed into the 128 rows (M) of
// one tcgen05 tile: row r holds head h0 + r / qpt at query position
// q0 + r % qpt, with qpt = floor(128 / g) query positions per tile.  One K/V
// tile of 128 keys, staged once in shared memory, therefore serves every head
// of the group ("Multi-Query Attention", "Implementation": the shared K/V head
// is read once and broadcast); the expanded K/V of the reference solution's
// repeat_interleave never exists.
//
// Per 128x128 tile:   S = Q K^T       tcgen05.mma, A and B from shared memory,
//                                     fp32 accumulator in tensor memory (TMEM)
//                     P = softmax(S)  256 softmax threads, two per TMEM lane
//                                     (row), 64 keys each: scale, mask,
//                                     online max / sum
//                     O += P V        tcgen05.mma, A = P (bf16) from TMEM,
//                                     B = V from shared memory, O in TMEM
//
// Warp roles (352 threads, one CTA per SM, persistent over work tiles):
//   warps 0-7  softmax, O rescale and epilogue: warp w owns rows 32*(w%4) ..
//              +31 (TMEM lanes) and column half w/4 of S, P and O
//   warp 8     TMA producer of Q tiles and K tiles
//   warp 9     TMEM allocator and single-thread MMA issuer
//   warp 10    TMA producer of V tiles
// S is double-buffered in TMEM so that QK^T of tile j+1 runs on the tensor
// cores while the softmax threads work on tile j, and PV of tile j-1 runs
// behind it.  The running maximum is rescaled lazily: exponentials use a
// reference that may trail the true maximum by up to 2^8, and O and l are
// rescaled (O in TMEM) only when the maximum grows past that.
//
// Causal tiles above the diagonal are never visited; with a bool mask a
// pre-pass classifies every (query tile, key tile) pair as hidden / mixed /
// visible, hidden tiles are skipped and only mixed tiles read mask bytes.
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int BM = 128;  // rows per tile = TMEM lanes
constexpr int BN = 128;  // keys per K/V tile
constexpr int kSoftmaxWarps = 8;
constexpr int kWarpQK = 8;
constexpr int kWarpMMA = 9;
constexpr int kWarpV = 10;
constexpr int kPrefillThreads = 11 * 32;
constexpr int kStages = 2;  // depth of the K ring and of the V ring
constexpr int kQBufs = 2;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
// Exponentials of every eight computed on the FMA pipe (exp2_poly) rather
// than the MUFU unit; the rest use ex2.approx.
#ifndef GQA_PREFILL_EXP_EMU
#define GQA_PREFILL_EXP_EMU 0
#endif
constexpr int kEmuPerEight = GQA_PREFILL_EXP_EMU;

template <int D>
struct Layout {
  static constexpr int CH = D / 64;                  // 64-column (128-byte) chunks
  static constexpr int kChunkBytes = 128 * 128;      // 128 rows x 128 bytes
  static constexpr int kTileBytes = CH * kChunkBytes;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBufs * kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  static constexpr int kNumBars = 2 * kQBufs + 4 * kStages + 2 + 2 + 4 + 2 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kRedOff = kMiscOff + 16;               // row max / sum exchange
  static constexpr int kBytes = kRedOff + 8 * BM * 4 + 1024;  // + alignment slack
  // TMEM columns.
  static constexpr uint32_t kSCol0 = 0;     // S buffers at 0 and 128
  static constexpr uint32_t kOCol = 256;    // O: D columns
  static constexpr uint32_t kPCol0 = 256 + D;  // P buffers (bf16 pairs): 64 columns each
};

struct Item {
  int b, kv, mt, q0, q_last, nt_end;
};

__device__ __forceinline__ Item item_of(int64_t x, const PrefillArgs& a, int m_tiles, int qpt,
                                        int n_tiles) {
  Item it;
  const int64_t bh = static_cast<int64_t>(a.B) * a.Hkv;
  it.mt = m_tiles - 1 - static_cast<int>(x / bh);  // longest causal rows first
  const int bk = static_cast<int>(x % bh);
  it.b = bk / a.Hkv;
  it.kv = bk % a.Hkv;
  it.q0 = it.mt * qpt;
  it.q_last = min(it.q0 + qpt, a.Sq) - 1;
  it.nt_end = a.causal ? min(n_tiles, it.q_last / BN + 1) : n_tiles;
  return it;
}

// 0: every key hidden from every row (skip), 1: mixed (mask per element),
// 2: every key visible to every row.
__device__ __forceinline__ int tile_class(const PrefillArgs& a, const Item& it, int nt,
                                          int m_tiles, int n_tiles) {
  int cls = 2;
  const int j0 = nt * BN, j1 = j0 + BN - 1;
  if (j1 >= a.Sk) cls = 1;
  if (a.causal && j1 > it.q0) cls = 1;
  if (a.has_mask) {
    const int s = a.summary[(static_cast<int64_t>(it.b) * m_tiles + it.mt) * n_tiles + nt];
    if (s == 0) return 0;
    if (s == 1) cls = 1;
  }
  return cls;
}

// Visibility of keys j0 .. j0+127 for query q, one bit per key: inside the
// sequence (j < Sk), not in the future (causal: j <= q), and allowed by the
// mask row (nonzero byte), which is read as 16-byte vectors when aligned.
__device__ __forceinline__ void visible_bits(uint32_t (&vb)[4], const uint8_t* mrow, int j0,
                                             int Sk, int causal, int q, bool vec) {
  int n = Sk - j0;  // keys inside the sequence
  if (causal && q - j0 + 1 < n) n = q - j0 + 1;
  n = n < 0 ? 0 : (n > BN ? BN : n);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int k = n - 32 * w;
    vb[w] = k >= 32 ? ~0u : (k <= 0 ? 0u : ((1u << k) - 1u));
  }
  if (mrow == nullptr) return;
  const uint8_t* m = mrow + j0;
  if (vec && n == BN) {
#pragma unroll
    for (int v = 0; v < 8; ++v) {
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

template <int D>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    gqa_prefill_kernel(const __grid_constant__ CUtensorMap tmq,
                       const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const PrefillArgs a,
                       const int qpt, const int rows, const int m_tiles, const int n_tiles,
                       const int64_t work) {
  using L = Layout<D>;
  constexpr int CH = L::CH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + kQBufs;
  uint64_t* k_full = q_empty + kQBufs;
  uint64_t* k_empty = k_full + kStages;
  uint64_t* v_full = k_empty + kStages;
  uint64_t* v_empty = v_full + kStages;
  uint64_t* s_full = v_empty + kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_ready = p_full + 2;
  uint64_t* o_final = o_ready + 1;
  uint64_t* o_free = o_final + 1;
  uint64_t* mma_done = o_free + 1;
  uint64_t* xchg = mma_done + 1;   // [2]: row-max exchange between column halves
  uint64_t* lxchg = xchg + 2;      // [2]: row-sum exchange at the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQBufs; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSoftmaxWarps);
    }
    mbar_init(o_ready, 1);
    mbar_init(o_final, 1);
    mbar_init(o_free, kSoftmaxWarps);
    mbar_init(mma_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&xchg[i], kSoftmaxWarps);
      mbar_init(&lxchg[i], kSoftmaxWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Rows past qpt * g of a query tile are never written by TMA: zero them once.
  if (rows < BM && threadIdx.x < BM) {
    for (int qb = 0; qb < kQBufs; ++qb)
      for (int c = 0; c < CH; ++c) {
        uint8_t* base = smem + L::kQOff + qb * L::kTileBytes + c * L::kChunkBytes;
        for (int r = rows; r < BM; ++r)
          if (threadIdx.x < 8)
            reinterpret_cast<uint4*>(base + r * 128)[threadIdx.x] = make_uint4(0, 0, 0, 0);
      }
    fence_proxy_async_smem();
  }
  if (warp == kWarpMMA) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpQK || warp == kWarpV) {
    // ------------------------------------------------------------- producers
    if (lane == 0) {
      const bool is_qk = warp == kWarpQK;
      const CUtensorMap* map = is_qk ? &tmk : &tmv;
      uint64_t* full = is_qk ? k_full : v_full;
      uint64_t* empty = is_qk ? k_empty : v_empty;
      uint8_t* ring = smem + (is_qk ? L::kKOff : L::kVOff);
      prefetch_tmap(map);
      if (is_qk) prefetch_tmap(&tmq);
      uint32_t kt = 0;
      int64_t it = 0;
      int32_t last_round[kStages] = {-1, -1};
      int32_t last_q_round[kQBufs] = {-1, -1};
      bool ok = true;
      for (int64_t x = blockIdx.x; x < work && ok; x += gridDim.x, ++it) {
        const Item item = item_of(x, a, m_tiles, qpt, n_tiles);
        if (is_qk) {
          const int qb = static_cast<int>(it & 1);
          const uint32_t round = static_cast<uint32_t>(it >> 1);
          if (round > 0 && !mbar_wait(&q_empty[qb], (round - 1) & 1u, abort_flag, a.err,
                                      kErrPrefillWait)) {
            ok = false;
            break;
          }
          uint8_t* qdst = smem + L::kQOff + qb * L::kTileBytes;
          mbar_arrive_expect_tx(&q_full[qb], static_cast<uint32_t>(rows * 128 * CH));
          for (int c = 0; c < CH; ++c)
            tma_load_4d(qdst + c * L::kChunkBytes, &tmq, &q_full[qb], c * 64, item.q0,
                        item.kv * a.g, item.b);
          last_q_round[qb] = static_cast<int32_t>(round);
        }
        for (int nt = 0; nt < item.nt_end; ++nt) {
          if (tile_class(a, item, nt, m_tiles, n_tiles) == 0) continue;
          const int s = static_cast<int>(kt % kStages);
          const uint32_t round = kt / kStages;
          if (round > 0 &&
              !mbar_wait(&empty[s], (round - 1) & 1u, abort_flag, a.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          uint8_t* dst = ring + s * L::kTileBytes;
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(L::kTileBytes));
          for (int c = 0; c < CH; ++c)
            tma_load_4d(dst + c * L::kChunkBytes, map, &full[s], c * 64, nt * BN, item.kv,
                        item.b);
          last_round[s] = static_cast<int32_t>(round);
          ++kt;
        }
      }
      if (*abort_flag) {  // let every copy in flight land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if (last_round[s] >= 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(last_round[s]) & 1u);
        if (is_qk)
          for (int qb = 0; qb < kQBufs; ++qb)
            if (last_q_round[qb] >= 0)
              mbar_wait_drain(&q_full[qb], static_cast<uint32_t>(last_q_round[qb]) & 1u);
      }
    }
  } else if (warp == kWarpMMA) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t q_base = smem_u32(smem + L::kQOff);
      const uint32_t k_base = smem_u32(smem + L::kKOff);
      const uint32_t v_base = smem_u32(smem + L::kVOff);
      uint32_t kt = 0, J = 0;
      int64_t it = 0;
      bool ok = true;

      // PV of the tile with global index Jp (K/V ring slot kp): O (+)= P V.
      auto issue_pv = [&](uint32_t Jp, uint32_t kp, int local, int64_t item_idx) -> bool {
        if (!mbar_wait(&p_full[Jp & 1], (Jp >> 1) & 1u, abort_flag, a.err, kErrPrefillWait))
          return false;
        const int s = static_cast<int>(kp % kStages);
        if (!mbar_wait(&v_full[s], (kp / kStages) & 1u, abort_flag, a.err, kErrPrefillWait))
          return false;
        if (local == 0 && item_idx > 0 &&
            !mbar_wait(o_free, static_cast<uint32_t>((item_idx - 1) & 1), abort_flag, a.err,
                       kErrPrefillWait))
          return false;
        tc_fence_after();
        const uint32_t vs = v_base + s * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint32_t a_tmem = tmem + L::kPCol0 + (Jp & 1) * 64 + ks * 8;
          const uint64_t bdesc = mnmajor_desc(vs + ks * 16 * 128, L::kChunkBytes);
          tc_mma_ts(tmem + L::kOCol, a_tmem, bdesc, idesc_pv, (local > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(&v_empty[s]);
        tc_commit(o_ready);
        return true;
      };

      for (int64_t x = blockIdx.x; x < work && ok; x += gridDim.x, ++it) {
        const Item item = item_of(x, a, m_tiles, qpt, n_tiles);
        const int qb = static_cast<int>(it & 1);
        if (!mbar_wait(&q_full[qb], static_cast<uint32_t>((it >> 1) & 1), abort_flag, a.err,
                       kErrPrefillWait)) {
          ok = false;
          break;
        }
        const uint32_t qs = q_base + qb * L::kTileBytes;
        bool pending = false;
        uint32_t pJ = 0, pk = 0;
        int nloc = 0;
        for (int nt = 0; nt < item.nt_end && ok; ++nt) {
          if (tile_class(a, item, nt, m_tiles, n_tiles) == 0) continue;
          const int s = static_cast<int>(kt % kStages);
          if (!mbar_wait(&k_full[s], (kt / kStages) & 1u, abort_flag, a.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ks_base = k_base + s * L::kTileBytes;
          const uint32_t d_s = tmem + L::kSCol0 + (J & 1) * 128;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks >> 2) * L::kChunkBytes + (ks & 3) * 32;
            tc_mma_ss(d_s, kmajor_desc(qs + off), kmajor_desc(ks_base + off), idesc_qk,
                      ks > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[J & 1]);
          tc_commit(&k_empty[s]);
          if (pending && !issue_pv(pJ, pk, nloc - 1, it)) {
            ok = false;
            break;
          }
          pending = true;
          pJ = J;
          pk = kt;
          ++nloc;
          ++J;
          ++kt;
        }
        if (!ok) break;
        if (pending && !issue_pv(pJ, pk, nloc - 1, it)) {
          ok = false;
          break;
        }
        tc_commit(&q_empty[qb]);
        if (nloc == 0 && it > 0 &&
            !mbar_wait(o_free, static_cast<uint32_t>((it - 1) & 1), abort_flag, a.err,
                       kErrPrefillWait)) {
          ok = false;
          break;
        }
        tc_commit(o_final);
      }
      // Every MMA issued so far has completed before TMEM is released.
      tc_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------- softmax
    // Eight warps: warp w serves TMEM lanes 32*(w % 4) .. +31 (its rows) and
    // column half hf = w / 4 of each S tile (64 keys), of P and of O, so two
    // warps per SM sub-partition share every row.  The halves exchange their
    // row maxima through shared memory and an mbarrier once per tile, and
    // their partial row sums once per work tile.
    const int quad = warp & 3, hf = warp >> 2;
    const int row = quad * 32 + lane;  // TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int hh = row / qpt, qi = row % qpt;
    constexpr int DH = D / 2;  // O columns per half
    // Mask rows can be read as 16-byte vectors when base and strides allow.
    const bool mask_vec = a.has_mask && ((reinterpret_cast<uintptr_t>(a.mask) & 15u) == 0) &&
                          (a.ms[0] % 16 == 0) && (a.ms[1] % 16 == 0);
    float* red = reinterpret_cast<float*>(smem + L::kRedOff);  // [2 parity][2 halves][BM]
    float* lred = red + 4 * BM;                                // [2 parity][2 halves][BM]
    uint32_t J = 0;
    int64_t it = 0;
    bool ok = true;
    for (int64_t x = blockIdx.x; x < work && ok; x += gridDim.x, ++it) {
      const Item item = item_of(x, a, m_tiles, qpt, n_tiles);
      const int q = item.q0 + qi;
      const bool row_valid = row < rows && q < a.Sq;
      const uint8_t* mrow =
          (a.has_mask && row_valid) ? a.mask + item.b * a.ms[0] + static_cast<int64_t>(q) * a.ms[1]
                                    : nullptr;
      float m_ref = -INFINITY, l = 0.f;
      int nloc = 0;
      for (int nt = 0; nt < item.nt_end; ++nt) {
        const int cls = tile_class(a, item, nt, m_tiles, n_tiles);
        if (cls == 0) continue;
        if (!mbar_wait(&s_full[J & 1], (J >> 1) & 1u, abort_flag, a.err, kErrPrefillWait)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // This half's 64 scores of the row.  Fully visible tiles keep raw
        // scores and fold the scale into one FMA per element; other tiles go
        // to the base-2 domain with -inf where a key is hidden.
        const bool fast = (cls == 2) && (a.scale_log2 >= 0.f);
        float t[64];
        {
          uint32_t r[64];
          const uint32_t sbase = tmem + lane_base + L::kSCol0 + (J & 1) * 128 + hf * 64;
          tmem_ld32(sbase, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(sbase + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_ld_wait();
          if (fast) {
#pragma unroll
            for (int c = 0; c < 64; ++c) t[c] = __uint_as_float(r[c]);
          } else {
            uint32_t vb[4];
            visible_bits(vb, row_valid ? mrow : nullptr, nt * BN, a.Sk, a.causal, q, mask_vec);
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int cc = hf * 64 + c;
              t[c] = ((vb[cc >> 5] >> (cc & 31)) & 1u) ? __uint_as_float(r[c]) * a.scale_log2
                                                       : -INFINITY;
            }
          }
        }
        float mx;
        {
          float part[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) part[e] = t[e];
#pragma unroll
          for (int c = 8; c < 64; ++c) part[c & 7] = fmaxf(part[c & 7], t[c]);
          mx = fmaxf(fmaxf(fmaxf(part[0], part[1]), fmaxf(part[2], part[3])),
                     fmaxf(fmaxf(part[4], part[5]), fmaxf(part[6], part[7])));
          if (fast) mx *= a.scale_log2;
        }
        // Row maximum over both halves.
        red[((J & 1) * 2 + hf) * BM + row] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xchg[J & 1]);
        if (!mbar_wait(&xchg[J & 1], (J >> 1) & 1u, abort_flag, a.err, kErrPrefillWait)) {
          ok = false;
          break;
        }
        mx = fmaxf(mx, red[((J & 1) * 2 + (hf ^ 1)) * BM + row]);
        const float m_new = fmaxf(m_ref, mx);
        const bool grow = m_new > m_ref + kRescaleLog2;  // also true for -inf -> finite
        const float alpha = grow ? fast_exp2(m_ref - m_new) : 1.f;  // 0 when m_ref = -inf
        const bool o_live = grow && nloc > 0 && m_ref != -INFINITY;
        if (__any_sync(0xffffffffu, o_live)) {
          // O holds earlier tiles' P V with the old reference: rescale this half.
          if (!mbar_wait(o_ready, (J - 1) & 1u, abort_flag, a.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = o_live ? alpha : 1.f;
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t r[32];
            const uint32_t oa = tmem + lane_base + L::kOCol + hf * DH + c * 32;
            tmem_ld32(oa, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
            tmem_st16(oa, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
            tmem_st16(oa + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
          }
          tmem_st_wait();
        }
        if (grow) {
          l *= alpha;
          m_ref = m_new;
        }
        const float ref = exp_ref(m_ref);
        // P = 2^(t - ref) as bf16 pairs into TMEM (A operand of the PV MMA);
        // kEmuPerEight of every eight exponentials run on the FMA pipe.
        float lp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) lp[e] = 0.f;
        const float sc = fast ? a.scale_log2 : 1.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = c * 32 + 2 * e, c1 = c0 + 1;
            const float x0 = fmaf(t[c0], sc, -ref);
            const float x1 = fmaf(t[c1], sc, -ref);
            const float p0 = ((c0 & 7) < kEmuPerEight) ? exp2_poly(x0) : fast_exp2(x0);
            const float p1 = ((c1 & 7) < kEmuPerEight) ? exp2_poly(x1) : fast_exp2(x1);
            lp[c0 & 7] += p0;
            lp[c1 & 7] += p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tmem + lane_base + L::kPCol0 + (J & 1) * 64 + hf * 32 + c * 16, pk);
        }
        l += ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[J & 1]);
        ++J;
        ++nloc;
      }
      if (!ok) break;
      // Epilogue: out = O / l for this row and this half of the columns.
      if (!mbar_wait(o_final, static_cast<uint32_t>(it & 1), abort_flag, a.err,
                     kErrPrefillWait)) {
        ok = false;
        break;
      }
      tc_fence_after();
      lred[((it & 1) * 2 + hf) * BM + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&lxchg[it & 1]);
      if (!mbar_wait(&lxchg[it & 1], static_cast<uint32_t>((it >> 1) & 1), abort_flag, a.err,
                     kErrPrefillWait)) {
        ok = false;
        break;
      }
      const float l_row = l + lred[((it & 1) * 2 + (hf ^ 1)) * BM + row];
      uint16_t* orow = a.out + item.b * a.os[0] +
                       static_cast<int64_t>(item.kv * a.g + (hh < a.g ? hh : 0)) * a.os[1] +
                       static_cast<int64_t>(q) * a.os[2] + hf * DH;
      const float inv_l = 1.f / l_row;  // l == 0: no visible key, NaN output
      if (nloc > 0) {
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + L::kOCol + hf * DH + c * 32, r);
          tmem_ld_wait();
          if (row_valid) {
#pragma unroll
            for (int v8 = 0; v8 < 4; ++v8) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(r[v8 * 8 + 0]) * inv_l,
                                __uint_as_float(r[v8 * 8 + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(r[v8 * 8 + 2]) * inv_l,
                                __uint_as_float(r[v8 * 8 + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(r[v8 * 8 + 4]) * inv_l,
                                __uint_as_float(r[v8 * 8 + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(r[v8 * 8 + 6]) * inv_l,
                                __uint_as_float(r[v8 * 8 + 7]) * inv_l);
              reinterpret_cast<uint4*>(orow + c * 32)[v8] = w;
            }
          }
        }
      } else if (row_valid) {
        const float nanv = __int_as_float(0x7fc00000);
        const uint32_t nn = pack_bf16x2(nanv, nanv);
        for (int d = 0; d < DH; d += 8)
          *reinterpret_cast<uint4*>(orow + d) = make_uint4(nn, nn, nn, nn);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

// summary[b][mt][nt] = 0 (all hidden), 1 (mixed) or 2 (all visible) over
// mask[b, q0 : q0 + qpt, nt*128 : nt*128 + 128].
__global__ void __launch_bounds__(128)
    gqa_mask_summary_kernel(const uint8_t* __restrict__ mask, int64_t ms0, int64_t ms1,
                            uint8_t* __restrict__ summary, int Sq, int Sk, int qpt, int m_tiles,
                            int n_tiles) {
  const int mt = blockIdx.x, b = blockIdx.y;
  const int q0 = mt * qpt;
  const int qn = min(qpt, Sq - q0);
  const uint8_t* base = mask + b * ms0;
  for (int nt = 0; nt < n_tiles; ++nt) {
    const int j = nt * BN + threadIdx.x;
    bool any1 = false, any0 = false;
    if (threadIdx.x < BN && j < Sk) {
      for (int r = 0; r < qn; ++r) {
        const uint8_t v = base[static_cast<int64_t>(q0 + r) * ms1 + j];
        any1 |= v != 0;
        any0 |= v == 0;
      }
    }
    const int o1 = __syncthreads_or(any1);
    const int o0 = __syncthreads_or(any0);
    if (threadIdx.x == 0)
      summary[(static_cast<int64_t>(b) * m_tiles + mt) * n_tiles + nt] =
          static_cast<uint8_t>(o1 ? (o0 ? 1 : 2) : 0);
  }
}

template <int D>
int launch_prefill_t(const PrefillShape& s, const PrefillArgs& a, const CUtensorMap& tmq,
                     const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream) {
  if (a.has_mask) {
    gqa_mask_summary_kernel<<<dim3(s.m_tiles, a.B), 128, 0, stream>>>(
        a.mask, a.ms[0], a.ms[1], a.summary, a.Sq, a.Sk, s.qpt, s.m_tiles, s.n_tiles);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  }
  auto kern = gqa_prefill_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Layout<D>::kBytes) != cudaSuccess)
    return GQA_ERR_CUDA;
  kern<<<s.grid, kPrefillThreads, Layout<D>::kBytes, stream>>>(tmq, tmk, tmv, a, s.qpt, s.rows,
                                                                s.m_tiles, s.n_tiles, s.work);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace

PrefillShape plan_prefill(const gqa_problem& p, int sm_count) {
  PrefillShape s{};
  const int64_t g = p.heads_q / p.heads_kv;
  s.D = static_cast<int>(p.head_dim);
  s.qpt = static_cast<int>(BM / g);
  s.rows = static_cast<int>(s.qpt * g);
  s.m_tiles = static_cast<int>((p.seq_q + s.qpt - 1) / s.qpt);
  s.n_tiles = static_cast<int>((p.seq_k + BN - 1) / BN);
  s.work = p.batch * p.heads_kv * s.m_tiles;
  s.grid = static_cast<int>(s.work < sm_count ? s.work : sm_count);
  if (s.grid < 1) s.grid = 1;
  s.smem_bytes = s.D == 128 ? Layout<128>::kBytes : Layout<64>::kBytes;
  s.summary_offset = 256;
  s.summary_bytes = p.has_mask ? p.batch * s.m_tiles * s.n_tiles : 0;
  return s;
}

int launch_prefill(const gqa_problem& p, const PrefillShape& s, const PrefillArgs& a,
                   const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                   cudaStream_t stream) {
  (void)p;
  if (s.D == 128) return launch_prefill_t<128>(s, a, tmq, tmk, tmv, stream);
  if (s.D == 64) return launch_prefill_t<64>(s, a, tmq, tmk, tmv, stream);
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace gqa
