// Prefill with two query tiles in flight per SM.
//
// The g query heads of a kv head are packed into 128-row tiles as in the
// other prefill kernel (row r: head h0 + r / qpt, query q0 + r % qpt), and
// one K / V tile serves every head of the group ("Multi-Query Attention",
// "Implementation": the shared K/V head is read once; the expanded K/V of
// "28. Grouped-Query Attention (GQA)", "Reference solution", never exists).
//
// A work item is two consecutive query tiles A = 2i and B = 2i + 1 of one
// (batch, kv head).  TMEM holds S_A, S_B (128 columns each) and O_A, O_B (D
// each); Q_A and Q_B stay in shared memory:
//
//   S_X = Q_X K^T    tcgen05.mma, A = Q_X and B = K from shared memory
//   O_X += P_X V     tcgen05.mma, A = P_X from TMEM (over the first half of
//                    S_X), B = V from shared memory
//
// One softmax warpgroup per query tile, one thread per row holding all 128
// keys of its S row: the maximum and the row sum need no exchange between
// threads, and while warpgroup A turns S_A into P_A the tensor core computes
// tile B's products, and the other way round.  The MMA warp issues, per
// key tile u:  PV_A(u), QK_A(u+1), PV_B(u), QK_B(u+1).  tcgen05 operations of
// one thread execute in issue order, so QK_X(u+1), which overwrites P_X(u),
// follows PV_X(u), and the commit that signals S_X(u+1) also means that
// PV_X(u) has completed: the softmax may rescale O_X as soon as it sees S_X.
// Each K / V tile is staged once for both query tiles.
//
// Warp roles (384 threads, one CTA per SM, persistent over items):
//   warps 0-3  softmax, O rescale and epilogue of tile A (thread t: row t)
//   warps 4-7  the same for tile B
//   warp 8     TMA producer of Q tiles and K tiles
//   warp 9     TMEM allocator and MMA warp (one elected lane issues)
//   warp 10    TMA producer of V tiles (warp 11 idles)
// Per-sequence lengths and paged caches (the KVX instances): an item's key
// range ends at its entry's length; the one key tile that reaches past it has
// its V rows there zeroed in shared memory by the V producer before its PVs
// (0 times a NaN left in the cache would still reach O); a paged cache's
// 128-key tile is two 64-key boxes, each inside one page.  With a mask or
// lengths the items' costs differ, and a one-CTA sort orders them heaviest
// first before the launch.
// Every wait is bounded; a thread that gives up sets the abort flag and the
// error word, every role leaves its loop, copies in flight are waited for and
// TMEM is freed after a block-wide barrier.
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "prefill_common.cuh"
#include "ptx.cuh"

namespace gqa {
namespace {

using namespace prefill;

constexpr int kPPThreads = 12 * 32;
constexpr int kWarpQK = 8;
constexpr int kWarpMMA = 9;
constexpr int kWarpV = 10;
// Register split (setmaxnreg): the softmax threads keep a whole S row (128
// values) in registers.
constexpr int kLaunchRegs = 168;
constexpr int kIoRegs = 120;
constexpr int kSoftmaxRegs = 192;
static_assert(128 * kIoRegs + 256 * kSoftmaxRegs <= kPPThreads * kLaunchRegs,
              "register split must fit in the launch allocation");
constexpr uint32_t kTmemCols = 512;
// At head dim 64, one pair of columns in four takes its exponentials on the
// FMA pipe (exp2_poly_x2), the others on the MUFU unit: 16 exponentials per
// clock per SM, which the two tiles' 2 x 128 x 128 per key tile otherwise keep
// busy for 2048 cycles, about 80% of the key tile's time at that head dim.  At
// head dim 128 the tensor core's share is twice as large and the exponentials
// all stay on the MUFU unit (a share on the FMA pipe was slower there), and so
// they do in the instances with lengths or a paged cache, whose softmax has no
// registers to spare for it.
template <int D, bool KVX>
__host__ __device__ constexpr bool poly_pair(int e) {
  return D == 64 && !KVX && e % 4 == 3;
}

// 2^x for two packed fp32 lanes on the FMA pipe.  Cody and Waite style
// reduction: n = round(x) (the low mantissa bits of x + 1.5 * 2^23), f = x - n
// in [-1/2, 1/2]; 2^f by the degree-3 polynomial of least maximum relative
// error on [-1/2, 1/2] (own Remez exchange fit: c3 = 5.517166853e-02,
// c2 = 2.426111251e-01, c1 = 6.932609677e-01, c0 = 9.999280572e-01, maximum
// relative error 7.5e-5, below the 16-bit rounding of P); 2^n by adding n to
// the exponent field ((t's bits << 23) is n << 23: the bits of 1.5 * 2^23
// shift out).  x is first raised to -126 (NaN kept) so that the exponent
// cannot wrap: -inf and anything below -126 give 2^-126 instead of 0, which
// the softmax tolerates (a row with no visible key is told by its running
// maximum, not by its sum).  One asm block, so that the packed constants live
// only inside it.
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x) {
  uint64_t y;
  asm("{\n\t"
      ".reg .f32 a0, a1;\n\t"
      ".reg .b64 xc, t, nf, f, q, k, k2;\n\t"
      ".reg .b32 q0, q1, t0, t1;\n\t"
      "mov.b64 {a0, a1}, %1;\n\t"
      "max.NaN.f32 a0, a0, 0fC2FC0000;\n\t"
      "max.NaN.f32 a1, a1, 0fC2FC0000;\n\t"
      "mov.b64 xc, {a0, a1};\n\t"
      "mov.b64 k, 0x4B4000004B400000;\n\t"
      "add.rn.f32x2 t, xc, k;\n\t"
      "mov.b64 k, 0xCB400000CB400000;\n\t"
      "add.rn.f32x2 nf, t, k;\n\t"
      "mov.b64 k, 0xBF800000BF800000;\n\t"
      "fma.rn.f32x2 f, nf, k, xc;\n\t"
      "mov.b64 k, 0x3D61FBB03D61FBB0;\n\t"
      "mov.b64 k2, 0x3E786F0D3E786F0D;\n\t"
      "fma.rn.f32x2 q, f, k, k2;\n\t"
      "mov.b64 k, 0x3F31798D3F31798D;\n\t"
      "fma.rn.f32x2 q, q, f, k;\n\t"
      "mov.b64 k, 0x3F7FFB493F7FFB49;\n\t"
      "fma.rn.f32x2 q, q, f, k;\n\t"
      "mov.b64 {q0, q1}, q;\n\t"
      "mov.b64 {t0, t1}, t;\n\t"
      "shl.b32 t0, t0, 23;\n\t"
      "shl.b32 t1, t1, 23;\n\t"
      "add.u32 q0, q0, t0;\n\t"
      "add.u32 q1, q1, t1;\n\t"
      "mov.b64 %0, {q0, q1};\n\t"
      "}"
      : "=l"(y)
      : "l"(x));
  return y;
}

template <int D>
struct PPLayout {
  static_assert(D == 64 || D == 128, "head_dim is padded to 64 or 128");
  static constexpr int CH = D / 64;                  // 64-column (128-byte) chunks
  static constexpr int kChunk = 128 * 128;           // 128 rows (or keys) x 128 bytes
  static constexpr int kTile = CH * kChunk;          // one Q, K or V tile
  static constexpr int kStages = D == 128 ? 2 : 4;   // depth of the K ring and of the V ring
  static constexpr int kQOff = 0;                    // Q_A, then Q_B
  static constexpr int kKOff = kQOff + 2 * kTile;
  static constexpr int kVOff = kKOff + kStages * kTile;
  static constexpr int kBarOff = kVOff + kStages * kTile;
  // q_full[2], q_empty[2], k_full[S], k_empty[S], v_full[S], v_empty[S],
  // s_full[2], p_full[2], o_final[2], o_free[2], mma_done, v_fix[S]
  static constexpr int kNumBars = 4 + 4 * kStages + 8 + 1 + kStages;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSchedOff = kMiscOff + 16;  // the MMA warp's key-tile list of an item
  static constexpr int kBytes = kSchedOff + kMaxPPTiles + 1024;  // + alignment slack
  // TMEM columns of S_X and O_X (X = 0: tile A, 1: tile B).
  __device__ static constexpr uint32_t s_col(int X) { return static_cast<uint32_t>(X) * 128u; }
  __device__ static constexpr uint32_t o_col(int X) {
    return 256u + static_cast<uint32_t>(X) * static_cast<uint32_t>(D);
  }
};

// Query tile X of item x (late, long causal items first), with its key
// range; a tile index past the last query tile gives a dead tile (no keys).
struct PPTile {
  Pair pr;
  Slot sl;
};

__device__ __forceinline__ PPTile pp_tile(int64_t x, int X, const PrefillArgs& a, int m_tiles,
                                          int qpt, int n_tiles) {
  PPTile t;
  const int64_t bh = static_cast<int64_t>(a.B) * a.Hkv;
  const int n2 = (m_tiles + 1) / 2;
  const int bk = static_cast<int>(x % bh);
  const int mt = 2 * (n2 - 1 - static_cast<int>(x / bh)) + X;
  t.pr.b = bk / a.Hkv;
  t.pr.kv = bk % a.Hkv;
  t.pr.mt0 = mt;
  t.pr.len = a.Sk;
  if (a.lens != nullptr) {  // out-of-range lengths are clamped (and reported at kernel start)
    const int len = a.lens[t.pr.b];
    t.pr.len = len < 0 ? 0 : (len > a.Sk ? a.Sk : len);
  }
  t.sl = slot_of(t.pr, a, qpt);
  t.sl.live = mt < m_tiles;
  if (!t.sl.live || t.sl.key_hi <= t.sl.key_lo) {
    t.pr.nt_beg = t.pr.nt_end = 0;
  } else {
    t.pr.nt_beg = static_cast<int>(t.sl.key_lo / BN);
    t.pr.nt_end = min(n_tiles, static_cast<int>((t.sl.key_hi + BN - 1) / BN));
    if (a.bounds != nullptr) {  // with a mask: drop the all-hidden tiles at either end
      const int2 bd = *reinterpret_cast<const int2*>(a.bounds + (static_cast<int64_t>(t.pr.b) *
                                                                 m_tiles + mt) * 2);
      t.pr.nt_beg = max(t.pr.nt_beg, bd.x);
      t.pr.nt_end = min(t.pr.nt_end, bd.y);
      if (t.pr.nt_end <= t.pr.nt_beg) t.pr.nt_beg = t.pr.nt_end = 0;
    }
  }
  return t;
}

// Class of key tile u for a query tile: 0 skipped, 1 mixed, 2 fully visible.
__device__ __forceinline__ int pp_class(const PPTile& q, int u, const PrefillArgs& a, int m_tiles,
                                        int n_tiles) {
  if (u < q.pr.nt_beg || u >= q.pr.nt_end) return 0;
  return tile_class(a, q.pr, q.sl, u, m_tiles, n_tiles);
}

// KVX: the launch has per-sequence lengths or a paged cache (the V rows past
// a length are zeroed before their PV; K / V tiles of a paged cache are two
// 64-key boxes, each inside one page).
template <int D, bool F16, bool KVX>
__global__ void __launch_bounds__(kPPThreads, 1)
    gqa_prefill_pp_kernel(const __grid_constant__ CUtensorMap tmq,
                          const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv, const PrefillArgs a,
                          const int qpt, const int rows, const int m_tiles, const int n_tiles,
                          const int64_t items, const PagedKV pg) {
  using L = PPLayout<D>;
  constexpr int CH = L::CH;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;              // [X] Q_X landed
  uint64_t* q_empty = q_full + 2;       // [X] the item's last QK_X done
  uint64_t* k_full = q_empty + 2;       // [stage] K tile landed
  uint64_t* k_empty = k_full + S;       // [stage] the QKs reading it done
  uint64_t* v_full = k_empty + S;       // [stage] V tile landed
  uint64_t* v_empty = v_full + S;       // [stage] the PVs reading it done
  uint64_t* s_full = v_empty + S;       // [X] S_X done (and every earlier PV_X)
  uint64_t* p_full = s_full + 2;        // [X] P_X written (one arrival per softmax warp)
  uint64_t* o_final = p_full + 2;       // [X] the item's last PV_X done
  uint64_t* o_free = o_final + 2;       // [X] O_X read by the epilogue (one arrival per warp)
  uint64_t* mma_done = o_free + 2;      // every MMA done
  uint64_t* v_fix = mma_done + 1;       // [stage] (KVX): the V rows past the length zeroed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  uint8_t* sched = smem + L::kSchedOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp
      mbar_init(&o_final[i], 1);
      mbar_init(&o_free[i], 4);  // one arrival per softmax warp
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    if (KVX)
      for (int i = 0; i < S; ++i) mbar_init(&v_fix[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (KVX && a.lens != nullptr && blockIdx.x == 0) {
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
      const int len = a.lens[b];
      if (len < 0 || len > a.Sk) atomicOr(a.err, kErrKvLength);
    }
  }
  // Q rows past qpt * g of a tile are never written by TMA: zero them once.
  if (rows < BM && threadIdx.x < 8) {
    for (int X = 0; X < 2; ++X)
      for (int c = 0; c < CH; ++c) {
        uint8_t* base = smem + L::kQOff + X * L::kTile + c * L::kChunk;
        for (int r = rows; r < BM; ++r)
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

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIoRegs));
    if ((warp == kWarpQK || warp == kWarpV) && lane == 0) {
      // ------------------------------------------------------------ producers
      const bool is_qk = warp == kWarpQK;
      const CUtensorMap* map = is_qk ? &tmk : &tmv;
      uint64_t* full = is_qk ? k_full : v_full;
      uint64_t* empty = is_qk ? k_empty : v_empty;
      uint8_t* ring = smem + (is_qk ? L::kKOff : L::kVOff);
      prefetch_tmap(map);
      if (is_qk) prefetch_tmap(&tmq);
      uint32_t kt = 0;         // key tiles loaded over the kernel
      uint32_t nq[2] = {0, 0};  // Q tiles loaded into each buffer
      int64_t it = 0;
      bool ok = true;
      for (int64_t x = snake(0, blockIdx.x, gridDim.x); x < items && ok;
           ++it, x = snake(it, blockIdx.x, gridDim.x)) {
        const int64_t xi = a.order != nullptr ? a.order[x] : x;
        const PPTile qa = pp_tile(xi, 0, a, m_tiles, qpt, n_tiles);
        const PPTile qb = pp_tile(xi, 1, a, m_tiles, qpt, n_tiles);
        if (is_qk) {
#pragma unroll
          for (int X = 0; X < 2; ++X) {
            if (it > 0 && !mbar_wait(&q_empty[X], static_cast<uint32_t>((it - 1) & 1), abort_flag,
                                     a.err, kErrPrefillWait)) {
              ok = false;
              break;
            }
            const Pair& pr = X == 0 ? qa.pr : qb.pr;
            mbar_arrive_expect_tx(&q_full[X], static_cast<uint32_t>(rows * 128 * CH));
            for (int c = 0; c < CH; ++c)
              tma_load_4d(smem + L::kQOff + X * L::kTile + c * L::kChunk, &tmq, &q_full[X], c * 64,
                          pr.mt0 * qpt, pr.kv * a.g, pr.b);
            ++nq[X];
          }
        }
        const int t_lo = min(qa.pr.nt_end > qa.pr.nt_beg ? qa.pr.nt_beg : 1 << 30,
                             qb.pr.nt_end > qb.pr.nt_beg ? qb.pr.nt_beg : 1 << 30);
        const int t_hi = max(qa.pr.nt_end, qb.pr.nt_end);
        for (int t = t_lo; t < t_hi && ok; ++t) {
          if (pp_class(qa, t, a, m_tiles, n_tiles) == 0 && pp_class(qb, t, a, m_tiles, n_tiles) == 0)
            continue;
          const int s = static_cast<int>(kt % S);
          const uint32_t round = kt / S;
          if (round > 0 &&
              !mbar_wait(&empty[s], (round - 1) & 1u, abort_flag, a.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], L::kTile);
          uint8_t* dst = ring + s * L::kTile;
          if (KVX && pg.bt != nullptr) {
            // Two 64-key boxes, each inside one page (page_size is a multiple
            // of 64).  A box that starts at or past the entry's length reads an
            // out-of-range page, which the copy fills with zeros; a page index
            // outside the pool for keys in use is reported and read the same way.
            for (int hb = 0; hb < 2; ++hb) {
              const int key = t * BN + hb * 64;
              int page = pg.num_pages;
              if (key < qa.pr.len) {
                page = __ldg(pg.bt + qa.pr.b * pg.bt_stride + key / pg.page_size);
                if (page < 0 || page >= pg.num_pages) {
                  atomicOr(a.err, kErrPage);
                  page = pg.num_pages;
                }
              }
              for (int c = 0; c < CH; ++c)
                tma_load_4d(dst + c * L::kChunk + hb * 64 * 128, map, &full[s], c * 64,
                            key % pg.page_size, qa.pr.kv, page);
            }
          } else {
            for (int c = 0; c < CH; ++c)
              tma_load_4d(dst + c * L::kChunk, map, &full[s], c * 64, t * BN, qa.pr.kv, qa.pr.b);
          }
          ++kt;
          // The V rows of the entry's last tile past its length hold whatever
          // the cache holds there (NaN included), and P = 0 does not hide a
          // NaN in P V: once the tile has landed they are zeroed, and the MMA
          // waits for that too.  Only the last tile an item visits can reach
          // past the length.
          if (KVX && !is_qk && (static_cast<int64_t>(t) + 1) * BN > qa.pr.len) {
            if (!mbar_wait(&full[s], round & 1u, abort_flag, a.err, kErrPrefillWait)) {
              ok = false;
              break;
            }
            const int valid = qa.pr.len - t * BN;  // 1 .. BN - 1: the tile holds a key below len
            for (int c = 0; c < CH; ++c) {
              uint4* row0 = reinterpret_cast<uint4*>(dst + c * L::kChunk + valid * 128);
              for (int i = 0; i < (BN - valid) * 8; ++i) row0[i] = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            mbar_arrive(&v_fix[s]);
          }
        }
      }
      // On an abort, the copies still in flight land before the CTA leaves.
      if (*abort_flag) {
        for (uint32_t j = kt > static_cast<uint32_t>(S) ? kt - S : 0; j < kt; ++j)
          mbar_wait_drain(&full[j % S], (j / S) & 1u);
        for (int X = 0; X < 2; ++X)
          if (nq[X] > 0) mbar_wait_drain(&q_full[X], (nq[X] - 1) & 1u);
      }
    } else if (warp == kWarpMMA) {
      // ------------------------------------------------------------ MMA warp
      // The whole warp walks the schedule and takes every wait (made
      // warp-uniform by a vote); one elected lane issues the MMAs and their
      // commits.  A lone issuing thread in a diverged warp leaves the tensor
      // core idle ~200 cycles at each wait or data-dependent branch between
      // MMA groups; a converged warp does not.  elect.sync picks the lowest
      // lane of a full warp, so one thread issues every tcgen05 operation
      // and they execute in issue order.
      constexpr uint32_t idesc_qk = F16 ? idesc_f16_f32(BM, BN, 0, 0) : idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = F16 ? idesc_f16_f32(BM, D, 0, 1) : idesc_bf16_f32(BM, D, 0, 1);
      const uint64_t dq0 = kmajor_desc(smem_u32(smem + L::kQOff));
      const uint64_t dk0 = kmajor_desc(smem_u32(smem + L::kKOff));
      const uint64_t dv0 = mnmajor_desc(smem_u32(smem + L::kVOff), L::kChunk);
      uint32_t kt = 0;          // key tiles (K / V stages) consumed over the kernel
      uint32_t np[2] = {0, 0};  // P_X tiles consumed over the kernel
      uint32_t fix_parity = 0;  // bit s (KVX): parity of the next v_fix[s] phase
      int64_t it = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_hot(bar, parity, abort_flag, a.err, kErrPrefillWait));
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
      };
      auto qk = [&](int X, uint32_t idx) {
        const uint64_t dq = dq0 + ((X * L::kTile) >> 4);
        const uint64_t dk = dk0 + (((idx % S) * L::kTile) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            tc_mma_ss(tmem + L::s_col(X), dq + (((k >> 2) * L::kChunk + (k & 3) * 32) >> 4),
                      dk + (((k >> 2) * L::kChunk + (k & 3) * 32) >> 4), idesc_qk, k > 0 ? 1u : 0u);
          tc_commit(&s_full[X]);
        }
        __syncwarp();
      };
      auto pv = [&](int X, uint32_t idx, bool first) {
        const uint64_t dv = dv0 + (((idx % S) * L::kTile) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < BN / 16; ++k)
            tc_mma_ts(tmem + L::o_col(X), tmem + L::s_col(X) + k * 8, dv + ((k * 16 * 128) >> 4),
                      idesc_pv, (!first || k > 0) ? 1u : 0u);
        }
        __syncwarp();
      };
      for (int64_t x = snake(0, blockIdx.x, gridDim.x); x < items && ok;
           ++it, x = snake(it, blockIdx.x, gridDim.x)) {
        const int64_t xi = a.order != nullptr ? a.order[x] : x;
        const PPTile qa = pp_tile(xi, 0, a, m_tiles, qpt, n_tiles);
        const PPTile qb = pp_tile(xi, 1, a, m_tiles, qpt, n_tiles);
        // The item's key tiles that some tile works on, in order, one byte
        // each in shared memory (bit X: tile X computes it); tile classes may
        // read mask summaries from global memory, so they are taken once per
        // item, 32 key tiles at a time across the warp, off the per-tile path.
        const int t_lo = min(qa.pr.nt_end > qa.pr.nt_beg ? qa.pr.nt_beg : 1 << 30,
                             qb.pr.nt_end > qb.pr.nt_beg ? qb.pr.nt_beg : 1 << 30);
        const int t_hi = max(qa.pr.nt_end, qb.pr.nt_end);
        int n = 0, nX[2] = {0, 0};
        int t_last = -1;  // the last key tile computed
        for (int t0 = t_lo; t0 < t_hi; t0 += 32) {
          const int t = t0 + lane;
          uint32_t f = 0;
          if (t < t_hi)
            f = (pp_class(qa, t, a, m_tiles, n_tiles) != 0 ? 1u : 0u) |
                (pp_class(qb, t, a, m_tiles, n_tiles) != 0 ? 2u : 0u);
          const uint32_t any = __ballot_sync(0xffffffffu, f != 0u);
          if (f != 0u) sched[n + __popc(any & ((1u << lane) - 1u))] = static_cast<uint8_t>(f);
          n += __popc(any);
          nX[0] += __popc(__ballot_sync(0xffffffffu, (f & 1u) != 0u));
          nX[1] += __popc(__ballot_sync(0xffffffffu, (f & 2u) != 0u));
          if (any != 0u) t_last = t0 + 31 - __clz(any);
        }
        __syncwarp();  // sched written by every lane, read by every lane below
        // That tile reaches past the entry's length: its V rows there are
        // zeroed by the V producer before its PVs.
        const bool last_fix = KVX && n > 0 && (static_cast<int64_t>(t_last) + 1) * BN > qa.pr.len;
#pragma unroll
        for (int X = 0; X < 2; ++X)
          if (ok) ok = wait(&q_full[X], static_cast<uint32_t>(it & 1));
        if (!ok) break;
        tc_fence_after();
        int qkX[2] = {0, 0};  // QK_X / PV_X issued for this item
        int pvX[2] = {0, 0};
        if (n > 0) {  // the first key tile: its QKs
          ok = wait(&k_full[kt % S], (kt / S) & 1u);
          if (!ok) break;
          tc_fence_after();
          const uint32_t f = sched[0];
#pragma unroll
          for (int X = 0; X < 2; ++X)
            if ((f >> X) & 1u) {
              qk(X, kt);
              if (++qkX[X] == nX[X]) commit(&q_empty[X]);
            }
          commit(&k_empty[kt % S]);
        }
        for (int i = 0; i < n && ok; ++i) {
          // Per key tile: PV_A(i), QK_A(i+1), PV_B(i), QK_B(i+1).
          const uint32_t f = sched[i];
          const uint32_t fn = i + 1 < n ? sched[i + 1] : 0u;
          const uint32_t cur = kt + static_cast<uint32_t>(i), nxt = cur + 1;
          ok = wait(&v_full[cur % S], (cur / S) & 1u);
          if (ok && last_fix && i == n - 1) {
            const uint32_t sf = cur % S;
            ok = wait(&v_fix[sf], (fix_parity >> sf) & 1u);
            fix_parity ^= 1u << sf;
          }
          if (!ok) break;
          bool k_ready = false;  // K(i+1) waited for, right before its first QK
#pragma unroll
          for (int X = 0; X < 2; ++X) {
            if (!ok) break;
            if ((f >> X) & 1u) {
              ok = wait(&p_full[X], np[X] & 1u);
              if (ok && pvX[X] == 0 && it > 0)  // O_X still holds the last item's result
                ok = wait(&o_free[X], static_cast<uint32_t>((it - 1) & 1));
              if (!ok) break;
              tc_fence_after();
              pv(X, cur, pvX[X] == 0);
              ++np[X];
              if (++pvX[X] == nX[X]) commit(&o_final[X]);
            }
            if ((fn >> X) & 1u) {
              if (!k_ready) {
                ok = wait(&k_full[nxt % S], (nxt / S) & 1u);
                if (!ok) break;
                tc_fence_after();
                k_ready = true;
              }
              qk(X, nxt);
              if (++qkX[X] == nX[X]) commit(&q_empty[X]);
            }
          }
          if (!ok) break;
          commit(&v_empty[cur % S]);          // V(i): its PVs are issued
          if (fn != 0u) commit(&k_empty[nxt % S]);  // K(i+1): its QKs are issued
        }
        if (!ok) break;
        kt += static_cast<uint32_t>(n);
        // A tile of the item that sees no key at all: release Q_X and let the
        // epilogue run (it writes NaN rows) once the last item's O_X is read.
#pragma unroll
        for (int X = 0; X < 2; ++X)
          if (ok && nX[X] == 0) {
            commit(&q_empty[X]);
            if (it > 0) ok = wait(&o_free[X], static_cast<uint32_t>((it - 1) & 1));
            commit(&o_final[X]);
          }
        __syncwarp();  // the next item's schedule overwrites sched
      }
      commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    const int X = warp >> 2;  // query tile of this warpgroup
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + L::s_col(X);
    const uint32_t o_col = tmem + lane_base + L::o_col(X);
    const int hh = row / qpt, qi = row % qpt;
    const bool mask_vec = a.has_mask && ((reinterpret_cast<uintptr_t>(a.mask) & 15u) == 0) &&
                          (a.ms[0] % 16 == 0) && (a.ms[1] % 16 == 0);
    uint32_t J = 0;  // S_X tiles over the kernel
    int64_t it = 0;
    bool ok = true;
    for (int64_t x = snake(0, blockIdx.x, gridDim.x); x < items && ok;
         ++it, x = snake(it, blockIdx.x, gridDim.x)) {
      const PPTile me = pp_tile(a.order != nullptr ? a.order[x] : x, X, a, m_tiles, qpt, n_tiles);
      const Pair& pr = me.pr;
      const int q = me.sl.q0 + qi;
      const bool row_valid = me.sl.live && row < rows && q < a.Sq;
      const uint8_t* mrow =
          (a.has_mask && row_valid) ? a.mask + pr.b * a.ms[0] + static_cast<int64_t>(q) * a.ms[1]
                                    : nullptr;
      float m_ref = -INFINITY, l = 0.f;
      int nloc = 0;
      for (int t = pr.nt_beg; t < pr.nt_end && ok; ++t) {
        const int cls = tile_class(a, pr, me.sl, t, m_tiles, n_tiles);
        if (cls == 0) continue;
        // okt: warp-uniform, so that every TMEM access it guards is made by
        // the whole warp.  The softmax warps meet no barrier of their own: each
        // signals the MMA warp per warp, and a warp that gives up leaves
        // while the others stop at their next wait, which sees the abort flag.
        const bool okt = __all_sync(0xffffffffu, mbar_wait_hot(&s_full[X], J & 1u, abort_flag,
                                                               a.err, kErrPrefillWait));
        if (okt) {
          tc_fence_after();
          uint32_t r[BN];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
            tmem_ld32(s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
          tmem_ld_wait();
          // Fully visible tiles work on raw scores and fold the scale into
          // one FMA per element below; other tiles test each key against the
          // row's visibility bits.
          const bool fast = cls == 2 && a.scale_log2 >= 0.f;
          if (!fast) {
            uint32_t vb[4];
            visible_bits<4>(vb, row_valid ? mrow : nullptr, t * BN, a, pr, q, mask_vec);
#pragma unroll
            for (int c = 0; c < BN; ++c)
              r[c] = __float_as_uint(((vb[c >> 5] >> (c & 31)) & 1u)
                                         ? __uint_as_float(r[c]) * a.scale_log2
                                         : -INFINITY);
          }
          // Eight independent running maxima, two elements per three-input max.
          float part[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) part[e] = -INFINITY;
#pragma unroll
          for (int c = 0; c < BN; c += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              part[e] = fmax3(part[e], __uint_as_float(r[c + e]), __uint_as_float(r[c + 8 + e]));
          float mx = fmax3(fmax3(part[0], part[1], part[2]), fmax3(part[3], part[4], part[5]),
                           fmaxf(part[6], part[7]));
          if (fast) mx *= a.scale_log2;
          const float m_new = fmaxf(m_ref, mx);
          const bool grow = m_new > m_ref + kRescaleLog2;  // also true for -inf -> finite
          const float alpha = grow ? fast_exp2(m_ref - m_new) : 1.f;
          const bool o_live = grow && nloc > 0 && m_ref != -INFINITY;
          if (grow) {
            l *= alpha;
            m_ref = m_new;
          }
          const float ref = exp_ref(m_ref);
          const float sc = fast ? a.scale_log2 : 1.f;
          // P = 2^(t - ref) as 16-bit pairs over the first 64 columns of S_X;
          // the scaling and the row sum take two columns per instruction.
          const uint64_t sc2 = f2_pack(sc, sc), nref2 = f2_pack(-ref, -ref);
          uint64_t lp[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) lp[e] = 0;
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c0 = c * 32 + 2 * e;
              const uint64_t x = f2_fma(f2_pack(__uint_as_float(r[c0]), __uint_as_float(r[c0 + 1])),
                                        sc2, nref2);
              float p0, p1;
              if (poly_pair<D, KVX>(e)) {
                const uint64_t pp = exp2_poly_x2(x);
                p0 = f2_lo(pp);
                p1 = f2_hi(pp);
              } else {
                p0 = fast_exp2(f2_lo(x));
                p1 = fast_exp2(f2_hi(x));
              }
              lp[e & 3] = f2_add(lp[e & 3], f2_pack(p0, p1));
              pk[e] = pack_p<F16>(p0, p1);
            }
            tmem_st16(s_col + c * 16, pk);
          }
          l += ((f2_lo(lp[0]) + f2_hi(lp[0])) + (f2_lo(lp[1]) + f2_hi(lp[1]))) +
               ((f2_lo(lp[2]) + f2_hi(lp[2])) + (f2_lo(lp[3]) + f2_hi(lp[3])));
          if (__any_sync(0xffffffffu, o_live)) {
            // O_X holds the earlier tiles' P V with the old reference; the
            // previous PV_X has completed (S_X follows it) and the next waits
            // for this tile's P: rescale it now, the S row being dead.
            const float f = o_live ? alpha : 1.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(o_col + c * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st16(o_col + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
              tmem_st16(o_col + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
            }
          }
        }
        tmem_st_wait();
        tc_fence_before();
        // Each warp reports its 32 rows of P_X on its own: a named barrier of
        // the warpgroup here would sit on every tile's critical path.  A warp
        // that gave up leaves; the others see the abort flag in their next wait.
        if (!okt) {
          ok = false;
          break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[X]);
        ++J;
        ++nloc;
      }
      if (!ok) break;
      // Epilogue: out = O / l for this row.
      const bool oke = __all_sync(
          0xffffffffu, mbar_wait_hot(&o_final[X], static_cast<uint32_t>(it & 1), abort_flag,
                                     a.err, kErrPrefillWait));
      if (oke) tc_fence_after();
      uint16_t* orow = a.out + pr.b * a.os[0] +
                       static_cast<int64_t>(pr.kv * a.g + (hh < a.g ? hh : 0)) * a.os[1] +
                       static_cast<int64_t>(q) * a.os[2];
      // No visible key (the running maximum never left -inf): NaN output.
      const float inv_l = m_ref == -INFINITY ? __int_as_float(0x7fc00000) : 1.f / l;
      if (nloc > 0) {
        // (After a failed wait the values read are discarded: the output of
        // an aborted launch is undefined.)
        uint32_t r[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          tmem_ld32(o_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        tmem_ld_wait();
        tc_fence_before();
        if (!oke) {
          ok = false;
          break;
        }
        // This warp's rows of O_X are in registers: once all four warps have
        // said so, the next item's first PV_X may overwrite O_X.
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[X]);
        if (row_valid) {
#pragma unroll
          for (int v8 = 0; v8 < D / 8; ++v8) {
            if (v8 * 8 >= a.Dv) break;
            uint4 w;
            w.x = pack2<F16>(__uint_as_float(r[v8 * 8 + 0]) * inv_l,
                             __uint_as_float(r[v8 * 8 + 1]) * inv_l);
            w.y = pack2<F16>(__uint_as_float(r[v8 * 8 + 2]) * inv_l,
                             __uint_as_float(r[v8 * 8 + 3]) * inv_l);
            w.z = pack2<F16>(__uint_as_float(r[v8 * 8 + 4]) * inv_l,
                             __uint_as_float(r[v8 * 8 + 5]) * inv_l);
            w.w = pack2<F16>(__uint_as_float(r[v8 * 8 + 6]) * inv_l,
                             __uint_as_float(r[v8 * 8 + 7]) * inv_l);
            reinterpret_cast<uint4*>(orow)[v8] = w;
          }
        }
      } else {
        if (row_valid) {
          const float nanv = __int_as_float(0x7fc00000);
          const uint32_t nn = pack2<F16>(nanv, nanv);
          for (int d = 0; d < a.Dv; d += 8)
            *reinterpret_cast<uint4*>(orow + d) = make_uint4(nn, nn, nn, nn);
        }
        tc_fence_before();
        if (!oke) {
          ok = false;
          break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[X]);
      }
    }
  }

  // Every role is done with TMEM (the MMA warp has seen its last MMA
  // complete) before it is freed.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

// The items of a launch with a mask or per-sequence lengths in decreasing
// order of cost (the key tiles that either query tile computes): a counting
// sort in one CTA, written to a.order.  Position x of the kernels' schedule then takes
// item a.order[x], so the heaviest items are spread first over the CTAs and
// the lightest fill in last.
__global__ void __launch_bounds__(1024)
    gqa_pp_order_kernel(const PrefillArgs a, const int qpt, const int m_tiles, const int n_tiles,
                        const int64_t items) {
  constexpr int kKeep = 8192;  // items whose bucket is kept in shared memory
  __shared__ int slot[1024];  // per cost bucket (bucket 0: the heaviest): count, then next position
  __shared__ int warp_base[32];
  __shared__ uint16_t kept[kKeep];
  const int tid = threadIdx.x;
  auto bucket_of = [&](int64_t x) -> int {
    const PPTile qa = pp_tile(x, 0, a, m_tiles, qpt, n_tiles);
    const PPTile qb = pp_tile(x, 1, a, m_tiles, qpt, n_tiles);
    int n = 0;
    if (!a.has_mask || a.bounds != nullptr) {
      // The union of the two query tiles' key-tile ranges (consecutive query
      // tiles: they overlap or touch).  Without a mask every tile of a range
      // is computed; with one the ranges are already trimmed to the first and
      // last tiles that are not all hidden (tiles hidden in between count too:
      // the order needs a cost, not the exact work).
      const int lo = min(qa.pr.nt_end > qa.pr.nt_beg ? qa.pr.nt_beg : 1 << 30,
                         qb.pr.nt_end > qb.pr.nt_beg ? qb.pr.nt_beg : 1 << 30);
      const int hi = max(qa.pr.nt_end, qb.pr.nt_end);
      n = hi > lo ? hi - lo : 0;
    } else if (!a.causal && a.lens == nullptr) {
      // Mask only: a key tile is computed iff its summary byte is nonzero
      // for either live query tile.
      const uint8_t* ra = a.summary + (static_cast<int64_t>(qa.pr.b) * m_tiles + qa.pr.mt0) * n_tiles;
      const uint8_t* rb = a.summary + (static_cast<int64_t>(qb.pr.b) * m_tiles + qb.pr.mt0) * n_tiles;
      const bool la = qa.pr.nt_end > qa.pr.nt_beg, lb = qb.pr.nt_end > qb.pr.nt_beg;
      for (int t = 0; t < n_tiles; ++t)
        n += ((la && ra[t] != 0) || (lb && rb[t] != 0)) ? 1 : 0;
    } else {
      const int t_lo = min(qa.pr.nt_end > qa.pr.nt_beg ? qa.pr.nt_beg : 1 << 30,
                           qb.pr.nt_end > qb.pr.nt_beg ? qb.pr.nt_beg : 1 << 30);
      const int t_hi = max(qa.pr.nt_end, qb.pr.nt_end);
      for (int t = t_lo; t < t_hi; ++t)
        n += (pp_class(qa, t, a, m_tiles, n_tiles) != 0 || pp_class(qb, t, a, m_tiles, n_tiles) != 0)
                 ? 1
                 : 0;
    }
    return 1023 - min(n, 1023);
  };
  slot[tid] = 0;
  __syncthreads();
  for (int64_t x = tid; x < items; x += blockDim.x) {
    const int k = bucket_of(x);
    if (x < kKeep) kept[x] = static_cast<uint16_t>(k);
    atomicAdd(&slot[k], 1);
  }
  __syncthreads();
  // Exclusive prefix sum of the bucket counts: the first position of each bucket.
  const int v = slot[tid];
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if ((tid & 31) >= o) incl += y;
  }
  if ((tid & 31) == 31) warp_base[tid >> 5] = incl;
  __syncthreads();
  if (tid < 32) {
    const int w = warp_base[tid];
    int wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (tid >= o) wi += y;
    }
    warp_base[tid] = wi - w;
  }
  __syncthreads();
  slot[tid] = warp_base[tid >> 5] + incl - v;
  __syncthreads();
  for (int64_t x = tid; x < items; x += blockDim.x)
    a.order[atomicAdd(&slot[x < kKeep ? kept[x] : bucket_of(x)], 1)] = static_cast<int32_t>(x);
}

template <int D, bool F16, bool KVX>
int launch_pp_t(const PrefillShape& s, const PrefillArgs& a, const PagedKV& pg,
                const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                cudaStream_t stream) {
  auto kern = gqa_prefill_pp_kernel<D, F16, KVX>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           PPLayout<D>::kBytes) != cudaSuccess)
    return GQA_ERR_CUDA;
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return GQA_ERR_CUDA;
  if (fa.numRegs != kLaunchRegs) return GQA_ERR_CUDA;  // the register split assumes it
  kern<<<s.grid, kPPThreads, PPLayout<D>::kBytes, stream>>>(tmq, tmk, tmv, a, s.qpt, s.rows,
                                                            s.m_tiles, s.n_tiles, s.work, pg);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace

int pp_smem_bytes(int D) { return D == 128 ? PPLayout<128>::kBytes : PPLayout<64>::kBytes; }

int launch_prefill_pp(const gqa_problem& p, const PrefillShape& s, const PrefillArgs& a,
                      const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                      cudaStream_t stream) {
  if (a.has_mask) {
    const int rc = launch_mask_summary(s, a, stream);
    if (rc != GQA_OK) return rc;
  }
  if (a.order != nullptr) {
    gqa_pp_order_kernel<<<1, 1024, 0, stream>>>(a, s.qpt, s.m_tiles, s.n_tiles, s.work);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  }
  const bool f16 = p.dtype == GQA_DTYPE_F16;
  PagedKV pg{};
  pg.bt = p.block_table;
  pg.bt_stride = p.block_table_stride;
  pg.page_size = static_cast<int>(p.page_size);
  pg.num_pages = static_cast<int>(p.num_pages);
  const bool kvx = a.lens != nullptr || pg.bt != nullptr;
  if (s.D == 128) {
    if (kvx)
      return f16 ? launch_pp_t<128, true, true>(s, a, pg, tmq, tmk, tmv, stream)
                 : launch_pp_t<128, false, true>(s, a, pg, tmq, tmk, tmv, stream);
    return f16 ? launch_pp_t<128, true, false>(s, a, pg, tmq, tmk, tmv, stream)
               : launch_pp_t<128, false, false>(s, a, pg, tmq, tmk, tmv, stream);
  }
  if (s.D == 64) {
    if (kvx)
      return f16 ? launch_pp_t<64, true, true>(s, a, pg, tmq, tmk, tmv, stream)
                 : launch_pp_t<64, false, true>(s, a, pg, tmq, tmk, tmv, stream);
    return f16 ? launch_pp_t<64, true, false>(s, a, pg, tmq, tmk, tmv, stream)
               : launch_pp_t<64, false, false>(s, a, pg, tmq, tmk, tmv, stream);
  }
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace gqa
