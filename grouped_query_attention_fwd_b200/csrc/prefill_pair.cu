// Prefill on pairs of SMs (clusters of two CTAs) with two query tiles in
// flight per SM.
//
// The g query heads of a kv head are packed into 128-row tiles as in the
// one-SM prefill kernel (row r: head h0 + r / qpt, query q0 + r % qpt), and
// one K / V tile serves every head of the group ("Multi-Query Attention",
// "Implementation": the shared K/V head is read once; the expanded K/V of
// "28. Grouped-Query Attention (GQA)", "Reference solution", never exists).
//
// A work item is four consecutive query tiles of one (batch, kv head): CTA
// rank r of the pair holds tiles A = 4i + r and B = 4i + 2 + r.  The pair's
// tensor cores compute each product for both CTAs at once (tcgen05.mma on a
// CTA pair, M = 256: each CTA supplies its own 128 rows of A; B is split by
// N between the two CTAs):
//
//   S_X = Q_X K^T    A = Q_X (this CTA's shared memory), B = K: CTA r holds
//                    keys [64 r, 64 r + 64) of the 128-key tile
//   O_X += P_X V     A = P_X (this CTA's tensor memory), B = V: CTA r holds
//                    head-dim columns [64 r, 64 r + 64)
//
// so every K / V byte is read once per 512 query rows of a group and each SM
// stages half of each tile.  TMEM of each CTA: S_A, S_B (128 columns each),
// O_A, O_B (D each).  One softmax warpgroup per query tile, one thread per
// row (all 128 keys of the row in registers: no exchange between threads);
// while warpgroup A turns S_A into P_A the tensor cores compute tile B's
// products, and the other way round.  The leader CTA's single MMA thread
// issues, per key tile u:  PV_A(u), QK_A(u+1), PV_B(u), QK_B(u+1).  P_X is
// written over the first half of S_X, so QK_X(u+1) follows PV_X(u) in issue
// order (tcgen05 operations of one thread execute in issue order).
//
// Barriers: the loads of both CTAs complete on the leader's full barriers,
// whose expected bytes the leader's producers set for both halves; the
// leader's MMA completions arrive on both CTAs' barriers (commit multicast);
// the peer's softmax warps arrive on the leader's P-ready and O-free barriers
// remotely.  Every wait is bounded; a CTA that gives up sets the error word
// and unwinds, and the pair meets at a cluster barrier before TMEM is freed.
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "prefill_common.cuh"
#include "ptx.cuh"

namespace gqa {
namespace {

using namespace prefill;

constexpr int kPairThreads = 12 * 32;
constexpr int kWarpQK = 8;   // TMA producer of Q tiles and K halves
constexpr int kWarpMMA = 9;  // TMEM allocation; the leader's MMA issuer
constexpr int kWarpV = 10;   // TMA producer of V halves (warp 11 idles)
constexpr int kStages = 4;  // K and V stages (a K half and a V half per key tile)
constexpr int kLaunchRegs = 168;
constexpr int kIoRegs = 120;
constexpr int kSoftmaxRegs = 192;
static_assert(128 * kIoRegs + 256 * kSoftmaxRegs <= kPairThreads * kLaunchRegs,
              "register split must fit in the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr uint16_t kBothCtas = 0x3;

template <int D>
struct PairLayout {
  static_assert(D == 128, "the pair kernel is built for head_dim 128 (padded)");
  static constexpr int CH = D / 64;                     // 64-column (128-byte) chunks
  static constexpr int kQChunk = BM * 128;              // 128 rows x 128 bytes
  static constexpr int kQTile = CH * kQChunk;
  static constexpr int kKChunk = (BN / 2) * 128;        // 64 keys x 128 bytes
  static constexpr int kKHalf = CH * kKChunk;           // this CTA's 64 keys of a K tile
  static constexpr int kVHalf = BN * 128;               // 128 keys x this CTA's 64 columns
  static constexpr int kQOff = 0;                       // Q_A, then Q_B
  static constexpr int kKOff = kQOff + 2 * kQTile;
  static constexpr int kVOff = kKOff + kStages * kKHalf;
  static constexpr int kBarOff = kVOff + kStages * kVHalf;
  // q_full[2], q_empty[2], k_full[S], v_full[S], kv_empty[S], s_full[2],
  // p_full[2], o_final[2], o_free[2], mma_done
  static constexpr int kNumBars = 4 + 3 * kStages + 8 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSchedOff = kMiscOff + 16;  // the MMA thread's key-tile list of an item
  static constexpr int kBytes = kSchedOff + kMaxPairTiles + 1024;  // + alignment slack
  // TMEM columns of S_X and O_X (X = 0: tile A, 1: tile B).
  __device__ static constexpr uint32_t s_col(int X) { return static_cast<uint32_t>(X) * 128u; }
  __device__ static constexpr uint32_t o_col(int X) { return 256u + static_cast<uint32_t>(X) * 128u; }
};

// Key tiles of one work item: the union over its four query tiles, and for
// tile X (0 = A, 1 = B) whether the pair computes it (some row of either CTA's
// query tile of X may see a key of the tile).
struct ItemGeom {
  Pair pr[2][2];   // [X][rank]: the query tile of rank r in X
  Slot sl[2][2];
  int t_lo, t_hi;  // union of the key tiles of all four query tiles
};

__device__ __forceinline__ Pair make_pair_tile(const PrefillArgs& a, int b, int kv, int mt,
                                               int qpt, int n_tiles) {
  Pair pr;
  pr.b = b;
  pr.kv = kv;
  pr.mt0 = mt;
  pr.len = a.Sk;
  const Slot s0 = slot_of(pr, a, qpt);
  if (mt * qpt >= a.Sq || s0.key_hi <= s0.key_lo) {
    pr.nt_beg = pr.nt_end = 0;
  } else {
    pr.nt_beg = static_cast<int>(s0.key_lo / BN);
    pr.nt_end = min(n_tiles, static_cast<int>((s0.key_hi + BN - 1) / BN));
  }
  return pr;
}

__device__ __forceinline__ ItemGeom item_geom(int64_t x, const PrefillArgs& a, int m_tiles, int qpt,
                                              int n_tiles) {
  ItemGeom it;
  const int64_t bh = static_cast<int64_t>(a.B) * a.Hkv;
  const int n4 = (m_tiles + 3) / 4;
  const int bk = static_cast<int>(x % bh);
  const int i4 = n4 - 1 - static_cast<int>(x / bh);  // late (long causal) items first
  const int b = bk / a.Hkv, kv = bk % a.Hkv;
  it.t_lo = 1 << 30;
  it.t_hi = 0;
  for (int X = 0; X < 2; ++X)
    for (int r = 0; r < 2; ++r) {
      it.pr[X][r] = make_pair_tile(a, b, kv, 4 * i4 + 2 * X + r, qpt, n_tiles);
      it.sl[X][r] = slot_of(it.pr[X][r], a, qpt);
      it.sl[X][r].live = 4 * i4 + 2 * X + r < m_tiles;
      if (it.pr[X][r].nt_end > it.pr[X][r].nt_beg) {
        it.t_lo = min(it.t_lo, it.pr[X][r].nt_beg);
        it.t_hi = max(it.t_hi, it.pr[X][r].nt_end);
      }
    }
  if (it.t_hi <= it.t_lo) it.t_lo = it.t_hi = 0;
  return it;
}

// Class of key tile t for rank r's query tile of X (0 hidden, 1 mixed, 2 visible).
__device__ __forceinline__ int cls_of(const ItemGeom& it, int X, int r, int t, const PrefillArgs& a,
                                      int m_tiles, int n_tiles) {
  const Pair& pr = it.pr[X][r];
  if (t < pr.nt_beg || t >= pr.nt_end) return 0;
  return tile_class(a, pr, it.sl[X][r], t, m_tiles, n_tiles);
}

// The pair computes QK_X / PV_X at key tile t.
__device__ __forceinline__ bool pair_does(const ItemGeom& it, int X, int t, const PrefillArgs& a,
                                          int m_tiles, int n_tiles) {
  return cls_of(it, X, 0, t, a, m_tiles, n_tiles) != 0 || cls_of(it, X, 1, t, a, m_tiles, n_tiles) != 0;
}

template <int D, bool F16>
__global__ void __launch_bounds__(kPairThreads, 1)
    gqa_prefill_pair_kernel(const __grid_constant__ CUtensorMap tmq,
                            const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, const PrefillArgs a,
                            const int qpt, const int rows, const int m_tiles, const int n_tiles,
                            const int64_t items) {
  using L = PairLayout<D>;
  constexpr int CH = L::CH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;                  // [X] leader: both CTAs' Q_X landed
  uint64_t* q_empty = q_full + 2;           // [X] every CTA: the item's QK_X done
  uint64_t* k_full = q_empty + 2;           // [stage] leader: both K halves landed
  uint64_t* v_full = k_full + kStages;      // [stage] leader: both V halves landed
  uint64_t* kv_empty = v_full + kStages;    // [stage] every CTA: the products reading it done
  // S_X done.  The commit follows QK_X, which follows the previous PV_X from
  // the same thread, so it also means that PV_X has completed: the softmax
  // may rescale O_X once it has seen S_X.
  uint64_t* s_full = kv_empty + kStages;    // [X] every CTA
  uint64_t* p_full = s_full + 2;            // [X] leader: P_X written (one arrival per CTA)
  uint64_t* o_final = p_full + 2;           // [X] every CTA: the item's last PV_X done
  uint64_t* o_free = o_final + 2;           // [X] leader: O_X read by both epilogues
  uint64_t* mma_done = o_free + 2;          // leader: every MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  uint8_t* sched = smem + L::kSchedOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int64_t pair = blockIdx.x >> 1;
  const int64_t npairs = gridDim.x >> 1;
  // Shared::cluster address of the leader's copy of a barrier.
  auto at_leader = [&](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 2);   // one arrival per CTA
      mbar_init(&o_final[i], 1);
      mbar_init(&o_free[i], 2);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Q rows past qpt * g of a tile are never written by TMA: zero them once.
  if (rows < BM && threadIdx.x < 8) {
    for (int X = 0; X < 2; ++X)
      for (int c = 0; c < CH; ++c) {
        uint8_t* base = smem + L::kQOff + X * L::kQTile + c * L::kQChunk;
        for (int r = rows; r < BM; ++r)
          reinterpret_cast<uint4*>(base + r * 128)[threadIdx.x] = make_uint4(0, 0, 0, 0);
      }
    fence_proxy_async_smem();
  }
  if (warp == kWarpMMA) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // Both CTAs' barriers are initialised and their TMEM allocated before any
  // remote arrival, load or MMA.
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIoRegs));
    if ((warp == kWarpQK || warp == kWarpV) && lane == 0) {
      // ------------------------------------------------------------ producers
      const bool is_qk = warp == kWarpQK;
      const CUtensorMap* map = is_qk ? &tmk : &tmv;
      uint64_t* full = is_qk ? k_full : v_full;
      uint64_t* empty = kv_empty;
      const int stages = kStages;
      const uint32_t bytes = is_qk ? L::kKHalf : L::kVHalf;
      uint8_t* ring = smem + (is_qk ? L::kKOff : L::kVOff);
      prefetch_tmap(map);
      if (is_qk) prefetch_tmap(&tmq);
      uint32_t kt = 0;
      int64_t it = 0;
      bool ok = true;
      for (int64_t x = snake(0, pair, npairs); x < items && ok; ++it, x = snake(it, pair, npairs)) {
        const ItemGeom g = item_geom(x, a, m_tiles, qpt, n_tiles);
        if (is_qk) {
          for (int X = 0; X < 2 && ok; ++X) {
            if (it > 0 && !mbar_wait(&q_empty[X], static_cast<uint32_t>((it - 1) & 1), abort_flag,
                                     a.err, kErrPrefillWait)) {
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(&q_full[X], static_cast<uint32_t>(2 * rows * 128 * CH));
            const Pair& pr = g.pr[X][rank];
            for (int c = 0; c < CH; ++c)
              tma_load_4d_pair(smem + L::kQOff + X * L::kQTile + c * L::kQChunk, &tmq,
                               at_leader(&q_full[X]), c * 64, pr.mt0 * qpt, pr.kv * a.g, pr.b);
          }
        }
        for (int t = g.t_lo; t < g.t_hi && ok; ++t) {
          if (!pair_does(g, 0, t, a, m_tiles, n_tiles) && !pair_does(g, 1, t, a, m_tiles, n_tiles))
            continue;
          const int s = static_cast<int>(kt % stages);
          const uint32_t round = kt / stages;
          if (round > 0 &&
              !mbar_wait(&empty[s], (round - 1) & 1u, abort_flag, a.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * bytes);
          uint8_t* dst = ring + s * bytes;
          const Pair& pr = g.pr[0][0];
          if (is_qk) {
            for (int c = 0; c < CH; ++c)
              tma_load_4d_pair(dst + c * L::kKChunk, map, at_leader(&full[s]), c * 64,
                               t * BN + static_cast<int>(rank) * (BN / 2), pr.kv, pr.b);
          } else {
            tma_load_4d_pair(dst, map, at_leader(&full[s]), static_cast<int>(rank) * 64, t * BN,
                             pr.kv, pr.b);
          }
          ++kt;
        }
      }
      // The leader's full barriers count both CTAs' bytes: on an abort the
      // leader waits for the copies in flight of both before the pair meets
      // at the closing cluster barrier.
      if (*abort_flag && leader)
        for (uint32_t j = kt > static_cast<uint32_t>(stages) ? kt - stages : 0; j < kt; ++j)
          mbar_wait_drain(&full[j % stages], (j / stages) & 1u);
    } else if (warp == kWarpMMA && lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_qk =
          F16 ? idesc_f16_f32(2 * BM, BN, 0, 0) : idesc_bf16_f32(2 * BM, BN, 0, 0);
      constexpr uint32_t idesc_pv =
          F16 ? idesc_f16_f32(2 * BM, D, 0, 1) : idesc_bf16_f32(2 * BM, D, 0, 1);
      const uint64_t dq0 = kmajor_desc(smem_u32(smem + L::kQOff));
      const uint64_t dk0 = kmajor_desc(smem_u32(smem + L::kKOff));
      const uint64_t dv0 = mnmajor_desc(smem_u32(smem + L::kVOff), L::kVHalf);
      uint32_t kt = 0;               // key tiles (K / V stages) consumed over the kernel
      uint32_t np[2] = {0, 0};       // P_X tiles consumed over the kernel
      int64_t it = 0;
      bool ok = true;
      auto qk = [&](int X, uint32_t idx) {
        const uint64_t dq = dq0 + ((X * L::kQTile) >> 4);
        const uint64_t dk = dk0 + (((idx % kStages) * L::kKHalf) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc_mma_ss_pair(tmem + L::s_col(X), dq + (((k >> 2) * L::kQChunk + (k & 3) * 32) >> 4),
                         dk + (((k >> 2) * L::kKChunk + (k & 3) * 32) >> 4), idesc_qk,
                         k > 0 ? 1u : 0u);
        tc_commit_pair_mc(&s_full[X], kBothCtas);
      };
      auto pv = [&](int X, uint32_t idx, bool first) {
        const uint64_t dv = dv0 + (((idx % kStages) * L::kVHalf) >> 4);
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          tc_mma_ts_pair(tmem + L::o_col(X), tmem + L::s_col(X) + k * 8,
                         dv + ((k * 16 * 128) >> 4), idesc_pv, (!first || k > 0) ? 1u : 0u);
      };
      for (int64_t x = snake(0, pair, npairs); x < items && ok; ++it, x = snake(it, pair, npairs)) {
        const ItemGeom g = item_geom(x, a, m_tiles, qpt, n_tiles);
        // The item's key tiles that some tile works on, in order, as one byte
        // each in shared memory (bit X: tile X computes it); tile classes read
        // mask summaries from global memory, so they are taken here once per
        // item, off the per-tile path.
        int n = 0, nX[2] = {0, 0};
        for (int t = g.t_lo; t < g.t_hi; ++t) {
          const uint32_t f = (pair_does(g, 0, t, a, m_tiles, n_tiles) ? 1u : 0u) |
                             (pair_does(g, 1, t, a, m_tiles, n_tiles) ? 2u : 0u);
          if (f != 0u) {
            sched[n++] = static_cast<uint8_t>(f);
            nX[0] += f & 1u;
            nX[1] += f >> 1;
          }
        }
        for (int X = 0; X < 2 && ok; ++X)
          ok = mbar_wait_hot(&q_full[X], static_cast<uint32_t>(it & 1), abort_flag, a.err,
                             kErrPrefillWait);
        if (!ok) break;
        tc_fence_after();
        int qkX[2] = {0, 0};  // QK_X / PV_X issued for this item
        int pvX[2] = {0, 0};
        if (n > 0) {  // the first key tile: its QKs
          ok = mbar_wait_hot(&k_full[kt % kStages], (kt / kStages) & 1u, abort_flag, a.err,
                             kErrPrefillWait);
          if (!ok) break;
          tc_fence_after();
          const uint32_t f = sched[0];
          for (int X = 0; X < 2; ++X)
            if ((f >> X) & 1u) {
              qk(X, kt);
              if (++qkX[X] == nX[X]) tc_commit_pair_mc(&q_empty[X], kBothCtas);
            }
        }
        for (int i = 0; i < n && ok; ++i) {
          // Per key tile: PV_A(i), QK_A(i+1), PV_B(i), QK_B(i+1).
          const uint32_t f = sched[i];
          const uint32_t fn = i + 1 < n ? sched[i + 1] : 0u;
          const uint32_t cur = kt + static_cast<uint32_t>(i), nxt = cur + 1;
          ok = mbar_wait_hot(&v_full[cur % kStages], (cur / kStages) & 1u, abort_flag, a.err,
                             kErrPrefillWait);
          if (!ok) break;
          bool k_ready = false;  // K(i+1) waited for, right before its first QK
          for (int X = 0; X < 2 && ok; ++X) {
            if ((f >> X) & 1u) {
              ok = mbar_wait_cluster(&p_full[X], np[X] & 1u, abort_flag, a.err, kErrPrefillWait);
              if (ok && pvX[X] == 0 && it > 0)  // O_X still holds the last item's result
                ok = mbar_wait_cluster(&o_free[X], static_cast<uint32_t>((it - 1) & 1), abort_flag,
                                       a.err, kErrPrefillWait);
              if (!ok) break;
              tc_fence_after();
              pv(X, cur, pvX[X] == 0);
              ++np[X];
              if (++pvX[X] == nX[X]) tc_commit_pair_mc(&o_final[X], kBothCtas);
            }
            if ((fn >> X) & 1u) {
              if (!k_ready) {
                ok = mbar_wait_hot(&k_full[nxt % kStages], (nxt / kStages) & 1u, abort_flag,
                                   a.err, kErrPrefillWait);
                if (!ok) break;
                tc_fence_after();
                k_ready = true;
              }
              qk(X, nxt);
              if (++qkX[X] == nX[X]) tc_commit_pair_mc(&q_empty[X], kBothCtas);
            }
          }
          if (!ok) break;
          // Stage i is free once its PVs (and the QKs issued before them) are done.
          tc_commit_pair_mc(&kv_empty[cur % kStages], kBothCtas);
        }
        if (!ok) break;
        kt += static_cast<uint32_t>(n);
        // A tile of the item that sees no key at all: release Q_X and let the
        // epilogue run (it writes NaN rows) once the last item's O_X is read.
        for (int X = 0; X < 2 && ok; ++X)
          if (nX[X] == 0) {
            tc_commit_pair_mc(&q_empty[X], kBothCtas);
            if (it > 0)
              ok = mbar_wait_cluster(&o_free[X], static_cast<uint32_t>((it - 1) & 1), abort_flag,
                                     a.err, kErrPrefillWait);
            tc_commit_pair_mc(&o_final[X], kBothCtas);
          }
      }
      tc_commit_pair_mc(mma_done, 1);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    const int X = warp >> 2;   // query tile of this warpgroup
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + L::s_col(X);
    const uint32_t o_col = tmem + lane_base + L::o_col(X);
    const uint32_t p_full_at = at_leader(&p_full[X]);
    const uint32_t o_free_at = at_leader(&o_free[X]);
    const int hh = row / qpt, qi = row % qpt;
    const bool mask_vec = a.has_mask && ((reinterpret_cast<uintptr_t>(a.mask) & 15u) == 0) &&
                          (a.ms[0] % 16 == 0) && (a.ms[1] % 16 == 0);
    uint32_t J = 0;  // S_X tiles over the kernel
    int64_t it = 0;
    bool ok = true;
    for (int64_t x = snake(0, pair, npairs); x < items && ok; ++it, x = snake(it, pair, npairs)) {
      const ItemGeom g = item_geom(x, a, m_tiles, qpt, n_tiles);
      const Pair& pr = g.pr[X][rank];
      const Slot& me = g.sl[X][rank];
      const int q = me.q0 + qi;
      const bool row_valid = me.live && row < rows && q < a.Sq;
      const uint8_t* mrow =
          (a.has_mask && row_valid) ? a.mask + pr.b * a.ms[0] + static_cast<int64_t>(q) * a.ms[1]
                                    : nullptr;
      float m_ref = -INFINITY, l = 0.f;
      int nloc = 0;
      for (int t = g.t_lo; t < g.t_hi && ok; ++t) {
        if (!pair_does(g, X, t, a, m_tiles, n_tiles)) continue;
        const int cls = cls_of(g, X, static_cast<int>(rank), t, a, m_tiles, n_tiles);
        // okt: warp-uniform, so that every TMEM access it guards is made by
        // the whole warp; the warpgroup meets once per tile below and leaves
        // the loop together.
        bool okt = __all_sync(0xffffffffu, mbar_wait_hot(&s_full[X], J & 1u, abort_flag, a.err,
                                                         kErrPrefillWait));
        if (!okt) {
        } else if (cls == 0) {
          tc_fence_after();
          // No row of this CTA's tile sees the tile: P = 0 for the pair's PV.
          uint32_t z[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) z[e] = 0u;
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_st16(s_col + c * 16, z);
        } else {
          tc_fence_after();
          uint32_t r[BN];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
          tmem_ld_wait();
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
          if (__any_sync(0xffffffffu, o_live)) {
            // O_X holds the earlier tiles' P V with the old reference; the
            // previous PV_X has completed (S_X follows it): rescale it.
            {
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
          if (grow) {
            l *= alpha;
            m_ref = m_new;
          }
          const float ref = exp_ref(m_ref);
          const float sc = fast ? a.scale_log2 : 1.f;
          float lp[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) lp[e] = 0.f;
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c0 = c * 32 + 2 * e, c1 = c0 + 1;
              const float p0 = fast_exp2(fmaf(__uint_as_float(r[c0]), sc, -ref));
              const float p1 = fast_exp2(fmaf(__uint_as_float(r[c1]), sc, -ref));
              lp[c0 & 7] += p0;
              lp[c1 & 7] += p1;
              pk[e] = pack_p<F16>(p0, p1);
            }
            tmem_st16(s_col + c * 16, pk);
          }
          l += ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
        }
        tmem_st_wait();
        tc_fence_before();
        // The four warps of the warpgroup have written P_X (or given up):
        // one arrival per CTA on the leader's barrier.
        if (!bar_and(1 + X, 128, okt)) {
          ok = false;
          break;
        }
        if ((threadIdx.x & 127) == 0) mbar_arrive_cluster(p_full_at);
        ++J;
        ++nloc;
      }
      if (!ok) break;
      // Epilogue: out = O / l for this row.
      bool oke = __all_sync(0xffffffffu, mbar_wait_hot(&o_final[X], static_cast<uint32_t>(it & 1),
                                                       abort_flag, a.err, kErrPrefillWait));
      if (oke) tc_fence_after();
      uint16_t* orow = a.out + pr.b * a.os[0] +
                       static_cast<int64_t>(pr.kv * a.g + (hh < a.g ? hh : 0)) * a.os[1] +
                       static_cast<int64_t>(q) * a.os[2];
      const float inv_l = 1.f / l;  // l == 0: no visible key, NaN output
      if (nloc > 0) {
        // (After a failed wait the values read are discarded: the output of
        // an aborted launch is undefined.)
        uint32_t r[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          tmem_ld32(o_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        tmem_ld_wait();
        tc_fence_before();
        if (!bar_and(1 + X, 128, oke)) {
          ok = false;
          break;
        }
        // O_X is in registers: the next item's first PV_X may overwrite it.
        if ((threadIdx.x & 127) == 0) mbar_arrive_cluster(o_free_at);
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
        if (!bar_and(1 + X, 128, oke)) {
          ok = false;
          break;
        }
        if ((threadIdx.x & 127) == 0) mbar_arrive_cluster(o_free_at);
      }
    }
  }

  // Both CTAs are done with their tensor memory and with every remote barrier
  // before TMEM is freed and either CTA exits.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == kWarpMMA) tmem_dealloc_pair(tmem, kTmemCols);
  cluster_sync();
}

template <bool F16>
int launch_pair_t(const PrefillShape& s, const PrefillArgs& a, const CUtensorMap& tmq,
                  const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = gqa_prefill_pair_kernel<128, F16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           PairLayout<128>::kBytes) != cudaSuccess)
    return GQA_ERR_CUDA;
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return GQA_ERR_CUDA;
  if (fa.numRegs != kLaunchRegs) return GQA_ERR_CUDA;  // the register split assumes it
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(s.grid));
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = PairLayout<128>::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tmq, tmk, tmv, a, s.qpt, s.rows, s.m_tiles, s.n_tiles,
                         s.work) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return GQA_OK;
}

}  // namespace

int pair_smem_bytes() { return PairLayout<128>::kBytes; }

int launch_prefill_pair(const gqa_problem& p, const PrefillShape& s, const PrefillArgs& a,
                        const CUtensorMap& tmq, const CUtensorMap& tmk_half,
                        const CUtensorMap& tmv, cudaStream_t stream) {
  if (a.has_mask) {
    const int rc = launch_mask_summary(s, a, stream);
    if (rc != GQA_OK) return rc;
  }
  return p.dtype == GQA_DTYPE_F16 ? launch_pair_t<true>(s, a, tmq, tmk_half, tmv, stream)
                                  : launch_pair_t<false>(s, a, tmq, tmk_half, tmv, stream);
}

}  // namespace gqa
