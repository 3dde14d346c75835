// Prefill kernel (longer query blocks) on the 5th-generation tensor cores,
// one query tile per SM.  Plans use it for key lengths beyond the two-tile
// kernel's per-item step list (more than 1024 key tiles); the two-tile
// kernel (prefill_pp.cu) takes every other prefill.
//
// The g query heads that share a kv head are packed into the 128 rows (M) of
// one tcgen05 tile: row r holds head h0 + r / qpt at query position
// q0 + r % qpt, with qpt = floor(128 / g) query positions per tile.  One K/V
// tile of 128 keys, staged once in shared memory, therefore serves every head
// of the group ("Multi-Query Attention", "Implementation": the shared K/V head
// is read once and broadcast); the expanded K/V of the reference solution's
// repeat_interleave never exists.
//
// Per 128x128 tile:   S = Q K^T       tcgen05.mma, A = Q from TMEM (copied
//                                     in once per query tile), B = K from
//                                     shared memory, fp32 accumulator in TMEM
//                     P = softmax(S)  256 softmax threads, two per TMEM lane
//                                     (row), 64 keys each: scale, mask, online
//                                     max / sum; P (bf16) overwrites the first
//                                     half of S
//                     O += P V        tcgen05.mma, A = P from TMEM, B = V from
//                                     shared memory, O in TMEM
// Both products read one operand from shared memory: with Q and K both there
// the QK product ran at about half the rate of the PV product, the shared
// memory operand bytes per FLOP being the limit.
//
// S is double-buffered in TMEM, so the tensor core computes the next tile's
// S (and the previous tile's PV) while the softmax threads work on this one:
// the order on the tensor core is QK(0), QK(1), PV(0), QK(2), PV(1), QK(3),
// ...; tcgen05 MMAs and copies from one thread execute in issue order, so
// QK(j + 2) may follow the PV(j) that reads the P stored in the same columns,
// and the next query tile's Q may be copied in after the last QK of this one.
// TMEM (512 columns): S0, S1 (128 each), Q (D / 2: bf16 pairs), O (D).
//
// Warp roles (384 threads, one CTA per SM, persistent over query tiles):
//   warps 0-3  softmax, O rescale and epilogue for keys 0-63 of each S tile
//              and the first half of the O columns (thread t: row t)
//   warps 4-7  the same for keys 64-127 and the second half of O
//   warp 8     TMA producer of Q tiles and K tiles
//   warp 9     TMEM allocator and single-thread MMA issuer
//   warp 10    TMA producer of V tiles (warp 11 idles)
// One warpgroup alone spent about 1 us of every 1.3 us tile on the softmax
// while the two products need about 0.75 us at the tensor cores' measured
// rate; two halves bring the softmax under the tensor-core time.  The two
// threads of a row trade their partial maxima every tile, so both pick the
// same reference, and their row sums once per query tile.
// The running maximum is rescaled lazily: exponentials use a reference that
// may trail the true maximum by up to 2^8, and O and l are rescaled (O in
// TMEM) only when the maximum grows past that.
//
// Causal tiles above the diagonal are never visited; with a bool mask a
// pre-pass classifies every (query tile, key tile) pair as hidden / mixed /
// visible, hidden tiles are skipped and only mixed tiles read mask bytes.
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "prefill_common.cuh"
#include "ptx.cuh"

namespace gqa {
namespace {

using namespace prefill;
constexpr int kSoftmaxWarps = 8;  // two warpgroups, one half of the key columns each
constexpr int kWarpQK = 8;
constexpr int kWarpMMA = 9;
constexpr int kWarpV = 10;  // warp 11 idles (it completes the third warpgroup)
constexpr int kKStages = 3;  // depth of the K ring
constexpr int kVStages = 2;  // depth of the V ring
// One Q landing buffer: it is free again as soon as Q has been copied into
// TMEM at the start of a query tile, long before the next tile's Q is due.
constexpr int kQBufs = 1;
constexpr int HK = BN / 2;  // keys of an S tile per softmax warpgroup
// Register split across the three warpgroups (setmaxnreg): the launch gives
// every thread kLaunchRegs; the producer / MMA warpgroup drops to kIoRegs and
// the two softmax warpgroups rise to kSoftmaxRegs, which must add up to the
// launch's total (setmaxnreg.inc waits for registers that a larger split
// would never free).
constexpr int kLaunchRegs = 168;
constexpr int kIoRegs = 152;
constexpr int kSoftmaxRegs = 176;
static_assert(128 * kIoRegs + 256 * kSoftmaxRegs <= kPrefillThreads * kLaunchRegs,
              "register split must fit in the launch allocation");
static_assert(kPrefillThreads == 12 * 32, "two softmax warpgroups and one producer / MMA warpgroup");
constexpr uint32_t kTmemCols = 512;

// KVX: the launch has per-sequence lengths or a paged cache (two more
// barriers, for the V rows past a length; without either the kernel is built
// without them).
template <int D, bool KVX>
struct Layout {
  static constexpr int CH = D / 64;                  // 64-column (128-byte) chunks
  static constexpr int kChunkBytes = 128 * 128;      // 128 rows x 128 bytes
  static constexpr int kTileBytes = CH * kChunkBytes;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBufs * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kNumBars =
      2 * kQBufs + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 3 + (KVX ? kVStages : 0);
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kXOff = kMiscOff + 16;  // float [2][2][128]: per-row values the halves trade
  static constexpr int kBytes = kXOff + 2 * 2 * 128 * 4 + 1024;  // + alignment slack
  static constexpr uint32_t kSCol = 0;     // S buffer s at 128 s (P in its first 64 columns)
  static constexpr uint32_t kQCol = 256;   // D / 2 columns
  static constexpr uint32_t kOCol = 384;   // D columns
};

// Item x: late (long causal) query tiles first.
__device__ __forceinline__ Pair pair_of(int64_t x, const PrefillArgs& a, int m_tiles, int qpt,
                                        int n_tiles) {
  Pair pr;
  const int64_t bh = static_cast<int64_t>(a.B) * a.Hkv;
  const int bk = static_cast<int>(x % bh);
  pr.b = bk / a.Hkv;
  pr.kv = bk % a.Hkv;
  pr.mt0 = m_tiles - 1 - static_cast<int>(x / bh);
  pr.len = a.Sk;
  if (a.lens != nullptr) {  // out-of-range lengths are clamped (and reported at kernel start)
    const int len = a.lens[pr.b];
    pr.len = len < 0 ? 0 : (len > a.Sk ? a.Sk : len);
  }
  const Slot s0 = slot_of(pr, a, qpt);
  if (s0.key_hi <= s0.key_lo) {
    pr.nt_beg = pr.nt_end = 0;
  } else {
    pr.nt_beg = static_cast<int>(s0.key_lo / BN);
    pr.nt_end = min(n_tiles, static_cast<int>((s0.key_hi + BN - 1) / BN));
  }
  return pr;
}

template <int D, bool F16, bool KVX>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    gqa_prefill_kernel(const __grid_constant__ CUtensorMap tmq,
                       const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const PrefillArgs a,
                       const int qpt, const int rows, const int m_tiles, const int n_tiles,
                       const int64_t work, const PagedKV pg) {
  using L = Layout<D, KVX>;
  constexpr int CH = L::CH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;                   // [Q buffer]
  uint64_t* q_empty = q_full + kQBufs;       // [Q buffer]: copied into TMEM
  uint64_t* k_full = q_empty + kQBufs;       // [stage]
  uint64_t* k_empty = k_full + kKStages;
  uint64_t* v_full = k_empty + kKStages;
  uint64_t* v_empty = v_full + kVStages;
  // Per-tile barriers come in pairs indexed by the tile's parity: QK runs two
  // tiles ahead of PV, so the softmax may finish P(J + 1) before the MMA
  // thread has looked at P(J), and one barrier would then have moved two
  // phases past it.
  uint64_t* s_full = v_empty + kVStages;     // [J & 1]: QK(J) done
  uint64_t* p_full = s_full + 2;             // [J & 1]: P(J) written (8 warps)
  uint64_t* o_ready = p_full + 2;            // [J & 1]: PV(J) into O has completed
  uint64_t* o_final = o_ready + 2;           // the item's last PV has completed
  uint64_t* o_free = o_final + 1;            // the epilogue has read O (8 warps)
  uint64_t* mma_done = o_free + 1;
  uint64_t* v_fix = mma_done + 1;            // [stage] (KVX): rows past the length zeroed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQBufs; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSoftmaxWarps);
      mbar_init(&o_ready[i], 1);
    }
    mbar_init(o_final, 1);
    mbar_init(o_free, kSoftmaxWarps);
    mbar_init(mma_done, 1);
    if (KVX)
      for (int i = 0; i < kVStages; ++i) mbar_init(&v_fix[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (a.lens != nullptr && blockIdx.x == 0) {
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
      const int len = a.lens[b];
      if (len < 0 || len > a.Sk) atomicOr(a.err, kErrKvLength);
    }
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

  if (warp >= kSoftmaxWarps) {
  // Producer / MMA warpgroup (warps 8-11): every warp drops its registers.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIoRegs));
  if (warp == kWarpQK || warp == kWarpV) {
    // ------------------------------------------------------------- producers
    if (lane == 0) {
      const bool is_qk = warp == kWarpQK;
      const CUtensorMap* map = is_qk ? &tmk : &tmv;
      uint64_t* full = is_qk ? k_full : v_full;
      uint64_t* empty = is_qk ? k_empty : v_empty;
      uint8_t* ring = smem + (is_qk ? L::kKOff : L::kVOff);
      const int stages = is_qk ? kKStages : kVStages;
      prefetch_tmap(map);
      if (is_qk) prefetch_tmap(&tmq);
      uint32_t kt = 0;
      int64_t it = 0, q_issued = 0;
      bool ok = true;
      for (int64_t x = snake(0, blockIdx.x, gridDim.x); x < work && ok;
           ++it, x = snake(it, blockIdx.x, gridDim.x)) {
        const Pair pr = pair_of(x, a, m_tiles, qpt, n_tiles);
        const Slot me = slot_of(pr, a, qpt);
        if (is_qk) {
          const int qb = static_cast<int>(it % kQBufs);
          if (it >= kQBufs &&
              !mbar_wait(&q_empty[qb], static_cast<uint32_t>((it / kQBufs - 1) & 1), abort_flag,
                         a.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          uint8_t* qdst = smem + L::kQOff + qb * L::kTileBytes;
          mbar_arrive_expect_tx(&q_full[qb], static_cast<uint32_t>(rows * 128 * CH));
          for (int c = 0; c < CH; ++c)
            tma_load_4d(qdst + c * L::kChunkBytes, &tmq, &q_full[qb], c * 64, me.q0,
                        pr.kv * a.g, pr.b);
          ++q_issued;
        }
        for (int nt = pr.nt_beg; nt < pr.nt_end; ++nt) {
          if (tile_class(a, pr, me, nt, m_tiles, n_tiles) == 0) continue;
          const int s = static_cast<int>(kt % stages);
          const uint32_t round = kt / stages;
          if (round > 0 &&
              !mbar_wait(&empty[s], (round - 1) & 1u, abort_flag, a.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          uint8_t* dst = ring + s * L::kTileBytes;
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(L::kTileBytes));
          if (KVX && pg.bt != nullptr) {
            // Two 64-key boxes, each inside one page (page_size is a multiple
            // of 64).  A box that starts at or past the entry's length reads an
            // out-of-range page, which the copy fills with zeros; a page index
            // outside the pool for keys in use is reported and read the same way.
            for (int hb = 0; hb < 2; ++hb) {
              const int key = nt * BN + hb * 64;
              int page = pg.num_pages;
              if (key < pr.len) {
                page = __ldg(pg.bt + pr.b * pg.bt_stride + key / pg.page_size);
                if (page < 0 || page >= pg.num_pages) {
                  atomicOr(a.err, kErrPage);
                  page = pg.num_pages;
                }
              }
              for (int c = 0; c < CH; ++c)
                tma_load_4d(dst + c * L::kChunkBytes + hb * 64 * 128, map, &full[s], c * 64,
                            key % pg.page_size, pr.kv, page);
            }
          } else {
            for (int c = 0; c < CH; ++c)
              tma_load_4d(dst + c * L::kChunkBytes, map, &full[s], c * 64, nt * BN, pr.kv, pr.b);
          }
          ++kt;
          // The V rows of the entry's last tile past its length hold whatever
          // the cache holds there (NaN included), and P = 0 does not hide a
          // NaN in P V: once the tile has landed they are zeroed, and the MMA
          // waits for that too.  Only the last tile a query tile visits can
          // reach past the length.
          if (KVX && !is_qk && (static_cast<int64_t>(nt) + 1) * BN > pr.len) {
            if (!mbar_wait(&full[s], round & 1u, abort_flag, a.err, kErrPrefillWait)) {
              ok = false;
              break;
            }
            const int valid = pr.len - nt * BN;  // 1 .. BN - 1: the tile holds a key below len
            for (int c = 0; c < CH; ++c) {
              uint4* row0 = reinterpret_cast<uint4*>(dst + c * L::kChunkBytes + valid * 128);
              for (int i = 0; i < (BN - valid) * 8; ++i) row0[i] = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            mbar_arrive(&v_fix[s]);
          }
        }
      }
      if (*abort_flag) {  // let every copy in flight land before the CTA exits
        for (uint32_t j = kt > static_cast<uint32_t>(stages) ? kt - stages : 0; j < kt; ++j)
          mbar_wait_drain(&full[j % stages], (j / stages) & 1u);
        if (is_qk)
          for (int64_t j = q_issued > kQBufs ? q_issued - kQBufs : 0; j < q_issued; ++j)
            mbar_wait_drain(&q_full[j % kQBufs], static_cast<uint32_t>((j / kQBufs) & 1));
      }
    }
  } else if (warp == kWarpMMA) {
    // ------------------------------------------------------------- MMA warp
    // The whole warp walks the work and takes every wait (made warp-uniform
    // by a vote); one elect.sync lane -- lane 0 of the full warp, so always
    // the same thread -- issues the copies, MMAs and commits.  A lone issuing
    // lane in a diverged warp leaves the tensor core idle for a while at each
    // wait or data-dependent branch between MMA groups; a converged warp does
    // not.
    {
      constexpr uint32_t idesc_qk = F16 ? idesc_f16_f32(BM, BN, 0, 0) : idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = F16 ? idesc_f16_f32(BM, D, 0, 1) : idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t q_base = smem_u32(smem + L::kQOff);
      const uint32_t t_q = tmem + L::kQCol, t_o = tmem + L::kOCol;
      // Descriptors of stage 0, k-step 0; every other (stage, k-step) adds a
      // constant to the 16-byte address field (shared memory stays below
      // 256 KB, so the 14-bit field never carries).
      const uint64_t dk0 = kmajor_desc(smem_u32(smem + L::kKOff));
      const uint64_t dv0 = mnmajor_desc(smem_u32(smem + L::kVOff), L::kChunkBytes);
      constexpr uint32_t kStageStep = L::kTileBytes >> 4;
      uint32_t Jq = 0, Jp = 0;  // tiles whose QK / PV have been issued, over the whole kernel
      uint32_t fix_parity = 0;  // bit s: parity of the next v_fix[s] phase
      int64_t it = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_hot(bar, parity, abort_flag, a.err, kErrPrefillWait));
      };

      // S(J & 1) = Q K(J)^T; the K stage is released when the MMA completes.
      auto issue_qk = [&](uint32_t J) -> bool {
        const uint32_t s = J % kKStages;
        if (!wait(&k_full[s], (J / kKStages) & 1u)) return false;
        tc_fence_after();
        const uint64_t dk = dk0 + s * kStageStep;
        const uint32_t d_s = tmem + L::kSCol + (J & 1u) * BN;
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            tc_mma_ts(d_s, t_q + ks * 8, dk + (((ks >> 2) * L::kChunkBytes + (ks & 3) * 32) >> 4),
                      idesc_qk, ks > 0 ? 1u : 0u);
          tc_commit(&s_full[J & 1u]);
          tc_commit(&k_empty[s]);
        }
        __syncwarp();
        return true;
      };
      // O (+)= P(J) V(J); `first`: the item's first PV overwrites O.
      auto issue_pv = [&](uint32_t J, bool first) -> bool {
        const uint32_t s = J % kVStages;
        if (!wait(&p_full[J & 1u], (J >> 1) & 1u) || !wait(&v_full[s], (J / kVStages) & 1u))
          return false;
        if (first && it > 0 && !wait(o_free, static_cast<uint32_t>((it - 1) & 1))) return false;
        tc_fence_after();
        const uint64_t dv = dv0 + s * kStageStep;
        const uint32_t p_t = tmem + L::kSCol + (J & 1u) * BN;
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            tc_mma_ts(t_o, p_t + ks * 8, dv + ((ks * 16 * 128) >> 4), idesc_pv,
                      (!first || ks > 0) ? 1u : 0u);
          tc_commit(&o_ready[J & 1u]);
          tc_commit(&v_empty[s]);
        }
        __syncwarp();
        return true;
      };

      for (int64_t x = snake(0, blockIdx.x, gridDim.x); x < work && ok;
           ++it, x = snake(it, blockIdx.x, gridDim.x)) {
        const Pair pr = pair_of(x, a, m_tiles, qpt, n_tiles);
        // Key tiles the query tile visits: without a mask every tile of
        // [nt_beg, nt_end) holds a key some row may see.
        int n = pr.nt_end - pr.nt_beg;
        // The last of them reaches past the entry's length: its V rows there
        // are zeroed by the V producer before its PV.
        bool last_fix = KVX && n > 0 && static_cast<int64_t>(pr.nt_end) * BN > pr.len;
        if (a.has_mask) {  // classes taken 32 key tiles at a time across the warp
          const Slot me = slot_of(pr, a, qpt);
          n = 0;
          for (int nt0 = pr.nt_beg; nt0 < pr.nt_end; nt0 += 32) {
            const int nt = nt0 + lane;
            n += __popc(__ballot_sync(
                0xffffffffu, nt < pr.nt_end && tile_class(a, pr, me, nt, m_tiles, n_tiles) != 0));
          }
          last_fix = last_fix && tile_class(a, pr, me, pr.nt_end - 1, m_tiles, n_tiles) != 0;
        }
        // Q from its landing buffer into TMEM (the A operand of every QK of
        // this query tile); the copy follows the previous tile's last QK on
        // the tensor core, and the buffer is released when the copy is done.
        const int qb = static_cast<int>(it % kQBufs);
        if (!wait(&q_full[qb], static_cast<uint32_t>((it / kQBufs) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t qs = q_base + qb * L::kTileBytes;
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            tc_cp_128x256b(t_q + ks * 8,
                           kmajor_desc(qs + (ks >> 2) * L::kChunkBytes + (ks & 3) * 32));
          tc_commit(&q_empty[qb]);
        }
        __syncwarp();
        // QK runs two tiles ahead of PV: QK(0), QK(1), PV(0), QK(2), PV(1), ...
        for (int i = 0; i < 2 && i < n && ok; ++i) ok = issue_qk(Jq++);
        for (int i = 0; i < n && ok; ++i) {
          if (last_fix && i == n - 1) {
            // The tile reaches past the entry's length: the V producer zeroes
            // those rows once it has landed (one phase of v_fix[stage] each).
            const uint32_t s = Jp % kVStages;
            ok = wait(&v_fix[s], (fix_parity >> s) & 1u);
            fix_parity ^= 1u << s;
            if (!ok) break;
          }
          ok = issue_pv(Jp++, i == 0);
          if (ok && i + 2 < n) ok = issue_qk(Jq++);
        }
        if (!ok) break;
        if (n == 0 && it > 0 &&  // no PV: O is left as it is, but the epilogue must be done
            !wait(o_free, static_cast<uint32_t>((it - 1) & 1))) {
          ok = false;
          break;
        }
        if (elect_one()) tc_commit(o_final);
        __syncwarp();
      }
      // Every MMA issued so far has completed before TMEM is released.
      if (elect_one()) tc_commit(mma_done);
      __syncwarp();
      mbar_wait_drain(mma_done, 0);
    }
  }
  } else {
    // ------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // Two warpgroups.  Thread t of warpgroup h owns row t (TMEM lane t), the
    // keys [64 h, 64 h + 64) of every S tile and the O columns
    // [h D / 2, (h + 1) D / 2).  The two threads of a row trade their partial
    // maxima (every tile) and row sums (every query tile) through shared
    // memory, under a named barrier per pair of warps that share TMEM lanes.
    constexpr int HD = D / 2;
    const int h = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t o_col = tmem + lane_base + L::kOCol + h * HD;
    const int pair_bar = 1 + (warp & 3);
    float* xch = reinterpret_cast<float*>(smem + L::kXOff);  // [X & 1][half][row]
    uint32_t X = 0;  // values traded so far (identical in both threads of a row)
    // Publish v, meet the partner, return its value; `flag` becomes the AND
    // of both threads' flags (and of the other 62 threads of the two warps).
    auto trade = [&](float v, bool& flag) -> float {
      float* slot = xch + (X & 1u) * 256;
      slot[h * 128 + row] = v;
      flag = bar_and(pair_bar, 64, flag);
      const float other = slot[(h ^ 1) * 128 + row];
      ++X;
      return other;
    };
    const int hh = row / qpt, qi = row % qpt;
    // Mask rows can be read as 16-byte vectors when base and strides allow.
    const bool mask_vec = a.has_mask && ((reinterpret_cast<uintptr_t>(a.mask) & 15u) == 0) &&
                          (a.ms[0] % 16 == 0) && (a.ms[1] % 16 == 0);
    uint32_t J = 0;
    int64_t it = 0;
    // `ok`: nothing this thread waited on has failed.  `live`: both threads
    // of the pair of warps still agree to go on; failures only end the loops
    // right after a trade, so the partner is never left at a named barrier.
    bool ok = true, live = true;
    for (int64_t x = snake(0, blockIdx.x, gridDim.x); x < work && live;
         ++it, x = snake(it, blockIdx.x, gridDim.x)) {
      const Pair pr = pair_of(x, a, m_tiles, qpt, n_tiles);
      const Slot me = slot_of(pr, a, qpt);
      const int q = me.q0 + qi;
      const bool row_valid = row < rows && q < a.Sq;
      const uint8_t* mrow =
          (a.has_mask && row_valid) ? a.mask + pr.b * a.ms[0] + static_cast<int64_t>(q) * a.ms[1]
                                    : nullptr;
      float m_ref = -INFINITY, l = 0.f;  // m_ref is the same in both threads of the row
      int nloc = 0;
      for (int nt = pr.nt_beg; nt < pr.nt_end; ++nt) {
        const int cls = tile_class(a, pr, me, nt, m_tiles, n_tiles);
        if (cls == 0) continue;
        const uint32_t s_col = tmem + lane_base + L::kSCol + (J & 1u) * BN;
        // tcgen05.ld / st are warp-collective: every decision that guards them
        // is made the same for the whole warp.
        bool okt = __all_sync(0xffffffffu, ok && mbar_wait_hot(&s_full[J & 1u], (J >> 1) & 1u,
                                                               abort_flag, a.err, kErrPrefillWait));
        // This half of the S row: its maximum.  Fully visible tiles work on
        // raw scores and fold the scale into one FMA per element below; other
        // tiles test each key against the row's visibility bits.
        const bool fast = (cls == 2) && (a.scale_log2 >= 0.f);
        uint32_t r[HK];
        float mx = -INFINITY;
        if (okt) {
          tc_fence_after();
          uint32_t vb[2] = {~0u, ~0u};
          if (!fast)
            visible_bits<2>(vb, row_valid ? mrow : nullptr, nt * BN + h * HK, a, pr, q, mask_vec);
          tmem_ld32(s_col + h * HK, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(s_col + h * HK + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_ld_wait();
          if (!fast) {
#pragma unroll
            for (int c = 0; c < HK; ++c)
              r[c] = __float_as_uint(((vb[c >> 5] >> (c & 31)) & 1u)
                                         ? __uint_as_float(r[c]) * a.scale_log2
                                         : -INFINITY);
          }
          // Eight independent running maxima, two elements per three-input max.
          float part[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) part[e] = -INFINITY;
#pragma unroll
          for (int c = 0; c < HK; c += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              part[e] = fmax3(part[e], __uint_as_float(r[c + e]), __uint_as_float(r[c + 8 + e]));
          mx = fmax3(fmax3(part[0], part[1], part[2]), fmax3(part[3], part[4], part[5]),
                     fmaxf(part[6], part[7]));
          if (fast) mx *= a.scale_log2;
        }
        // Both halves of S are in registers once the trade is done: P may then
        // overwrite the first 64 columns, half of which the other warpgroup read.
        tc_fence_before();
        const float mx_other = trade(mx, okt);
        tc_fence_after();
        if (!okt) {
          live = false;
          break;
        }
        const float m_new = fmaxf(m_ref, fmaxf(mx, mx_other));
        const bool grow = m_new > m_ref + kRescaleLog2;  // also true for -inf -> finite
        const float alpha = grow ? fast_exp2(m_ref - m_new) : 1.f;  // 0 when m_ref = -inf
        const bool o_live = grow && nloc > 0 && m_ref != -INFINITY;
        if (__any_sync(0xffffffffu, o_live)) {
          // O holds the earlier tiles' P V with the old reference: rescale this
          // half once the previous tile's PV has completed.
          if (__all_sync(0xffffffffu, mbar_wait(&o_ready[(J - 1) & 1u], ((J - 1) >> 1) & 1u,
                                                abort_flag, a.err, kErrPrefillWait))) {
            tc_fence_after();
            const float f = o_live ? alpha : 1.f;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(o_col + c * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st16(o_col + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
              tmem_st16(o_col + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
            }
            tmem_st_wait();
          } else {
            ok = false;  // carried to the next trade
          }
        }
        if (grow) {
          l *= alpha;
          m_ref = m_new;
        }
        const float ref = exp_ref(m_ref);
        // P = 2^(t - ref) as 16-bit pairs: keys [64 h, 64 h + 64) land in the
        // P columns [32 h, 32 h + 32) of S (A operand of the PV MMA).
        float lp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) lp[e] = 0.f;
        const float sc = fast ? a.scale_log2 : 1.f;
#pragma unroll
        for (int c = 0; c < HK / 32; ++c) {
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
          tmem_st16(s_col + h * (HK / 2) + c * 16, pk);
        }
        l += ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[J & 1u]);
        ++J;
        ++nloc;
      }
      if (!live) break;
      // Epilogue: out = O / l for this half row, l being both halves' sum.
      bool oke = ok && mbar_wait_hot(o_final, static_cast<uint32_t>(it & 1), abort_flag, a.err,
                                     kErrPrefillWait);
      const float l_other = trade(l, oke);
      if (!oke) {
        live = false;
        break;
      }
      tc_fence_after();
      uint16_t* orow = a.out + pr.b * a.os[0] +
                       static_cast<int64_t>(pr.kv * a.g + (hh < a.g ? hh : 0)) * a.os[1] +
                       static_cast<int64_t>(q) * a.os[2] + h * HD;
      const int dv = a.Dv - h * HD;        // columns of this half inside head_dim_v
      const float inv_l = 1.f / (l + l_other);  // l == 0: no visible key, NaN output
      if (nloc > 0) {
        // The half O row in registers: every TMEM load in flight, one wait.
        uint32_t r[HD];
#pragma unroll
        for (int c = 0; c < HD / 32; ++c)
          tmem_ld32(o_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        tmem_ld_wait();
        // O is in registers: the next tile's first PV may overwrite it now.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
        if (row_valid) {
#pragma unroll
          for (int v8 = 0; v8 < HD / 8; ++v8) {
            if (v8 * 8 >= dv) break;
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
          for (int d = 0; d < dv && d < HD; d += 8)
            *reinterpret_cast<uint4*>(orow + d) = make_uint4(nn, nn, nn, nn);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

// summary[b][mt][nt] = 0 (all hidden), 1 (mixed) or 2 (all visible) over
// mask[b, q0 : q0 + qpt, nt*BN : nt*BN + BN].  Each thread owns a 16-byte
// column piece and reads it down the tile's rows (one 16-byte load per row
// when the rows are 16-byte aligned); the BN / 16 threads of a key tile then
// combine their flags with warp shuffles.  bounds[b][mt] = the first key tile
// not all hidden and one past the last (0, 0 when every tile is hidden), so
// that the prefill kernels never walk the hidden tiles at either end.
__global__ void __launch_bounds__(128)
    gqa_mask_summary_kernel(const uint8_t* __restrict__ mask, int64_t ms0, int64_t ms1,
                            uint8_t* __restrict__ summary, int32_t* __restrict__ bounds, int Sq,
                            int Sk, int qpt, int m_tiles, int n_tiles, int BN, int vec) {
  __shared__ int lo_s, hi_s;
  if (threadIdx.x == 0) {
    lo_s = n_tiles;
    hi_s = 0;
  }
  __syncthreads();
  const int mt = blockIdx.x, b = blockIdx.y;
  const int q0 = mt * qpt;
  const int qn = min(qpt, Sq - q0);
  const uint8_t* base = mask + b * ms0 + static_cast<int64_t>(q0) * ms1;
  const int pieces = (Sk + 15) / 16;
  const int per_tile = BN / 16;  // 4 or 8: divides the warp, and 128 divides by it
  for (int c0 = 0; c0 < pieces; c0 += 128) {
    const int c = c0 + threadIdx.x;
    bool any1 = false, any0 = false;
    if (c < pieces) {
      const int j0 = c * 16;
      const int nv = min(16, Sk - j0);
      if (vec && nv == 16) {
#pragma unroll 4
        for (int r = 0; r < qn; ++r) {
          const uint4 x = *reinterpret_cast<const uint4*>(base + r * ms1 + j0);
          any1 |= (x.x | x.y | x.z | x.w) != 0u;
          any0 |= (__vcmpeq4(x.x, 0u) | __vcmpeq4(x.y, 0u) | __vcmpeq4(x.z, 0u) |
                   __vcmpeq4(x.w, 0u)) != 0u;
        }
      } else {
        for (int r = 0; r < qn; ++r)
          for (int e = 0; e < nv; ++e) {
            const uint8_t v = base[r * ms1 + j0 + e];
            any1 |= v != 0;
            any0 |= v == 0;
          }
      }
    }
    for (int o = 1; o < per_tile; o <<= 1) {
      any1 |= __shfl_xor_sync(0xffffffffu, any1, o) != 0;
      any0 |= __shfl_xor_sync(0xffffffffu, any0, o) != 0;
    }
    if (c < pieces && threadIdx.x % per_tile == 0) {
      summary[(static_cast<int64_t>(b) * m_tiles + mt) * n_tiles + c / per_tile] =
          static_cast<uint8_t>(any1 ? (any0 ? 1 : 2) : 0);
      if (any1) {
        atomicMin(&lo_s, c / per_tile);
        atomicMax(&hi_s, c / per_tile + 1);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && bounds != nullptr) {
    int32_t* bd = bounds + (static_cast<int64_t>(b) * m_tiles + mt) * 2;
    bd[0] = hi_s > lo_s ? lo_s : 0;
    bd[1] = hi_s > lo_s ? hi_s : 0;
  }
}

template <int D, bool F16, bool KVX>
int launch_prefill_t(const PrefillShape& s, const PrefillArgs& a, const PagedKV& pg,
                     const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                     cudaStream_t stream) {
  if (a.has_mask) {
    const int rc = launch_mask_summary(s, a, stream);
    if (rc != GQA_OK) return rc;
  }
  auto kern = gqa_prefill_kernel<D, F16, KVX>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Layout<D, KVX>::kBytes) != cudaSuccess)
    return GQA_ERR_CUDA;
  // The register split assumes the launch allocation it was sized for: with
  // fewer registers per thread, setmaxnreg.inc could never be granted.
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return GQA_ERR_CUDA;
  if (fa.numRegs != kLaunchRegs) return GQA_ERR_CUDA;
  kern<<<s.grid, kPrefillThreads, Layout<D, KVX>::kBytes, stream>>>(
      tmq, tmk, tmv, a, s.qpt, s.rows, s.m_tiles, s.n_tiles, s.work, pg);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace

int launch_mask_summary(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  const bool vec = (reinterpret_cast<uintptr_t>(a.mask) & 15u) == 0 && a.ms[0] % 16 == 0 &&
                   a.ms[1] % 16 == 0;
  gqa_mask_summary_kernel<<<dim3(s.m_tiles, a.B), 128, 0, stream>>>(
      a.mask, a.ms[0], a.ms[1], a.summary, a.bounds, a.Sq, a.Sk, s.qpt, s.m_tiles, s.n_tiles, BN,
      vec ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

PrefillShape plan_prefill(const gqa_problem& p, int sm_count) {
  PrefillShape s{};
  const int64_t g = p.heads_q / p.heads_kv;
  s.D = p.head_dim <= 64 ? 64 : 128;  // padded: TMA fills the columns past head_dim with zeros
  s.qpt = static_cast<int>(BM / g);
  s.rows = static_cast<int>(s.qpt * g);
  s.m_tiles = static_cast<int>((p.seq_q + s.qpt - 1) / s.qpt);
  s.n_tiles = static_cast<int>((p.seq_k + BN - 1) / BN);
  // Two query tiles per SM; one query tile per SM when an item's key tiles
  // would overflow the two-tile kernel's per-item step list.
  s.pp = s.n_tiles <= kMaxPPTiles;
  if (s.pp) {
    s.work = p.batch * p.heads_kv * ((s.m_tiles + 1) / 2);  // pairs of query tiles
    s.grid = static_cast<int>(s.work < sm_count ? s.work : sm_count);
    if (s.grid < 1) s.grid = 1;
    s.smem_bytes = pp_smem_bytes(s.D);
  } else {
    s.work = p.batch * p.heads_kv * s.m_tiles;  // query tiles
    s.grid = static_cast<int>(s.work < sm_count ? s.work : sm_count);
    if (s.grid < 1) s.grid = 1;
    s.smem_bytes = (p.kv_lens != nullptr || p.block_table != nullptr)
                       ? (s.D == 128 ? Layout<128, true>::kBytes : Layout<64, true>::kBytes)
                       : (s.D == 128 ? Layout<128, false>::kBytes : Layout<64, false>::kBytes);
  }
  s.summary_offset = kScratchOffset;
  s.workspace_end = s.summary_offset + (p.has_mask ? p.batch * s.m_tiles * s.n_tiles : 0);
  s.bounds_offset = -1;
  if (p.has_mask) {
    s.bounds_offset = ((s.workspace_end + 255) / 256) * 256;
    s.workspace_end = s.bounds_offset + p.batch * s.m_tiles * 8;
  }
  s.order_offset = -1;
  // With a mask or per-sequence lengths the items' costs vary (with each
  // entry's length): the two-tile kernel takes them heaviest first, in an
  // order sorted on the device, when sorting is cheap (a mask: every item's
  // tiles are classified; lengths alone: a range per item).
  const bool sort_cost = p.has_mask ? s.work * s.n_tiles <= kMaxOrderWork
                                    : (p.kv_lens != nullptr && s.work <= kMaxOrderWork);
  if (s.pp && sort_cost) {
    s.order_offset = ((s.workspace_end + 255) / 256) * 256;
    s.workspace_end = s.order_offset + s.work * 4;
  }
  return s;
}

int launch_prefill(const gqa_problem& p, const PrefillShape& s, const PrefillArgs& a,
                   const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                   cudaStream_t stream) {
  const bool f16 = p.dtype == GQA_DTYPE_F16;
  PagedKV pg{};
  pg.bt = p.block_table;
  pg.bt_stride = p.block_table_stride;
  pg.page_size = static_cast<int>(p.page_size);
  pg.num_pages = static_cast<int>(p.num_pages);
  const bool kvx = a.lens != nullptr || pg.bt != nullptr;
  if (s.D == 128) {
    if (kvx)
      return f16 ? launch_prefill_t<128, true, true>(s, a, pg, tmq, tmk, tmv, stream)
                 : launch_prefill_t<128, false, true>(s, a, pg, tmq, tmk, tmv, stream);
    return f16 ? launch_prefill_t<128, true, false>(s, a, pg, tmq, tmk, tmv, stream)
               : launch_prefill_t<128, false, false>(s, a, pg, tmq, tmk, tmv, stream);
  }
  if (s.D == 64) {
    if (kvx)
      return f16 ? launch_prefill_t<64, true, true>(s, a, pg, tmq, tmk, tmv, stream)
                 : launch_prefill_t<64, false, true>(s, a, pg, tmq, tmk, tmv, stream);
    return f16 ? launch_prefill_t<64, true, false>(s, a, pg, tmq, tmk, tmv, stream)
               : launch_prefill_t<64, false, false>(s, a, pg, tmq, tmk, tmv, stream);
  }
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace gqa
