// Split-K decode kernel (seq_q == 1) with its split merge fused in.
//
// Decoding re-reads the whole KV cache once per generated token and does
// about one multiply-add per byte it reads, so its time is the KV bytes over
// HBM bandwidth ("Multi-Query Attention", "Theory"; "Grouped-Query Attention
// Explained Simply", "Why it matters").  The kernel is built around that
// bound:
//
//  * Work unit = one 128-key tile of one (batch, kv head, head pass).  All units
//    of the problem are laid end to end and cut into one contiguous range per
//    CTA (a persistent grid of one CTA per SM), so every SM streams the same
//    number of bytes whatever B * Hkv is; a range may start or end inside a
//    kv head's key sequence (split-K), which leaves a partial softmax state.
//  * A producer warp streams K and V tiles with TMA (128-byte swizzled boxes,
//    so the ldmatrix reads below are bank-conflict free) into a ring of
//    shared-memory stages guarded by mbarriers; each tile crosses HBM once.
//  * Eight consumer warps (two per SM sub-partition, so that one hides the
//    other's MMA and shuffle latency) take 16 keys each of every staged
//    128-key tile and serve all g query heads of the group from it: the kv head is never expanded
//    ("Multi-Query Attention": a zero stride over the head dimension).  The
//    dot products run on the tensor cores as S^T = K Q^T with keys in the MMA
//    M dimension and the group's heads in N (g <= 8 fills one 8-wide column
//    tile), then O^T += V^T P^T; at g = 8 a CUDA-core version would need about
//    as many FMA issue slots as the HBM time allows, the MMA needs a few %.
//  * Online softmax in fp32 with warp-shuffle max/sum reductions; at the end
//    of a group the eight warps merge in shared memory.  A group handled by
//    one CTA is normalised and written straight to `out`.  A group split over
//    several CTAs leaves one partial (m, l, O) per head and CTA in the
//    workspace; each contributor then takes a ticket from the group's counter
//    and the last one merges all partials and writes bf16 `out` (the counters
//    are zeroed on the stream before the launch).  No CTA ever waits for
//    another one.
//  * The CTA that finishes a split group last usually knows it in advance:
//    the group's other contributors flushed it early in their ranges.  Once
//    the consumers are on the range's last tile, the producer warp (idle by
//    then) reads the final group's ticket count; if every other partial is
//    already published the consumers merge them directly with their own
//    states and write `out`, without publishing a partial or taking a ticket,
//    which shortens the launch's tail.
//  * Launched with programmatic stream serialisation: the next launch's CTAs
//    may start, initialise their barriers and wait (griddepcontrol.wait) while
//    this grid's last CTAs finish; before that wait nothing global is written,
//    and global memory is read only to place L2 prefetch hints for the first
//    tiles of a contiguous cache (lengths read then are clamped, and read
//    again after the wait).
//  * Per-sequence cache lengths (kv_lens): each CTA reads the B lengths,
//    counts the tiles every batch entry needs and prefix-sums them in shared
//    memory, so the units -- and the cut into CTA ranges -- cover only keys
//    that exist, and the split stays even however ragged the batch is.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int KT = kDecodeKeysPerTile;  // keys per tile
constexpr int NCW = kDecodeConsumerWarps;
constexpr int kMergeWarps = NCW / 2;    // warps whose states are merged per element
constexpr int CHUNK_BYTES = KT * 128;   // one 64-wide bf16 column chunk of a tile
constexpr int kFastMerge = 4;           // split groups merged with all loads in flight

__host__ __device__ inline int range_start(int c, int T, int P) {
  // floor(c T / P) = c q + floor(c r / P) with T = q P + r: 32-bit operations
  // only (c <= P, so c r < P^2), on every CTA's path to its first copy.
  const int q = T / P, r = T - q * P;
  return c * q + (c * r) / P;
}

// The CTA whose range [range_start(c), range_start(c + 1)) holds unit u:
// the largest c with floor(c T / P) <= u, i.e. ceil((u + 1) P / T) - 1.
__host__ __device__ inline int cta_of_unit(int u, int T, int P) {
  return static_cast<int>(((static_cast<int64_t>(u) + 1) * P + T - 1) / T) - 1;
}

// Shared memory of one CTA: the K / V ring, one Q area per stage (one 8-row
// column tile: a group's Q rows arrive with its first K tile), the flush
// scratch, the barriers and flags, then (ragged launches) the B lengths and
// B + 1 prefix sums.
template <int D, int NT>
struct DecodeSmem {
  static constexpr int kTileBytes = KT * D * 2;        // K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;   // K + V
  static constexpr int HP = 8 * NT;
  static constexpr int kQRow = D * 2 + 16;             // bytes per Q row (padded: no bank conflicts)
  static constexpr int kQAreaBytes = NT == 1 ? HP * kQRow : 0;
  static constexpr int kScrRow = D + 4;  // one row's O, then (m, l), padded (floats)
  static constexpr int kScrOBytes = kMergeWarps * HP * kScrRow * 4;
  static int bytes(int stages, int ragged_batch) {
    return 1024 /*alignment slack*/ + stages * (kStageBytes + kQAreaBytes) + kScrOBytes +
           3 * stages * 8 + 16 + (ragged_batch > 0 ? ((8 * ragged_batch + 4 + 15) / 16) * 16 : 0);
  }
};

// Unit layout of one launch.  Units run over batch entries, then kv heads,
// then head passes, then key tiles; every group (one kv head and pass of one
// batch entry) of entry b has the same number of tiles, so the units of b
// start at pre[b] (ragged) or b * per_b.
struct Sched {
  const int* pre;  // ragged: B + 1 prefix sums (shared memory), else nullptr
  const int* len;  // ragged: cache length per entry (shared memory), else nullptr
  int per_b;       // uniform: units per batch entry
  int gpb;         // groups per batch entry = Hkv * passes
  int B;
  int total;       // units of the launch (< 2^31, checked by the planner)
  int P;           // CTAs that get units: min(grid, total)

  __device__ int batch_of(int u) const {
    if (pre == nullptr) return u / per_b;
    int lo = 0, hi = B - 1;  // largest b with pre[b] <= u (pre is strictly increasing)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= u)
        lo = mid;
      else
        hi = mid - 1;
    }
    return lo;
  }
  __device__ int start_of(int b) const { return pre ? pre[b] : b * per_b; }
};

// Batch entry of the unit last looked up, with its key range.
struct Cursor {
  int b = -1;
  int beg = 0, end = 0;  // units [beg, end) belong to entry b
  KeyRange kr{};
};

__device__ __forceinline__ void seek(Cursor& c, int u, const Sched& sc, const DecodeArgs& a) {
  if (c.b >= 0 && u >= c.beg && u < c.end) return;
  c.b = sc.batch_of(u);
  c.beg = sc.start_of(c.b);
  c.kr = decode_key_range(sc.len ? sc.len[c.b] : a.Sk, a.Sk, a.Sq, a.causal, a.causal_offset,
                          a.window);
  c.end = c.beg + sc.gpb * c.kr.tiles;
}

// Group of unit u (its index over the whole launch).
__device__ __forceinline__ int group_of(int u, const Sched& sc, const DecodeArgs& a) {
  Cursor c;
  seek(c, u, sc, a);
  return c.b * sc.gpb + (u - c.beg) / c.kr.tiles;
}

// MQ: several query positions per kv head (seq_q > 1): the rows of a pass
// are (head, query) pairs, row r = head * seq_q + query, each with its own
// visible key range and mask row.
// D: the padded head dim the kernel is built for (64 or 128); columns past
// a.Dv (the problem's head dim, a multiple of 8) arrive as zeros from TMA and
// are never written.  F16: fp16 operands instead of bf16.
template <int D, int NT, bool MQ, bool F16>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const DecodeArgs a,
                      const int tiles_per_group, const int passes, const int units,
                      const int stages, uint32_t* __restrict__ counters) {
  using L = DecodeSmem<D, NT>;
  constexpr int HP = L::HP;
  constexpr int KSTEPS = D / 16;
  constexpr int CHUNKS = D / 64;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint8_t* qarea = ring + stages * L::kStageBytes;  // stage s: qarea + s * kQAreaBytes
  float* scr_o = reinterpret_cast<float*>(qarea + stages * L::kQAreaBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(scr_o) + L::kScrOBytes);
  uint64_t* full_v = full + stages;  // full: the stage's K tile landed; full_v: its V tile
  uint64_t* empty = full_v + stages;
  uint8_t* tail = reinterpret_cast<uint8_t*>(empty + stages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail);
  volatile int* last_flag = abort_flag + 1;
  int* len_s = reinterpret_cast<int*>(tail + 16);
  int* pre_s = len_s + a.B;

  volatile int* fast_flag = abort_flag + 2;  // the final split group is merged here directly
  // Ticket count of the final split group read by the producer near the end
  // of the range (kNoPeek until then; the producer's fence precedes the write).
  volatile uint32_t* peek_count = reinterpret_cast<volatile uint32_t*>(abort_flag + 3);
  constexpr uint32_t kNoPeek = 0xFFFFFFFFu;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool ragged = a.lens != nullptr;
  const int gpb = a.Hkv * passes;
  // Trace record of this CTA (diagnostics only; the address is recomputed
  // from the parameter at each use rather than held in a register).
  auto trace = [&]() { return a.trace + blockIdx.x * kDecodeTraceWords; };
  const uint64_t t_entry = (a.trace != nullptr && threadIdx.x == 0) ? globaltimer_ns() : 0;

  if (warp == NCW) {
    // The tensor maps are kernel parameters: fetch them before the wait.
    if (lane == 0) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
    }
    // Contiguous caches: start the range's first two tiles towards L2 before
    // the grid dependency resolves.  Lengths may still be being written by
    // earlier work on the stream: they are read here only to place these
    // prefetch hints, clamped into range (a stale one warms the wrong lines,
    // nothing more), and read again after the wait.  (With a block table the
    // page entries would cost a second dependent round trip before the wait,
    // which measured slower than no hints.)
    auto hint_len = [&](int b) -> int {
      if (!ragged) return a.Sk;
      const int l = __ldcg(a.lens + b);
      return l < 0 ? 0 : (l > a.Sk ? a.Sk : l);
    };
    auto hint_tiles = [&](int b) -> int {  // key tiles of each group of entry b
      return decode_key_range(hint_len(b), a.Sk, a.Sq, a.causal, a.causal_offset, a.window).tiles;
    };
    // With lengths, a batch of more than 32 entries gets no hints: its scan
    // would take a round trip per 32 entries before the wait.
    int total = a.bt == nullptr && (!ragged || a.B <= 32) ? units : 0;
    if (ragged && total > 0) {
      total = 0;
      for (int b0 = 0; b0 < a.B; b0 += 32)
        total += __reduce_add_sync(0xffffffffu, b0 + lane < a.B ? gpb * hint_tiles(b0 + lane) : 0);
    }
    const int P = static_cast<int>(gridDim.x) < total ? static_cast<int>(gridDim.x) : total;
    if (static_cast<int>(blockIdx.x) < P) {
      const int ub = range_start(blockIdx.x, total, P);
      const int ue = range_start(blockIdx.x + 1, total, P);
      for (int u = ub; u < ub + 2 && u < ue; ++u) {
        int b = -1, beg = 0;  // entry of unit u and its first unit
        if (!ragged) {
          b = u / (gpb * tiles_per_group);
          beg = b * gpb * tiles_per_group;
        } else {
          int carry = 0;
          for (int b0 = 0; b0 < a.B && b < 0; b0 += 32) {
            const int bb = b0 + lane;
            const int v = bb < a.B ? gpb * hint_tiles(bb) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int n = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += n;
            }
            const uint32_t hit = __ballot_sync(0xffffffffu, bb < a.B && carry + incl > u);
            if (hit != 0u) {
              const int l = __ffs(hit) - 1;
              b = b0 + l;
              beg = carry + __shfl_sync(0xffffffffu, incl - v, l);
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
          }
          if (b < 0) break;
        }
        const int len = hint_len(b);
        const KeyRange kr = decode_key_range(len, a.Sk, a.Sq, a.causal, a.causal_offset, a.window);
        const int tpg = ragged ? kr.tiles : tiles_per_group;
        if (tpg <= 0) break;
        const int r = u - beg, gi = r / tpg;
        const int kv = gi / passes, key0 = (r - gi * tpg + kr.t0) * KT;
        if (lane == 0) {
          if (a.bt == nullptr) {
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c) {
              tma_prefetch_4d(&tmk, c * 64, key0, kv, b);
              tma_prefetch_4d(&tmv, c * 64, key0, kv, b);
            }
          }
        }
      }
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&full_v[s], 1);
      mbar_init(&empty[s], NCW);
    }
    *abort_flag = 0;
    *fast_flag = 0;
    *peek_count = kNoPeek;
    fence_mbar_init();
  }
  // Q areas: columns past head_dim and rows past the group stay zero.
  for (int x = threadIdx.x; x < stages * L::kQAreaBytes / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(qarea)[x] = make_uint4(0u, 0u, 0u, 0u);
  if (L::kQAreaBytes > 0) fence_proxy_async_smem();  // before the bulk copies into it
  // Above, only shared memory is written and global memory is read for L2
  // hints alone; from here on global memory written by earlier work on the
  // stream (lengths, caches, counters) is read.
  griddep_wait();
  griddep_launch_dependents();
  if (ragged) {
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
      int len = a.lens[b];
      if (len < 0 || len > a.Sk) {
        if (blockIdx.x == 0) atomicOr(a.err, kErrKvLength);
        len = len < 0 ? 0 : a.Sk;
      }
      len_s[b] = len;
    }
  }
  __syncthreads();
  if (a.trace != nullptr && threadIdx.x == 0) {
    uint64_t* tr = trace();
    for (int w = 0; w < kDecodeTraceWords; ++w) tr[w] = 0;
    tr[kTrEntry] = t_entry;
    tr[kTrReady] = globaltimer_ns();
  }
  if (ragged) {
    if (warp == 0) {
      // pre[b + 1] = sum over entries <= b of (groups per entry) x (tiles of the entry).
      int carry = 0;
      for (int b0 = 0; b0 < a.B; b0 += 32) {
        const int b = b0 + lane;
        int v = 0;
        if (b < a.B)
          v = gpb * decode_key_range(len_s[b], a.Sk, a.Sq, a.causal, a.causal_offset, a.window)
                        .tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += n;
        }
        if (b < a.B) pre_s[b + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) pre_s[0] = 0;
    }
    __syncthreads();
  }
  Sched sc;
  sc.pre = ragged ? pre_s : nullptr;
  sc.len = ragged ? len_s : nullptr;
  sc.per_b = gpb * tiles_per_group;
  sc.gpb = gpb;
  sc.B = a.B;
  sc.total = ragged ? pre_s[a.B] : units;
  sc.P = static_cast<int>(gridDim.x) < sc.total ? static_cast<int>(gridDim.x) : sc.total;
  // CTAs past P (a ragged batch with fewer units than CTAs) get no range; a
  // split group counts only CTAs that hold some of its units.
  const bool has_range = static_cast<int>(blockIdx.x) < sc.P;
  const int u_begin = has_range ? range_start(blockIdx.x, sc.total, sc.P) : 0;
  const int u_end = has_range ? range_start(blockIdx.x + 1, sc.total, sc.P) : 0;

  if (warp == NCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      Cursor cu;
      // Paged cache: each 128-key tile is two 64-key boxes, each in one page.
      // The block-table entries of the next unit are loaded one iteration
      // ahead, so their latency overlaps the wait for a free stage.  A box
      // past the sequence's length takes page index num_pages, out of range:
      // TMA fills it with zeros and reads nothing.
      const bool paged = a.bt != nullptr;
      Cursor cn;
      int npage[2] = {0, 0}, nrow[2] = {0, 0};
      bool nuse[2] = {false, false};
      auto fetch_pages = [&](int u) {
        seek(cn, u, sc, a);
        const int r = u - cn.beg;
        const int gi = r / cn.kr.tiles;
        const int key0 = (r - gi * cn.kr.tiles + cn.kr.t0) * KT;
        const int len = sc.len ? sc.len[cn.b] : a.Sk;
#pragma unroll
        for (int h = 0; h < KT / kDecodePageBox; ++h) {
          const int key = key0 + h * kDecodePageBox;
          nuse[h] = key < len;
          nrow[h] = key % a.page_size;
          npage[h] = nuse[h] ? __ldg(a.bt + cn.b * a.bt_stride + key / a.page_size) : a.num_pages;
        }
      };
      if (paged && u_begin < u_end) fetch_pages(u_begin);
      for (int u = u_begin; u < u_end; ++u, ++it) {
        const int s = it % stages;
        const uint32_t round = static_cast<uint32_t>(it / stages);
        if (round > 0 &&
            !mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, a.err, kErrDecodeWait, a.wait_ns))
          break;
        if (u == a.withhold_unit) {
          // Test of the bounded waits (gqa_debug_decode_withhold): this
          // unit's copies are never issued, so the consumers' wait for it
          // runs out and aborts the CTA; nothing more is issued, so every
          // copy in flight belongs to an earlier unit and lands.
          const uint64_t t0 = globaltimer_ns();
          while (!*abort_flag && globaltimer_ns() - t0 < 4 * a.wait_ns) {
          }
          break;
        }
        seek(cu, u, sc, a);
        const int r = u - cu.beg;
        const int gi = r / cu.kr.tiles;  // group within the entry: kv * passes + pass
        const int key0 = (r - gi * cu.kr.tiles + cu.kr.t0) * KT;
        const int kv = gi / passes;
        const int b = cu.b;
        uint8_t* st = ring + s * L::kStageBytes;
        // The first tile of a group in this range brings the group's Q rows
        // (one 8-row column tile) into the stage's Q area, on the same
        // barrier: the consumers then start the group without a global load.
        const bool q_rows = L::kQAreaBytes > 0 && (u == u_begin || r - gi * cu.kr.tiles == 0);
        const int pass = gi % passes;
        const int nq = q_rows ? min(HP, a.rows - pass * HP) : 0;
        const uint32_t q_bytes = static_cast<uint32_t>(nq * a.Dv * 2);
        auto issue_q = [&]() {
          uint8_t* qd = qarea + s * L::kQAreaBytes;
          for (int hr = 0; hr < nq; ++hr) {
            const int hl = pass * HP + hr;
            const int hh = MQ ? hl / a.Sq : hl;
            const int qi = MQ ? hl % a.Sq : 0;
            const uint16_t* src = a.q + b * a.qs[0] + static_cast<int64_t>(kv * a.g + hh) * a.qs[1] +
                                  static_cast<int64_t>(qi) * a.qs[2];
            bulk_load(qd + hr * L::kQRow, src, static_cast<uint32_t>(a.Dv * 2), &full[s]);
          }
        };
        if (paged) {
          int page[2], prow[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            page[h] = npage[h];
            prow[h] = nrow[h];
            if (nuse[h] && (page[h] < 0 || page[h] >= a.num_pages)) {
              atomicOr(a.err, kErrPage);
              page[h] = a.num_pages;  // read as zeros
            }
          }
          if (u + 1 < u_end) fetch_pages(u + 1);
          mbar_arrive_expect_tx(&full[s], L::kTileBytes + q_bytes);
          issue_q();
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c)
              tma_load_4d(st + c * CHUNK_BYTES + h * kDecodePageBox * 128, &tmk, &full[s], c * 64,
                          prow[h], kv, page[h]);
          mbar_arrive_expect_tx(&full_v[s], L::kTileBytes);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c)
              tma_load_4d(st + L::kTileBytes + c * CHUNK_BYTES + h * kDecodePageBox * 128, &tmv,
                          &full_v[s], c * 64, prow[h], kv, page[h]);
          if (a.trace != nullptr && it == 0) trace()[kTrFirstIssue] = globaltimer_ns();
          continue;
        }
        mbar_arrive_expect_tx(&full[s], L::kTileBytes + q_bytes);
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c)
          tma_load_4d(st + c * CHUNK_BYTES, &tmk, &full[s], c * 64, key0, kv, b);
        issue_q();
        if (a.trace != nullptr && it == 0) trace()[kTrFirstIssue] = globaltimer_ns();
        mbar_arrive_expect_tx(&full_v[s], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c)
          tma_load_4d(st + L::kTileBytes + c * CHUNK_BYTES, &tmv, &full_v[s], c * 64, key0, kv, b);
      }
      if (a.trace != nullptr) trace()[kTrLastIssue] = globaltimer_ns();
      // Final group split over several CTAs: once the consumers have released
      // the range's second-to-last tile, read the group's ticket count for
      // the consumers' final flush (a fence makes the partials published
      // before those tickets visible to this CTA).
      if (!*abort_flag && u_begin < u_end) {
        seek(cu, u_end - 1, sc, a);
        const int gi = (u_end - 1 - cu.beg) / cu.kr.tiles;
        const int g_beg = cu.beg + gi * cu.kr.tiles;
        if (cta_of_unit(g_beg, sc.total, sc.P) !=
            cta_of_unit(g_beg + cu.kr.tiles - 1, sc.total, sc.P)) {
          const int j = it - 2;  // second-to-last unit of the range
          const bool ready =
              j < 0 || mbar_wait(&empty[j % stages], static_cast<uint32_t>((j / stages) & 1),
                                 abort_flag, a.err, kErrDecodeWait, a.wait_ns);
          if (ready) {
            const uint32_t n = ld_relaxed_gpu(&counters[cu.b * gpb + gi]);
            fence_acq_rel_gpu();
            *peek_count = n;
          }
        }
      }
      // Unwind: make sure no copy is still landing in this CTA's shared memory.
      if (*abort_flag) {
        const int issued = it;
        for (int j = (issued > stages ? issued - stages : 0); j < issued; ++j) {
          mbar_wait_drain(&full[j % stages], static_cast<uint32_t>((j / stages) & 1),
                          a.wait_ns / 4);
          mbar_wait_drain(&full_v[j % stages], static_cast<uint32_t>((j / stages) & 1),
                          a.wait_ns / 4);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // Q as MMA B fragments: for one column tile, in registers, read from the
    // Q area of the stage that brought the group's first tile; for two, in
    // shared memory (head rows padded to D * 2 + 16 bytes, conflict-free for
    // ldmatrix), aliasing the flush scratch, to stay within the registers
    // that 288 threads may hold.
    constexpr bool kQSmem = NT == 2;
    constexpr int kQRow = L::kQRow;
    static_assert(!kQSmem || HP * kQRow <= L::kScrOBytes, "Q rows must fit the scratch");
    uint32_t bq[kQSmem ? 1 : NT][kQSmem ? 1 : KSTEPS][2];
    uint8_t* q_smem = reinterpret_cast<uint8_t*>(scr_o);
    float o[NT][KSTEPS][4];
    float m_run[NT][2], l_run[NT][2];
    int cur = -1;                // group being accumulated
    int cur_beg = 0;             // its first unit
    int cur_tiles = 1;           // its units
    int cur_lo = 0, cur_hi = 0, cur_len = 0;  // its key range and cache length
    int b = 0, kv = 0, pass = 0;
    const uint8_t* mrow = nullptr;
    const int first_grp = u_begin < u_end ? group_of(u_begin, sc, a) : -1;
    bool q_pending = false;  // the group's Q fragments come with its first stage

    auto reset_state = [&]() {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
          for (int c = 0; c < 4; ++c) o[nt][mt][c] = 0.f;
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
      }
    };

    // Visible keys [vlo, vhi) and mask row of the two rows (columns) this
    // thread's S^T fragments hold in each column tile.
    int vlo[NT][2], vhi[NT][2];
    const uint8_t* vmask[NT][2];

    // Global address of row hl (a head, or a (head, query) pair) of this pass.
    auto q_row = [&](int hl) -> const uint16_t* {
      const int hh = MQ ? hl / a.Sq : hl;
      const int qi = MQ ? hl % a.Sq : 0;
      return a.q + b * a.qs[0] + (int64_t)(kv * a.g + hh) * a.qs[1] + (int64_t)qi * a.qs[2];
    };

    auto load_q = [&]() {
      if (kQSmem) {
        // 16-byte pieces of the pass's HP rows; rows past the group are zero.
        for (int x = threadIdx.x; x < HP * (D / 8); x += NCW * 32) {
          const int r = x / (D / 8), c = x % (D / 8);
          const int hl = pass * HP + r;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (hl < a.rows && c * 8 < a.Dv) v = *reinterpret_cast<const uint4*>(q_row(hl) + c * 8);
          *reinterpret_cast<uint4*>(q_smem + r * kQRow + c * 16) = v;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (MQ) {
            const int r = pass * HP + nt * 8 + (lane & 3) * 2 + e;
            const int i = (r < a.rows ? r : 0) % a.Sq;
            const int64_t lim = i + a.causal_offset + (cur_len - a.Sk);  // query i's diagonal
            int64_t lo = 0, hi = cur_len;
            if (a.causal) {
              hi = lim + 1 < hi ? lim + 1 : hi;
              if (a.window > 0 && lim - a.window + 1 > 0) lo = lim - a.window + 1;
            }
            vlo[nt][e] = static_cast<int>(lo < cur_len ? lo : cur_len);  // within [0, len]
            vhi[nt][e] = static_cast<int>(hi > 0 ? hi : 0);
            vmask[nt][e] = a.mask ? a.mask + b * a.ms[0] + static_cast<int64_t>(i) * a.ms[1] : nullptr;
          } else {
            vlo[nt][e] = cur_lo;
            vhi[nt][e] = cur_hi;
            vmask[nt][e] = mrow;
          }
        }
      }
    };

    // One column tile: the group's B fragments from the Q area of stage st
    // (rows past the group and columns past head_dim are zero there).
    auto load_q_stage = [&](int st) {
      if (!kQSmem) {
        const uint8_t* qrow = qarea + st * L::kQAreaBytes + (lane >> 2) * kQRow;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int d0 = ks * 16 + (lane & 3) * 2;
          bq[0][kQSmem ? 0 : ks][0] = *reinterpret_cast<const uint32_t*>(qrow + d0 * 2);
          bq[0][kQSmem ? 0 : ks][1] = *reinterpret_cast<const uint32_t*>(qrow + (d0 + 8) * 2);
        }
      }
    };

    // Merge the eight warps' states of the finished group and write it out
    // (whole in this CTA) or publish one partial (split).  Warps w and w + 4
    // hold the same fragment positions of different keys: w + 4 hands its
    // state over, then the four merged states combine per output element.
    // The scratch rows keep (m, l) in the padding after the D values.
    auto flush = [&](bool final_flush) {
      constexpr int R = L::kScrRow;
      // CTAs sharing this group (every CTA computes the same ranges).
      const int c_lo = cta_of_unit(cur_beg, sc.total, sc.P);
      const int c_hi = cta_of_unit(cur_beg + cur_tiles - 1, sc.total, sc.P);
      const int n_contrib = c_hi - c_lo + 1;
      // Fast final merge: every other contributor has published (the early
      // ticket read saw n - 1) and one 4-wide column group per thread covers
      // the group's output.
      constexpr bool kOneQuadPerThread = HP * D / 4 <= NCW * 32;
      if (kOneQuadPerThread && final_flush && threadIdx.x == 0) {
        int fast = 0;
        if (n_contrib > 1 && n_contrib <= kFastMerge &&
            *peek_count == static_cast<uint32_t>(n_contrib - 1)) {
          // The producer read the tickets and fenced at gpu scope before
          // publishing the count in shared memory; acquiring that store at
          // CTA scope orders the partial loads below after the other CTAs'
          // releases.
          fence_acq_rel_cta();
          fast = 1;
        }
        *fast_flag = fast;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float l = l_run[nt][e];
          l += __shfl_xor_sync(0xffffffffu, l, 4);
          l += __shfl_xor_sync(0xffffffffu, l, 8);
          l += __shfl_xor_sync(0xffffffffu, l, 16);
          l_run[nt][e] = l;
        }
      float* my_rows = scr_o + (warp & 3) * HP * R;
      // Q lives in the scratch: every warp must be done with its last S first.
      if (kQSmem) asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      auto put_state = [&]() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int h = nt * 8 + (lane & 3) * 2 + (c & 1);
              const int d = mt * 16 + (lane >> 2) + ((c & 2) ? 8 : 0);
              my_rows[h * R + d] = o[nt][mt][c];
            }
          if (lane < 4) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int h = nt * 8 + lane * 2 + e;
              my_rows[h * R + D] = m_run[nt][e];
              my_rows[h * R + D + 1] = l_run[nt][e];
            }
          }
        }
      };
      if (warp >= kMergeWarps) put_state();
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      // Partial slot of CTA cc for this group: only a range's first and last
      // groups can be split, so two slots per CTA suffice.
      auto slot_of = [&](int cc) -> int {
        const int first = group_of(range_start(cc, sc.total, sc.P), sc, a);
        return (cc * 2 + (first == cur ? 0 : 1)) * HP;
      };
      // Fast final merge: this thread's quad of every other partial is
      // requested now, so that the loads overlap the eight-warp merge.
      const bool fast = kOneQuadPerThread && final_flush && *fast_flag != 0;
      float2 rml[kFastMerge];
      float4 rov[kFastMerge];
      if (fast && threadIdx.x < HP * D / 4) {
        const int h = threadIdx.x / (D / 4), d = (threadIdx.x % (D / 4)) * 4;
#pragma unroll
        for (int k = 0; k < kFastMerge; ++k) {
          const int cc = c_lo + k;
          if (k < n_contrib && cc != static_cast<int>(blockIdx.x)) {
            const int base = slot_of(cc);
            rml[k] = __ldcg(&a.part_ml[base + h]);
            rov[k] = __ldcg(reinterpret_cast<const float4*>(&a.part_o[(base + h) * D + d]));
          }
        }
      }
      if (warp < kMergeWarps) {
        float wa[NT][2], wb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = nt * 8 + (lane & 3) * 2 + e;
            const float mp = my_rows[h * R + D], lp = my_rows[h * R + D + 1];
            const float M = fmaxf(m_run[nt][e], mp);
            wa[nt][e] = M == -INFINITY ? 0.f : fast_exp2(m_run[nt][e] - M);
            wb[nt][e] = M == -INFINITY ? 0.f : fast_exp2(mp - M);
            l_run[nt][e] = l_run[nt][e] * wa[nt][e] + lp * wb[nt][e];
            m_run[nt][e] = M;
          }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int h = nt * 8 + (lane & 3) * 2 + (c & 1);
              const int d = mt * 16 + (lane >> 2) + ((c & 2) ? 8 : 0);
              o[nt][mt][c] = o[nt][mt][c] * wa[nt][c & 1] + my_rows[h * R + d] * wb[nt][c & 1];
            }
        __syncwarp();
        put_state();
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      if (a.trace != nullptr && final_flush && threadIdx.x == 0) trace()[kTrFinalMerged] = globaltimer_ns();
      auto m_of = [&](int w, int h) { return scr_o[(w * HP + h) * R + D]; };
      auto l_of = [&](int w, int h) { return scr_o[(w * HP + h) * R + D + 1]; };
      // Output row of row hr of this pass (a head, or a (head, query) pair).
      auto out_row = [&](int hr) -> uint16_t* {
        const int r = pass * HP + hr;
        const int hh = MQ ? r / a.Sq : r;
        const int qi = MQ ? r % a.Sq : 0;
        return a.out + b * a.os[0] + static_cast<int64_t>(kv * a.g + hh) * a.os[1] +
               static_cast<int64_t>(qi) * a.os[2];
      };
      if (c_lo == c_hi) {
        // The whole group is in this CTA: normalise and write out, two
        // elements per thread.
        for (int idx = threadIdx.x; idx < HP * D / 2; idx += NCW * 32) {
          const int h = idx / (D / 2), d = (idx % (D / 2)) * 2;
          if (pass * HP + h >= a.rows || d >= a.Dv) continue;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kMergeWarps; ++w) M = fmaxf(M, m_of(w, h));
          float l = 0.f, acc0 = 0.f, acc1 = 0.f;
          if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kMergeWarps; ++w) {
              const float sc = fast_exp2(m_of(w, h) - M);
              l += sc * l_of(w, h);
              const float2 ov = *reinterpret_cast<const float2*>(&scr_o[(w * HP + h) * R + d]);
              acc0 += sc * ov.x;
              acc1 += sc * ov.y;
            }
          }
          const float inv = 1.f / l;  // l == 0: NaN
          *reinterpret_cast<uint32_t*>(out_row(h) + d) = pack2<F16>(acc0 * inv, acc1 * inv);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
        if (a.trace != nullptr && final_flush && threadIdx.x == 0) {
          trace()[kTrFinalDone] = globaltimer_ns();
          trace()[kTrFinalKind] = 0;
        }
        return;
      }
      if (fast) {
        // Every other partial of the group is published and was requested
        // above: merge them with the eight warps' states and write out.
        if (threadIdx.x < HP * D / 4) {
          const int h = threadIdx.x / (D / 4), d = (threadIdx.x % (D / 4)) * 4;
          if (pass * HP + h < a.rows && d < a.Dv) {
            auto other = [&](int k) { return k < n_contrib && c_lo + k != static_cast<int>(blockIdx.x); };
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kMergeWarps; ++w) M = fmaxf(M, m_of(w, h));
#pragma unroll
            for (int k = 0; k < kFastMerge; ++k)
              if (other(k)) M = fmaxf(M, rml[k].x);
            float Lsum = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (M != -INFINITY) {
#pragma unroll
              for (int w = 0; w < kMergeWarps; ++w) {
                const float wt = fast_exp2(m_of(w, h) - M);
                Lsum += wt * l_of(w, h);
                const float4 ov = *reinterpret_cast<const float4*>(&scr_o[(w * HP + h) * R + d]);
                acc.x += wt * ov.x;
                acc.y += wt * ov.y;
                acc.z += wt * ov.z;
                acc.w += wt * ov.w;
              }
#pragma unroll
              for (int k = 0; k < kFastMerge; ++k) {
                if (other(k)) {
                  const float wt = fast_exp2(rml[k].x - M);
                  Lsum += wt * rml[k].y;
                  acc.x += wt * rov[k].x;
                  acc.y += wt * rov[k].y;
                  acc.z += wt * rov[k].z;
                  acc.w += wt * rov[k].w;
                }
              }
            }
            const float inv = 1.f / Lsum;  // Lsum == 0: NaN
            uint2 pk;
            pk.x = pack2<F16>(acc.x * inv, acc.y * inv);
            pk.y = pack2<F16>(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2*>(out_row(h) + d) = pk;
          }
        }
        // Every contributor has arrived: the counter goes back to zero for
        // the next launch (which reads it only after this grid completes).
        if (threadIdx.x == 0) counters[cur] = 0u;
        asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
        if (a.trace != nullptr && threadIdx.x == 0) {
          trace()[kTrFinalDone] = globaltimer_ns();
          trace()[kTrFinalKind] = 2;
        }
        return;
      }
      // Split group: publish this CTA's partial (float4 stores), then take a
      // ticket on the group's counter.
      const int slot = (static_cast<int>(blockIdx.x) * 2 + (cur == first_grp ? 0 : 1)) * HP;
      for (int idx = threadIdx.x; idx < HP * D / 4; idx += NCW * 32) {
        const int h = idx / (D / 4), d = (idx % (D / 4)) * 4;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kMergeWarps; ++w) M = fmaxf(M, m_of(w, h));
        float l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kMergeWarps; ++w) {
            const float sc = fast_exp2(m_of(w, h) - M);
            l += sc * l_of(w, h);
            const float4 ov = *reinterpret_cast<const float4*>(&scr_o[(w * HP + h) * R + d]);
            acc.x += sc * ov.x;
            acc.y += sc * ov.y;
            acc.z += sc * ov.z;
            acc.w += sc * ov.w;
          }
        }
        *reinterpret_cast<float4*>(&a.part_o[(slot + h) * D + d]) = acc;
        if (d == 0) a.part_ml[slot + h] = make_float2(M, l);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      if (threadIdx.x == 0) {
        // The barrier above makes every thread's partial visible to thread 0;
        // its acquire-release add at gpu scope publishes them (release) and,
        // for the last arriver, makes the others' partials visible (acquire).
        const uint32_t n = static_cast<uint32_t>(c_hi - c_lo + 1);
        const uint32_t old = atom_add_acq_rel_gpu(&counters[cur], 1u);
        *last_flag = (old == n - 1) ? 1 : 0;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      if (*last_flag) {
        // Last contributor: every other partial of the group is published.
        const int n = static_cast<int>(c_hi - c_lo + 1);
        if (n <= kFastMerge) {
          // Few contributors: every load of a thread's elements in flight at once.
          int base[kFastMerge];
#pragma unroll
          for (int k = 0; k < kFastMerge; ++k) base[k] = slot_of(c_lo + (k < n ? k : 0));
          for (int idx = threadIdx.x; idx < HP * D / 4; idx += NCW * 32) {
            const int h = idx / (D / 4), d = (idx % (D / 4)) * 4;
            if (pass * HP + h >= a.rows || d >= a.Dv) continue;
            float2 ml[kFastMerge];
            float4 ov[kFastMerge];
#pragma unroll
            for (int k = 0; k < kFastMerge; ++k) {
              if (k < n) {
                ml[k] = __ldcg(&a.part_ml[base[k] + h]);
                ov[k] = __ldcg(reinterpret_cast<const float4*>(&a.part_o[(base[k] + h) * D + d]));
              }
            }
            float M = -INFINITY;
#pragma unroll
            for (int k = 0; k < kFastMerge; ++k)
              if (k < n) M = fmaxf(M, ml[k].x);
            float Lsum = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (M != -INFINITY) {
#pragma unroll
              for (int k = 0; k < kFastMerge; ++k) {
                if (k < n) {
                  const float w = fast_exp2(ml[k].x - M);
                  Lsum += w * ml[k].y;
                  acc.x += w * ov[k].x;
                  acc.y += w * ov[k].y;
                  acc.z += w * ov[k].z;
                  acc.w += w * ov[k].w;
                }
              }
            }
            const float inv = 1.f / Lsum;  // Lsum == 0: NaN
            uint2 pk;
            pk.x = pack2<F16>(acc.x * inv, acc.y * inv);
            pk.y = pack2<F16>(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2*>(out_row(h) + d) = pk;
          }
        } else {
          // Many contributors: stage each one's slot and each row's merged
          // (max, sum) in shared memory (the scratch rows are free now), then
          // accumulate O with 16-byte loads.
          int* sm_slot = reinterpret_cast<int*>(scr_o);
          float* sm_ml = scr_o + kMergeWarps * HP * R / 2;  // HP x (M, L), past the slots
          for (int k = threadIdx.x; k < n; k += NCW * 32)
            sm_slot[k] = slot_of(c_lo + k);
          asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
          if (threadIdx.x < HP) {
            const int h = threadIdx.x;
            float M = -INFINITY;
#pragma unroll 4
            for (int k = 0; k < n; ++k) M = fmaxf(M, __ldcg(&a.part_ml[sm_slot[k] + h]).x);
            float Lsum = 0.f;
            if (M != -INFINITY) {
#pragma unroll 4
              for (int k = 0; k < n; ++k) {
                const float2 ml = __ldcg(&a.part_ml[sm_slot[k] + h]);
                Lsum += fast_exp2(ml.x - M) * ml.y;
              }
            }
            sm_ml[2 * h] = M;
            sm_ml[2 * h + 1] = Lsum;
          }
          asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
          for (int idx = threadIdx.x; idx < HP * D / 4; idx += NCW * 32) {
            const int h = idx / (D / 4), d = (idx % (D / 4)) * 4;
            if (pass * HP + h >= a.rows || d >= a.Dv) continue;
            const float M = sm_ml[2 * h], Lsum = sm_ml[2 * h + 1];
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (M != -INFINITY) {
#pragma unroll 4
              for (int k = 0; k < n; ++k) {
                const int sl = sm_slot[k] + h;
                const float w = fast_exp2(__ldcg(&a.part_ml[sl]).x - M);
                const float4 ov = __ldcg(reinterpret_cast<const float4*>(&a.part_o[sl * D + d]));
                acc.x += w * ov.x;
                acc.y += w * ov.y;
                acc.z += w * ov.z;
                acc.w += w * ov.w;
              }
            }
            const float inv = 1.f / Lsum;  // Lsum == 0: NaN
            uint2 pk;
            pk.x = pack2<F16>(acc.x * inv, acc.y * inv);
            pk.y = pack2<F16>(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2*>(out_row(h) + d) = pk;
          }
        }
        if (threadIdx.x == 0) atomicExch(&counters[cur], 0u);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      if (a.trace != nullptr && final_flush && threadIdx.x == 0) {
        trace()[kTrFinalDone] = globaltimer_ns();
        trace()[kTrFinalKind] = 1;
      }
    };

    int it = 0;
    Cursor cu;
    for (int u = u_begin; u < u_end; ++u, ++it) {
      seek(cu, u, sc, a);
      const int r = u - cu.beg;
      const int gi = r / cu.kr.tiles;
      const int grp = cu.b * gpb + gi;
      const int tile = r - gi * cu.kr.tiles + cu.kr.t0;
      if (grp != cur) {
        if (cur >= 0) {
          const uint64_t t0 = (a.trace != nullptr && threadIdx.x == 0) ? globaltimer_ns() : 0;
          flush(false);
          if (a.trace != nullptr && threadIdx.x == 0) {
            trace()[kTrMidFlushNs] += globaltimer_ns() - t0;
            trace()[kTrFlushes] += 1;
          }
        }
        cur = grp;
        cur_beg = cu.beg + gi * cu.kr.tiles;
        cur_tiles = cu.kr.tiles;
        cur_lo = cu.kr.lo;
        cur_hi = cu.kr.hi;
        cur_len = sc.len ? sc.len[cu.b] : a.Sk;
        pass = gi % passes;
        kv = gi / passes;
        b = cu.b;
        mrow = a.mask ? a.mask + b * a.ms[0] : nullptr;
        load_q();
        reset_state();
        q_pending = true;
      }
      const int s = it % stages;
      const uint32_t round = static_cast<uint32_t>(it / stages);
      // A wait that gives up sets the abort flag; from then on every wait
      // fails at once and the warps skip the arithmetic but keep walking the
      // units, so that all eight reach the same flush() barriers.
      if (!mbar_wait(&full[s], round & 1u, abort_flag, a.err, kErrDecodeWait, a.wait_ns)) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        continue;
      }
      if (a.trace != nullptr && it == 0 && threadIdx.x == 0) trace()[kTrFirstLand] = globaltimer_ns();
      if (q_pending) {
        load_q_stage(s);
        q_pending = false;
      }
      const uint32_t kbase = smem_u32(ring + s * L::kStageBytes);
      const uint32_t vbase = kbase + L::kTileBytes;

      // S^T[16 keys x 8 heads] = K[16 x D] Q^T[D x 8] per column tile.  With
      // one column tile, even and odd k-steps go to two accumulators (half the
      // dependent MMA chain); two column tiles already interleave two chains.
      constexpr bool kSplit = NT == 1;
      float sc[NT][4], sc2[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[nt][c] = sc2[nt][c] = 0.f;
      {
        const int mi = lane >> 3;
        const int r = warp * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int u16 = ((ks & 3) << 1) + (mi >> 1);
          const uint32_t addr =
              kbase + (ks >> 2) * CHUNK_BYTES + r * 128 + ((u16 ^ (r & 7)) << 4);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(a0, a1, a2, a3, addr);
          if (kQSmem) {
            // B fragments of both column tiles: matrices (rows 0-7 | 8-15) x
            // (d ks*16 + 0-7 | + 8-15), row and half picked by the lane.
            const int qr = ((lane >> 4) << 3) + (lane & 7);
            const uint32_t qaddr =
                smem_u32(q_smem) + qr * kQRow + ks * 32 + ((lane >> 3) & 1) * 16;
            uint32_t q0, q1, q2, q3;
            ldmatrix_x4(q0, q1, q2, q3, qaddr);
            mma_16816<F16>(sc[0], a0, a1, a2, a3, q0, q1);
            mma_16816<F16>(sc[NT - 1], a0, a1, a2, a3, q2, q3);
          } else {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_16816<F16>((kSplit && (ks & 1)) ? sc2[nt] : sc[nt], a0, a1, a2, a3,
                             bq[kQSmem ? 0 : nt][kQSmem ? 0 : ks][0],
                             bq[kQSmem ? 0 : nt][kQSmem ? 0 : ks][1]);
          }
        }
        if (kSplit) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) sc[nt][c] += sc2[nt][c];
        }
      }

      // Visibility of this thread's two keys for its rows.
      const int key0 = tile * KT + warp * 16 + (lane >> 2);
      const int key1 = key0 + 8;
      auto vis = [&](int key, int nt, int e) -> bool {
        return key >= vlo[nt][e] && key < vhi[nt][e] && mask_allows(vmask[nt][e], key);
      };

      uint32_t pt0[NT], pt1[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float tv[4];
        tv[0] = vis(key0, nt, 0) ? sc[nt][0] * a.scale_log2 : -INFINITY;
        tv[1] = vis(key0, nt, 1) ? sc[nt][1] * a.scale_log2 : -INFINITY;
        tv[2] = vis(key1, nt, 0) ? sc[nt][2] * a.scale_log2 : -INFINITY;
        tv[3] = vis(key1, nt, 1) ? sc[nt][3] * a.scale_log2 : -INFINITY;
        float alpha[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mx = fmaxf(tv[e], tv[e + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_run[nt][e], mx);
          const float ref = exp_ref(m_new);
          alpha[e] = fast_exp2(m_run[nt][e] - ref);
          m_run[nt][e] = m_new;
          tv[e] = fast_exp2(tv[e] - ref);
          tv[e + 2] = fast_exp2(tv[e + 2] - ref);
          l_run[nt][e] = l_run[nt][e] * alpha[e] + tv[e] + tv[e + 2];
        }
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
          o[nt][mt][0] *= alpha[0];
          o[nt][mt][1] *= alpha[1];
          o[nt][mt][2] *= alpha[0];
          o[nt][mt][3] *= alpha[1];
        }
        // P^T as the B operand: transpose the two 8x8 (keys x heads) blocks.
        pt0[nt] = movmatrix_trans(pack2<F16>(tv[0], tv[1]));
        pt1[nt] = movmatrix_trans(pack2<F16>(tv[2], tv[3]));
      }

      // O^T[D x 8] += V^T[D x 16 keys] P^T[16 keys x 8], once the V tile is in.
      if (!mbar_wait(&full_v[s], round & 1u, abort_flag, a.err, kErrDecodeWait, a.wait_ns)) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        continue;
      }
      // Cache rows past the sequence's length may hold anything (NaN
      // included), and zero weights would not cancel them: their V values
      // are cleared in the A fragments.  Fragments a0 / a1 hold keys
      // 2 (lane % 4) + {0, 1} of this warp's 16, a2 / a3 the same + 8, one
      // key per 16-bit half.
      uint32_t vm_lo = ~0u, vm_hi = ~0u;
      if ((tile + 1) * KT > cur_len) {
        const int kb = tile * KT + warp * 16 + (lane & 3) * 2;
        vm_lo = (kb < cur_len ? 0xFFFFu : 0u) | (kb + 1 < cur_len ? 0xFFFF0000u : 0u);
        vm_hi = (kb + 8 < cur_len ? 0xFFFFu : 0u) | (kb + 9 < cur_len ? 0xFFFF0000u : 0u);
      }
      {
        const int mi = lane >> 3;
        const int key = warp * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
          const int dcol = mt * 16 + (mi & 1) * 8;
          const int u16 = (dcol & 63) >> 3;
          const uint32_t addr =
              vbase + (dcol >> 6) * CHUNK_BYTES + key * 128 + ((u16 ^ (key & 7)) << 4);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(a0, a1, a2, a3, addr);
          a0 &= vm_lo;
          a1 &= vm_lo;
          a2 &= vm_hi;
          a3 &= vm_hi;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_16816<F16>(o[nt][mt], a0, a1, a2, a3, pt0[nt], pt1[nt]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (a.trace != nullptr && threadIdx.x == 0) trace()[kTrLastTile] = globaltimer_ns();
    if (cur >= 0) {
      flush(true);  // after an abort too (its output is undefined, the error word set)
      if (a.trace != nullptr && threadIdx.x == 0) trace()[kTrFlushes] += 1;
    }
  }
  __syncthreads();
  if (a.trace != nullptr && threadIdx.x == 0) {
    uint64_t* tr = trace();
    tr[kTrExit] = globaltimer_ns();
    tr[kTrSm] = static_cast<uint64_t>(sm_id()) | (static_cast<uint64_t>(blockIdx.x) << 32);
    tr[kTrUnits] = static_cast<uint64_t>(u_end - u_begin);
  }
}

template <int D, int NT, bool MQ, bool F16>
int launch_decode_t(const DecodeShape& s, const DecodeArgs& a, const CUtensorMap& tmk,
                    const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = gqa_decode_kernel<D, NT, MQ, F16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, s.smem_bytes) !=
      cudaSuccess)
    return GQA_ERR_CUDA;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(s.grid));
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(s.smem_bytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tmk, tmv, a, s.tiles_per_group, s.passes,
                         static_cast<int>(s.units), s.stages, a.counters) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return GQA_OK;
}

}  // namespace

DecodeShape plan_decode(const gqa_problem& p, int sm_count) {
  DecodeShape s{};
  const int64_t g = p.heads_q / p.heads_kv;
  const int64_t rows = g * p.seq_q;  // (head, query) rows per kv head
  s.D = p.head_dim <= 64 ? 64 : 128;  // padded: TMA fills the columns past head_dim with zeros
  s.NT = rows <= 8 ? 1 : 2;
  s.HP = 8 * s.NT;
  s.passes = static_cast<int>((rows + s.HP - 1) / s.HP);
  s.ragged = p.kv_lens != nullptr;
  // Without kv_lens every group streams the same tiles; with them a group
  // needs at most the tiles of the whole capacity.
  s.tiles_per_group =
      s.ragged ? static_cast<int>((p.seq_k + KT - 1) / KT)
               : decode_key_range(p.seq_k, p.seq_k, p.seq_q, p.causal, p.causal_offset, p.window)
                     .tiles;
  if (s.tiles_per_group < 1) s.tiles_per_group = 1;
  s.groups = p.batch * p.heads_kv * s.passes;
  s.units = s.groups * s.tiles_per_group;
  s.grid = static_cast<int>(s.units < sm_count ? s.units : sm_count);
  if (s.grid < 1) s.grid = 1;
  const int rb = s.ragged ? static_cast<int>(p.batch) : 0;
  s.stages = s.D == 128 ? 3 : 6;  // 192 KB of K/V in flight per SM
  for (;; --s.stages) {
    if (s.D == 128 && s.NT == 1)
      s.smem_bytes = DecodeSmem<128, 1>::bytes(s.stages, rb);
    else if (s.D == 128)
      s.smem_bytes = DecodeSmem<128, 2>::bytes(s.stages, rb);
    else if (s.NT == 1)
      s.smem_bytes = DecodeSmem<64, 1>::bytes(s.stages, rb);
    else
      s.smem_bytes = DecodeSmem<64, 2>::bytes(s.stages, rb);
    if (s.smem_bytes <= kDecodeMaxSmem || s.stages <= 2) break;
  }
  // Two partial slots per CTA: its first and its last group.  The ticket
  // counters sit in the workspace's counter region, which stays zero between
  // calls; a launch with more groups keeps them past it and zeroes them.
  const int64_t slots = static_cast<int64_t>(s.grid) * 2 * s.HP;
  int64_t at = kScratchOffset;
  s.zero_counters = s.groups * 4 > kCounterRegionBytes;
  if (s.zero_counters) {
    s.counters_offset = at;
    at += ((s.groups * 4 + 255) / 256) * 256;
  } else {
    s.counters_offset = kWorkspaceHeadBytes;
  }
  s.part_ml_offset = at;
  s.part_o_offset = s.part_ml_offset + ((slots * 8 + 255) / 256) * 256;
  s.workspace_end = s.part_o_offset + slots * s.D * 4;
  return s;
}

DecodeArgs make_decode_args(const gqa_problem& p, const DecodeShape& s, const void* q,
                            const uint8_t* mask, void* out, uint8_t* ws) {
  DecodeArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  for (int d = 0; d < 4; ++d) a.qs[d] = p.q_stride[d], a.os[d] = p.o_stride[d];
  a.mask = p.has_mask ? mask : nullptr;
  for (int d = 0; d < 3; ++d) a.ms[d] = p.mask_stride[d];
  a.out = static_cast<uint16_t*>(out);
  a.part_ml = reinterpret_cast<float2*>(ws + s.part_ml_offset);
  a.part_o = reinterpret_cast<float*>(ws + s.part_o_offset);
  a.counters = reinterpret_cast<uint32_t*>(ws + s.counters_offset);
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.lens = p.kv_lens;
  a.Dv = static_cast<int>(p.head_dim);
  a.bt = p.block_table;
  a.bt_stride = p.block_table_stride;
  a.page_size = static_cast<int>(p.page_size);
  a.num_pages = static_cast<int>(p.num_pages);
  a.B = static_cast<int>(p.batch);
  a.Hq = static_cast<int>(p.heads_q);
  a.Hkv = static_cast<int>(p.heads_kv);
  a.Sk = static_cast<int>(p.seq_k);
  a.g = static_cast<int>(p.heads_q / p.heads_kv);
  a.Sq = static_cast<int>(p.seq_q);
  a.rows = static_cast<int>(a.g * p.seq_q);
  a.causal = p.causal;
  a.causal_offset = p.causal_offset;
  a.window = p.window;
  a.scale_log2 = static_cast<float>(static_cast<double>(p.scale) * 1.4426950408889634073599);
  a.trace = decode_trace_slot(s.grid);
  decode_test_settings(&a.withhold_unit, &a.wait_ns);
  return a;
}

template <int D, int NT>
int launch_decode_dt(const DecodeShape& s, const DecodeArgs& a, const CUtensorMap& tmk,
                     const CUtensorMap& tmv, cudaStream_t stream, bool mq, bool f16) {
  if (f16)
    return mq ? launch_decode_t<D, NT, true, true>(s, a, tmk, tmv, stream)
              : launch_decode_t<D, NT, false, true>(s, a, tmk, tmv, stream);
  return mq ? launch_decode_t<D, NT, true, false>(s, a, tmk, tmv, stream)
            : launch_decode_t<D, NT, false, false>(s, a, tmk, tmv, stream);
}

int launch_decode(const gqa_problem& p, const DecodeShape& s, const DecodeArgs& a,
                  const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream) {
  const bool mq = a.Sq > 1;
  const bool f16 = p.dtype == GQA_DTYPE_F16;
  if (s.D == 128 && s.NT == 1) return launch_decode_dt<128, 1>(s, a, tmk, tmv, stream, mq, f16);
  if (s.D == 128 && s.NT == 2) return launch_decode_dt<128, 2>(s, a, tmk, tmv, stream, mq, f16);
  if (s.D == 64 && s.NT == 1) return launch_decode_dt<64, 1>(s, a, tmk, tmv, stream, mq, f16);
  if (s.D == 64 && s.NT == 2) return launch_decode_dt<64, 2>(s, a, tmk, tmv, stream, mq, f16);
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace gqa
