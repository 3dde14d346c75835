// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gqa.h"

namespace gqa {

// ------------------------------------------------------------ decode
// Keys per streamed tile and consumer warps per CTA of the decode kernel.
constexpr int kDecodeKeysPerTile = 128;
constexpr int kDecodeConsumerWarps = 8;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;
constexpr int kDecodeMaxRowsPerPass = 16;  // (head, query) rows in the MMA N dimension
constexpr int kDecodeMaxSmem = 227 * 1024;  // dynamic shared memory one CTA may take
constexpr int kDecodePageBox = 64;          // keys per TMA box of a paged cache
constexpr int64_t kMaxRaggedBatch = 16384;  // batch entries with per-sequence lengths

// Workspace layout shared by every call: bytes [0, 256) hold the error word
// (and the append ticket), [256, 256 + kCounterRegionBytes) the decode ticket
// counters, which each group's last contributor resets, so the region stays
// zero between calls; other scratch (decode partials, prefill tile classes)
// starts after it and never touches it.
constexpr int64_t kWorkspaceHeadBytes = 256;
constexpr int64_t kCounterRegionBytes = 64 * 1024;
constexpr int64_t kScratchOffset = kWorkspaceHeadBytes + kCounterRegionBytes;

// Keys [lo, hi) of one batch entry that some query of the block can see,
// and the decode key tiles [t0, t0 + tiles) that hold them.  `len` is the entry's
// cache length (seq_k without per-sequence lengths); the causal diagonal
// moves with it by len - seq_k.  A range with no visible key still gets one
// tile, streamed fully hidden, so that its rows come out NaN.
struct KeyRange {
  int lo, hi;
  int t0, tiles;
};

__host__ __device__ inline KeyRange decode_key_range(int64_t len, int64_t Sk, int64_t Sq,
                                                     int causal, int64_t off, int64_t window) {
  const int64_t shift = len - Sk;
  int64_t lo = 0, hi = len;
  if (causal) {
    if (Sq + off + shift < hi) hi = Sq + off + shift;  // last query: j <= Sq - 1 + off + shift
    if (window > 0 && off + shift - window + 1 > 0) lo = off + shift - window + 1;  // query 0
  }
  KeyRange r;
  if (hi <= lo) {
    r.lo = r.hi = 0;
    r.t0 = 0;
    r.tiles = 1;
  } else {  // 0 <= lo < hi <= len <= Sk < 2^31
    r.lo = static_cast<int>(lo);
    r.hi = static_cast<int>(hi);
    r.t0 = r.lo / kDecodeKeysPerTile;
    r.tiles = (r.hi + kDecodeKeysPerTile - 1) / kDecodeKeysPerTile - r.t0;
  }
  return r;
}

struct DecodeShape {
  int D;            // 64 or 128: head_dim rounded up (the kernel's width)
  int NT;           // 8-head MMA column tiles per pass (1 or 2)
  int HP;           // rows per pass = 8 * NT (a row: one head, or one (head, query))
  int passes;       // ceil(g * seq_q / HP)
  int tiles_per_group;  // without kv_lens; with them, the most any group can need
  int64_t groups;   // batch * heads_kv * passes
  int64_t units;    // groups * tiles_per_group (an upper bound with kv_lens)
  int grid;         // CTAs (<= units)
  int stages;       // shared-memory ring depth
  int smem_bytes;
  bool ragged;      // per-sequence kv_lens: the partition is computed on the device
  bool zero_counters;  // more groups than the counter region holds: zero them per call
  int64_t counters_offset, part_o_offset, part_ml_offset;
  int64_t workspace_end;  // bytes of workspace the launch uses
};

DecodeShape plan_decode(const gqa_problem& p, int sm_count);

struct DecodeArgs {
  const uint16_t* q;
  int64_t qs[4];
  const uint8_t* mask;
  int64_t ms[3];
  uint16_t* out;
  int64_t os[4];
  float* part_o;
  float2* part_ml;
  uint32_t* counters;  // one ticket counter per group; zeroed before each launch
  uint32_t* err;
  const int32_t* lens;  // per-sequence cache lengths, or nullptr (all seq_k)
  int Dv;                  // head_dim (<= the kernel's D; a multiple of 8)
  const int32_t* bt;       // paged cache: block table, or nullptr (contiguous k / v)
  int64_t bt_stride;
  int page_size, num_pages;
  int B, Hq, Hkv, Sk, g;
  int Sq, rows;            // queries per kv head; rows = g * Sq
  int causal;
  int64_t causal_offset, window;
  float scale_log2;  // scale * log2(e)
  uint64_t* trace;   // per-CTA phase timestamps (kDecodeTraceWords each), or nullptr
  uint64_t wait_ns;  // limit of every wait of the launch (1 s unless a test shortens it)
  int withhold_unit; // test only (gqa_debug_decode_withhold): the producer never issues
                     // this unit's copies and stops there; -1 = none
};

// One-shot settings of the next decode launch made by gqa_debug_decode_withhold
// (api.cu): the unit to withhold (-1: none) and the wait limit.
void decode_test_settings(int* withhold_unit, uint64_t* wait_ns);

// Diagnostic trace of the decode kernel: one record of kDecodeTraceWords
// 64-bit words per CTA and launch (gqa_debug_decode_trace).
constexpr int kDecodeTraceWords = 16;
enum DecodeTraceWord : int {
  kTrSm = 0,           // SM id (low 32 bits), CTA index (high 32 bits)
  kTrEntry = 1,        // %globaltimer at kernel entry
  kTrReady = 2,        // set-up done, earlier grids complete (after the dependent-launch wait)
  kTrFirstIssue = 3,   // producer: first K tile copy issued
  kTrLastIssue = 4,    // producer: last V tile copy issued
  kTrFirstLand = 5,    // consumer warp 0: first K tile landed
  kTrLastTile = 6,     // consumer warp 0: last tile consumed
  kTrFinalMerged = 7,  // final group merged across the eight warps
  kTrFinalDone = 8,    // final group written (out, or a partial and its ticket)
  kTrExit = 9,         // after the closing barrier
  kTrUnits = 10,       // tiles in this CTA's range
  kTrFlushes = 11,     // groups flushed
  kTrMidFlushNs = 12,  // consumer warp 0: time spent in flushes before the final one
  kTrFinalKind = 13,   // final group: 0 whole, 1 split (published), 2 split (merged here directly)
};
// Device buffer and slot count set by gqa_debug_decode_trace (api.cu), or
// nullptr; each decode launch takes the next slot.
uint64_t* decode_trace_slot(int grid);

// Arguments of one decode launch; the workspace `ws` holds the error word at
// offset 0 and the plan's counters and partials.
DecodeArgs make_decode_args(const gqa_problem& p, const DecodeShape& s, const void* q,
                            const uint8_t* mask, void* out, uint8_t* ws);

int launch_decode(const gqa_problem& p, const DecodeShape& s, const DecodeArgs& a,
                  const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream);

// TMA map of a K or V tensor with the decode kernel's box (api.cu).
int encode_decode_kv_map(CUtensorMap* map, const void* base, const gqa_problem& p,
                         const int64_t st[4]);

// ------------------------------------------------------------ prefill
constexpr int kPrefillThreads = 12 * 32;  // two softmax warpgroups, load, MMA and V-load warps

// Key tiles a work item of the two-tile prefill kernel may span (Sk <= 131072).
constexpr int kMaxPPTiles = 1024;
// Largest items x key tiles for which the two-tile kernel's item order is
// sorted on the device (one CTA classifies every item's key tiles).
constexpr int64_t kMaxOrderWork = int64_t(1) << 21;

struct PrefillShape {
  bool pp;           // two query tiles per SM (prefill_pp.cu); else one (prefill.cu)
  int D;             // 64 or 128
  int qpt;           // query positions per 128-row tile (rows = qpt * g)
  int rows;          // qpt * g <= 128
  int m_tiles;       // ceil(Sq / qpt)
  int n_tiles;       // ceil(Sk / 128)
  int64_t work;      // batch * heads_kv * m_tiles
  int grid;
  int smem_bytes;
  int64_t summary_offset, workspace_end;
  // Two-tile kernel with a mask: the order in which the items are taken
  // (heaviest first, from the mask summary), int32 per item, or -1 (none).
  int64_t order_offset;
  int64_t bounds_offset;  // with a mask: the summary's per-query-tile key-tile bounds
};

PrefillShape plan_prefill(const gqa_problem& p, int sm_count);

struct PrefillArgs {
  const uint8_t* mask;
  int64_t ms[3];
  uint16_t* out;
  int64_t os[4];
  uint8_t* summary;  // [B][m_tiles][n_tiles]: 0 all hidden, 1 mixed, 2 all visible
  int32_t* order;    // item taken at position x of the schedule, or nullptr (x itself)
  int32_t* bounds;   // with a mask: [B][m_tiles][2] first and past-last key tile not hidden
  uint32_t* err;
  const int32_t* lens;  // per-sequence cache lengths, or nullptr (all seq_k)
  int Dv;               // head_dim (<= the kernel's D; a multiple of 8)
  int B, Hq, Hkv, Sq, Sk, g;
  int causal, has_mask;
  int64_t causal_offset, window;
  float scale_log2;
};

// Mask pre-pass shared by both prefill kernels: per (batch, query tile, key
// tile) 0 all hidden, 1 mixed, 2 all visible.
int launch_mask_summary(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream);

// Two query tiles per SM: K and V with 128-key boxes, as for the one-tile kernel.
int pp_smem_bytes(int D);
int launch_prefill_pp(const gqa_problem& p, const PrefillShape& s, const PrefillArgs& a,
                      const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                      cudaStream_t stream);

int launch_prefill(const gqa_problem& p, const PrefillShape& s, const PrefillArgs& a,
                   const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                   cudaStream_t stream);

// ------------------------------------------------------------ fp32 path
int launch_f32(const gqa_problem& p, const float* q, const float* k, const float* v,
               const uint8_t* mask, float* out, uint32_t* err, cudaStream_t stream);

// ------------------------------------------------------------ KV-cache append
struct AppendArgs {
  uint8_t* ck;          // cache_k, cache_v (bytes)
  uint8_t* cv;
  const uint8_t* kn;    // k_new, v_new (bytes)
  const uint8_t* vn;
  int32_t* lens;        // read, then advanced by n_new by the last CTA
  uint32_t* err;
  uint32_t* ticket;     // CTAs done; zero between launches
  int64_t cks[3], cvs[3], kns[3], vns[3];  // byte strides over (b, h, row)
  int B, H;
  int64_t cap, n_new;
  int row_bytes;        // head_dim * element bytes
  int vec;              // bytes per copied vector: 16, 4 or 2
  const int32_t* bt;    // paged cache: block table, or nullptr
  int64_t bt_stride, page_size, num_pages;
};

int launch_kv_append(const AppendArgs& a, cudaStream_t stream);

// ------------------------------------------------------------ fill: zeros (seq_k == 0) or NaN
int launch_zero(const gqa_problem& p, void* out, cudaStream_t stream, bool nan);

}  // namespace gqa
