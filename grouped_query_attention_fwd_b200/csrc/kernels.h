// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gqa.h"

namespace gqa {

// ------------------------------------------------------------ decode
// Keys per streamed tile and consumer warps per CTA of the decode kernel.
constexpr int kDecodeKeysPerTile = 64;
constexpr int kDecodeConsumerWarps = 4;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;
constexpr int kDecodeMaxRowsPerPass = 16;  // (head, query) rows in the MMA N dimension

struct DecodeShape {
  int D;            // 64 or 128
  int NT;           // 8-head MMA column tiles per pass (1 or 2)
  int HP;           // rows per pass = 8 * NT (a row: one head, or one (head, query))
  int passes;       // ceil(g * seq_q / HP)
  int tiles_per_group;
  int t0;           // first 64-key tile any query can see (window)
  int64_t key_lo, key_hi;  // keys [key_lo, key_hi) pass the causal / window rules
  int64_t groups;   // batch * heads_kv * passes
  int64_t units;    // groups * tiles_per_group
  int grid;         // CTAs (<= units)
  int segmax;       // partial segments per CTA
  int stages;       // shared-memory ring depth
  int smem_bytes;
  int64_t counters_offset, part_o_offset, part_ml_offset, part_bytes;
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
  int B, Hq, Hkv, Sk, g;
  int Sq, rows;            // queries per kv head; rows = g * Sq
  int causal;
  int64_t causal_offset, window;
  int t0;                  // tile offset of the streamed key range
  int64_t key_lo, key_hi;  // keys outside [key_lo, key_hi) are hidden (causal / window)
  float scale_log2;  // scale * log2(e)
};

int launch_decode(const gqa_problem& p, const DecodeShape& s, const DecodeArgs& a,
                  const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream);

// TMA map of a K or V tensor with the decode kernel's box (api.cu).
int encode_decode_kv_map(CUtensorMap* map, const void* base, const gqa_problem& p,
                         const int64_t st[4]);

// ------------------------------------------------------------ prefill
constexpr int kPrefillThreads = 12 * 32;  // two softmax warpgroups, load, MMA and V-load warps

struct PrefillShape {
  int D;             // 64 or 128
  int qpt;           // query positions per 128-row tile (rows = qpt * g)
  int rows;          // qpt * g <= 128
  int m_tiles;       // ceil(Sq / qpt)
  int n_tiles;       // ceil(Sk / 128)
  int64_t work;      // batch * heads_kv * m_tiles
  int grid;
  int smem_bytes;
  int64_t summary_offset, summary_bytes;
};

PrefillShape plan_prefill(const gqa_problem& p, int sm_count);

struct PrefillArgs {
  const uint8_t* mask;
  int64_t ms[3];
  uint16_t* out;
  int64_t os[4];
  uint8_t* summary;  // [B][m_tiles][n_tiles]: 0 all hidden, 1 mixed, 2 all visible
  uint32_t* err;
  int B, Hq, Hkv, Sq, Sk, g;
  int causal, has_mask;
  int64_t causal_offset, window;
  float scale_log2;
};

int launch_prefill(const gqa_problem& p, const PrefillShape& s, const PrefillArgs& a,
                   const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmv,
                   cudaStream_t stream);

// ------------------------------------------------------------ fp32 path
int launch_f32(const gqa_problem& p, const float* q, const float* k, const float* v,
               const uint8_t* mask, float* out, cudaStream_t stream);

// ------------------------------------------------------------ fill: zeros (seq_k == 0) or NaN
int launch_zero(const gqa_problem& p, void* out, cudaStream_t stream, bool nan);

}  // namespace gqa
