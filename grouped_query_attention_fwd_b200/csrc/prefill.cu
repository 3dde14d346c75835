// Prefill kernel (seq_q >= 2): placeholder until the tcgen05 kernel lands.
#include <cuda_runtime.h>

#include "kernels.h"

namespace gqa {

PrefillShape plan_prefill(const gqa_problem& p, int sm_count) {
  PrefillShape s{};
  const int64_t g = p.heads_q / p.heads_kv;
  s.D = static_cast<int>(p.head_dim);
  s.qpt = static_cast<int>(128 / g);
  s.rows = static_cast<int>(s.qpt * g);
  s.m_tiles = static_cast<int>((p.seq_q + s.qpt - 1) / s.qpt);
  s.n_tiles = static_cast<int>((p.seq_k + 127) / 128);
  s.work = p.batch * p.heads_kv * s.m_tiles;
  s.grid = static_cast<int>(s.work < sm_count ? s.work : sm_count);
  s.summary_offset = 256;
  s.summary_bytes = p.has_mask ? p.batch * s.m_tiles * s.n_tiles : 0;
  return s;
}

int launch_prefill(const gqa_problem&, const PrefillShape&, const PrefillArgs&,
                   const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, cudaStream_t) {
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace gqa
