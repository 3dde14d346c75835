// fp64 CPU oracle for the grouped-query attention forward.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
// load this file: it is used by tests/, by __graft_entry__.smoke() and by the
// benchmark's cpu_baseline / reference arm, and by nothing else.  It shares no
// code, header, table or helper with the CUDA library.
//
// What it computes is the plain definition, written out, single-threaded, in
// double precision, with a two-pass softmax (row max first, then exponentials
// and their sum) and no blocking, fusion or reordering:
//
//   g            = Hq / Hkv                        (Hq must be a multiple of Hkv)
//   kv(h)        = h / g                           (integer division)
//   s[b,h,i,j]   = scale * sum_d Q[b,h,i,d] * K[b,kv(h),j,d]
//   s[b,h,i,j]   = -inf  if a mask is given and mask[b,i,j] == 0
//   s[b,h,i,j]   = -inf  if causal and j > i
//   w[b,h,i,j]   = exp(s - max_j s) / sum_j exp(s - max_j s)
//   out[b,h,i,d] = sum_j w[b,h,i,j] * V[b,kv(h),j,d]
//
// Sources, by page and section:
//  * "28. Grouped-Query Attention (GQA)" (anandmoghan problems, page 28),
//    "Step-by-Step Approach" steps 1-4 and "Reference solution": the group size
//    read from the head counts, the contiguous repeat_interleave head map
//    (query head h uses kv head h // group), the scaled scores, the boolean
//    mask [B, Sq, Sk] broadcast over heads with false -> -inf, the row softmax
//    and the product with V.
//  * "Grouped-Query Attention Explained Simply" (lzwjava), "Minimal
//    implementation": the causal variant (is_causal=True, key j visible to
//    query i when j <= i).
//  * "Multi-Query Attention" (aiwiki), "Implementation": the same map and a
//    boolean attn_mask in the library attention call.
//
// Readings where the pages are silent or differ:
//  * the scale is an argument and multiplies the dot product (the reference
//    solution divides by sqrt(head_dim); callers pass 1/sqrt(D) for that);
//  * a mask value of 1 means "attend" (the reference solution fills where the
//    mask is false);
//  * mask and causal together: a key is visible only if both allow it;
//  * a row in which every key is hidden has max = -inf, so its weights and its
//    output are NaN, as in the reference solution's softmax of an all -inf row;
//  * causal is top-left aligned (j <= i) and, in the plain entry points, only
//    defined for Sq == Sk.  The "_ex" entry points take an explicit offset:
//    key j is visible to query i iff j <= i + causal_offset (bottom-right
//    alignment is causal_offset = Sk - Sq), and an optional sliding window of
//    `window` keys ending at that diagonal (Mistral's sliding-window attention,
//    named on "28. Grouped-Query Attention (GQA)", "Problem"): key j is also
//    hidden when j <= i + causal_offset - window.
//  * a ragged KV cache (the "_ex" entry points' kv_lens, one length per batch
//    entry, NULL = all seq_k): keys j >= kv_lens[b] are hidden, and the causal
//    diagonal of batch entry b moves with its length: causal_offset is given
//    for a full cache and becomes causal_offset + kv_lens[b] - seq_k.
//
// Layout: every array is contiguous, Q and out [B, Hq, Sq, D], K and V
// [B, Hkv, Sk, D], probs [B, Hq, Sq, Sk], mask [B, Sq, Sk] (uint8, nonzero =
// attend).  Return value: 0 on success, -1 on an invalid shape.

#include <cmath>
#include <cstdint>
#include <limits>
#include <vector>

namespace {

struct Problem {
  const double* q;
  const double* k;
  const double* v;
  const uint8_t* mask;  // may be null
  int64_t B, Hq, Hkv, Sq, Sk, D;
  int causal;
  double scale;
  int64_t causal_offset;  // key j visible to query i iff j <= i + causal_offset
  int64_t window;         // > 0: also hidden iff j <= i + causal_offset - window
  bool explicit_offset;   // false: the pages' causal, Sq == Sk required
  const int32_t* kv_lens = nullptr;  // per batch entry: keys j >= kv_lens[b] hidden
};

bool valid(const Problem& p) {
  if (p.B < 0 || p.Hq <= 0 || p.Hkv <= 0 || p.Sq < 0 || p.Sk < 0 || p.D <= 0) return false;
  if (p.Hq % p.Hkv != 0) return false;
  if (p.causal && !p.explicit_offset && p.Sq != p.Sk) return false;
  if (p.window < 0 || (p.window > 0 && !p.causal)) return false;
  return true;
}

// Softmax weights of one (b, h, i) row into w[0..Sk).
void row_weights(const Problem& p, int64_t b, int64_t h, int64_t i, double* w) {
  const int64_t g = p.Hq / p.Hkv;
  const int64_t kv = h / g;
  const double* qrow = p.q + ((b * p.Hq + h) * p.Sq + i) * p.D;
  const double* kbase = p.k + ((b * p.Hkv + kv) * p.Sk) * p.D;
  const double neg_inf = -std::numeric_limits<double>::infinity();
  const int64_t len = p.kv_lens ? p.kv_lens[b] : p.Sk;
  const int64_t off = p.causal_offset + (len - p.Sk);

  // Pass 1: scores and their maximum.
  double m = neg_inf;
  for (int64_t j = 0; j < p.Sk; ++j) {
    double dot = 0.0;
    const double* krow = kbase + j * p.D;
    for (int64_t d = 0; d < p.D; ++d) dot += qrow[d] * krow[d];
    double s = p.scale * dot;
    if (p.mask != nullptr && p.mask[(b * p.Sq + i) * p.Sk + j] == 0) s = neg_inf;
    if (j >= len) s = neg_inf;
    if (p.causal && j > i + off) s = neg_inf;
    if (p.window > 0 && j <= i + off - p.window) s = neg_inf;
    w[j] = s;
    if (s > m) m = s;
  }
  // Pass 2: exponentials and their sum; then normalise.  With m = -inf every
  // s - m is NaN, which is the defined result for a fully hidden row.
  double l = 0.0;
  for (int64_t j = 0; j < p.Sk; ++j) {
    w[j] = std::exp(w[j] - m);
    l += w[j];
  }
  for (int64_t j = 0; j < p.Sk; ++j) w[j] = w[j] / l;
}

void row_output(const Problem& p, int64_t b, int64_t h, int64_t i, const double* w, double* out) {
  const int64_t g = p.Hq / p.Hkv;
  const int64_t kv = h / g;
  const double* vbase = p.v + ((b * p.Hkv + kv) * p.Sk) * p.D;
  for (int64_t d = 0; d < p.D; ++d) out[d] = 0.0;
  for (int64_t j = 0; j < p.Sk; ++j) {
    const double* vrow = vbase + j * p.D;
    for (int64_t d = 0; d < p.D; ++d) out[d] += w[j] * vrow[d];
  }
}

}  // namespace

extern "C" {

// Attention weights [B, Hq, Sq, Sk].
int oracle_gqa_probs(const double* q, const double* k, const uint8_t* mask, int64_t B,
                     int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Sk, int64_t D, int causal,
                     double scale, double* probs) {
  Problem p{q, k, nullptr, mask, B, Hq, Hkv, Sq, Sk, D, causal, scale, 0, 0, false};
  if (!valid(p)) return -1;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < Hq; ++h)
      for (int64_t i = 0; i < Sq; ++i)
        row_weights(p, b, h, i, probs + ((b * Hq + h) * Sq + i) * Sk);
  return 0;
}

// Full output [B, Hq, Sq, D].
int oracle_gqa_forward(const double* q, const double* k, const double* v, const uint8_t* mask,
                       int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Sk, int64_t D,
                       int causal, double scale, double* out) {
  Problem p{q, k, v, mask, B, Hq, Hkv, Sq, Sk, D, causal, scale, 0, 0, false};
  if (!valid(p)) return -1;
  std::vector<double> w(static_cast<size_t>(Sk > 0 ? Sk : 1));
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < Hq; ++h)
      for (int64_t i = 0; i < Sq; ++i) {
        row_weights(p, b, h, i, w.data());
        row_output(p, b, h, i, w.data(), out + ((b * Hq + h) * Sq + i) * D);
      }
  return 0;
}

// Selected rows only: rows[3*r .. 3*r+2] = (b, h, i); out is [n, D].
int oracle_gqa_forward_rows(const double* q, const double* k, const double* v,
                            const uint8_t* mask, int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq,
                            int64_t Sk, int64_t D, int causal, double scale, const int64_t* rows,
                            int64_t n, double* out) {
  Problem p{q, k, v, mask, B, Hq, Hkv, Sq, Sk, D, causal, scale, 0, 0, false};
  if (!valid(p)) return -1;
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= Sq) return -1;
  }
  std::vector<double> w(static_cast<size_t>(Sk > 0 ? Sk : 1));
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    row_weights(p, b, h, i, w.data());
    row_output(p, b, h, i, w.data(), out + r * D);
  }
  return 0;
}

// Selected rows with an explicit causal offset and sliding window (see the
// header); rows[3*r .. 3*r+2] = (b, h, i); out is [n, D].
int oracle_gqa_forward_rows_ex(const double* q, const double* k, const double* v,
                               const uint8_t* mask, const int32_t* kv_lens, int64_t B, int64_t Hq,
                               int64_t Hkv, int64_t Sq, int64_t Sk, int64_t D, int causal,
                               int64_t causal_offset, int64_t window, double scale,
                               const int64_t* rows, int64_t n, double* out) {
  Problem p{q, k, v, mask, B, Hq, Hkv, Sq, Sk, D, causal, scale, causal_offset, window, true,
            kv_lens};
  if (!valid(p)) return -1;
  for (int64_t b = 0; kv_lens != nullptr && b < B; ++b)
    if (kv_lens[b] < 0 || kv_lens[b] > Sk) return -1;
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= Sq) return -1;
  }
  std::vector<double> w(static_cast<size_t>(Sk > 0 ? Sk : 1));
  for (int64_t r = 0; r < n; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    row_weights(p, b, h, i, w.data());
    row_output(p, b, h, i, w.data(), out + r * D);
  }
  return 0;
}

// Full output with an explicit causal offset and sliding window.
int oracle_gqa_forward_ex(const double* q, const double* k, const double* v, const uint8_t* mask,
                          const int32_t* kv_lens, int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq,
                          int64_t Sk, int64_t D, int causal, int64_t causal_offset,
                          int64_t window, double scale, double* out) {
  Problem p{q, k, v, mask, B, Hq, Hkv, Sq, Sk, D, causal, scale, causal_offset, window, true,
            kv_lens};
  if (!valid(p)) return -1;
  for (int64_t b = 0; kv_lens != nullptr && b < B; ++b)
    if (kv_lens[b] < 0 || kv_lens[b] > Sk) return -1;
  std::vector<double> w(static_cast<size_t>(Sk > 0 ? Sk : 1));
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < Hq; ++h)
      for (int64_t i = 0; i < Sq; ++i) {
        row_weights(p, b, h, i, w.data());
        row_output(p, b, h, i, w.data(), out + ((b * Hq + h) * Sq + i) * D);
      }
  return 0;
}

// KV-cache size in bytes, "Multi-Query Attention" (aiwiki), "Theory":
// bytes_KV = 2 * L * n * h_kv * d_head * b * sizeof(dtype)
// (L layers, n tokens of context, h_kv kv heads, d_head, b sequences).
int64_t oracle_kv_cache_bytes(int64_t layers, int64_t tokens, int64_t h_kv, int64_t d_head,
                              int64_t batch, int64_t elem_bytes) {
  return 2 * layers * tokens * h_kv * d_head * batch * elem_bytes;
}

}  // extern "C"
