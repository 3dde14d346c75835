// Split-K decode kernel (seq_q == 1) with its split merge fused in.
//
// Decoding re-reads the whole KV cache once per generated token and does
// about one multiply-add per byte it reads, so its time is the KV bytes over
// HBM bandwidth ("Multi-Query Attention", "Theory"; "Grouped-Query Attention
// Explained Simply", "Why it matters").  The kernel is built around that
// bound:
//
//  * Work unit = one 64-key tile of one (batch, kv head, head pass).  All units
//    of the problem are laid end to end and cut into one contiguous range per
//    CTA (a persistent grid of one CTA per SM), so every SM streams the same
//    number of bytes whatever B * Hkv is; a range may start or end inside a
//    kv head's key sequence (split-K), which leaves a partial softmax state.
//  * A producer warp streams K and V tiles with TMA (128-byte swizzled boxes,
//    so the ldmatrix reads below are bank-conflict free) into a ring of
//    shared-memory stages guarded by mbarriers; each tile crosses HBM once.
//  * Four consumer warps take 16 keys each of every staged tile and serve all
//    g query heads of the group from it: the kv head is never expanded
//    ("Multi-Query Attention": a zero stride over the head dimension).  The
//    dot products run on the tensor cores as S^T = K Q^T with keys in the MMA
//    M dimension and the group's heads in N (g <= 8 fills one 8-wide column
//    tile), then O^T += V^T P^T; at g = 8 a CUDA-core version would need about
//    as many FMA issue slots as the HBM time allows, the MMA needs a few %.
//  * Online softmax in fp32 with warp-shuffle max/sum reductions; at the end
//    of a range the four warps merge in shared memory.  A group handled by
//    one CTA is normalised and written straight to `out`.  A group split over
//    several CTAs leaves one partial (m, l, O) per head and CTA in the
//    workspace; each contributor then takes a ticket from the group's counter
//    and the last one merges all partials and writes bf16 `out` (the counters
//    are zeroed on the stream before the launch).  No CTA ever waits for
//    another one.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int KT = kDecodeKeysPerTile;  // keys per tile
constexpr int NCW = kDecodeConsumerWarps;
constexpr int CHUNK_BYTES = KT * 128;   // one 64-wide bf16 column chunk of a tile
constexpr int kFastMerge = 4;           // split groups merged with all loads in flight

__host__ __device__ inline int64_t range_start(int64_t c, int64_t T, int64_t P) {
  return (c * T) / P;
}

// The CTA whose range [range_start(c), range_start(c + 1)) holds unit u:
// the largest c with floor(c T / P) <= u, i.e. ceil((u + 1) P / T) - 1.
__host__ __device__ inline int64_t cta_of_unit(int64_t u, int64_t T, int64_t P) {
  return ((u + 1) * P + T - 1) / T - 1;
}

template <int D, int NT>
struct DecodeSmem {
  static constexpr int kTileBytes = KT * D * 2;        // K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;   // K + V
  static constexpr int HP = 8 * NT;
  static constexpr int kScrRow = D + 4;                // padded head row (floats)
  static constexpr int kScrOBytes = NCW * HP * kScrRow * 4;
  static constexpr int kScrMLBytes = NCW * HP * 2 * 4;
  static int bytes(int stages) {
    return 1024 /*alignment slack*/ + stages * kStageBytes + kScrOBytes + kScrMLBytes +
           2 * stages * 8 + 16;
  }
};

// MQ: several query positions per kv head (seq_q > 1): the rows of a pass
// are (head, query) pairs, row r = head * seq_q + query, each with its own
// visible key range and mask row.
template <int D, int NT, bool MQ>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const DecodeArgs a,
                      const int tiles_per_group, const int passes, const int64_t units,
                      const int segmax, const int stages, uint32_t* __restrict__ counters) {
  using L = DecodeSmem<D, NT>;
  constexpr int HP = L::HP;
  constexpr int KSTEPS = D / 16;
  constexpr int CHUNKS = D / 64;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  float* scr_o = reinterpret_cast<float*>(ring + stages * L::kStageBytes);
  float* scr_ml = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(scr_o) + L::kScrOBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(scr_ml) +
                                               L::kScrMLBytes);
  uint64_t* empty = full + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);
  volatile int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t u_begin = range_start(blockIdx.x, units, P);
  const int64_t u_end = range_start(blockIdx.x + 1, units, P);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
      int64_t it = 0;
      for (int64_t u = u_begin; u < u_end; ++u, ++it) {
        const int s = static_cast<int>(it % stages);
        const uint32_t round = static_cast<uint32_t>(it / stages);
        if (round > 0 &&
            !mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, a.err, kErrDecodeWait))
          break;
        const int64_t grp = u / tiles_per_group;
        const int t = static_cast<int>(u % tiles_per_group);
        const int64_t bk = grp / passes;  // b * Hkv + kv
        const int kv = static_cast<int>(bk % a.Hkv);
        const int b = static_cast<int>(bk / a.Hkv);
        uint8_t* st = ring + s * L::kStageBytes;
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          tma_load_4d(st + c * CHUNK_BYTES, &tmk, &full[s], c * 64, (t + a.t0) * KT, kv, b);
          tma_load_4d(st + L::kTileBytes + c * CHUNK_BYTES, &tmv, &full[s], c * 64,
                      (t + a.t0) * KT, kv, b);
        }
      }
      // Unwind: make sure no copy is still landing in this CTA's shared memory.
      if (*abort_flag) {
        const int64_t issued = it;
        for (int64_t j = (issued > stages ? issued - stages : 0); j < issued; ++j)
          mbar_wait_drain(&full[j % stages], static_cast<uint32_t>((j / stages) & 1));
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    uint32_t bq[NT][KSTEPS][2];
    float o[NT][KSTEPS][4];
    float m_run[NT][2], l_run[NT][2];
    int64_t cur = -1;
    int seg = 0;
    int b = 0, kv = 0, pass = 0;
    const uint8_t* mrow = nullptr;

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
    int64_t vlo[NT][2], vhi[NT][2];
    const uint8_t* vmask[NT][2];

    auto load_q = [&]() {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hl = pass * HP + nt * 8 + (lane >> 2);  // row within the group
        const bool ok = hl < a.rows;
        const int hh = MQ ? (ok ? hl / a.Sq : 0) : (ok ? hl : 0);
        const int qi = MQ ? (ok ? hl % a.Sq : 0) : 0;
        const uint16_t* qrow = a.q + b * a.qs[0] + (int64_t)(kv * a.g + hh) * a.qs[1] +
                               (int64_t)qi * a.qs[2];
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int d0 = ks * 16 + (lane & 3) * 2;
          bq[nt][ks][0] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
          bq[nt][ks][1] = ok ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 8) : 0u;
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (MQ) {
            const int r = pass * HP + nt * 8 + (lane & 3) * 2 + e;
            const int i = (r < a.rows ? r : 0) % a.Sq;
            int64_t lo = 0, hi = a.Sk;
            if (a.causal) {
              hi = i + a.causal_offset + 1 < hi ? i + a.causal_offset + 1 : hi;
              if (a.window > 0 && i + a.causal_offset - a.window + 1 > 0)
                lo = i + a.causal_offset - a.window + 1;
            }
            vlo[nt][e] = lo;
            vhi[nt][e] = hi;
            vmask[nt][e] = a.mask ? a.mask + b * a.ms[0] + static_cast<int64_t>(i) * a.ms[1] : nullptr;
          } else {
            vlo[nt][e] = a.key_lo;
            vhi[nt][e] = a.key_hi;
            vmask[nt][e] = mrow;
          }
        }
      }
    };

    // Merge the four warps' states of the finished range and write one partial.
    auto flush = [&]() {
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
      float* my_o = scr_o + warp * HP * L::kScrRow;
      float* my_ml = scr_ml + warp * HP * 2;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int h = nt * 8 + (lane & 3) * 2 + (c & 1);
            const int d = mt * 16 + (lane >> 2) + ((c & 2) ? 8 : 0);
            my_o[h * L::kScrRow + d] = o[nt][mt][c];
          }
        if (lane < 4) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = nt * 8 + lane * 2 + e;
            my_ml[h * 2 + 0] = m_run[nt][e];
            my_ml[h * 2 + 1] = l_run[nt][e];
          }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      // Which CTAs share this group?  Ranges are static, so every CTA can tell.
      const int64_t g_u0 = cur * tiles_per_group, g_u1 = g_u0 + tiles_per_group;
      const int64_t c_lo = cta_of_unit(g_u0, units, P);
      const int64_t c_hi = cta_of_unit(g_u1 - 1, units, P);
      // Output row of row hr of this pass (a head, or a (head, query) pair).
      auto out_row = [&](int hr) -> uint16_t* {
        const int r = pass * HP + hr;
        const int hh = MQ ? r / a.Sq : r;
        const int qi = MQ ? r % a.Sq : 0;
        return a.out + b * a.os[0] + static_cast<int64_t>(kv * a.g + hh) * a.os[1] +
               static_cast<int64_t>(qi) * a.os[2];
      };
      if (c_lo == c_hi) {
        // The whole group is in this CTA: normalise and write out.
        for (int idx = threadIdx.x; idx < HP * D; idx += NCW * 32) {
          const int h = idx / D, d = idx % D;
          if (pass * HP + h >= a.rows) continue;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < NCW; ++w) M = fmaxf(M, scr_ml[(w * HP + h) * 2]);
          float l = 0.f, acc = 0.f;
          if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NCW; ++w) {
              const float sc = fast_exp2(scr_ml[(w * HP + h) * 2] - M);
              l += sc * scr_ml[(w * HP + h) * 2 + 1];
              acc += sc * scr_o[(w * HP + h) * L::kScrRow + d];
            }
          }
          out_row(h)[d] = bf16_bits_rn(acc / l);  // l == 0: NaN
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
        return;
      }
      // Split group: publish this CTA's partial (float4 stores), then take a
      // ticket: the CTA barrier orders every thread's stores before thread
      // 0's gpu-scope fence and atomic (release), and thread 0's fence after
      // the atomic orders the reads of the others' partials (acquire).
      const int64_t slot = (static_cast<int64_t>(blockIdx.x) * segmax + seg) * HP;
      for (int idx = threadIdx.x; idx < HP * D / 4; idx += NCW * 32) {
        const int h = idx / (D / 4), d = (idx % (D / 4)) * 4;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, scr_ml[(w * HP + h) * 2]);
        float l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < NCW; ++w) {
            const float sc = fast_exp2(scr_ml[(w * HP + h) * 2] - M);
            l += sc * scr_ml[(w * HP + h) * 2 + 1];
            const float* src = scr_o + (w * HP + h) * L::kScrRow + d;
            acc.x += sc * src[0];
            acc.y += sc * src[1];
            acc.z += sc * src[2];
            acc.w += sc * src[3];
          }
        }
        *reinterpret_cast<float4*>(&a.part_o[(slot + h) * D + d]) = acc;
        if (d == 0) a.part_ml[slot + h] = make_float2(M, l);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      if (threadIdx.x == 0) {
        const uint32_t n = static_cast<uint32_t>(c_hi - c_lo + 1);
        __threadfence();
        const uint32_t old = atomicAdd(&counters[cur], 1u);
        __threadfence();
        *last_flag = (old == n - 1) ? 1 : 0;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
      if (*last_flag) {
        // Last contributor: every other partial of the group is published.
        const int n = static_cast<int>(c_hi - c_lo + 1);
        if (n <= kFastMerge) {
          // Few contributors: every load of a thread's elements in flight at once.
          int64_t base[kFastMerge];
#pragma unroll
          for (int k = 0; k < kFastMerge; ++k) {
            const int64_t cc = c_lo + (k < n ? k : 0);
            base[k] = (cc * segmax + (cur - range_start(cc, units, P) / tiles_per_group)) * HP;
          }
          for (int idx = threadIdx.x; idx < HP * D / 4; idx += NCW * 32) {
            const int h = idx / (D / 4), d = (idx % (D / 4)) * 4;
            if (pass * HP + h >= a.rows) continue;
            float2 ml[kFastMerge];
            float4 o[kFastMerge];
#pragma unroll
            for (int k = 0; k < kFastMerge; ++k) {
              if (k < n) {
                ml[k] = __ldcg(&a.part_ml[base[k] + h]);
                o[k] = __ldcg(reinterpret_cast<const float4*>(&a.part_o[(base[k] + h) * D + d]));
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
                  acc.x += w * o[k].x;
                  acc.y += w * o[k].y;
                  acc.z += w * o[k].z;
                  acc.w += w * o[k].w;
                }
              }
            }
            const float inv = 1.f / Lsum;  // Lsum == 0: NaN
            uint2 pk;
            pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
            pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2*>(out_row(h) + d) = pk;
          }
        } else {
        // Many contributors: stage each one's segment index and each head's
        // merged (max, sum) in shared memory, then accumulate O with 16-byte
        // loads, several contributors in flight at once.
        int* sm_seg = reinterpret_cast<int*>(scr_o);          // n ints (scr_o is free now)
        float* sm_ml = scr_ml;                                 // HP x (M, L)
        for (int k = threadIdx.x; k < n; k += NCW * 32)
          sm_seg[k] = static_cast<int>(cur - range_start(c_lo + k, units, P) / tiles_per_group);
        asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
        if (threadIdx.x < HP) {
          const int h = threadIdx.x;
          float M = -INFINITY;
#pragma unroll 4
          for (int k = 0; k < n; ++k)
            M = fmaxf(M, __ldcg(&a.part_ml[((c_lo + k) * segmax + sm_seg[k]) * HP + h]).x);
          float Lsum = 0.f;
          if (M != -INFINITY) {
#pragma unroll 4
            for (int k = 0; k < n; ++k) {
              const float2 ml = __ldcg(&a.part_ml[((c_lo + k) * segmax + sm_seg[k]) * HP + h]);
              Lsum += fast_exp2(ml.x - M) * ml.y;
            }
          }
          sm_ml[2 * h] = M;
          sm_ml[2 * h + 1] = Lsum;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
        for (int idx = threadIdx.x; idx < HP * D / 4; idx += NCW * 32) {
          const int h = idx / (D / 4), d = (idx % (D / 4)) * 4;
          if (pass * HP + h >= a.rows) continue;
          const float M = sm_ml[2 * h], Lsum = sm_ml[2 * h + 1];
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          if (M != -INFINITY) {
#pragma unroll 4
            for (int k = 0; k < n; ++k) {
              const int64_t sl = ((c_lo + k) * segmax + sm_seg[k]) * HP + h;
              const float w = fast_exp2(__ldcg(&a.part_ml[sl]).x - M);
              const float4 o = __ldcg(reinterpret_cast<const float4*>(&a.part_o[sl * D + d]));
              acc.x += w * o.x;
              acc.y += w * o.y;
              acc.z += w * o.z;
              acc.w += w * o.w;
            }
          }
          const float inv = 1.f / Lsum;  // Lsum == 0: NaN
          uint2 pk;
          pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
          pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
          *reinterpret_cast<uint2*>(out_row(h) + d) = pk;
        }
        }
        if (threadIdx.x == 0) atomicExch(&counters[cur], 0u);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
    };

    int64_t it = 0;
    bool ok = true;
    for (int64_t u = u_begin; u < u_end; ++u, ++it) {
      const int64_t grp = u / tiles_per_group;
      const int t = static_cast<int>(u % tiles_per_group);
      if (grp != cur) {
        if (cur >= 0) {
          flush();
          ++seg;
        }
        cur = grp;
        const int64_t bk = grp / passes;
        pass = static_cast<int>(grp % passes);
        kv = static_cast<int>(bk % a.Hkv);
        b = static_cast<int>(bk / a.Hkv);
        mrow = a.mask ? a.mask + b * a.ms[0] : nullptr;
        load_q();
        reset_state();
      }
      const int s = static_cast<int>(it % stages);
      const uint32_t round = static_cast<uint32_t>(it / stages);
      if (!mbar_wait(&full[s], round & 1u, abort_flag, a.err, kErrDecodeWait)) {
        ok = false;
        break;
      }
      const uint32_t kbase = smem_u32(ring + s * L::kStageBytes);
      const uint32_t vbase = kbase + L::kTileBytes;

      // S^T[16 keys x 8 heads] = K[16 x D] Q^T[D x 8] per column tile.
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[nt][c] = 0.f;
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
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_bf16_16816(sc[nt], a0, a1, a2, a3, bq[nt][ks][0], bq[nt][ks][1]);
        }
      }

      // Visibility of this thread's two keys for its rows.
      const int64_t key0 = static_cast<int64_t>(t + a.t0) * KT + warp * 16 + (lane >> 2);
      const int64_t key1 = key0 + 8;
      auto vis = [&](int64_t key, int nt, int e) -> bool {
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
        pt0[nt] = movmatrix_trans(pack_bf16x2(tv[0], tv[1]));
        pt1[nt] = movmatrix_trans(pack_bf16x2(tv[2], tv[3]));
      }

      // O^T[D x 8] += V^T[D x 16 keys] P^T[16 keys x 8].
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
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_bf16_16816(o[nt][mt], a0, a1, a2, a3, pt0[nt], pt1[nt]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ok && cur >= 0) flush();
    if (!ok) {
      // Keep the named barrier count consistent for warps still in flush():
      // nothing else to do, the error word is already set.
    }
  }
  __syncthreads();
}

template <int D, int NT, bool MQ>
int launch_decode_t(const DecodeShape& s, const DecodeArgs& a, const CUtensorMap& tmk,
                    const CUtensorMap& tmv, cudaStream_t stream) {
  auto kern = gqa_decode_kernel<D, NT, MQ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, s.smem_bytes) !=
      cudaSuccess)
    return GQA_ERR_CUDA;
  kern<<<s.grid, kDecodeThreads, s.smem_bytes, stream>>>(tmk, tmv, a, s.tiles_per_group,
                                                          s.passes, s.units, s.segmax, s.stages,
                                                          a.counters);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace

DecodeShape plan_decode(const gqa_problem& p, int sm_count) {
  DecodeShape s{};
  const int64_t g = p.heads_q / p.heads_kv;
  const int64_t rows = g * p.seq_q;  // (head, query) rows per kv head
  s.D = static_cast<int>(p.head_dim);
  s.NT = rows <= 8 ? 1 : 2;
  s.HP = 8 * s.NT;
  s.passes = static_cast<int>((rows + s.HP - 1) / s.HP);
  // Keys some query can see: [key_lo, key_hi) (query 0's lower limit, the
  // last query's upper limit).
  s.key_hi = p.seq_k;
  s.key_lo = 0;
  if (p.causal) {
    if (p.seq_q - 1 + p.causal_offset + 1 < s.key_hi) s.key_hi = p.seq_q + p.causal_offset;
    if (p.window > 0 && p.causal_offset - p.window + 1 > 0) s.key_lo = p.causal_offset - p.window + 1;
  }
  s.t0 = static_cast<int>(s.key_lo / KT);
  s.tiles_per_group = static_cast<int>((s.key_hi + KT - 1) / KT) - s.t0;
  if (s.tiles_per_group < 1) s.tiles_per_group = 1;
  s.groups = p.batch * p.heads_kv * s.passes;
  s.units = s.groups * s.tiles_per_group;
  s.grid = static_cast<int>(s.units < sm_count ? s.units : sm_count);
  if (s.grid < 1) s.grid = 1;
  const int64_t per_cta = (s.units + s.grid - 1) / s.grid;
  s.segmax = static_cast<int>((per_cta + s.tiles_per_group - 1) / s.tiles_per_group + 1);
  const int stage_bytes = 2 * KT * s.D * 2;
  if (s.D == 128)
    s.stages = s.NT == 1 ? 6 : 5;
  else
    s.stages = 8;
  if (s.D == 128 && s.NT == 1)
    s.smem_bytes = DecodeSmem<128, 1>::bytes(s.stages);
  else if (s.D == 128)
    s.smem_bytes = DecodeSmem<128, 2>::bytes(s.stages);
  else if (s.NT == 1)
    s.smem_bytes = DecodeSmem<64, 1>::bytes(s.stages);
  else
    s.smem_bytes = DecodeSmem<64, 2>::bytes(s.stages);
  (void)stage_bytes;
  const int64_t slots = static_cast<int64_t>(s.grid) * s.segmax * s.HP;
  s.counters_offset = 256;
  s.part_ml_offset = s.counters_offset + ((s.groups * 4 + 255) / 256) * 256;
  s.part_o_offset = s.part_ml_offset + ((slots * 8 + 255) / 256) * 256;
  s.part_bytes = (s.part_o_offset - 256) + slots * s.D * 4;
  return s;
}

int launch_decode(const gqa_problem& p, const DecodeShape& s, const DecodeArgs& a,
                  const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream) {
  (void)p;
  const bool mq = a.Sq > 1;
  if (s.D == 128 && s.NT == 1)
    return mq ? launch_decode_t<128, 1, true>(s, a, tmk, tmv, stream)
              : launch_decode_t<128, 1, false>(s, a, tmk, tmv, stream);
  if (s.D == 128 && s.NT == 2)
    return mq ? launch_decode_t<128, 2, true>(s, a, tmk, tmv, stream)
              : launch_decode_t<128, 2, false>(s, a, tmk, tmv, stream);
  if (s.D == 64 && s.NT == 1)
    return mq ? launch_decode_t<64, 1, true>(s, a, tmk, tmv, stream)
              : launch_decode_t<64, 1, false>(s, a, tmk, tmv, stream);
  if (s.D == 64 && s.NT == 2)
    return mq ? launch_decode_t<64, 2, true>(s, a, tmk, tmv, stream)
              : launch_decode_t<64, 2, false>(s, a, tmk, tmv, stream);
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace gqa
