// CUDA-core sparse attention of single query rows (fp32 prefill path and the
// per-chunk partials of decode).
//
// HiLS paper, hotpaper.ai abstract and aitrends.kr article, sections "방법론"
// (Methodology) and glossary "계층적 소프트맥스" (hierarchical softmax): each
// query attends independently to each kept chunk (intra-chunk softmax), and
// the chunk outputs are fused by a softmax over the chunk scores.  The own
// chunk is attended under the causal mask and fused with its exact
// log-sum-exp as score.
//
// One warp per query row.  Key and value rows stream with one 16-byte load
// per lane (LPK lanes per row, KPI rows per iteration, fully coalesced), each
// key group keeps an online softmax state, and the groups merge with xor
// shuffles.  The fusion over chunks is a second online softmax.
#pragma once
#include "common.cuh"

namespace hils {

// Softmax attention of one query over keys [j0, j1) (j1 - j0 <= 64) of one
// (b, kv head) slab.  Returns the log-sum-exp of the logits; out receives this
// lane's slice (sub*E .. sub*E+E) of the normalised output.  Warp-collective.
template <typename T, int D>
__device__ __forceinline__ float attend_range(const float (&qv)[RowLayout<T, D>::E], const T* __restrict__ kbh,
                                              const T* __restrict__ vbh, int64_t j0, int64_t j1, float tau,
                                              float (&out)[RowLayout<T, D>::E]) {
  using L = RowLayout<T, D>;
  constexpr int E = L::E, LPK = L::LPK, KPI = L::KPI;
  const int lane = threadIdx.x & 31;
  const int grp = lane / LPK, sub = lane % LPK;
  SoftAcc<E> st;
  st.init();
#pragma unroll 4
  for (int it = 0; it < kChunk / KPI; ++it) {
    const int64_t j = j0 + it * KPI + grp;
    const bool ok = j < j1;
    const int64_t jj = ok ? j : j0;
    float kv[E], vv[E];
    Vec16<T>::load(kbh + jj * D + sub * E, kv);
    Vec16<T>::load(vbh + jj * D + sub * E, vv);
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) part = fmaf(qv[e], kv[e], part);
    const float z = group_sum<LPK>(part) * tau;
    if (ok) st.add(z, vv);
    if (j0 + (it + 1) * KPI >= j1) break;   // uniform across the warp
  }
#pragma unroll
  for (int off = LPK; off < 32; off <<= 1) st.merge_xor(off);
  const float inv = 1.f / st.l;
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = st.acc[e] * inv;
  return st.m + logf(st.l);
}

// Running fusion over chunks: softmax over chunk scores u of normalised chunk outputs.
template <int E> struct Fusion {
  float M, Z, acc[E];
  __device__ __forceinline__ void init(float u, const float (&o)[E]) {
    M = u;
    Z = 1.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = o[e];
  }
  __device__ __forceinline__ void add(float u, const float (&o)[E]) {
    const float Mn = fmaxf(M, u);
    const float a = expf(M - Mn), w = expf(u - Mn);
    Z = Z * a + w;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] * a + w * o[e];
    M = Mn;
  }
};

// Prefill, fp32 / CUDA-core path: one warp per row (b, hq, i).
template <typename T, int D>
__global__ void __launch_bounds__(128)
prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    const int32_t* __restrict__ ids, const float* __restrict__ scores, T* __restrict__ o,
                    float* __restrict__ lse_own, int64_t n_tok, int Hq, int G, int Hkv, int K, float tau,
                    int64_t n_rows, int wm1, const float* __restrict__ kp, const float* __restrict__ bp,
                    const __nv_bfloat16* __restrict__ kmma) {
  using L = RowLayout<T, D>;
  constexpr int E = L::E, LPK = L::LPK;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPK;
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= n_rows) return;
  const int64_t bhq = row / n_tok, i = row % n_tok;
  const int64_t b = bhq / Hq, hq = bhq % Hq;
  const int64_t bh = b * Hkv + hq / G;
  const T* kbh = k + bh * n_tok * D;
  const T* vbh = v + bh * n_tok * D;
  float qv[E];
  Vec16<T>::load(q + row * D + sub * E, qv);
  const int64_t own = i / kChunk;

  float oc[E];
  // the local window: the own chunk (causal) and the wm1 chunks before it,
  // each fused at its exact log-sum-exp, which together is one branch over
  // the window's keys at the window's log-sum-exp lo
  float lo = attend_range<T, D>(qv, kbh, vbh, own * kChunk, i + 1, tau, oc);
  Fusion<E> f;
  f.init(lo, oc);
  for (int64_t c = own - 1; c >= 0 && c >= own - wm1; --c) {
    const float lc = attend_range<T, D>(qv, kbh, vbh, c * kChunk, (c + 1) * kChunk, tau, oc);
    f.add(lc, oc);
    lo = fmaxf(lo, lc) + log1pf(expf(-fabsf(lo - lc)));
  }
  const int64_t n_cand = n_candidates(i, wm1);
  for (int t = 0; t < K; ++t) {
    const int32_t c = __ldg(ids + row * K + t);
    if (c < 0) continue;
    if (c >= n_cand) {
      if (lane == 0) record_error(HILS_ERR_DEVICE_BOUNDS);
      continue;
    }
    // the chunk score from select, or (scores NULL) recomputed as select
    // computes it: fp32 tau <q, k'> + b', or from the bf16 scoring operand
    float u;
    if (scores != nullptr) {
      u = __ldg(scores + row * K + t);
    } else {
      const int64_t cr = bh * (n_tok / kChunk) + c;
      float part = 0.f;
      if (kmma != nullptr) {   // bf16 rows (E = 8): one 16-byte piece of the bf16 k' row per lane
        float kv[8];
        Vec16<__nv_bfloat16>::load(kmma + cr * (D + kExt) + sub * 8, kv);
#pragma unroll
        for (int e = 0; e < E && e < 8; ++e) part = fmaf(qv[e], kv[e], part);
        const float x = __bfloat162float(kmma[cr * (D + kExt) + D]) + __bfloat162float(kmma[cr * (D + kExt) + D + 1]);
        u = tau * (group_sum<LPK>(part) + x);
      } else {
        float kv[4];
#pragma unroll
        for (int e = 0; e < E; e += 4) {
          Vec16<float>::load(kp + cr * D + sub * E + e, kv);
#pragma unroll
          for (int z = 0; z < 4; ++z) part = fmaf(qv[e + z], kv[z], part);
        }
        u = fmaf(tau, group_sum<LPK>(part), __ldg(bp + cr));
      }
    }
    attend_range<T, D>(qv, kbh, vbh, int64_t(c) * kChunk, int64_t(c + 1) * kChunk, tau, oc);
    f.add(u, oc);
  }
  if (lane < LPK) {
    float res[E];
    const float inv = 1.f / f.Z;
#pragma unroll
    for (int e = 0; e < E; ++e) res[e] = f.acc[e] * inv;
    Vec16<T>::store(o + row * D + sub * E, res);
  }
  if (lse_own != nullptr && lane == 0) lse_own[row] = lo;
}

}  // namespace hils
