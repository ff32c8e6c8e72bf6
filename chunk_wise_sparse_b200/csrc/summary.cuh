// Kernel (a): landmark chunk summary.
//
// HiLS paper, aitrends.kr article, sections "방법론" (Methodology) and
// "기술 상세" (Technical details): the landmark query of chunk c attends over
// the chunk's C keys; the weighted key sum is the compressed key k'_c and the
// entropy of the attention distribution is the bias b'_c.
//
// One warp per chunk.  The chunk's 64 key rows stream through the warp with
// one 16-byte load per lane (LPK lanes per key row, KPI rows per iteration),
// so every 128-byte line of K is read once, coalesced.  Each key group keeps
// an online-softmax state (max, sum, sum p*z, sum p*k) that the groups merge
// with xor shuffles at the end.  HBM-bound: algorithmic bytes per chunk are
// C*d*sizeof(T) (keys) + d*sizeof(T) (landmark) + 4d + 4 (k', b' fp32)
// + 2(d+16) (bf16 scoring operand).
#pragma once
#include "common.cuh"

namespace hils {

template <typename T, int D>
__global__ void __launch_bounds__(256)
summary_kernel(const T* __restrict__ k, const T* __restrict__ lq, int64_t n_tok, int64_t nc,
               int64_t chunk_begin, int64_t span, int64_t n_units, float* __restrict__ kp,
               float* __restrict__ bp, __nv_bfloat16* __restrict__ kmma, float tau, PagedKv pk, int Hkv) {
  using L = RowLayout<T, D>;
  constexpr int E = L::E, LPK = L::LPK, KPI = L::KPI;
  constexpr int ITERS = kChunk / KPI;
  constexpr int BATCH = ITERS < 8 ? ITERS : 8;
  const int lane = threadIdx.x & 31;
  const int64_t unit = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (unit >= n_units) return;
  const int64_t bh = unit / span, c = chunk_begin + unit % span;
  const int grp = lane / LPK, sub = lane % LPK;

  const int64_t koff = kv_chunk_offset(pk, bh / Hkv, bh % Hkv, c, Hkv, n_tok, nc, D);
  if (koff < 0) return;   // page outside the pool: recorded, chunk left unwritten
  float lqv[E];
  Vec16<T>::load(lq + (bh * nc + c) * D + sub * E, lqv);
  const T* kc = k + koff + sub * E;

  // online state of this key group: max m, sum l of exp(z-m), sum s of exp(z-m)*z, acc of exp(z-m)*k
  float m = -INFINITY, l = 0.f, s = 0.f, acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;

  for (int it0 = 0; it0 < ITERS; it0 += BATCH) {
    float kv[BATCH][E];
#pragma unroll
    for (int u = 0; u < BATCH; ++u) Vec16<T>::load_stream(kc + int64_t((it0 + u) * KPI + grp) * D, kv[u]);
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) part = fmaf(lqv[e], kv[u][e], part);
      const float z = group_sum<LPK>(part) * tau;
      const float mn = fmaxf(m, z);
      const float a = expf(m - mn);
      const float p = expf(z - mn);
      l = l * a + p;
      s = s * a + p * z;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = acc[e] * a + p * kv[u][e];
      m = mn;
    }
  }
  // merge the KPI key groups (lanes sub, sub+LPK, ...)
#pragma unroll
  for (int off = LPK; off < 32; off <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off);
    const float lo = __shfl_xor_sync(0xffffffffu, l, off);
    const float so = __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(m, mo);
    const float a = expf(m - mn), b = expf(mo - mn);
    l = l * a + lo * b;
    s = s * a + so * b;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float ao = __shfl_xor_sync(0xffffffffu, acc[e], off);
      acc[e] = acc[e] * a + ao * b;
    }
    m = mn;
  }
  if (grp != 0) return;
  const float inv = 1.f / l;
  float kpv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) kpv[e] = acc[e] * inv;
  float* kout = kp + (bh * nc + c) * D + sub * E;
#pragma unroll
  for (int e = 0; e < E; e += 4) *reinterpret_cast<float4*>(kout + e) = make_float4(kpv[e], kpv[e + 1], kpv[e + 2], kpv[e + 3]);
  // b' = LSE(z) - sum p z  (= -sum p log p)
  const float bias = m + logf(l) - s * inv;
  if (sub == 0) bp[bh * nc + c] = bias;
  if (kmma != nullptr) {
    __nv_bfloat16* row = kmma + (bh * nc + c) * (D + kExt);
#pragma unroll
    for (int e = 0; e < E; e += 2)
      *reinterpret_cast<__nv_bfloat162*>(row + sub * E + e) = __floats2bfloat162_rn(kpv[e], kpv[e + 1]);
    if (sub == 0) {
      // the bias rides in the MMA as x_hi + x_lo (x = b'/tau) against q-extension [1, 1, 0...]
      const float x = bias / tau;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      __nv_bfloat162 hl;
      hl.x = hi;
      hl.y = lo;
      uint4 z4 = make_uint4(*reinterpret_cast<uint32_t*>(&hl), 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(row + D) = z4;
      *reinterpret_cast<uint4*>(row + D + 8) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

}  // namespace hils
