// Kernel (d): one decode step of HiLS attention.
//
// HiLS paper, aitrends.kr article, section "방법론" (Methodology) for the
// scoring and top-K, and ai-papers.net article, section "実験結果と性能",
// for the per-token decode with sparse KV access.  The query of (b, hq) sits
// at position t = seqlens[b]-1; its candidates are the fully-past chunks
// c < floor(t/C); its own chunk (keys floor(t/C)*C .. t) is attended under
// the causal mask.
//
// Four short kernels, all HBM- or latency-bound:
//   D1 scores   : s^ for every candidate chunk of every query head; one warp
//                 streams 32 compressed-key rows and scores them against the
//                 G query heads that share the kv head (one read of k' per
//                 kv head).
//   D2 top-K    : exact radix select (4 passes of 8 bits over an
//                 order-preserving integer image of the score), then a
//                 stable compaction in ascending chunk id; ties among equal
//                 scores go to the lower ids.
//   D3 partials : split-K over the K kept chunks plus the own chunk: one warp
//                 per (row, chunk) computes the intra-chunk softmax output
//                 and carries the chunk's fusion score.
//   D4 combine  : softmax over the chunk scores fuses the partials.
#pragma once
#include "attend_simt.cuh"

namespace hils {

struct DecodeWs {
  float* scores;      // [B*Hq, nc]
  int32_t* sel_ids;   // [B*Hq, K]
  float* sel_scores;  // [B*Hq, K]
  float* part_u;      // [B*Hq, K+1]
  float* part_o;      // [B*Hq, K+1, D]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t decode_ws_layout(int64_t rows, int64_t nc, int K, int D, char* base, DecodeWs* ws) {
  size_t off = 0;
  auto take = [&](size_t bytes) { char* p = base ? base + off : nullptr; off += align256(bytes); return p; };
  char* a = take(sizeof(float) * rows * nc);
  char* b = take(sizeof(int32_t) * rows * K);
  char* c = take(sizeof(float) * rows * K);
  char* d = take(sizeof(float) * rows * (K + 1));
  char* e = take(sizeof(float) * rows * (K + 1) * D);
  if (ws) {
    ws->scores = reinterpret_cast<float*>(a);
    ws->sel_ids = reinterpret_cast<int32_t*>(b);
    ws->sel_scores = reinterpret_cast<float*>(c);
    ws->part_u = reinterpret_cast<float*>(d);
    ws->part_o = reinterpret_cast<float*>(e);
  }
  return off;
}

// Number of candidate chunks of batch b (own chunk index); -1 if seqlens[b] is invalid.
__device__ __forceinline__ int64_t decode_own_chunk(const int32_t* seqlens, int b, int64_t cap) {
  const int32_t s = __ldg(seqlens + b);
  if (s < 1 || int64_t(s) > cap) return -1;
  return int64_t(s - 1) / kChunk;
}

constexpr int kDecChunksPerCta = 128;

template <typename T, int D, bool MMA_OPERAND>
__global__ void __launch_bounds__(128)
decode_scores_kernel(const T* __restrict__ q, const float* __restrict__ kp, const float* __restrict__ bp,
                     const __nv_bfloat16* __restrict__ kmma, const int32_t* __restrict__ seqlens, int64_t cap,
                     int64_t nc, int Hq, int G, int Hkv, float tau, float* __restrict__ ws_scores) {
  using KT = typename std::conditional<MMA_OPERAND, __nv_bfloat16, float>::type;
  using L = RowLayout<KT, D>;
  constexpr int E = L::E, LPK = L::LPK, KPI = L::KPI;
  constexpr int RS = MMA_OPERAND ? D + kExt : D;  // row stride of the k' rows
  extern __shared__ __align__(16) float sq[];       // [G][D]
  const int bh = blockIdx.y;
  const int b = bh / Hkv, h = bh % Hkv;
  const int64_t own = decode_own_chunk(seqlens, b, cap);
  if (own < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) record_error(HILS_ERR_DEVICE_BOUNDS);
    return;
  }
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, t = idx % D;
    const T x = q[(int64_t(b) * Hq + h * G + g) * D + t];
    if constexpr (sizeof(T) == 2) sq[idx] = __bfloat162float(x);
    else sq[idx] = x;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPK, sub = lane % LPK;
  const int64_t cw0 = int64_t(blockIdx.x) * kDecChunksPerCta + warp * 32;
  const KT* base = MMA_OPERAND ? reinterpret_cast<const KT*>(kmma) : reinterpret_cast<const KT*>(kp);
  base += int64_t(bh) * nc * RS;
  for (int it = 0; it < 32 / KPI; ++it) {
    const int64_t c = cw0 + it * KPI + grp;
    if (cw0 + it * KPI >= own) break;               // uniform
    const bool ok = c < own;
    const int64_t cc = ok ? c : cw0;
    float kv[E];
    Vec16<KT>::load(base + cc * RS + sub * E, kv);
    float bias;
    if constexpr (MMA_OPERAND) {
      const __nv_bfloat16* ext = kmma + (int64_t(bh) * nc + cc) * RS + D;
      bias = __bfloat162float(ext[0]) + __bfloat162float(ext[1]);
    } else {
      bias = __ldg(bp + int64_t(bh) * nc + cc);
    }
    for (int g = 0; g < G; ++g) {
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) part = fmaf(sq[g * D + sub * E + e], kv[e], part);
      const float dot = group_sum<LPK>(part);
      if (ok && sub == 0) {
        const float s = MMA_OPERAND ? tau * (dot + bias) : fmaf(tau, dot, bias);
        ws_scores[(int64_t(b) * Hq + h * G + g) * nc + c] = s;
      }
    }
  }
}

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix sum over 256 threads; also returns the total.
__device__ __forceinline__ int block_exclusive_scan256(int x, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int t = warp_tot[w];
    if (w < warp) before += t;
    total += t;
  }
  return before + incl - x;
}

__global__ void __launch_bounds__(256)
decode_topk_kernel(const float* __restrict__ ws_scores, const int32_t* __restrict__ seqlens, int64_t cap,
                   int64_t nc, int Hq, int K, int32_t* __restrict__ sel_ids, float* __restrict__ sel_scores) {
  __shared__ uint32_t hist[256];
  __shared__ int warp_tot[8];
  __shared__ uint32_t s_digit, s_above;
  const int row = blockIdx.x, b = row / Hq, tid = threadIdx.x;
  int64_t n = decode_own_chunk(seqlens, b, cap);
  if (n < 0) n = 0;
  const float* sc = ws_scores + int64_t(row) * nc;
  int32_t* oid = sel_ids + int64_t(row) * K;
  float* osc = sel_scores + int64_t(row) * K;
  if (n <= K) {
    for (int t = tid; t < K; t += 256) {
      oid[t] = t < n ? t : -1;
      osc[t] = t < n ? sc[t] : -INFINITY;
    }
    return;
  }
  uint32_t prefix = 0, mask = 0;
  int krem = K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[tid] = 0;
    __syncthreads();
    for (int64_t c = tid; c < n; c += 256) {
      const uint32_t key = order_key(sc[c]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t loc[8], lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { loc[j] = hist[255 - 8 * tid - j]; lsum += loc[j]; }
      uint32_t incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t excl = incl - lsum;
      if (excl < uint32_t(krem) && uint32_t(krem) <= incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + loc[j] >= uint32_t(krem)) { s_digit = 255 - 8 * tid - j; s_above = cum; break; }
          cum += loc[j];
        }
      }
    }
    __syncthreads();
    krem -= int(s_above);
    prefix |= s_digit << shift;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  // prefix = key of the K-th largest score; take all keys above it and the
  // krem lowest-id keys equal to it.
  const int64_t seg = (n + 255) / 256;
  const int64_t s0 = tid * seg, s1 = (s0 + seg < n) ? s0 + seg : n;
  int gt = 0, eq = 0;
  for (int64_t c = s0; c < s1; ++c) {
    const uint32_t key = order_key(sc[c]);
    gt += key > prefix;
    eq += key == prefix;
  }
  int tot;
  const int eq_before = block_exclusive_scan256(eq, warp_tot, tot);
  int take_eq = krem - eq_before;
  take_eq = take_eq < 0 ? 0 : (take_eq > eq ? eq : take_eq);
  const int pos0 = block_exclusive_scan256(gt + take_eq, warp_tot, tot);
  int pos = pos0, eq_seen = 0;
  for (int64_t c = s0; c < s1; ++c) {
    const float s = sc[c];
    const uint32_t key = order_key(s);
    bool take = key > prefix;
    if (key == prefix) take = eq_seen++ < take_eq;
    if (take && pos < K) { oid[pos] = int32_t(c); osc[pos] = s; ++pos; }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
decode_partial_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                      const int32_t* __restrict__ seqlens, int64_t cap, int Hq, int G, int Hkv, int K,
                      float tau, const int32_t* __restrict__ sel_ids, const float* __restrict__ sel_scores,
                      float* __restrict__ part_u, float* __restrict__ part_o, int64_t n_units) {
  using L = RowLayout<T, D>;
  constexpr int E = L::E, LPK = L::LPK;
  const int lane = threadIdx.x & 31, sub = lane % LPK;
  const int64_t unit = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (unit >= n_units) return;
  const int64_t row = unit / (K + 1);
  const int slot = int(unit % (K + 1));
  const int b = int(row / Hq), hq = int(row % Hq);
  const int64_t own = decode_own_chunk(seqlens, b, cap);
  float* uo = part_u + row * (K + 1) + slot;
  float* po = part_o + (row * (K + 1) + slot) * D;
  if (own < 0) {
    if (lane == 0) *uo = -INFINITY;
    return;
  }
  const int64_t t = int64_t(__ldg(seqlens + b)) - 1;
  const int64_t bh = int64_t(b) * Hkv + hq / G;
  const T* kbh = kc + bh * cap * D;
  const T* vbh = vc + bh * cap * D;
  float qv[E];
  Vec16<T>::load(q + row * D + sub * E, qv);
  float oc[E];
  float u;
  if (slot == K) {
    u = attend_range<T, D>(qv, kbh, vbh, own * kChunk, t + 1, tau, oc);
  } else {
    const int32_t c = sel_ids[row * K + slot];
    if (c < 0 || c >= own) {
      if (lane == 0) *uo = -INFINITY;
      return;
    }
    attend_range<T, D>(qv, kbh, vbh, int64_t(c) * kChunk, int64_t(c + 1) * kChunk, tau, oc);
    u = sel_scores[row * K + slot];
  }
  if (lane < LPK) {
#pragma unroll
    for (int e = 0; e < E; e += 4)
      *reinterpret_cast<float4*>(po + sub * E + e) = make_float4(oc[e], oc[e + 1], oc[e + 2], oc[e + 3]);
  }
  if (lane == 0) *uo = u;
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(const float* __restrict__ part_u, const float* __restrict__ part_o,
                      const int32_t* __restrict__ seqlens, int64_t cap, int Hq, int K,
                      const int32_t* __restrict__ sel_ids, const float* __restrict__ sel_scores,
                      T* __restrict__ o, int32_t* __restrict__ ids_out, float* __restrict__ scores_out,
                      int64_t n_rows) {
  constexpr int EL = D / 32;   // output elements per lane
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= n_rows) return;
  const int b = int(row / Hq);
  const bool valid = decode_own_chunk(seqlens, b, cap) >= 0;
  float M = -INFINITY;
  for (int s = 0; s <= K; ++s) M = fmaxf(M, part_u[row * (K + 1) + s]);
  float Z = 0.f, acc[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) acc[e] = 0.f;
  if (valid) {
    for (int s = 0; s <= K; ++s) {
      const float u = part_u[row * (K + 1) + s];
      if (u == -INFINITY) continue;
      const float w = expf(u - M);
      Z += w;
      const float* po = part_o + (row * (K + 1) + s) * D + lane * EL;
#pragma unroll
      for (int e = 0; e < EL; ++e) acc[e] += w * po[e];
    }
  }
  const float inv = Z > 0.f ? 1.f / Z : 0.f;
#pragma unroll
  for (int e = 0; e < EL; ++e) {
    const float x = acc[e] * inv;
    if constexpr (sizeof(T) == 2) o[row * D + lane * EL + e] = __float2bfloat16_rn(x);
    else o[row * D + lane * EL + e] = x;
  }
  for (int t = lane; t < K; t += 32) {
    if (ids_out) ids_out[row * K + t] = valid ? sel_ids[row * K + t] : -1;
    if (scores_out) scores_out[row * K + t] = valid ? sel_scores[row * K + t] : -INFINITY;
  }
}

}  // namespace hils
