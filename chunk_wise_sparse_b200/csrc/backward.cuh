// Backward of the forward pass for a fixed selection.
//
// AI Trends article, section "방법론" (Methodology): the chunk score s^ is
// part of the forward attention, so the gradient of the loss reaches the
// landmark queries (through k', b') and the Q-Cal adapter (through the
// scoring query); the top-K choice itself is not differentiated.
//
// Per row i with g = dL/dO_i, Dg = <g, O_i>, fusion normaliser M' and, per
// branch c (a selected chunk, or the local window w), a_c = exp(u_c - M'),
// p = the softmax inside the branch, X_c = <g, o_c>:
//   selected c:  dz_j = a_c p_j (<g, v_j> - X_c),   du_c = a_c (X_c - Dg)
//                dq^ += tau du_c k'_c,  dk'_c += tau du_c q^,  db'_c += du_c
//   window w:    dz_j = P_ij (<g, v_j> - Dg),  P_ij = exp(tau s_ij - M')
//   every key:   dq += tau dz_j k_j,  dk_j += tau dz_j q,  dv_j += a_c p_j g
// and the landmark summaries pass dk', db' on to the keys and the landmark
// queries.
//
// Kernels (CUDA cores; a first, exact design):
//   bwd_prep     per row: M' = log(sum_kept exp(s^) + exp(lse_w)) and Dg.
//   (index)      the forward's chunk-centric index: per (kv head, window,
//                chunk) the list of (row, slot) pairs with s^ - M'.
//   bwd_window   one CTA per (chunk of positions, query head): the window
//                branch of those 64 rows, one key chunk at a time; dq is
//                written (plain stores), dk, dv receive the chunk's sums.
//   bwd_chunk    persistent over the index's tiles (up to 128 pairs of one
//                chunk): per pair a warp forms dz, a p and the pair's dq
//                (added to dq); the chunk's dk, dv are two small GEMMs over
//                the tile's pairs (dZ^T Q and (a P)^T dO) held in registers,
//                added to dk, dv once per tile; dk', db' of the chunk are
//                summed in shared memory.
//   bwd_summary  one warp per chunk: the landmark softmax again, dlq, and
//                the keys' share of dk'.
#pragma once
#include "prefill_cc.cuh"

namespace hils {

template <typename T>
__device__ __forceinline__ float ldf(const T* p) {
  if constexpr (sizeof(T) == 2) return __bfloat162float(*p);
  else return *p;
}

// ---------------------------------------------------------------- per-row statistics
// One warp per row: M' from the kept scores and the window's log-sum-exp,
// Dg = <dO, O>.
template <typename T, int D>
__global__ void __launch_bounds__(128)
bwd_prep_kernel(const int32_t* __restrict__ ids, const float* __restrict__ scores, const float* __restrict__ lse_w,
                const T* __restrict__ o, const T* __restrict__ d_o, int64_t n_tok, int K, int wm1, int64_t n_rows,
                float* __restrict__ rowstat, float* __restrict__ dvec) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= n_rows) return;
  const int64_t i = row % n_tok;
  const int64_t n_cand = n_candidates(i, wm1);
  float dg = 0.f;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) dg = fmaf(ldf(o + row * D + lane + 32 * e), ldf(d_o + row * D + lane + 32 * e), dg);
  float mx = -INFINITY;
  for (int t = lane; t < K; t += 32) {
    const int32_t c = ids[row * K + t];
    if (c >= 0 && c < n_cand) mx = fmaxf(mx, scores[row * K + t]);
  }
  const float lw = lse_w[row];
  mx = fmaxf(mx, lw);
#pragma unroll
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float z = lane == 0 ? expf(lw - mx) : 0.f;
  for (int t = lane; t < K; t += 32) {
    const int32_t c = ids[row * K + t];
    if (c >= 0 && c < n_cand) z += expf(scores[row * K + t] - mx);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    z += __shfl_xor_sync(0xffffffffu, z, off);
    dg += __shfl_xor_sync(0xffffffffu, dg, off);
  }
  if (lane == 0) {
    rowstat[row] = mx + logf(z);
    dvec[row] = dg;
  }
}

// ---------------------------------------------------------------- shared pieces
// Shared-memory tiles of the two per-chunk kernels (fp32):
//   ks, vs      [64][D+1]  the chunk's keys and values (padded rows: lane j
//                          reading column t of row j hits bank (j + t) % 32)
//   qs, gs      [SUB][D]   the rows' queries and output gradients
//   dzs, pws    [SUB][64]  per row: tau dz_j and the weight of v_j
template <int D>
struct BwdTiles {
  static constexpr int SUB = 64;        // rows per pass
  static constexpr int KS = D + 1;
  static constexpr int THREADS = 256;
  static constexpr int TJ = 4;          // keys per thread in the GEMMs
  static constexpr int TT = D / 16;     // dims per thread in the GEMMs (16 x 16 threads)
  static constexpr size_t KV_BYTES = size_t(2) * kChunk * KS * 4;
  static constexpr size_t ROW_BYTES = size_t(2) * SUB * D * 4;
  static constexpr size_t P_BYTES = size_t(2) * SUB * kChunk * 4;
};

// The chunk's keys and values into shared memory as fp32.
template <typename T, int D>
__device__ __forceinline__ void bwd_load_kv(const T* __restrict__ k, const T* __restrict__ v, int64_t row0,
                                            float* ks, float* vs) {
  using BT = BwdTiles<D>;
  for (int idx = threadIdx.x; idx < kChunk * D; idx += blockDim.x) {
    const int j = idx / D, t = idx % D;
    ks[j * BT::KS + t] = ldf(k + (row0 + j) * D + t);
    vs[j * BT::KS + t] = ldf(v + (row0 + j) * D + t);
  }
}

// dk[j][t] += sum_r dzs[r][j] qs[r][t] and dv[j][t] += sum_r pws[r][j] gs[r][t]
// over the n rows of the pass; thread (jb, tb) of a 16 x 16 grid owns keys
// 4 jb .. 4 jb + 3 and dims tb * TT .. tb * TT + TT - 1.
template <int D>
__device__ __forceinline__ void bwd_gemm_acc(const float* dzs, const float* pws, const float* qs, const float* gs,
                                             int n, float (&ak)[4][D / 16], float (&av)[4][D / 16]) {
  using BT = BwdTiles<D>;
  const int jb = threadIdx.x >> 4, tb = threadIdx.x & 15;
  for (int r = 0; r < n; ++r) {
    const float4 dz = *reinterpret_cast<const float4*>(dzs + r * kChunk + 4 * jb);
    const float4 pw = *reinterpret_cast<const float4*>(pws + r * kChunk + 4 * jb);
    const float dza[4] = {dz.x, dz.y, dz.z, dz.w}, pwa[4] = {pw.x, pw.y, pw.z, pw.w};
    float qv[BT::TT], gv[BT::TT];
#pragma unroll
    for (int t = 0; t < BT::TT; t += 4) {
      const float4 q4 = *reinterpret_cast<const float4*>(qs + r * D + tb * BT::TT + t);
      const float4 g4 = *reinterpret_cast<const float4*>(gs + r * D + tb * BT::TT + t);
      qv[t] = q4.x; qv[t + 1] = q4.y; qv[t + 2] = q4.z; qv[t + 3] = q4.w;
      gv[t] = g4.x; gv[t + 1] = g4.y; gv[t + 2] = g4.z; gv[t + 3] = g4.w;
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int t = 0; t < BT::TT; ++t) {
        ak[a][t] = fmaf(dza[a], qv[t], ak[a][t]);
        av[a][t] = fmaf(pwa[a], gv[t], av[a][t]);
      }
  }
}

template <int D>
__device__ __forceinline__ void bwd_gemm_flush(float (&ak)[4][D / 16], float (&av)[4][D / 16], float* dk, float* dv,
                                               int64_t row0) {
  using BT = BwdTiles<D>;
  const int jb = threadIdx.x >> 4, tb = threadIdx.x & 15;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int t = 0; t < BT::TT; ++t) {
      const int64_t at = (row0 + 4 * jb + a) * D + tb * BT::TT + t;
      atomicAdd(dk + at, ak[a][t]);
      atomicAdd(dv + at, av[a][t]);
      ak[a][t] = 0.f;
      av[a][t] = 0.f;
    }
}

// Scores of one row against the 64 keys in shared memory: lane owns keys
// lane and lane + 32; q from shared memory (broadcast).
template <int D>
__device__ __forceinline__ void bwd_row_dots(const float* x, const float* ks, float& s0, float& s1) {
  using BT = BwdTiles<D>;
  const int lane = threadIdx.x & 31;
  s0 = 0.f;
  s1 = 0.f;
#pragma unroll 8
  for (int t = 0; t < D; ++t) {
    const float xt = x[t];
    s0 = fmaf(xt, ks[lane * BT::KS + t], s0);
    s1 = fmaf(xt, ks[(lane + 32) * BT::KS + t], s1);
  }
}

// sum_j w_j k_j[t] for the dims t = lane + 32 e of one row (w_j held by lane j % 32)
template <int D>
__device__ __forceinline__ void bwd_row_combine(float w0, float w1, const float* ks, float (&out)[D / 32]) {
  using BT = BwdTiles<D>;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) out[e] = 0.f;
#pragma unroll 4
  for (int j = 0; j < 32; ++j) {
    const float a = __shfl_sync(0xffffffffu, w0, j), c = __shfl_sync(0xffffffffu, w1, j);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
      out[e] = fmaf(a, ks[j * BT::KS + lane + 32 * e], out[e]);
      out[e] = fmaf(c, ks[(j + 32) * BT::KS + lane + 32 * e], out[e]);
    }
  }
}

// ---------------------------------------------------------------- window branch
// One CTA per (chunk o of positions, (b, hq)): the 64 rows at positions
// 64 o .. 64 o + 63 attend their windows, the key chunks o - wm1 .. o (the
// last under the causal mask), with weights P = exp(tau s - M').
template <typename T, int D>
__global__ void __launch_bounds__(BwdTiles<D>::THREADS)
bwd_window_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ d_o, const float* __restrict__ rowstat, const float* __restrict__ dvec,
                  int64_t n_tok, int Hq, int G, int Hkv, int wm1, float tau, float* __restrict__ dq,
                  float* __restrict__ dk, float* __restrict__ dv) {
  using BT = BwdTiles<D>;
  extern __shared__ __align__(16) float sm[];
  float* ks = sm;
  float* vs = ks + kChunk * BT::KS;
  float* qs = vs + kChunk * BT::KS;
  float* gs = qs + BT::SUB * D;
  float* dzs = gs + BT::SUB * D;
  float* pws = dzs + BT::SUB * kChunk;
  float* dqa = pws + BT::SUB * kChunk;   // [SUB][D] the rows' dq
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t own = blockIdx.x;
  const int bhq = int(blockIdx.y), b = bhq / Hq, hq = bhq % Hq, h = hq / G;
  const int64_t p0 = own * kChunk;
  const int64_t row0 = int64_t(bhq) * n_tok + p0;
  const int64_t kv0 = (int64_t(b) * Hkv + h) * n_tok;
  for (int idx = tid; idx < BT::SUB * D; idx += BT::THREADS) {
    qs[idx] = ldf(q + row0 * D + idx);
    gs[idx] = ldf(d_o + row0 * D + idx);
    dqa[idx] = 0.f;
  }
  float ak[4][BT::TT], av[4][BT::TT];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int t = 0; t < BT::TT; ++t) ak[a][t] = av[a][t] = 0.f;
  const int64_t c_lo = own - wm1 > 0 ? own - wm1 : 0;
  for (int64_t cj = c_lo; cj <= own; ++cj) {
    __syncthreads();
    bwd_load_kv<T, D>(k, v, kv0 + cj * kChunk, ks, vs);
    __syncthreads();
    for (int r = warp; r < BT::SUB; r += BT::THREADS / 32) {
      const int64_t pos = p0 + r;
      const float mp = rowstat[row0 + r], dg = dvec[row0 + r];
      float s0, s1, g0, g1;
      bwd_row_dots<D>(qs + r * D, ks, s0, s1);
      bwd_row_dots<D>(gs + r * D, vs, g0, g1);
      const bool ok0 = cj * kChunk + lane <= pos, ok1 = cj * kChunk + lane + 32 <= pos;
      const float P0 = ok0 ? expf(tau * s0 - mp) : 0.f, P1 = ok1 ? expf(tau * s1 - mp) : 0.f;
      const float dz0 = tau * P0 * (g0 - dg), dz1 = tau * P1 * (g1 - dg);
      dzs[r * kChunk + lane] = dz0;
      dzs[r * kChunk + lane + 32] = dz1;
      pws[r * kChunk + lane] = P0;
      pws[r * kChunk + lane + 32] = P1;
      float acc[D / 32];
      bwd_row_combine<D>(dz0, dz1, ks, acc);
#pragma unroll
      for (int e = 0; e < D / 32; ++e) dqa[r * D + lane + 32 * e] += acc[e];
    }
    __syncthreads();
    bwd_gemm_acc<D>(dzs, pws, qs, gs, BT::SUB, ak, av);
    bwd_gemm_flush<D>(ak, av, dk, dv, kv0 + cj * kChunk);
  }
  __syncthreads();
  // the window kernel runs first: dq is written here, the selected chunks add to it
  for (int idx = tid; idx < BT::SUB * D; idx += BT::THREADS) dq[row0 * D + idx] = dqa[idx];
}

// ---------------------------------------------------------------- selected chunks
// Persistent over the index's tiles (up to 128 (row, slot) pairs of one
// chunk), the rows taken SUB at a time.
template <typename T, int D>
__global__ void __launch_bounds__(BwdTiles<D>::THREADS)
bwd_chunk_kernel(const T* __restrict__ q, const T* __restrict__ q_score, const T* __restrict__ k,
                 const T* __restrict__ v, const T* __restrict__ d_o, const float* __restrict__ kprime,
                 const float* __restrict__ dvec, const int32_t* __restrict__ tile_start, const int4* __restrict__ items,
                 const int2* __restrict__ e_pair, const CcDims c,
                 float* dq, float* dqs, float* __restrict__ dk, float* __restrict__ dv,   // dqs may be dq
                 float* __restrict__ dkp, float* __restrict__ dbp) {
  using BT = BwdTiles<D>;
  extern __shared__ __align__(16) float sm[];
  float* ks = sm;
  float* vs = ks + kChunk * BT::KS;
  float* qs = vs + kChunk * BT::KS;
  float* gs = qs + BT::SUB * D;
  float* dzs = gs + BT::SUB * D;
  float* pws = dzs + BT::SUB * kChunk;
  float* kpc = pws + BT::SUB * kChunk;   // [D] the chunk's k'
  float* dkpa = kpc + D;                 // [D] sum of tau du q^ over the tile's pairs
  float* dbpa = dkpa + D;                // [1] sum of du
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float tau = c.tau;
  const int n_all = tile_start[c.n_keys];
  float ak[4][BT::TT], av[4][BT::TT];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int t = 0; t < BT::TT; ++t) ak[a][t] = av[a][t] = 0.f;
  for (int tile = blockIdx.x; tile < n_all; tile += gridDim.x) {
    const int4 it = items[tile];   // first entry, K/V row, pair count
    const int64_t first = it.x, kvrow = it.y;
    const int n = it.z;
    const int64_t bh = kvrow / c.n_tok, chunk = (kvrow % c.n_tok) / kChunk;
    __syncthreads();
    bwd_load_kv<T, D>(k, v, kvrow, ks, vs);
    for (int t = tid; t < D; t += BT::THREADS) {
      kpc[t] = kprime[(bh * c.nc + chunk) * D + t];
      dkpa[t] = 0.f;
    }
    if (tid == 0) dbpa[0] = 0.f;
    for (int s0 = 0; s0 < n; s0 += BT::SUB) {
      const int ns = n - s0 < BT::SUB ? n - s0 : BT::SUB;
      __syncthreads();
      for (int idx = tid; idx < ns * D; idx += BT::THREADS) {
        const int r = idx / D, t = idx % D;
        const int64_t row = e_pair[first + s0 + r].x;
        qs[idx] = ldf(q + row * D + t);
        gs[idx] = ldf(d_o + row * D + t);
      }
      __syncthreads();
      for (int r = warp; r < ns; r += BT::THREADS / 32) {
        const int2 ep = e_pair[first + s0 + r];
        const int64_t row = ep.x;
        const float a = expf(__int_as_float(ep.y));   // exp(s^ - M')
        const float dg = dvec[row];
        float s0v, s1v, g0, g1;
        bwd_row_dots<D>(qs + r * D, ks, s0v, s1v);
        bwd_row_dots<D>(gs + r * D, vs, g0, g1);
        const float z0 = tau * s0v, z1 = tau * s1v;
        float m = fmaxf(z0, z1);
#pragma unroll
        for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float e0 = expf(z0 - m), e1 = expf(z1 - m);
        float l = e0 + e1;
#pragma unroll
        for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        const float p0 = e0 / l, p1 = e1 / l;
        float X = p0 * g0 + p1 * g1;
#pragma unroll
        for (int off = 16; off; off >>= 1) X += __shfl_xor_sync(0xffffffffu, X, off);
        const float dz0 = tau * a * p0 * (g0 - X), dz1 = tau * a * p1 * (g1 - X);
        const float du = a * (X - dg);
        dzs[r * kChunk + lane] = dz0;
        dzs[r * kChunk + lane + 32] = dz1;
        pws[r * kChunk + lane] = a * p0;
        pws[r * kChunk + lane + 32] = a * p1;
        float acc[D / 32];
        bwd_row_combine<D>(dz0, dz1, ks, acc);
#pragma unroll
        for (int e = 0; e < D / 32; ++e) {
          const int t = lane + 32 * e;
          const float sg = tau * du * kpc[t];   // through the chunk score
          if (dqs == dq) {
            atomicAdd(dq + row * D + t, acc[e] + sg);
          } else {
            atomicAdd(dq + row * D + t, acc[e]);
            atomicAdd(dqs + row * D + t, sg);
          }
          const float qv = q_score ? ldf(q_score + row * D + t) : qs[r * D + t];
          atomicAdd(dkpa + t, tau * du * qv);
        }
        if (lane == 0) atomicAdd(dbpa, du);
      }
      __syncthreads();
      bwd_gemm_acc<D>(dzs, pws, qs, gs, ns, ak, av);
    }
    bwd_gemm_flush<D>(ak, av, dk, dv, kvrow);
    __syncthreads();
    for (int t = tid; t < D; t += BT::THREADS) atomicAdd(dkp + (bh * c.nc + chunk) * D + t, dkpa[t]);
    if (tid == 0) atomicAdd(dbp + bh * c.nc + chunk, dbpa[0]);
  }
}

// ---------------------------------------------------------------- landmark summaries
// One warp per chunk (four per CTA), the chunk's keys staged in shared
// memory: the landmark softmax pl over the chunk, then
//   dzl_j = pl_j <dk', k_j - k'> - db' pl_j (zl_j - sum pl zl)
//   dlq = tau sum_j dzl_j k_j,   dk_j += tau dzl_j lq + pl_j dk'.
template <typename T, int D>
__global__ void __launch_bounds__(128)
bwd_summary_kernel(const T* __restrict__ k, const T* __restrict__ lq, const float* __restrict__ kprime,
                   const float* __restrict__ dkp, const float* __restrict__ dbp, int64_t n_tok, int64_t nc,
                   int64_t n_units, float tau, float* __restrict__ dk, float* __restrict__ dlq) {
  using BT = BwdTiles<D>;
  constexpr int WS = kChunk * BT::KS + 3 * D;   // floats per warp
  extern __shared__ __align__(16) float sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = int64_t(blockIdx.x) * 4 + warp;   // (b, kv head) * nc + chunk
  if (unit >= n_units) return;
  float* ks = sm + warp * WS;
  float* lqw = ks + kChunk * BT::KS;
  float* dkw = lqw + D;
  float* kpw = dkw + D;
  const int64_t bh = unit / nc, cidx = unit % nc;
  const int64_t kv0 = bh * n_tok + cidx * kChunk;
  for (int idx = lane; idx < kChunk * D; idx += 32) {
    const int j = idx / D, t = idx % D;
    ks[j * BT::KS + t] = ldf(k + (kv0 + j) * D + t);
  }
  for (int t = lane; t < D; t += 32) {
    lqw[t] = ldf(lq + unit * D + t);
    dkw[t] = dkp[unit * D + t];
    kpw[t] = kprime[unit * D + t];
  }
  __syncwarp();
  const float db = dbp[unit];
  float z0, z1, d0, d1;
  bwd_row_dots<D>(lqw, ks, z0, z1);
  bwd_row_dots<D>(dkw, ks, d0, d1);
  z0 *= tau;
  z1 *= tau;
  float c0 = 0.f;   // <dk', k'>
  for (int t = lane; t < D; t += 32) c0 = fmaf(dkw[t], kpw[t], c0);
  float m = fmaxf(z0, z1);
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    c0 += __shfl_xor_sync(0xffffffffu, c0, off);
  }
  const float e0 = expf(z0 - m), e1 = expf(z1 - m);
  float l = e0 + e1;
#pragma unroll
  for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  const float p0 = e0 / l, p1 = e1 / l;
  float zbar = p0 * z0 + p1 * z1;
#pragma unroll
  for (int off = 16; off; off >>= 1) zbar += __shfl_xor_sync(0xffffffffu, zbar, off);
  const float dz0 = p0 * (d0 - c0) - db * p0 * (z0 - zbar);
  const float dz1 = p1 * (d1 - c0) - db * p1 * (z1 - zbar);
  float acc[D / 32];
  bwd_row_combine<D>(tau * dz0, tau * dz1, ks, acc);
#pragma unroll
  for (int e = 0; e < D / 32; ++e) dlq[unit * D + lane + 32 * e] = acc[e];
  // the keys' share: each key of the chunk belongs to this warp alone
  for (int j = 0; j < kChunk; ++j) {
    const float a = __shfl_sync(0xffffffffu, j < 32 ? tau * dz0 : tau * dz1, j & 31);
    const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
      const int t = lane + 32 * e;
      dk[(kv0 + j) * D + t] += a * lqw[t] + pj * dkw[t];
    }
  }
}

}  // namespace hils
