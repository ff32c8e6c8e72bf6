// Backward of the selected chunks on tensor cores (bf16, mma.sync).
//
// AI Trends article, section "방법론" (Methodology): the chunk score s^ is
// part of the forward attention, so the gradient reaches the queries, keys,
// values and (through k', b') the landmark queries.  Per pair (row i, kept
// chunk c) with g = dL/dO_i, Dg = <g, O_i>, a = exp(s^ - M') and p the softmax
// of the row over the chunk's 64 keys:
//   X = <g, o_c> = sum_j p_j <g, v_j>
//   dz_j = tau a p_j (<g, v_j> - X),  du = a (X - Dg)
//   dq_i += sum_j dz_j k_j + tau du k'_c
//   dk_j += sum_i dz_j q_i,  dv_j += sum_i a p_j g_i
//   dk'_c += tau du q_i,  db'_c += du
// The same arithmetic as bwd_chunk_kernel (CUDA cores), tile by tile of the
// forward's chunk-centric index (up to 128 pairs of one chunk).  The five
// products run as m16n8k16 bf16 MMAs with fp32 accumulators:
//   S = Q K^T and G = dO V^T   (warp w: the tile's rows 16w .. 16w+15)
//   dQ = dZ K                  (dZ straight from the S accumulators, bf16)
//   dK = dZ^T Q, dV = (aP)^T dO (warp w: dK or dV of keys 16(w%4) .. +15,
//                               summed over the tile's rows)
// dZ and aP enter the MMAs rounded to bf16 (the inputs are bf16); every sum
// is fp32.  Rows of a tile are gathered into shared memory by 16-byte
// cp.async copies (the next tile's keys, values and row list while the
// current tile's dK, dV products run); every row-major bf16 tile keeps its 16-byte blocks of row r
// at block ^ (r mod 8), so that the eight rows an ldmatrix reads hit
// distinct banks.  No TMEM and no mbarrier: the only waits are block
// barriers that every thread reaches.
#pragma once
#include "backward.cuh"

namespace hils {

// ldmatrix of four 8x8 b16 matrices (lane i gives row i % 8 of matrix i / 8),
// plain or transposed, and mma m16n8k16 bf16 -> fp32.
__device__ __forceinline__ void bm_ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void bm_ldsm4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void bm_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
               "{%0, %1, %2, %3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t bm_pack(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// Two rows' fragment pairs -> one 16-byte atomic per lane: lanes tq and
// tq ^ 1 hold dims t0, t0+1 and t0+2, t0+3 (t0 = 4 (tq / 2) + 8n) of rows ra
// and rb; after one exchange the even lane adds row ra's four dims and the
// odd lane row rb's (16-byte aligned: t0 is a multiple of 4).
__device__ __forceinline__ void bm_red4(float* base_a, float* base_b, int t0, int tq, float a0, float a1,
                                        float b0, float b1, bool live_a, bool live_b) {
  const bool even = (tq & 1) == 0;
  const float x = __shfl_xor_sync(0xffffffffu, even ? b0 : a0, 1);
  const float y = __shfl_xor_sync(0xffffffffu, even ? b1 : a1, 1);
  if (even) {
    if (live_a) atomicAdd(reinterpret_cast<float4*>(base_a + t0), make_float4(a0, a1, x, y));
  } else {
    if (live_b) atomicAdd(reinterpret_cast<float4*>(base_b + t0 - 2), make_float4(x, y, b0, b1));
  }
}

__device__ __forceinline__ void bm_cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <int D>
struct BwdMma {
  static constexpr int M = kCcTileRows;          // pairs per tile (128)
  static constexpr int RB = D * 2;               // bytes per bf16 row of d
  static constexpr int NB = RB / 16;             // 16-byte blocks per row
  static constexpr int THREADS = 256;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + kChunk * RB;
  static constexpr uint32_t OFF_Q = OFF_V + kChunk * RB;
  static constexpr uint32_t OFF_G = OFF_Q + M * RB;
  static constexpr uint32_t OFF_DZ = OFF_G + M * RB;       // [M][64] bf16
  static constexpr uint32_t OFF_PW = OFF_DZ + M * 128;     // [M][64] bf16
  static constexpr uint32_t OFF_DU = OFF_PW + M * 128;     // [M] fp32
  static constexpr uint32_t OFF_KP = OFF_DU + M * 4;       // [D] fp32, the chunk's k'
  static constexpr uint32_t OFF_DKP = OFF_KP + D * 4;      // [D] fp32: tau sum du q over the tile, then sum du
  static constexpr uint32_t OFF_ROWS = OFF_DKP + D * 4 + 16;  // [M] int32: the tile's pair rows
  // d = 128 (one CTA per SM, shared memory to spare): a second query and
  // output-gradient row buffer, so that the next tile's rows are gathered
  // while the current tile's dK, dV products still read the first
  static constexpr bool DB = D == 128;
  static constexpr uint32_t OFF_Q2 = (OFF_ROWS + M * 4 + 127u) & ~127u;
  static constexpr uint32_t OFF_G2 = OFF_Q2 + M * RB;
  static constexpr uint32_t SMEM = DB ? OFF_G2 + M * RB : OFF_ROWS + M * 4;
  static constexpr int CTAS_PER_SM = D == 64 ? 2 : 1;
};

// byte offset of 16-byte block `blk` of row r in a row-major tile of `rb`-byte rows
__device__ __forceinline__ uint32_t bm_at(int r, int blk, int rb) {
  return uint32_t(r * rb + ((blk ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(BwdMma<D>::THREADS, BwdMma<D>::CTAS_PER_SM)
bwd_chunk_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ d_o,
                     const float* __restrict__ kprime, const float* __restrict__ dvec,
                     const int32_t* __restrict__ tile_start, const int4* __restrict__ items,
                     const int2* __restrict__ e_pair, const CcDims c, float* __restrict__ dq,
                     float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dkp,
                     float* __restrict__ dbp) {
  using C = BwdMma<D>;
  extern __shared__ __align__(16) uint8_t bsm[];
  const uint32_t sbase = uint32_t(__cvta_generic_to_shared(bsm));
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sQ = sbase + C::OFF_Q, sG = sbase + C::OFF_G;
  const uint32_t sDZ = sbase + C::OFF_DZ, sPW = sbase + C::OFF_PW;
  float* s_du = reinterpret_cast<float*>(bsm + C::OFF_DU);
  float* s_kp = reinterpret_cast<float*>(bsm + C::OFF_KP);
  float* s_dkp = reinterpret_cast<float*>(bsm + C::OFF_DKP);   // [D], then [D] the tile's sum of du
  int32_t* s_rows = reinterpret_cast<int32_t*>(bsm + C::OFF_ROWS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;   // fragment row group and column pair
  const int mi = lane >> 3, ri = lane & 7;   // ldmatrix: the matrix and row this lane addresses
  const float tau = c.tau;
  const int n_all = tile_start[c.n_keys];
  // a tile's keys, values and k' and its pair rows, staged ahead: the first
  // tile's before the loop, the next tile's while the current one's dK, dV
  // products run (they read neither K, V, k' nor the row list)
  auto stage = [&](int t) {
    const int4 st = items[t];
    const int64_t kvr = st.y;
    for (int u = tid; u < 2 * kChunk * C::NB; u += C::THREADS) {
      const int which = u / (kChunk * C::NB), rem = u % (kChunk * C::NB);
      const int r = rem / C::NB, blk = rem % C::NB;
      bm_cp16((which ? sV : sK) + bm_at(r, blk, C::RB), (which ? v : k) + (kvr + r) * D + blk * 8);
    }
    for (int r = tid; r < st.z; r += C::THREADS) s_rows[r] = e_pair[st.x + r].x;
    const int64_t sbh = kvr / c.n_tok, sch = (kvr % c.n_tok) / kChunk;
    for (int d2 = tid; d2 < D; d2 += C::THREADS) s_kp[d2] = kprime[(sbh * c.nc + sch) * D + d2];
  };
  // DB: the pairs' query and output-gradient rows of tile t into the buffer
  // pair (qb, gb), row ids read from the index (rows past the pairs zeroed)
  auto gather = [&](int t, uint32_t qb, uint32_t gb) {
    const int4 gt = items[t];
    const int gn = gt.z, gn16 = (gn + 15) & ~15;
    for (int u = tid; u < 2 * gn16 * C::NB; u += C::THREADS) {
      const int which = u / (gn16 * C::NB), rem = u % (gn16 * C::NB);
      const int r = rem / C::NB, blk = rem % C::NB;
      const uint32_t dst = (which ? gb : qb) + bm_at(r, blk, C::RB);
      if (r < gn) {
        bm_cp16(dst, (which ? d_o : q) + int64_t(e_pair[gt.x + r].x) * D + blk * 8);
      } else {
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
      }
    }
  };
  const uint32_t sQ2 = sbase + C::OFF_Q2, sG2 = sbase + C::OFF_G2;
  if (int(blockIdx.x) < n_all) {
    stage(blockIdx.x);
    if constexpr (C::DB) gather(blockIdx.x, sQ, sG);
  }
  int pb = 0;   // DB: the buffer pair of the current tile
  for (int tile = blockIdx.x; tile < n_all; tile += gridDim.x, pb ^= 1) {
    const int4 it = items[tile];   // first entry, K/V row, pair count
    const int64_t first = it.x, kvrow = it.y;
    const int n = it.z;
    const int64_t bh = kvrow / c.n_tok, chunk = (kvrow % c.n_tok) / kChunk;
    const int n16 = (n + 15) & ~15;   // rows the products read (the rest of the last 16 zeroed)
    const uint32_t cQ = (C::DB && pb) ? sQ2 : sQ, cG = (C::DB && pb) ? sG2 : sG;   // this tile's rows
    __syncthreads();   // the previous tile's shared memory is no longer read; this tile's rows are staged
    if constexpr (!C::DB) {
      // ---- the pairs' query and output-gradient rows (the keys and values are on their way)
      for (int u = tid; u < 2 * n16 * C::NB; u += C::THREADS) {
        const int which = u / (n16 * C::NB), rem = u % (n16 * C::NB);
        const int r = rem / C::NB, blk = rem % C::NB;
        const uint32_t dst = (which ? sG : sQ) + bm_at(r, blk, C::RB);
        if (r < n) {
          bm_cp16(dst, (which ? d_o : q) + int64_t(s_rows[r]) * D + blk * 8);
        } else {
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
        }
      }
    }
    for (int t = tid; t < D; t += C::THREADS) s_dkp[t] = 0.f;
    if (tid == 0) s_dkp[D] = 0.f;
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    // ---- per warp, rows rb .. rb+15: S, G, the softmax, dZ, aP, du, dQ
    const int rb = warp * 16;
    if (rb < n) {
      float sacc[8][4], gacc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = gacc[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t aq[4], ag[4];
        const int ar = rb + ri + ((mi & 1) << 3), ablk = 2 * kk + (mi >> 1);
        bm_ldsm4(cQ + bm_at(ar, ablk, C::RB), aq);
        bm_ldsm4(cG + bm_at(ar, ablk, C::RB), ag);
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          // keys 8nt .. 8nt+15 as the B operand (k = dims): b0, b1 of n-tiles nt and nt+1
          uint32_t bk[4], bv[4];
          const int key = 8 * nt + ri + ((mi >> 1) << 3), bblk = 2 * kk + (mi & 1);
          bm_ldsm4(sK + bm_at(key, bblk, C::RB), bk);
          bm_ldsm4(sV + bm_at(key, bblk, C::RB), bv);
          bm_mma(sacc[nt], aq, bk[0], bk[1]);
          bm_mma(sacc[nt + 1], aq, bk[2], bk[3]);
          bm_mma(gacc[nt], ag, bv[0], bv[1]);
          bm_mma(gacc[nt + 1], ag, bv[2], bv[3]);
        }
      }
      // accumulators: [nt][0..1] row rb+gq, keys 8nt+2tq, +1; [nt][2..3] row rb+gq+8
      const int r0 = rb + gq, r1 = rb + gq + 8;
      const bool live0 = r0 < n, live1 = r1 < n;
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        m0 = fmaxf(m0, fmaxf(sacc[nt][0], sacc[nt][1]));
        m1 = fmaxf(m1, fmaxf(sacc[nt][2], sacc[nt][3]));
      }
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
      }
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        sacc[nt][0] = expf(tau * (sacc[nt][0] - m0));
        sacc[nt][1] = expf(tau * (sacc[nt][1] - m0));
        sacc[nt][2] = expf(tau * (sacc[nt][2] - m1));
        sacc[nt][3] = expf(tau * (sacc[nt][3] - m1));
        l0 += sacc[nt][0] + sacc[nt][1];
        l1 += sacc[nt][2] + sacc[nt][3];
      }
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      const float il0 = 1.f / l0, il1 = 1.f / l1;
      float x0 = 0.f, x1 = 0.f;   // X = sum_j p_j <g, v_j>
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        sacc[nt][0] *= il0;
        sacc[nt][1] *= il0;
        sacc[nt][2] *= il1;
        sacc[nt][3] *= il1;
        x0 = fmaf(sacc[nt][0], gacc[nt][0], fmaf(sacc[nt][1], gacc[nt][1], x0));
        x1 = fmaf(sacc[nt][2], gacc[nt][2], fmaf(sacc[nt][3], gacc[nt][3], x1));
      }
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        x0 += __shfl_xor_sync(0xffffffffu, x0, off);
        x1 += __shfl_xor_sync(0xffffffffu, x1, off);
      }
      int64_t grow0 = 0, grow1 = 0;
      float a0 = 0.f, a1 = 0.f, du0 = 0.f, du1 = 0.f;
      if (live0) {
        const int2 ep = e_pair[first + r0];
        grow0 = ep.x;
        a0 = expf(__int_as_float(ep.y));   // exp(s^ - M')
        du0 = a0 * (x0 - dvec[grow0]);
      }
      if (live1) {
        const int2 ep = e_pair[first + r1];
        grow1 = ep.x;
        a1 = expf(__int_as_float(ep.y));
        du1 = a1 * (x1 - dvec[grow1]);
      }
      // dZ (tau a p (G - X)) into the S accumulators, aP into G's; both to
      // shared memory as bf16 rows for dK, dV (rows past the pairs: zeros)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p00 = sacc[nt][0], p01 = sacc[nt][1], p10 = sacc[nt][2], p11 = sacc[nt][3];
        sacc[nt][0] = tau * a0 * p00 * (gacc[nt][0] - x0);
        sacc[nt][1] = tau * a0 * p01 * (gacc[nt][1] - x0);
        sacc[nt][2] = tau * a1 * p10 * (gacc[nt][2] - x1);
        sacc[nt][3] = tau * a1 * p11 * (gacc[nt][3] - x1);
        gacc[nt][0] = a0 * p00;
        gacc[nt][1] = a0 * p01;
        gacc[nt][2] = a1 * p10;
        gacc[nt][3] = a1 * p11;
        const uint32_t o0 = bm_at(r0, nt, 128) + 4 * tq, o1 = bm_at(r1, nt, 128) + 4 * tq;
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sDZ + o0), "r"(bm_pack(sacc[nt][0], sacc[nt][1])) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sDZ + o1), "r"(bm_pack(sacc[nt][2], sacc[nt][3])) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sPW + o0), "r"(bm_pack(gacc[nt][0], gacc[nt][1])) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sPW + o1), "r"(bm_pack(gacc[nt][2], gacc[nt][3])) : "memory");
      }
      if (tq == 0) {
        s_du[r0] = du0;
        s_du[r1] = du1;
      }
      __syncwarp();
      // this warp's share of dk'_c (tau sum du q over its 16 rows) and db'_c
      {
        float dsum = tq == 0 ? du0 + du1 : 0.f;
#pragma unroll
        for (int off = 16; off; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
        if (lane == 0) atomicAdd(s_dkp + D, dsum);
#pragma unroll
        for (int e = 0; e < D / 32; ++e) {
          const int t = lane + 32 * e;
          float acc_t = 0.f;
#pragma unroll 4
          for (int r = 0; r < 16; ++r) {
            unsigned short hb;
            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(hb) : "r"(cQ + bm_at(rb + r, t >> 3, C::RB) + uint32_t((t & 7) * 2)));
            acc_t = fmaf(s_du[rb + r], __uint_as_float(uint32_t(hb) << 16), acc_t);
          }
          atomicAdd(s_dkp + t, tau * acc_t);
        }
      }
      // dQ = dZ K (k = keys: the A fragments are the dZ accumulators), plus tau du k'
#pragma unroll
      for (int nd = 0; nd < D / 8; nd += 2) {
        float qa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t a[4] = {bm_pack(sacc[2 * kk][0], sacc[2 * kk][1]), bm_pack(sacc[2 * kk][2], sacc[2 * kk][3]),
                                 bm_pack(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]),
                                 bm_pack(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3])};
          // keys 16kk .. 16kk+15 as the B operand rows (k = keys), dims 8nd .. 8nd+15
          uint32_t b[4];
          const int key = 16 * kk + ri + ((mi & 1) << 3), bblk = nd + (mi >> 1);
          bm_ldsm4_t(sK + bm_at(key, bblk, C::RB), b);
          bm_mma(qa[0], a, b[0], b[1]);
          bm_mma(qa[1], a, b[2], b[3]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int t0 = 8 * (nd + h) + 2 * tq;
          bm_red4(dq + grow0 * D, dq + grow1 * D, t0, tq, qa[h][0] + tau * du0 * s_kp[t0],
                  qa[h][1] + tau * du0 * s_kp[t0 + 1], qa[h][2] + tau * du1 * s_kp[t0],
                  qa[h][3] + tau * du1 * s_kp[t0 + 1], live0, live1);
        }
      }
    }
    __syncthreads();
    // the next tile's keys, values, k' and rows (DB: and its query and
    // output-gradient rows, into the other buffer pair) start while dK, dV run
    if (tile + int(gridDim.x) < n_all) {
      stage(tile + int(gridDim.x));
      if constexpr (C::DB) gather(tile + int(gridDim.x), pb ? sQ : sQ2, pb ? sG : sG2);
    }
    // ---- dK = dZ^T Q (warps 0-3) and dV = (aP)^T dO (warps 4-7), keys 16 (w % 4) .. +15
    {
      const uint32_t sA = warp < 4 ? sDZ : sPW, sB = warp < 4 ? cQ : cG;
      float* gout = warp < 4 ? dk : dv;
      const int mt = warp & 3;
      float acc[D / 8][4];
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd) acc[nd][0] = acc[nd][1] = acc[nd][2] = acc[nd][3] = 0.f;
      for (int kk = 0; kk < n16 / 16; ++kk) {
        // A = X^T (m = keys, k = rows) from the row-major [row][key] tile, transposed
        uint32_t a[4];
        const int ar = 16 * kk + ri + ((mi >> 1) << 3), ablk = 2 * mt + (mi & 1);
        bm_ldsm4_t(sA + bm_at(ar, ablk, 128), a);
#pragma unroll
        for (int nd = 0; nd < D / 8; nd += 2) {
          // B = the rows (k) x dims (n) of Q or dO, transposed
          uint32_t b[4];
          const int br = 16 * kk + ri + ((mi & 1) << 3), bblk = nd + (mi >> 1);
          bm_ldsm4_t(sB + bm_at(br, bblk, C::RB), b);
          bm_mma(acc[nd], a, b[0], b[1]);
          bm_mma(acc[nd + 1], a, b[2], b[3]);
        }
      }
      // acc[nd]: (key 16mt+gq, dims 8nd+2tq, +1), then (key 16mt+gq+8, same dims)
      const int64_t k0 = kvrow + 16 * mt + gq;
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd)
        bm_red4(gout + k0 * D, gout + (k0 + 8) * D, 8 * nd + 2 * tq, tq, acc[nd][0], acc[nd][1], acc[nd][2],
                acc[nd][3], true, true);
    }
    // ---- dk'_c += tau sum_i du_i q_i, db'_c += sum_i du_i (the warps' shares, summed)
    for (int t = tid; t < D; t += C::THREADS) atomicAdd(dkp + (bh * c.nc + chunk) * D + t, s_dkp[t]);
    if (tid == C::THREADS - 1) atomicAdd(dbp + bh * c.nc + chunk, s_dkp[D]);
  }
}

// The window branch on tensor cores: one CTA per (chunk o of positions,
// (b, hq)), the 64 rows at positions 64 o .. 64 o + 63 against the key
// chunks o - wm1 .. o (the last under the causal mask), with weights
// P = exp(tau s - M'):
//   dz_j = tau P_j (<g, v_j> - Dg),  dq = sum_j dz_j k_j (written: this
//   kernel runs first), dk_j += sum_i dz_j q_i, dv_j += sum_i P_j g_i.
// Warps 0-3 take 16 rows each for S, G, the weights and dQ (kept in
// registers across the window's chunks); all eight warps take dK or dV of
// 16 keys of each chunk, as in bwd_chunk_mma_kernel.
template <int D>
struct BwdWinMma {
  static constexpr int RB = D * 2;
  static constexpr int NB = RB / 16;
  static constexpr int THREADS = 256;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + kChunk * RB;
  static constexpr uint32_t OFF_Q = OFF_V + kChunk * RB;
  static constexpr uint32_t OFF_G = OFF_Q + kChunk * RB;
  static constexpr uint32_t OFF_DZ = OFF_G + kChunk * RB;   // [64][64] bf16
  static constexpr uint32_t OFF_PW = OFF_DZ + kChunk * 128;
  static constexpr uint32_t SMEM = OFF_PW + kChunk * 128;
  static constexpr int CTAS_PER_SM = D == 64 ? 2 : 1;
};

template <int D>
__global__ void __launch_bounds__(BwdWinMma<D>::THREADS, BwdWinMma<D>::CTAS_PER_SM)
bwd_window_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ d_o,
                      const float* __restrict__ rowstat, const float* __restrict__ dvec, int64_t n_tok, int Hq,
                      int G, int Hkv, int wm1, float tau, float* __restrict__ dq, float* __restrict__ dk,
                      float* __restrict__ dv) {
  using C = BwdWinMma<D>;
  extern __shared__ __align__(16) uint8_t bsm[];
  const uint32_t sbase = uint32_t(__cvta_generic_to_shared(bsm));
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sQ = sbase + C::OFF_Q, sG = sbase + C::OFF_G;
  const uint32_t sDZ = sbase + C::OFF_DZ, sPW = sbase + C::OFF_PW;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int mi = lane >> 3, ri = lane & 7;
  const int64_t own = blockIdx.x;
  const int bhq = int(blockIdx.y), b = bhq / Hq, hq = bhq % Hq, h = hq / G;
  const int64_t p0 = own * kChunk;
  const int64_t row0 = int64_t(bhq) * n_tok + p0;
  const int64_t kv0 = (int64_t(b) * Hkv + h) * n_tok;
  // the 64 rows' queries and output gradients (contiguous rows)
  for (int u = tid; u < 2 * kChunk * C::NB; u += C::THREADS) {
    const int which = u / (kChunk * C::NB), rem = u % (kChunk * C::NB);
    const int r = rem / C::NB, blk = rem % C::NB;
    bm_cp16((which ? sG : sQ) + bm_at(r, blk, C::RB), (which ? d_o : q) + (row0 + r) * D + blk * 8);
  }
  const int rb = warp * 16;
  const int r0 = rb + gq, r1 = rb + gq + 8;   // this lane's rows (warps 0-3)
  float mp0 = 0.f, mp1 = 0.f, dg0 = 0.f, dg1 = 0.f;
  if (warp < 4) {
    mp0 = rowstat[row0 + r0];
    mp1 = rowstat[row0 + r1];
    dg0 = dvec[row0 + r0];
    dg1 = dvec[row0 + r1];
  }
  float qacc[D / 8][4];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) qacc[nd][0] = qacc[nd][1] = qacc[nd][2] = qacc[nd][3] = 0.f;
  const int64_t c_lo = own - wm1 > 0 ? own - wm1 : 0;
  for (int64_t cj = c_lo; cj <= own; ++cj) {
    __syncthreads();   // the previous chunk's K, V, dZ, aP are no longer read
    for (int u = tid; u < 2 * kChunk * C::NB; u += C::THREADS) {
      const int which = u / (kChunk * C::NB), rem = u % (kChunk * C::NB);
      const int r = rem / C::NB, blk = rem % C::NB;
      bm_cp16((which ? sV : sK) + bm_at(r, blk, C::RB), (which ? v : k) + (kv0 + cj * kChunk + r) * D + blk * 8);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (warp < 4) {
      float sacc[8][4], gacc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = gacc[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t aq[4], ag[4];
        const int ar = rb + ri + ((mi & 1) << 3), ablk = 2 * kk + (mi >> 1);
        bm_ldsm4(sQ + bm_at(ar, ablk, C::RB), aq);
        bm_ldsm4(sG + bm_at(ar, ablk, C::RB), ag);
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          uint32_t bk[4], bv[4];
          const int key = 8 * nt + ri + ((mi >> 1) << 3), bblk = 2 * kk + (mi & 1);
          bm_ldsm4(sK + bm_at(key, bblk, C::RB), bk);
          bm_ldsm4(sV + bm_at(key, bblk, C::RB), bv);
          bm_mma(sacc[nt], aq, bk[0], bk[1]);
          bm_mma(sacc[nt + 1], aq, bk[2], bk[3]);
          bm_mma(gacc[nt], ag, bv[0], bv[1]);
          bm_mma(gacc[nt + 1], ag, bv[2], bv[3]);
        }
      }
      // P (causal in the own chunk), dZ into sacc, P into gacc; both to shared memory
      const int64_t kbase = cj * kChunk;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t key = kbase + 8 * nt + 2 * tq + (e & 1);
          const int64_t pos = p0 + (e < 2 ? r0 : r1);
          const float mp = e < 2 ? mp0 : mp1, dg = e < 2 ? dg0 : dg1;
          const float P = key <= pos ? expf(tau * sacc[nt][e] - mp) : 0.f;
          sacc[nt][e] = tau * P * (gacc[nt][e] - dg);
          gacc[nt][e] = P;
        }
        const uint32_t o0 = bm_at(r0, nt, 128) + 4 * tq, o1 = bm_at(r1, nt, 128) + 4 * tq;
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sDZ + o0), "r"(bm_pack(sacc[nt][0], sacc[nt][1])) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sDZ + o1), "r"(bm_pack(sacc[nt][2], sacc[nt][3])) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sPW + o0), "r"(bm_pack(gacc[nt][0], gacc[nt][1])) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sPW + o1), "r"(bm_pack(gacc[nt][2], gacc[nt][3])) : "memory");
      }
      // dQ += dZ K
#pragma unroll
      for (int nd = 0; nd < D / 8; nd += 2) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t a[4] = {bm_pack(sacc[2 * kk][0], sacc[2 * kk][1]), bm_pack(sacc[2 * kk][2], sacc[2 * kk][3]),
                                 bm_pack(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]),
                                 bm_pack(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3])};
          uint32_t bq[4];
          const int key = 16 * kk + ri + ((mi & 1) << 3), bblk = nd + (mi >> 1);
          bm_ldsm4_t(sK + bm_at(key, bblk, C::RB), bq);
          bm_mma(qacc[nd], a, bq[0], bq[1]);
          bm_mma(qacc[nd + 1], a, bq[2], bq[3]);
        }
      }
    }
    __syncthreads();
    // dK = dZ^T Q (warps 0-3), dV = P^T dO (warps 4-7) for this chunk's keys 16 (w % 4) .. +15
    {
      const uint32_t sA = warp < 4 ? sDZ : sPW, sB = warp < 4 ? sQ : sG;
      float* gout = warp < 4 ? dk : dv;
      const int mt = warp & 3;
      float acc[D / 8][4];
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd) acc[nd][0] = acc[nd][1] = acc[nd][2] = acc[nd][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kChunk / 16; ++kk) {
        uint32_t a[4];
        const int ar = 16 * kk + ri + ((mi >> 1) << 3), ablk = 2 * mt + (mi & 1);
        bm_ldsm4_t(sA + bm_at(ar, ablk, 128), a);
#pragma unroll
        for (int nd = 0; nd < D / 8; nd += 2) {
          uint32_t bb[4];
          const int br = 16 * kk + ri + ((mi & 1) << 3), bblk = nd + (mi >> 1);
          bm_ldsm4_t(sB + bm_at(br, bblk, C::RB), bb);
          bm_mma(acc[nd], a, bb[0], bb[1]);
          bm_mma(acc[nd + 1], a, bb[2], bb[3]);
        }
      }
      const int64_t k0 = kv0 + cj * kChunk + 16 * mt + gq;
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd)
        bm_red4(gout + k0 * D, gout + (k0 + 8) * D, 8 * nd + 2 * tq, tq, acc[nd][0], acc[nd][1], acc[nd][2],
                acc[nd][3], true, true);
    }
  }
  // the window kernel runs first: dq is written here, the selected chunks add to it
  if (warp < 4) {
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      const int t0 = 8 * nd + 2 * tq;
      *reinterpret_cast<float2*>(dq + (row0 + r0) * D + t0) = make_float2(qacc[nd][0], qacc[nd][1]);
      *reinterpret_cast<float2*>(dq + (row0 + r1) * D + t0) = make_float2(qacc[nd][2], qacc[nd][3]);
    }
  }
}

}  // namespace hils
