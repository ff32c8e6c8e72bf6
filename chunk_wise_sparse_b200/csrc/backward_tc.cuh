// Backward, selected chunks, on tensor cores (bf16).
//
// The same quantities as bwd_chunk_kernel (see backward.cuh) for one tile of
// up to 128 (row, slot) pairs of one chunk c, with the five contractions on
// tcgen05 (fp32 accumulators in TMEM):
//   S    = Q K_c^T         [128 x 64]   the logits again
//   dP   = dO V_c^T        [128 x 64]   <dO_i, v_j>
//   (one thread per pair: p = softmax(tau S), X = sum p dP, a = exp(s^ - M'),
//    dZ = tau a p (dP - X) and aP in bf16, du = a (X - <dO, O>))
//   dQ   = dZ K_c          [128 x d]    added to the pairs' rows of dq
//   dK^T = Q^T dZ          [d x 64]     added to the chunk's rows of dk
//   dV^T = dO^T (aP)       [d x 64]     added to the chunk's rows of dv
// The Q and dO tiles (pairs x d, d contiguous) serve both as K-major A
// operands (S, dP) and, read transposed, as MN-major A operands (dK^T, dV^T);
// dZ and aP (pairs x 64 keys) are K-major A (dQ) and MN-major B operands;
// K_c (keys x d) is K-major B for S and MN-major B for dQ.  With d = 64 the
// transposed A has only 64 of its 128 rows: the other 64 come from a zeroed
// tile and give zero rows in TMEM.  dk'_c += tau sum_i du_i q_i and
// db'_c += sum_i du_i come from the Q tile in shared memory (one thread per
// dim).
//
// Persistent over the index's tiles, one tile at a time per CTA; 128 threads:
// thread 0 issues the copies and the MMAs, every thread owns one pair row
// (TMEM lane) in the softmax and one dim in the epilogues.  Every wait is
// bounded; a time-out records HILS_ERR_DEVICE_TIMEOUT and the kernel drains
// and returns.
#pragma once
#include "backward.cuh"

namespace hils {

// global[addr] += v in L2, no return value
__device__ __forceinline__ void red_add_f32(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

template <int D>
struct BwdTc {
  static constexpr int M = 128;
  static constexpr int KATOMS = D / 64;
  static constexpr uint32_t ROW_ATOM = M * 128;        // 128 rows x 64 elements
  static constexpr uint32_t KV_ATOM = kChunk * 128;    // 64 rows x 64 elements
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_G = OFF_Q + KATOMS * ROW_ATOM;    // dO rows
  static constexpr uint32_t OFF_K = OFF_G + KATOMS * ROW_ATOM;
  static constexpr uint32_t OFF_V = OFF_K + KATOMS * KV_ATOM;
  static constexpr uint32_t OFF_DZ = OFF_V + KATOMS * KV_ATOM;    // 128 pairs x 64 keys bf16
  static constexpr uint32_t OFF_PW = OFF_DZ + ROW_ATOM;
  static constexpr uint32_t OFF_ZERO = OFF_PW + ROW_ATOM;         // d = 64: the zero half of the transposed A
  static constexpr uint32_t ZERO_BYTES = D == 64 ? ROW_ATOM : 0u;
  static constexpr uint32_t OFF_META = OFF_ZERO + ZERO_BYTES;     // rows[128], fac[128], du[128], kp[D]
  static constexpr uint32_t OFF_BAR = OFF_META + (3 * M + D) * 4;
  static constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
  static constexpr uint32_t TX_BYTES = 2 * KATOMS * ROW_ATOM + 2 * KATOMS * KV_ATOM;
  // TMEM columns: [0, 64) S then dK^T, [64, 128) dP then dV^T, [128, 128 + d) dQ
  static constexpr uint32_t T_S = 0, T_P = 64, T_Q = 128;
  static constexpr uint32_t TMEM_COLS = 256;
  // more CTAs than 512 / TMEM_COLS per SM (228 KB of shared memory, 1 KB
  // reserved per CTA) could make a tcgen05.alloc wait for columns that a
  // co-resident CTA never frees
  static_assert((512 / TMEM_COLS + 1) * (SMEM + 1024) > 233472u, "TMEM never oversubscribed");
  static constexpr uint32_t IDESC_S = sm100::idesc_bf16(M, kChunk);
  static constexpr uint32_t IDESC_Q = sm100::idesc_bf16(M, D) | (1u << 16);                  // B MN-major
  static constexpr uint32_t IDESC_T = sm100::idesc_bf16(M, kChunk) | (1u << 15) | (1u << 16);   // A, B MN-major
  static constexpr int THREADS = 128;
};

template <int D>
__global__ void __launch_bounds__(128)
bwd_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const float* __restrict__ kprime, const float* __restrict__ dvec,
                    const int32_t* __restrict__ tile_start, const int4* __restrict__ items,
                    const int2* __restrict__ e_pair, const CcDims c,
                    float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dkp,
                    float* __restrict__ dbp) {
  using C = BwdTc<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  uint64_t* ld_bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* mma_bar = ld_bar + 1;
  uint64_t* done_bar = ld_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 28);
  int32_t* s_rows = reinterpret_cast<int32_t*>(smem + C::OFF_META);
  float* s_fac = reinterpret_cast<float*>(s_rows + C::M);
  float* s_du = s_fac + C::M;
  float* s_kp = s_du + C::M;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float tau = c.tau;

  if (tid == 0) {
    mbar_init(ld_bar, 1);
    mbar_init(mma_bar, 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (C::ZERO_BYTES) {
    for (uint32_t i = tid; i < C::ZERO_BYTES / 16; i += C::THREADS)
      reinterpret_cast<uint4*>(smem + C::OFF_ZERO)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_lane = tmem + (uint32_t(warp * 32) << 16);
  const int n_all = tile_start[c.n_keys];
  bool ok = true;
  int it = 0;
  for (int tile = blockIdx.x; tile < n_all && ok; tile += gridDim.x, ++it) {
    const int4 rec = items[tile];   // first entry, K/V row, pair count
    const int64_t first = rec.x, kvrow = rec.y;
    const int n = rec.z;
    const int64_t bh = kvrow / c.n_tok, chunk = (kvrow % c.n_tok) / kChunk;
    // the tile's pair rows (entries are padded with valid rows past the end)
    const int2 ep = e_pair[first + tid];
    s_rows[tid] = ep.x;
    s_fac[tid] = __int_as_float(ep.y);
    for (int t = tid; t < D; t += C::THREADS) s_kp[t] = kprime[(bh * c.nc + chunk) * D + t];
    __syncthreads();
    if (tid == 0) {
      mbar_arrive_expect_tx(ld_bar, C::TX_BYTES);
#pragma unroll
      for (int a = 0; a < C::KATOMS; ++a) {
        tma_load_2d(smem + C::OFF_K + a * C::KV_ATOM, &tm_k, ld_bar, a * 64, int(kvrow));
        tma_load_2d(smem + C::OFF_V + a * C::KV_ATOM, &tm_v, ld_bar, a * 64, int(kvrow));
      }
    }
    __syncthreads();   // expect_tx before any complete_tx of the gathers
    if (warp < 2) {
      // warp 0 gathers the Q rows, warp 1 the dO rows: lane l owns rows 4l .. 4l + 3
      const CUtensorMap* map = warp == 0 ? &tm_q : &tm_g;
      const uint32_t dst = smem_u32(smem + (warp == 0 ? C::OFF_Q : C::OFF_G)) + uint32_t(4 * lane) * 128;
#pragma unroll
      for (int a = 0; a < C::KATOMS; ++a)
        tma_gather4(dst + a * C::ROW_ATOM, map, ld_bar, a * 64, s_rows[4 * lane], s_rows[4 * lane + 1],
                    s_rows[4 * lane + 2], s_rows[4 * lane + 3]);
    }
    if (tid == 0) {
      ok = mbar_wait(ld_bar, it & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        const uint32_t sq = smem_u32(smem + C::OFF_Q), sg = smem_u32(smem + C::OFF_G);
        const uint32_t sk = smem_u32(smem + C::OFF_K), sv = smem_u32(smem + C::OFF_V);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offa = uint32_t((kk >> 2) * C::ROW_ATOM + (kk & 3) * 32);
          const uint32_t offb = uint32_t((kk >> 2) * C::KV_ATOM + (kk & 3) * 32);
          mma_bf16(tmem + C::T_S, desc_sw128(sq + offa), desc_sw128(sk + offb), C::IDESC_S, kk > 0 ? 1u : 0u);
          mma_bf16(tmem + C::T_P, desc_sw128(sg + offa), desc_sw128(sv + offb), C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(mma_bar);
      }
    }
    ok = __syncthreads_and(ok);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(mma_bar, 0, abort_flag));
    // ---- softmax of the pair row r = tid
    const int r = tid;
    const bool live = r < n;
    float du = 0.f;
    if (ok) {
      tc_fence_after();
      // the row's 64 logits and <dO, v_j> in two halves of 32 registers each
      float sa[32], sb[32], ga[32], gb[32];
      tmem_ld32(t_lane + C::T_S, sa);
      tmem_ld32(t_lane + C::T_S + 32, sb);
      tmem_ld32(t_lane + C::T_P, ga);
      tmem_ld32(t_lane + C::T_P + 32, gb);
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) m = fmaxf(m, fmaxf(sa[j], sb[j]));
      float l = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        sa[j] = expf(tau * (sa[j] - m));
        sb[j] = expf(tau * (sb[j] - m));
        l += sa[j] + sb[j];
      }
      const float inv = 1.f / l;
      float X = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        sa[j] *= inv;   // p_j
        sb[j] *= inv;
        X = fmaf(sa[j], ga[j], X);
        X = fmaf(sb[j], gb[j], X);
      }
      const float a = live ? expf(s_fac[r]) : 0.f;
      du = live ? a * (X - dvec[s_rows[r]]) : 0.f;
      uint8_t* zrow = smem + C::OFF_DZ + r * 128;
      uint8_t* prow = smem + C::OFF_PW + r * 128;
#pragma unroll
      for (int pc = 0; pc < 8; ++pc) {
        uint32_t wz[4], wp[4];
#pragma unroll
        for (int v2 = 0; v2 < 4; ++v2) {
          const int j = (pc & 3) * 8 + 2 * v2;   // within the half
          const float p0 = pc < 4 ? sa[j] : sb[j], p1 = pc < 4 ? sa[j + 1] : sb[j + 1];
          const float g0 = pc < 4 ? ga[j] : gb[j], g1 = pc < 4 ? ga[j + 1] : gb[j + 1];
          __nv_bfloat162 z2 = __floats2bfloat162_rn(tau * a * p0 * (g0 - X), tau * a * p1 * (g1 - X));
          __nv_bfloat162 p2 = __floats2bfloat162_rn(a * p0, a * p1);
          wz[v2] = *reinterpret_cast<uint32_t*>(&z2);
          wp[v2] = *reinterpret_cast<uint32_t*>(&p2);
        }
        const uint32_t off = uint32_t((pc ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(zrow + off) = make_uint4(wz[0], wz[1], wz[2], wz[3]);
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(wp[0], wp[1], wp[2], wp[3]);
      }
    }
    s_du[r] = du;
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (tid == 0 && ok) {
      tc_fence_after();
      const uint32_t sq = smem_u32(smem + C::OFF_Q), sg = smem_u32(smem + C::OFF_G);
      const uint32_t sk = smem_u32(smem + C::OFF_K);
      const uint32_t sz = smem_u32(smem + C::OFF_DZ), sp = smem_u32(smem + C::OFF_PW);
      // the second 64-row block of the transposed A: the Q / dO tile's second
      // atom (d = 128) or the zero tile (d = 64)
      const uint32_t lbo_q = C::ZERO_BYTES ? (smem_u32(smem + C::OFF_ZERO) - sq) : C::ROW_ATOM;
      const uint32_t lbo_g = C::ZERO_BYTES ? (smem_u32(smem + C::OFF_ZERO) - sg) : C::ROW_ATOM;
#pragma unroll
      for (int kk = 0; kk < kChunk / 16; ++kk)
        mma_bf16(tmem + C::T_Q, desc_sw128(sz + kk * 32), desc_sw128_mn(sk + kk * 2048, C::KV_ATOM), C::IDESC_Q,
                 kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < C::M / 16; ++kk) {
        mma_bf16(tmem + C::T_S, desc_sw128_mn(sq + kk * 2048, lbo_q), desc_sw128_mn(sz + kk * 2048, C::ROW_ATOM),
                 C::IDESC_T, kk > 0 ? 1u : 0u);
        mma_bf16(tmem + C::T_P, desc_sw128_mn(sg + kk * 2048, lbo_g), desc_sw128_mn(sp + kk * 2048, C::ROW_ATOM),
                 C::IDESC_T, kk > 0 ? 1u : 0u);
      }
      mma_commit(mma_bar);
    }
    // dk'_c and db'_c from the Q tile (one thread per dim), while the MMAs run
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(ld_bar, it & 1, abort_flag));   // the tiles, seen by this thread
    if (ok) {
      for (int t = tid; t < D; t += C::THREADS) {
        const uint8_t* col = smem + C::OFF_Q + (t >> 6) * C::ROW_ATOM + ((t & 63) & 7) * 2;
        const int pc = (t & 63) >> 3;
        float acc = 0.f;
        for (int rr = 0; rr < n; ++rr) {
          const __nv_bfloat16 x = *reinterpret_cast<const __nv_bfloat16*>(col + rr * 128 + ((pc ^ (rr & 7)) << 4));
          acc = fmaf(s_du[rr], __bfloat162float(x), acc);
        }
        red_add_f32(dkp + (bh * c.nc + chunk) * D + t, tau * acc);
      }
      float sd = du;
#pragma unroll
      for (int off = 16; off; off >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, off);
      if (lane == 0) red_add_f32(dbp + bh * c.nc + chunk, sd);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(mma_bar, 1, abort_flag));
    if (ok) {
      tc_fence_after();
      // dQ of pair row r (+ tau du k'_c, the chunk score's share).  The TMEM
      // loads are warp-collective: every lane issues them, only live rows add.
      float* dst = dq + int64_t(s_rows[r]) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float v[32];
        tmem_ld32(t_lane + C::T_Q + uint32_t(cc * 32), v);
        if (live) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const int t = cc * 32 + e;
            red_add_v4(dst + t, v[e] + tau * du * s_kp[t], v[e + 1] + tau * du * s_kp[t + 1],
                       v[e + 2] + tau * du * s_kp[t + 2], v[e + 3] + tau * du * s_kp[t + 3]);
          }
        }
      }
      // dK^T and dV^T: TMEM lane = dim (rows >= d of the d = 64 case are zero)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float kt[32], vt[32];
        tmem_ld32(t_lane + C::T_S + uint32_t(h * 32), kt);
        tmem_ld32(t_lane + C::T_P + uint32_t(h * 32), vt);
        if (tid < D) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            red_add_f32(dk + (kvrow + h * 32 + j) * D + tid, kt[j]);
            red_add_f32(dv + (kvrow + h * 32 + j) * D + tid, vt[j]);
          }
        }
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);   // the tile's shared memory and TMEM are free again
  }
  if (tid == 0 && !ok && it > 0) {
    // after a time-out: let the last tile's copies land and issued MMAs finish
    // before TMEM is freed (the loop counted that tile already)
    mbar_wait_drain(ld_bar, (it - 1) & 1);
    mma_commit(done_bar);
    mbar_wait_drain(done_bar, 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace hils
