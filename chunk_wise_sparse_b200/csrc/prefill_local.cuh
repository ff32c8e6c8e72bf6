// Kernel (c), local window branch on tensor cores (bf16, a window of more
// than one chunk).
//
// AI Trends article, section "기술 상세": beside the K selected chunks each
// query attends a sliding window of recent tokens.  Read chunk-aligned, the
// window of a row at position i in chunk o is the key range
// max(0, (o - wm1) C) .. i, one fusion branch whose score is its exact
// log-sum-exp (the own-chunk rule of the hotpaper.ai abstract and the
// aitrends.kr glossary entry "계층적 소프트맥스", widened to the window).
//
// This kernel takes the place of the own-chunk kernel when wm1 > 0; the
// count / scan / fill / attend / final kernels are unchanged, with the
// candidates of a row being the chunks before its window.
//
// One CTA per tile of 128 rows (P = 128/G consecutive positions of the G
// query heads of one kv head), the same tiles as the own-chunk kernel.  The
// tile's window keys are the chunks cw0 .. c_last (at most wm1 + 2 chunks).
// Two passes over them, one chunk (64 keys) per step:
//   pass 1: S = Q K_c^T on tcgen05; each row takes the max of its valid
//           scores (no exponentials);
//   pass 2: S again; P = exp(tau (s - m)) in bf16 into shared memory, the row
//           sum l in fp32, O += P V_c on tcgen05 (accumulated in TMEM).
// Then lse = tau m + log l, the fusion normaliser M' over the kept chunks and
// the window, and exp(tau m - M') O goes to the fp32 accumulator.
// Recomputing S costs a second Q K^T (small next to the exponentials) and
// avoids rescaling O, so each key takes one exponential.
//
// Warp 0 lane 0 loads (TMA: the Q tile once, K or K and V per step into a
// ring of NS stages), warp 1 lane 0 issues the MMAs, warps 2-5 own one row
// per thread (TMEM lane quarter = warp % 4).  S is double-buffered in TMEM,
// P in shared memory, so the loads, the MMAs and the softmax of neighbouring
// steps overlap.
#pragma once
#include "prefill_cc.cuh"

namespace hils {

template <int D>
struct CcLocal {
  static constexpr int M = 128;
  static constexpr int KATOMS = D / 64;
  static constexpr int NS = 3;                           // K/V load stages
  static constexpr uint32_t Q_ATOM = M * 128;           // 16 KB
  static constexpr uint32_t KV_ATOM = kChunk * 128;     // 8 KB
  static constexpr uint32_t Q_BYTES = KATOMS * Q_ATOM;
  static constexpr uint32_t K_BYTES = KATOMS * KV_ATOM;
  static constexpr uint32_t STAGE = 2 * K_BYTES;        // K, then V
  static constexpr uint32_t P_BYTES = M * 128;          // 128 rows x 64 keys bf16
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_ST = Q_BYTES;
  static constexpr uint32_t OFF_P = OFF_ST + NS * STAGE;
  static constexpr uint32_t OFF_BAR = OFF_P + 2 * P_BYTES;
  // q_full, load_full[NS], load_empty[NS], s_full[2], s_empty[2], p_full[2],
  // p_empty[2], o_full, done
  static constexpr int N_BARS = 1 + 2 * NS + 8 + 2;
  static constexpr uint32_t SMEM = OFF_BAR + N_BARS * 8 + 16 + 1024;
  // S[2] x 64 columns, then O (D columns).  Shared memory holds at most two
  // CTAs per SM (d = 64) or one (d = 128), so 256 columns each always fit.
  static constexpr uint32_t TMEM_COLS = 256;
  // more CTAs than 512 / TMEM_COLS per SM (228 KB of shared memory, 1 KB
  // reserved per CTA) could make a tcgen05.alloc wait for columns that a
  // co-resident CTA never frees
  static_assert((512 / TMEM_COLS + 1) * (SMEM + 1024) > 233472u, "TMEM never oversubscribed");
  static constexpr uint32_t T_O = 2 * kChunk;
  static constexpr uint32_t IDESC_S = sm100::idesc_bf16(M, kChunk);
  static constexpr uint32_t IDESC_O = sm100::idesc_bf16(M, D) | (1u << 16);   // V is MN-major
  static constexpr int THREADS = 192;
  static_assert(3 * (SMEM + 1024) > 233472u, "at most two CTAs per SM share the TMEM");
};

template <int D>
__global__ void __launch_bounds__(CcLocal<D>::THREADS)
cc_local_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const CcOwnParams p) {
  using C = CcLocal<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* load_full = bars + 1;              // [NS] producer -> MMA
  uint64_t* load_empty = load_full + C::NS;    // [NS] MMA -> producer
  uint64_t* s_full = load_empty + C::NS;       // [2]  MMA -> rows
  uint64_t* s_empty = s_full + 2;              // [2]  rows -> MMA
  uint64_t* p_full = s_empty + 2;              // [2]  rows -> MMA
  uint64_t* p_empty = p_full + 2;              // [2]  MMA -> rows
  uint64_t* o_full = p_empty + 2;
  uint64_t* done = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + C::N_BARS) + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const CcDims& c = p.c;
  const int P = p.P, G = c.G;
  const int64_t bh = blockIdx.y, b = bh / c.Hkv, h = bh % c.Hkv;
  const int64_t p0 = int64_t(blockIdx.x) * P;
  const int64_t p_last = (p0 + P < c.n_tok ? p0 + P : c.n_tok) - 1;
  const int64_t cw0 = p0 / kChunk - c.wm1 > 0 ? p0 / kChunk - c.wm1 : 0;   // first window chunk of the tile
  const int KB = int(p_last / kChunk - cw0 + 1);                          // chunks per pass
  const int n_steps = 2 * KB;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&load_full[s], 1);
      mbar_init(&load_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int g = 0; g < G; ++g) {
        const int y = int((b * c.Hq + h * G + g) * c.n_tok + p0);
#pragma unroll
        for (int a = 0; a < C::KATOMS; ++a)
          tma_load_2d(smem + C::OFF_Q + a * C::Q_ATOM + g * P * 128, &tm_q, q_full, a * 64, y);
      }
      int t = 0;
      for (; t < n_steps; ++t) {
        const int s = t % C::NS, u = t / C::NS;
        if (!mbar_wait(&load_empty[s], (u & 1) ^ 1, abort_flag)) break;
        const bool pass2 = t >= KB;
        const int yk = int(bh * c.n_tok + (cw0 + (pass2 ? t - KB : t)) * kChunk);
        uint8_t* st = smem + C::OFF_ST + s * C::STAGE;
        mbar_arrive_expect_tx(&load_full[s], pass2 ? 2 * C::K_BYTES : C::K_BYTES);
#pragma unroll
        for (int a = 0; a < C::KATOMS; ++a) {
          tma_load_2d(st + a * C::KV_ATOM, &tm_k, &load_full[s], a * 64, yk);
          if (pass2) tma_load_2d(st + C::K_BYTES + a * C::KV_ATOM, &tm_v, &load_full[s], a * 64, yk);
        }
      }
      // only the last NS issued loads can still be in flight: let them land
      mbar_wait_drain(q_full, 0);
      for (int t2 = t > C::NS ? t - C::NS : 0; t2 < t; ++t2) mbar_wait_drain(&load_full[t2 % C::NS], (t2 / C::NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int t = 0;
      const bool q_ok = mbar_wait(q_full, 0, abort_flag);
      for (; q_ok && t < n_steps; ++t) {
        const int s = t % C::NS, u = t / C::NS, sb = t & 1;
        if (!mbar_wait(&load_full[s], u & 1, abort_flag)) break;
        if (!mbar_wait(&s_empty[sb], ((t >> 1) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t sq = smem_u32(smem + C::OFF_Q), sk = smem_u32(smem + C::OFF_ST + s * C::STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16(tmem + uint32_t(sb * kChunk), desc_sw128(sq + uint32_t((kk >> 2) * C::Q_ATOM + (kk & 3) * 32)),
                   desc_sw128(sk + uint32_t((kk >> 2) * C::KV_ATOM + (kk & 3) * 32)), C::IDESC_S, kk > 0 ? 1u : 0u);
        mma_commit(&s_full[sb]);
        if (t < KB) {
          mma_commit(&load_empty[s]);
          continue;
        }
        const int j = t - KB, pb = j & 1;
        if (!mbar_wait(&p_full[pb], (j >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t sp = smem_u32(smem + C::OFF_P + pb * C::P_BYTES), sv = sk + C::K_BYTES;
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          mma_bf16(tmem + C::T_O, desc_sw128(sp + uint32_t(kk * 32)), desc_sw128_mn(sv + uint32_t(kk * 2048), C::KV_ATOM),
                   C::IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&p_empty[pb]);
        mma_commit(&load_empty[s]);
      }
      if (q_ok && t == n_steps) mma_commit(o_full);
      mma_commit(done);
    }
  } else {
    // ------------------------------------------------------------ one row per thread
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t t_lane = uint32_t(quarter * 32) << 16;
    const int g = r / P;
    const int64_t pos = p0 + r % P;
    const bool live = pos < c.n_tok;
    const int64_t row = (b * c.Hq + h * G + g) * c.n_tok + pos;
    const int64_t own = pos / kChunk;
    const int64_t lo = own - c.wm1 > 0 ? own - c.wm1 : 0;   // first window chunk = number of candidates
    const int jpos = int(pos % kChunk);
    const float k2 = c.tau * 1.4426950408889634f;
    // largest kept score (the loads overlap the first MMAs)
    float smax = -INFINITY;
    if (live) {
      for (int t = 0; t < c.K; ++t) {
        const int32_t ci = __ldg(p.ids + row * c.K + t);
        if (ci >= 0 && ci < lo) smax = fmaxf(smax, __ldg(p.scores + row * c.K + t));
      }
    }
    // last valid key of window chunk cj for this row (-1: none)
    auto last_key = [&](int64_t cj) -> int { return (live && cj >= lo && cj <= own) ? (cj < own ? kChunk - 1 : jpos) : -1; };
    bool ok = true;
    float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // independent chains
    for (int t = 0; t < KB; ++t) {
      const int sb = t & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (t >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float sa[32], sc[32];
      tmem_ld32(tmem + t_lane + uint32_t(sb * kChunk), sa);
      tmem_ld32(tmem + t_lane + uint32_t(sb * kChunk + 32), sc);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      const int jmax = last_key(cw0 + t);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        mp[e & 3] = fmaxf(mp[e & 3], e <= jmax ? sa[e] : -INFINITY);
        mp[(e + 2) & 3] = fmaxf(mp[(e + 2) & 3], e + 32 <= jmax ? sc[e] : -INFINITY);
      }
    }
    const float m = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
    const float mb = (live ? m : 0.f) * k2;
    float lp[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; ok && j < KB; ++j) {
      const int t = KB + j, sb = t & 1, pb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (t >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float sa[32], sc[32];
      tmem_ld32(tmem + t_lane + uint32_t(sb * kChunk), sa);
      tmem_ld32(tmem + t_lane + uint32_t(sb * kChunk + 32), sc);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      const int jmax = last_key(cw0 + j);
      ok = __all_sync(0xffffffffu, mbar_wait(&p_empty[pb], ((j >> 1) & 1) ^ 1, abort_flag));
      if (!ok) break;
      // P row: 64 keys bf16 = 128 bytes, K-major with the 128-byte swizzle
      uint8_t* prow = smem + C::OFF_P + pb * C::P_BYTES + r * 128;
#pragma unroll
      for (int piece = 0; piece < 8; ++piece) {
        uint32_t wd[4];
#pragma unroll
        for (int v2 = 0; v2 < 4; ++v2) {
          const int e0 = piece * 8 + 2 * v2;
          const float x0 = e0 < 32 ? sa[e0] : sc[e0 - 32];
          const float x1 = e0 + 1 < 32 ? sa[e0 + 1] : sc[e0 - 31];
          const float y0 = e0 <= jmax ? ex2_approx(fmaf(x0, k2, -mb)) : 0.f;
          const float y1 = e0 + 1 <= jmax ? ex2_approx(fmaf(x1, k2, -mb)) : 0.f;
          lp[v2] += y0 + y1;
          __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
          wd[v2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(prow + ((piece ^ (r & 7)) << 4)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&p_full[pb]);
    }
    // window log-sum-exp and the fusion normaliser over the kept chunks and the window
    const float l = (lp[0] + lp[1]) + (lp[2] + lp[3]);
    const float lse = (live ? m : 0.f) * c.tau + logf(l);
    float Mp = lse;
    if (live && ok) {
      const float Mx = fmaxf(smax, lse);
      float Z = expf(lse - Mx);
      for (int t = 0; t < c.K; ++t) {
        const int32_t ci = __ldg(p.ids + row * c.K + t);
        if (ci >= 0 && ci < lo) Z += expf(__ldg(p.scores + row * c.K + t) - Mx);
      }
      Mp = Mx + logf(Z);
      p.rowstat[row] = Mp;
      if (p.lse_own) p.lse_own[row] = lse;
    }
    // O = sum exp(tau (s - m)) v  ->  the accumulator gets exp(tau m - M') O
    const float scale = live ? expf(m * c.tau - Mp) : 0.f;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_full, 0, abort_flag));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        tmem_ld32(tmem + t_lane + C::T_O + uint32_t(cc * 32), o);
        if (live) {
          float* dst = p.oacc + row * D + cc * 32;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + e) =
                make_float4(o[e] * scale, o[e + 1] * scale, o[e + 2] * scale, o[e + 3] * scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA this CTA issued has finished before its TMEM is freed
    if (lane == 0) mbar_wait_drain(done, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace hils
