// Kernel (b), tensor-core variant (bf16): chunk scoring on tcgen05 + fused
// per-row top-K.
//
// HiLS paper, aitrends.kr article, section "방법론" (Methodology):
//   s^_{i,c} = <q_i, k'_c>/sqrt(d) + b'_c over the fully-past chunks; keep the
//   K largest.
//
// One CTA scores a tile of 128 query rows -- P = 128/G consecutive positions
// of the G query heads that share a kv head, so the compressed keys are read
// once for all G heads -- against the causal prefix of compressed keys, in
// tiles of 128 chunks:
//   warp 0 (one lane)  TMA producer: the Q tile once, then k' tiles into a
//                      STAGES-deep shared-memory ring (128B swizzle).
//   warp 1 (one lane)  MMA issuer: S = Q . K'^T with tcgen05.mma (M=128,
//                      N=128, bf16 in, fp32 accumulators in TMEM, two TMEM
//                      buffers so the epilogue of tile j overlaps the MMA of
//                      tile j+1).  The entropy bias enters the MMA: the
//                      scoring operand carries x = b'/tau as a bf16 hi/lo
//                      pair in 16 extra K columns, and a constant A slice
//                      [1, 1, 0, ...] multiplies it, so TMEM holds
//                      <q,k'> + b'/tau and s^ = tau * acc.
//   warps 2-5          epilogue, one thread per row (= TMEM lane): 32 scores
//                      per tcgen05.ld; each is tested against the row's
//                      current K-th best with one FFMA and its sign bit is
//                      funnel-shifted into a 32-bit mask.  Passing scores go,
//                      one per lane and round with all lanes in step, into a
//                      values-only sorted list in registers (two min/max per
//                      slot, no branches) and, with their chunk ids, into a
//                      per-row log in shared memory; the result's ids are
//                      read back from the log.  Ties keep the lower chunk id
//                      (chunks are visited in ascending order).
// Every wait is bounded in time; a time-out records HILS_ERR_DEVICE_TIMEOUT,
// drains in-flight copies and MMAs, frees TMEM and returns.
#pragma once
#include "sm100.cuh"

namespace hils {

template <int D, int KCAP>
struct SelTc {
  static constexpr int M = 128;           // rows per tile (TMEM lanes)
  static constexpr int NT = 128;          // chunks per k' tile (MMA N)
  static constexpr int KATOMS = D / 64;   // 128-byte swizzle atoms along K
  static constexpr uint32_t A_ATOM = M * 128;
  static constexpr uint32_t A_BYTES = KATOMS * A_ATOM;
  static constexpr uint32_t AEXT_BYTES = M * 32;
  static constexpr uint32_t B_ATOM = NT * 128;
  static constexpr uint32_t B_MAIN = KATOMS * B_ATOM;
  static constexpr uint32_t B_EXT = NT * 32;
  static constexpr uint32_t B_STAGE = B_MAIN + B_EXT;
  static constexpr int STG_STRIDE = 36;   // floats per thread in the staging area (conflict-free float4)
  // KCAP > 0: the per-row top-K values live in registers (K <= KCAP) and the
  // (score, chunk) pairs that entered them in a per-row shared-memory log of
  // `cap` entries (K + 32 at least, host-chosen); KCAP == 0: a sorted
  // (score, chunk) list of K entries in shared memory.
  static constexpr int MIN_CAP = KCAP + 32;
  // d = 64 with K <= 16 runs two CTAs per SM; every other shape runs one
  static constexpr bool TWO_PER_SM = D == 64 && KCAP == 16;
  // STAGED: a row with passing scores in a 32-score group stages the group in
  // shared memory and reads the passing ones back by column.  Otherwise they
  // are picked out of the registers by a 5-level select (31 selects per
  // append).  Staging wins where there is room for it next to two k' stages,
  // i.e. with one CTA per SM; with two CTAs per SM it would cost a k' stage,
  // which measured slower.
  static constexpr bool STAGED = KCAP > 0 && !TWO_PER_SM;
  // staging area (the shared-memory list path, K > 32, always uses it)
  static constexpr uint32_t STG_BYTES = (KCAP == 0 || STAGED) ? uint32_t(M) * STG_STRIDE * 4 : 0u;
  static constexpr int THREADS = 192;
  // two CTAs per SM, two TMEM accumulators each (the MMA of tile j+1 runs
  // during the epilogue of tile j; three CTAs with one accumulator each
  // measured slower)
  static constexpr int CTAS_PER_SM = 2;
  static constexpr int BUFS = 2;
  static constexpr uint32_t TMEM_COLS = BUFS * NT;
  static constexpr uint32_t IDESC = sm100::idesc_bf16(M, NT);

  struct Layout {
    uint32_t a, aext, b, stg, topv, topi, bars, misc, total;
    int stages;
  };
  // Shared-memory layout (offsets from a 1024-byte aligned base).
  __host__ __device__ static Layout layout(int K, int stages, int cap) {
    Layout L;
    L.stages = stages;
    L.a = 0;
    L.aext = A_BYTES;
    L.b = (L.aext + AEXT_BYTES + 1023u) & ~1023u;
    L.stg = L.b + uint32_t(stages) * B_STAGE;
    const uint32_t list_bytes = uint32_t(KCAP > 0 ? cap : K) * M * 4;
    L.topv = L.stg + STG_BYTES;
    L.topi = L.topv + list_bytes;
    L.bars = L.topi + list_bytes;
    L.misc = L.bars + uint32_t(2 * stages + 6) * 8;
    L.total = L.misc + 16 + 1024;  // + slack for aligning the dynamic base
    return L;
  }
};

struct SelTcParams {
  int64_t n_tok, nc;
  int Hq, Hkv, G, K, P;  // P = 128 / G positions per tile
  int n_row_tiles, stages, cap;
  int wm1;   // chunks of the local window before the own chunk
  float tau;
  int32_t* ids;
  float* scores;
};

// sign bits (as words) of c - t*a0 and c - t*a1, one packed FMA
__device__ __forceinline__ void fma2_signs(float a0, float a1, uint64_t nt2, uint64_t c2, uint32_t& s0, uint32_t& s1) {
  asm("{\n\t.reg .b64 va, vd;\n\t"
      "mov.b64 va, {%2, %3};\n\t"
      "fma.rn.f32x2 vd, va, %4, %5;\n\t"
      "mov.b64 {%0, %1}, vd;\n\t}"
      : "=r"(s0), "=r"(s1)
      : "f"(a0), "f"(a1), "l"(nt2), "l"(c2));
}

// max of three floats in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint64_t pack2(float x) {
  const uint64_t u = __float_as_uint(x);
  return (u << 32) | u;
}

template <int D, int KCAP>
__global__ void __launch_bounds__(SelTc<D, KCAP>::THREADS, SelTc<D, KCAP>::CTAS_PER_SM)
select_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kb,
                 const __grid_constant__ CUtensorMap tm_ke, const SelTcParams p) {
  using C = SelTc<D, KCAP>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const typename C::Layout L = C::layout(p.K, p.stages, p.cap);
  uint8_t* sA = smem + L.a;
  uint8_t* sAext = smem + L.aext;
  uint8_t* sB = smem + L.b;
  float* stg = reinterpret_cast<float*>(smem + L.stg);
  float* topv = reinterpret_cast<float*>(smem + L.topv);
  int32_t* topi = reinterpret_cast<int32_t*>(smem + L.topi);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + L.stages;
  uint64_t* tfull = bars + 2 * L.stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* qfull = tempty + 2;
  uint64_t* done = qfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  int* issued_slot = reinterpret_cast<int*>(smem + L.misc + 8);
  int* consumed_slot = reinterpret_cast<int*>(smem + L.misc + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = p.n_row_tiles - 1 - int(blockIdx.x);  // longest causal prefixes first
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const int64_t pos0 = int64_t(tile) * p.P;
  const int64_t pos_end = (pos0 + p.P < p.n_tok) ? pos0 + p.P : p.n_tok;
  const int64_t c_hi = n_candidates(pos_end - 1, p.wm1);   // candidates of the tile's last row
  const int n_tiles = int((c_hi + C::NT - 1) / C::NT);
  // K <= KCAP: when every row of the tile has at least 8 K candidates, a
  // first pass over the chunks splits each row's scores into disjoint groups
  // of g and finds the K-th largest group maximum: K distinct scores reach
  // it, so it is a lower bound of the row's K-th best score, and the second
  // pass keeps only the scores that reach it.  The MMAs of both passes are
  // the same.  g: 128 from 128 K candidates on, else 32, 16 or 8 (the
  // largest that leaves K groups); smaller groups bound tighter but cost a
  // list insertion each, and on long rows a group of 128 is the cheaper.
  const int64_t n_min = n_candidates(pos0, p.wm1);   // candidates of the tile's first row
  const int64_t kk = p.K;
  const int group = n_min >= 128 * kk ? 128 : n_min >= 32 * kk ? 32 : n_min >= 16 * kk ? 16 : n_min >= 8 * kk ? 8 : 0;
  const int n_pass = (KCAP > 0 && group > 0) ? 2 : 1;
  const int n_steps = n_pass * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&tfull[t], 1);
      mbar_init(&tempty[t], 4);
    }
    mbar_init(qfull, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    *issued_slot = 0;
    *consumed_slot = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // constant A slice [1, 1, 0, ...] in the 32-byte swizzled K-major layout:
    // the two 16-byte halves of row r swap when bit 2 of r is set.
    const int r = int(threadIdx.x) - 64;
    uint4* row = reinterpret_cast<uint4*>(sAext + r * 32);
    const int sw = (r >> 2) & 1;
    row[sw] = make_uint4(0x3F803F80u, 0u, 0u, 0u);
    row[sw ^ 1] = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0 && n_tiles > 0) {
    // ------------------------------------------------------------ producer
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kb);
    prefetch_tmap(&tm_ke);
    mbar_arrive_expect_tx(qfull, C::A_BYTES);
    for (int g = 0; g < p.G; ++g) {
      const int y = int((int64_t(b) * p.Hq + int64_t(h) * p.G + g) * p.n_tok + pos0);
      for (int a = 0; a < C::KATOMS; ++a) tma_load_2d(sA + a * C::A_ATOM + g * p.P * 128, &tm_q, qfull, a * 64, y);
    }
    int j = 0;
    for (; j < n_steps; ++j) {
      const int s = j % L.stages, u = j / L.stages;
      if (!mbar_wait(&empty[s], (u & 1) ^ 1, abort_flag)) break;
      mbar_arrive_expect_tx(&full[s], C::B_STAGE);
      uint8_t* bs = sB + s * C::B_STAGE;
      const int y = int(int64_t(bh) * p.nc + int64_t(j % n_tiles) * C::NT);
      for (int a = 0; a < C::KATOMS; ++a) tma_load_2d(bs + a * C::B_ATOM, &tm_kb, &full[s], a * 64, y);
      tma_load_2d(bs + C::B_MAIN, &tm_ke, &full[s], D, y);
    }
    *issued_slot = j;
  } else if (warp == 1 && lane == 0 && n_tiles > 0) {
    // ------------------------------------------------------------ MMA issuer
    int j = 0;
    if (mbar_wait(qfull, 0, abort_flag)) {
      const uint32_t a0 = smem_u32(sA), ae = smem_u32(sAext);
      for (; j < n_steps; ++j) {
        const int s = j % L.stages, u = j / L.stages, buf = j % C::BUFS, ub = j / C::BUFS;
        if (!mbar_wait(&full[s], u & 1, abort_flag)) break;
        if (!mbar_wait(&tempty[buf], (ub & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(buf * C::NT);
        const uint32_t b0 = smem_u32(sB + s * C::B_STAGE);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = uint32_t((k >> 2) * C::A_ATOM + (k & 3) * 32);
          const uint32_t offb = uint32_t((k >> 2) * C::B_ATOM + (k & 3) * 32);
          mma_bf16(d, desc_sw128(a0 + off), desc_sw128(b0 + offb), C::IDESC, k > 0 ? 1u : 0u);
        }
        mma_bf16(d, desc_sw32(ae), desc_sw32(b0 + C::B_MAIN), C::IDESC, 1u);
        mma_commit(&empty[s]);
        mma_commit(&tfull[buf]);
      }
    }
    *consumed_slot = j;
    mma_commit(done);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int g = r / p.P;
    const int64_t pos = pos0 + r % p.P;
    const bool valid = pos < p.n_tok;
    const int64_t n_cand = valid ? n_candidates(pos, p.wm1) : 0;
    const int K = p.K;
    const float tau = p.tau;
    const uint64_t ntau2 = pack2(-tau);
    float* my_stg = stg + r * C::STG_STRIDE;
    float* tv = topv + r;
    int32_t* ti = topi + r;
    // KCAP > 0: tv/ti is the row's candidate buffer, (score, chunk) pairs in
    // ascending chunk order; KCAP == 0: its sorted top-K list.  `count` entries.
    int count = 0;
    // a score passes when tau * acc > thr, exactly (the sign of one FMA)
    float thr = -INFINITY;
    // KCAP > 0: values-only list sorted descending; slots [0, KCAP-K) hold
    // +inf so that the K-th value is always the last slot.  It ranks the group
    // maxima of the first pass and the candidate buffer.
    constexpr int KR = KCAP > 0 ? KCAP : 1;
    float rv[KR];
    auto rv_reset = [&]() {
#pragma unroll
      for (int t = 0; t < KR; ++t) rv[t] = t < KR - K ? INFINITY : -INFINITY;
    };
    rv_reset();
    // sorted insertion without branches: slot t takes max(old t, min(old t-1, x));
    // x = -inf leaves the list unchanged
    auto rv_insert = [&](float x) {
#pragma unroll
      for (int t = KR - 1; t >= 1; --t) rv[t] = fmaxf(rv[t], fminf(rv[t - 1], x));
      rv[0] = fmaxf(rv[0], x);
    };
    // rv <- the best K scores of the buffer, all lanes in step
    auto rank_buffer = [&]() {
      rv_reset();
      const int m = __reduce_max_sync(0xffffffffu, count);
      for (int i = 0; i < m; ++i) rv_insert(i < count ? tv[i * C::M] : -INFINITY);
    };
    // Walk the buffer in chunk order and keep what its best K are: every
    // score above their K-th value w, then the first scores equal to w.
    // Compaction (emit false): the kept entries move to the front of the
    // buffer and later scores must beat w.  Emission: they are written to
    // out_i/out_s (if not null) in chunk order and padded with -1.  All lanes
    // call it together.
    auto keep_best = [&](bool emit, int32_t* out_i, float* out_s) {
      rank_buffer();
      const float w = rv[KR - 1];
      int quota = K;
#pragma unroll
      for (int t = 0; t < KR; ++t) quota -= (t >= KR - K) & (rv[t] > w);
      int n = 0;
      for (int i = 0; i < count; ++i) {
        const float val = tv[i * C::M];
        const bool eq = val == w;
        const bool keep = val > w || (eq && quota > 0);
        quota -= eq && keep;
        if (keep) {
          const int32_t id = ti[i * C::M];
          if (emit) {
            if (out_i) out_i[n] = id;
            if (out_s) out_s[n] = val;
          } else {
            tv[n * C::M] = val;
            ti[n * C::M] = id;
          }
          ++n;
        }
      }
      if (emit) {
        for (int t = n; t < K && out_i; ++t) {
          out_i[t] = -1;
          if (out_s) out_s[t] = -INFINITY;
        }
      } else {
        count = n;
        thr = fmaxf(thr, w);
      }
    };
    float tmax = -INFINITY;
    // ---- first pass, one 32-column group: its maxima, ranked in rv
    auto max_group = [&](uint32_t (&rg)[32], int lim) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(rg[e]);
      if (__any_sync(0xffffffffu, lim < 32)) {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = e < lim ? v[e] : -INFINITY;
      }
      if (group == C::NT) {
        // one maximum per tile: a tree of three-input maxima, 16 instructions
        // for 32 scores plus the running maximum
        float m[11];
#pragma unroll
        for (int t = 0; t < 10; ++t) m[t] = fmax3(v[3 * t], v[3 * t + 1], v[3 * t + 2]);
        m[10] = fmaxf(v[30], v[31]);
        const float a = fmax3(m[0], m[1], m[2]), bb = fmax3(m[3], m[4], m[5]), cc = fmax3(m[6], m[7], m[8]);
        tmax = fmaxf(fmax3(a, bb, cc), fmax3(m[9], m[10], tmax));
        return;
      }
      // max tree: after the step of width w, v[t] (t < w) is the maximum of
      // the scores e = t (mod w) -- disjoint groups of 32 / w.
      // tau > 0 and rounding is monotone: tau * max = max of the scores.
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = fmaxf(v[e], v[e + 16]);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = fmaxf(v[e], v[e + 8]);
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = fmaxf(v[e], v[e + 4]);
      if (group == 8) {
#pragma unroll
        for (int e = 0; e < 4; ++e) rv_insert(tau * v[e]);
        return;
      }
      v[0] = fmaxf(v[0], v[2]);
      v[1] = fmaxf(v[1], v[3]);
      if (group == 16) {
        rv_insert(tau * v[0]);
        rv_insert(tau * v[1]);
        return;
      }
      v[0] = fmaxf(v[0], v[1]);
      rv_insert(tau * v[0]);   // group == 32
    };
    // ---- scan, one 32-column group: test every score against thr, keep the
    // passing ones
    auto scan_group = [&](uint32_t (&rg)[32], int lim, int64_t cbase) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(rg[e]);
      uint32_t bits = 0;
      if (lim > 0) {
        // bit (31-e) = [tau * v[e] > thr], exactly: sign of fma(-tau, v, thr);
        // four independent 8-bit chains keep the dependency depth short
        uint32_t part[4] = {0u, 0u, 0u, 0u};
        const uint64_t thr2 = pack2(thr);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t s0, s1;
            fma2_signs(v[8 * q4 + e], v[8 * q4 + e + 1], ntau2, thr2, s0, s1);
            part[q4] = __funnelshift_l(s0, part[q4], 1);
            part[q4] = __funnelshift_l(s1, part[q4], 1);
          }
        }
        bits = (part[0] << 24) | ((part[1] & 0xFFu) << 16) | ((part[2] & 0xFFu) << 8) | (part[3] & 0xFFu);
        if (lim < 32) bits &= ~(0xFFFFFFFFu >> lim);
      }
      if constexpr (KCAP > 0) {
        // the buffer holds at least K + 32 entries and a compaction leaves at
        // most K, so one check per group makes room for all its scores
        if (__any_sync(0xffffffffu, count + __popc(bits) > p.cap)) keep_best(false, nullptr, nullptr);
        if constexpr (C::STAGED) {
          // append the passing scores: a row with any stages its 32 scores,
          // then reads each passing one back by its column
          if (bits) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(my_stg + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          }
          while (bits) {
            const int e = __clz(bits);
            bits &= ~(0x80000000u >> e);
            tv[count * C::M] = tau * my_stg[e];
            ti[count * C::M] = int32_t(cbase + e);
            ++count;
          }
        } else {
          // append the passing scores, one per lane and round; the score is
          // picked out of the registers by a 5-level select on its column
          while (__any_sync(0xffffffffu, bits != 0u)) {
            const bool has = bits != 0u;
            const int e = __clz(bits) & 31;
            bits &= ~(0x80000000u >> e);
            float w16[16], w8[8], w4[4], w2[2];
#pragma unroll
            for (int t = 0; t < 16; ++t) w16[t] = (e & 16) ? v[t + 16] : v[t];
#pragma unroll
            for (int t = 0; t < 8; ++t) w8[t] = (e & 8) ? w16[t + 8] : w16[t];
#pragma unroll
            for (int t = 0; t < 4; ++t) w4[t] = (e & 4) ? w8[t + 4] : w8[t];
#pragma unroll
            for (int t = 0; t < 2; ++t) w2[t] = (e & 2) ? w4[t + 2] : w4[t];
            const float x = tau * ((e & 1) ? w2[1] : w2[0]);
            if (has) {
              tv[count * C::M] = x;
              ti[count * C::M] = int32_t(cbase + e);
              ++count;
            }
          }
        }
      } else {
        if (!__any_sync(0xffffffffu, bits != 0)) return;
        if (bits) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(my_stg + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
        while (bits) {
          const int e = __clz(bits);
          bits &= ~(0x80000000u >> e);
          const float sc = tau * my_stg[e];
          const int32_t cid = int32_t(cbase + e);
          if (count == K && !(sc > thr)) continue;
          int q = count < K ? count : K - 1;
          while (q > 0 && tv[(q - 1) * C::M] < sc) {
            tv[q * C::M] = tv[(q - 1) * C::M];
            ti[q * C::M] = ti[(q - 1) * C::M];
            --q;
          }
          tv[q * C::M] = sc;
          ti[q * C::M] = cid;
          if (count < K) ++count;
          if (count == K) thr = tv[(K - 1) * C::M];
        }
      }
    };
    for (int jg = 0; jg < n_steps; ++jg) {
      const int buf = jg % C::BUFS, ub = jg / C::BUFS;
      const int j = jg % n_tiles;
      if (!mbar_wait(&tfull[buf], ub & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(buf * C::NT);
      const int64_t c0 = int64_t(j) * C::NT;
      // candidates of this row left in the tile (clamped to 0..128)
      const int64_t left64 = n_cand - c0;
      const int left = left64 <= 0 ? 0 : (left64 >= C::NT ? C::NT : int(left64));
      // the tile's four 32-column groups (loading the next group while one is
      // processed measured slower: more registers, more code)
      uint32_t ra[32];
      if (KCAP > 0 && n_pass == 2 && jg < n_tiles) {
#pragma unroll 1
        for (int gi = 0; gi < C::NT / 32; ++gi) {
          tmem_ld32_async(tb + gi * 32, ra);
          tmem_ld_wait(ra);
          max_group(ra, left - gi * 32);
        }
        if (group == C::NT) {
          rv_insert(tau * tmax);
          tmax = -INFINITY;
        }
      } else {
#pragma unroll 1
        for (int gi = 0; gi < C::NT / 32; ++gi) {
          tmem_ld32_async(tb + gi * 32, ra);
          tmem_ld_wait(ra);
          scan_group(ra, left - gi * 32, c0 + gi * 32);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (KCAP > 0 && n_pass == 2 && jg == n_tiles - 1) {
        // every score >= the K-th group maximum T passes: thr = the float below T
        const float t_lb = rv[KR - 1];
        thr = t_lb > -INFINITY ? nextafterf(t_lb, -INFINITY) : -INFINITY;
      }
    }
    const int64_t row = (int64_t(b) * p.Hq + int64_t(h) * p.G + g) * p.n_tok + pos;
    int32_t* out_i = valid ? p.ids + row * K : nullptr;
    float* out_s = valid && p.scores ? p.scores + row * K : nullptr;
    if constexpr (KCAP > 0) {
      keep_best(true, out_i, out_s);
    } else if (valid) {
      for (int a = 1; a < count; ++a) {
        const int32_t ci = ti[a * C::M];
        const float cv = tv[a * C::M];
        int q = a;
        while (q > 0 && ti[(q - 1) * C::M] > ci) {
          ti[q * C::M] = ti[(q - 1) * C::M];
          tv[q * C::M] = tv[(q - 1) * C::M];
          --q;
        }
        ti[q * C::M] = ci;
        tv[q * C::M] = cv;
      }
      for (int t = 0; t < K; ++t) {
        out_i[t] = t < count ? ti[t * C::M] : -1;
        if (out_s) out_s[t] = t < count ? tv[t * C::M] : -INFINITY;
      }
    }
  }
  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (threadIdx.x == 0 && n_tiles > 0) {
    // copies still in flight (only after an abort): wait for them to land
    mbar_wait_drain(qfull, 0);
    for (int j = *consumed_slot; j < *issued_slot; ++j)
      mbar_wait_drain(&full[j % L.stages], (j / L.stages) & 1);
  }
  if (warp == 1) {
    if (lane == 0 && n_tiles > 0) mbar_wait_drain(done, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace hils
