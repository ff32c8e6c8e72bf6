// Kernel (c), tensor-core variant (bf16): chunk-centric sparse prefill.
//
// HiLS paper, hotpaper.ai abstract and aitrends.kr article, section "방법론"
// (Methodology) and glossary "계층적 소프트맥스": each query attends to each
// retrieved chunk separately (intra-chunk softmax) and the chunk outputs are
// fused by a softmax over the retrieval scores; the own chunk is attended
// under the causal mask and fused with its exact log-sum-exp.
//
// The pages' kernel loads, for a block of adjacent queries, the union of
// their selected chunks.  On i.i.d. inputs adjacent queries share few chunks
// (a 128-row block selects hundreds of distinct chunks), so that design would
// spend most tensor-core work on rows that did not select the chunk.  Here the
// work is regrouped by chunk instead:
//   own    : per row, the causal own-chunk attention (or, with a local
//            window of more than one chunk, the window branch of
//            prefill_local.cuh), the fusion normaliser
//            M' = log(sum_c exp(s^_c) + exp(lse_own)) and the own branch's
//            share exp(lse_own - M') o_own written to an fp32 accumulator.
//   count  : the number of (row, slot) pairs per key (kv head, window,
//            chunk) and each pair's rank within its key.
//   scan   : offsets of every key's pair list and of its 128-row tiles.
//   fill   : the inverted index: per key its list of (row, s^ - M') records.
//   attend : per tile of up to 128 pairs of one chunk: the chunk's K and V
//            arrive by TMA, the rows' queries by TMA gather4 into a
//            128B-swizzled tile, S = Q K^T on tcgen05 (fp32 in TMEM), one
//            thread per row turns its 64 scores into
//            P = exp(s - lse_c + s^_c - M'), P V on tcgen05, and the row's
//            partial output is added to its accumulator in L2 (bulk or
//            16-byte vector reductions).  The weights are final, so partials
//            simply add.
//   final  : accumulator -> bf16 output.
// Windows: a key's rows lie in one window of W positions; tiles are ordered
// window by window, so the accumulators of the rows being updated stay
// resident in L2.
#pragma once
#include "attend_simt.cuh"
#include "sm100.cuh"

namespace hils {

struct CcDims {
  int64_t n_tok, nc;
  int Hq, Hkv, G, K;
  int wm1;         // chunks of the local window before the own chunk
  int win_shift;   // L2 window of a row = pos >> win_shift
  int n_win;
  int64_t n_keys;  // B*Hkv*n_win*nc
  float tau;
};

__device__ __forceinline__ int64_t cc_key(const CcDims& c, int64_t bh, int64_t pos, int64_t chunk) {
  return (bh * c.n_win + (pos >> c.win_shift)) * c.nc + chunk;
}

// MN-major, 128B-swizzled operand: 64-element rows along N, 8-row groups
// (along K) 1024 bytes apart, 64-wide N blocks `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// global[dst .. dst+bytes) += shared[src .. src+bytes) as fp32, done by the
// bulk-copy unit as whole-sector reductions in L2; per-thread bulk group.
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src_smem, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
               "r"(src_smem), "r"(bytes)
               : "memory");
}
// global[addr .. addr+16) += {a, b, c, d} as fp32, in L2
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
// D[tmem] (+)= A[tmem] x B[smem desc]^T, bf16 inputs, fp32 accumulate.  A sits
// in tensor memory: row m in lane m, its K elements in consecutive columns,
// two bf16 per 32-bit column (the lower element in the low half).
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns from registers (thread t of the
// warp writes lane (warp%4)*32 + t), then a wait until the stores are done.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk groups except the newest n have finished reading shared memory
template <int n>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Four rows y0..y3 of a tensor map whose box is one row of 64 elements.
__device__ __forceinline__ void tma_gather4(uint32_t smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y0,
                                            int y1, int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(sm100::smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

// max of three floats in one instruction (sm_100)
__device__ __forceinline__ float fmax3_f32(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two fp32 lanes per instruction (sm_100), each rounded as its scalar form.
__device__ __forceinline__ void fma2_f32(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                         float c1) {
  asm("{\n\t.reg .b64 va, vb, vc, vd;\n\t"
      "mov.b64 va, {%2, %3};\n\tmov.b64 vb, {%4, %5};\n\tmov.b64 vc, {%6, %7};\n\t"
      "fma.rn.f32x2 vd, va, vb, vc;\n\t"
      "mov.b64 {%0, %1}, vd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add2_f32(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 va, vb, vd;\n\t"
      "mov.b64 va, {%2, %3};\n\tmov.b64 vb, {%4, %5};\n\t"
      "add.rn.f32x2 vd, va, vb;\n\t"
      "mov.b64 {%0, %1}, vd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul2_f32(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 va, vb, vd;\n\t"
      "mov.b64 va, {%2, %3};\n\tmov.b64 vb, {%4, %5};\n\t"
      "mul.rn.f32x2 vd, va, vb;\n\t"
      "mov.b64 {%0, %1}, vd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- own chunk + counts (tcgen05)
// One CTA per tile of 128 rows: P = 128/G consecutive positions of the G query
// heads of one kv head.  The tile's keys are the NK = max(64, P) keys of the
// chunks that hold those positions; S = Q K^T and O = P V run on tcgen05 and
// one thread per row applies the causal own-chunk mask.  Per row it also forms
// the fusion normaliser M' = log(sum_kept exp(s^) + exp(lse_own)) and writes
// the own chunk's weighted output exp(lse_own - M') softmax(s) V
// (= exp(s - M') V) to the fp32 accumulator.
template <int D>
struct CcOwn {
  static constexpr int M = 128;
  static constexpr int KATOMS = D / 64;
  static constexpr uint32_t ATOM = 128 * 128;   // 128 rows x 128 bytes
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = KATOMS * ATOM;
  static constexpr uint32_t OFF_V = OFF_K + KATOMS * ATOM;
  // P (up to 128 keys = two atoms) overwrites Q and K once S = Q K^T is done
  static constexpr uint32_t OFF_P = OFF_Q;
  static constexpr uint32_t OFF_BAR = OFF_V + KATOMS * ATOM;
  static constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
  // S (NK <= 128 columns) is read out before P V overwrites its first D columns
  static constexpr uint32_t TMEM_COLS = 128;
  // more CTAs than 512 / TMEM_COLS per SM (228 KB of shared memory, 1 KB
  // reserved per CTA) could make a tcgen05.alloc wait for columns that a
  // co-resident CTA never frees
  static_assert((512 / TMEM_COLS + 1) * (SMEM + 1024) > 233472u, "TMEM never oversubscribed");
};

struct CcOwnParams {
  CcDims c;
  const int32_t* ids;
  const float* scores;
  float* oacc;
  float* rowstat;
  float* lse_own;
  int P;            // positions per tile
  int n_tiles;      // tiles per kv head
};

template <int D>
__global__ void __launch_bounds__(128)
cc_own_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const CcOwnParams p) {
  using C = CcOwn<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  uint64_t* ld_bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* mma_bar = ld_bar + 1;
  uint64_t* done_bar = ld_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 28);
  const int tid = threadIdx.x, warp = tid >> 5;
  const CcDims& c = p.c;
  const int P = p.P, G = c.G;
  const int NK = P >= kChunk ? P : kChunk;
  const int tile = int(blockIdx.x);
  const int64_t bh = blockIdx.y, b = bh / c.Hkv, h = bh % c.Hkv;
  const int64_t p0 = int64_t(tile) * P;
  const int64_t kbase = (p0 / kChunk) * kChunk;

  if (tid == 0) {
    mbar_init(ld_bar, 1);
    mbar_init(mma_bar, 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    const uint32_t kv_bytes = uint32_t(NK) * 128;
    mbar_arrive_expect_tx(ld_bar, C::KATOMS * (C::ATOM + 2 * kv_bytes));
    for (int g = 0; g < G; ++g) {
      const int y = int((b * c.Hq + h * G + g) * c.n_tok + p0);
#pragma unroll
      for (int a = 0; a < C::KATOMS; ++a) tma_load_2d(smem + C::OFF_Q + a * C::ATOM + g * P * 128, &tm_q, ld_bar, a * 64, y);
    }
    const int yk = int(bh * c.n_tok + kbase);
#pragma unroll
    for (int a = 0; a < C::KATOMS; ++a) {
      tma_load_2d(smem + C::OFF_K + a * C::ATOM, &tm_k, ld_bar, a * 64, yk);
      tma_load_2d(smem + C::OFF_V + a * C::ATOM, &tm_v, ld_bar, a * 64, yk);
    }
  }
  // this thread's row and its kept slots (loads overlap the copies and the MMA)
  const int r = tid;                         // TMEM lane == row of the tile
  const int g = r / P;
  const int64_t pos = p0 + r % P;
  const bool live = pos < c.n_tok;
  const int64_t row = (b * c.Hq + h * G + g) * c.n_tok + pos;
  const int64_t own = pos / kChunk;
  float smax = -INFINITY;
  // K <= 32 (a multiple of 4): the row's kept ids and scores are loaded once,
  // all loads in flight, and kept in registers for both passes
  const bool reg_k = c.K <= 32 && (c.K & 3) == 0;
  int32_t kid[32];
  float ksc[32];
  if (live && reg_k) {
    const int4* i4 = reinterpret_cast<const int4*>(p.ids + row * c.K);
    const float4* s4 = reinterpret_cast<const float4*>(p.scores + row * c.K);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      int4 ci = make_int4(-1, -1, -1, -1);
      float4 sc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < c.K / 4) {
        ci = __ldg(i4 + t);
        sc = __ldg(s4 + t);
      }
      kid[4 * t] = ci.x; kid[4 * t + 1] = ci.y; kid[4 * t + 2] = ci.z; kid[4 * t + 3] = ci.w;
      ksc[4 * t] = sc.x; ksc[4 * t + 1] = sc.y; ksc[4 * t + 2] = sc.z; ksc[4 * t + 3] = sc.w;
    }
#pragma unroll
    for (int t = 0; t < 32; ++t)
      if (kid[t] >= 0 && kid[t] < own) smax = fmaxf(smax, ksc[t]);
  } else if (live) {
    if ((c.K & 3) == 0) {
      const int4* i4 = reinterpret_cast<const int4*>(p.ids + row * c.K);
      const float4* s4 = reinterpret_cast<const float4*>(p.scores + row * c.K);
      for (int t = 0; t < c.K / 4; ++t) {
        const int4 ci = __ldg(i4 + t);
        const float4 sc = __ldg(s4 + t);
        if (ci.x >= 0 && ci.x < own) smax = fmaxf(smax, sc.x);
        if (ci.y >= 0 && ci.y < own) smax = fmaxf(smax, sc.y);
        if (ci.z >= 0 && ci.z < own) smax = fmaxf(smax, sc.z);
        if (ci.w >= 0 && ci.w < own) smax = fmaxf(smax, sc.w);
      }
    } else {
      for (int t = 0; t < c.K; ++t) {
        const int32_t ci = __ldg(p.ids + row * c.K + t);
        if (ci >= 0 && ci < own) smax = fmaxf(smax, __ldg(p.scores + row * c.K + t));
      }
    }
  }
  bool ok = true;
  if (tid == 0) {
    ok = mbar_wait(ld_bar, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const uint32_t sq = smem_u32(smem + C::OFF_Q), sk = smem_u32(smem + C::OFF_K);
      const uint32_t idesc = idesc_bf16(C::M, NK);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = uint32_t((kk >> 2) * C::ATOM + (kk & 3) * 32);
        mma_bf16(tmem, desc_sw128(sq + off), desc_sw128(sk + off), idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(mma_bar);
    }
  }
  ok = __syncthreads_and(ok);
  if (ok) ok = mbar_wait(mma_bar, 0, abort_flag);
  tc_fence_after();
  // causal softmax statistics over the own chunk's keys: tile key j is key
  // kbase + j, valid for j in [jlo, jhi] (same chunk as the row, not after it)
  const uint32_t t_row = tmem + (uint32_t(warp * 32) << 16);
  const int jlo = int(own * kChunk - kbase), jhi = int(pos - kbase);
  const float k2 = c.tau * 1.4426950408889634f;
  float m = -INFINITY;
#pragma unroll 1
  for (int q4 = 0; q4 < NK / 32; ++q4) {
    float tmp[32];
    tmem_ld32(t_row + uint32_t(q4 * 32), tmp);
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const int j = q4 * 32 + t;
      if (j >= jlo && j <= jhi) m = fmaxf(m, tmp[t]);
    }
  }
  float l = 0.f;
#pragma unroll 1
  for (int q4 = 0; q4 < NK / 32; ++q4) {
    float tmp[32];
    tmem_ld32(t_row + uint32_t(q4 * 32), tmp);
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const int j = q4 * 32 + t;
      if (j >= jlo && j <= jhi) l += ex2_approx(fmaf(tmp[t], k2, -m * k2));
    }
  }
  const float lse = m * c.tau + logf(l);   // log sum_j exp(tau s_j)
  // fusion normaliser over the valid kept chunks and the own chunk
  float Mp = lse;
  if (live) {
    const float Mx = fmaxf(smax, lse);
    float Z = expf(lse - Mx);
    if (reg_k) {
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (kid[t] >= 0 && kid[t] < own) Z += expf(ksc[t] - Mx);
    } else {
      for (int t = 0; t < c.K; ++t) {
        const int32_t ci = __ldg(p.ids + row * c.K + t);
        if (ci >= 0 && ci < own) Z += expf(__ldg(p.scores + row * c.K + t) - Mx);
      }
    }
    Mp = Mx + logf(Z);
    p.rowstat[row] = Mp;
    if (p.lse_own) p.lse_own[row] = lse;
  }
  // P = exp(tau s - M') on the causal own-chunk keys, bf16, 128B-swizzled K-major
  const float mb = Mp * 1.4426950408889634f;
#pragma unroll 1
  for (int q4 = 0; q4 < NK / 32; ++q4) {
    float tmp[32];
    tmem_ld32(t_row + uint32_t(q4 * 32), tmp);
    uint8_t* prow = smem + C::OFF_P + (q4 >> 1) * C::ATOM + r * 128;
#pragma unroll
    for (int t = 0; t < 4; ++t) {           // four 16-byte pieces of 8 keys
      uint32_t wd[4];
#pragma unroll
      for (int v2 = 0; v2 < 4; ++v2) {
        float e2[2];
#pragma unroll
        for (int z = 0; z < 2; ++z) {
          const int tt = 8 * t + 2 * v2 + z;
          const int j = q4 * 32 + tt;
          e2[z] = (live && j >= jlo && j <= jhi) ? ex2_approx(fmaf(tmp[tt], k2, -mb)) : 0.f;
        }
        __nv_bfloat162 h2 = __floats2bfloat162_rn(e2[0], e2[1]);
        wd[v2] = *reinterpret_cast<uint32_t*>(&h2);
      }
      const int piece = (q4 & 1) * 4 + t;   // 16-byte piece within the 128-byte row
      *reinterpret_cast<uint4*>(prow + ((piece ^ (r & 7)) << 4)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (tid == 0 && ok) {
    tc_fence_after();
    const uint32_t sp = smem_u32(smem + C::OFF_P), svv = smem_u32(smem + C::OFF_V);
    const uint32_t idesc = idesc_bf16(C::M, D) | (1u << 16);
    for (int kk = 0; kk < NK / 16; ++kk)
      mma_bf16(tmem, desc_sw128(sp + (kk >> 2) * C::ATOM + (kk & 3) * 32),
               desc_sw128_mn(svv + kk * 2048, C::ATOM), idesc, kk > 0 ? 1u : 0u);
    mma_commit(mma_bar);
  }
  if (ok) ok = mbar_wait(mma_bar, 1, abort_flag);
  tc_fence_after();
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    float o[32];
    tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + uint32_t(cc * 32), o);
    if (live && ok) {
      float* dst = p.oacc + row * D + cc * 32;
#pragma unroll
      for (int t = 0; t < 32; t += 4) *reinterpret_cast<float4*>(dst + t) = make_float4(o[t], o[t + 1], o[t + 2], o[t + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && !ok) {
    // after a time-out: let the copies land and any issued MMA finish before TMEM is freed
    mbar_wait_drain(ld_bar, 0);
    mma_commit(done_bar);
    mbar_wait_drain(done_bar, 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- pair counts
// Each CTA takes kCountRows consecutive rows of one query head (inside one
// window) and counts their kept pairs per chunk in a shared-memory histogram;
// a pair's rank among the CTA's pairs of its chunk is the histogram's old
// value.  Then each touched chunk's count goes to the global per-key count
// with one atomic, whose old value -- the base of this CTA's pairs of that
// chunk -- is stored in cbase[CTA][chunk].  A pair's position within its key
// is cbase + its rank; the fill adds the two, so the ids and ranks are read
// once here.  Ids outside the row's candidates are recorded as
// HILS_ERR_DEVICE_BOUNDS and skipped.
constexpr int kCountRows = 4096;
constexpr int kCountThreads = 1024;

__global__ void __launch_bounds__(kCountThreads)
cc_count_kernel(const int32_t* __restrict__ ids, int32_t* __restrict__ counts, int32_t* __restrict__ ranks,
                int32_t* __restrict__ cbase, const CcDims c) {
  extern __shared__ int32_t hist[];   // [nc]
  const int64_t row0 = int64_t(blockIdx.x) * kCountRows;   // rows of one (b, hq); kCountRows | n_tok
  const int64_t bhq = row0 / c.n_tok, i0 = row0 % c.n_tok;
  const int64_t b = bhq / c.Hq, hq = bhq % c.Hq;
  const int64_t bh = b * c.Hkv + hq / c.G;
  const int64_t key0 = cc_key(c, bh, i0, 0);
  const int64_t nch = (i0 + kCountRows - 1) / kChunk;   // candidates of the last row
  for (int64_t t = threadIdx.x; t < nch; t += blockDim.x) hist[t] = 0;
  __syncthreads();
  const int64_t n = int64_t(kCountRows) * c.K;
  const int32_t* id0 = ids + row0 * c.K;
  int32_t* rk0 = ranks + row0 * c.K;
  if ((c.K & 3) == 0) {
    // four slots of one row per step, 16-byte loads and stores
    const int64_t n4 = n / 4;
    const int4* id4 = reinterpret_cast<const int4*>(id0);
    int4* rk4 = reinterpret_cast<int4*>(rk0);
#pragma unroll 4
    for (int64_t t = threadIdx.x; t < n4; t += blockDim.x) {
      const int4 ci = __ldg(id4 + t);
      const int64_t nc_i = n_candidates(i0 + (4 * t) / c.K, c.wm1);
      const int32_t cv[4] = {ci.x, ci.y, ci.z, ci.w};
      int32_t r[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        r[e] = 0;
        if (cv[e] >= nc_i) record_error(HILS_ERR_DEVICE_BOUNDS);
        if (cv[e] >= 0 && cv[e] < nc_i) r[e] = atomicAdd(hist + cv[e], 1);
      }
      rk4[t] = make_int4(r[0], r[1], r[2], r[3]);
    }
  } else {
    for (int64_t t = threadIdx.x; t < n; t += blockDim.x) {
      const int32_t ci = __ldg(id0 + t);
      if (ci < 0) continue;
      const int64_t i = i0 + t / c.K;
      if (ci >= n_candidates(i, c.wm1)) {
        record_error(HILS_ERR_DEVICE_BOUNDS);
        continue;
      }
      rk0[t] = atomicAdd(hist + ci, 1);
    }
  }
  __syncthreads();
  // chunks no pair of this CTA touched keep stale entries: no pair reads them
  int32_t* cb = cbase + int64_t(blockIdx.x) * c.nc;
  for (int64_t t = threadIdx.x; t < nch; t += blockDim.x) {
    const int32_t h = hist[t];
    if (h > 0) cb[t] = atomicAdd(counts + key0 + t, h);
  }
}

// Fallback for shapes the histogram does not fit: one global atomic per pair.
__global__ void __launch_bounds__(256)
cc_count_direct_kernel(const int32_t* __restrict__ ids, int32_t* __restrict__ counts, int32_t* __restrict__ ranks,
                       const CcDims c, int64_t n_slots) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n_slots) return;
  const int32_t ci = __ldg(ids + idx);
  if (ci < 0) return;
  const int64_t row = idx / c.K;
  const int64_t bhq = row / c.n_tok, i = row % c.n_tok;
  if (ci >= n_candidates(i, c.wm1)) {
    record_error(HILS_ERR_DEVICE_BOUNDS);
    return;
  }
  const int64_t b = bhq / c.Hq, hq = bhq % c.Hq;
  const int64_t bh = b * c.Hkv + hq / c.G;
  ranks[idx] = atomicAdd(counts + cc_key(c, bh, i, ci), 1);
}

// ---------------------------------------------------------------- scan (three passes)
constexpr int kCcTileRows = 128;
constexpr int kScanBlock = 4096;   // keys per CTA (256 threads x 16)

__device__ __forceinline__ int64_t cc_tiles(int64_t cnt) { return (cnt + kCcTileRows - 1) / kCcTileRows; }

// pass 1: per-CTA totals of pairs and tiles
__global__ void __launch_bounds__(256)
cc_scan_sums_kernel(const int32_t* __restrict__ counts, int64_t n_keys, int64_t* __restrict__ sums) {
  __shared__ int64_t sa[8], st[8];
  const int64_t k0 = int64_t(blockIdx.x) * kScanBlock + threadIdx.x * 16;
  int64_t a = 0, t = 0;
#pragma unroll 4
  for (int e = 0; e < 16; ++e) {
    const int64_t kk = k0 + e;
    const int64_t c = kk < n_keys ? counts[kk] : 0;
    a += c;
    t += cc_tiles(c);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  if ((threadIdx.x & 31) == 0) { sa[threadIdx.x >> 5] = a; st[threadIdx.x >> 5] = t; }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t A = 0, T = 0;
    for (int w = 0; w < 8; ++w) { A += sa[w]; T += st[w]; }
    sums[2 * blockIdx.x] = A;
    sums[2 * blockIdx.x + 1] = T;
  }
}

// pass 2 (one CTA): exclusive prefix of the per-CTA totals, in place; also the grand totals
__global__ void __launch_bounds__(1024)
cc_scan_blocks_kernel(int64_t* __restrict__ sums, int64_t n_blocks, int64_t n_keys, int64_t* __restrict__ offsets,
                      int32_t* __restrict__ tile_start) {
  __shared__ int64_t wa[32], wt[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t per = (n_blocks + 1023) / 1024;
  const int64_t b0 = tid * per, b1 = (b0 + per < n_blocks) ? b0 + per : n_blocks;
  int64_t a = 0, t = 0;
  for (int64_t b = b0; b < b1; ++b) { a += sums[2 * b]; t += sums[2 * b + 1]; }
  int64_t ia = a, it = t;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t ya = __shfl_up_sync(0xffffffffu, ia, o), yt = __shfl_up_sync(0xffffffffu, it, o);
    if (lane >= o) { ia += ya; it += yt; }
  }
  if (lane == 31) { wa[warp] = ia; wt[warp] = it; }
  __syncthreads();
  int64_t pa = 0, pt = 0, TA = 0, TT = 0;
  for (int w = 0; w < 32; ++w) {
    if (w < warp) { pa += wa[w]; pt += wt[w]; }
    TA += wa[w];
    TT += wt[w];
  }
  int64_t ra = pa + ia - a, rt = pt + it - t;
  for (int64_t b = b0; b < b1; ++b) {
    const int64_t xa = sums[2 * b], xt = sums[2 * b + 1];
    sums[2 * b] = ra;
    sums[2 * b + 1] = rt;
    ra += xa;
    rt += xt;
  }
  if (tid == 0) {
    offsets[n_keys] = TA;
    tile_start[n_keys] = int32_t(TT);
  }
}

// pass 3: per-key offsets, tile starts and the tile -> key table
__global__ void __launch_bounds__(256)
cc_scan_apply_kernel(const int32_t* __restrict__ counts, const CcDims c, const int64_t* __restrict__ sums,
                     int64_t* __restrict__ offsets, int32_t* __restrict__ tile_start, int4* __restrict__ items) {
  const int64_t n_keys = c.n_keys;
  __shared__ int64_t sa[8], st[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t k0 = int64_t(blockIdx.x) * kScanBlock + threadIdx.x * 16;
  int64_t cnt[16];
  int64_t a = 0, t = 0;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int64_t kk = k0 + e;
    cnt[e] = kk < n_keys ? counts[kk] : 0;
    a += cnt[e];
    t += cc_tiles(cnt[e]);
  }
  int64_t ia = a, it = t;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t ya = __shfl_up_sync(0xffffffffu, ia, o), yt = __shfl_up_sync(0xffffffffu, it, o);
    if (lane >= o) { ia += ya; it += yt; }
  }
  if (lane == 31) { sa[warp] = ia; st[warp] = it; }
  __syncthreads();
  int64_t pa = sums[2 * blockIdx.x], pt = sums[2 * blockIdx.x + 1];
  for (int w = 0; w < warp; ++w) { pa += sa[w]; pt += st[w]; }
  int64_t ra = pa + ia - a, rt = pt + it - t;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int64_t kk = k0 + e;
    if (kk >= n_keys) break;
    offsets[kk] = ra;
    tile_start[kk] = int32_t(rt);
    const int64_t tl = cc_tiles(cnt[e]);
    const int64_t bh = kk / (int64_t(c.n_win) * c.nc), chunk = kk % c.nc;
    const int32_t kvrow = int32_t(bh * c.n_tok + chunk * kChunk);
    for (int64_t u = 0; u < tl; ++u) {
      const int64_t left = cnt[e] - u * kCcTileRows;
      items[rt + u] = make_int4(int32_t(ra + u * kCcTileRows), kvrow, int32_t(left < kCcTileRows ? left : kCcTileRows), 0);
    }
    ra += cnt[e];
    rt += tl;
  }
}

// ---------------------------------------------------------------- fill the inverted index
// A pair's position within its key's list is known from the count: its rank
// among its count CTA's pairs of the chunk (ranks[slot]) plus that CTA's base
// for the chunk (cbase; null when the count took one global atomic per pair,
// whose old value is the position itself), so filling is a plain scatter of
// the pair's global row id and its fusion factor s^ - M'.
__global__ void __launch_bounds__(256)
cc_fill_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ ranks, const int32_t* __restrict__ cbase,
               const float* __restrict__ scores, const float* __restrict__ rowstat,
               const int64_t* __restrict__ offsets, int2* __restrict__ e_pair, const CcDims c, int64_t n_slots) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n_slots) return;
  const int32_t ci = __ldg(ids + idx);
  if (ci < 0) return;
  const int64_t row = idx / c.K;
  const int64_t bhq = row / c.n_tok, i = row % c.n_tok;
  if (ci >= n_candidates(i, c.wm1)) return;   // out of range: recorded when counting
  const int64_t b = bhq / c.Hq, hq = bhq % c.Hq;
  const int64_t bh = b * c.Hkv + hq / c.G;
  int64_t at = offsets[cc_key(c, bh, i, ci)] + __ldg(ranks + idx);
  if (cbase) at += __ldg(cbase + (row / kCountRows) * c.nc + ci);
  // one 8-byte record per pair: the row and its fusion factor
  e_pair[at] = make_int2(int32_t(row), __float_as_int(__ldg(scores + idx) - __ldg(rowstat + row)));
}

// The same scatter four slots of one row per thread (K a multiple of 4):
// 16-byte loads of ids, ranks and scores, one row statistic, and the four
// independent offset loads in flight together.
__global__ void __launch_bounds__(256)
cc_fill4_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ ranks, const int32_t* __restrict__ cbase,
                const float* __restrict__ scores, const float* __restrict__ rowstat,
                const int64_t* __restrict__ offsets, int2* __restrict__ e_pair, const CcDims c, int64_t n_quads) {
  const int64_t qd = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (qd >= n_quads) return;
  const int64_t idx = qd * 4;
  const int4 ci = __ldg(reinterpret_cast<const int4*>(ids) + qd);
  const int4 rk = __ldg(reinterpret_cast<const int4*>(ranks) + qd);
  const float4 sc = __ldg(reinterpret_cast<const float4*>(scores) + qd);
  const int64_t row = idx / c.K;
  const int64_t bhq = row / c.n_tok, i = row % c.n_tok;
  const int64_t n_cand = n_candidates(i, c.wm1);
  const int64_t b = bhq / c.Hq, hq = bhq % c.Hq;
  const int64_t bh = b * c.Hkv + hq / c.G;
  const float ms = __ldg(rowstat + row);
  const int32_t cv[4] = {ci.x, ci.y, ci.z, ci.w};
  const int32_t rv[4] = {rk.x, rk.y, rk.z, rk.w};
  const float sv[4] = {sc.x, sc.y, sc.z, sc.w};
  const int32_t* cb = cbase ? cbase + (row / kCountRows) * c.nc : nullptr;
  int64_t at[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {   // out-of-range ids were recorded when counting
    const bool ok = cv[e] >= 0 && cv[e] < n_cand;
    at[e] = ok ? offsets[cc_key(c, bh, i, cv[e])] + rv[e] + (cb ? __ldg(cb + cv[e]) : 0) : -1;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (at[e] >= 0) e_pair[at[e]] = make_int2(int32_t(row), __float_as_int(sv[e] - ms));
}

// ---------------------------------------------------------------- chunk scores, recomputed
// For a prefill called without the scores hils_select returned: s^ of every
// kept (row, slot) from the query row and the bf16 scoring operand, with the
// tensor-core selection's arithmetic (aitrends.kr article, section "방법론":
// s^ = tau <q, k'> + b'; here tau * (<q, k'_bf16> + x_hi + x_lo), products
// exact and summed in fp32, so only the order of the sums differs).  One
// thread per slot; the K threads of a row read the same query row.  Padding
// (-1) and ids outside the row's candidates (recorded when the pairs are
// counted) get -inf.
template <int D>
__global__ void __launch_bounds__(256)
cc_rescore_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kmma,
                  const int32_t* __restrict__ ids, float* __restrict__ scores, const CcDims c, int64_t n_slots) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n_slots) return;
  const int32_t ci = __ldg(ids + idx);
  const int64_t row = idx / c.K;
  const int64_t bhq = row / c.n_tok, i = row % c.n_tok;
  if (ci < 0 || ci >= n_candidates(i, c.wm1)) {
    scores[idx] = -INFINITY;
    return;
  }
  const int64_t b = bhq / c.Hq, hq = bhq % c.Hq;
  const int64_t bh = b * c.Hkv + hq / c.G;
  const __nv_bfloat16* kr = kmma + (bh * c.nc + ci) * (D + kExt);
  const __nv_bfloat16* qr = q + row * D;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < D; t += 8) {
    float qv[8], kv[8];
    Vec16<__nv_bfloat16>::load(qr + t, qv);
    Vec16<__nv_bfloat16>::load(kr + t, kv);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e & 3] = fmaf(qv[e], kv[e], acc[e & 3]);
  }
  const float x = __bfloat162float(kr[D]) + __bfloat162float(kr[D + 1]);
  scores[idx] = c.tau * (((acc[0] + acc[1]) + (acc[2] + acc[3])) + x);
}

// ---------------------------------------------------------------- accumulator -> output
template <int D>
__global__ void __launch_bounds__(256)
cc_final_kernel(const float* __restrict__ oacc, __nv_bfloat16* __restrict__ o, int64_t n_vec8) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n_vec8) return;
  const float4 a = __ldcs(reinterpret_cast<const float4*>(oacc) + 2 * idx);
  const float4 b = __ldcs(reinterpret_cast<const float4*>(oacc) + 2 * idx + 1);
  float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  Vec16<__nv_bfloat16>::store(o + idx * 8, x);
}

// ---------------------------------------------------------------- chunk tiles on tcgen05
// Warp-specialised, two-stage pipeline per CTA over its tiles (item = blockIdx.x
// + j * gridDim.x), persistent with two CTAs per SM:
//   warp 0       producer: tile records three tiles ahead and their entries
//                (row id, fusion factor s^ - M') two tiles ahead, held in named
//                registers; per tile the entries go to the stage's shared
//                memory, one lane issues TMA loads of the chunk's K and V, and
//                every lane issues the gather4 loads of its four query rows
//                (128B swizzle);
//   warp 1       one lane issues S = Q K^T into TMEM buffer b, and once the
//                softmax warps have written P, O = P V into TMEM buffer b
//                (A = P from tensor memory), then releases the stage;
//   warps 2-5    one thread per row: softmax of its 64 scores into P (bf16,
//                over the row's own S columns in tensor memory, so no shared
//                memory store and no proxy fence); the softmax of tile j+1 runs before
//                tile j's output rows are staged in a separate padded buffer
//                and added to the accumulator (one bulk reduction per row at
//                d = 64, coalesced 16-byte reductions per warp row at d = 128).
// Stage / TMEM buffer b = j & 1, so loading tile j+1 and the MMAs of tile j+1
// overlap the softmax and reductions of tile j.
template <int D>
struct CcTc {
  static constexpr int M = kCcTileRows;
  static constexpr int KATOMS = D / 64;
  static constexpr int NS = 2;                      // shared-memory load stages
  static constexpr uint32_t Q_ATOM = M * 128;       // 16 KB
  static constexpr uint32_t KV_ATOM = kChunk * 128; // 8 KB
  static constexpr uint32_t Q_BYTES = KATOMS * Q_ATOM;
  static constexpr uint32_t K_BYTES = KATOMS * KV_ATOM;
  // P (bf16, two per 32-bit column) overwrites its own S columns in tensor
  // memory and is the A operand of P V from there; the stage goes back to
  // the producer as soon as P V is done.  A separate buffer holds a
  // tile's fp32 output rows (4D bytes each, padded to a 4D + 16 byte stride
  // so the row-per-thread stores of 8 consecutive rows hit distinct banks)
  // until the bulk reductions have read them.
  static constexpr uint32_t O_ROW = D * 4;
  static constexpr uint32_t O_STRIDE = O_ROW + 16;
  static constexpr uint32_t STAGE = Q_BYTES + 2 * K_BYTES;
  static constexpr uint32_t OFF_Q = 0, OFF_K = Q_BYTES, OFF_V = OFF_K + K_BYTES;
  static constexpr uint32_t OFF_O = NS * STAGE;
  static constexpr uint32_t O_BYTES = (M * O_STRIDE + 1023u) & ~1023u;
  static constexpr uint32_t OFF_META = OFF_O + O_BYTES;           // per stage: rows[128] i32, fac[128] f32, n
  static constexpr uint32_t META = M * 4 + M * 4 + 16;
  static constexpr uint32_t OFF_BAR = OFF_META + NS * META;
  static constexpr uint32_t SMEM_MIN = OFF_BAR + 16 * 8 + 32 + 1024;
  static constexpr uint32_t TMEM_COLS = D == 64 ? 256 : 512;    // S[2] x 64 + O[2] x D
  static constexpr uint32_t MAX_CTAS = 512 / TMEM_COLS;
  // at most MAX_CTAS CTAs may share an SM, or a tcgen05.alloc could wait for
  // columns that a co-resident persistent CTA never frees
  static constexpr uint32_t SMEM_FLOOR = 233472u / (MAX_CTAS + 1) + 1024u;
  static constexpr uint32_t SMEM = SMEM_MIN > SMEM_FLOOR ? SMEM_MIN : SMEM_FLOOR;
  static_assert((512 / TMEM_COLS + 1) * (SMEM + 1024) > 233472u, "TMEM never oversubscribed");
  static constexpr uint32_t TX_BYTES = M * D * 2 + 2 * K_BYTES;
  static constexpr uint32_t IDESC_S = sm100::idesc_bf16(M, kChunk);
  // P (in tensor memory, K-major) x V (MN-major: d contiguous in each key row)
  static constexpr uint32_t IDESC_O = sm100::idesc_bf16(M, D) | (1u << 16);
  static constexpr int THREADS = 192;
};

struct CcTcParams {
  CcDims c;
  const int32_t* tile_start;   // [n_keys + 1]; the last entry is the number of tiles
  const int4* items;           // per tile: first entry, K/V row, pair count
  const int2* e_pair;          // per entry: global row id, s^ - M' (float bits)
  float* oacc;
};

template <int D>
__global__ void __launch_bounds__(CcTc<D>::THREADS, 1)
cc_attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const CcTcParams p) {
  using C = CcTc<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* load_full = bars;        // [NS] producer -> MMA, softmax
  uint64_t* load_empty = bars + 3;   // [NS] MMA (after P V) -> producer
  uint64_t* p_full = bars + 6;       // [NS] softmax -> MMA
  uint64_t* s_full = bars + 9;       // [2] MMA -> softmax
  uint64_t* o_full = bars + 11;      // [2] MMA -> epilogue
  uint64_t* t_empty = bars + 13;     // [2] epilogue -> MMA
  uint64_t* done = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 16 * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 16 * 8 + 4);
  int* issued_slot = reinterpret_cast<int*>(smem + C::OFF_BAR + 16 * 8 + 8);
  int* consumed_slot = reinterpret_cast<int*>(smem + C::OFF_BAR + 16 * 8 + 12);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const CcDims& c = p.c;

  if (tid == 0) {
    for (int t = 0; t < C::NS; ++t) {
      mbar_init(&load_full[t], 1);
      mbar_init(&load_empty[t], 1);
      mbar_init(&p_full[t], 4);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&o_full[t], 1);
      mbar_init(&t_empty[t], 4);
    }
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t n_items = p.tile_start[c.n_keys];
  const int n_my = n_items > int32_t(blockIdx.x) ? (n_items - 1 - int32_t(blockIdx.x)) / int32_t(gridDim.x) + 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane l owns rows 4l..4l+3 of every tile: it loads their row ids and
    // fusion factors two tiles ahead and issues their gather4 itself, so the
    // 32 gathers of a tile are issued in parallel.
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    // Tile records are fetched three tiles ahead and their entries two tiles
    // ahead, held in named registers that shift by one tile per iteration
    // (an array indexed by the tile counter would live in local memory and
    // make every load wait at once).
    auto fetch_rec = [&](int jj) {
      return __ldg(p.items + int32_t(blockIdx.x) + jj * int32_t(gridDim.x));
    };
    auto fetch_entries = [&](const int4& r, int32_t (&row)[4], float (&fac)[4]) {
      const int base = r.x + 4 * lane;   // entries are padded past the last tile
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int2 e = __ldg(p.e_pair + base + t);
        row[t] = e.x;
        fac[t] = __int_as_float(e.y);
      }
    };
    int4 r0 = make_int4(0, 0, 0, 0), r1 = r0, r2 = r0;
    int32_t row0[4] = {0, 0, 0, 0}, row1[4] = {0, 0, 0, 0};
    float fac0[4] = {0.f, 0.f, 0.f, 0.f}, fac1[4] = {0.f, 0.f, 0.f, 0.f};
    if (n_my > 0) { r0 = fetch_rec(0); fetch_entries(r0, row0, fac0); }
    if (n_my > 1) { r1 = fetch_rec(1); fetch_entries(r1, row1, fac1); }
    if (n_my > 2) r2 = fetch_rec(2);
    int j = 0;
    for (; j < n_my; ++j) {
      const int s = j % C::NS, u = j / C::NS;
      const int4 cur = r0;
      int32_t crow[4];
      float cfac[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        crow[t] = row0[t];
        cfac[t] = fac0[t];
        row0[t] = row1[t];
        fac0[t] = fac1[t];
      }
      r0 = r1;
      r1 = r2;
      if (j + 3 < n_my) r2 = fetch_rec(j + 3);
      if (j + 2 < n_my) fetch_entries(r1, row1, fac1);
      if (!mbar_wait(&load_empty[s], (u & 1) ^ 1, abort_flag)) break;
      uint8_t* meta = smem + C::OFF_META + s * C::META;
      *reinterpret_cast<int4*>(meta + 16 * lane) = make_int4(crow[0], crow[1], crow[2], crow[3]);
      *reinterpret_cast<float4*>(meta + C::M * 4 + 16 * lane) = make_float4(cfac[0], cfac[1], cfac[2], cfac[3]);
      if (lane == 0) reinterpret_cast<int32_t*>(meta + C::M * 8)[0] = cur.z;
      uint8_t* st = smem + s * C::STAGE;
      if (lane == 0) {
        mbar_arrive_expect_tx(&load_full[s], C::TX_BYTES);
#pragma unroll
        for (int a = 0; a < C::KATOMS; ++a) {
          tma_load_2d(st + C::OFF_K + a * C::KV_ATOM, &tm_k, &load_full[s], a * 64, cur.y);
          tma_load_2d(st + C::OFF_V + a * C::KV_ATOM, &tm_v, &load_full[s], a * 64, cur.y);
        }
      }
      __syncwarp();
      const uint32_t qdst = smem_u32(st + C::OFF_Q) + uint32_t(4 * lane) * 128;
#pragma unroll
      for (int a = 0; a < C::KATOMS; ++a)
        tma_gather4(qdst + a * C::Q_ATOM, &tm_q, &load_full[s], a * 64, crow[0], crow[1], crow[2], crow[3]);
      __syncwarp();
    }
    if (lane == 0) *issued_slot = j;
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int j = 0;
      for (; j < n_my; ++j) {
        const int s = j % C::NS, u = j / C::NS, b = j & 1, ub = j >> 1;
        if (!mbar_wait(&load_full[s], u & 1, abort_flag)) break;
        if (!mbar_wait(&t_empty[b], (ub & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * C::STAGE);
        const uint32_t sq = st + C::OFF_Q, sk = st + C::OFF_K, sv = st + C::OFF_V;
        const uint32_t t_s = tmem + uint32_t(b * kChunk), t_o = tmem + uint32_t(2 * kChunk + b * D);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = uint32_t((kk >> 2) * C::Q_ATOM + (kk & 3) * 32);
          const uint32_t offk = uint32_t((kk >> 2) * C::KV_ATOM + (kk & 3) * 32);
          mma_bf16(t_s, desc_sw128(sq + off), desc_sw128(sk + offk), C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[b]);
        if (!mbar_wait(&p_full[s], u & 1, abort_flag)) { ++j; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          mma_bf16_tmem_a(t_o, t_s + uint32_t(kk * 8), desc_sw128_mn(sv + kk * 2048, C::KV_ATOM), C::IDESC_O,
                          kk > 0 ? 1u : 0u);
        mma_commit(&o_full[b]);
        mma_commit(&load_empty[s]);
      }
      *consumed_slot = j;
      mma_commit(done);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Software-pipelined: the softmax of tile j+1 runs while the tensor core
    // does P V of tile j, then tile j's output is written.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t t_lane = uint32_t(quarter * 32) << 16;
    const float k2 = c.tau * 1.4426950408889634f;   // scores in log2 units
    // softmax of tile jj: P into its own S columns in tensor memory; returns
    // the row's global row id (-1 when the row is not live) or -2 on abort
    auto softmax_tile = [&](int jj) -> int64_t {
      const int s = jj % C::NS, u = jj / C::NS, b = jj & 1, ub = jj >> 1;
      if (!mbar_wait(&load_full[s], u & 1, abort_flag)) return -2;
      const uint8_t* meta = smem + C::OFF_META + s * C::META;
      const int n = reinterpret_cast<const int32_t*>(meta + C::M * 8)[0];
      const bool live = r < n;
      const int64_t grow = reinterpret_cast<const int32_t*>(meta)[r];
      const float fac = reinterpret_cast<const float*>(meta + C::M * 4)[r];
      if (!mbar_wait(&s_full[b], ub & 1, abort_flag)) return -2;
      tc_fence_after();
      float sc[64];
      {
        float tmp[32];
        tmem_ld32(tmem + t_lane + uint32_t(b * kChunk), tmp);
#pragma unroll
        for (int t = 0; t < 32; ++t) sc[t] = tmp[t];
        tmem_ld32(tmem + t_lane + uint32_t(b * kChunk + 32), tmp);
#pragma unroll
        for (int t = 0; t < 32; ++t) sc[32 + t] = tmp[t];
      }
      uint32_t pw[32];   // the row's P, two bf16 per word (zero when the row is not live)
      if (live) {
        // short dependency chains: a tree of three-input maxima, four partial sums
        float mx[22];
#pragma unroll
        for (int t = 0; t < 21; ++t) mx[t] = fmax3_f32(sc[3 * t], sc[3 * t + 1], sc[3 * t + 2]);
        mx[21] = sc[63];
#pragma unroll
        for (int t = 0; t < 7; ++t) mx[t] = fmax3_f32(mx[3 * t], mx[3 * t + 1], mx[3 * t + 2]);
        const float m = fmaxf(fmax3_f32(fmax3_f32(mx[0], mx[1], mx[2]), fmax3_f32(mx[3], mx[4], mx[5]), mx[6]), mx[21]);
        const float mb = m * k2;
        // scores in pairs: one packed FMA, two exponentials, one packed add
        // into four partial sums (lane pairs (0,1) and (2,3) of each 4 keys)
        float lp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          float x0, x1;
          fma2_f32(x0, x1, sc[2 * t], sc[2 * t + 1], k2, k2, -mb, -mb);
          sc[2 * t] = ex2_approx(x0);
          sc[2 * t + 1] = ex2_approx(x1);
          const int a = 2 * (t & 1);
          add2_f32(lp[a], lp[a + 1], lp[a], lp[a + 1], sc[2 * t], sc[2 * t + 1]);
        }
        const float l = (lp[0] + lp[1]) + (lp[2] + lp[3]);
        const float w = expf(fac) / l;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          float y0, y1;
          mul2_f32(y0, y1, sc[2 * t], sc[2 * t + 1], w, w);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
          pw[t] = *reinterpret_cast<uint32_t*>(&h2);
        }
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) pw[t] = 0u;
      }
      // the whole warp, converged: S of this tile has been read into registers
      tmem_st32(tmem + t_lane + uint32_t(b * kChunk), pw);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[s]);
      return live ? grow : -1;
    };
    // output of tile jj: each thread stages its fp32 output row in the output
    // buffer (once the previous tile's rows have been read out of it), then
    // the rows are added to the accumulator.  d = 64: one bulk reduction per
    // row (256 B) by the bulk-copy unit.  d = 128: the warp reads its 32 rows
    // back D / 4 lanes per row and adds them with coalesced 16-byte
    // reductions, one row per instruction (measured faster at d = 128,
    // slower at d = 64).
    constexpr int LPR = D / 4;            // lanes per row
    constexpr int RPI = 32 / LPR;         // rows per instruction
    constexpr bool kBulk = D == 64;
    const uint32_t orow = smem_u32(smem + C::OFF_O) + uint32_t(r) * C::O_STRIDE;
    const uint32_t obase = smem_u32(smem + C::OFF_O) + uint32_t(quarter * 32) * C::O_STRIDE;
    auto output_tile = [&](int jj, int64_t grow) -> bool {
      const int b = jj & 1, ub = jj >> 1;
      if (!mbar_wait(&o_full[b], ub & 1, abort_flag)) return false;
      tc_fence_after();
      if constexpr (kBulk) bulk_wait_read<0>();
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        tmem_ld32(tmem + t_lane + uint32_t(2 * kChunk + b * D + cc * 32), o);
#pragma unroll
        for (int t = 0; t < 32; t += 4)
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(orow + uint32_t(cc * 32 + t) * 4), "f"(o[t]),
                       "f"(o[t + 1]), "f"(o[t + 2]), "f"(o[t + 3])
                       : "memory");
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[b]);
      if constexpr (kBulk) {
        fence_proxy_async_smem();
        if (grow >= 0) bulk_reduce_add_f32(p.oacc + grow * D, orow, C::O_ROW);
        bulk_commit();
      } else {
        const int32_t g32 = int32_t(grow);   // rows < 2^31; -1 when the row is not live
        const int sub = lane / LPR, col = (lane % LPR) * 4;
#pragma unroll 4
        for (int i = 0; i < 32; i += RPI) {
          const int rr = i + sub;
          const int32_t g = __shfl_sync(0xffffffffu, g32, rr);
          float4 val;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(val.x), "=f"(val.y), "=f"(val.z), "=f"(val.w)
                       : "r"(obase + uint32_t(rr) * C::O_STRIDE + uint32_t(col) * 4)
                       : "memory");
          if (g >= 0) red_add_v4(p.oacc + int64_t(g) * D + col, val.x, val.y, val.z, val.w);
        }
        __syncwarp();
      }
      return true;
    };
    int64_t g_cur = n_my > 0 ? softmax_tile(0) : -2;
    for (int j = 0; j < n_my && g_cur != -2; ++j) {
      const int64_t g_next = j + 1 < n_my ? softmax_tile(j + 1) : -1;
      if (g_next == -2) break;
      if (!output_tile(j, g_cur)) break;
      g_cur = g_next;
    }
    bulk_wait_all();
  }
  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (tid == 0) {
    // loads still in flight (only after an abort): wait for them to land
    for (int j = *consumed_slot; j < *issued_slot; ++j) mbar_wait_drain(&load_full[j % C::NS], (j / C::NS) & 1);
  }
  if (warp == 1) {
    if (lane == 0 && n_my > 0) mbar_wait_drain(done, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace hils
