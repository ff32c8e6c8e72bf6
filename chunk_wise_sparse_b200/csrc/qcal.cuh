// Q-Cal: low-rank query calibration for the chunk scores.
//
// aitrends.kr article, section "방법론" (Methodology) and glossary entry
// "저계수 쿼리 보정" (low-rank query calibration): a light adapter applies a
// low-rank down/up projection to the query; the calibrated query q^ scores
// the chunks.  Read as residual and per query head:
//     q^ = q + W_up (W_down q),   W_down [r x d], W_up [d x r],
// q^ replaces q in s^ = tau <q^, k'_c> + b'_c (selection and fusion
// weights); the attention inside chunks keeps q.
//
// Two kernels:
//   qcal_tc_kernel   bf16, tiles of 128 positions of one (b, hq): two chained
//                    tcgen05 MMAs, T = Q W_down^T (128 x 64, the rank
//                    zero-padded to 64) and D = T W_up^T (128 x d), T passing
//                    through shared memory in bf16; q^ = q + D is written
//                    over the Q tile and leaves by a TMA store that clips at
//                    the end of the sequence.  HBM-bound: 4d bytes per row.
//   qcal_simt_kernel fp32 (and bf16 with few positions, e.g. a decode
//                    step): one warp per row, r lanes for W_down q, the d
//                    outputs spread over the lanes.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace hils {

constexpr int kQcalMaxRank = 64;

template <typename T, int D>
__global__ void __launch_bounds__(128)
qcal_simt_kernel(const T* q, const T* __restrict__ w_down, const T* __restrict__ w_up, int r,
                 int64_t n_pos, int Hq, int64_t n_rows, T* out) {   // out may be q (in place)
  constexpr int EL = D / 32;   // outputs per lane
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= n_rows) return;
  const int hq = int((row / n_pos) % Hq);
  const T* wd = w_down + int64_t(hq) * r * D;
  const T* wu = w_up + int64_t(hq) * D * r;
  auto f = [](T x) -> float {
    if constexpr (sizeof(T) == 2) return __bfloat162float(x);
    else return x;
  };
  float xv[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) xv[e] = f(q[row * D + lane * EL + e]);
  // z_a = <W_down[a], q>: lane a (and a + 32) owns z_a
  float z0 = 0.f, z1 = 0.f;
#pragma unroll
  for (int t = 0; t < D; ++t) {
    const float xt = __shfl_sync(0xffffffffu, xv[t % EL], t / EL);
    if (lane < r) z0 = fmaf(f(__ldg(wd + int64_t(lane) * D + t)), xt, z0);
    if (lane + 32 < r) z1 = fmaf(f(__ldg(wd + int64_t(lane + 32) * D + t)), xt, z1);
  }
  float y[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) y[e] = xv[e];
  for (int a = 0; a < r; ++a) {
    const float za = __shfl_sync(0xffffffffu, a < 32 ? z0 : z1, a & 31);
#pragma unroll
    for (int e = 0; e < EL; ++e) y[e] = fmaf(f(__ldg(wu + int64_t(lane * EL + e) * r + a)), za, y[e]);
  }
#pragma unroll
  for (int e = 0; e < EL; ++e) {
    if constexpr (sizeof(T) == 2) out[row * D + lane * EL + e] = __float2bfloat16_rn(y[e]);
    else out[row * D + lane * EL + e] = y[e];
  }
}

template <int D>
struct QcalTc {
  static constexpr int M = 128;
  static constexpr int KATOMS = D / 64;
  static constexpr int RP = kQcalMaxRank;               // padded rank
  static constexpr uint32_t Q_ATOM = M * 128;           // 128 rows x 64 elements
  static constexpr uint32_t WD_ATOM = RP * 128;         // 64 rank rows x 64 elements
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_WD = OFF_Q + KATOMS * Q_ATOM;
  static constexpr uint32_t OFF_WU = OFF_WD + KATOMS * WD_ATOM;   // D rows x 64 rank elements
  static constexpr uint32_t OFF_T = OFF_WU + D * 128;              // 128 rows x 64 rank elements
  static constexpr uint32_t OFF_BAR = OFF_T + M * 128;
  static constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
  // T (64 columns) is read out before D (D columns) overwrites it
  static constexpr uint32_t TMEM_COLS = D;
  static_assert((512 / TMEM_COLS + 1) * (SMEM + 1024) > 233472u, "TMEM never oversubscribed");
};

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(sm100::smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(sm100::smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(sm100::smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(128)
qcal_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
               const __nv_bfloat16* __restrict__ w_down, const __nv_bfloat16* __restrict__ w_up, int r, int Hq) {
  using C = QcalTc<D>;
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
  const int p0 = int(blockIdx.x) * C::M;
  const int bhq = int(blockIdx.y), hq = bhq % Hq;

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
    mbar_arrive_expect_tx(ld_bar, C::KATOMS * C::Q_ATOM);
#pragma unroll
    for (int a = 0; a < C::KATOMS; ++a) tma_load_3d(smem + C::OFF_Q + a * C::Q_ATOM, &tm_q, ld_bar, a * 64, p0, bhq);
  }
  // the head's projections in the 128-byte-swizzled K-major layout, the rank
  // zero-padded to 64: W_down as 64 rows of d (K = d), W_up as d rows of 64 (K = rank)
  {
    const __nv_bfloat16* wd = w_down + int64_t(hq) * r * D;
    const __nv_bfloat16* wu = w_up + int64_t(hq) * D * r;
    constexpr int PD = D / 8;   // 16-byte pieces per W_down row
    for (int idx = tid; idx < C::RP * PD; idx += 128) {
      const int n = idx / PD, kc = idx % PD;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (n < r) v = __ldg(reinterpret_cast<const uint4*>(wd + int64_t(n) * D + kc * 8));
      *reinterpret_cast<uint4*>(smem + C::OFF_WD + (kc >> 3) * C::WD_ATOM + n * 128 + (((kc & 7) ^ (n & 7)) << 4)) = v;
    }
    for (int idx = tid; idx < D * 8; idx += 128) {
      const int n = idx >> 3, kc = idx & 7;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (kc * 8 < r) v = __ldg(reinterpret_cast<const uint4*>(wu + int64_t(n) * r + kc * 8));
      *reinterpret_cast<uint4*>(smem + C::OFF_WU + n * 128 + ((kc ^ (n & 7)) << 4)) = v;
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  bool ok = true;
  if (tid == 0) {
    ok = mbar_wait(ld_bar, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const uint32_t sq = smem_u32(smem + C::OFF_Q), swd = smem_u32(smem + C::OFF_WD);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_bf16(tmem, desc_sw128(sq + uint32_t((kk >> 2) * C::Q_ATOM + (kk & 3) * 32)),
                 desc_sw128(swd + uint32_t((kk >> 2) * C::WD_ATOM + (kk & 3) * 32)), idesc_bf16(C::M, C::RP),
                 kk > 0 ? 1u : 0u);
      mma_commit(mma_bar);
    }
  }
  ok = __syncthreads_and(ok);
  if (ok) ok = mbar_wait(mma_bar, 0, abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  const uint32_t t_row = tmem + (uint32_t(warp * 32) << 16);
  if (ok) {
    // T row -> bf16 A operand of the second MMA (row = TMEM lane = thread)
    tc_fence_after();
    uint8_t* trow = smem + C::OFF_T + tid * 128;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float t32[32];
      tmem_ld32(t_row + uint32_t(h * 32), t32);
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t w[4];
#pragma unroll
        for (int v2 = 0; v2 < 4; ++v2) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(t32[pc * 8 + 2 * v2], t32[pc * 8 + 2 * v2 + 1]);
          w[v2] = *reinterpret_cast<uint32_t*>(&b2);
        }
        const int piece = h * 4 + pc;
        *reinterpret_cast<uint4*>(trow + ((piece ^ (tid & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (tid == 0 && ok) {
    tc_fence_after();
    const uint32_t st = smem_u32(smem + C::OFF_T), swu = smem_u32(smem + C::OFF_WU);
#pragma unroll
    for (int kk = 0; kk < C::RP / 16; ++kk)
      mma_bf16(tmem, desc_sw128(st + uint32_t(kk * 32)), desc_sw128(swu + uint32_t(kk * 32)), idesc_bf16(C::M, D),
               kk > 0 ? 1u : 0u);
    mma_commit(mma_bar);
  }
  if (ok) ok = mbar_wait(mma_bar, 1, abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) ok = __all_sync(0xffffffffu, mbar_wait(ld_bar, 0, abort_flag));   // the Q tile, seen by this thread
  if (ok) {
    // q^ = q + D, written over this thread's row of the Q tile
    tc_fence_after();
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      float dl[32];
      tmem_ld32(t_row + uint32_t(cc * 32), dl);
      uint8_t* qrow = smem + C::OFF_Q + (cc >> 1) * C::Q_ATOM + tid * 128;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        const int piece = (cc & 1) * 4 + pc;
        uint4* p = reinterpret_cast<uint4*>(qrow + ((piece ^ (tid & 7)) << 4));
        const uint4 u = *p;
        const uint32_t w_in[4] = {u.x, u.y, u.z, u.w};
        uint32_t w[4];
#pragma unroll
        for (int v2 = 0; v2 < 4; ++v2) {
          const float x0 = __uint_as_float(w_in[v2] << 16), x1 = __uint_as_float(w_in[v2] & 0xFFFF0000u);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(x0 + dl[pc * 8 + 2 * v2], x1 + dl[pc * 8 + 2 * v2 + 1]);
          w[v2] = *reinterpret_cast<uint32_t*>(&b2);
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (tid == 0) {
    if (ok) {
#pragma unroll
      for (int a = 0; a < C::KATOMS; ++a) tma_store_3d(&tm_out, smem + C::OFF_Q + a * C::Q_ATOM, a * 64, p0, bhq);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    } else {
      // after a time-out: let the load land and any issued MMA finish before TMEM is freed
      mbar_wait_drain(ld_bar, 0);
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace hils
