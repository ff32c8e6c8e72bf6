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
//   own    : per row, the causal own-chunk attention, the fusion normaliser
//            M' = log(sum_c exp(s^_c) + exp(lse_own)), the own chunk's share
//            exp(lse_own - M') o_own written to an fp32 accumulator, and a
//            count of (row, slot) pairs per key (kv head, window, chunk).
//   scan   : offsets of every key's pair list and of its 128-row tiles.
//   fill   : the inverted index: each key's list of (row, slot) entries.
//   attend : per tile of up to 128 pairs of one chunk: the chunk's K and V
//            arrive by TMA, the rows' queries are gathered with cp.async into
//            a 128B-swizzled tile, S = Q K^T on tcgen05 (fp32 in TMEM), one
//            thread per row turns its 64 scores into
//            P = exp(s - lse_c + s^_c - M'), P V on tcgen05, and the row's
//            partial output is added to its accumulator with 16-byte vector
//            reductions.  The weights are final, so partials simply add.
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
  int win_shift;   // window = pos >> win_shift
  int n_win;
  int64_t n_keys;  // B*Hkv*n_win*nc
  float tau;
};

__device__ __forceinline__ int64_t cc_key(const CcDims& c, int64_t bh, int64_t pos, int64_t chunk) {
  return (bh * c.n_win + (pos >> c.win_shift)) * c.nc + chunk;
}

// ---------------------------------------------------------------- own chunk + counts
template <typename T, int D>
__global__ void __launch_bounds__(128)
cc_own_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
              const int32_t* __restrict__ ids, const float* __restrict__ scores, float* __restrict__ oacc,
              float* __restrict__ rowstat, float* __restrict__ lse_own, int32_t* __restrict__ counts,
              const CcDims c, int64_t n_rows) {
  using L = RowLayout<T, D>;
  constexpr int E = L::E, LPK = L::LPK;
  const int lane = threadIdx.x & 31, sub = lane % LPK;
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= n_rows) return;
  const int64_t bhq = row / c.n_tok, i = row % c.n_tok;
  const int64_t b = bhq / c.Hq, hq = bhq % c.Hq;
  const int64_t bh = b * c.Hkv + hq / c.G;
  const T* kbh = k + bh * c.n_tok * D;
  const T* vbh = v + bh * c.n_tok * D;
  float qv[E];
  Vec16<T>::load(q + row * D + sub * E, qv);
  const int64_t own = i / kChunk;
  float oc[E];
  const float lo = attend_range<T, D>(qv, kbh, vbh, own * kChunk, i + 1, c.tau, oc);
  // fusion normaliser over the valid selected chunks and the own chunk
  float M = lo;
  for (int t = lane; t < c.K; t += 32) {
    const int32_t ci = __ldg(ids + row * c.K + t);
    if (ci >= 0 && ci < own) M = fmaxf(M, __ldg(scores + row * c.K + t));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float Z = 0.f;
  for (int t = lane; t < c.K; t += 32) {
    const int32_t ci = __ldg(ids + row * c.K + t);
    if (ci < 0) continue;
    if (ci >= own) {
      record_error(HILS_ERR_DEVICE_BOUNDS);
      continue;
    }
    Z += expf(__ldg(scores + row * c.K + t) - M);
    atomicAdd(counts + cc_key(c, bh, i, ci), 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
  Z += expf(lo - M);
  const float Mp = M + logf(Z);
  const float w_own = expf(lo - Mp);
  if (lane < LPK) {
    float* dst = oacc + row * D + sub * E;
#pragma unroll
    for (int e = 0; e < E; e += 4)
      *reinterpret_cast<float4*>(dst + e) = make_float4(w_own * oc[e], w_own * oc[e + 1], w_own * oc[e + 2], w_own * oc[e + 3]);
  }
  if (lane == 0) {
    rowstat[row] = Mp;
    if (lse_own) lse_own[row] = lo;
  }
}

// ---------------------------------------------------------------- scan (one CTA)
constexpr int kCcTileRows = 128;

// Each of the 1024 threads owns a contiguous segment of keys: local sums,
// one block-wide exclusive scan, then the segment's offsets.
__global__ void __launch_bounds__(1024)
cc_scan_kernel(const int32_t* __restrict__ counts, int64_t n_keys, int64_t* __restrict__ offsets,
               int32_t* __restrict__ tile_start, int32_t* __restrict__ cursor) {
  __shared__ int64_t s_a[32], s_t[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t seg = (n_keys + 1023) / 1024;
  const int64_t k0 = tid * seg, k1 = (k0 + seg < n_keys) ? k0 + seg : n_keys;
  int64_t sa = 0, st = 0;
  for (int64_t kk = k0; kk < k1; ++kk) {
    const int64_t cnt = counts[kk];
    sa += cnt;
    st += (cnt + kCcTileRows - 1) / kCcTileRows;
  }
  int64_t a = sa, t = st;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t ya = __shfl_up_sync(0xffffffffu, a, o), yt = __shfl_up_sync(0xffffffffu, t, o);
    if (lane >= o) { a += ya; t += yt; }
  }
  if (lane == 31) { s_a[warp] = a; s_t[warp] = t; }
  __syncthreads();
  int64_t pa = 0, pt = 0, ta = 0, tt = 0;
  for (int w = 0; w < 32; ++w) {
    if (w < warp) { pa += s_a[w]; pt += s_t[w]; }
    ta += s_a[w];
    tt += s_t[w];
  }
  int64_t ra = pa + a - sa, rt = pt + t - st;   // exclusive prefix of this segment
  for (int64_t kk = k0; kk < k1; ++kk) {
    const int64_t cnt = counts[kk];
    offsets[kk] = ra;
    tile_start[kk] = int32_t(rt);
    cursor[kk] = 0;
    ra += cnt;
    rt += (cnt + kCcTileRows - 1) / kCcTileRows;
  }
  if (tid == 0) {
    offsets[n_keys] = ta;
    tile_start[n_keys] = int32_t(tt);
  }
}

// ---------------------------------------------------------------- fill the inverted index
__global__ void __launch_bounds__(256)
cc_fill_kernel(const int32_t* __restrict__ ids, const int64_t* __restrict__ offsets, int32_t* __restrict__ cursor,
               int32_t* __restrict__ entries, const CcDims c, int64_t n_slots) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n_slots) return;
  const int32_t ci = __ldg(ids + idx);
  if (ci < 0) return;
  const int64_t row = idx / c.K;
  const int slot = int(idx % c.K);
  const int64_t bhq = row / c.n_tok, i = row % c.n_tok;
  const int64_t b = bhq / c.Hq, hq = bhq % c.Hq;
  if (ci >= i / kChunk) return;   // recorded by cc_own_kernel
  const int64_t bh = b * c.Hkv + hq / c.G;
  const int64_t key = cc_key(c, bh, i, ci);
  const int32_t at = atomicAdd(cursor + key, 1);
  const int64_t row_in_bh = (hq % c.G) * c.n_tok + i;   // (g, position) within the kv head
  entries[offsets[key] + at] = int32_t((row_in_bh << 6) | slot);
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
template <int D>
struct CcTc {
  static constexpr int M = kCcTileRows;
  static constexpr int KATOMS = D / 64;
  static constexpr uint32_t Q_ATOM = M * 128;       // 16 KB
  static constexpr uint32_t KV_ATOM = kChunk * 128; // 8 KB
  static constexpr uint32_t Q_BYTES = KATOMS * Q_ATOM;
  static constexpr uint32_t K_BYTES = KATOMS * KV_ATOM;
  static constexpr uint32_t P_BYTES = M * 128;      // 128 rows x 64 keys bf16
  static constexpr uint32_t OFF_Q = 0, OFF_K = Q_BYTES, OFF_V = OFF_K + K_BYTES, OFF_P = OFF_V + K_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
  static constexpr uint32_t TMEM_COLS = D == 64 ? 128 : 256;   // S: 64 columns, O: D columns
  static constexpr uint32_t SMEM_MIN = OFF_BAR + 64 + 1024;
  // at most 512 / TMEM_COLS CTAs may share an SM, or a tcgen05.alloc could wait
  // for columns that a co-resident persistent CTA never frees: request enough
  // shared memory that no more CTAs fit.
  static constexpr uint32_t MAX_CTAS = 512 / TMEM_COLS;
  static constexpr uint32_t SMEM_FLOOR = 233472u / (MAX_CTAS + 1) + 1024u;
  static constexpr uint32_t SMEM = SMEM_MIN > SMEM_FLOOR ? SMEM_MIN : SMEM_FLOOR;
  static constexpr uint32_t IDESC_S = sm100::idesc_bf16(M, kChunk);
  // P (K-major) x V (MN-major: d contiguous in each key row)
  static constexpr uint32_t IDESC_O = sm100::idesc_bf16(M, D) | (1u << 16);
};

// MN-major, 128B-swizzled operand: 64-element rows along N, 8-row groups
// (along K) 1024 bytes apart, 64-wide N blocks `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

struct CcTcParams {
  CcDims c;
  const int64_t* offsets;
  const int32_t* tile_start;
  const int32_t* entries;
  const float* scores;
  const float* rowstat;
  const __nv_bfloat16* q;
  float* oacc;
};

template <int D>
__global__ void __launch_bounds__(128)
cc_attend_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const CcTcParams p) {
  using C = CcTc<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  uint64_t* kv_bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* mma_bar = kv_bar + 1;
  uint64_t* done_bar = kv_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 28);
  int64_t* s_item = reinterpret_cast<int64_t*>(smem + C::OFF_BAR + 32);   // key, first entry, count
  const uint32_t sQ = smem_u32(smem + C::OFF_Q), sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V), sP = smem_u32(smem + C::OFF_P);
  const int tid = threadIdx.x, warp = tid >> 5;
  const CcDims& c = p.c;

  if (tid == 0) {
    mbar_init(kv_bar, 1);
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
  const uint32_t t_lane = uint32_t(warp * 32) << 16;
  const int32_t n_items = p.tile_start[c.n_keys];
  uint32_t kv_phase = 0, mma_phase = 0;
  bool ok = true, issued_mma = false;

  for (int32_t item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
    if (tid == 0) {
      // key = last index with tile_start[key] <= item
      int64_t lo = 0, hi = c.n_keys - 1;
      while (lo < hi) {
        const int64_t mid = (lo + hi + 1) >> 1;
        if (p.tile_start[mid] <= item) lo = mid; else hi = mid - 1;
      }
      const int64_t key = lo;
      const int64_t t = item - p.tile_start[key];
      const int64_t first = p.offsets[key] + t * C::M;
      const int64_t cnt = p.offsets[key + 1] - first;
      s_item[0] = key;
      s_item[1] = first;
      s_item[2] = cnt < C::M ? cnt : C::M;
      // chunk K and V tiles
      const int64_t chunk = key % c.nc;
      const int64_t bh = key / (c.nc * c.n_win);
      const int y = int(bh * c.n_tok + chunk * kChunk);
      mbar_arrive_expect_tx(kv_bar, 2 * C::K_BYTES);
#pragma unroll
      for (int a = 0; a < C::KATOMS; ++a) {
        tma_load_2d(smem + C::OFF_K + a * C::KV_ATOM, &tm_k, kv_bar, a * 64, y);
        tma_load_2d(smem + C::OFF_V + a * C::KV_ATOM, &tm_v, kv_bar, a * 64, y);
      }
    }
    __syncthreads();
    const int64_t key = s_item[0], first = s_item[1];
    const int n = int(s_item[2]);
    const int64_t bh = key / (c.nc * c.n_win);
    const int64_t b = bh / c.Hkv, h = bh % c.Hkv;
    // row of this thread and its fusion factor s^ - M'
    int64_t grow = -1;
    float fac = 0.f;
    if (tid < n) {
      const int32_t e = p.entries[first + tid];
      const int64_t row_in_bh = e >> 6;
      const int slot = e & 63;
      const int64_t g = row_in_bh / c.n_tok, pos = row_in_bh % c.n_tok;
      grow = (b * c.Hq + h * c.G + g) * c.n_tok + pos;
      fac = p.scores[grow * c.K + slot] - p.rowstat[grow];
      const __nv_bfloat16* src = p.q + grow * D;
#pragma unroll
      for (int a = 0; a < C::KATOMS; ++a)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          cp_async16(sQ + a * C::Q_ATOM + tid * 128 + ((j ^ (tid & 7)) << 4), src + a * 64 + j * 8);
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncthreads();
    // S = Q K^T
    if (tid == 0) {
      ok = mbar_wait(kv_bar, kv_phase, abort_flag);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = uint32_t((kk >> 2) * C::Q_ATOM + (kk & 3) * 32);
          const uint32_t offk = uint32_t((kk >> 2) * C::KV_ATOM + (kk & 3) * 32);
          mma_bf16(tmem, desc_sw128(sQ + off), desc_sw128(sK + offk), C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(mma_bar);
        issued_mma = true;
      }
    }
    kv_phase ^= 1;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    ok = mbar_wait(mma_bar, mma_phase, abort_flag);
    mma_phase ^= 1;
    tc_fence_after();
    {
      float s[64];
      float tmp[32];
      tmem_ld32(tmem + t_lane + 0, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) s[j] = tmp[j];
      tmem_ld32(tmem + t_lane + 32, tmp);
#pragma unroll
      for (int j = 0; j < 32; ++j) s[32 + j] = tmp[j];
      const float k2 = c.tau * 1.4426950408889634f;   // scores in log2 units
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) m = fmaxf(m, s[j]);
      const float mb = m * k2;
      float l = 0.f;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        s[j] = exp2f(fmaf(s[j], k2, -mb));
        l += s[j];
      }
      const float w = expf(fac) / l;
      uint8_t* prow = smem + C::OFF_P + tid * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t wd[4] = {0u, 0u, 0u, 0u};
        if (tid < n) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(s[8 * j + 2 * u] * w, s[8 * j + 2 * u + 1] * w);
            wd[u] = *reinterpret_cast<uint32_t*>(&h2);
          }
        }
        *reinterpret_cast<uint4*>(prow + ((j ^ (tid & 7)) << 4)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    // O = P V
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kChunk / 16; ++kk)
        mma_bf16(tmem + 64, desc_sw128(sP + kk * 32), desc_sw128_mn(sV + kk * 2048, C::KV_ATOM), C::IDESC_O,
                 kk > 0 ? 1u : 0u);
      mma_commit(mma_bar);
    }
    __syncwarp();
    ok = mbar_wait(mma_bar, mma_phase, abort_flag);
    mma_phase ^= 1;
    tc_fence_after();
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      float o[32];
      tmem_ld32(tmem + t_lane + 64 + cc * 32, o);
      if (grow >= 0) {
        float* dst = p.oacc + grow * D + cc * 32;
#pragma unroll
        for (int j = 0; j < 32; j += 4) red_add_v4(dst + j, o[j], o[j + 1], o[j + 2], o[j + 3]);
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);
  }
  // teardown: no copy or MMA may still be in flight when TMEM is freed
  __syncthreads();
  if (tid == 0) {
    if (!ok) mbar_wait_drain(kv_bar, kv_phase ^ 1);
    if (issued_mma) {
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
