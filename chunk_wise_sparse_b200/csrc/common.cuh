// Device helpers shared by the HiLS kernels (sm_100a only).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hils.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library is built for sm_100a only"
#endif

namespace hils {

constexpr int kChunk = 64;      // C: tokens per chunk
constexpr int kMaxTopK = 64;    // largest supported K
constexpr int kExt = 16;        // extra bf16 columns of the scoring operand (b'/tau hi, lo, zeros)

// Device status word: the first error a kernel records since the last read.
__device__ int32_t g_status;

__device__ __forceinline__ void record_error(int32_t code) { atomicCAS(&g_status, 0, code); }

// Candidates of a query at position i: the chunks before its local window,
// which spans the own chunk and the wm1 chunks before it (wm1 = 0: the own
// chunk alone).
__host__ __device__ __forceinline__ int64_t n_candidates(int64_t i, int wm1) {
  const int64_t n = i / kChunk - wm1;
  return n > 0 ? n : 0;
}

// Where the keys / values of chunk c of (b, h) live.  Contiguous cache
// (table == nullptr): [B, Hkv, n_tok, d], chunk c at token c*C.  Chunk-paged
// cache: a pool [n_pages, Hkv, C, d] and table[b * nc + c] = the page of
// logical chunk c of sequence b.
struct PagedKv {
  const int32_t* table;
  int64_t n_pages;
};
// Element offset of the chunk's first row, or -1 (recorded as
// HILS_ERR_DEVICE_BOUNDS) when its page is outside the pool.
__device__ __forceinline__ int64_t kv_chunk_offset(const PagedKv& pk, int64_t b, int64_t h, int64_t c, int64_t Hkv,
                                                   int64_t n_tok, int64_t nc, int64_t D) {
  if (pk.table == nullptr) return ((b * Hkv + h) * n_tok + c * kChunk) * D;
  const int64_t page = __ldg(pk.table + b * nc + c);
  if (page < 0 || page >= pk.n_pages) {
    record_error(HILS_ERR_DEVICE_BOUNDS);
    return -1;
  }
  return (page * Hkv + h) * kChunk * D;
}

// ---------------------------------------------------------------------------
// 16-byte vectors of bf16 (8 elements) or fp32 (4 elements), widened to fp32.
template <typename T> struct Vec16;

template <> struct Vec16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    unpack(u, x);
  }
  __device__ __forceinline__ static void load_stream(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    unpack(u, x);
  }
  __device__ __forceinline__ static void unpack(uint4 u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      x[2 * t] = __uint_as_float(w[t] << 16);
      x[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
    }
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float (&x)[8]) {
    uint4 u;
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * t], x[2 * t + 1]);
      w[t] = *reinterpret_cast<uint32_t*>(&h);
    }
    u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
    *reinterpret_cast<uint4*>(p) = u;
  }
};

template <> struct Vec16<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void load(const float* p, float (&x)[4]) {
    float4 f = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  }
  __device__ __forceinline__ static void load_stream(const float* p, float (&x)[4]) {
    float4 f = __ldcs(reinterpret_cast<const float4*>(p));
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  }
  __device__ __forceinline__ static void store(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};

// Lane layout used by the row-streaming kernels: a key row of D elements is
// read by LPK lanes with one 16-byte vector each; a warp covers KPI rows.
template <typename T, int D> struct RowLayout {
  static constexpr int E = Vec16<T>::E;
  static constexpr int VPR = D / E;                  // vectors per row
  static_assert(VPR >= 1 && VPR <= 32 && (VPR & (VPR - 1)) == 0, "row must be 1..32 vectors");
  static constexpr int LPK = VPR;                    // lanes per key row
  static constexpr int KPI = 32 / LPK;               // rows per warp iteration
};

// Sum over the LPK lanes that share a row (xor shuffles inside the group).
template <int LPK>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = 1; o < LPK; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Online softmax-weighted accumulator for one key group: (max, sum, acc[E]).
template <int E> struct SoftAcc {
  float m, l;
  float acc[E];
  __device__ __forceinline__ void init() {
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
  }
  // add one logit z with value vector v
  __device__ __forceinline__ void add(float z, const float (&v)[E]) {
    const float mn = fmaxf(m, z);
    const float a = expf(m - mn);   // m = -inf first time -> 0
    const float p = expf(z - mn);
    l = l * a + p;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] * a + p * v[e];
    m = mn;
  }
  // merge with the state held by lane (lane ^ off)
  __device__ __forceinline__ void merge_xor(int off) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off);
    const float lo = __shfl_xor_sync(0xffffffffu, l, off);
    const float mn = fmaxf(m, mo);
    const float a = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float b = (mo == -INFINITY) ? 0.f : expf(mo - mn);
    l = l * a + lo * b;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float ao = __shfl_xor_sync(0xffffffffu, acc[e], off);
      acc[e] = acc[e] * a + ao * b;
    }
    m = mn;
  }
};

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

}  // namespace hils
