// Kernel (b), CUDA-core variant: chunk scoring + top-K selection.
//
// HiLS paper, aitrends.kr article, section "방법론" (Methodology):
//   s^_{i,c} = <q_i, k'_c>/sqrt(d) + b'_c over the fully-past chunks, keep the
//   K largest.
//
// This is the fp32 path (fp32 has no tensor-core MMA that meets a 1e-5
// tolerance), and the path for a listed subset of query positions (row_pos,
// any order).  One CTA scores 128 rows of one (b, hq) -- consecutive
// positions, or 128 consecutive entries of row_pos -- against tiles of 32
// compressed keys staged in shared memory.  q is stored
// transposed ([d][128]) so each thread reads its own row conflict-free; k'
// is transposed ([d][32]) so a float4 read broadcasts four chunks.  Each
// thread keeps its row's running top-K (sorted, ties to the lower id, which
// is the chunk seen first) in shared memory.
#pragma once
#include "common.cuh"

namespace hils {

constexpr int kSelRows = 128;   // rows per CTA
constexpr int kSelTile = 32;    // compressed keys per shared-memory tile

template <int D>
constexpr size_t select_simt_smem(int K) {
  return sizeof(float) * (size_t(D) * kSelRows + size_t(D) * kSelTile + kSelTile) +
         size_t(K) * kSelRows * (sizeof(float) + sizeof(int32_t));
}

// MMA_OPERAND: read k' from the bf16 scoring operand (k' in bf16, bias as
// x_hi + x_lo = b'/tau) and compute s^ = tau * (<q, k'> + x), the same
// quantity the tensor-core path computes; otherwise read fp32 k', b'.
template <typename T, int D, bool MMA_OPERAND>
__global__ void __launch_bounds__(kSelRows)
select_simt_kernel(const T* __restrict__ q, const float* __restrict__ kp, const float* __restrict__ bp,
                   const __nv_bfloat16* __restrict__ kmma, int64_t n_tok, int64_t nc, int Hq, int G,
                   int Hkv, int K, float tau, int32_t* __restrict__ ids, float* __restrict__ scores, int wm1,
                   const int64_t* __restrict__ row_pos, int64_t n_rows) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qT = reinterpret_cast<float*>(smem_raw);          // [D][128]
  float* kT = qT + D * kSelRows;                           // [D][32]
  float* kb = kT + D * kSelTile;                           // [32]
  float* topv = kb + kSelTile;                             // [K][128]
  int32_t* topi = reinterpret_cast<int32_t*>(topv + K * kSelRows);  // [K][128]

  const int tid = threadIdx.x;
  const int64_t bhq = blockIdx.y;
  const int b = int(bhq / Hq), hq = int(bhq % Hq);
  const int64_t bh = int64_t(b) * Hkv + hq / G;
  __shared__ int64_t pos_s[kSelRows];
  __shared__ int c_end_s;
  // this thread's output row r (0 .. n_rows-1) and its query position
  const int64_t r = int64_t(blockIdx.x) * kSelRows + tid;
  const bool in_rows = r < n_rows;
  int64_t i = in_rows ? (row_pos ? __ldg(row_pos + r) : r) : -1;
  if (in_rows && (i < 0 || i >= n_tok)) {
    record_error(HILS_ERR_DEVICE_BOUNDS);   // listed position outside the sequence: ids -1
    i = -1;
  }
  const bool valid = i >= 0;
  const int64_t n_cand = valid ? n_candidates(i, wm1) : 0;
  pos_s[tid] = i;
  if (tid == 0) c_end_s = 0;
  __syncthreads();
  if (n_cand > 0) atomicMax(&c_end_s, int(n_cand));   // candidates of the tile's longest row

  // stage q (transposed)
  for (int idx = tid; idx < kSelRows * D; idx += kSelRows) {
    const int rr = idx / D, t = idx % D;
    const int64_t ii = pos_s[rr];
    float x = 0.f;
    if (ii >= 0) {
      if constexpr (sizeof(T) == 2) x = __bfloat162float(q[(bhq * n_tok + ii) * D + t]);
      else x = q[(bhq * n_tok + ii) * D + t];
    }
    qT[t * kSelRows + rr] = x;
  }
  int count = 0;
  float thr = -INFINITY;
  __syncthreads();
  const int64_t c_end = c_end_s;

  for (int64_t c0 = 0; c0 < c_end; c0 += kSelTile) {
    __syncthreads();
    for (int idx = tid; idx < kSelTile * D; idx += kSelRows) {
      const int cc = idx / D, t = idx % D;
      const int64_t c = c0 + cc;
      float x = 0.f;
      if (c < c_end) {
        if constexpr (MMA_OPERAND) x = __bfloat162float(kmma[(bh * nc + c) * (D + kExt) + t]);
        else x = kp[(bh * nc + c) * D + t];
      }
      kT[t * kSelTile + cc] = x;
    }
    if (tid < kSelTile) {
      const int64_t c = c0 + tid;
      float x = 0.f;
      if (c < c_end) {
        if constexpr (MMA_OPERAND) {
          const __nv_bfloat16* ext = kmma + (bh * nc + c) * (D + kExt) + D;
          x = __bfloat162float(ext[0]) + __bfloat162float(ext[1]);
        } else {
          x = bp[bh * nc + c];
        }
      }
      kb[tid] = x;
    }
    __syncthreads();
    for (int cc = 0; cc < kSelTile; cc += 4) {
      if (c0 + cc >= n_cand) break;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int t = 0; t < D; ++t) {
        const float qv = qT[t * kSelRows + tid];
        const float4 kv = *reinterpret_cast<const float4*>(kT + t * kSelTile + cc);
        acc[0] = fmaf(qv, kv.x, acc[0]);
        acc[1] = fmaf(qv, kv.y, acc[1]);
        acc[2] = fmaf(qv, kv.z, acc[2]);
        acc[3] = fmaf(qv, kv.w, acc[3]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t c = c0 + cc + u;
        if (c >= n_cand) break;
        const float s = MMA_OPERAND ? tau * (acc[u] + kb[cc + u]) : fmaf(tau, acc[u], kb[cc + u]);
        if (s > thr) {
          int j = count < K ? count : K - 1;
          while (j > 0 && topv[(j - 1) * kSelRows + tid] < s) {
            topv[j * kSelRows + tid] = topv[(j - 1) * kSelRows + tid];
            topi[j * kSelRows + tid] = topi[(j - 1) * kSelRows + tid];
            --j;
          }
          topv[j * kSelRows + tid] = s;
          topi[j * kSelRows + tid] = int32_t(c);
          if (count < K) ++count;
          if (count == K) thr = topv[(K - 1) * kSelRows + tid];
        }
      }
    }
  }
  if (!in_rows) return;
  // ascending chunk id order
  for (int a = 1; a < count; ++a) {
    const int32_t ci = topi[a * kSelRows + tid];
    const float cv = topv[a * kSelRows + tid];
    int j = a;
    while (j > 0 && topi[(j - 1) * kSelRows + tid] > ci) {
      topi[j * kSelRows + tid] = topi[(j - 1) * kSelRows + tid];
      topv[j * kSelRows + tid] = topv[(j - 1) * kSelRows + tid];
      --j;
    }
    topi[j * kSelRows + tid] = ci;
    topv[j * kSelRows + tid] = cv;
  }
  const int64_t row = bhq * n_rows + r;
  for (int t = 0; t < K; ++t) {
    ids[row * K + t] = t < count ? topi[t * kSelRows + tid] : -1;
    if (scores) scores[row * K + t] = t < count ? topv[t * kSelRows + tid] : -INFINITY;
  }
}

}  // namespace hils
