// Kernel (d): one decode step of HiLS attention.
//
// HiLS paper, aitrends.kr article, section "방법론" (Methodology) for the
// scoring and top-K, and ai-papers.net article, section "実験結果と性能",
// for the per-token decode with sparse KV access.  The query of (b, hq) sits
// at position t = seqlens[b]-1.  Its local window is the own chunk
// o = floor(t/C) and the wm1 chunks before it (keys max(0, (o - wm1) C) .. t,
// causal), one fusion branch whose score is its exact log-sum-exp; its top-K
// candidates are the chunks before the window, c < o - wm1.
//
// Four short kernels, all HBM- or latency-bound:
//   D1 scores   : s^ for every candidate chunk of every query head; one
//                 thread per chunk scores its compressed-key row against the
//                 G query heads that share the kv head (one read of k' per
//                 kv head); the bf16 rows of a CTA arrive in shared memory by
//                 one bulk copy.
//   D2 top-K    : exact radix select (4 passes of 8 bits over an
//                 order-preserving integer image of the score), then a
//                 stable compaction in ascending chunk id; ties among equal
//                 scores go to the lower ids.
//   D3 partials : per (batch, kv head), each distinct chunk kept by any of the
//                 G query heads (plus each chunk of the local window) is read
//                 once and attended by every head that kept it; one partial
//                 (score, output) per (row, slot).  A window chunk's score is
//                 its exact log-sum-exp, so the window chunks' partials fuse
//                 to the one window branch.
//   D4 combine  : softmax over the chunk scores fuses the partials.
// D2-D4 are launched with programmatic stream serialisation: each may start
// while its predecessor finishes and waits for it (pdl_wait) before reading
// its results.
#pragma once
#include "attend_simt.cuh"
#include "sm100.cuh"

namespace hils {

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialisation may start while the kernel before it in the stream is still
// running; pdl_wait() returns once that kernel has completed and its memory
// writes are visible (at once for a kernel launched without the attribute).
// pdl_trigger() lets the next such kernel be scheduled as soon as every block
// of this one has called it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

struct DecodeWs {
  float* scores;      // [B*Hq, nc]
  int32_t* sel_ids;   // [B*Hq, K]
  float* sel_scores;  // [B*Hq, K]
  float* part_u;      // [B*Hq, K+WC]: K selected slots, then the WC window chunks
  float* part_o;      // [B*Hq, K+WC, D]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t decode_ws_layout(int64_t rows, int64_t nc, int K, int WC, int D, char* base, DecodeWs* ws) {
  size_t off = 0;
  auto take = [&](size_t bytes) { char* p = base ? base + off : nullptr; off += align256(bytes); return p; };
  char* a = take(sizeof(float) * rows * nc);
  char* b = take(sizeof(int32_t) * rows * K);
  char* c = take(sizeof(float) * rows * K);
  char* d = take(sizeof(float) * rows * (K + WC));
  char* e = take(sizeof(float) * rows * (K + WC) * D);
  if (ws) {
    ws->scores = reinterpret_cast<float*>(a);
    ws->sel_ids = reinterpret_cast<int32_t*>(b);
    ws->sel_scores = reinterpret_cast<float*>(c);
    ws->part_u = reinterpret_cast<float*>(d);
    ws->part_o = reinterpret_cast<float*>(e);
  }
  return off;
}

// Own chunk of batch b's query; -1 if seqlens[b] is invalid.
__device__ __forceinline__ int64_t decode_own_chunk(const int32_t* seqlens, int b, int64_t cap) {
  const int32_t s = __ldg(seqlens + b);
  if (s < 1 || int64_t(s) > cap) return -1;
  return int64_t(s - 1) / kChunk;
}

constexpr int kDecChunksPerCta = 128;

// Shared memory of decode_scores_kernel: the G query rows (fp32), then, for
// the bf16 scoring operand, the CTA's operand rows and an mbarrier.
template <int D, bool MMA_OPERAND>
__host__ __device__ constexpr size_t decode_scores_smem(int G) {
  return sizeof(float) * size_t(G) * D +
         (MMA_OPERAND ? size_t(kDecChunksPerCta) * (D + kExt) * sizeof(__nv_bfloat16) + 16 : 0);
}

// One thread per candidate chunk scores the chunk's compressed key against
// the G query heads of the kv head (query rows broadcast from shared memory),
// four heads per pass over the row.  No cross-lane reductions.  The bf16
// scoring operand rows of the CTA's chunks are contiguous in memory: one bulk
// copy brings them into shared memory (whole lines from HBM instead of a
// 16-byte piece of 32 rows per load instruction) and each thread reads its row
// there; fp32 rows are read from global memory with 16-byte loads.
template <typename T, int D, bool MMA_OPERAND>
__global__ void __launch_bounds__(kDecChunksPerCta)
decode_scores_kernel(const T* __restrict__ q, const float* __restrict__ kp, const float* __restrict__ bp,
                     const __nv_bfloat16* __restrict__ kmma, const int32_t* __restrict__ seqlens, int64_t cap,
                     int64_t nc, int Hq, int G, int Hkv, float tau, float* __restrict__ ws_scores, int wm1) {
  using KT = typename std::conditional<MMA_OPERAND, __nv_bfloat16, float>::type;
  constexpr int E = Vec16<KT>::E;                   // elements per 16-byte load
  constexpr int RS = MMA_OPERAND ? D + kExt : D;    // row stride of the k' rows
  extern __shared__ __align__(16) float sq[];       // [G][D]
  __shared__ int s_abort;
  pdl_trigger();
  const int bh = blockIdx.y;
  const int b = bh / Hkv, h = bh % Hkv;
  const int64_t own = decode_own_chunk(seqlens, b, cap);
  if (own < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) record_error(HILS_ERR_DEVICE_BOUNDS);
    return;
  }
  const int64_t c0 = int64_t(blockIdx.x) * kDecChunksPerCta;
  const int64_t n_cand = own - wm1;
  if (c0 >= n_cand) return;   // the whole CTA: no candidate chunk
  __nv_bfloat16* srows = reinterpret_cast<__nv_bfloat16*>(sq + G * D);   // [rows][RS]
  uint64_t* bar = reinterpret_cast<uint64_t*>(srows + kDecChunksPerCta * RS);
  if constexpr (MMA_OPERAND) {
    if (threadIdx.x == 0) {
      // rows c0 .. c0+nv-1: 16-byte aligned (the operand base is, and a row is
      // (D + 16) x 2 bytes), a multiple of 16 bytes long
      const int nv = n_cand - c0 < kDecChunksPerCta ? int(n_cand - c0) : kDecChunksPerCta;
      const uint32_t bytes = uint32_t(nv) * RS * 2u;
      s_abort = 0;
      sm100::mbar_init(bar, 1);
      sm100::fence_barrier_init();
      sm100::mbar_arrive_expect_tx(bar, bytes);
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              sm100::smem_u32(srows)),
          "l"(kmma + (int64_t(bh) * nc + c0) * RS), "r"(bytes), "r"(sm100::smem_u32(bar))
          : "memory");
    }
  }
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, t = idx % D;
    const T x = q[(int64_t(b) * Hq + h * G + g) * D + t];
    if constexpr (sizeof(T) == 2) sq[idx] = __bfloat162float(x);
    else sq[idx] = x;
  }
  __syncthreads();
  if constexpr (MMA_OPERAND) {
    if (!sm100::mbar_wait(bar, 0, &s_abort)) {
      // the copy did not land within the time limit (recorded): let it land
      // before the CTA's shared memory is released
      if (threadIdx.x == 0) sm100::mbar_wait_drain(bar, 0);
      return;
    }
  }
  const int64_t c = c0 + threadIdx.x;
  if (c >= n_cand) return;
  const KT* row = MMA_OPERAND ? reinterpret_cast<const KT*>(srows + threadIdx.x * RS)
                              : reinterpret_cast<const KT*>(kp) + (int64_t(bh) * nc + c) * RS;
  float bias;
  if constexpr (MMA_OPERAND) {
    const __nv_bfloat16* ext = srows + threadIdx.x * RS + D;
    bias = __bfloat162float(ext[0]) + __bfloat162float(ext[1]);
  } else {
    bias = __ldg(bp + int64_t(bh) * nc + c);
  }
  float* out = ws_scores + (int64_t(b) * Hq + h * G) * nc + c;
  for (int g0 = 0; g0 < G; g0 += 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int k0 = 0; k0 < D; k0 += E) {
      float kv[E];
      if constexpr (MMA_OPERAND) Vec16<KT>::unpack(*reinterpret_cast<const uint4*>(row + k0), kv);
      else Vec16<KT>::load(row + k0, kv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (g0 + j < G) {
          const float* qg = sq + (g0 + j) * D + k0;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[j] = fmaf(qg[e], kv[e], acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (g0 + j < G) out[int64_t(g0 + j) * nc] = MMA_OPERAND ? tau * (acc[j] + bias) : fmaf(tau, acc[j], bias);
  }
}

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix sum over 256 threads; also returns the total.
__device__ __forceinline__ int block_exclusive_scan256(int x, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int t = warp_tot[w];
    if (w < warp) before += t;
    total += t;
  }
  return before + incl - x;
}

__global__ void __launch_bounds__(256)
decode_topk_kernel(const float* __restrict__ ws_scores, const int32_t* __restrict__ seqlens, int64_t cap,
                   int64_t nc, int Hq, int K, int32_t* __restrict__ sel_ids, float* __restrict__ sel_scores,
                   int wm1) {
  __shared__ uint32_t hist[256];
  __shared__ int warp_tot[8];
  __shared__ uint32_t s_digit, s_above;
  pdl_wait();      // the scores of the step's first kernel
  pdl_trigger();
  const int row = blockIdx.x, b = row / Hq, tid = threadIdx.x;
  int64_t n = decode_own_chunk(seqlens, b, cap) - wm1;   // candidates
  if (n < 0) n = 0;
  const float* sc = ws_scores + int64_t(row) * nc;
  int32_t* oid = sel_ids + int64_t(row) * K;
  float* osc = sel_scores + int64_t(row) * K;
  if (n <= K) {
    for (int t = tid; t < K; t += 256) {
      oid[t] = t < n ? t : -1;
      osc[t] = t < n ? sc[t] : -INFINITY;
    }
    return;
  }
  uint32_t prefix = 0, mask = 0;
  int krem = K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[tid] = 0;
    __syncthreads();
    for (int64_t c = tid; c < n; c += 256) {
      const uint32_t key = order_key(sc[c]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t loc[8], lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { loc[j] = hist[255 - 8 * tid - j]; lsum += loc[j]; }
      uint32_t incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t excl = incl - lsum;
      if (excl < uint32_t(krem) && uint32_t(krem) <= incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + loc[j] >= uint32_t(krem)) { s_digit = 255 - 8 * tid - j; s_above = cum; break; }
          cum += loc[j];
        }
      }
    }
    __syncthreads();
    krem -= int(s_above);
    prefix |= s_digit << shift;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  // prefix = key of the K-th largest score; take all keys above it and the
  // krem lowest-id keys equal to it.
  const int64_t seg = (n + 255) / 256;
  const int64_t s0 = tid * seg, s1 = (s0 + seg < n) ? s0 + seg : n;
  int gt = 0, eq = 0;
  for (int64_t c = s0; c < s1; ++c) {
    const uint32_t key = order_key(sc[c]);
    gt += key > prefix;
    eq += key == prefix;
  }
  int tot;
  const int eq_before = block_exclusive_scan256(eq, warp_tot, tot);
  int take_eq = krem - eq_before;
  take_eq = take_eq < 0 ? 0 : (take_eq > eq ? eq : take_eq);
  const int pos0 = block_exclusive_scan256(gt + take_eq, warp_tot, tot);
  int pos = pos0, eq_seen = 0;
  for (int64_t c = s0; c < s1; ++c) {
    const float s = sc[c];
    const uint32_t key = order_key(s);
    bool take = key > prefix;
    if (key == prefix) take = eq_seen++ < take_eq;
    if (take && pos < K) { oid[pos] = int32_t(c); osc[pos] = s; ++pos; }
  }
}

// D2 for rows of at most 256 * IT candidates: the same radix select and
// stable compaction with each thread's contiguous segment of order keys held
// in registers, so the scores are read once instead of once per pass.
template <int IT>
__global__ void __launch_bounds__(256)
decode_topk_reg_kernel(const float* __restrict__ ws_scores, const int32_t* __restrict__ seqlens, int64_t cap,
                       int64_t nc, int Hq, int K, int32_t* __restrict__ sel_ids, float* __restrict__ sel_scores,
                       int wm1) {
  __shared__ uint32_t hist[256];
  __shared__ int warp_tot[8];
  __shared__ uint32_t s_digit, s_above;
  pdl_wait();      // the scores of the step's first kernel
  pdl_trigger();
  const int row = blockIdx.x, b = row / Hq, tid = threadIdx.x;
  int64_t n = decode_own_chunk(seqlens, b, cap) - wm1;   // candidates
  if (n < 0) n = 0;
  const float* sc = ws_scores + int64_t(row) * nc;
  int32_t* oid = sel_ids + int64_t(row) * K;
  float* osc = sel_scores + int64_t(row) * K;
  if (n <= K) {
    for (int t = tid; t < K; t += 256) {
      oid[t] = t < n ? t : -1;
      osc[t] = t < n ? sc[t] : -INFINITY;
    }
    return;
  }
  const int seg = int((n + 255) / 256);   // <= IT
  const int s0 = tid * seg;
  const int cnt = s0 >= n ? 0 : (s0 + seg <= n ? seg : int(n - s0));
  uint32_t key[IT];
  float val[IT];
#pragma unroll
  for (int e = 0; e < IT; ++e) {
    val[e] = e < cnt ? sc[s0 + e] : -INFINITY;
    key[e] = order_key(val[e]);
  }
  uint32_t prefix = 0, mask = 0;
  int krem = K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[tid] = 0;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < IT; ++e)
      if (e < cnt && (key[e] & mask) == prefix) atomicAdd(&hist[(key[e] >> shift) & 255u], 1u);
    __syncthreads();
    if (tid < 32) {
      uint32_t loc[8], lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { loc[j] = hist[255 - 8 * tid - j]; lsum += loc[j]; }
      uint32_t incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t excl = incl - lsum;
      if (excl < uint32_t(krem) && uint32_t(krem) <= incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + loc[j] >= uint32_t(krem)) { s_digit = 255 - 8 * tid - j; s_above = cum; break; }
          cum += loc[j];
        }
      }
    }
    __syncthreads();
    krem -= int(s_above);
    prefix |= s_digit << shift;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  // prefix = key of the K-th largest score; take every key above it and the
  // krem lowest-id keys equal to it, in chunk order
  int gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < IT; ++e) {
    gt += e < cnt && key[e] > prefix;
    eq += e < cnt && key[e] == prefix;
  }
  int tot;
  const int eq_before = block_exclusive_scan256(eq, warp_tot, tot);
  int take_eq = krem - eq_before;
  take_eq = take_eq < 0 ? 0 : (take_eq > eq ? eq : take_eq);
  int pos = block_exclusive_scan256(gt + take_eq, warp_tot, tot);
  int eq_seen = 0;
#pragma unroll
  for (int e = 0; e < IT; ++e) {
    if (e >= cnt) continue;
    bool take = key[e] > prefix;
    if (key[e] == prefix) take = eq_seen++ < take_eq;
    if (take && pos < K) { oid[pos] = int32_t(s0 + e); osc[pos] = val[e]; ++pos; }
  }
}

// D3, grouped by kv head: the G query heads of a kv head select overlapping
// chunk sets, so each distinct chunk is read once and attended by all heads
// that kept it.  One CTA per candidate slot (g, k) of the (b, kv head)'s
// G x K selections, plus one per chunk of the local window.  Thread 0 reads
// the slot's chunk id and starts the copies of its 64 key rows into shared
// memory at once (cp.async, 16 bytes per copy, all in flight; the 16-byte
// blocks of row r rotated by r mod 8 so that the key-per-lane reads hit
// distinct banks), after an L2 prefetch of the key and value rows.  While
// they land, warp 0 finds the heads that kept the chunk (binary search in
// their ascending id lists, one lane per head); a slot whose chunk an earlier
// head also kept is skipped (its copies are drained first).  Then, for up to
// four kept heads at a time, the four warps split the 64 keys: each scores
// its 16 keys (two lanes per key, half of the dimensions each) and keeps
// their weights, maximum and sum; the value rows replace the key rows in the
// same buffer (from L2 by then), each warp accumulates its keys' weighted
// values (lanes own dims), and the four partial results merge through shared
// memory.  One 64-row buffer instead of two keeps eight CTAs per SM instead
// of six.  A chunk is usually kept by one head only, so splitting its keys
// over the warps keeps all four busy.  Each head's partial goes to its own
// slot; invalid slots get score -inf.
template <typename T, int D>
struct DecUnion {
  static constexpr int RB = D * int(sizeof(T));   // bytes per key / value row
  static constexpr int NB = RB / 16;             // 16-byte blocks per row
  static constexpr uint32_t TILE = uint32_t(kChunk) * RB;
  // the key-then-value rows, queries, kept ids, per-head slots, a flag and the
  // copy offset, the kept heads' selection scores, then per warp its keys'
  // maximum, sum and partial output row (D + 4 floats), and per head of a
  // batch each thread's key weight and each warp's (max, sum) (all dynamic:
  // the kernel may be given the largest dynamic size, which leaves no room
  // for static shared memory)
  static constexpr int RED = D + 4;
  static size_t smem(int G, int K) {
    return size_t(TILE) + sizeof(float) * size_t(G) * D + sizeof(int32_t) * size_t(G) * K + sizeof(int32_t) * 36 +
           sizeof(float) * 32 + 16 + sizeof(float) * 4 * RED + sizeof(float) * (4 * 128 + 4 * 4 * 2) + 16;
  }
};

// 16 bytes from shared memory (shared-window address) as 8 bf16 or 4 fp32 values
template <typename T>
__device__ __forceinline__ void lds16(uint32_t saddr, float (&x)[16 / sizeof(T)]) {
  uint32_t w[4];
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(saddr));
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
      x[2 * i] = __low2float(v);
      x[2 * i + 1] = __high2float(v);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __uint_as_float(w[i]);
  }
}

__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <typename T, int D>
__global__ void __launch_bounds__(128, sizeof(T) == 2 ? 8 : 6)
decode_partial_union_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                            const int32_t* __restrict__ seqlens, int64_t cap, int Hq, int G, int Hkv, int K,
                            float tau, const int32_t* __restrict__ sel_ids, const float* __restrict__ sel_scores,
                            float* __restrict__ part_u, float* __restrict__ part_o, PagedKv pk, int wm1) {
  using U = DecUnion<T, D>;
  constexpr int EL = D / 32;                 // output dims per lane
  constexpr int EB = 16 / int(sizeof(T));    // elements per 16-byte block
  extern __shared__ __align__(16) uint8_t dsm[];
  // one [64][D] buffer: the chunk's keys (16-byte blocks rotated), then its values
  uint8_t* sk = dsm;
  float* sq = reinterpret_cast<float*>(dsm + U::TILE);          // [G][D] queries
  int32_t* sid = reinterpret_cast<int32_t*>(sq + G * D);        // [G][K] kept ids, ascending
  int* s_slot = sid + G * K;   // [32] per head: the chunk's slot in its list, -1 if not kept
  int& s_go = s_slot[32];
  int* s_off = s_slot + 34;   // [2] element offset of the chunk's rows, low and high words; -1: no copies
  float* s_sel = reinterpret_cast<float*>(s_slot + 36);   // [32] per kept head: its selection score
  // [4][RED] per-warp softmax statistics and partial outputs, 16-byte aligned
  float* s_red = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(s_sel + 32) + 15) & ~uintptr_t(15));
  // per head of a batch: each thread's key weight [4][128], then each warp's (max, sum) [4][4][2]
  float* s_pk = s_red + 4 * U::RED;
  float* s_ml = s_pk + 4 * 128;
  pdl_wait();      // the top-K lists
  pdl_trigger();
  const int bh = blockIdx.y, b = bh / Hkv, h = bh % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row0 = int64_t(b) * Hq + int64_t(h) * G;
  const int PS = K + wm1 + 1;    // partial slots per row
  // candidate slot g * K + k, or G * K + w for window chunk own - w
  const int pidx = blockIdx.x;
  const bool window = pidx >= G * K;
  const int64_t own = decode_own_chunk(seqlens, b, cap);
  if (own < 0 || (window && own < pidx - G * K)) {
    if (tid == 0 && !window) part_u[(row0 + pidx / K) * PS + pidx % K] = -INFINITY;
    if (tid < G && window) part_u[(row0 + tid) * PS + K + (pidx - G * K)] = -INFINITY;
    return;
  }
  const int64_t n_cand = own - wm1 > 0 ? own - wm1 : 0;
  int64_t j0, j1;
  if (tid == 0) {
    // the chunk and where its rows live (contiguous cache or chunk page; a
    // page outside the pool is recorded); the copies start right after the
    // barrier below, before the slot bookkeeping, and are drained if the
    // chunk turns out to belong to an earlier head
    int64_t c = -1;
    if (window) {
      c = own - (pidx - G * K);
    } else {
      const int32_t ci = sel_ids[row0 * K + pidx];
      if (ci >= 0 && ci < n_cand) c = ci;
    }
    const int64_t off = c >= 0 ? kv_chunk_offset(pk, b, h, c, Hkv, cap, cap / kChunk, D) : -1;
    if (off >= 0) {
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(kc + off), "r"(U::TILE) : "memory");
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(vc + off), "r"(U::TILE) : "memory");
    }
    s_off[0] = int(uint32_t(uint64_t(off)));
    s_off[1] = int(uint32_t(uint64_t(off) >> 32));
  }
  if (!window)
    for (int idx = tid; idx < G * K; idx += 128) sid[idx] = sel_ids[row0 * K + idx];
  for (int idx = tid; idx < G * D; idx += 128) {
    const T x = q[row0 * D + idx];
    if constexpr (sizeof(T) == 2) sq[idx] = __bfloat162float(x);
    else sq[idx] = x;
  }
  __syncthreads();
  const int64_t koff = int64_t((uint64_t(uint32_t(s_off[1])) << 32) | uint64_t(uint32_t(s_off[0])));
  // the chunk's 64 key and value rows, all copies in flight at once (the own
  // chunk lies inside the cache, whose capacity is a multiple of 64; keys
  // after the query are masked below)
  const uint8_t* kg = reinterpret_cast<const uint8_t*>(kc + (koff > 0 ? koff : 0));
  const uint8_t* vg = reinterpret_cast<const uint8_t*>(vc + (koff > 0 ? koff : 0));
  const uint32_t sk_a = uint32_t(__cvta_generic_to_shared(sk));
  // the chunk's 64 key rows (blocks rotated) or value rows into the buffer,
  // all copies in flight at once
  auto load_rows = [&](const uint8_t* src, bool keys) {
#pragma unroll 4
    for (int t = tid; t < kChunk * U::NB; t += 128) {
      const int r = t / U::NB, blk = t % U::NB;
      cp_async16(sk_a + (keys ? uint32_t(r * U::RB + ((blk ^ (r & 7)) << 4)) : uint32_t(t) * 16), src + size_t(t) * 16);
    }
  };
  if (koff >= 0) load_rows(kg, true);
  if (window) {
    const int w = pidx - G * K;
    j0 = (own - w) * kChunk;
    j1 = w == 0 ? int64_t(__ldg(seqlens + b)) : j0 + kChunk;
    if (tid < G) s_slot[tid] = koff >= 0 ? K + w : -1;
    if (tid == 0) s_go = 1;
  } else {
    const int g = pidx / K, k = pidx % K;
    const int32_t c = sid[g * K + k];
    j0 = int64_t(c) * kChunk;
    j1 = j0 + kChunk;
    if (warp == 0) {
      const bool bad = c < 0 || c >= n_cand;
      int my_slot = -1;
      if (!bad && lane < G) {
        const int32_t* ids = sid + lane * K;
        int lo = 0, hi = K - 1;
        while (lo <= hi) {
          const int mid = (lo + hi) >> 1;
          const int32_t v = ids[mid];
          if (v == c) { my_slot = mid; break; }
          // -1 padding sorts after the real ids
          if (v >= 0 && v < c) lo = mid + 1; else hi = mid - 1;
        }
      }
      const uint32_t mask = __ballot_sync(0xffffffffu, my_slot >= 0);
      // an earlier head's CTA takes a chunk that head also kept
      const bool go = !bad && !(mask & ((1u << g) - 1u));
      if (go && my_slot >= 0) {
        s_sel[lane] = sel_scores[(row0 + lane) * K + my_slot];
        // a page outside the pool: the chunk counts as not kept
        if (koff < 0) part_u[(row0 + lane) * PS + my_slot] = -INFINITY;
      }
      if (lane < G) s_slot[lane] = my_slot;
      if (lane == 0) {
        if (bad) {
          part_u[(row0 + g) * PS + k] = -INFINITY;
          if (c >= n_cand) record_error(HILS_ERR_DEVICE_BOUNDS);
        }
        s_go = go;
      }
    }
  }
  __syncthreads();
  if (window && koff < 0 && tid < G) part_u[(row0 + tid) * PS + K + (pidx - G * K)] = -INFINITY;
  // a skipped chunk's copies (if any) land before the CTA's shared memory is released
  cp_async_wait_all();
  if (!s_go || koff < 0) return;
  __syncthreads();
  // The heads that kept the chunk are taken in batches of up to four.  The
  // buffer first holds the keys: all four warps score the batch's heads,
  // warp w the keys 16w .. 16w+15 (lanes l and l+16 share key 16w + l%16,
  // each summing half of the dimensions), and keep each head's weights, key
  // maximum and sum.  Then the values replace the keys (they are in L2 by
  // now), each warp accumulates its keys' weighted values per head, and the
  // four warps' partial results merge through shared memory.  A chunk is
  // kept by one head of the kv head in most cases: one batch, each row read
  // once; a later batch reads the keys again.
  const int key = warp * 16 + (lane & 15), half = lane >> 4;
  const bool vk = j0 + key < j1;
  float* my_red = s_red + warp * U::RED;
  int next = 0;            // the next head to look at
  bool keys_in = true;     // the buffer holds the keys
  while (true) {
    uint32_t hb = 0;       // the batch, a head per byte (the same for the whole CTA)
    int nb = 0;
    while (next < G && nb < 4) {
      if (s_slot[next] >= 0) hb |= uint32_t(next) << (8 * nb++);
      ++next;
    }
    if (nb == 0) break;
    if (!keys_in) {
      load_rows(kg, true);
      cp_async_wait_all();
      __syncthreads();
    }
#pragma unroll 1
    for (int i = 0; i < nb; ++i) {
      const float* qg = sq + int((hb >> (8 * i)) & 255u) * D;
      float sd = 0.f;
#pragma unroll
      for (int bb = 0; bb < U::NB / 2; ++bb) {
        const int blk = half * (U::NB / 2) + bb;
        float x[EB];
        lds16<T>(sk_a + uint32_t(key * U::RB + ((blk ^ (key & 7)) << 4)), x);
#pragma unroll
        for (int e = 0; e < EB; ++e) sd = fmaf(qg[blk * EB + e], x[e], sd);
      }
      sd += __shfl_xor_sync(0xffffffffu, sd, 16);
      const float z = vk ? sd * tau : -INFINITY;
      float m = z;
#pragma unroll
      for (int off = 8; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const float p = (vk && m > -INFINITY) ? expf(z - m) : 0.f;
      float l = p;
#pragma unroll
      for (int off = 8; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      s_pk[i * 128 + tid] = p;
      if (lane == 0) {
        s_ml[(i * 4 + warp) * 2] = m;
        s_ml[(i * 4 + warp) * 2 + 1] = l;
      }
    }
    __syncthreads();   // every warp is done with the keys
    load_rows(vg, false);
    cp_async_wait_all();
    __syncthreads();
    keys_in = false;
#pragma unroll 1
    for (int i = 0; i < nb; ++i) {
      const int g = int((hb >> (8 * i)) & 255u), slot = s_slot[g];
      // the warp's 16 keys' weighted values: lane owns dims lane * EL .. + EL - 1
      float o[EL];
#pragma unroll
      for (int e = 0; e < EL; ++e) o[e] = 0.f;
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const T* vrow = reinterpret_cast<const T*>(sk + (warp * 16 + jj) * U::RB) + lane * EL;
        const float pj = s_pk[i * 128 + warp * 32 + jj];   // key 16w + jj, as lane jj holds it
#pragma unroll
        for (int e = 0; e < EL; ++e) {
          float xv;
          if constexpr (sizeof(T) == 2) xv = __bfloat162float(vrow[e]);
          else xv = vrow[e];
          o[e] = fmaf(pj, xv, o[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < EL; ++e) my_red[lane * EL + e] = o[e];
      if (lane == 0) {
        my_red[D] = s_ml[(i * 4 + warp) * 2];
        my_red[D + 1] = s_ml[(i * 4 + warp) * 2 + 1];
      }
      __syncthreads();
      // merge the four warps: M = max m_w, L = sum l_w e^(m_w - M), O = sum o_w e^(m_w - M) / L
      float mw[4], M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        mw[w] = s_red[w * U::RED + D];
        M = fmaxf(M, mw[w]);
      }
      float L = 0.f, f[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        f[w] = mw[w] > -INFINITY ? expf(mw[w] - M) : 0.f;
        L = fmaf(s_red[w * U::RED + D + 1], f[w], L);
      }
      const int64_t row = row0 + g;
      if (tid < D) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) acc = fmaf(s_red[w * U::RED + tid], f[w], acc);
        part_o[(row * PS + slot) * D + tid] = acc / L;
      }
      if (tid == 0) part_u[row * PS + slot] = slot >= K ? M + logf(L) : s_sel[g];
      __syncthreads();   // s_red is reused by the next head
    }
  }
}

// D4: one CTA of D threads per row, thread t owns output dim t.  Every
// thread reads the row's slot scores itself (the same addresses for the
// whole CTA, so no shared memory and no block barrier) together with its
// dim of the slots' partial rows, kCombBlock slots per round with all
// loads in flight, and folds each round into a running softmax (maximum,
// sum of weights, weighted sum).  A slot with score -inf was not written
// with a partial row: its load is made but its value is discarded by a
// select, never multiplied.  The kernel is load-latency bound: one round
// trip per kCombBlock slots.
constexpr int kCombBlock = 24;

template <typename T, int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const float* __restrict__ part_u, const float* __restrict__ part_o,
                      const int32_t* __restrict__ seqlens, int64_t cap, int Hq, int K,
                      const int32_t* __restrict__ sel_ids, const float* __restrict__ sel_scores,
                      T* __restrict__ o, int32_t* __restrict__ ids_out, float* __restrict__ scores_out,
                      int64_t n_rows, int wm1) {
  pdl_wait();      // the partial outputs
  const int t = threadIdx.x;
  const int64_t row = blockIdx.x;
  const int b = int(row / Hq);
  const bool valid = decode_own_chunk(seqlens, b, cap) >= 0;
  const int PS = K + wm1 + 1;
  const float* pu = part_u + row * PS;
  const float* po = part_o + row * PS * D + t;
  float M = -INFINITY, Z = 0.f, acc = 0.f;
  for (int s0 = 0; s0 < PS; s0 += kCombBlock) {
    float u[kCombBlock], x[kCombBlock];
#pragma unroll
    for (int e = 0; e < kCombBlock; ++e) {
      const bool in = s0 + e < PS;
      u[e] = in ? __ldg(pu + s0 + e) : -INFINITY;
      x[e] = in ? po[int64_t(s0 + e) * D] : 0.f;
    }
    float m = M;
#pragma unroll
    for (int e = 0; e < kCombBlock; ++e) m = fmaxf(m, u[e]);
    if (!valid || m == -INFINITY) continue;
    // rescale what the earlier rounds summed to the new maximum
    const float r = M == -INFINITY ? 0.f : expf(M - m);
    Z *= r;
    acc *= r;
#pragma unroll
    for (int e = 0; e < kCombBlock; ++e) {
      const bool live = u[e] != -INFINITY;
      const float w = live ? expf(u[e] - m) : 0.f;
      Z += w;
      acc = fmaf(w, live ? x[e] : 0.f, acc);
    }
    M = m;
  }
  const float y = Z > 0.f ? acc / Z : 0.f;
  if constexpr (sizeof(T) == 2) o[row * D + t] = __float2bfloat16_rn(y);
  else o[row * D + t] = y;
  for (int k = t; k < K; k += D) {
    if (ids_out) ids_out[row * K + k] = valid ? sel_ids[row * K + k] : -1;
    if (scores_out) scores_out[row * K + k] = valid ? sel_scores[row * K + k] : -INFINITY;
  }
}

}  // namespace hils
