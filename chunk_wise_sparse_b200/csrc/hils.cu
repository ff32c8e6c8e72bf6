// C ABI of the HiLS attention forward library: argument validation, dispatch
// on (dtype, head_dim) and kernel launches.  See include/hils.h for the
// contract of every entry point.
#include <atomic>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "hils.h"
#include "common.cuh"
#include "summary.cuh"
#include "select_simt.cuh"
#include "attend_simt.cuh"
#include "decode.cuh"
#include "select_tc.cuh"
#include "prefill_cc.cuh"
#include "prefill_local.cuh"
#include "qcal.cuh"
#include "backward.cuh"
#include "backward_mma.cuh"

using namespace hils;

namespace {

std::atomic<uint64_t> g_launches{0};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }

int check_dims(const hils_dims* d) {
  if (d == nullptr) return HILS_ERR_INVALID_ARGUMENT;
  if (d->batch < 1 || d->heads_q < 1 || d->heads_kv < 1 || d->heads_q % d->heads_kv != 0)
    return HILS_ERR_INVALID_ARGUMENT;
  if (d->seqlen < 1 || d->chunk < 1) return HILS_ERR_INVALID_ARGUMENT;
  if (d->window < 0 || d->window % kChunk != 0) return HILS_ERR_INVALID_ARGUMENT;
  if (d->window > 16 * kChunk) return HILS_ERR_UNSUPPORTED;
  if (d->dtype != HILS_BF16 && d->dtype != HILS_FP32) return HILS_ERR_INVALID_ARGUMENT;
  if (d->chunk != kChunk) return HILS_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128) return HILS_ERR_UNSUPPORTED;
  if (d->topk < 1 || d->topk > kMaxTopK) return HILS_ERR_UNSUPPORTED;
  if (d->seqlen % d->chunk != 0) return HILS_ERR_INVALID_ARGUMENT;
  if (d->seqlen > (int64_t(1) << 31)) return HILS_ERR_UNSUPPORTED;
  return HILS_OK;
}

// chunks of the local window before the own chunk
inline int window_wm1(const hils_dims* d) { return d->window > kChunk ? d->window / kChunk - 1 : 0; }

// Launch with programmatic stream serialisation: the kernel may be scheduled
// before the previous kernel in the stream completes and must call pdl_wait()
// before it touches that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*fn)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, static_cast<KArgs>(args)...);
}

inline int launched(int n) {
  g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

constexpr int kMaxSmem = 227 * 1024;

// cudaFuncSetAttribute to the largest dynamic shared memory, once per (kernel, device).
template <auto FN>
cudaError_t set_smem_max() {
  static std::atomic<uint32_t> done_mask{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint32_t bit = 1u << (dev & 31);
  if (done_mask.load(std::memory_order_acquire) & bit) return cudaSuccess;
  // the per-block limit covers static and dynamic shared memory together
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, FN);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(FN, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem - int(fa.sharedSizeBytes));
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<void*> fn{nullptr};
  void* f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn.store(f, std::memory_order_release);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// 2D bf16 tensor map: `rows` rows of `inner` elements, `row_bytes` apart.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 tensor map [planes][rows][inner], 128-byte swizzle, box {64, box_rows, 1}.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t planes,
                 uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {inner, rows, planes};
  cuuint64_t strides[2] = {inner * 2, inner * 2 * rows};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core selection handles bf16 with G a power of two up to 16.
bool select_tc_supported(const hils_dims* d) {
  const int G = d->heads_q / d->heads_kv;
  const int64_t rows_q = int64_t(d->batch) * d->heads_q * d->seqlen;
  return d->dtype == HILS_BF16 && G <= 16 && (G & (G - 1)) == 0 && rows_q < (int64_t(1) << 31);
}

template <int D, int KCAP>
int launch_select_tc(const hils_dims* d, const void* q, const void* kmma, int32_t* ids, float* scores,
                     cudaStream_t st) {
  using C = SelTc<D, KCAP>;
  const int G = d->heads_q / d->heads_kv, P = C::M / G;
  const int64_t N = d->seqlen, nc = N / kChunk;
  const uint64_t rows_q = uint64_t(d->batch) * d->heads_q * N, rows_k = uint64_t(d->batch) * d->heads_kv * nc;
  CUtensorMap tq, tkb, tke;
  if (!make_map_2d(&tq, q, D, rows_q, D * 2, 64, P, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tkb, kmma, D + kExt, rows_k, (D + kExt) * 2, 64, C::NT, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tke, kmma, D + kExt, rows_k, (D + kExt) * 2, kExt, C::NT, CU_TENSOR_MAP_SWIZZLE_32B))
    return HILS_ERR_CUDA;
  // d = 64 with K <= 16 keeps two CTAs per SM (228 KB per SM, 1 KB of it
  // reserved per CTA); the rest run one CTA per SM.  Two k' stages; the
  // candidate buffer takes what shared memory is left (it is compacted less
  // often the longer it is), at most 128 entries.
  const uint32_t per_cta = C::TWO_PER_SM ? 115712u : uint32_t(kMaxSmem);
  const int stages = 2;
  int cap = KCAP > 0 ? C::MIN_CAP : 0;
  if (KCAP > 0)
    while (cap + 8 <= 128 && C::layout(d->topk, stages, cap + 8).total <= per_cta) cap += 8;
  const uint32_t smem = C::layout(d->topk, stages, cap).total;
  if (smem > uint32_t(kMaxSmem)) return HILS_ERR_UNSUPPORTED;
  // no more CTAs per SM than 512 TMEM columns hold (a tcgen05.alloc would
  // otherwise wait for columns a co-resident persistent CTA never frees)
  if ((512u / C::TMEM_COLS + 1u) * (smem + 1024u) <= 233472u) return HILS_ERR_UNSUPPORTED;
  constexpr auto fn = select_tc_kernel<D, KCAP>;
  if (set_smem_max<fn>() != cudaSuccess) return HILS_ERR_CUDA;
  SelTcParams p;
  p.n_tok = N;
  p.nc = nc;
  p.Hq = d->heads_q;
  p.Hkv = d->heads_kv;
  p.G = G;
  p.K = d->topk;
  p.P = P;
  p.n_row_tiles = int((N + P - 1) / P);
  p.stages = stages;
  p.cap = cap;
  p.wm1 = window_wm1(d);
  p.tau = 1.f / sqrtf(float(D));
  p.ids = ids;
  p.scores = scores;
  dim3 grid(unsigned(p.n_row_tiles), unsigned(d->batch * d->heads_kv));
  fn<<<grid, C::THREADS, smem, st>>>(tq, tkb, tke, p);
  return launched(1);
}

// ---------------------------------------------------------------- chunk-centric prefill (bf16)
struct CcPlan {
  CcDims c;
  int64_t rows, n_slots, max_items, n_scan_blocks;
  int P, own_tiles;
  size_t off_oacc, off_rowstat, off_counts, off_ranks, off_cbase, off_offsets, off_tiles, off_items, off_sums, off_epair,
      off_rescore, total;
};

bool cc_supported(const hils_dims* d) {
  const int64_t G = d->heads_q / d->heads_kv;
  const int64_t rows = int64_t(d->batch) * d->heads_q * d->seqlen;
  return d->dtype == HILS_BF16 && G <= 16 && (G & (G - 1)) == 0 &&
         G * d->seqlen <= (int64_t(1) << 25) &&
         rows * d->topk < (int64_t(1) << 31);
}

// Sizes of the chunk-centric index over (kv head, window, chunk) keys.
CcDims make_cc_dims(const hils_dims* d) {
  CcDims c;
  const int64_t N = d->seqlen, D = d->head_dim, G = d->heads_q / d->heads_kv;
  c.n_tok = N;
  c.nc = N / kChunk;
  c.Hq = d->heads_q;
  c.Hkv = d->heads_kv;
  c.G = int(G);
  c.K = d->topk;
  c.wm1 = window_wm1(d);
  c.tau = 1.f / sqrtf(float(D));
  // window: the fp32 accumulators and bf16 queries of one window of one kv head
  // (G x W positions) stay within 64 MiB of L2
  int shift = 6;
  while ((int64_t(1) << (shift + 1)) <= N && G * (int64_t(1) << (shift + 1)) * D * 6 <= (int64_t(64) << 20)) ++shift;
  c.win_shift = shift;
  c.n_win = int((N + (int64_t(1) << shift) - 1) >> shift);
  c.n_keys = int64_t(d->batch) * d->heads_kv * c.n_win * c.nc;
  return c;
}

// The count takes one shared-memory histogram per kCountRows rows when those
// rows stay in one window and the chunk histogram fits; its per-(CTA, chunk)
// bases then need a table of rows / kCountRows x nc entries.
bool cc_two_level_count(const CcDims& c) {
  return c.n_tok % kCountRows == 0 && (int64_t(1) << c.win_shift) % kCountRows == 0 &&
         sizeof(int32_t) * size_t(c.nc) <= 96 * 1024;
}
size_t cc_cbase_entries(const CcDims& c, int64_t rows) {
  return cc_two_level_count(c) ? size_t(rows / kCountRows) * size_t(c.nc) : 0;
}

// The chunk-centric index of a selection (counts zeroed by the caller): pair
// counts and ranks, the scan into per-key offsets and tiles, and the fill of
// the (row, s^ - M') records.  Five launches.
int launch_cc_index(const CcDims& c, int64_t rows, int64_t n_slots, int64_t n_scan_blocks, const int32_t* ids,
                    const float* scores, const float* rowstat, int32_t* counts, int32_t* ranks, int32_t* cbase,
                    int64_t* offsets, int32_t* tiles, int4* items, int64_t* sums, int2* e_pair, cudaStream_t st) {
  if (cc_two_level_count(c)) {
    const size_t hist_bytes = sizeof(int32_t) * size_t(c.nc);
    constexpr auto cfn = cc_count_kernel;
    if (hist_bytes > 48 * 1024 && set_smem_max<cfn>() != cudaSuccess) return HILS_ERR_CUDA;
    cfn<<<unsigned(rows / kCountRows), kCountThreads, hist_bytes, st>>>(ids, counts, ranks, cbase, c);
  } else {
    cbase = nullptr;
    cc_count_direct_kernel<<<unsigned((n_slots + 255) / 256), 256, 0, st>>>(ids, counts, ranks, c, n_slots);
  }
  const unsigned nsb = unsigned(n_scan_blocks);
  cc_scan_sums_kernel<<<nsb, 256, 0, st>>>(counts, c.n_keys, sums);
  cc_scan_blocks_kernel<<<1, 1024, 0, st>>>(sums, n_scan_blocks, c.n_keys, offsets, tiles);
  cc_scan_apply_kernel<<<nsb, 256, 0, st>>>(counts, c, sums, offsets, tiles, items);
  if (c.K % 4 == 0)
    cc_fill4_kernel<<<unsigned((n_slots / 4 + 255) / 256), 256, 0, st>>>(ids, ranks, cbase, scores, rowstat, offsets,
                                                                          e_pair, c, n_slots / 4);
  else
    cc_fill_kernel<<<unsigned((n_slots + 255) / 256), 256, 0, st>>>(ids, ranks, cbase, scores, rowstat, offsets,
                                                                     e_pair, c, n_slots);
  return HILS_OK;
}

CcPlan cc_plan(const hils_dims* d) {
  CcPlan P;
  const int64_t N = d->seqlen, D = d->head_dim, G = d->heads_q / d->heads_kv;
  P.c = make_cc_dims(d);
  P.rows = int64_t(d->batch) * d->heads_q * N;
  P.n_slots = P.rows * d->topk;
  P.P = int(128 / G);
  P.own_tiles = int((N + P.P - 1) / P.P);
  P.n_scan_blocks = (P.c.n_keys + kScanBlock - 1) / kScanBlock;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~size_t(255); return o; };
  P.off_oacc = take(sizeof(float) * P.rows * D);
  P.off_rowstat = take(sizeof(float) * P.rows);
  P.off_counts = take(sizeof(int32_t) * P.c.n_keys);
  P.off_ranks = take(sizeof(int32_t) * P.n_slots);
  P.off_cbase = take(sizeof(int32_t) * cc_cbase_entries(P.c, P.rows));
  P.off_offsets = take(sizeof(int64_t) * (P.c.n_keys + 1));
  P.off_tiles = take(sizeof(int32_t) * (P.c.n_keys + 1));
  P.max_items = P.n_slots / kCcTileRows + P.c.n_keys + 1;
  P.off_items = take(sizeof(int4) * P.max_items);
  P.off_sums = take(sizeof(int64_t) * 2 * P.n_scan_blocks);
  // entries are padded by one tile so that tile loads never run past the end
  P.off_epair = take(sizeof(int2) * (P.n_slots + kCcTileRows));
  // the recomputed chunk scores of a call without the selection's scores
  P.off_rescore = take(sizeof(float) * P.n_slots);
  P.total = off;
  return P;
}

int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  int v = cached[dev & 63].load(std::memory_order_relaxed);
  if (v == 0) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached[dev & 63].store(v, std::memory_order_relaxed);
  }
  return v;
}

template <int D>
int launch_prefill_cc(const hils_dims* d, const void* q, const void* k, const void* v, const void* kmma,
                      const int32_t* ids, const float* scores, void* o, float* lse, void* ws, cudaStream_t st) {
  using C = CcTc<D>;
  using CO = CcOwn<D>;
  const CcPlan P = cc_plan(d);
  char* base = static_cast<char*>(ws);
  float* oacc = reinterpret_cast<float*>(base + P.off_oacc);
  float* rowstat = reinterpret_cast<float*>(base + P.off_rowstat);
  int32_t* counts = reinterpret_cast<int32_t*>(base + P.off_counts);
  int32_t* ranks = reinterpret_cast<int32_t*>(base + P.off_ranks);
  int32_t* cbase = reinterpret_cast<int32_t*>(base + P.off_cbase);
  int64_t* offsets = reinterpret_cast<int64_t*>(base + P.off_offsets);
  int32_t* tiles = reinterpret_cast<int32_t*>(base + P.off_tiles);
  int4* items = reinterpret_cast<int4*>(base + P.off_items);
  int64_t* sums = reinterpret_cast<int64_t*>(base + P.off_sums);
  int2* e_pair = reinterpret_cast<int2*>(base + P.off_epair);
  const uint64_t kv_rows = uint64_t(d->batch) * d->heads_kv * d->seqlen;
  const uint32_t nk_own = P.P >= kChunk ? uint32_t(P.P) : uint32_t(kChunk);
  CUtensorMap tq_tile, tq_row, tk, tv, tk_own, tv_own;
  if (!make_map_2d(&tq_tile, q, D, uint64_t(P.rows), D * 2, 64, uint32_t(P.P), CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tq_row, q, D, uint64_t(P.rows), D * 2, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tk, k, D, kv_rows, D * 2, 64, kChunk, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tv, v, D, kv_rows, D * 2, 64, kChunk, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tk_own, k, D, kv_rows, D * 2, 64, nk_own, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tv_own, v, D, kv_rows, D * 2, 64, nk_own, CU_TENSOR_MAP_SWIZZLE_128B))
    return HILS_ERR_CUDA;
  // own (or local window), count, three scans, fill, attend, final
  int n_launch = 8;
  if (scores == nullptr) {
    // no scores from the selection: recompute s^ of the kept ids
    float* rescore = reinterpret_cast<float*>(base + P.off_rescore);
    cc_rescore_kernel<D><<<unsigned((P.n_slots + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(kmma), ids, rescore, P.c, P.n_slots);
    scores = rescore;
    ++n_launch;
  }
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * P.c.n_keys, st) != cudaSuccess) return HILS_ERR_CUDA;
  // the padding after the last entry must hold valid row ids (row 0)
  if (cudaMemsetAsync(base + P.off_epair + sizeof(int2) * P.n_slots, 0, sizeof(int2) * kCcTileRows, st) !=
      cudaSuccess)
    return HILS_ERR_CUDA;
  CcOwnParams op;
  op.c = P.c;
  op.ids = ids;
  op.scores = scores;
  op.oacc = oacc;
  op.rowstat = rowstat;
  op.lse_own = lse;
  op.P = P.P;
  op.n_tiles = P.own_tiles;
  const dim3 own_grid(unsigned(P.own_tiles), unsigned(d->batch * d->heads_kv));
  if (P.c.wm1 == 0) {
    constexpr auto own_fn = cc_own_tc_kernel<D>;
    if (set_smem_max<own_fn>() != cudaSuccess) return HILS_ERR_CUDA;
    own_fn<<<own_grid, 128, CO::SMEM, st>>>(tq_tile, tk_own, tv_own, op);
  } else {
    // the local window spans more than the own chunk
    using CL = CcLocal<D>;
    constexpr auto loc_fn = cc_local_tc_kernel<D>;
    if (set_smem_max<loc_fn>() != cudaSuccess) return HILS_ERR_CUDA;
    loc_fn<<<own_grid, CL::THREADS, CL::SMEM, st>>>(tq_tile, tk, tv, op);
  }
  const int ix = launch_cc_index(P.c, P.rows, P.n_slots, P.n_scan_blocks, ids, scores, rowstat, counts, ranks, cbase,
                                 offsets, tiles, items, sums, e_pair, st);
  if (ix != HILS_OK) return ix;
  constexpr auto fn = cc_attend_kernel<D>;
  if (set_smem_max<fn>() != cudaSuccess) return HILS_ERR_CUDA;
  CcTcParams prm;
  prm.c = P.c;
  prm.tile_start = tiles;
  prm.items = items;
  prm.e_pair = e_pair;
  prm.oacc = oacc;
  fn<<<unsigned(sm_count() * C::MAX_CTAS), C::THREADS, C::SMEM, st>>>(tq_row, tk, tv, prm);
  const int64_t n8 = P.rows * D / 8;
  cc_final_kernel<D><<<unsigned((n8 + 255) / 256), 256, 0, st>>>(oacc, static_cast<__nv_bfloat16*>(o), n8);
  return launched(n_launch);
}

// ---------------------------------------------------------------- backward
struct BwdPlan {
  CcDims c;
  int64_t rows, n_slots, max_items, n_scan_blocks, n_units;
  size_t off_rowstat, off_dvec, off_counts, off_ranks, off_cbase, off_offsets, off_tiles, off_items, off_sums,
      off_epair, off_dkp, off_dbp, total;
};

BwdPlan bwd_plan(const hils_dims* d) {
  BwdPlan P;
  P.c = make_cc_dims(d);
  const int64_t D = d->head_dim;
  P.rows = int64_t(d->batch) * d->heads_q * d->seqlen;
  P.n_slots = P.rows * d->topk;
  P.n_units = int64_t(d->batch) * d->heads_kv * P.c.nc;
  P.n_scan_blocks = (P.c.n_keys + kScanBlock - 1) / kScanBlock;
  P.max_items = P.n_slots / kCcTileRows + P.c.n_keys + 1;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~size_t(255); return o; };
  P.off_rowstat = take(sizeof(float) * P.rows);
  P.off_dvec = take(sizeof(float) * P.rows);
  P.off_counts = take(sizeof(int32_t) * P.c.n_keys);
  P.off_ranks = take(sizeof(int32_t) * P.n_slots);
  P.off_cbase = take(sizeof(int32_t) * cc_cbase_entries(P.c, P.rows));
  P.off_offsets = take(sizeof(int64_t) * (P.c.n_keys + 1));
  P.off_tiles = take(sizeof(int32_t) * (P.c.n_keys + 1));
  P.off_items = take(sizeof(int4) * P.max_items);
  P.off_sums = take(sizeof(int64_t) * 2 * P.n_scan_blocks);
  P.off_epair = take(sizeof(int2) * (P.n_slots + kCcTileRows));
  P.off_dkp = take(sizeof(float) * P.n_units * D);
  P.off_dbp = take(sizeof(float) * P.n_units);
  P.total = off;
  return P;
}

template <typename T, int D>
int launch_backward(const hils_dims* d, const void* q, const void* q_score, const void* k, const void* v,
                    const void* lq, const float* kprime, const int32_t* ids, const float* scores, const float* lse_w,
                    const void* o, const void* d_o, float* dq, float* dq_score, float* dk, float* dv, float* dlq,
                    void* ws, cudaStream_t st) {
  using BT = BwdTiles<D>;
  const BwdPlan P = bwd_plan(d);
  char* base = static_cast<char*>(ws);
  float* rowstat = reinterpret_cast<float*>(base + P.off_rowstat);
  float* dvec = reinterpret_cast<float*>(base + P.off_dvec);
  int32_t* counts = reinterpret_cast<int32_t*>(base + P.off_counts);
  int32_t* ranks = reinterpret_cast<int32_t*>(base + P.off_ranks);
  int32_t* cbase = reinterpret_cast<int32_t*>(base + P.off_cbase);
  int64_t* offsets = reinterpret_cast<int64_t*>(base + P.off_offsets);
  int32_t* tiles = reinterpret_cast<int32_t*>(base + P.off_tiles);
  int4* items = reinterpret_cast<int4*>(base + P.off_items);
  int64_t* sums = reinterpret_cast<int64_t*>(base + P.off_sums);
  int2* e_pair = reinterpret_cast<int2*>(base + P.off_epair);
  float* dkp = reinterpret_cast<float*>(base + P.off_dkp);
  float* dbp = reinterpret_cast<float*>(base + P.off_dbp);
  const int64_t N = d->seqlen, kv_elems = int64_t(d->batch) * d->heads_kv * N * D;
  const int G = d->heads_q / d->heads_kv;
  const T* tq = static_cast<const T*>(q);
  const T* tk = static_cast<const T*>(k);
  const T* tv = static_cast<const T*>(v);
  const T* tdo = static_cast<const T*>(d_o);
  if (cudaMemsetAsync(dk, 0, sizeof(float) * kv_elems, st) != cudaSuccess ||
      cudaMemsetAsync(dv, 0, sizeof(float) * kv_elems, st) != cudaSuccess ||
      cudaMemsetAsync(dkp, 0, sizeof(float) * P.n_units * (D + 0), st) != cudaSuccess ||
      cudaMemsetAsync(dbp, 0, sizeof(float) * P.n_units, st) != cudaSuccess ||
      cudaMemsetAsync(counts, 0, sizeof(int32_t) * P.c.n_keys, st) != cudaSuccess ||
      cudaMemsetAsync(base + P.off_epair + sizeof(int2) * P.n_slots, 0, sizeof(int2) * kCcTileRows, st) !=
          cudaSuccess)
    return HILS_ERR_CUDA;
  if (dq_score && cudaMemsetAsync(dq_score, 0, sizeof(float) * P.rows * D, st) != cudaSuccess) return HILS_ERR_CUDA;
  bwd_prep_kernel<T, D><<<unsigned((P.rows * 32 + 127) / 128), 128, 0, st>>>(
      ids, scores, lse_w, static_cast<const T*>(o), tdo, N, d->topk, P.c.wm1, P.rows, rowstat, dvec);
  // the forward's index: per (kv head, window, chunk) its (row, slot) pairs and s^ - M'
  const int ix = launch_cc_index(P.c, P.rows, P.n_slots, P.n_scan_blocks, ids, scores, rowstat, counts, ranks, cbase,
                                 offsets, tiles, items, sums, e_pair, st);
  if (ix != HILS_OK) return ix;
  const float tau = 1.f / sqrtf(float(D));
  if (std::is_same<T, __nv_bfloat16>::value) {
    // bf16: the window branch's products on tensor cores
    using WT = BwdWinMma<D>;
    constexpr auto wfn = bwd_window_mma_kernel<D>;
    if (set_smem_max<wfn>() != cudaSuccess) return HILS_ERR_CUDA;
    wfn<<<dim3(unsigned(P.c.nc), unsigned(d->batch * d->heads_q)), WT::THREADS, WT::SMEM, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(d_o), rowstat, dvec, N,
        d->heads_q, G, d->heads_kv, P.c.wm1, tau, dq, dk, dv);
  } else {
    const size_t smem_w = BT::KV_BYTES + BT::ROW_BYTES + BT::P_BYTES + size_t(BT::SUB) * D * 4;
    constexpr auto wfn = bwd_window_kernel<T, D>;
    if (set_smem_max<wfn>() != cudaSuccess) return HILS_ERR_CUDA;
    wfn<<<dim3(unsigned(P.c.nc), unsigned(d->batch * d->heads_q)), BT::THREADS, smem_w, st>>>(
        tq, tk, tv, tdo, rowstat, dvec, N, d->heads_q, G, d->heads_kv, P.c.wm1, tau, dq, dk, dv);
  }
  if (std::is_same<T, __nv_bfloat16>::value && q_score == nullptr && dq_score == nullptr) {
    // bf16 with the attention query as the scoring query: the selected
    // chunks' five products on tensor cores (mma.sync)
    using MT = BwdMma<D>;
    constexpr auto mfn = bwd_chunk_mma_kernel<D>;
    if (set_smem_max<mfn>() != cudaSuccess) return HILS_ERR_CUDA;
    mfn<<<unsigned(sm_count() * MT::CTAS_PER_SM), MT::THREADS, MT::SMEM, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(d_o), kprime, dvec, tiles, items,
        e_pair, P.c, dq, dk, dv, dkp, dbp);
  } else {
    const size_t smem_c = BT::KV_BYTES + BT::ROW_BYTES + BT::P_BYTES + size_t(2 * D + 4) * 4;
    constexpr auto cfn2 = bwd_chunk_kernel<T, D>;
    if (set_smem_max<cfn2>() != cudaSuccess) return HILS_ERR_CUDA;
    cfn2<<<unsigned(sm_count() * 2), BT::THREADS, smem_c, st>>>(
        tq, static_cast<const T*>(q_score), tk, tv, tdo, kprime, dvec, tiles, items, e_pair, P.c, dq,
        dq_score ? dq_score : dq, dk, dv, dkp, dbp);
  }
  const size_t smem_s = size_t(4) * (kChunk * BT::KS + 3 * D) * 4;
  constexpr auto sfn = bwd_summary_kernel<T, D>;
  if (set_smem_max<sfn>() != cudaSuccess) return HILS_ERR_CUDA;
  sfn<<<unsigned((P.n_units + 3) / 4), 128, smem_s, st>>>(tk, static_cast<const T*>(lq), kprime, dkp, dbp, N, P.c.nc,
                                                          P.n_units, tau, dk, dlq);
  // prep, count, three scans, fill, window, chunks, summary
  return launched(9);
}

template <typename T, int D>
int launch_summary(const hils_dims* d, const void* k, const void* lq, int64_t c0, int64_t c1, float* kp,
                   float* bp, void* kmma, cudaStream_t st, PagedKv pk = PagedKv{nullptr, 0}) {
  const int64_t nc = d->seqlen / kChunk, span = c1 - c0;
  const int64_t units = int64_t(d->batch) * d->heads_kv * span;
  const int64_t blocks = (units * 32 + 255) / 256;
  summary_kernel<T, D><<<dim3(unsigned(blocks)), 256, 0, st>>>(
      static_cast<const T*>(k), static_cast<const T*>(lq), d->seqlen, nc, c0, span, units, kp, bp,
      static_cast<__nv_bfloat16*>(kmma), 1.f / sqrtf(float(D)), pk, d->heads_kv);
  return launched(1);
}

template <typename T, int D, bool MMA>
int launch_select_simt(const hils_dims* d, const void* q, const float* kp, const float* bp, const void* kmma,
                       const int64_t* row_pos, int64_t n_rows, int32_t* ids, float* scores, cudaStream_t st) {
  const size_t smem = select_simt_smem<D>(d->topk);
  constexpr auto fn = select_simt_kernel<T, D, MMA>;
  if (set_smem_max<fn>() != cudaSuccess) return HILS_ERR_CUDA;
  dim3 grid(unsigned((n_rows + kSelRows - 1) / kSelRows), unsigned(d->batch * d->heads_q));
  fn<<<grid, kSelRows, smem, st>>>(static_cast<const T*>(q), kp, bp, static_cast<const __nv_bfloat16*>(kmma),
                                  d->seqlen, d->seqlen / kChunk, d->heads_q, d->heads_q / d->heads_kv,
                                  d->heads_kv, d->topk, 1.f / sqrtf(float(D)), ids, scores, window_wm1(d), row_pos,
                                  n_rows);
  return launched(1);
}

template <typename T, int D>
int launch_prefill_simt(const hils_dims* d, const void* q, const void* k, const void* v, const float* kp,
                        const float* bp, const void* kmma, const int32_t* ids, const float* scores, void* o,
                        float* lse, cudaStream_t st) {
  const int64_t rows = int64_t(d->batch) * d->heads_q * d->seqlen;
  const int64_t blocks = (rows + 3) / 4;
  prefill_simt_kernel<T, D><<<dim3(unsigned(blocks)), 128, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), ids, scores,
      static_cast<T*>(o), lse, d->seqlen, d->heads_q, d->heads_q / d->heads_kv, d->heads_kv, d->topk,
      1.f / sqrtf(float(D)), rows, window_wm1(d), kp, bp, static_cast<const __nv_bfloat16*>(kmma));
  return launched(1);
}

template <typename T, int D>
int launch_decode(const hils_dims* d, const void* q, const void* kc, const void* vc, const float* kp,
                  const float* bp, const void* kmma, const int32_t* seqlens, void* o, int32_t* ids_out,
                  float* scores_out, void* ws_ptr, cudaStream_t st, PagedKv pk = PagedKv{nullptr, 0},
                  const void* q_score = nullptr) {
  constexpr bool BF = std::is_same<T, __nv_bfloat16>::value;
  const int64_t nc = d->seqlen / kChunk, rows = int64_t(d->batch) * d->heads_q;
  const int G = d->heads_q / d->heads_kv, K = d->topk;
  const float tau = 1.f / sqrtf(float(D));
  DecodeWs ws;
  const int wm1 = window_wm1(d);
  decode_ws_layout(rows, nc, K, wm1 + 1, D, static_cast<char*>(ws_ptr), &ws);
  const size_t smem1 = decode_scores_smem<D, BF>(G);
  constexpr auto k1 = decode_scores_kernel<T, D, BF>;
  if (smem1 > 48 * 1024 && set_smem_max<k1>() != cudaSuccess) return HILS_ERR_CUDA;
  dim3 g1(unsigned((nc + kDecChunksPerCta - 1) / kDecChunksPerCta), unsigned(d->batch * d->heads_kv));
  k1<<<g1, kDecChunksPerCta, smem1, st>>>(static_cast<const T*>(q_score ? q_score : q), kp, bp, static_cast<const __nv_bfloat16*>(kmma), seqlens,
                            d->seqlen, nc, d->heads_q, G, d->heads_kv, tau, ws.scores, wm1);
  // the next three kernels start while their predecessor finishes and wait
  // for it on the device (programmatic dependent launch)
  const dim3 g2(static_cast<unsigned>(rows));
  cudaError_t e;
  if (nc <= 256 * 16)
    e = launch_pdl(decode_topk_reg_kernel<16>, g2, 256, 0, st, ws.scores, seqlens, d->seqlen, nc, d->heads_q, K,
                   ws.sel_ids, ws.sel_scores, wm1);
  else if (nc <= 256 * 32)
    e = launch_pdl(decode_topk_reg_kernel<32>, g2, 256, 0, st, ws.scores, seqlens, d->seqlen, nc, d->heads_q, K,
                   ws.sel_ids, ws.sel_scores, wm1);
  else
    e = launch_pdl(decode_topk_kernel, g2, 256, 0, st, ws.scores, seqlens, d->seqlen, nc, d->heads_q, K, ws.sel_ids,
                   ws.sel_scores, wm1);
  if (e != cudaSuccess) return HILS_ERR_CUDA;
  const size_t smem3 = DecUnion<T, D>::smem(G, K);
  constexpr auto k3 = decode_partial_union_kernel<T, D>;
  if (smem3 > 48 * 1024 && set_smem_max<k3>() != cudaSuccess) return HILS_ERR_CUDA;
  const dim3 g3(unsigned(G * K + wm1 + 1), unsigned(d->batch * d->heads_kv));
  e = launch_pdl(k3, g3, 128, smem3, st, static_cast<const T*>(q), static_cast<const T*>(kc),
                 static_cast<const T*>(vc), seqlens, d->seqlen, d->heads_q, G, d->heads_kv, K, tau,
                 static_cast<const int32_t*>(ws.sel_ids), static_cast<const float*>(ws.sel_scores), ws.part_u,
                 ws.part_o, pk, wm1);
  if (e != cudaSuccess) return HILS_ERR_CUDA;
  e = launch_pdl(decode_combine_kernel<T, D>, dim3(unsigned(rows)), D, 0, st,
                 static_cast<const float*>(ws.part_u), static_cast<const float*>(ws.part_o), seqlens, d->seqlen,
                 d->heads_q, K, static_cast<const int32_t*>(ws.sel_ids), static_cast<const float*>(ws.sel_scores),
                 static_cast<T*>(o), ids_out, scores_out, rows, wm1);
  if (e != cudaSuccess) return HILS_ERR_CUDA;
  return launched(4);
}

}  // namespace

extern "C" {

static int summary_entry(const hils_dims* d, const void* k, const void* lq, int64_t chunk_begin,
                         int64_t chunk_end, float* kprime, float* bprime, void* kprime_mma, hils_stream_t stream,
                         PagedKv pk) {
  int rc = check_dims(d);
  if (rc) return rc;
  const int64_t nc = d->seqlen / kChunk;
  if (!ptr_ok(k) || !ptr_ok(lq) || !ptr_ok(kprime) || !ptr_ok(bprime)) return HILS_ERR_INVALID_ARGUMENT;
  if (kprime_mma != nullptr && (d->dtype != HILS_BF16 || !aligned16(kprime_mma))) return HILS_ERR_INVALID_ARGUMENT;
  if (chunk_begin < 0 || chunk_end < chunk_begin || chunk_end > nc) return HILS_ERR_INVALID_ARGUMENT;
  if (chunk_end == chunk_begin) return HILS_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == HILS_BF16) {
    if (d->head_dim == 64) return launch_summary<__nv_bfloat16, 64>(d, k, lq, chunk_begin, chunk_end, kprime, bprime, kprime_mma, st, pk);
    return launch_summary<__nv_bfloat16, 128>(d, k, lq, chunk_begin, chunk_end, kprime, bprime, kprime_mma, st, pk);
  }
  if (d->head_dim == 64) return launch_summary<float, 64>(d, k, lq, chunk_begin, chunk_end, kprime, bprime, nullptr, st, pk);
  return launch_summary<float, 128>(d, k, lq, chunk_begin, chunk_end, kprime, bprime, nullptr, st, pk);
}

int hils_landmark_summary(const hils_dims* d, const void* k, const void* lq, int64_t chunk_begin,
                          int64_t chunk_end, float* kprime, float* bprime, void* kprime_mma,
                          hils_stream_t stream) {
  return summary_entry(d, k, lq, chunk_begin, chunk_end, kprime, bprime, kprime_mma, stream, PagedKv{nullptr, 0});
}

int hils_landmark_summary_paged(const hils_dims* d, const void* k_pages, const int32_t* page_table, int64_t n_pages,
                                const void* lq, int64_t chunk_begin, int64_t chunk_end, float* kprime,
                                float* bprime, void* kprime_mma, hils_stream_t stream) {
  if (page_table == nullptr || n_pages < 1) return HILS_ERR_INVALID_ARGUMENT;
  return summary_entry(d, k_pages, lq, chunk_begin, chunk_end, kprime, bprime, kprime_mma, stream,
                       PagedKv{page_table, n_pages});
}

size_t hils_kprime_mma_bytes(const hils_dims* d) {
  if (check_dims(d) != HILS_OK) return 0;
  return size_t(d->batch) * d->heads_kv * size_t(d->seqlen / kChunk) * size_t(d->head_dim + kExt) * 2;
}

int hils_select(const hils_dims* d, const void* q, const float* kprime, const float* bprime, const void* kprime_mma,
                const int64_t* row_pos, int64_t n_rows, int32_t* ids, float* scores, hils_stream_t stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if (!ptr_ok(q) || !ptr_ok(ids) || (scores != nullptr && !aligned16(scores))) return HILS_ERR_INVALID_ARGUMENT;
  // every position (row_pos NULL: n_rows 0 or seqlen) or a listed subset
  if (row_pos == nullptr ? (n_rows != 0 && n_rows != d->seqlen) : (n_rows < 0 || !aligned16(row_pos)))
    return HILS_ERR_INVALID_ARGUMENT;
  if (row_pos == nullptr) n_rows = d->seqlen;
  if (n_rows == 0) return HILS_OK;
  if (int64_t(d->batch) * d->heads_q > 65535) return HILS_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == HILS_BF16) {
    if (!ptr_ok(kprime_mma)) return HILS_ERR_INVALID_ARGUMENT;
    if (row_pos == nullptr && select_tc_supported(d)) {
      const int K = d->topk;
      if (d->head_dim == 64) {
        if (K <= 16) return launch_select_tc<64, 16>(d, q, kprime_mma, ids, scores, st);
        if (K <= 32) return launch_select_tc<64, 32>(d, q, kprime_mma, ids, scores, st);
        return launch_select_tc<64, 0>(d, q, kprime_mma, ids, scores, st);
      }
      if (K <= 16) return launch_select_tc<128, 16>(d, q, kprime_mma, ids, scores, st);
      if (K <= 32) return launch_select_tc<128, 32>(d, q, kprime_mma, ids, scores, st);
      return launch_select_tc<128, 0>(d, q, kprime_mma, ids, scores, st);
    }
    if (d->head_dim == 64)
      return launch_select_simt<__nv_bfloat16, 64, true>(d, q, nullptr, nullptr, kprime_mma, row_pos, n_rows, ids,
                                                         scores, st);
    return launch_select_simt<__nv_bfloat16, 128, true>(d, q, nullptr, nullptr, kprime_mma, row_pos, n_rows, ids,
                                                        scores, st);
  }
  if (!ptr_ok(kprime) || !ptr_ok(bprime)) return HILS_ERR_INVALID_ARGUMENT;
  if (d->head_dim == 64)
    return launch_select_simt<float, 64, false>(d, q, kprime, bprime, nullptr, row_pos, n_rows, ids, scores, st);
  return launch_select_simt<float, 128, false>(d, q, kprime, bprime, nullptr, row_pos, n_rows, ids, scores, st);
}

size_t hils_prefill_workspace_bytes(const hils_dims* d) {
  if (check_dims(d) != HILS_OK) return 0;
  if (!cc_supported(d)) return 0;
  return cc_plan(d).total;
}

int hils_attn_prefill(const hils_dims* d, const void* q, const void* k, const void* v, const float* kprime,
                      const float* bprime, const void* kprime_mma, const int32_t* ids, const float* scores, void* o,
                      float* lse_own, void* workspace, size_t workspace_bytes, hils_stream_t stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(ids) || !ptr_ok(o)) return HILS_ERR_INVALID_ARGUMENT;
  if (scores != nullptr && !aligned16(scores)) return HILS_ERR_INVALID_ARGUMENT;
  if (lse_own != nullptr && !aligned16(lse_own)) return HILS_ERR_INVALID_ARGUMENT;
  // without scores the chunk scores are recomputed: bf16 from the scoring
  // operand, fp32 from k' and b'
  if (scores == nullptr && (d->dtype == HILS_BF16 ? !ptr_ok(kprime_mma) : (!ptr_ok(kprime) || !ptr_ok(bprime))))
    return HILS_ERR_INVALID_ARGUMENT;
  const size_t need = hils_prefill_workspace_bytes(d);
  if (workspace_bytes < need) return HILS_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && !ptr_ok(workspace)) return HILS_ERR_INVALID_ARGUMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const void* kmma = scores == nullptr ? kprime_mma : nullptr;
  const float* kp = scores == nullptr ? kprime : nullptr;
  const float* bp = scores == nullptr ? bprime : nullptr;
  if (d->dtype == HILS_BF16 && need > 0) {
    if (d->head_dim == 64) return launch_prefill_cc<64>(d, q, k, v, kmma, ids, scores, o, lse_own, workspace, st);
    return launch_prefill_cc<128>(d, q, k, v, kmma, ids, scores, o, lse_own, workspace, st);
  }
  if (d->dtype == HILS_BF16) {
    if (d->head_dim == 64)
      return launch_prefill_simt<__nv_bfloat16, 64>(d, q, k, v, nullptr, nullptr, kmma, ids, scores, o, lse_own, st);
    return launch_prefill_simt<__nv_bfloat16, 128>(d, q, k, v, nullptr, nullptr, kmma, ids, scores, o, lse_own, st);
  }
  if (d->head_dim == 64) return launch_prefill_simt<float, 64>(d, q, k, v, kp, bp, nullptr, ids, scores, o, lse_own, st);
  return launch_prefill_simt<float, 128>(d, q, k, v, kp, bp, nullptr, ids, scores, o, lse_own, st);
}

size_t hils_decode_workspace_bytes(const hils_dims* d) {
  if (check_dims(d) != HILS_OK) return 0;
  return decode_ws_layout(int64_t(d->batch) * d->heads_q, d->seqlen / kChunk, d->topk, window_wm1(d) + 1,
                          d->head_dim, nullptr, nullptr);
}

static int decode_entry(const hils_dims* d, const void* q, const void* k_cache, const void* v_cache,
                        const float* kprime, const float* bprime, const void* kprime_mma, const int32_t* seqlens,
                        void* o, int32_t* ids_out, float* scores_out, void* workspace, size_t workspace_bytes,
                        hils_stream_t stream, PagedKv pk, const void* q_score = nullptr) {
  int rc = check_dims(d);
  if (rc) return rc;
  if (d->heads_q / d->heads_kv > 32) return HILS_ERR_UNSUPPORTED;   // one lane per query head of a kv head
  if (!ptr_ok(q) || !ptr_ok(k_cache) || !ptr_ok(v_cache) || !ptr_ok(seqlens) || !ptr_ok(o) || !ptr_ok(workspace))
    return HILS_ERR_INVALID_ARGUMENT;
  if (q_score != nullptr && !aligned16(q_score)) return HILS_ERR_INVALID_ARGUMENT;
  if ((ids_out != nullptr && !aligned16(ids_out)) || (scores_out != nullptr && !aligned16(scores_out)))
    return HILS_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < hils_decode_workspace_bytes(d)) return HILS_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == HILS_BF16) {
    if (!ptr_ok(kprime_mma)) return HILS_ERR_INVALID_ARGUMENT;
    if (d->head_dim == 64)
      return launch_decode<__nv_bfloat16, 64>(d, q, k_cache, v_cache, nullptr, nullptr, kprime_mma, seqlens, o, ids_out, scores_out, workspace, st, pk, q_score);
    return launch_decode<__nv_bfloat16, 128>(d, q, k_cache, v_cache, nullptr, nullptr, kprime_mma, seqlens, o, ids_out, scores_out, workspace, st, pk, q_score);
  }
  if (!ptr_ok(kprime) || !ptr_ok(bprime)) return HILS_ERR_INVALID_ARGUMENT;
  if (d->head_dim == 64)
    return launch_decode<float, 64>(d, q, k_cache, v_cache, kprime, bprime, nullptr, seqlens, o, ids_out, scores_out, workspace, st, pk, q_score);
  return launch_decode<float, 128>(d, q, k_cache, v_cache, kprime, bprime, nullptr, seqlens, o, ids_out, scores_out, workspace, st, pk, q_score);
}

int hils_attn_decode(const hils_dims* d, const void* q, const void* k_cache, const void* v_cache,
                     const float* kprime, const float* bprime, const void* kprime_mma, const int32_t* seqlens,
                     void* o, int32_t* ids_out, float* scores_out, void* workspace, size_t workspace_bytes,
                     hils_stream_t stream) {
  return decode_entry(d, q, k_cache, v_cache, kprime, bprime, kprime_mma, seqlens, o, ids_out, scores_out, workspace,
                      workspace_bytes, stream, PagedKv{nullptr, 0});
}

int hils_attn_decode_paged(const hils_dims* d, const void* q, const void* k_pages, const void* v_pages,
                           const int32_t* page_table, int64_t n_pages, const float* kprime, const float* bprime,
                           const void* kprime_mma, const int32_t* seqlens, void* o, int32_t* ids_out,
                           float* scores_out, void* workspace, size_t workspace_bytes, hils_stream_t stream) {
  if (page_table == nullptr || n_pages < 1) return HILS_ERR_INVALID_ARGUMENT;
  return decode_entry(d, q, k_pages, v_pages, kprime, bprime, kprime_mma, seqlens, o, ids_out, scores_out, workspace,
                      workspace_bytes, stream, PagedKv{page_table, n_pages});
}

int hils_attn_decode_qcal(const hils_dims* d, const void* q, const void* q_score, const void* k_cache,
                          const void* v_cache, const int32_t* page_table, int64_t n_pages, const float* kprime,
                          const float* bprime, const void* kprime_mma, const int32_t* seqlens, void* o,
                          int32_t* ids_out, float* scores_out, void* workspace, size_t workspace_bytes,
                          hils_stream_t stream) {
  if (q_score == nullptr) return HILS_ERR_INVALID_ARGUMENT;
  if (page_table != nullptr && n_pages < 1) return HILS_ERR_INVALID_ARGUMENT;
  return decode_entry(d, q, k_cache, v_cache, kprime, bprime, kprime_mma, seqlens, o, ids_out, scores_out, workspace,
                      workspace_bytes, stream, PagedKv{page_table, page_table ? n_pages : 0}, q_score);
}

int hils_query_calibrate(const hils_dims* d, const void* q, int64_t n_pos, const void* w_down, const void* w_up,
                         int32_t rank, void* q_hat, hils_stream_t stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if (n_pos < 1 || rank < 8 || rank > kQcalMaxRank || rank % 8 != 0) return HILS_ERR_INVALID_ARGUMENT;
  if (!ptr_ok(q) || !ptr_ok(w_down) || !ptr_ok(w_up) || !ptr_ok(q_hat)) return HILS_ERR_INVALID_ARGUMENT;
  const int64_t rows = int64_t(d->batch) * d->heads_q * n_pos;
  const size_t es = d->dtype == HILS_BF16 ? 2 : 4;
  // q_hat may be q itself (in place) but must not overlap it otherwise
  const uintptr_t a = reinterpret_cast<uintptr_t>(q), b = reinterpret_cast<uintptr_t>(q_hat);
  const uintptr_t span = uintptr_t(rows) * d->head_dim * es;
  if (a != b && a < b + span && b < a + span) return HILS_ERR_INVALID_ARGUMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t bhq = int64_t(d->batch) * d->heads_q;
  if (d->dtype == HILS_BF16 && n_pos >= 64 && bhq <= 65535 && n_pos <= (int64_t(1) << 31) - 128) {
    CUtensorMap tq, to;
    if (!make_map_3d(&tq, q, d->head_dim, n_pos, bhq, 128) || !make_map_3d(&to, q_hat, d->head_dim, n_pos, bhq, 128))
      return HILS_ERR_CUDA;
    const dim3 grid(unsigned((n_pos + 127) / 128), unsigned(bhq));
    const auto* wd = static_cast<const __nv_bfloat16*>(w_down);
    const auto* wu = static_cast<const __nv_bfloat16*>(w_up);
    if (d->head_dim == 64) {
      constexpr auto fn = qcal_tc_kernel<64>;
      if (set_smem_max<fn>() != cudaSuccess) return HILS_ERR_CUDA;
      fn<<<grid, 128, QcalTc<64>::SMEM, st>>>(tq, to, wd, wu, rank, d->heads_q);
    } else {
      constexpr auto fn = qcal_tc_kernel<128>;
      if (set_smem_max<fn>() != cudaSuccess) return HILS_ERR_CUDA;
      fn<<<grid, 128, QcalTc<128>::SMEM, st>>>(tq, to, wd, wu, rank, d->heads_q);
    }
    return launched(1);
  }
  const unsigned blocks = unsigned((rows * 32 + 127) / 128);
  if (d->dtype == HILS_BF16) {
    const auto* qq = static_cast<const __nv_bfloat16*>(q);
    const auto* wd = static_cast<const __nv_bfloat16*>(w_down);
    const auto* wu = static_cast<const __nv_bfloat16*>(w_up);
    auto* out = static_cast<__nv_bfloat16*>(q_hat);
    if (d->head_dim == 64) qcal_simt_kernel<__nv_bfloat16, 64><<<blocks, 128, 0, st>>>(qq, wd, wu, rank, n_pos, d->heads_q, rows, out);
    else qcal_simt_kernel<__nv_bfloat16, 128><<<blocks, 128, 0, st>>>(qq, wd, wu, rank, n_pos, d->heads_q, rows, out);
  } else {
    const auto* qq = static_cast<const float*>(q);
    const auto* wd = static_cast<const float*>(w_down);
    const auto* wu = static_cast<const float*>(w_up);
    auto* out = static_cast<float*>(q_hat);
    if (d->head_dim == 64) qcal_simt_kernel<float, 64><<<blocks, 128, 0, st>>>(qq, wd, wu, rank, n_pos, d->heads_q, rows, out);
    else qcal_simt_kernel<float, 128><<<blocks, 128, 0, st>>>(qq, wd, wu, rank, n_pos, d->heads_q, rows, out);
  }
  return launched(1);
}

size_t hils_attn_backward_workspace_bytes(const hils_dims* d) {
  if (check_dims(d) != HILS_OK) return 0;
  return bwd_plan(d).total;
}

int hils_attn_backward(const hils_dims* d, const void* q, const void* q_score, const void* k, const void* v,
                       const void* lq, const float* kprime, const int32_t* ids, const float* scores,
                       const float* lse_own, const void* o, const void* d_o, float* dq, float* dq_score, float* dk,
                       float* dv, float* dlq, void* workspace, size_t workspace_bytes, hils_stream_t stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(lq) || !ptr_ok(kprime) || !ptr_ok(ids) || !ptr_ok(scores) ||
      !ptr_ok(lse_own) || !ptr_ok(o) || !ptr_ok(d_o) || !ptr_ok(dq) || !ptr_ok(dk) || !ptr_ok(dv) || !ptr_ok(dlq) ||
      !ptr_ok(workspace))
    return HILS_ERR_INVALID_ARGUMENT;
  if ((q_score != nullptr && !aligned16(q_score)) || (dq_score != nullptr && !aligned16(dq_score)))
    return HILS_ERR_INVALID_ARGUMENT;
  const int64_t rows = int64_t(d->batch) * d->heads_q * d->seqlen;
  if (rows * d->topk >= (int64_t(1) << 31) || int64_t(d->batch) * d->heads_kv * d->seqlen >= (int64_t(1) << 31))
    return HILS_ERR_UNSUPPORTED;
  if (int64_t(d->batch) * d->heads_q > 65535) return HILS_ERR_UNSUPPORTED;
  if (workspace_bytes < hils_attn_backward_workspace_bytes(d)) return HILS_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == HILS_BF16) {
    if (d->head_dim == 64)
      return launch_backward<__nv_bfloat16, 64>(d, q, q_score, k, v, lq, kprime, ids, scores, lse_own, o, d_o, dq,
                                                dq_score, dk, dv, dlq, workspace, st);
    return launch_backward<__nv_bfloat16, 128>(d, q, q_score, k, v, lq, kprime, ids, scores, lse_own, o, d_o, dq,
                                               dq_score, dk, dv, dlq, workspace, st);
  }
  if (d->head_dim == 64)
    return launch_backward<float, 64>(d, q, q_score, k, v, lq, kprime, ids, scores, lse_own, o, d_o, dq, dq_score, dk,
                                      dv, dlq, workspace, st);
  return launch_backward<float, 128>(d, q, q_score, k, v, lq, kprime, ids, scores, lse_own, o, d_o, dq, dq_score, dk,
                                     dv, dlq, workspace, st);
}

}  // extern "C"

namespace {

// Scratch of hils_attn_decode_fixed_scratch: one array per device, shared by
// every call, kept until the process exits.
__device__ __align__(256) unsigned char g_decode_scratch[HILS_DECODE_FIXED_SCRATCH_BYTES];

// Device address of g_decode_scratch on the current device.  Host code cannot
// use the symbol itself as a device pointer, so it is looked up on every call
// (a host-side table lookup once the module is loaded): a cached address would
// go stale if the caller reset the device and the module came back elsewhere.
void* decode_scratch_address() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace

extern "C" {

int hils_attn_decode_fixed_scratch(const hils_dims* d, const void* q, const void* k_cache, const void* v_cache,
                                   const float* kprime, const float* bprime, const void* kprime_mma,
                                   const int32_t* seqlens, void* o, int32_t* ids_out, float* scores_out,
                                   hils_stream_t stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if (d->heads_q / d->heads_kv > 32) return HILS_ERR_UNSUPPORTED;
  const size_t need = hils_decode_workspace_bytes(d);
  if (need > size_t(HILS_DECODE_FIXED_SCRATCH_BYTES)) return HILS_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = decode_scratch_address();
  if (scratch == nullptr) return HILS_ERR_CUDA;
  return hils_attn_decode(d, q, k_cache, v_cache, kprime, bprime, kprime_mma, seqlens, o, ids_out, scores_out,
                          scratch, size_t(HILS_DECODE_FIXED_SCRATCH_BYTES), stream);
}

int hils_get_status(int32_t* host_status, hils_stream_t stream) {
  if (host_status == nullptr) return HILS_ERR_INVALID_ARGUMENT;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HILS_ERR_CUDA;
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return HILS_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return HILS_ERR_CUDA;
  *host_status = v;
  return HILS_OK;
}

int hils_selftest_bounded_wait(int32_t limit_ms, hils_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000) return HILS_ERR_INVALID_ARGUMENT;
  sm100::bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      uint64_t(limit_ms) * 1000000ull);
  return launched(1);
}

const char* hils_strerror(int s) {
  switch (s) {
    case HILS_OK: return "ok";
    case HILS_ERR_INVALID_ARGUMENT: return "invalid argument (null or misaligned pointer, or bad size)";
    case HILS_ERR_UNSUPPORTED: return "unsupported sizes (chunk must be 64, head_dim 64 or 128, topk 1..64)";
    case HILS_ERR_CUDA: return "CUDA error";
    case HILS_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case HILS_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case HILS_ERR_DEVICE_BOUNDS: return "a device-side index (chunk id or seqlen) was out of range and skipped";
    default: return "unknown status";
  }
}

uint64_t hils_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
