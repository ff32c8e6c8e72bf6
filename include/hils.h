/*
 * hils.h -- C ABI of the B200 (sm_100a) HiLS attention forward library.
 *
 * HiLS = Hierarchical Landmark Sparse attention ("Hierarchical Sparse
 * Attention Done Right: Toward Infinite Context Modeling").  Citations below
 * name the page and its section:
 *   [HP-Abs]    hotpaper.ai page on the paper, abstract
 *   [AIT-Meth]  aitrends.kr article, section "방법론" (Methodology)
 *   [AIT-Tech]  aitrends.kr article, section "기술 상세" (Technical details)
 *   [AIT-Gloss] aitrends.kr article, glossary "계층적 소프트맥스"
 *   [AIP-Perf]  ai-papers.net article, section "実験結果と性能"
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers, 16-byte aligned, row-major with
 *   head_dim innermost.  The caller allocates and frees every buffer; the
 *   library never allocates, frees or synchronises (hils_get_status is the
 *   one call that synchronises its stream).
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and returns an int status:
 *     HILS_OK (0)                    launched (or nothing to do)
 *     HILS_ERR_INVALID_ARGUMENT (1)  null / misaligned pointer, bad size;
 *                                    nothing was launched
 *     HILS_ERR_UNSUPPORTED (2)       sizes outside the compiled set
 *                                    (chunk != 64, head_dim not 64/128,
 *                                    topk outside 1..64, fp32 on a
 *                                    bf16-only call); nothing was launched
 *     HILS_ERR_CUDA (3)              a CUDA launch error
 *     HILS_ERR_WORKSPACE_TOO_SMALL (4)
 *   Device-side faults are never raised by trapping.  A kernel that meets a
 *   bad value (a chunk id or seqlen out of range) or a bounded wait that ran
 *   out records a code in a device status word and skips the access:
 *     HILS_ERR_DEVICE_TIMEOUT (5), HILS_ERR_DEVICE_BOUNDS (6)
 *   Read (and clear) that word with hils_get_status.
 * - No C++ exception crosses this boundary.  Calls are re-entrant across
 *   streams (they keep no host state besides a launch counter).
 * - Row = (b, hq, i).  Its kv head is h = hq / G with G = heads_q/heads_kv
 *   (contiguous query-head groups share a kv head).  Its own chunk is
 *   o = floor(i/chunk); its local window is o and the W-1 chunks before it
 *   (W = max(1, dims.window/chunk)), keys max(0, (o-W+1) chunk) .. i; its
 *   candidate chunks are the ones before the window, c < o - W + 1.
 *   tau = 1/sqrt(head_dim).
 */
#ifndef HILS_H_
#define HILS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hils_stream_t; /* identical to cudaStream_t */

enum hils_dtype { HILS_BF16 = 0, HILS_FP32 = 1 };

enum hils_status {
  HILS_OK = 0,
  HILS_ERR_INVALID_ARGUMENT = 1,
  HILS_ERR_UNSUPPORTED = 2,
  HILS_ERR_CUDA = 3,
  HILS_ERR_WORKSPACE_TOO_SMALL = 4,
  HILS_ERR_DEVICE_TIMEOUT = 5,
  HILS_ERR_DEVICE_BOUNDS = 6
};

typedef struct hils_dims {
  int32_t batch;     /* B */
  int32_t heads_q;   /* Hq */
  int32_t heads_kv;  /* Hkv; heads_q % heads_kv == 0 */
  int32_t head_dim;  /* d in {64, 128} */
  int32_t chunk;     /* C; must be 64 ([AIT-Tech]: chunk size 64) */
  int32_t topk;      /* K in 1..64 */
  int64_t seqlen;    /* prefill: N tokens; decode: KV-cache capacity in tokens.
                        Must be a positive multiple of chunk. */
  int32_t dtype;     /* HILS_BF16 (bf16 storage, fp32 accumulation) or HILS_FP32 */
  int32_t window;    /* local window in tokens ([AIT-Tech]: a sliding window of
                        512): 0 or chunk = the own chunk alone; else a multiple
                        of chunk, at most 16 chunks.  Read chunk-aligned: the
                        own chunk o and the window/C - 1 chunks before it, keys
                        max(0, (o - window/C + 1) C) .. i, one fusion branch
                        scored by its exact log-sum-exp; the top-K candidates
                        are the chunks before the window. */
} hils_dims;

/*
 * Landmark summary of chunks [chunk_begin, chunk_end) -- [AIT-Meth], [AIT-Tech]:
 * for each (b, h, c) the landmark query lq_c attends over the chunk's C keys,
 *     z_j = tau * <lq_c, k_j>,  p = softmax(z),
 *     k'_c = sum_j p_j k_j          (compressed key)
 *     b'_c = -sum_j p_j log p_j     (entropy bias, natural log)
 * so that tau*<q, k'_c> + b'_c is the first-order Taylor surrogate of the
 * chunk's log-sum-exp log sum_j exp(tau*<q,k_j>).
 *   k           [B, Hkv, seqlen, d]   dtype
 *   lq          [B, Hkv, seqlen/C, d] dtype (one landmark query per chunk)
 *   kprime      [B, Hkv, seqlen/C, d] fp32, written for the chunk range
 *   bprime      [B, Hkv, seqlen/C]    fp32, written for the chunk range
 *   kprime_mma  bf16 only (NULL for fp32; optional for bf16): the scoring
 *               operand, hils_kprime_mma_bytes() bytes, written for the
 *               range.  Layout [B, Hkv, seqlen/C, d+16] bf16: k'_c rounded to
 *               bf16, then x_hi, x_lo with x_hi + x_lo ~ b'_c / tau, then 14
 *               zeros.  hils_select and hils_attn_decode read it for bf16.
 * 0 <= chunk_begin <= chunk_end <= seqlen/C.  Decode appends one chunk at a
 * time by passing [c, c+1) once chunk c is full.
 */
int hils_landmark_summary(const hils_dims* dims, const void* k, const void* lq,
                          int64_t chunk_begin, int64_t chunk_end,
                          float* kprime, float* bprime, void* kprime_mma,
                          hils_stream_t stream);

/* Bytes of the bf16 scoring operand written by hils_landmark_summary. */
size_t hils_kprime_mma_bytes(const hils_dims* dims);

/*
 * Chunk scoring and top-K selection for the query rows of a prefill --
 * [AIT-Meth]: s^_{i,c} = tau*<q_i, k'_c> + b'_c over the candidates
 * c < floor(i/C) - W + 1 (W = window chunks); keep the K largest.  Ties go to
 * the lower chunk id.
 *   q          [B, Hq, seqlen, d] dtype (every position, also when a subset
 *              of rows is selected)
 *   kprime     fp32 [B,Hkv,nc,d]  (fp32 path; may be NULL for bf16)
 *   bprime     fp32 [B,Hkv,nc]    (fp32 path; may be NULL for bf16)
 *   kprime_mma bf16 scoring operand (required for bf16, ignored for fp32);
 *              the bf16 path scores with bf16 k' and fp32 accumulation.
 *   row_pos    NULL: every position 0 .. seqlen-1 (n_rows 0 or seqlen), on
 *              tensor cores where the shape allows.  Otherwise a device
 *              int64 array of n_rows query positions (any order, repeats
 *              allowed, 16-byte aligned), selected on CUDA cores: row r of
 *              every (b, hq) is position row_pos[r].  A position outside
 *              [0, seqlen) is recorded as HILS_ERR_DEVICE_BOUNDS and its ids
 *              are all -1.  This serves checks on a sample of rows and
 *              queries that need only some positions' selection.
 *   n_rows     number of listed positions (>= 0; 0 with a list: no work)
 *   ids        [B, Hq, n_rows, K] int32 out: the kept chunk ids in
 *              ascending order; rows with fewer than K candidates are padded
 *              with -1.
 *   scores     [B, Hq, n_rows, K] fp32 out (nullable): s^ of each id, -inf
 *              for padding.  hils_attn_prefill can take it or recompute it.
 */
int hils_select(const hils_dims* dims, const void* q, const float* kprime, const float* bprime,
                const void* kprime_mma, const int64_t* row_pos, int64_t n_rows, int32_t* ids, float* scores,
                hils_stream_t stream);

/*
 * Device workspace bytes hils_attn_prefill needs for these dims (0 when the
 * call needs none: the fp32 path).  For bf16 it holds an fp32 output
 * accumulator (rows x d), the fusion normaliser of every row, the inverted
 * index of (row, slot) pairs per (kv head, window, chunk), the pair count's
 * per-(4096 rows, chunk) bases and room for the recomputed chunk scores of a
 * call without scores: about rows x (4d + 4 + 16K + nc/1024) bytes, nc =
 * seqlen / 64.
 */
size_t hils_prefill_workspace_bytes(const hils_dims* dims);

/*
 * Prefill sparse attention with hierarchical fusion -- [HP-Abs], [AIT-Meth],
 * [AIT-Gloss]: for each row and each kept chunk c, an intra-chunk softmax
 * over the chunk's C keys gives o_c and its log-sum-exp; the row's local
 * window (keys max(0, (floor(i/C)-W+1) C) .. i, causal) is one branch that
 * enters the fusion with its exact log-sum-exp lse_own as score; the fusion
 * weights are a softmax over {s^_c : c kept} U {lse_own}:
 *     O_i = sum_c w_c o_c + w_own o_own.
 *   q, k, v   [B,Hq,N,d] / [B,Hkv,N,d] / [B,Hkv,N,d] dtype
 *   kprime, bprime, kprime_mma
 *             the summaries of hils_landmark_summary; read only when scores
 *             is NULL (bf16: kprime_mma required, the others may be NULL;
 *             fp32: kprime and bprime required)
 *   ids       [B,Hq,N,K] int32 from hils_select (-1 entries are skipped; an id
 *             outside the candidates [0, floor(i/C)-W+1) is recorded as
 *             HILS_ERR_DEVICE_BOUNDS and skipped)
 *   scores    [B,Hq,N,K] fp32 from hils_select, or NULL: then s^ of every
 *             kept id is recomputed from q and the summaries as hils_select
 *             computes it ([AIT-Meth]; bf16: tau (<q, k'_bf16> + x_hi + x_lo)
 *             with fp32 sums in another order, so within rounding of the
 *             selection's values), and the caller needs no [B,Hq,N,K] scores
 *             buffer.  Pass the scores when the selection scored another
 *             query than q (Q-Cal's q^).
 *   o         [B,Hq,N,d] dtype out
 *   lse_own   [B,Hq,N] fp32 out (nullable): log-sum-exp of the local window
 *   workspace device scratch of at least hils_prefill_workspace_bytes(dims)
 *             (may be NULL when that is 0); HILS_ERR_WORKSPACE_TOO_SMALL
 *             otherwise
 * bf16 outputs: the chunk outputs are summed in fp32 by reductions whose
 * order is not fixed, so two runs on the same inputs may differ by one bf16
 * ulp in an output element (the fp32 sums differ only in their last bits,
 * and rounding to bf16 can then land on the neighbouring value), or by about
 * 1e-6 for an output that is almost zero (its sum cancels); ids and lse_own
 * are reproducible.
 */
int hils_attn_prefill(const hils_dims* dims, const void* q, const void* k, const void* v, const float* kprime,
                      const float* bprime, const void* kprime_mma, const int32_t* ids, const float* scores, void* o,
                      float* lse_own, void* workspace, size_t workspace_bytes, hils_stream_t stream);

/* Device workspace bytes hils_attn_decode needs for these dims. */
size_t hils_decode_workspace_bytes(const hils_dims* dims);

/*
 * One decode step -- [AIT-Meth] scoring and selection plus the fused sparse
 * attention of hils_attn_prefill, for one new query per (b, hq) at position
 * t_b = seqlens[b] - 1 whose key/value are already in the cache ([AIP-Perf]:
 * per-token decode with sparse KV access).  The candidate chunks
 * 0 .. floor(t_b/C)-W must have summaries.
 *   dims.seqlen  KV-cache capacity in tokens
 *   q            [B, Hq, d] dtype
 *   k_cache, v_cache [B, Hkv, seqlen, d] dtype
 *   kprime, bprime   fp32 summaries (fp32 path)
 *   kprime_mma   bf16 scoring operand (bf16 path)
 *   seqlens      device int32 [B], 1 <= seqlens[b] <= seqlen (violations are
 *                recorded as HILS_ERR_DEVICE_BOUNDS and the row is zeroed)
 *   o            [B, Hq, d] dtype out
 *   ids_out      [B, Hq, K] int32 out (nullable)
 *   scores_out   [B, Hq, K] fp32 out (nullable)
 *   workspace    device scratch of at least hils_decode_workspace_bytes(dims)
 * heads_q / heads_kv must be at most 32 (HILS_ERR_UNSUPPORTED otherwise).
 * The step is four kernels on `stream`, ordered like any stream work.  The
 * first is launched normally; the other three with programmatic stream
 * serialisation, so each may be scheduled while the one before it finishes
 * and waits for it on the device.  Only the library's own kernels overlap this
 * way; work the caller enqueues before or after the call is not affected.
 */
int hils_attn_decode(const hils_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                     const float* kprime, const float* bprime, const void* kprime_mma,
                     const int32_t* seqlens, void* o, int32_t* ids_out, float* scores_out,
                     void* workspace, size_t workspace_bytes, hils_stream_t stream);

/*
 * Decode step that allocates nothing.  This entry point has no counterpart in
 * the paper; it exists for callers that cannot call cudaMalloc -- for example
 * a plugin inside a host inference engine that owns all device memory and
 * hands its plugins no workspace, or a latency-critical decode loop where the
 * device-wide synchronisation implied by cudaMalloc would stall other work.
 *
 * Same arguments and results as hils_attn_decode, minus the workspace: the
 * scratch lives in a file-scope device array of
 * HILS_DECODE_FIXED_SCRATCH_BYTES (16 MiB) inside the library, which every
 * GPU that loads the library keeps until the process exits.
 * - Sizes whose hils_decode_workspace_bytes() exceeds that maximum are
 *   rejected with HILS_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 * - The 16 MiB are taken on a device when the library's device code is loaded
 *   there.  Under CUDA's lazy module loading (the default) that happens at the
 *   first library call or symbol lookup on the device, so that call may
 *   allocate and synchronise inside the driver: make the first call on each
 *   device during set-up, before any stream capture.
 * - Each call looks up the array's device address (cudaGetSymbolAddress,
 *   with the call's device current), so a device reset in between is safe.
 * - Every call uses the same array and it keeps the previous call's
 *   contents.  Each byte a call reads is written earlier in that same call,
 *   so nothing has to start at zero.  Calls whose executions overlap on the
 *   GPU (other streams, other host threads) race on the array: serialise
 *   them.
 * - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define HILS_DECODE_FIXED_SCRATCH_BYTES (16u << 20)
int hils_attn_decode_fixed_scratch(const hils_dims* dims, const void* q, const void* k_cache,
                                   const void* v_cache, const float* kprime, const float* bprime,
                                   const void* kprime_mma, const int32_t* seqlens, void* o,
                                   int32_t* ids_out, float* scores_out, hils_stream_t stream);

/*
 * Chunk-paged KV cache -- [AIT-Tech] lists chunk-unit KV paging among what
 * the implementation needs (its limits section counts it as engineering cost
 * of deployment).  Here each page holds one chunk (C = 64 tokens) of all kv
 * heads of one sequence, taken from a pool; a page table maps every
 * sequence's logical chunks to pages.
 *   k_pages, v_pages  [n_pages, Hkv, C, d] dtype (16-byte aligned)
 *   page_table        device int32 [B, seqlen/C] (dims.seqlen is the
 *                     capacity in tokens): page of logical chunk c of
 *                     sequence b; only the entries of chunks the call reads
 *                     are looked at
 *   n_pages           pool size, >= 1
 * All other arguments, layouts and results are those of
 * hils_landmark_summary / hils_attn_decode: both compute exactly what the
 * contiguous calls compute on the cache the table describes (same kernels,
 * same arithmetic; only the addresses of the key and value rows differ).  A
 * table entry outside [0, n_pages) is recorded as HILS_ERR_DEVICE_BOUNDS:
 * the summary leaves that chunk's k', b' unwritten; the decode step leaves
 * that chunk out of every query's fusion.  NULL page_table or n_pages < 1:
 * HILS_ERR_INVALID_ARGUMENT.
 */
int hils_landmark_summary_paged(const hils_dims* dims, const void* k_pages, const int32_t* page_table,
                                int64_t n_pages, const void* lq, int64_t chunk_begin, int64_t chunk_end,
                                float* kprime, float* bprime, void* kprime_mma, hils_stream_t stream);
int hils_attn_decode_paged(const hils_dims* dims, const void* q, const void* k_pages, const void* v_pages,
                           const int32_t* page_table, int64_t n_pages, const float* kprime,
                           const float* bprime, const void* kprime_mma, const int32_t* seqlens, void* o,
                           int32_t* ids_out, float* scores_out, void* workspace, size_t workspace_bytes,
                           hils_stream_t stream);

/*
 * Low-rank query calibration (Q-Cal) -- [AIT-Meth] and the glossary entry
 * "저계수 쿼리 보정" of the same article: a light adapter maps each query to
 *     q^ = q + W_up (W_down q)
 * with per-query-head projections of rank r (read as residual, on the query).
 * q^ is the scoring query: pass it to hils_select (prefill) or
 * hils_attn_decode_qcal (decode) in place of q for the chunk scores; the
 * attention inside chunks keeps q (hils_attn_prefill takes q and the scores
 * that hils_select returned for q^).
 *   q       [B, Hq, n_pos, d] dtype; n_pos = dims.seqlen for a prefill, 1 for
 *           a decode step (dims.seqlen is otherwise not used here)
 *   w_down  [Hq, r, d] dtype
 *   w_up    [Hq, d, r] dtype
 *   rank    r: a multiple of 8, 8 <= r <= 64
 *   q_hat   [B, Hq, n_pos, d] dtype out; may be q itself (in place) but must
 *           not overlap it otherwise
 * bf16: products accumulate in fp32 on tensor cores, W_down q is rounded to
 * bf16 before the up projection and q^ is rounded to bf16 (RNE).  fp32:
 * fp32 arithmetic throughout.
 */
int hils_query_calibrate(const hils_dims* dims, const void* q, int64_t n_pos, const void* w_down,
                         const void* w_up, int32_t rank, void* q_hat, hils_stream_t stream);

/*
 * Decode step whose chunk scores use a separate scoring query, e.g. the
 * Q-Cal output of hils_query_calibrate: q_score [B, Hq, d] dtype scores and
 * selects the chunks and gives the fusion weights; q attends.  page_table
 * NULL: contiguous caches as in hils_attn_decode; otherwise chunk pages as in
 * hils_attn_decode_paged (n_pages >= 1).  Other arguments, workspace and
 * errors as in hils_attn_decode; q_score NULL is HILS_ERR_INVALID_ARGUMENT.
 */
int hils_attn_decode_qcal(const hils_dims* dims, const void* q, const void* q_score, const void* k_cache,
                          const void* v_cache, const int32_t* page_table, int64_t n_pages,
                          const float* kprime, const float* bprime, const void* kprime_mma,
                          const int32_t* seqlens, void* o, int32_t* ids_out, float* scores_out,
                          void* workspace, size_t workspace_bytes, hils_stream_t stream);

/* Device workspace bytes hils_attn_backward needs for these dims. */
size_t hils_attn_backward_workspace_bytes(const hils_dims* dims);

/*
 * Backward pass of the prefill (hils_landmark_summary + the chunk scores of
 * hils_select + hils_attn_prefill) for the selection the forward made --
 * [AIT-Meth]: the chunk score is part of the forward attention, so the loss
 * gradient reaches the landmark queries through k', b' and the scoring query
 * (Q-Cal) through s^; the top-K choice itself is not differentiated.
 * Given dO = dL/dO it returns the gradients of L with respect to q, k, v and
 * lq.  Per row, with M' the fusion normaliser and a_c = exp(u_c - M'):
 *   selected chunk c: dz_j = a_c p_j (<dO, v_j> - <dO, o_c>),
 *                     du_c = a_c (<dO, o_c> - <dO, O>) -> q_score, k', b'
 *   window:           dz_j = P_ij (<dO, v_j> - <dO, O>)
 *   dq += tau dz_j k_j, dk_j += tau dz_j q, dv_j += a_c p_j dO, and the
 *   landmark softmax passes dk', db' on to k and lq.
 *   q, k, v, lq  the forward's inputs (dtype, layouts as in the forward)
 *   q_score      the scoring query the selection used ([B,Hq,N,d] dtype, the
 *                output of hils_query_calibrate), or NULL when it was q
 *   kprime       fp32 [B,Hkv,nc,d] from hils_landmark_summary
 *   ids, scores  [B,Hq,N,K] from hils_select
 *   lse_own      [B,Hq,N] fp32 from hils_attn_prefill (required here)
 *   o, d_o       [B,Hq,N,d] dtype: the forward output and dL/dO
 *   dq           [B,Hq,N,d] fp32 out: through the attention, plus through
 *                the chunk scores when dq_score is NULL
 *   dq_score     [B,Hq,N,d] fp32 out (nullable): the scoring query's gradient
 *   dk, dv       [B,Hkv,N,d] fp32 out;  dlq [B,Hkv,nc,d] fp32 out
 * Outputs are overwritten.  fp32 arithmetic on CUDA cores, except for bf16:
 * there the window branch's products, and with q_score == NULL also the
 * selected chunks', run on tensor cores with bf16 operands (dZ and the
 * weights rounded to bf16) and fp32 sums.
 * Gradients are summed with fp32 atomics (the order of the sums is not
 * fixed).  Any G;
 * B * Hq <= 65535.  Ids outside a row's candidates are recorded as
 * HILS_ERR_DEVICE_BOUNDS and skipped.
 */
int hils_attn_backward(const hils_dims* dims, const void* q, const void* q_score, const void* k, const void* v,
                       const void* lq, const float* kprime, const int32_t* ids, const float* scores,
                       const float* lse_own, const void* o, const void* d_o, float* dq, float* dq_score,
                       float* dk, float* dv, float* dlq, void* workspace, size_t workspace_bytes,
                       hils_stream_t stream);

/*
 * Synchronises `stream`, copies the device status word of the current device
 * into *host_status (HILS_OK or a HILS_ERR_DEVICE_* code recorded by a kernel
 * since the last call) and clears it.  Returns HILS_ERR_CUDA if the
 * synchronisation itself failed.
 */
int hils_get_status(int32_t* host_status, hils_stream_t stream);

/*
 * Self-test of the bounded device waits that every tcgen05 kernel uses (no
 * counterpart in the paper).  Launches one CTA whose thread waits for an
 * mbarrier phase that nothing completes, with a limit of limit_ms
 * milliseconds (1..2000).  The wait gives up, records HILS_ERR_DEVICE_TIMEOUT
 * in the device status word and the kernel returns normally, so the context
 * stays usable; read the result with hils_get_status.  Nothing traps or hangs.
 */
int hils_selftest_bounded_wait(int32_t limit_ms, hils_stream_t stream);

/* Static English description of a status code. */
const char* hils_strerror(int status);

/* Number of kernels this library has launched in this process. */
uint64_t hils_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* HILS_H_ */
