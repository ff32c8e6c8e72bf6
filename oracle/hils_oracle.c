/*
 * HiLS attention forward pass -- fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the CUDA path computes.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or constant with the CUDA library, and the library never
 * calls it.
 *
 * Sources (the HiLS paper, "Hierarchical Sparse Attention Done Right: Toward
 * Infinite Context Modeling", as summarised on these pages):
 *   [HP-Abs]   hotpaper.ai page on the paper, abstract: each query attends
 *              independently to each retrieved chunk, and the chunk outputs
 *              are fused according to the chunk retrieval scores.
 *   [AIT-Meth] aitrends.kr article, section "방법론" (Methodology): the
 *              landmark query of a chunk attends over the chunk's keys; the
 *              weighted key sum is the compressed key k'_c and the entropy
 *              of that distribution is b'_c; the chunk score is
 *              s^_{i,c} = q_i . k'_c / sqrt(d) + b'_c; the top-K chunks are
 *              kept and an intra-chunk softmax gives token weights.  Worked
 *              example: d = 64, q.k'/sqrt(64) = 2.0, b' = 0.7 -> 2.7,
 *              exp(2.7) ~ 14.9.
 *   [AIT-Tech] same article, section "기술 상세" (Technical details): the
 *              first-order Taylor view log sum_j exp(s_j) ~ q.k'_c/sqrt(d)
 *              + b'_c, with b'_c the entropy of the intra-chunk attention
 *              distribution; chunk size 64.
 *   [AIT-Gloss] same article, glossary entry "계층적 소프트맥스"
 *              (hierarchical softmax): an inter-chunk softmax over the chunk
 *              scores, then an intra-chunk softmax.
 *   [AIT-QCal] same article, section "방법론" and glossary entry "저계수
 *              쿼리 보정" (low-rank query calibration): a light adapter that
 *              applies a low-rank down/up projection to the query, giving a
 *              calibrated query for the chunk-level scores.
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes of the repository):
 *   - the landmark softmax uses the same scale 1/sqrt(d) as the chunk score
 *     (the only choice that makes the Taylor surrogate exact at q = lq);
 *   - natural logarithm for the entropy;
 *   - candidates of a query at position i are the chunks c < floor(i/C)
 *     (fully past); the query's own chunk is always attended under the
 *     causal mask and enters the fusion with its exact log-sum-exp as score;
 *   - with a local window of W tokens (W a multiple of C; [AIT-Tech] gives a
 *     sliding window of 512) the window is chunk-aligned: the own chunk o
 *     and the W/C - 1 chunks before it, keys max(0, (o - W/C + 1) C) .. i.
 *     The window is one fusion branch scored by its exact log-sum-exp (it
 *     replaces the own-chunk branch), and the candidates are the chunks
 *     before it, c < o - W/C + 1.  W = 0 or W = C is the own chunk alone;
 *   - the fusion softmax runs over the selected chunks and the own chunk
 *     (the window) only;
 *   - query head hq reads kv head floor(hq / G);
 *   - top-K ties: the lower chunk id wins; fewer than K candidates: keep
 *     them all, pad the id list with -1; ids are reported in ascending order;
 *   - Q-Cal ([AIT-QCal]) is residual, per query head, and acts on the query
 *     (not on a hidden state, which this path does not see):
 *     q^ = q + W_up (W_down q), W_down [r x d], W_up [d x r].  q^ replaces q
 *     in the chunk score s^ = tau <q^, k'_c> + b'_c, so it steers both the
 *     selection and the fusion weights; the attention inside chunks keeps q.
 *
 * Everything is computed in double precision from the exact stored input
 * values (bf16 and fp32 values are exactly representable in double).
 *
 * Layouts (row-major, head_dim innermost):
 *   K, V  [B, Hkv, N, d]    (N = token capacity)
 *   LQ    [B, Hkv, N/C, d]  landmark queries
 *   kp    [B, Hkv, N/C, d]  compressed keys (double)
 *   bp    [B, Hkv, N/C]     entropy biases (double)
 * Rows are given explicitly: for row r, its batch rb[r], query head rhq[r],
 * position rpos[r] and its query vector qrows[r*d .. r*d+d).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct hils_oracle_dims {
  int64_t B, Hq, Hkv, N, d, C, K;
  int64_t W;   /* local window in tokens (0 or C: the own chunk only) */
} hils_oracle_dims;

/* chunks in the local window, own chunk included */
static int64_t window_chunks(const hils_oracle_dims* D) { return D->W > D->C ? D->W / D->C : 1; }

/* candidates of a query at position i: the chunks before its window */
static int64_t n_candidates(const hils_oracle_dims* D, int64_t i) {
  const int64_t n = i / D->C - (window_chunks(D) - 1);
  return n > 0 ? n : 0;
}

static double dot_fd(const float* a, const float* b, int64_t d) {
  double s = 0.0;
  for (int64_t t = 0; t < d; ++t) s += (double)a[t] * (double)b[t];
  return s;
}

static double dot_fdd(const float* a, const double* b, int64_t d) {
  double s = 0.0;
  for (int64_t t = 0; t < d; ++t) s += (double)a[t] * b[t];
  return s;
}

/*
 * Landmark summary of chunks [chunk_begin, chunk_end) of every (b, kv head)
 * ([AIT-Meth], [AIT-Tech]):
 *   z_j  = <lq_c, k_j> / sqrt(d)       for the C keys j of chunk c
 *   p    = softmax(z)
 *   k'_c = sum_j p_j k_j
 *   b'_c = -sum_j p_j log p_j          (natural log)
 * The entropy is evaluated as  log sum_j exp(z_j) - sum_j p_j z_j , which is
 * the same quantity (log p_j = z_j - LSE(z)) and never takes log(0).
 */
void hils_oracle_summary(const hils_oracle_dims* D, const float* K, const float* LQ,
                         int64_t chunk_begin, int64_t chunk_end, double* kp, double* bp) {
  const int64_t d = D->d, C = D->C, nc = D->N / D->C;
  const double tau = 1.0 / sqrt((double)d);
  const int64_t nbh = D->B * D->Hkv;
  const int64_t span = chunk_end - chunk_begin;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t u = 0; u < nbh * span; ++u) {
    const int64_t bh = u / span, c = chunk_begin + u % span;
    const float* lq = LQ + (bh * nc + c) * d;
    const float* kc = K + (bh * D->N + c * C) * d;
    double* z = (double*)malloc(sizeof(double) * (size_t)C);
    double m = -INFINITY;
    for (int64_t j = 0; j < C; ++j) {
      z[j] = tau * dot_fd(lq, kc + j * d, d);
      if (z[j] > m) m = z[j];
    }
    double Z = 0.0;
    for (int64_t j = 0; j < C; ++j) Z += exp(z[j] - m);
    const double lse = m + log(Z);
    double* out = kp + (bh * nc + c) * d;
    for (int64_t t = 0; t < d; ++t) out[t] = 0.0;
    double pz = 0.0;
    for (int64_t j = 0; j < C; ++j) {
      const double p = exp(z[j] - m) / Z;
      pz += p * z[j];
      for (int64_t t = 0; t < d; ++t) out[t] += p * (double)kc[j * d + t];
    }
    bp[bh * nc + c] = lse - pz;
    free(z);
  }
}

/*
 * Chunk scores of the given rows ([AIT-Meth]):
 *   s^_{i,c} = <q_i, k'_c> / sqrt(d) + b'_c     for every candidate c < floor(i/C)
 * out[r, c] = -inf for chunks that are not candidates of row r.
 */
void hils_oracle_scores(const hils_oracle_dims* D, const double* kp, const double* bp,
                        int64_t n_rows, const int32_t* rb, const int32_t* rhq, const int64_t* rpos,
                        const float* qrows, double* out) {
  const int64_t d = D->d, nc = D->N / D->C, G = D->Hq / D->Hkv;
  const double tau = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < n_rows; ++r) {
    const int64_t bh = (int64_t)rb[r] * D->Hkv + rhq[r] / G;
    const int64_t own = n_candidates(D, rpos[r]);   /* scores exist for c < own */
    const float* q = qrows + r * d;
    for (int64_t c = 0; c < nc; ++c) {
      out[r * nc + c] = (c < own) ? tau * dot_fdd(q, kp + (bh * nc + c) * d, d) + bp[bh * nc + c]
                                  : -INFINITY;
    }
  }
}

typedef struct { double s; int64_t c; } scored_chunk;

static int by_score_desc_id_asc(const void* x, const void* y) {
  const scored_chunk* a = (const scored_chunk*)x;
  const scored_chunk* b = (const scored_chunk*)y;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->c < b->c) ? -1 : (a->c > b->c);
}

static int by_id_asc(const void* x, const void* y) {
  const scored_chunk* a = (const scored_chunk*)x;
  const scored_chunk* b = (const scored_chunk*)y;
  return (a->c < b->c) ? -1 : (a->c > b->c);
}

/*
 * Top-K chunk selection ([AIT-Meth]: keep the K chunks of largest score).
 * Candidates are sorted by (score descending, chunk id ascending) and the
 * first min(K, #candidates) are kept.  ids[r, :] lists them in ascending chunk
 * id, padded with -1; sel[r, :] holds their scores (-inf for padding).
 * gap[r] = (K-th best score) - ((K+1)-th best score), +inf when a row has at
 * most K candidates.
 */
void hils_oracle_select(const hils_oracle_dims* D, const double* kp, const double* bp,
                        int64_t n_rows, const int32_t* rb, const int32_t* rhq, const int64_t* rpos,
                        const float* qrows, int32_t* ids, double* sel, double* gap) {
  const int64_t d = D->d, nc = D->N / D->C, G = D->Hq / D->Hkv, K = D->K;
  const double tau = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < n_rows; ++r) {
    const int64_t bh = (int64_t)rb[r] * D->Hkv + rhq[r] / G;
    const int64_t n_cand = n_candidates(D, rpos[r]);   /* candidates: the chunks 0 .. n_cand-1 */
    const float* q = qrows + r * d;
    scored_chunk* cand = (scored_chunk*)malloc(sizeof(scored_chunk) * (size_t)(n_cand + 1));
    for (int64_t c = 0; c < n_cand; ++c) {
      cand[c].s = tau * dot_fdd(q, kp + (bh * nc + c) * d, d) + bp[bh * nc + c];
      cand[c].c = c;
    }
    qsort(cand, (size_t)n_cand, sizeof(scored_chunk), by_score_desc_id_asc);
    const int64_t keep = n_cand < K ? n_cand : K;
    if (gap) gap[r] = (n_cand > K) ? cand[K - 1].s - cand[K].s : INFINITY;
    qsort(cand, (size_t)keep, sizeof(scored_chunk), by_id_asc);
    for (int64_t t = 0; t < K; ++t) {
      ids[r * K + t] = (t < keep) ? (int32_t)cand[t].c : -1;
      if (sel) sel[r * K + t] = (t < keep) ? cand[t].s : -INFINITY;
    }
    free(cand);
  }
}

/*
 * Softmax attention of query q over keys [j0, j1) of one (b, kv head):
 * s_j = <q, k_j>/sqrt(d); returns LSE(s) and writes o = sum_j softmax(s)_j v_j.
 */
static double attend_keys(const float* q, const float* Kbh, const float* Vbh, int64_t j0, int64_t j1,
                          int64_t d, double tau, double* s, double* o) {
  double m = -INFINITY;
  for (int64_t j = j0; j < j1; ++j) {
    s[j - j0] = tau * dot_fd(q, Kbh + j * d, d);
    if (s[j - j0] > m) m = s[j - j0];
  }
  double l = 0.0;
  for (int64_t t = 0; t < d; ++t) o[t] = 0.0;
  for (int64_t j = j0; j < j1; ++j) {
    const double e = exp(s[j - j0] - m);
    l += e;
    for (int64_t t = 0; t < d; ++t) o[t] += e * (double)Vbh[j * d + t];
  }
  for (int64_t t = 0; t < d; ++t) o[t] /= l;
  return m + log(l);
}

/*
 * Hierarchical attention of the given rows ([HP-Abs], [AIT-Meth], [AIT-Gloss]):
 *   for each selected chunk c (ids[r, :], -1 entries skipped):
 *       o_c = softmax_j(<q, k_j>/sqrt(d)) V   over the chunk's C keys
 *       u_c = s^_{i,c}                      (score_mode 0: the surrogate,
 *                                              with the scoring query qscore
 *                                              when given, else q)
 *           = log sum_j exp(<q,k_j>/sqrt(d))  (score_mode 1: the exact chunk
 *                                              log-sum-exp; used by the
 *                                              dense-equivalence pin)
 *   own chunk o = floor(i/C): keys j in [o*C, i] (causal),
 *       o_own = softmax V, u_own = exact log-sum-exp of those logits
 *   w = softmax(u over selected chunks and the own chunk)
 *   O = sum w_c o_c + w_own o_own
 * lse_own (nullable) receives u_own.
 */
void hils_oracle_attend(const hils_oracle_dims* D, const float* K, const float* V,
                        const double* kp, const double* bp,
                        int64_t n_rows, const int32_t* rb, const int32_t* rhq, const int64_t* rpos,
                        const float* qrows, const float* qscore, const int32_t* ids, int64_t ids_stride,
                        int score_mode, double* O, double* lse_own) {
  const int64_t d = D->d, C = D->C, nc = D->N / D->C, G = D->Hq / D->Hkv;
  const double tau = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 8)
  for (int64_t r = 0; r < n_rows; ++r) {
    const int64_t bh = (int64_t)rb[r] * D->Hkv + rhq[r] / G;
    const int64_t i = rpos[r], own = i / C;
    const float* q = qrows + r * d;
    const float* qs = qscore ? qscore + r * d : q;
    const float* Kbh = K + bh * D->N * d;
    const float* Vbh = V + bh * D->N * d;
    const int64_t nsel = ids_stride;
    double* u = (double*)malloc(sizeof(double) * (size_t)(nsel + 1));
    double* oc = (double*)malloc(sizeof(double) * (size_t)((nsel + 1) * d));
    double* s = (double*)malloc(sizeof(double) * (size_t)(C * window_chunks(D)));
    int64_t m_used = 0;
    for (int64_t t = 0; t < nsel; ++t) {
      const int64_t c = ids[r * ids_stride + t];
      if (c < 0) continue;
      const double lse = attend_keys(q, Kbh, Vbh, c * C, (c + 1) * C, d, tau, s, oc + m_used * d);
      u[m_used] = (score_mode == 0) ? tau * dot_fdd(qs, kp + (bh * nc + c) * d, d) + bp[bh * nc + c]
                                    : lse;
      ++m_used;
    }
    /* the own chunk, or with a window the W/C chunks ending at it (causal) */
    int64_t w0 = (own - (window_chunks(D) - 1)) * C;
    if (w0 < 0) w0 = 0;
    const double lo = attend_keys(q, Kbh, Vbh, w0, i + 1, d, tau, s, oc + m_used * d);
    u[m_used] = lo;
    if (lse_own) lse_own[r] = lo;
    ++m_used;
    double M = -INFINITY;
    for (int64_t t = 0; t < m_used; ++t) if (u[t] > M) M = u[t];
    double Z = 0.0;
    for (int64_t t = 0; t < m_used; ++t) Z += exp(u[t] - M);
    double* out = O + r * d;
    for (int64_t x = 0; x < d; ++x) out[x] = 0.0;
    for (int64_t t = 0; t < m_used; ++t) {
      const double w = exp(u[t] - M) / Z;
      for (int64_t x = 0; x < d; ++x) out[x] += w * oc[t * d + x];
    }
    free(u);
    free(oc);
    free(s);
  }
}

/*
 * Q-Cal ([AIT-QCal]): q^ = q + W_up (W_down q) for each row, with the
 * projections of the row's query head.
 *   q      [n_rows, d] float      rhq [n_rows] query head of each row
 *   w_down [Hq, r, d] float       w_up [Hq, d, r] float
 *   out    [n_rows, d] double
 */
void hils_oracle_qcal(int64_t n_rows, int64_t d, int64_t r, const int32_t* rhq, const float* q,
                      const float* w_down, const float* w_up, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_rows; ++row) {
    const float* x = q + row * d;
    const float* Wd = w_down + (int64_t)rhq[row] * r * d;
    const float* Wu = w_up + (int64_t)rhq[row] * d * r;
    double* y = out + row * d;
    double z[256];   /* W_down q, r <= 256 */
    for (int64_t a = 0; a < r; ++a) {
      double acc = 0.0;
      for (int64_t t = 0; t < d; ++t) acc += (double)Wd[a * d + t] * (double)x[t];
      z[a] = acc;
    }
    for (int64_t t = 0; t < d; ++t) {
      double acc = (double)x[t];
      for (int64_t a = 0; a < r; ++a) acc += (double)Wu[t * r + a] * z[a];
      y[t] = acc;
    }
  }
}

/*
 * One branch of a row's fusion: keys [j0, j1) of one (b, kv head), their
 * logits z_j = <q, k_j>/sqrt(d), the softmax p over them, the branch output
 * o = sum p_j v_j and its log-sum-exp.
 */
typedef struct {
  int64_t j0, j1;
  double lse;
  double u;        /* fusion score: s^ for a selected chunk, lse for the window */
  int64_t chunk;   /* selected chunk id, -1 for the window branch */
} branch_t;

/*
 * Backward of the forward pass for a fixed selection.  [AIT-Meth]: the chunk
 * score s^ is part of the forward attention, so the gradient of the loss
 * reaches the landmark queries (through k', b') and the Q-Cal adapter
 * (through the scoring query); the top-K choice itself is not differentiated.
 * Forward, per row i (query q, scoring query q^ = q unless dQs is given):
 *   branch c (a selected chunk):  z_j = tau <q, k_j>, p = softmax(z),
 *       o_c = sum p_j v_j,  u_c = tau <q^, k'_c> + b'_c
 *   window branch w: the causal window keys, u_w = log sum_j exp(z_j)
 *   a = softmax(u),  O = sum_c a_c o_c
 * With g = dL/dO_i and Dg = <g, O>, per branch X_c = <g, o_c>:
 *   du_c = a_c (X_c - Dg)
 *   dz_j = a_c p_j (<g, v_j> - X_c)        (+ du_w p_j on the window branch,
 *                                            since u_w = lse: together
 *                                            a_w p_j (<g, v_j> - Dg))
 *   dv_j += a_c p_j g,  dq += tau dz_j k_j,  dk_j += tau dz_j q
 *   selected c: dq^ += tau du_c k'_c,  dk'_c += tau du_c q^,  db'_c += du_c
 * Summary ([AIT-Meth], [AIT-Tech]), per chunk with zl_j = tau <lq, k_j>,
 * pl = softmax(zl), k' = sum pl_j k_j, b' = lse(zl) - sum pl_j zl_j:
 *   dzl_j = pl_j <dk', k_j - k'> - db' pl_j (zl_j - sum_k pl_k zl_k)
 *   dlq += tau dzl_j k_j,  dk_j += tau dzl_j lq + pl_j dk'
 * Inputs: Q [B,Hq,N,d], K, V [B,Hkv,N,d], LQ [B,Hkv,nc,d] (float, stored
 * values), Qs (nullable; the scoring query, e.g. the Q-Cal output, else Q),
 * ids [B,Hq,N,ids_stride] (-1 skipped), dO [B,Hq,N,d].  Outputs (double,
 * overwritten): dQ, dQs (nullable: then the scoring-query gradient is added
 * into dQ), dK, dV, dLQ.  Rows of different (b, kv head) touch disjoint
 * gradients, so those run in parallel.
 */
void hils_oracle_backward(const hils_oracle_dims* D, const float* Q, const float* Qs, const float* Kt,
                          const float* Vt, const float* LQ, const int32_t* ids, int64_t ids_stride,
                          const float* dO, double* dQ, double* dQs, double* dK, double* dV, double* dLQ) {
  const int64_t d = D->d, C = D->C, N = D->N, nc = N / C, G = D->Hq / D->Hkv;
  const double tau = 1.0 / sqrt((double)d);
  const int64_t nbh = D->B * D->Hkv;
  double* kp = (double*)malloc(sizeof(double) * (size_t)(nbh * nc * d));
  double* bp = (double*)malloc(sizeof(double) * (size_t)(nbh * nc));
  double* dkp = (double*)calloc((size_t)(nbh * nc * d), sizeof(double));
  double* dbp = (double*)calloc((size_t)(nbh * nc), sizeof(double));
  hils_oracle_summary(D, Kt, LQ, 0, nc, kp, bp);
  memset(dQ, 0, sizeof(double) * (size_t)(D->B * D->Hq * N * d));
  if (dQs) memset(dQs, 0, sizeof(double) * (size_t)(D->B * D->Hq * N * d));
  memset(dK, 0, sizeof(double) * (size_t)(nbh * N * d));
  memset(dV, 0, sizeof(double) * (size_t)(nbh * N * d));
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < nbh; ++bh) {
    const int64_t b = bh / D->Hkv, h = bh % D->Hkv;
    const float* Kbh = Kt + bh * N * d;
    const float* Vbh = Vt + bh * N * d;
    branch_t* br = (branch_t*)malloc(sizeof(branch_t) * (size_t)(ids_stride + 1));
    double* z = (double*)malloc(sizeof(double) * (size_t)(C * window_chunks(D)));
    double* o = (double*)malloc(sizeof(double) * (size_t)((ids_stride + 1) * d));
    double* Orow = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t g = 0; g < G; ++g) {
      const int64_t hq = h * G + g;
      for (int64_t i = 0; i < N; ++i) {
        const int64_t row = (b * D->Hq + hq) * N + i;
        const float* q = Q + row * d;
        const float* qs = Qs ? Qs + row * d : q;
        const float* gr = dO + row * d;
        double* dq = dQ + row * d;
        double* dqs = dQs ? dQs + row * d : dq;
        /* the row's branches: selected chunks, then the window */
        int64_t nb = 0;
        for (int64_t t = 0; t < ids_stride; ++t) {
          const int64_t c = ids[row * ids_stride + t];
          if (c < 0) continue;
          br[nb].j0 = c * C;
          br[nb].j1 = (c + 1) * C;
          br[nb].chunk = c;
          br[nb].u = tau * dot_fdd(qs, kp + (bh * nc + c) * d, d) + bp[bh * nc + c];
          ++nb;
        }
        int64_t w0 = (i / C - (window_chunks(D) - 1)) * C;
        if (w0 < 0) w0 = 0;
        br[nb].j0 = w0;
        br[nb].j1 = i + 1;
        br[nb].chunk = -1;
        ++nb;
        for (int64_t c = 0; c < nb; ++c) {
          br[c].lse = attend_keys(q, Kbh, Vbh, br[c].j0, br[c].j1, d, tau, z, o + c * d);
          if (br[c].chunk < 0) br[c].u = br[c].lse;
        }
        double M = -INFINITY;
        for (int64_t c = 0; c < nb; ++c) if (br[c].u > M) M = br[c].u;
        double Zs = 0.0;
        for (int64_t c = 0; c < nb; ++c) Zs += exp(br[c].u - M);
        for (int64_t t = 0; t < d; ++t) Orow[t] = 0.0;
        for (int64_t c = 0; c < nb; ++c) {
          const double a = exp(br[c].u - M) / Zs;
          for (int64_t t = 0; t < d; ++t) Orow[t] += a * o[c * d + t];
        }
        double Dg = 0.0;
        for (int64_t t = 0; t < d; ++t) Dg += (double)gr[t] * Orow[t];
        for (int64_t c = 0; c < nb; ++c) {
          const double a = exp(br[c].u - M) / Zs;
          double X = 0.0;
          for (int64_t t = 0; t < d; ++t) X += (double)gr[t] * o[c * d + t];
          const double du = a * (X - Dg);
          for (int64_t j = br[c].j0; j < br[c].j1; ++j) {
            const double zj = tau * dot_fd(q, Kbh + j * d, d);
            const double pj = exp(zj - br[c].lse);
            const double dP = dot_fd(gr, Vbh + j * d, d);
            double dz = a * pj * (dP - X);
            if (br[c].chunk < 0) dz += du * pj;
            double* dkj = dK + (bh * N + j) * d;
            double* dvj = dV + (bh * N + j) * d;
            for (int64_t t = 0; t < d; ++t) {
              dvj[t] += a * pj * (double)gr[t];
              dq[t] += tau * dz * (double)Kbh[j * d + t];
              dkj[t] += tau * dz * (double)q[t];
            }
          }
          if (br[c].chunk >= 0) {
            const int64_t cc = br[c].chunk;
            for (int64_t t = 0; t < d; ++t) {
              dqs[t] += tau * du * kp[(bh * nc + cc) * d + t];
              dkp[(bh * nc + cc) * d + t] += tau * du * (double)qs[t];
            }
            dbp[bh * nc + cc] += du;
          }
        }
      }
    }
    /* the landmark summaries of this (b, kv head) */
    for (int64_t c = 0; c < nc; ++c) {
      const float* lq = LQ + (bh * nc + c) * d;
      const float* kc = Kbh + c * C * d;
      const double* kpc = kp + (bh * nc + c) * d;
      const double* dkpc = dkp + (bh * nc + c) * d;
      const double dbpc = dbp[bh * nc + c];
      double* zl = z;   /* the landmark logits of chunk c */
      double m = -INFINITY;
      for (int64_t j = 0; j < C; ++j) {
        zl[j] = tau * dot_fd(lq, kc + j * d, d);
        if (zl[j] > m) m = zl[j];
      }
      double Zl = 0.0;
      for (int64_t j = 0; j < C; ++j) Zl += exp(zl[j] - m);
      double zbar = 0.0;
      for (int64_t j = 0; j < C; ++j) zbar += exp(zl[j] - m) / Zl * zl[j];
      double* dlq = dLQ + (bh * nc + c) * d;
      for (int64_t t = 0; t < d; ++t) dlq[t] = 0.0;
      for (int64_t j = 0; j < C; ++j) {
        const double pj = exp(zl[j] - m) / Zl;
        double proj = 0.0;
        for (int64_t t = 0; t < d; ++t) proj += dkpc[t] * ((double)kc[j * d + t] - kpc[t]);
        const double dz = pj * proj - dbpc * pj * (zl[j] - zbar);
        double* dkj = dK + (bh * N + c * C + j) * d;
        for (int64_t t = 0; t < d; ++t) {
          dlq[t] += tau * dz * (double)kc[j * d + t];
          dkj[t] += tau * dz * (double)lq[t] + pj * dkpc[t];
        }
      }
    }
    free(br);
    free(z);
    free(o);
    free(Orow);
  }
  free(kp);
  free(bp);
  free(dkp);
  free(dbp);
}

int hils_oracle_max_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
