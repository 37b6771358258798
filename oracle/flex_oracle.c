/*
 * flex_oracle.c -- plain fp64 CPU oracle for flex attention (forward, backward, decode).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; every rule below is
 * written again from the method's definition.
 *
 * What it computes (one query row i of batch b, query head h):
 *
 *   hk     = h / (H / Hkv)                       GQA: contiguous head groups
 *                                                 (torch-mlir PR 4366 "[TORCH] Added
 *                                                 flex_attention hop function",
 *                                                 Description: enable_gqa operand)
 *   x_j    = scale * sum_d Q[b,h,i,d] K[b,hk,j,d]  score, scaled first
 *   x_j   += score_mod(...)                      alibi: slope_h * (j - i),
 *                                                 slope_h = 2^(-8 (h+1) / H)
 *                                                 (FlyDSL PR 931 "Add flex_attention
 *                                                 (score_mod / mask_mod) ...",
 *                                                 Summary: score_mod runs after the
 *                                                 scale and before the mask)
 *   keep_j = mask_mod(b,h,i,j)                   causal: j <= i;
 *                                                 sliding window W: j <= i && i-j < W;
 *                                                 offset o: j <= i + o
 *   M      = max over kept j of x_j
 *   l      = sum over kept j of exp(x_j - M)
 *   O[i]   = sum over kept j of exp(x_j - M) / l * V[b,hk,j,:]
 *   LSE[i] = M + ln l        (natural log)
 *   no kept j  ->  O[i] = 0, LSE[i] = -inf       (FlyDSL PR 931, Summary:
 *                                                 fully-masked rows give 0/-inf)
 *
 * Decode (IREE issue 19015 "[ROCM] Support dynamic key-value cache sequence
 * length", example IR: one query row against a KV cache of dynamic length and an
 * f16 additive mask operand): x_j = scale * q.k_j + mask[b,h,j] for j < kv_len[b];
 * keep_j = (x_j != -inf); then the same softmax as above.
 *
 * Tensor-capturing mods (FlyDSL PR 931, Out of scope: a later phase, undefined; the
 * readings are stated at keep_rule below): alibi with a captured per-head slope table,
 * and a document mask (optionally causal) over per-batch document boundaries.
 *
 * Block-sparse forward (BlockMask; FlyDSL PR 931, "Out of scope (future phases)":
 * block sparsity named as the next phase, with no definition given).  Reading: the
 * PyTorch BlockMask convention.  For query tile t = i / BM of (b, h), a key j with
 * block u = j / BN is kept iff j < Skv and (u is in the full list of t, or u is in
 * the partial list of t and mask_mod(i, j) holds).  Unlisted blocks are dropped.
 * Everything else (scale, score_mod, softmax, 0/-inf rows) is the forward above, and
 * the block-sparse backward is the backward below with this keep rule.
 *
 * Tile map: for a BM x BN grid over (query, key) positions, a tile is
 *   EMPTY(0)   if no element with i < Sq has keep && j < Skv,
 *   FULL(1)    if every element with i < Sq has keep && j < Skv,
 *   PARTIAL(2) otherwise.
 *
 * Everything is a direct loop in double precision; rows are split across
 * POSIX threads and nothing else is reordered.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Oracle-local identifiers; the Python wrapper maps names onto these. */
#define OR_SCORE_NONE 0
#define OR_SCORE_ALIBI 1

#define OR_MASK_NONE 0
#define OR_MASK_CAUSAL 1
#define OR_MASK_SLIDING 2
#define OR_MASK_OFFSET 3
#define OR_MASK_DOC 5
#define OR_MASK_DOC_CAUSAL 6

#define OR_DT_BF16 0
#define OR_DT_F16 1
#define OR_DT_E4M3 2  /* 8-bit e4m3 (OCP E4M3FN): the buffers hold bytes */

/* ---- exact conversion of stored 16-bit values to double ---------------- */

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double f16_bits_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(m + 1024), e - 25);   /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* e4m3: sign, 4 exponent bits (bias 7), 3 mantissa bits; no infinities; S.1111.111 is NaN */
static double e4m3_bits_to_double(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 15;
  int m = b & 7;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -9);              /* subnormal: m/8 * 2^-6 */
  } else if (e == 15 && m == 7) {
    v = NAN;
  } else {
    v = ldexp((double)(m + 8), e - 10);    /* (1 + m/8) * 2^(e-7) */
  }
  return sign ? -v : v;
}

double oracle_e4m3_value(int bits) { return e4m3_bits_to_double((uint8_t)bits); }

static double elem(const uint16_t* p, int64_t idx, int dtype) {
  if (dtype == OR_DT_E4M3) return e4m3_bits_to_double(((const uint8_t*)p)[idx]);
  return dtype == OR_DT_BF16 ? bf16_bits_to_double(p[idx]) : f16_bits_to_double(p[idx]);
}

/* ---- the hooks, written from their definitions -------------------------- */

double oracle_alibi_slope(int h, int H) { return pow(2.0, -8.0 * (double)(h + 1) / (double)H); }

int oracle_mask_keep(int mask_mod, int64_t i, int64_t j, int window, int offset) {
  switch (mask_mod) {
    case OR_MASK_NONE: return 1;
    case OR_MASK_CAUSAL: return j <= i;
    case OR_MASK_SLIDING: return (j <= i) && (i - j < (int64_t)window);
    case OR_MASK_OFFSET: return j <= i + (int64_t)offset;
    default: return 0;
  }
}

/* Tensor-capturing mods (FlyDSL PR 931, Out of scope: "tensor-capturing mods" named as a
 * later phase, undefined).  Readings:
 *  - alibi with a captured per-head slope table: s += slopes[h] * (j - i);
 *  - document mask over packed sequences: the captured tensors give, per batch b, the
 *    document boundaries off_q[b][0..n_docs] of the query positions and off_kv[b][..]
 *    of the key positions; position p is in document d iff off[d] <= p < off[d+1], and
 *    in none if no such d.  Keep (i, j) iff i and j are in the same document d (and,
 *    for the causal form, j <= i in absolute positions). */
typedef struct {
  const double* slopes;          /* [H], or NULL for the built-in slopes */
  const int32_t *off_q, *off_kv; /* [B][n_docs + 1] */
  int n_docs;
} captured_mods;

/* Document d with off[d] <= pos < off[d+1], or -1 (a plain scan of the boundaries). */
static int64_t doc_of(const int32_t* off, int n_docs, int64_t pos) {
  for (int d = 0; d < n_docs; ++d)
    if ((int64_t)off[d] <= pos && pos < (int64_t)off[d + 1]) return d;
  return -1;
}

/* The keep rule of element (i, j) of batch b, mask_mod with its parameters. */
static int keep_rule(int mask_mod, int window, int offset, const captured_mods* C, int b, int64_t i,
                     int64_t j) {
  if (mask_mod == OR_MASK_DOC || mask_mod == OR_MASK_DOC_CAUSAL) {
    const int32_t* oq = C->off_q + (int64_t)b * (C->n_docs + 1);
    const int32_t* okv = C->off_kv + (int64_t)b * (C->n_docs + 1);
    int64_t dq = doc_of(oq, C->n_docs, i);
    if (dq < 0 || dq != doc_of(okv, C->n_docs, j)) return 0;
    return mask_mod == OR_MASK_DOC || j <= i;
  }
  return oracle_mask_keep(mask_mod, i, j, window, offset);
}

/* Block mask (BlockMask).  Reading: PyTorch's convention.  For query tile t of one
 * (b, h) (tile_row = (b*H + h) * n_qtiles + t), the key blocks u listed in
 * full_idx[tile_row, 0 .. full_num) are kept wholesale (only j < Skv applies), those in
 * kv_idx[tile_row, 0 .. kv_num) keep (i, j) iff mask_mod(i, j) && j < Skv, and every
 * other block is dropped.  A block on both lists counts as full.  Counts are clamped
 * to [0, max_blocks]; an index outside [0, ceil(Skv/BN)) matches no key. */
typedef struct {
  const int32_t *kv_num, *kv_idx, *full_num, *full_idx;
  int max_blocks, BM, BN, n_qtiles;
} block_lists;

static int block_listed(const int32_t* num, const int32_t* idx, int64_t row, int max_blocks, int64_t u) {
  if (!num || !idx) return 0;
  int32_t cnt = num[row];
  if (cnt > max_blocks) cnt = max_blocks;
  for (int32_t c = 0; c < cnt; ++c)
    if ((int64_t)idx[row * max_blocks + c] == u) return 1;
  return 0;
}

static int block_keep(const block_lists* L, int64_t bh, int mask_mod, int64_t i, int64_t j, int Skv,
                      int window, int offset, const captured_mods* C, int b) {
  if (j >= Skv) return 0;
  int64_t tile_row = bh * L->n_qtiles + i / L->BM;
  int64_t u = j / L->BN;
  if (block_listed(L->full_num, L->full_idx, tile_row, L->max_blocks, u)) return 1;
  if (block_listed(L->kv_num, L->kv_idx, tile_row, L->max_blocks, u)) return keep_rule(mask_mod, window, offset, C, b, i, j);
  return 0;
}

/* ---- forward -------------------------------------------------------------- */

typedef struct {
  const uint16_t *q, *k, *v;
  int dtype, B, H, Hkv, Sq, Skv, D;
  double scale;
  int score_mod, mask_mod, window, offset;
  const int64_t* rows;   /* flattened (b*H + h)*Sq + i; NULL = all rows */
  int64_t n_rows;
  double* o;             /* [n_rows, D] */
  double* lse;           /* [n_rows] */
  double* probs;         /* optional [n_rows, Skv] normalised weights */
  const block_lists* blk; /* block mask, or NULL for mask_mod alone */
  captured_mods cap;      /* captured tensors of the mods */
  int64_t r0, r1;
} fwd_job;

/* Key/value head of query head h (GQA: contiguous groups of H / Hkv query heads). */
static int kv_head(const fwd_job* J, int h) {
  int G = J->H / J->Hkv;
  int hk = h / G;
  return hk;
}

/* x_ij = scale * q_i . k_j + score_mod bias, for row i of (b, h) and key j. */
static double score_ij(const fwd_job* J, int b, int h, int64_t i, int64_t j) {
  int D = J->D;
  const int64_t qbase = (((int64_t)b * J->H + h) * J->Sq + i) * D;
  const int64_t kvbase = ((int64_t)b * J->Hkv + kv_head(J, h)) * (int64_t)J->Skv * D;
  double slope = 0.0;
  if (J->score_mod == OR_SCORE_ALIBI) slope = J->cap.slopes ? J->cap.slopes[h] : oracle_alibi_slope(h, J->H);
  double dot = 0.0;
  for (int d = 0; d < D; ++d)
    dot += elem(J->q, qbase + d, J->dtype) * elem(J->k, kvbase + j * D + d, J->dtype);
  double s = J->scale * dot;
  if (J->score_mod == OR_SCORE_ALIBI) s += slope * (double)(j - i);
  return s;
}

/* The keep decision of element (i, j) of (b, h): the block mask if any, else mask_mod. */
static int keep_ij(const fwd_job* J, int b, int h, int64_t i, int64_t j) {
  int64_t bh = (int64_t)b * J->H + h;
  return J->blk ? block_keep(J->blk, bh, J->mask_mod, i, j, J->Skv, J->window, J->offset, &J->cap, b)
                : keep_rule(J->mask_mod, J->window, J->offset, &J->cap, b, i, j);
}

static void fwd_row(const fwd_job* J, int64_t r, double* x, unsigned char* keep) {
  int64_t flat = J->rows ? J->rows[r] : r;
  int64_t i = flat % J->Sq;
  int64_t bh = flat / J->Sq;
  int h = (int)(bh % J->H);
  int b = (int)(bh / J->H);
  int D = J->D;
  const int64_t kvbase = ((int64_t)b * J->Hkv + kv_head(J, h)) * (int64_t)J->Skv * D;

  double M = -INFINITY;
  int any = 0;
  for (int64_t j = 0; j < J->Skv; ++j) {
    double s = score_ij(J, b, h, i, j);
    x[j] = s;
    keep[j] = (unsigned char)keep_ij(J, b, h, i, j);
    if (keep[j]) {
      any = 1;
      if (s > M) M = s;
    }
  }
  double* o = J->o + r * D;
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (!any) {
    J->lse[r] = -INFINITY;
    if (J->probs)
      for (int64_t j = 0; j < J->Skv; ++j) J->probs[r * J->Skv + j] = 0.0;
    return;
  }
  double l = 0.0;
  for (int64_t j = 0; j < J->Skv; ++j)
    if (keep[j]) l += exp(x[j] - M);
  for (int64_t j = 0; j < J->Skv; ++j) {
    double p = keep[j] ? exp(x[j] - M) / l : 0.0;
    if (J->probs) J->probs[r * J->Skv + j] = p;
    if (p != 0.0)
      for (int d = 0; d < D; ++d) o[d] += p * elem(J->v, kvbase + j * D + d, J->dtype);
  }
  J->lse[r] = M + log(l);
}

static void* fwd_worker(void* arg) {
  fwd_job* J = (fwd_job*)arg;
  double* x = (double*)malloc(sizeof(double) * (size_t)J->Skv);
  unsigned char* keep = (unsigned char*)malloc((size_t)J->Skv);
  if (x && keep)
    for (int64_t r = J->r0; r < J->r1; ++r) fwd_row(J, r, x, keep);
  free(x);
  free(keep);
  return NULL;
}

static int run_jobs(fwd_job* base, int64_t n_rows, int nthreads, void* (*fn)(void*), size_t job_size) {
  if (nthreads < 1) nthreads = 1;
  if ((int64_t)nthreads > n_rows) nthreads = (int)(n_rows > 0 ? n_rows : 1);
  char* jobs = (char*)malloc(job_size * (size_t)nthreads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!jobs || !th) { free(jobs); free(th); return -1; }
  for (int t = 0; t < nthreads; ++t) {
    fwd_job* J = (fwd_job*)(jobs + job_size * (size_t)t);
    memcpy(J, base, job_size);
    J->r0 = n_rows * t / nthreads;
    J->r1 = n_rows * (t + 1) / nthreads;
  }
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, fn, jobs + job_size * (size_t)t) != 0) break;
    started = t;
  }
  fn(jobs);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  /* any worker that failed to start: run it here */
  for (int t = started + 1; t < nthreads; ++t) fn(jobs + job_size * (size_t)t);
  free(jobs);
  free(th);
  return 0;
}

/* Forward over selected rows (rows == NULL: all B*H*Sq rows). */
/* slopes, off_q, off_kv: the captured tensors (NULL when the mods take none). */
int oracle_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dtype,
               int B, int H, int Hkv, int Sq, int Skv, int D, double scale,
               int score_mod, int mask_mod, int window, int offset,
               const double* slopes, const int32_t* off_q, const int32_t* off_kv, int n_docs,
               const int64_t* rows, int64_t n_rows,
               double* o, double* lse, double* probs, int nthreads) {
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || Sq <= 0 || Skv <= 0 || D <= 0) return -1;
  fwd_job J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v; J.dtype = dtype;
  J.B = B; J.H = H; J.Hkv = Hkv; J.Sq = Sq; J.Skv = Skv; J.D = D;
  J.scale = scale; J.score_mod = score_mod; J.mask_mod = mask_mod;
  J.window = window; J.offset = offset;
  J.rows = rows;
  J.n_rows = rows ? n_rows : (int64_t)B * H * Sq;
  J.o = o; J.lse = lse; J.probs = probs;
  J.cap.slopes = slopes; J.cap.off_q = off_q; J.cap.off_kv = off_kv; J.cap.n_docs = n_docs;
  if ((mask_mod == OR_MASK_DOC || mask_mod == OR_MASK_DOC_CAUSAL) && (!off_q || !off_kv || n_docs < 0)) return -2;
  return run_jobs(&J, J.n_rows, nthreads, fwd_worker, sizeof J);
}

/* ---- backward ---------------------------------------------------------------
 * Gradients of the forward above (FlyDSL PR 931, Out of scope: the backward pass as a
 * later phase; xformers 1094 reports dq/dk/dv mean errors of its own backward).  With an
 * upstream gradient dO, per query row i of (b, h) and kept key j:
 *   P_ij  = exp(x_ij - M_i) / l_i            (the forward's probabilities, 0 if dropped)
 *   O_i   = sum_j P_ij V_j,   delta_i = sum_d dO_id O_id
 *   dP_ij = dO_i . V_j,       dS_ij = P_ij (dP_ij - delta_i)
 *   dQ_i  = scale sum_j dS_ij K_j
 *   dK_j  = scale sum_{h, i} dS_ij Q_i,   dV_j = sum_{h, i} P_ij dO_i
 * where the sums over h run over the query heads that share key/value head hk (GQA).
 * score_mod adds a bias that does not depend on Q or K, so it enters only through P.
 * Two passes per (b, hk) group: rows (statistics, delta, dQ), then keys (dK, dV, with P
 * and dS recomputed from the row statistics). */

typedef struct {
  fwd_job f;                 /* inputs, mods and the keep rule of the forward */
  const uint16_t* dout;      /* dO [B, H, Sq, D] */
  const int64_t* groups;     /* b * Hkv + hk of each group computed */
  int64_t n_groups;
  double *dq, *dk, *dv;      /* [n_groups, G, Sq, D], [n_groups, Skv, D] x 2 */
  double *M, *l, *delta;     /* [n_groups, G, Sq] row statistics */
  int pass;                  /* 1: rows, 2: keys */
} bwd_job;

static void* bwd_worker(void* arg) {
  bwd_job* W = (bwd_job*)arg;
  const fwd_job* J = &W->f;
  const int D = J->D, G = J->H / J->Hkv;
  const int64_t Sq = J->Sq, Skv = J->Skv;
  double* x = (double*)malloc(sizeof(double) * (size_t)Skv);
  unsigned char* keep = (unsigned char*)malloc((size_t)Skv);
  double* acc = (double*)malloc(sizeof(double) * (size_t)D * 2);
  if (x && keep && acc) {
    for (int64_t t = J->r0; t < J->r1; ++t) {
      if (W->pass == 1) {
        /* task t = (group, head in group, row) */
        int64_t gi = t / (G * Sq), rem = t % (G * Sq);
        int hg = (int)(rem / Sq);
        int64_t i = rem % Sq;
        int64_t g = W->groups[gi];
        int b = (int)(g / J->Hkv), hk = (int)(g % J->Hkv), h = hk * G + hg;  /* kv_head(J, h) == hk */
        const int64_t kvbase = ((int64_t)b * J->Hkv + hk) * Skv * D;
        const int64_t obase = (((int64_t)b * J->H + h) * Sq + i) * D;
        for (int64_t j = 0; j < Skv; ++j) {
          x[j] = score_ij(J, b, h, i, j);
          keep[j] = (unsigned char)keep_ij(J, b, h, i, j);
        }
        double M = -INFINITY, l = 0.0;
        for (int64_t j = 0; j < Skv; ++j)
          if (keep[j] && x[j] > M) M = x[j];
        double* dq = W->dq + ((gi * G + hg) * Sq + i) * D;
        for (int d = 0; d < D; ++d) dq[d] = 0.0;
        int64_t srow = (gi * G + hg) * Sq + i;
        W->M[srow] = M;
        if (M == -INFINITY) {  /* no kept key: no gradient through this row */
          W->l[srow] = 0.0;
          W->delta[srow] = 0.0;
          continue;
        }
        for (int64_t j = 0; j < Skv; ++j)
          if (keep[j]) l += exp(x[j] - M);
        W->l[srow] = l;
        /* O_i and delta_i */
        for (int d = 0; d < D; ++d) acc[d] = 0.0;
        for (int64_t j = 0; j < Skv; ++j) {
          if (!keep[j]) continue;
          double pij = exp(x[j] - M) / l;
          for (int d = 0; d < D; ++d) acc[d] += pij * elem(J->v, kvbase + j * D + d, J->dtype);
        }
        double delta = 0.0;
        for (int d = 0; d < D; ++d) delta += elem(W->dout, obase + d, J->dtype) * acc[d];
        W->delta[srow] = delta;
        /* dQ_i */
        for (int64_t j = 0; j < Skv; ++j) {
          if (!keep[j]) continue;
          double pij = exp(x[j] - M) / l, dp = 0.0;
          for (int d = 0; d < D; ++d) dp += elem(W->dout, obase + d, J->dtype) * elem(J->v, kvbase + j * D + d, J->dtype);
          double ds = pij * (dp - delta);
          for (int d = 0; d < D; ++d) dq[d] += J->scale * ds * elem(J->k, kvbase + j * D + d, J->dtype);
        }
      } else {
        /* task t = (group, key) */
        int64_t gi = t / Skv, j = t % Skv;
        int64_t g = W->groups[gi];
        int b = (int)(g / J->Hkv), hk = (int)(g % J->Hkv);
        const int64_t kvbase = ((int64_t)b * J->Hkv + hk) * Skv * D;
        double* dk = acc;
        double* dv = acc + D;
        for (int d = 0; d < 2 * D; ++d) acc[d] = 0.0;
        for (int hg = 0; hg < G; ++hg) {
          int h = hk * G + hg;
          for (int64_t i = 0; i < Sq; ++i) {
            int64_t srow = (gi * G + hg) * Sq + i;
            if (W->M[srow] == -INFINITY) continue;
            if (!keep_ij(J, b, h, i, j)) continue;
            const int64_t qbase = (((int64_t)b * J->H + h) * Sq + i) * D;
            double dp = 0.0;
            for (int d = 0; d < D; ++d)
              dp += elem(W->dout, qbase + d, J->dtype) * elem(J->v, kvbase + j * D + d, J->dtype);
            double pij = exp(score_ij(J, b, h, i, j) - W->M[srow]) / W->l[srow];
            double ds = pij * (dp - W->delta[srow]);
            for (int d = 0; d < D; ++d) {
              dk[d] += J->scale * ds * elem(J->q, qbase + d, J->dtype);
              dv[d] += pij * elem(W->dout, qbase + d, J->dtype);
            }
          }
        }
        for (int d = 0; d < D; ++d) {
          W->dk[(gi * Skv + j) * D + d] = dk[d];
          W->dv[(gi * Skv + j) * D + d] = dv[d];
        }
      }
    }
  }
  free(x);
  free(keep);
  free(acc);
  return NULL;
}

static int run_bwd_pass(bwd_job* base, int64_t n_tasks, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if ((int64_t)nthreads > n_tasks) nthreads = (int)(n_tasks > 0 ? n_tasks : 1);
  bwd_job* jobs = (bwd_job*)malloc(sizeof(bwd_job) * (size_t)nthreads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!jobs || !th) { free(jobs); free(th); return -3; }
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = *base;
    jobs[t].f.r0 = n_tasks * t / nthreads;
    jobs[t].f.r1 = n_tasks * (t + 1) / nthreads;
  }
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, bwd_worker, &jobs[t]) != 0) break;
    started = t;
  }
  bwd_worker(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  for (int t = started + 1; t < nthreads; ++t) bwd_worker(&jobs[t]);
  free(jobs);
  free(th);
  return 0;
}

/* Backward for the (b, hk) groups listed (groups == NULL: all B*Hkv), with the keep rule
 * of mask_mod, or of the block lists when blk is given.  dq: [n_groups, G, Sq, D]; dk, dv:
 * [n_groups, Skv, D] (G = H / Hkv query heads per group, in order). */
static int bwd_run(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout, int dtype,
                   int B, int H, int Hkv, int Sq, int Skv, int D, double scale,
                   int score_mod, int mask_mod, int window, int offset,
                   const double* slopes, const int32_t* off_q, const int32_t* off_kv, int n_docs,
                   const block_lists* blk, const int64_t* groups, int64_t n_groups, double* dq, double* dk,
                   double* dv, int nthreads) {
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || Sq <= 0 || Skv <= 0 || D <= 0) return -1;
  if ((mask_mod == OR_MASK_DOC || mask_mod == OR_MASK_DOC_CAUSAL) && (!off_q || !off_kv || n_docs < 0)) return -2;
  int64_t ng = groups ? n_groups : (int64_t)B * Hkv;
  int64_t* all = NULL;
  if (!groups) {
    all = (int64_t*)malloc(sizeof(int64_t) * (size_t)ng);
    if (!all) return -3;
    for (int64_t g = 0; g < ng; ++g) all[g] = g;
  }
  const int G = H / Hkv;
  bwd_job W;
  memset(&W, 0, sizeof W);
  fwd_job* J = &W.f;
  J->q = q; J->k = k; J->v = v; J->dtype = dtype;
  J->B = B; J->H = H; J->Hkv = Hkv; J->Sq = Sq; J->Skv = Skv; J->D = D;
  J->scale = scale; J->score_mod = score_mod; J->mask_mod = mask_mod;
  J->window = window; J->offset = offset;
  J->cap.slopes = slopes; J->cap.off_q = off_q; J->cap.off_kv = off_kv; J->cap.n_docs = n_docs;
  J->blk = blk;
  W.dout = dout;
  W.groups = groups ? groups : all;
  W.n_groups = ng;
  W.dq = dq; W.dk = dk; W.dv = dv;
  size_t nrows = (size_t)ng * G * Sq;
  W.M = (double*)malloc(sizeof(double) * nrows);
  W.l = (double*)malloc(sizeof(double) * nrows);
  W.delta = (double*)malloc(sizeof(double) * nrows);
  int rc = -3;
  if (W.M && W.l && W.delta) {
    W.pass = 1;
    rc = run_bwd_pass(&W, ng * G * (int64_t)Sq, nthreads);
    if (rc == 0) {
      W.pass = 2;
      rc = run_bwd_pass(&W, ng * (int64_t)Skv, nthreads);
    }
  }
  free(W.M);
  free(W.l);
  free(W.delta);
  free(all);
  return rc;
}

int oracle_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout, int dtype,
               int B, int H, int Hkv, int Sq, int Skv, int D, double scale,
               int score_mod, int mask_mod, int window, int offset,
               const double* slopes, const int32_t* off_q, const int32_t* off_kv, int n_docs,
               const int64_t* groups, int64_t n_groups, double* dq, double* dk, double* dv, int nthreads) {
  return bwd_run(q, k, v, dout, dtype, B, H, Hkv, Sq, Skv, D, scale, score_mod, mask_mod, window, offset, slopes,
                 off_q, off_kv, n_docs, NULL, groups, n_groups, dq, dk, dv, nthreads);
}

/* Backward of the block-sparse forward: the gradients of the forward whose keep rule is
 * the block lists' (oracle_fwd_block_sparse).  The lists are laid out as there. */
int oracle_bwd_block_sparse(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                            int dtype, int B, int H, int Hkv, int Sq, int Skv, int D, double scale,
                            int score_mod, int mask_mod, int window, int offset,
                            const double* slopes, const int32_t* off_q, const int32_t* off_kv, int n_docs,
                            const int32_t* kv_num, const int32_t* kv_idx, const int32_t* full_num,
                            const int32_t* full_idx, int max_blocks, int BM, int BN,
                            const int64_t* groups, int64_t n_groups, double* dq, double* dk, double* dv,
                            int nthreads) {
  if (BM <= 0 || BN <= 0 || max_blocks < 0 || Sq <= 0) return -1;
  block_lists L;
  L.kv_num = kv_num; L.kv_idx = kv_idx; L.full_num = full_num; L.full_idx = full_idx;
  L.max_blocks = max_blocks; L.BM = BM; L.BN = BN; L.n_qtiles = (Sq + BM - 1) / BM;
  return bwd_run(q, k, v, dout, dtype, B, H, Hkv, Sq, Skv, D, scale, score_mod, mask_mod, window, offset, slopes,
                 off_q, off_kv, n_docs, &L, groups, n_groups, dq, dk, dv, nthreads);
}

/* ---- decode ---------------------------------------------------------------- */

typedef struct {
  const uint16_t *q, *kc, *vc, *mask;
  const int32_t* kv_len;
  int dtype, mask_dtype, B, H, Hkv, cap, D;
  double scale;
  double* o;    /* [B*H, D] */
  double* lse;  /* [B*H]    */
  int64_t r0, r1;
} dec_job;

static void dec_row(const dec_job* J, int64_t r, double* x) {
  int h = (int)(r % J->H);
  int b = (int)(r / J->H);
  int hk = h / (J->H / J->Hkv);
  int D = J->D;
  int64_t L = J->kv_len[b];
  const int64_t kvbase = ((int64_t)b * J->Hkv + hk) * (int64_t)J->cap * D;
  double M = -INFINITY;
  for (int64_t j = 0; j < L; ++j) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d)
      dot += elem(J->q, r * D + d, J->dtype) * elem(J->kc, kvbase + j * D + d, J->dtype);
    double s = J->scale * dot;
    if (J->mask) s += elem(J->mask, r * (int64_t)J->cap + j, J->mask_dtype);
    x[j] = s;
    if (s > M) M = s;
  }
  double* o = J->o + r * D;
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (M == -INFINITY) {   /* kv_len == 0 or every position masked */
    J->lse[r] = -INFINITY;
    return;
  }
  double l = 0.0;
  for (int64_t j = 0; j < L; ++j)
    if (x[j] != -INFINITY) l += exp(x[j] - M);
  for (int64_t j = 0; j < L; ++j) {
    if (x[j] == -INFINITY) continue;
    double p = exp(x[j] - M) / l;
    for (int d = 0; d < D; ++d) o[d] += p * elem(J->vc, kvbase + j * D + d, J->dtype);
  }
  J->lse[r] = M + log(l);
}

static void* dec_worker(void* arg) {
  dec_job* J = (dec_job*)arg;
  double* x = (double*)malloc(sizeof(double) * (size_t)(J->cap > 0 ? J->cap : 1));
  if (x)
    for (int64_t r = J->r0; r < J->r1; ++r) dec_row(J, r, x);
  free(x);
  return NULL;
}

int oracle_decode(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                  const int32_t* kv_len, const uint16_t* mask, int mask_dtype, int dtype,
                  int B, int H, int Hkv, int cap, int D, double scale,
                  double* o, double* lse, int nthreads) {
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || cap <= 0 || D <= 0) return -1;
  for (int b = 0; b < B; ++b)
    if (kv_len[b] < 0 || kv_len[b] > cap) return -2;
  dec_job J;
  memset(&J, 0, sizeof J);
  J.q = q; J.kc = kc; J.vc = vc; J.mask = mask; J.kv_len = kv_len;
  J.dtype = dtype; J.mask_dtype = mask_dtype;
  J.B = B; J.H = H; J.Hkv = Hkv; J.cap = cap; J.D = D; J.scale = scale;
  J.o = o; J.lse = lse;
  int64_t n = (int64_t)B * H;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > n) nthreads = (int)(n > 0 ? n : 1);
  dec_job* jobs = (dec_job*)malloc(sizeof(dec_job) * (size_t)nthreads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!jobs || !th) { free(jobs); free(th); return -3; }
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = J;
    jobs[t].r0 = n * t / nthreads;
    jobs[t].r1 = n * (t + 1) / nthreads;
  }
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, dec_worker, &jobs[t]) != 0) break;
    started = t;
  }
  dec_worker(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  for (int t = started + 1; t < nthreads; ++t) dec_worker(&jobs[t]);
  free(jobs);
  free(th);
  return 0;
}

/* Block-sparse forward over selected rows: the forward above with the keep rule of the
 * block lists.  kv_num/full_num are [B*H*n_qtiles] and kv_idx/full_idx
 * [B*H*n_qtiles*max_blocks] int32, n_qtiles = ceil(Sq/BM); either pair may be NULL. */
int oracle_fwd_block_sparse(const uint16_t* q, const uint16_t* k, const uint16_t* v, int dtype,
                            int B, int H, int Hkv, int Sq, int Skv, int D, double scale,
                            int score_mod, int mask_mod, int window, int offset,
                            const double* slopes, const int32_t* off_q, const int32_t* off_kv, int n_docs,
                            const int32_t* kv_num, const int32_t* kv_idx, const int32_t* full_num,
                            const int32_t* full_idx, int max_blocks, int BM, int BN,
                            const int64_t* rows, int64_t n_rows, double* o, double* lse, int nthreads) {
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || Sq <= 0 || Skv <= 0 || D <= 0) return -1;
  if (BM <= 0 || BN <= 0 || max_blocks < 0) return -1;
  block_lists L;
  L.kv_num = kv_num; L.kv_idx = kv_idx; L.full_num = full_num; L.full_idx = full_idx;
  L.max_blocks = max_blocks; L.BM = BM; L.BN = BN; L.n_qtiles = (Sq + BM - 1) / BM;
  fwd_job J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v; J.dtype = dtype;
  J.B = B; J.H = H; J.Hkv = Hkv; J.Sq = Sq; J.Skv = Skv; J.D = D;
  J.scale = scale; J.score_mod = score_mod; J.mask_mod = mask_mod;
  J.window = window; J.offset = offset;
  J.rows = rows;
  J.n_rows = rows ? n_rows : (int64_t)B * H * Sq;
  J.o = o; J.lse = lse; J.blk = &L;
  J.cap.slopes = slopes; J.cap.off_q = off_q; J.cap.off_kv = off_kv; J.cap.n_docs = n_docs;
  if ((mask_mod == OR_MASK_DOC || mask_mod == OR_MASK_DOC_CAUSAL) && (!off_q || !off_kv || n_docs < 0)) return -2;
  return run_jobs(&J, J.n_rows, nthreads, fwd_worker, sizeof J);
}

/* ---- element mask and tile map (brute force) ------------------------------- */

/* keep[i*Skv + j] = mask_mod(i, j) for every i < Sq, j < Skv (document masks: the
 * boundaries off_q / off_kv of one batch, n_docs + 1 entries each). */
int oracle_mask_matrix(int mask_mod, int Sq, int Skv, int window, int offset, const int32_t* off_q,
                       const int32_t* off_kv, int n_docs, uint8_t* keep) {
  captured_mods C = {NULL, off_q, off_kv, n_docs};
  if ((mask_mod == OR_MASK_DOC || mask_mod == OR_MASK_DOC_CAUSAL) && (!off_q || !off_kv)) return -2;
  for (int64_t i = 0; i < Sq; ++i)
    for (int64_t j = 0; j < Skv; ++j)
      keep[i * Skv + j] = (uint8_t)keep_rule(mask_mod, window, offset, &C, 0, i, j);
  return 0;
}

/* map[t*nkv + u] in {0 EMPTY, 1 FULL, 2 PARTIAL}; nq = ceil(Sq/BM), nkv = ceil(Skv/BN). */
int oracle_tile_map(int mask_mod, int Sq, int Skv, int window, int offset, const int32_t* off_q,
                    const int32_t* off_kv, int n_docs, int BM, int BN, uint8_t* map) {
  captured_mods C = {NULL, off_q, off_kv, n_docs};
  if (BM <= 0 || BN <= 0) return -1;
  if ((mask_mod == OR_MASK_DOC || mask_mod == OR_MASK_DOC_CAUSAL) && (!off_q || !off_kv)) return -2;
  int nq = (Sq + BM - 1) / BM, nkv = (Skv + BN - 1) / BN;
  for (int t = 0; t < nq; ++t) {
    for (int u = 0; u < nkv; ++u) {
      int64_t kept = 0, total = 0;
      for (int64_t i = (int64_t)t * BM; i < (int64_t)(t + 1) * BM && i < Sq; ++i) {
        for (int64_t j = (int64_t)u * BN; j < (int64_t)(u + 1) * BN; ++j) {
          ++total;
          if (j < Skv && keep_rule(mask_mod, window, offset, &C, 0, i, j)) ++kept;
        }
      }
      map[(int64_t)t * nkv + u] = (uint8_t)(kept == 0 ? 0 : (kept == total ? 1 : 2));
    }
  }
  return 0;
}
