/*
 * sp_oracle.c -- plain fp64 CPU oracle for the sequence/head-parallel attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library path links, loads or calls this file; only the
 * tests, the package's smoke check and the benchmark's CPU-baseline leg do.  It shares no code,
 * header, table or constant with the CUDA implementation.
 *
 * What it computes, and where the pages define it:
 *
 *  orc_attn       Exact per-head scaled-dot-product attention, written out as its definition:
 *                 s_j = q.k_j / sqrt(D); p_j = exp(s_j - m) / l with m = max_j s_j and
 *                 l = sum_j exp(s_j - m); o = sum_j p_j v_j; lse = m + ln l.  Two passes per row, no
 *                 tiling, no online rescaling.
 *                 - "LLM Lab Notes 05: Attention Tensor Parallelism", section 2 (code walkthrough),
 *                   step 4 "local attention" and the explanation under "Local projections and local
 *                   attention": per head, q @ k^T / sqrt(head_dim), softmax over the keys, then a
 *                   weighted sum of v.  Layout (batch, seq, heads, head_dim), same section, step 3.
 *                 - Key subsets: the KV range [kv_begin, kv_end) is one Ring-Attention round
 *                   ("CHARM+: How Cross-Hardware Attention Breaks Through ...", section "Where Does
 *                   the Communication Bottleneck of Distributed Attention Come From?": each round
 *                   computes local attention on one KV block and accumulates partial results).
 *                 - A per-head block mask keeps or drops whole 128x128 (query tile, key tile) blocks
 *                   ("db-SP: Accelerating Sparse Attention ...", abstract: block-wise sparse
 *                   attention whose sparsity varies across heads).
 *                 - Causal: key j is allowed for query i iff j <= i, positions global.
 *                 - A row with no allowed key returns o = 0, lse = -inf.
 *  orc_attn_probs The probability matrix p of the same definition, for tiny inputs.
 *  orc_merge      Combination of KV-block partials (o_b, lse_b) into the result over the union of
 *                 the blocks ("CHARM+: Cross-Hardware Attention with Re-Merge Multistream
 *                 Mechanism", abstract: re-merge of partial results).  Written as the log-sum-exp
 *                 identity: lse = M + ln sum_b exp(lse_b - M), M = max_b lse_b, and
 *                 o = sum_b exp(lse_b - lse) o_b.  All lse_b = -inf gives o = 0, lse = -inf.
 *  orc_seq_to_head / orc_head_to_seq
 *                 The Ulysses all-to-all layout permutation between P rank buffers ("HCMS:
 *                 Head-Chunked Multi-Stream Pipeline ...", abstract: all-to-all based sequence
 *                 parallelism; "db-SP ...", abstract: parallelism along the head dimension as in
 *                 Ulysses).  Rank r holds sequence shard r of all heads before, and all positions of
 *                 head group r after:  out_r[b, s, h', :] = in_{s / (S/P)}[b, s % (S/P), r*H/P + h', :].
 *                 Byte copies, element by element.
 *  orc_split_heads / orc_merge_heads
 *                 The local halves of that all-to-all when the ranks are separate processes: a rank cuts
 *                 its sequence shard into P head groups before the exchange (split) and joins the head
 *                 groups it gets back after it (merge).  Byte copies, element by element.
 *  orc_tile_list  The compacted per-(head, query tile) list of kept key tiles of a block mask, in
 *                 increasing key-tile order (CSR: row_ptr, col_idx).
 *  orc_attn_bwd   The gradients of the attention above (dense or causal, all keys) for an upstream
 *                 gradient dO of O: the backward pass whose speed the CHARM+ pages report ("CHARM+ ...",
 *                 abstract: forward and backward speedups).  Plain calculus on the definition: with
 *                 p_ij the softmax of s_ij = q_i.k_j / sqrt(D) over the allowed j and o_i = sum_j p_ij v_j,
 *                   dV_j = sum_i p_ij dO_i;   dp_ij = dO_i . v_j;   delta_i = sum_j p_ij dp_ij (= dO_i . o_i);
 *                   ds_ij = p_ij (dp_ij - delta_i);   dQ_i = sum_j ds_ij k_j / sqrt(D);
 *                   dK_j = sum_i ds_ij q_i / sqrt(D).
 *                 Per (batch, head), rows in order, p from the same two-pass softmax as orc_attn.
 *
 * Threads: rows are split over POSIX threads; each row is computed by exactly one thread in a fixed
 * order, so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2

/* ------------------------------------------------------------------------------------------------ */
/* Which keys a query may see.                                                                       */
/* ------------------------------------------------------------------------------------------------ */
typedef struct {
  int S, H, causal, tile, kv_begin, kv_end, n_tiles;
  const uint8_t* block_mask; /* [H, n_tiles, n_tiles], nonzero = keep, or NULL */
} key_rule;

static int key_allowed(const key_rule* r, int h, int i, int j) {
  if (j < r->kv_begin || j >= r->kv_end || j >= r->S) return 0;
  if (r->causal && j > i) return 0;
  if (r->block_mask) {
    size_t idx = ((size_t)h * r->n_tiles + (size_t)(i / r->tile)) * r->n_tiles + (size_t)(j / r->tile);
    if (!r->block_mask[idx]) return 0;
  }
  return 1;
}

/* ------------------------------------------------------------------------------------------------ */
/* Attention                                                                                          */
/* ------------------------------------------------------------------------------------------------ */
typedef struct {
  const double *q, *k, *v;
  double *o, *lse, *probs;
  int B, S, H, D;
  key_rule rule;
  const int* rows; /* query positions to evaluate, or NULL for all S */
  int n_rows;
  long next; /* shared work counter, guarded by mu */
  pthread_mutex_t mu;
} attn_job;

static void attn_one_row(attn_job* J, int b, int h, int ri, double* s, unsigned char* ok) {
  const int S = J->S, H = J->H, D = J->D;
  const int i = J->rows ? J->rows[ri] : ri;
  const int n_out = J->rows ? J->n_rows : S;
  const double scale = 1.0 / sqrt((double)D);
  const double* qi = J->q + (((size_t)b * S + i) * H + h) * D;
  double* oi = J->o + (((size_t)b * n_out + ri) * H + h) * D;
  double* lsei = J->lse + ((size_t)b * H + h) * n_out + ri;

  /* pass 1: scores of the allowed keys and their maximum */
  double m = -INFINITY;
  int any = 0;
  for (int j = 0; j < S; ++j) {
    ok[j] = (unsigned char)key_allowed(&J->rule, h, i, j);
    if (!ok[j]) continue;
    const double* kj = J->k + (((size_t)b * S + j) * H + h) * D;
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
    s[j] = dot * scale;
    if (!any || s[j] > m) m = s[j];
    any = 1;
  }
  if (!any) {
    for (int d = 0; d < D; ++d) oi[d] = 0.0;
    *lsei = -INFINITY;
    if (J->probs) {
      double* pr = J->probs + (((size_t)b * H + h) * n_out + ri) * S;
      for (int j = 0; j < S; ++j) pr[j] = 0.0;
    }
    return;
  }
  /* pass 2: normaliser, then the weighted sum of values */
  double l = 0.0;
  for (int j = 0; j < S; ++j)
    if (ok[j]) l += exp(s[j] - m);
  for (int d = 0; d < D; ++d) oi[d] = 0.0;
  for (int j = 0; j < S; ++j) {
    if (!ok[j]) continue;
    const double p = exp(s[j] - m) / l;
    const double* vj = J->v + (((size_t)b * S + j) * H + h) * D;
    for (int d = 0; d < D; ++d) oi[d] += p * vj[d];
  }
  *lsei = m + log(l);
  if (J->probs) {
    double* pr = J->probs + (((size_t)b * H + h) * n_out + ri) * S;
    for (int j = 0; j < S; ++j) pr[j] = ok[j] ? exp(s[j] - m) / l : 0.0;
  }
}

static void* attn_worker(void* arg) {
  attn_job* J = (attn_job*)arg;
  const int n_out = J->rows ? J->n_rows : J->S;
  const long total = (long)J->B * J->H * n_out;
  double* s = (double*)malloc(sizeof(double) * (size_t)J->S);
  unsigned char* ok = (unsigned char*)malloc((size_t)J->S);
  if (!s || !ok) {
    free(s);
    free(ok);
    return (void*)1;
  }
  for (;;) {
    pthread_mutex_lock(&J->mu);
    long w = J->next;
    J->next += 16;
    pthread_mutex_unlock(&J->mu);
    if (w >= total) break;
    long w_end = w + 16 < total ? w + 16 : total;
    for (; w < w_end; ++w) {
      /* unit w = ((b * H) + h) * n_out + row */
      const int ri = (int)(w % n_out);
      const int h = (int)((w / n_out) % J->H);
      const int b = (int)(w / ((long)n_out * J->H));
      attn_one_row(J, b, h, ri, s, ok);
    }
  }
  free(s);
  free(ok);
  return NULL;
}

static int run_attn(attn_job* J, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  int started = 0, rc = ORC_OK;
  pthread_mutex_init(&J->mu, NULL);
  J->next = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, attn_worker, J) != 0) break;
    ++started;
  }
  if (attn_worker(J) != NULL) rc = ORC_ENOMEM;
  for (int t = 1; t <= started; ++t) {
    void* ret = NULL;
    pthread_join(th[t], &ret);
    if (ret != NULL) rc = ORC_ENOMEM;
  }
  pthread_mutex_destroy(&J->mu);
  return rc;
}

static int check_rule_args(int B, int S, int H, int D, int tile, int kv_begin, int kv_end) {
  if (B < 0 || S < 0 || H < 1 || D < 1) return ORC_EINVAL;
  if (tile < 1) return ORC_EINVAL;
  if (kv_begin < 0 || kv_end < kv_begin) return ORC_EINVAL;
  return ORC_OK;
}

/*
 * q, k, v: [B, S, H, D] fp64.  rows: NULL (all S query positions) or n_rows positions in [0, S).
 * o: [B, n_out, H, D], lse: [B, H, n_out] with n_out = rows ? n_rows : S.
 * block_mask: NULL or [H, ceil(S/tile), ceil(S/tile)] bytes, shared by all b.
 * Keys are those j with kv_begin <= j < min(kv_end, S); pass kv_begin = 0, kv_end = S for all.
 */
int orc_attn(const double* q, const double* k, const double* v, double* o, double* lse, int B, int S,
             int H, int D, int causal, const uint8_t* block_mask, int tile, int kv_begin, int kv_end,
             const int* rows, int n_rows, int nthreads) {
  int rc = check_rule_args(B, S, H, D, tile, kv_begin, kv_end);
  if (rc) return rc;
  if (rows)
    for (int r = 0; r < n_rows; ++r)
      if (rows[r] < 0 || rows[r] >= S) return ORC_EINVAL;
  attn_job J;
  memset(&J, 0, sizeof(J));
  J.q = q; J.k = k; J.v = v; J.o = o; J.lse = lse; J.probs = NULL;
  J.B = B; J.S = S; J.H = H; J.D = D;
  J.rule.S = S; J.rule.H = H; J.rule.causal = causal; J.rule.tile = tile;
  J.rule.kv_begin = kv_begin; J.rule.kv_end = kv_end;
  J.rule.n_tiles = (S + tile - 1) / tile; J.rule.block_mask = block_mask;
  J.rows = rows; J.n_rows = rows ? n_rows : S;
  if ((long)B * H * (rows ? n_rows : S) == 0) return ORC_OK;
  return run_attn(&J, nthreads);
}

/* Same definition; also writes probs [B, H, S, S] (row i: p_j over all key positions j). */
int orc_attn_probs(const double* q, const double* k, const double* v, double* o, double* lse,
                   double* probs, int B, int S, int H, int D, int causal, const uint8_t* block_mask,
                   int tile, int kv_begin, int kv_end) {
  int rc = check_rule_args(B, S, H, D, tile, kv_begin, kv_end);
  if (rc) return rc;
  attn_job J;
  memset(&J, 0, sizeof(J));
  J.q = q; J.k = k; J.v = v; J.o = o; J.lse = lse; J.probs = probs;
  J.B = B; J.S = S; J.H = H; J.D = D;
  J.rule.S = S; J.rule.H = H; J.rule.causal = causal; J.rule.tile = tile;
  J.rule.kv_begin = kv_begin; J.rule.kv_end = kv_end;
  J.rule.n_tiles = (S + tile - 1) / tile; J.rule.block_mask = block_mask;
  J.rows = NULL; J.n_rows = S;
  if ((long)B * H * S == 0) return ORC_OK;
  return run_attn(&J, 1);
}

/* ------------------------------------------------------------------------------------------------ */
/* Re-merge of KV-block partials                                                                      */
/* ------------------------------------------------------------------------------------------------ */
/*
 * o_parts[b_]: [B, S, H, D] fp64, lse_parts[b_]: [B, H, S] fp64, for b_ in [0, n).
 * o: [B, S, H, D], lse: [B, H, S].
 */
int orc_merge(const double* const* o_parts, const double* const* lse_parts, int n, double* o,
              double* lse, int B, int S, int H, int D) {
  if (n < 1 || B < 0 || S < 0 || H < 1 || D < 1) return ORC_EINVAL;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s) {
        const size_t li = ((size_t)b * H + h) * S + s;
        const size_t oi = (((size_t)b * S + s) * H + h) * D;
        double M = -INFINITY;
        for (int p = 0; p < n; ++p)
          if (lse_parts[p][li] > M) M = lse_parts[p][li];
        if (M == -INFINITY) {
          for (int d = 0; d < D; ++d) o[oi + d] = 0.0;
          lse[li] = -INFINITY;
          continue;
        }
        double sum = 0.0;
        for (int p = 0; p < n; ++p)
          if (lse_parts[p][li] != -INFINITY) sum += exp(lse_parts[p][li] - M);
        const double L = M + log(sum);
        for (int d = 0; d < D; ++d) o[oi + d] = 0.0;
        for (int p = 0; p < n; ++p) {
          if (lse_parts[p][li] == -INFINITY) continue;
          const double w = exp(lse_parts[p][li] - L);
          for (int d = 0; d < D; ++d) o[oi + d] += w * o_parts[p][oi + d];
        }
        lse[li] = L;
      }
  return ORC_OK;
}

/* ------------------------------------------------------------------------------------------------ */
/* Ulysses relayout between P rank buffers                                                            */
/* ------------------------------------------------------------------------------------------------ */
/*
 * seq -> head: in_ranks[r] is [B, S/P, H, D], out_ranks[r] is [B, S, H/P, D]; elem_bytes per element.
 */
int orc_seq_to_head(const void* const* in_ranks, void* const* out_ranks, int P, int B, int S, int H,
                    int D, int elem_bytes) {
  if (P < 1 || B < 0 || S < 0 || H < 1 || D < 1 || elem_bytes < 1) return ORC_EINVAL;
  if (S % P || H % P) return ORC_EINVAL;
  const int Sl = S / P, Hl = H / P;
  for (int r = 0; r < P; ++r)
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < S; ++s)
        for (int hh = 0; hh < Hl; ++hh) {
          const int src_rank = s / Sl, src_s = s % Sl, src_h = r * Hl + hh;
          const unsigned char* src = (const unsigned char*)in_ranks[src_rank] +
                                     ((((size_t)b * Sl + src_s) * H + src_h) * D) * elem_bytes;
          unsigned char* dst =
              (unsigned char*)out_ranks[r] + ((((size_t)b * S + s) * Hl + hh) * D) * elem_bytes;
          for (size_t e = 0; e < (size_t)D * elem_bytes; ++e) dst[e] = src[e];
        }
  return ORC_OK;
}

/* head -> seq: in_ranks[r] is [B, S, H/P, D], out_ranks[r] is [B, S/P, H, D]; inverse of the above. */
int orc_head_to_seq(const void* const* in_ranks, void* const* out_ranks, int P, int B, int S, int H,
                    int D, int elem_bytes) {
  if (P < 1 || B < 0 || S < 0 || H < 1 || D < 1 || elem_bytes < 1) return ORC_EINVAL;
  if (S % P || H % P) return ORC_EINVAL;
  const int Sl = S / P, Hl = H / P;
  for (int r = 0; r < P; ++r)
    for (int b = 0; b < B; ++b)
      for (int sl = 0; sl < Sl; ++sl)
        for (int h = 0; h < H; ++h) {
          const int src_rank = h / Hl, src_h = h % Hl, s = r * Sl + sl;
          const unsigned char* src = (const unsigned char*)in_ranks[src_rank] +
                                     ((((size_t)b * S + s) * Hl + src_h) * D) * elem_bytes;
          unsigned char* dst =
              (unsigned char*)out_ranks[r] + ((((size_t)b * Sl + sl) * H + h) * D) * elem_bytes;
          for (size_t e = 0; e < (size_t)D * elem_bytes; ++e) dst[e] = src[e];
        }
  return ORC_OK;
}

/*
 * The two local halves of the Ulysses all-to-all when the P ranks are P processes ("HCMS ...", abstract:
 * all-to-all based sequence parallelism).  Before the exchange, rank g cuts its sequence shard [B, S, H, D]
 * (S = its own positions) into P head groups, one per destination rank:
 *   split_heads:  out_r[b, s, h', :] = in[b, s, r*H/P + h', :]          (out_r is [B, S, H/P, D])
 * after the way back it joins the P head groups it received into its sequence shard:
 *   merge_heads:  out[b, s, r*H/P + h', :] = in_r[b, s, h', :]
 * Byte copies, element by element.
 */
int orc_split_heads(const void* in, void* const* out_ranks, int P, int B, int S, int H, int D, int elem_bytes) {
  if (P < 1 || B < 0 || S < 0 || H < 1 || D < 1 || elem_bytes < 1 || H % P) return ORC_EINVAL;
  const int Hl = H / P;
  for (int r = 0; r < P; ++r)
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < S; ++s)
        for (int hh = 0; hh < Hl; ++hh) {
          const unsigned char* src =
              (const unsigned char*)in + ((((size_t)b * S + s) * H + r * Hl + hh) * D) * elem_bytes;
          unsigned char* dst = (unsigned char*)out_ranks[r] + ((((size_t)b * S + s) * Hl + hh) * D) * elem_bytes;
          for (size_t e = 0; e < (size_t)D * elem_bytes; ++e) dst[e] = src[e];
        }
  return ORC_OK;
}

int orc_merge_heads(const void* const* in_ranks, void* out, int P, int B, int S, int H, int D, int elem_bytes) {
  if (P < 1 || B < 0 || S < 0 || H < 1 || D < 1 || elem_bytes < 1 || H % P) return ORC_EINVAL;
  const int Hl = H / P;
  for (int r = 0; r < P; ++r)
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < S; ++s)
        for (int hh = 0; hh < Hl; ++hh) {
          const unsigned char* src =
              (const unsigned char*)in_ranks[r] + ((((size_t)b * S + s) * Hl + hh) * D) * elem_bytes;
          unsigned char* dst = (unsigned char*)out + ((((size_t)b * S + s) * H + r * Hl + hh) * D) * elem_bytes;
          for (size_t e = 0; e < (size_t)D * elem_bytes; ++e) dst[e] = src[e];
        }
  return ORC_OK;
}

/* ------------------------------------------------------------------------------------------------ */
/* Compacted tile list of a block mask                                                                */
/* ------------------------------------------------------------------------------------------------ */
/*
 * mask: [H, Tq, Tk] bytes, nonzero = keep.  row_ptr: [H*Tq + 1], col_idx: [nnz] (capacity cap).
 * Row (h, i) lists the kept key tiles j in increasing order.  Returns ORC_EINVAL if cap is too small.
 */
/* ------------------------------------------------------------------------------------------------ */
/* Backward: one (batch, head) per task.                                                            */
/* ------------------------------------------------------------------------------------------------ */
typedef struct {
  const double *q, *k, *v, *dout;
  double *dq, *dk, *dv;
  int B, S, H, D, causal;
  int next;
  pthread_mutex_t mu;
} bwd_job;

static void bwd_head(bwd_job* J, int b, int h) {
  const int S = J->S, H = J->H, D = J->D;
  const double scale = 1.0 / sqrt((double)D);
#define IDX(t, i, d) ((((size_t)(b) * S + (i)) * H + (h)) * D + (d))
  double* p = (double*)malloc(sizeof(double) * (size_t)S);
  double* o = (double*)malloc(sizeof(double) * (size_t)D);
  for (int j = 0; j < S; ++j)
    for (int d = 0; d < D; ++d) {
      J->dk[IDX(k, j, d)] = 0.0;
      J->dv[IDX(v, j, d)] = 0.0;
    }
  for (int i = 0; i < S; ++i) {
    const int n = J->causal ? i + 1 : S;  /* allowed keys 0 .. n-1 */
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
      double s = 0.0;
      for (int d = 0; d < D; ++d) s += J->q[IDX(q, i, d)] * J->k[IDX(k, j, d)];
      p[j] = s * scale;
      if (p[j] > m) m = p[j];
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
      p[j] = exp(p[j] - m);
      l += p[j];
    }
    for (int j = 0; j < n; ++j) p[j] /= l;
    for (int d = 0; d < D; ++d) {
      double acc = 0.0;
      for (int j = 0; j < n; ++j) acc += p[j] * J->v[IDX(v, j, d)];
      o[d] = acc;
    }
    double delta = 0.0;
    for (int d = 0; d < D; ++d) delta += J->dout[IDX(dout, i, d)] * o[d];
    for (int d = 0; d < D; ++d) J->dq[IDX(q, i, d)] = 0.0;
    for (int j = 0; j < n; ++j) {
      double dp = 0.0;
      for (int d = 0; d < D; ++d) dp += J->dout[IDX(dout, i, d)] * J->v[IDX(v, j, d)];
      const double ds = p[j] * (dp - delta);
      for (int d = 0; d < D; ++d) {
        J->dq[IDX(q, i, d)] += ds * J->k[IDX(k, j, d)] * scale;
        J->dk[IDX(k, j, d)] += ds * J->q[IDX(q, i, d)] * scale;
        J->dv[IDX(v, j, d)] += p[j] * J->dout[IDX(dout, i, d)];
      }
    }
  }
#undef IDX
  free(p);
  free(o);
}

static void* bwd_worker(void* arg) {
  bwd_job* J = (bwd_job*)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    const int t = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (t >= J->B * J->H) break;
    bwd_head(J, t / J->H, t % J->H);
  }
  return NULL;
}

int orc_attn_bwd(const double* q, const double* k, const double* v, const double* dout, double* dq, double* dk,
                 double* dv, int B, int S, int H, int D, int causal, int nthreads) {
  if (B < 1 || S < 1 || H < 1 || D < 1 || (causal != 0 && causal != 1)) return ORC_EINVAL;
  bwd_job J = {q, k, v, dout, dq, dk, dv, B, S, H, D, causal, 0, PTHREAD_MUTEX_INITIALIZER};
  if (nthreads < 1) nthreads = 1;
  if (nthreads > B * H) nthreads = B * H;
  pthread_t th[256];
  if (nthreads > 256) nthreads = 256;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, bwd_worker, &J) != 0) break;
    ++started;
  }
  if (started == 0) bwd_worker(&J);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
  return ORC_OK;
}

int orc_tile_list(const uint8_t* mask, int H, int Tq, int Tk, int32_t* row_ptr, int32_t* col_idx,
                  long cap) {
  if (H < 1 || Tq < 0 || Tk < 0) return ORC_EINVAL;
  long nnz = 0;
  row_ptr[0] = 0;
  for (int h = 0; h < H; ++h)
    for (int i = 0; i < Tq; ++i) {
      for (int j = 0; j < Tk; ++j) {
        if (!mask[((size_t)h * Tq + i) * Tk + j]) continue;
        if (nnz >= cap) return ORC_EINVAL;
        col_idx[nnz++] = j;
      }
      row_ptr[(size_t)h * Tq + i + 1] = (int32_t)nnz;
    }
  return ORC_OK;
}
