/*
 * tls_oracle.c -- TEST INFRASTRUCTURE ONLY (the oracle).
 *
 * A plain, slow, fp64 CPU restatement of the per-decode-step two-level sparse
 * attention described for AsyncTLS ("AsyncTLS: Efficient Generative LLM
 * Inference with Asynchronous Two-level Sparse Attention": arXiv abstract on
 * mlsanity.com; gist.science explainers (de) section 2.A and (es) section 2.A).
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * this file.  It shares no code, header, table or helper with the CUDA library
 * and includes nothing from it.
 *
 * Every step is written from its definition, in the order the pages give:
 *   1. per-block channel max / min of the keys (compressed block summary),
 *   2. Quest-style block bound from that summary, summed over the query heads
 *      that share the KV head,
 *   3. top-K_b blocks,
 *   4. label-channel (Double-Sparsity style) token scores inside those blocks,
 *   5. top-K_t tokens,
 *   6. exact softmax attention over the gathered K/V of those tokens.
 * Readings where the pages are silent (sum over heads, ties to the lower
 * index, clamping, empty selections) are stated at each function.
 *
 * Inputs are read in their stored type (fp32, or bf16 bits) and widened
 * exactly to double; all arithmetic is double, except the codes and scales of
 * the quantised label slab (a variant), which are integers and scales decided
 * in fp32 (ora_quantize_labels).  Tensor layouts:
 *   q    [B][H_q][d_qk]           K [B][H_kv][max_ctx][d_qk]
 *   V    [B][H_kv][max_ctx][d_v]  (or V = K[..., :d_v] when v_is_k_prefix)
 *   query head h uses KV head h / (H_q / H_kv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int batch, n_q_heads, n_kv_heads, d_qk, d_v, v_is_k_prefix;
  int block_size, n_label, k_b, k_t, max_ctx, dtype; /* dtype 0: fp32, 1: bf16 bits */
  int block_agg;                                      /* 0: sum of the heads' bounds, 1: their max */
  int slab_bits;                                      /* 0: exact label channels, 8: int8 codes */
  double softmax_scale;
} ora_shape;

/* ---- input widening (exact) ------------------------------------------- */
static double ora_in(const void *base, int dtype, size_t i) {
  if (dtype == 0) return (double)((const float *)base)[i];
  uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static int ora_nblocks_max(const ora_shape *s) { return (s->max_ctx + s->block_size - 1) / s->block_size; }
static int ora_nblocks(const ora_shape *s, int seq_len) { return (seq_len + s->block_size - 1) / s->block_size; }

int ora_abi_version(void) { return 1; }

/* ---- step 1: per-block channel max / min -------------------------------
 * gist.science (de) section 2.A, "Stufe 1": each block is summarised by the
 * per-channel maximum and minimum of its keys.  Only the block's valid tokens
 * (t < seq_len) count; a partial last block is summarised over its valid part.
 * meta: [B][H_kv][N_b_max][2][d_qk], row 0 = max, row 1 = min.  Blocks with no
 * valid token are filled with NAN (never read by later steps). */
void ora_build_meta(const ora_shape *s, const void *K, const int32_t *seq_lens, double *meta) {
  const int nbm = ora_nblocks_max(s), d = s->d_qk;
  for (int b = 0; b < s->batch; ++b)
    for (int g = 0; g < s->n_kv_heads; ++g)
      for (int j = 0; j < nbm; ++j) {
        double *mx = meta + ((((size_t)b * s->n_kv_heads + g) * nbm + j) * 2) * d;
        double *mn = mx + d;
        int t0 = j * s->block_size, t1 = t0 + s->block_size;
        if (t1 > seq_lens[b]) t1 = seq_lens[b];
        for (int i = 0; i < d; ++i) {
          if (t0 >= t1) { mx[i] = NAN; mn[i] = NAN; continue; }
          double hi = -INFINITY, lo = INFINITY;
          for (int t = t0; t < t1; ++t) {
            double v = ora_in(K, s->dtype, (((size_t)b * s->n_kv_heads + g) * s->max_ctx + t) * d + i);
            if (v > hi) hi = v;
            if (v < lo) lo = v;
          }
          mx[i] = hi;
          mn[i] = lo;
        }
      }
}

/* ---- step 2: block bound -------------------------------------------------
 * gist.science (es) section 2.A.1 ("basado en Quest") and (de) section 2.A:
 * for a query head h and block j, the largest value q_h . k can take for any
 * key k inside the box [min_j, max_j] is
 *     u_{h,j} = sum_i max(q_{h,i} * max_{j,i}, q_{h,i} * min_{j,i}).
 * The heads sharing one KV head (GQA) or one latent (MLA) share one selection;
 * their bounds are added:  score_j = sum_{h in group} u_{h,j}  (block_agg 0),
 * or, as the variant, the largest one is taken: score_j = max_h u_{h,j}
 * (block_agg 1).
 * score: [B][H_kv][N_b_max]; blocks at or beyond ceil(seq_len / bs) get -inf. */
void ora_block_scores(const ora_shape *s, const void *q, const double *meta, const int32_t *seq_lens,
                      double *score) {
  const int nbm = ora_nblocks_max(s), d = s->d_qk, G = s->n_q_heads / s->n_kv_heads;
  for (int b = 0; b < s->batch; ++b)
    for (int g = 0; g < s->n_kv_heads; ++g) {
      const int nb = ora_nblocks(s, seq_lens[b]);
      for (int j = 0; j < nbm; ++j) {
        double *out = score + ((size_t)b * s->n_kv_heads + g) * nbm + j;
        if (j >= nb) { *out = -INFINITY; continue; }
        const double *mx = meta + ((((size_t)b * s->n_kv_heads + g) * nbm + j) * 2) * d;
        const double *mn = mx + d;
        double total = s->block_agg ? -INFINITY : 0.0;
        for (int hh = 0; hh < G; ++hh) {
          const int h = g * G + hh;
          double u = 0.0;
          for (int i = 0; i < d; ++i) {
            double qi = ora_in(q, s->dtype, ((size_t)b * s->n_q_heads + h) * d + i);
            double a = qi * mx[i], c = qi * mn[i];
            u += (a > c) ? a : c;
          }
          if (s->block_agg) total = (u > total) ? u : total;
          else total += u;
        }
        *out = total;
      }
    }
}

/* ---- steps 3 and 5: top-k ------------------------------------------------
 * gist.science (es) section 2.A: "the K_b most relevant blocks" / "the K_t most
 * salient tokens".  Reading: rank by score descending; equal scores rank the
 * lower id first; keep the first min(k, n) entries; return their ids in
 * ascending order, padded with -1 up to out_cap.  When decide_f32 is set the
 * scores are first rounded to fp32 (the precision a caller decides in), so that
 * ties are judged in that precision. */
typedef struct { double s; int32_t id; } ora_pair;

static int ora_pair_cmp(const void *pa, const void *pb) {
  const ora_pair *a = (const ora_pair *)pa, *b = (const ora_pair *)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->id < b->id) ? -1 : (a->id > b->id);
}

static int ora_int_cmp(const void *pa, const void *pb) {
  int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
  return (a > b) - (a < b);
}

int ora_topk(const double *score, const int32_t *ids, int n, int k, int decide_f32, int32_t *out, int out_cap) {
  ora_pair *p = (ora_pair *)malloc(sizeof(ora_pair) * (size_t)(n > 0 ? n : 1));
  for (int i = 0; i < n; ++i) {
    p[i].s = decide_f32 ? (double)(float)score[i] : score[i];
    p[i].id = ids ? ids[i] : i;
  }
  qsort(p, (size_t)n, sizeof(ora_pair), ora_pair_cmp);
  int m = k < n ? k : n;
  if (m > out_cap) m = out_cap;
  if (m < 0) m = 0;
  for (int i = 0; i < m; ++i) out[i] = p[i].id;
  qsort(out, (size_t)m, sizeof(int32_t), ora_int_cmp);
  for (int i = m; i < out_cap; ++i) out[i] = -1;
  free(p);
  return m;
}

/* Block selection for every (b, kv head): top-K_b over the valid blocks.
 * block_idx: [B][H_kv][k_b]. */
void ora_select_blocks(const ora_shape *s, const double *score, const int32_t *seq_lens, int decide_f32,
                       int32_t *block_idx) {
  const int nbm = ora_nblocks_max(s);
  for (int b = 0; b < s->batch; ++b)
    for (int g = 0; g < s->n_kv_heads; ++g) {
      const size_t bg = (size_t)b * s->n_kv_heads + g;
      ora_topk(score + bg * nbm, NULL, ora_nblocks(s, seq_lens[b]), s->k_b, decide_f32, block_idx + bg * s->k_b,
               s->k_b);
    }
}

/* ---- step 4: label-channel token scores ----------------------------------
 * gist.science (de) section 2.A "Stufe 2" and (es) section 2.A.2: inside the
 * kept blocks every token is scored on a fixed subset L of r channels
 * ("label channels", Double Sparsity):
 *     s_t = sum_{h in group} sum_{c in L} q_{h,c} * K[t, c].
 * Candidate j of a (b, kv head) is token block_idx[j / bs] * bs + j % bs; it is
 * invalid when that block id is -1 or the token is at or beyond seq_len.
 * cand_score / cand_tok: [B][H_kv][k_b * bs]; invalid -> -inf / -1.
 * The scores are computed from K itself (not from any copied slab). */
void ora_quantize_labels(const ora_shape *s, const void *K, const int32_t *seq_lens, const int32_t *label_idx,
                         int8_t *codes, float *scales);

void ora_token_scores(const ora_shape *s, const void *q, const void *K, const int32_t *label_idx,
                      const int32_t *block_idx, const int32_t *seq_lens, double *cand_score, int32_t *cand_tok) {
  const int d = s->d_qk, G = s->n_q_heads / s->n_kv_heads, bs = s->block_size;
  const int C = s->k_b * bs;
  int8_t *codes = NULL;
  float *scales = NULL;
  if (s->slab_bits == 8) {  /* the quantised variant: K[t, L_c] is replaced by scale_c * code */
    codes = (int8_t *)malloc((size_t)s->batch * s->n_kv_heads * s->max_ctx * s->n_label);
    scales = (float *)malloc(sizeof(float) * (size_t)s->batch * s->n_kv_heads * s->n_label);
    ora_quantize_labels(s, K, seq_lens, label_idx, codes, scales);
  }
  for (int b = 0; b < s->batch; ++b)
    for (int g = 0; g < s->n_kv_heads; ++g) {
      const size_t bg = (size_t)b * s->n_kv_heads + g;
      for (int j = 0; j < C; ++j) {
        const int blk = block_idx[bg * s->k_b + j / bs];
        const int t = blk * bs + j % bs;
        double *os = cand_score + bg * C + j;
        int32_t *ot = cand_tok + bg * C + j;
        if (blk < 0 || t >= seq_lens[b]) { *os = -INFINITY; *ot = -1; continue; }
        double acc = 0.0;
        for (int hh = 0; hh < G; ++hh) {
          const int h = g * G + hh;
          for (int c = 0; c < s->n_label; ++c) {
            const int ch = label_idx[c];
            if (ch < 0 || ch >= d) continue;
            const double kv = codes ? (double)scales[bg * s->n_label + c] *
                                          (double)codes[(bg * s->max_ctx + t) * s->n_label + c]
                                    : ora_in(K, s->dtype, (bg * s->max_ctx + t) * d + ch);
            acc += ora_in(q, s->dtype, ((size_t)b * s->n_q_heads + h) * d + ch) * kv;
          }
        }
        *os = acc;
        *ot = t;
      }
    }
  free(codes);
  free(scales);
}

/* ---- the quantised label slab (variant) -----------------------------------
 * gist.science (de) section 2.A "Stufe 2": the token stage reads the label
 * channels "durch Quantisierung und Kanalauswahl" (through quantisation and
 * channel choice).  Reading: per sequence, KV head and label channel c, a
 * symmetric scale = max |K[t, L_c]| over the valid tokens / 127 and codes
 * round-half-even(K / scale) clamped to [-127, 127] (scale 0: codes 0).  The
 * scale and the codes are integers decided from fp32 values, so they are
 * computed in fp32 here (IEEE division, rint) as any implementation that
 * shares the reading must; the token score then uses scale * code in fp64.
 * codes: [B][H_kv][max_ctx][r] (rows >= seq_len: 0); scales: [B][H_kv][r]. */
void ora_quantize_labels(const ora_shape *s, const void *K, const int32_t *seq_lens, const int32_t *label_idx,
                         int8_t *codes, float *scales) {
  const int d = s->d_qk, r = s->n_label;
  for (int b = 0; b < s->batch; ++b)
    for (int g = 0; g < s->n_kv_heads; ++g) {
      const size_t bg = (size_t)b * s->n_kv_heads + g;
      const int L = seq_lens[b] < 0 ? 0 : (seq_lens[b] > s->max_ctx ? s->max_ctx : seq_lens[b]);
      for (int c = 0; c < r; ++c) {
        const int ch = label_idx[c];
        float maxabs = 0.0f;
        if (ch >= 0 && ch < d)
          for (int t = 0; t < L; ++t) {
            const size_t ki = (bg * s->max_ctx + t) * d + ch;
            const float v = (float)ora_in(K, s->dtype, ki);
            const float a = v < 0.0f ? -v : v;
            if (a > maxabs) maxabs = a;
          }
        const float scale = maxabs / 127.0f;
        scales[bg * r + c] = scale;
        for (int t = 0; t < s->max_ctx; ++t) {
          int code = 0;
          if (t < L && scale > 0.0f && ch >= 0 && ch < d) {
            const size_t ki = (bg * s->max_ctx + t) * d + ch;
            const float v = (float)ora_in(K, s->dtype, ki);
            const float qv = rintf(v / scale);
            code = qv > 127.0f ? 127 : (qv < -127.0f ? -127 : (int)qv);
          }
          codes[(bg * s->max_ctx + t) * r + c] = (int8_t)code;
        }
      }
    }
}

/* Token selection for every (b, kv head): top-K_t over the valid candidates,
 * ranked by score, ties to the lower token index.  token_idx: [B][H_kv][k_t]. */
void ora_select_tokens(const ora_shape *s, const double *cand_score, const int32_t *cand_tok, int decide_f32,
                       int32_t *token_idx) {
  const int C = s->k_b * s->block_size;
  double *sc = (double *)malloc(sizeof(double) * (size_t)C);
  int32_t *id = (int32_t *)malloc(sizeof(int32_t) * (size_t)C);
  for (int b = 0; b < s->batch; ++b)
    for (int g = 0; g < s->n_kv_heads; ++g) {
      const size_t bg = (size_t)b * s->n_kv_heads + g;
      int n = 0;
      for (int j = 0; j < C; ++j)
        if (cand_tok[bg * C + j] >= 0) { sc[n] = cand_score[bg * C + j]; id[n] = cand_tok[bg * C + j]; ++n; }
      ora_topk(sc, id, n, s->k_t, decide_f32, token_idx + bg * s->k_t, s->k_t);
    }
  free(sc);
  free(id);
}

/* ---- step 6: exact attention over the selected tokens --------------------
 * gist.science (es) section 2.A.2: the final attention is computed at token
 * precision over the K_t selected tokens.  For each query head h:
 *     a_t = tau * q_h . K[t, :]   (t in the selection S)
 *     p_t = exp(a_t - max a) / sum_t' exp(a_t' - max a)
 *     o_h = sum_t p_t V[t, :],    lse_h = log sum_t exp(a_t)
 * Entries of token_idx that are -1 (or beyond max_ctx) are skipped.  An empty selection gives
 * o_h = 0 and lse_h = -inf.  out: [B][H_q][d_v], lse: [B][H_q]. */
void ora_attention(const ora_shape *s, const void *q, const void *K, const void *V, const int32_t *token_idx,
                   double *out, double *lse) {
  const int d = s->d_qk, dv = s->d_v, G = s->n_q_heads / s->n_kv_heads;
  const void *Vb = s->v_is_k_prefix ? K : V;
  const int vstride = s->v_is_k_prefix ? d : dv;
  double *a = (double *)malloc(sizeof(double) * (size_t)(s->k_t > 0 ? s->k_t : 1));
  for (int b = 0; b < s->batch; ++b)
    for (int g = 0; g < s->n_kv_heads; ++g) {
      const size_t bg = (size_t)b * s->n_kv_heads + g;
      const int32_t *sel = token_idx + bg * s->k_t;
      for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        double *o = out + ((size_t)b * s->n_q_heads + h) * dv;
        for (int c = 0; c < dv; ++c) o[c] = 0.0;
        double mx = -INFINITY;
        for (int j = 0; j < s->k_t; ++j) {
          if (sel[j] < 0 || sel[j] >= s->max_ctx) continue;
          double acc = 0.0;
          for (int i = 0; i < d; ++i)
            acc += ora_in(q, s->dtype, ((size_t)b * s->n_q_heads + h) * d + i) *
                   ora_in(K, s->dtype, (bg * s->max_ctx + sel[j]) * d + i);
          a[j] = s->softmax_scale * acc;
          if (a[j] > mx) mx = a[j];
        }
        if (mx == -INFINITY) { lse[(size_t)b * s->n_q_heads + h] = -INFINITY; continue; }
        double l = 0.0;
        for (int j = 0; j < s->k_t; ++j) {
          if (sel[j] < 0 || sel[j] >= s->max_ctx) continue;
          const double p = exp(a[j] - mx);
          l += p;
          for (int c = 0; c < dv; ++c) o[c] += p * ora_in(Vb, s->dtype, (bg * s->max_ctx + sel[j]) * vstride + c);
        }
        for (int c = 0; c < dv; ++c) o[c] /= l;
        lse[(size_t)b * s->n_q_heads + h] = mx + log(l);
      }
    }
  free(a);
}

/* ---- one whole decode step (steps 2-6, given the step-1 summary) --------
 * Chains the functions above.  Any output pointer may be NULL except the
 * ones a later step needs internally (those are allocated here).  Used for
 * the CPU baseline timing and for end-to-end parity. */
void ora_decode_step(const ora_shape *s, const void *q, const void *K, const void *V, const double *meta,
                     const int32_t *seq_lens, const int32_t *label_idx, int decide_f32, int32_t *block_idx_out,
                     int32_t *token_idx_out, double *out, double *lse) {
  const size_t BG = (size_t)s->batch * s->n_kv_heads;
  const size_t C = (size_t)s->k_b * s->block_size;
  double *score = (double *)malloc(sizeof(double) * BG * (size_t)ora_nblocks_max(s));
  int32_t *bidx = block_idx_out ? block_idx_out : (int32_t *)malloc(sizeof(int32_t) * BG * (size_t)s->k_b);
  double *cs = (double *)malloc(sizeof(double) * BG * C);
  int32_t *ct = (int32_t *)malloc(sizeof(int32_t) * BG * C);
  int32_t *tidx = token_idx_out ? token_idx_out : (int32_t *)malloc(sizeof(int32_t) * BG * (size_t)s->k_t);
  ora_block_scores(s, q, meta, seq_lens, score);
  ora_select_blocks(s, score, seq_lens, decide_f32, bidx);
  ora_token_scores(s, q, K, label_idx, bidx, seq_lens, cs, ct);
  ora_select_tokens(s, cs, ct, decide_f32, tidx);
  if (out && lse) ora_attention(s, q, K, V, tidx, out, lse);
  free(score);
  free(cs);
  free(ct);
  if (!block_idx_out) free(bidx);
  if (!token_idx_out) free(tidx);
}
