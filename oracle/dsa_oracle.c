/*
 * CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  The GPU product path never calls it,
 * and it shares no code, header, table or helper with the CUDA sources.
 *
 * Plain fp64 loops, one query row per call, written straight from the
 * definitions on the pages:
 *   - indexer score, "DeepSeek-V3.2" analysis page (PaperTrace), sec. 1.1, eq. (1)
 *   - top-k selection set S_t, same page, sec. 1.1, eq. (2) and eq. (4)
 *   - attention over the selected latents in MLA's MQA mode, same page,
 *     sec. 1.1 eq. (2) and the MQA-mode paragraph (shared 576-d latent,
 *     512 value dims); renormalised form, sec. 5.2 eq. (19)
 *   - target distribution p: main-attention probabilities summed over heads
 *     and L1-normalised, "DSA Continued Pre-Training" page, Stage 1
 *   - sparse-stage indexer loss L^I = sum_t KL(p[t,S_t] || Softmax(I[t,S_t])),
 *     "DSA Continued Pre-Training" page, Stage 2, and the analysis page eq. (4)
 *   - dense warm-up loss L^I = sum_t KL(p[t,:] || Softmax(I[t,:])) over every s <= t, with p
 *     the dense main attention summed over heads and L1-normalised, "DSA Continued
 *     Pre-Training" page, Stage 1, and the analysis page eq. (3)
 *   - masked MHA for short prefill: MLA's MHA mode (per-head decompressed keys and values) with
 *     every position outside S_t masked, which gives DSA's attention (V3.2-Exp page, sec. 3,
 *     inference costs; the analysis page's MHA/MQA-mode paragraph, Fig. 7)
 *   - HISA's two-stage retrieval: blocks scored by a block representative, the best blocks'
 *     tokens scored exactly, top-k among them (analysis page, sec. 5.3, eq. (24)-(25) and the
 *     block-mean paragraph)
 *   - the gradient of one row's L^I with respect to the indexer's inputs q_I, w and k_I (the
 *     indexer is trained from L^I alone, on a detached input: "DSA Continued Pre-Training",
 *     Stage 2), with the selected set held fixed (top-k is piecewise constant)
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - causal visibility includes the query's own position: s <= t;
 *   - the indexer has no extra scale or dequantisation factors (eq. (1) as printed);
 *   - masked scores (s > t) are -infinity;
 *   - ties in top-k go to the smaller key index;
 *   - value = latent dims [0, d_v), key = all d_qk latent dims;
 *   - "main attention scores" are post-softmax probabilities;
 *   - KL uses natural logs, 0 * ln 0 = 0, and is summed (not averaged) over t.
 *
 * Parity pins: every function here is pinned by a CPU test against a value or
 * property fixed independently of this file (hand-worked example, library
 * routines in fp64, closed forms, invariants).  None is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

/* ---- storage decoders ------------------------------------------------------------------- */

/* OCP FP8 E4M3 (fn variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 * exponent 15 with mantissa 7 is NaN; exponent 0 is subnormal m/8 * 2^-6. */
double ref_e4m3_to_double(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 0xF;
  int m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* bfloat16 = the top 16 bits of an IEEE binary32. */
double ref_bf16_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---- a1: lightning indexer, eq. (1) ----------------------------------------------------- */
/* I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]) for s <= t; -inf for s > t.
 * q_row: [H_I][d_I] e4m3 of this query; k_seq: [Lk][d_I] e4m3 of its sequence;
 * w_row: [H_I]; out: [Lk]. */
void ref_indexer_row(const uint8_t* q_row, const uint8_t* k_seq, const float* w_row, int Lk,
                     int t, int H_I, int d_I, double* out) {
  for (int s = 0; s < Lk; ++s) {
    if (s > t) {
      out[s] = -INFINITY;
      continue;
    }
    double score = 0.0;
    for (int j = 0; j < H_I; ++j) {
      double dot = 0.0;
      for (int d = 0; d < d_I; ++d)
        dot += ref_e4m3_to_double(q_row[j * d_I + d]) * ref_e4m3_to_double(k_seq[(int64_t)s * d_I + d]);
      double relu = dot > 0.0 ? dot : 0.0;
      score += (double)w_row[j] * relu;
    }
    out[s] = score;
  }
}

/* ---- a2: top-k selection S_t, eq. (2)/(4) ----------------------------------------------- */
typedef struct {
  double score;
  int32_t s;
} scored_t;

static int by_score_desc_then_index(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->s < y->s) ? -1 : (x->s > y->s);
}

/* S_t = the min(k, t+1) positions s <= t with the largest scores; ties -> smaller s.
 * Full sort of all candidates, then the first entries.  idx[0..n) holds them in ascending
 * position order, idx[n..k) = -1.  Returns n. */
int ref_topk_row(const double* scores, int t, int k, int32_t* idx) {
  int n_cand = t + 1;
  scored_t* c = (scored_t*)malloc(sizeof(scored_t) * (size_t)n_cand);
  for (int s = 0; s < n_cand; ++s) {
    c[s].score = scores[s];
    c[s].s = s;
  }
  qsort(c, (size_t)n_cand, sizeof(scored_t), by_score_desc_then_index);
  int n = n_cand < k ? n_cand : k;
  /* mark the chosen positions, then list them in ascending order */
  unsigned char* chosen = (unsigned char*)calloc((size_t)n_cand, 1);
  for (int i = 0; i < n; ++i) chosen[c[i].s] = 1;
  int w = 0;
  for (int s = 0; s < n_cand; ++s)
    if (chosen[s]) idx[w++] = s;
  for (int i = n; i < k; ++i) idx[i] = -1;
  free(chosen);
  free(c);
  return n;
}

/* ---- a3/a4: attention in MQA mode over the selected latents ----------------------------- */
/* For each head h: z_i = scale * <q[h,:], c[idx_i,:]> over all d_qk dims (valid i only),
 * P_h,i = softmax_i(z), o[h,:] = sum_i P_h,i * c[idx_i, 0:d_v], lse[h] = ln sum_i exp(z_i).
 * q_row: [H][d_qk] bf16; kv_seq: [Lk][d_qk] bf16; idx: [k] (-1 = empty slot).
 * out: [H][d_v]; lse: [H] (nullable); P: [H][k] (nullable, 0 for empty slots). */
void ref_sparse_mla_row(const uint16_t* q_row, const uint16_t* kv_seq, const int32_t* idx, int k,
                        int H, int d_qk, int d_v, double scale, double* out, double* lse,
                        double* P) {
  double* z = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  for (int h = 0; h < H; ++h) {
    double m = -INFINITY;
    for (int i = 0; i < k; ++i) {
      if (idx[i] < 0) continue;
      double dot = 0.0;
      for (int d = 0; d < d_qk; ++d)
        dot += ref_bf16_to_double(q_row[h * d_qk + d]) *
               ref_bf16_to_double(kv_seq[(int64_t)idx[i] * d_qk + d]);
      z[i] = scale * dot;
      if (z[i] > m) m = z[i];
    }
    double denom = 0.0;
    for (int i = 0; i < k; ++i)
      if (idx[i] >= 0) denom += exp(z[i] - m);
    for (int e = 0; e < d_v; ++e) out[h * d_v + e] = 0.0;
    for (int i = 0; i < k; ++i) {
      double p = idx[i] >= 0 ? exp(z[i] - m) / denom : 0.0;
      if (P) P[(int64_t)h * k + i] = p;
      if (idx[i] < 0) continue;
      for (int e = 0; e < d_v; ++e)
        out[h * d_v + e] += p * ref_bf16_to_double(kv_seq[(int64_t)idx[i] * d_qk + e]);
    }
    if (lse) lse[h] = m + log(denom);
  }
  free(z);
}

/* Target distribution over S_t ("DSA Continued Pre-Training", Stage 1 and Stage 2):
 * main-attention probabilities summed over all heads, then L1-normalised along the
 * selected positions.  P: [H][k] from ref_sparse_mla_row.  p: [k], 0 for empty slots. */
void ref_p_sel_row(const double* P, const int32_t* idx, int k, int H, double* p) {
  double total = 0.0;
  for (int i = 0; i < k; ++i) {
    double acc = 0.0;
    if (idx[i] >= 0)
      for (int h = 0; h < H; ++h) acc += P[(int64_t)h * k + i];
    p[i] = acc;
    total += acc;
  }
  for (int i = 0; i < k; ++i) p[i] = total > 0.0 ? p[i] / total : 0.0;
}

/* ---- a5: sparse-stage indexer loss, one row of eq. (4) ---------------------------------- */
/* KL(p || q) with q = Softmax(I[t, S_t]) over the valid selected positions:
 * sum_i p_i (ln p_i - ln q_i), ln q_i = I_i - ln sum_j exp(I_j); terms with p_i = 0 are 0. */
double ref_kl_row(const double* scores_row, const int32_t* idx, const double* p, int k) {
  double m = -INFINITY;
  for (int i = 0; i < k; ++i)
    if (idx[i] >= 0 && scores_row[idx[i]] > m) m = scores_row[idx[i]];
  double denom = 0.0;
  for (int i = 0; i < k; ++i)
    if (idx[i] >= 0) denom += exp(scores_row[idx[i]] - m);
  double log_z = m + log(denom);
  double kl = 0.0;
  for (int i = 0; i < k; ++i) {
    if (idx[i] < 0 || p[i] == 0.0) continue;
    double log_q = scores_row[idx[i]] - log_z;
    kl += p[i] * (log(p[i]) - log_q);
  }
  return kl;
}

/* ---- f3: dense warm-up target and loss, eq. (3) ------------------------------------------- */
/* Target of the dense warm-up ("DSA Continued Pre-Training", Stage 1): for query t, the dense
 * main attention over every s <= t (MQA mode: logits scale * <q[h,:], c[s,:]> over all d_qk
 * latent dims, softmax over s per head), summed over the H heads and L1-normalised along s.
 * q_row: [H][d_qk] bf16; kv_seq: [>= t+1][d_qk] bf16; p: [t+1]. */
void ref_dense_p_row(const uint16_t* q_row, const uint16_t* kv_seq, int t, int H, int d_qk,
                     double scale, double* p) {
  int n = t + 1;
  double* z = (double*)malloc(sizeof(double) * (size_t)n);
  for (int s = 0; s < n; ++s) p[s] = 0.0;
  for (int h = 0; h < H; ++h) {
    double m = -INFINITY;
    for (int s = 0; s < n; ++s) {
      double dot = 0.0;
      for (int d = 0; d < d_qk; ++d)
        dot += ref_bf16_to_double(q_row[h * d_qk + d]) * ref_bf16_to_double(kv_seq[(int64_t)s * d_qk + d]);
      z[s] = scale * dot;
      if (z[s] > m) m = z[s];
    }
    double denom = 0.0;
    for (int s = 0; s < n; ++s) denom += exp(z[s] - m);
    for (int s = 0; s < n; ++s) p[s] += exp(z[s] - m) / denom;  /* this head's probabilities */
  }
  double total = 0.0;
  for (int s = 0; s < n; ++s) total += p[s];
  for (int s = 0; s < n; ++s) p[s] /= total;
  free(z);
}

/* One row of eq. (3): KL(p[t,:] || Softmax(I[t,:])) over every s <= t, natural log,
 * 0 * ln 0 = 0.  scores_row: I[t, 0..t]; p: [t+1]. */
double ref_dense_kl_row(const double* scores_row, int t, const double* p) {
  int n = t + 1;
  double m = -INFINITY;
  for (int s = 0; s < n; ++s)
    if (scores_row[s] > m) m = scores_row[s];
  double denom = 0.0;
  for (int s = 0; s < n; ++s) denom += exp(scores_row[s] - m);
  double log_z = m + log(denom);
  double kl = 0.0;
  for (int s = 0; s < n; ++s) {
    if (p[s] == 0.0) continue;
    kl += p[s] * (log(p[s]) - (scores_row[s] - log_z));
  }
  return kl;
}

/* ---- f4: masked MHA (MLA's MHA mode restricted to S_t) ------------------------------------ */
/* For each head h: z_s = scale * <q[h,:], k[s,h,:]> over the selected positions s of idx (-1 =
 * empty slot), P = softmax(z), out[h,:] = sum_s P_s v[s,h,:], lse[h] = ln sum_s exp(z_s); a head
 * with no selected position gets out = 0, lse = -inf.  Real (fp64) inputs: q [H][dqk],
 * k_seq [L][H][dqk], v_seq [L][H][dv]. */
void ref_masked_mha_row(const double* q_row, const double* k_seq, const double* v_seq, const int32_t* idx, int k,
                        int H, int dqk, int dv, double scale, double* out, double* lse) {
  double* z = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  for (int h = 0; h < H; ++h) {
    double m = -INFINITY;
    for (int i = 0; i < k; ++i) {
      if (idx[i] < 0) continue;
      double dot = 0.0;
      for (int d = 0; d < dqk; ++d) dot += q_row[h * dqk + d] * k_seq[((int64_t)idx[i] * H + h) * dqk + d];
      z[i] = scale * dot;
      if (z[i] > m) m = z[i];
    }
    for (int e = 0; e < dv; ++e) out[h * dv + e] = 0.0;
    if (m == -INFINITY) {
      lse[h] = -INFINITY;
      continue;
    }
    double denom = 0.0;
    for (int i = 0; i < k; ++i)
      if (idx[i] >= 0) denom += exp(z[i] - m);
    for (int i = 0; i < k; ++i) {
      if (idx[i] < 0) continue;
      double p = exp(z[i] - m) / denom;
      for (int e = 0; e < dv; ++e) out[h * dv + e] += p * v_seq[((int64_t)idx[i] * H + h) * dv + e];
    }
    lse[h] = m + log(denom);
  }
  free(z);
}

/* ---- f4: HISA, block -> token retrieval (analysis page, sec. 5.3) ----------------------- */
/* Representative of a block of keys: the mean of its keys [s0, s0 + n) (the block-mean
 * representation the page discusses).  k_seq: [..][d_I] e4m3; mean: [d_I]. */
void ref_block_mean(const uint8_t* k_seq, int s0, int n, int d_I, double* mean) {
  for (int d = 0; d < d_I; ++d) {
    double acc = 0.0;
    for (int s = s0; s < s0 + n; ++s) acc += ref_e4m3_to_double(k_seq[(int64_t)s * d_I + d]);
    mean[d] = acc / (double)n;
  }
}

/* Coarse score of a block for one query: the indexer's score formula with the block's mean
 * key in place of a token key, sum_j w_j ReLU(q_j . mean). */
double ref_block_score(const uint8_t* q_row, const double* mean, const float* w_row, int H_I, int d_I) {
  double score = 0.0;
  for (int j = 0; j < H_I; ++j) {
    double dot = 0.0;
    for (int d = 0; d < d_I; ++d) dot += ref_e4m3_to_double(q_row[j * d_I + d]) * mean[d];
    score += (double)w_row[j] * (dot > 0.0 ? dot : 0.0);
  }
  return score;
}

/* HISA selection for query t: the keys are cut into blocks [b*bsize, b*bsize + bsize); a block
 * starting at or before t is a candidate, represented by the mean of its keys s <= t; the r
 * candidate blocks with the largest coarse scores are kept (ties -> smaller block); their keys
 * s <= t form U; every key of U gets its exact indexer score (eq. (1)); S = the min(k, |U|) keys
 * of U with the largest scores (ties -> smaller position).
 * idx [k]: S ascending, -1 padded.  blocks [r]: the kept blocks ascending, -1 padded.
 * Returns |S|. */
int ref_hisa_row(const uint8_t* q_row, const uint8_t* k_seq, const float* w_row, int Lk, int t, int H_I,
                 int d_I, int bsize, int r, int k, int32_t* idx, int32_t* blocks) {
  int nb = t / bsize + 1; /* candidate blocks: those starting at or before t */
  double* bscore = (double*)malloc(sizeof(double) * (size_t)nb);
  double* mean = (double*)malloc(sizeof(double) * (size_t)d_I);
  for (int b = 0; b < nb; ++b) {
    int s0 = b * bsize;
    int n = (t + 1 - s0) < bsize ? (t + 1 - s0) : bsize;
    ref_block_mean(k_seq, s0, n, d_I, mean);
    bscore[b] = ref_block_score(q_row, mean, w_row, H_I, d_I);
  }
  /* the r best blocks: the same full sort and tie rule as the token top-k */
  int32_t* bsel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(r > 0 ? r : 1));
  int nsel = ref_topk_row(bscore, nb - 1, r, bsel);
  for (int i = 0; i < r; ++i) blocks[i] = bsel[i];
  /* exact scores on U (every other key -inf), then the token top-k */
  double* sc = (double*)malloc(sizeof(double) * (size_t)(t + 1));
  for (int s = 0; s <= t; ++s) sc[s] = -INFINITY;
  int n_u = 0;
  double* one = (double*)malloc(sizeof(double) * (size_t)Lk);
  ref_indexer_row(q_row, k_seq, w_row, Lk, t, H_I, d_I, one);
  for (int i = 0; i < nsel; ++i) {
    int s0 = bsel[i] * bsize;
    for (int s = s0; s < s0 + bsize && s <= t; ++s) {
      sc[s] = one[s];
      ++n_u;
    }
  }
  /* top-k over U: rank the keys of U only (the others are not candidates) */
  scored_t* c = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n_u > 0 ? n_u : 1));
  int m = 0;
  for (int i = 0; i < nsel; ++i) {
    int s0 = bsel[i] * bsize;
    for (int s = s0; s < s0 + bsize && s <= t; ++s) {
      c[m].score = sc[s];
      c[m].s = s;
      ++m;
    }
  }
  qsort(c, (size_t)m, sizeof(scored_t), by_score_desc_then_index);
  int n = m < k ? m : k;
  unsigned char* chosen = (unsigned char*)calloc((size_t)(t + 1), 1);
  for (int i = 0; i < n; ++i) chosen[c[i].s] = 1;
  int wpos = 0;
  for (int s = 0; s <= t; ++s)
    if (chosen[s]) idx[wpos++] = s;
  for (int i = n; i < k; ++i) idx[i] = -1;
  free(chosen);
  free(c);
  free(one);
  free(sc);
  free(bsel);
  free(mean);
  free(bscore);
  return n;
}

/* ---- f2: gradient of the indexer loss with respect to the indexer's inputs -------------- */
/* Real-valued inputs (fp64) so that the loss can be differentiated numerically as well:
 * q_row [H_I][d_I], k_seq [Lk][d_I], w_row [H_I]; idx [k] (-1 = empty slot, the set held fixed);
 * p [k] the target over the slots.  One row's loss of eq. (4) (eq. (3) when idx lists every
 * s <= t):  L = sum_i p_i (ln p_i - ln q_i),  q = Softmax_i(I_i),
 * I_i = sum_j w_j ReLU(q_j . k_{idx_i}). */
double ref_indexer_loss_row_f64(const double* q_row, const double* k_seq, const double* w_row,
                                const int32_t* idx, const double* p, int k, int H_I, int d_I) {
  double* I = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  double m = -INFINITY;
  for (int i = 0; i < k; ++i) {
    if (idx[i] < 0) continue;
    double score = 0.0;
    for (int j = 0; j < H_I; ++j) {
      double dot = 0.0;
      for (int d = 0; d < d_I; ++d) dot += q_row[j * d_I + d] * k_seq[(int64_t)idx[i] * d_I + d];
      score += w_row[j] * (dot > 0.0 ? dot : 0.0);
    }
    I[i] = score;
    if (score > m) m = score;
  }
  double denom = 0.0;
  for (int i = 0; i < k; ++i)
    if (idx[i] >= 0) denom += exp(I[i] - m);
  double log_z = m + log(denom);
  double loss = 0.0;
  for (int i = 0; i < k; ++i) {
    if (idx[i] < 0 || p[i] == 0.0) continue;
    loss += p[i] * (log(p[i]) - (I[i] - log_z));
  }
  free(I);
  return loss;
}

/* Its gradient, by the chain rule through the definitions above:
 *   dL/dI_i = q_i * (sum_i' p_i') - p_i                        (softmax and KL)
 *   dL/dw_j = sum_i dL/dI_i * ReLU(a_ji),   a_ji = q_j . k_{idx_i}
 *   dL/dq_j = sum_i dL/dI_i * w_j * [a_ji > 0] * k_{idx_i}
 *   dL/dk_s += sum_{i: idx_i = s} dL/dI_i * sum_j w_j [a_ji > 0] q_j
 * with ReLU'(0) taken as 0.  dq [H_I][d_I] and dw [H_I] are written; dk [Lk][d_I] is
 * ACCUMULATED (several query rows add into the same keys); g [k] (nullable) gets dL/dI. */
void ref_indexer_grad_row(const double* q_row, const double* k_seq, const double* w_row,
                          const int32_t* idx, const double* p, int k, int H_I, int d_I, double* dq,
                          double* dw, double* dk, double* g) {
  double* I = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  double* a = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1) * (size_t)H_I);
  double m = -INFINITY;
  for (int i = 0; i < k; ++i) {
    if (idx[i] < 0) continue;
    double score = 0.0;
    for (int j = 0; j < H_I; ++j) {
      double dot = 0.0;
      for (int d = 0; d < d_I; ++d) dot += q_row[j * d_I + d] * k_seq[(int64_t)idx[i] * d_I + d];
      a[(int64_t)i * H_I + j] = dot;
      score += w_row[j] * (dot > 0.0 ? dot : 0.0);
    }
    I[i] = score;
    if (score > m) m = score;
  }
  double denom = 0.0, p_total = 0.0;
  for (int i = 0; i < k; ++i) {
    if (idx[i] < 0) continue;
    denom += exp(I[i] - m);
    p_total += p[i];
  }
  for (int j = 0; j < H_I; ++j) {
    dw[j] = 0.0;
    for (int d = 0; d < d_I; ++d) dq[j * d_I + d] = 0.0;
  }
  for (int i = 0; i < k; ++i) {
    if (idx[i] < 0) {
      if (g) g[i] = 0.0;
      continue;
    }
    double gi = exp(I[i] - m) / denom * p_total - p[i];
    if (g) g[i] = gi;
    const double* ks = k_seq + (int64_t)idx[i] * d_I;
    double* dks = dk + (int64_t)idx[i] * d_I;
    for (int j = 0; j < H_I; ++j) {
      double aj = a[(int64_t)i * H_I + j];
      dw[j] += gi * (aj > 0.0 ? aj : 0.0);
      if (aj > 0.0) {
        for (int d = 0; d < d_I; ++d) {
          dq[j * d_I + d] += gi * w_row[j] * ks[d];
          dks[d] += gi * w_row[j] * q_row[j * d_I + d];
        }
      }
    }
  }
  free(a);
  free(I);
}

/* ---- dense causal MQA over all s <= t (for the k >= t+1 and eq. (19)/(20) checks) ------- */
void ref_dense_mla_row(const uint16_t* q_row, const uint16_t* kv_seq, int t, int H, int d_qk,
                       int d_v, double scale, double* out, double* lse, double* A /* [H][t+1] */) {
  int n = t + 1;
  int32_t* all = (int32_t*)malloc(sizeof(int32_t) * (size_t)n);
  for (int s = 0; s < n; ++s) all[s] = s;
  ref_sparse_mla_row(q_row, kv_seq, all, n, H, d_qk, d_v, scale, out, lse, A);
  free(all);
}

/* ---- whole-path driver over a set of query rows (CPU baseline timing) ------------------- */
/* Runs indexer -> top-k -> sparse MLA (-> p -> KL when emit_p) for each listed flat row
 * r = b*Lq + i, rows spread over nthreads POSIX threads; each row is computed by the
 * single-threaded functions above, so threading changes no arithmetic.
 * Outputs per listed row j: scores [Lk], idx [k], out [H][d_v], lse [H], p [k], kl [1].
 * Any output pointer may be NULL. */
typedef struct {
  const uint8_t *qI, *kI;
  const float* w;
  const uint16_t *q, *kv;
  const int64_t* rows;
  int64_t nrows;
  int B, Lq, Lk, H_I, d_I, k, H, d_qk, d_v, emit_p;
  double scale;
  double *scores, *out, *lse, *p, *kl;
  int32_t* idx;
  int tid, nthreads;
  /* which inputs are stored densely per listed row rather than for every row */
  int rows_packed;
} path_job_t;

static void* path_worker(void* arg) {
  path_job_t* J = (path_job_t*)arg;
  double* sc = (double*)malloc(sizeof(double) * (size_t)J->Lk);
  int32_t* id = (int32_t*)malloc(sizeof(int32_t) * (size_t)J->k);
  double* o = (double*)malloc(sizeof(double) * (size_t)J->H * J->d_v);
  double* l = (double*)malloc(sizeof(double) * (size_t)J->H);
  double* P = (double*)malloc(sizeof(double) * (size_t)J->H * J->k);
  double* pp = (double*)malloc(sizeof(double) * (size_t)J->k);
  for (int64_t j = J->tid; j < J->nrows; j += J->nthreads) {
    int64_t r = J->rows[j];
    int b = (int)(r / J->Lq), i = (int)(r % J->Lq);
    int t = i + J->Lk - J->Lq;
    int64_t src = J->rows_packed ? j : r;
    const uint8_t* q_row = J->qI + src * J->H_I * J->d_I;
    const uint8_t* k_seq = J->kI + (int64_t)b * J->Lk * J->d_I;
    const float* w_row = J->w + src * J->H_I;
    ref_indexer_row(q_row, k_seq, w_row, J->Lk, t, J->H_I, J->d_I, sc);
    ref_topk_row(sc, t, J->k, id);
    const uint16_t* qa = J->q + src * J->H * J->d_qk;
    const uint16_t* kvs = J->kv + (int64_t)b * J->Lk * J->d_qk;
    ref_sparse_mla_row(qa, kvs, id, J->k, J->H, J->d_qk, J->d_v, J->scale, o, l,
                       J->emit_p ? P : NULL);
    double klv = 0.0;
    if (J->emit_p) {
      ref_p_sel_row(P, id, J->k, J->H, pp);
      klv = ref_kl_row(sc, id, pp, J->k);
    }
    if (J->scores) memcpy(J->scores + j * J->Lk, sc, sizeof(double) * (size_t)J->Lk);
    if (J->idx) memcpy(J->idx + j * J->k, id, sizeof(int32_t) * (size_t)J->k);
    if (J->out) memcpy(J->out + j * J->H * J->d_v, o, sizeof(double) * (size_t)J->H * J->d_v);
    if (J->lse) memcpy(J->lse + j * J->H, l, sizeof(double) * (size_t)J->H);
    if (J->p && J->emit_p) memcpy(J->p + j * J->k, pp, sizeof(double) * (size_t)J->k);
    if (J->kl) J->kl[j] = klv;
  }
  free(sc);
  free(id);
  free(o);
  free(l);
  free(P);
  free(pp);
  return NULL;
}

int ref_path_rows(const uint8_t* qI, const uint8_t* kI, const float* w, const uint16_t* q,
                  const uint16_t* kv, int rows_packed, const int64_t* rows, int64_t nrows, int B,
                  int Lq, int Lk, int H_I, int d_I, int k, int H, int d_qk, int d_v, double scale,
                  int emit_p, double* scores, int32_t* idx, double* out, double* lse, double* p,
                  double* kl, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  path_job_t* jobs = (path_job_t*)malloc(sizeof(path_job_t) * (size_t)nthreads);
  for (int i = 0; i < nthreads; ++i) {
    path_job_t J = {qI, kI, w, q, kv, rows, nrows, B, Lq, Lk, H_I, d_I, k, H, d_qk, d_v, emit_p,
                    scale, scores, out, lse, p, kl, idx, i, nthreads, rows_packed};
    jobs[i] = J;
    pthread_create(&th[i], NULL, path_worker, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(th);
  free(jobs);
  return 0;
}
