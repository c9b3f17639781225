/*
 * HiLS oracle — a plain, slow, fp64 CPU restatement of Hierarchical Landmark
 * Sparse (HiLS) attention: the forward pass and, at the end of the file, its
 * gradients with the chunk selection held fixed.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library and it includes no CUDA header.
 *
 * Sources (cited by page and section):
 *   [M]  hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section
 *        "方法" (Method): uniform chunking, the chunk-aligned sliding window,
 *        the chunk mass Z_{i,c}, the surrogate score
 *        s^_{i,c} = q_i.k'_c / sqrt(d) + b'_c, the landmark summary
 *        (k'_c = p-weighted sum of the chunk's keys, b'_c = entropy of p),
 *        the partition estimate Z^_i = sum_{c in I_i} exp(s^_{i,c}) + Z_{i,swa},
 *        the hierarchical factorisation of w_{i,j}, Q-Cal
 *        (dq_i = W_up W_down h_i, scoring only) and the GQA rule
 *        (per-head scores, max over the group's heads, then top-K).
 *   [A]  "Hierarchical Landmark Sparse Attention" abstract (chatpaper page):
 *        each query attends each retrieved chunk on its own and the chunk
 *        outputs are fused by the retrieval scores.
 *
 * Readings where the pages leave a step open:
 *   - window of query i = keys [max(0,(cur(i)-n_w+1)*S), i], cur(i)=floor(i/S),
 *     n_w = W/S; candidates = complete chunks c <= cur(i)-n_w;
 *   - the landmark softmax uses the same 1/sqrt(d) temperature as the
 *     attention logits; the entropy is in nats;
 *   - every head uses its own s^ in Z^ and in the fusion weights; the group
 *     max only ranks chunks;  Z_swa is the exact window mass (self included);
 *   - top-K ties go to the smaller chunk index; the chosen set is stored in
 *     ascending chunk order, padded with -1 (scores padded with -inf);
 *   - fewer candidates than K: all are taken; none: pure window attention.
 *
 * All inputs arrive as float32 (bf16 inputs are widened exactly by the
 * caller); every intermediate and every output is double.  OpenMP only
 * splits independent rows across threads and does not change any result.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t B;       /* batch */
  int64_t Hq;      /* query heads */
  int64_t Hkv;     /* key/value heads; G = Hq / Hkv */
  int64_t N;       /* keys per sequence (prefill length, or decode cache length L) */
  int64_t d;       /* head dimension */
  int64_t S;       /* chunk size */
  int64_t W;       /* window size, a multiple of S */
  int64_t K;       /* number of selected chunks */
  int64_t nq;      /* query rows stored per (b, head): N for prefill, 1 for decode */
  int64_t q_pos0;  /* sequence position of stored query row 0: 0 prefill, L-1 decode */
  double scale;    /* logit scale, 1/sqrt(d) */
} hils_oracle_dims;

static int64_t n_chunks(const hils_oracle_dims *dm) { return dm->N / dm->S; }

/* first key of the window of position i ([M], chunk-aligned sliding window) */
static int64_t window_start(const hils_oracle_dims *dm, int64_t i) {
  int64_t nw = dm->W / dm->S;
  int64_t first_chunk = i / dm->S - nw + 1;
  return first_chunk > 0 ? first_chunk * dm->S : 0;
}

/* number of candidate chunks of position i: complete chunks before the window */
static int64_t n_candidates(const hils_oracle_dims *dm, int64_t i) {
  int64_t nw = dm->W / dm->S;
  int64_t last = i / dm->S - nw; /* last candidate chunk, may be negative */
  return last >= 0 ? last + 1 : 0;
}

static double dot_fd(const float *a, const float *b, int64_t n) {
  double s = 0.0;
  for (int64_t e = 0; e < n; ++e) s += (double)a[e] * (double)b[e];
  return s;
}

static double dot_dd(const double *a, const float *b, int64_t n) {
  double s = 0.0;
  for (int64_t e = 0; e < n; ++e) s += a[e] * (double)b[e];
  return s;
}

/*
 * Landmark summaries ([M], the paragraph after the surrogate-score equation):
 * for every (b, query head h, complete chunk c), the landmark query q'_{h,c}
 * induces p = softmax_j(q'.k_j / sqrt(d)) over the S keys j of chunk c (keys of
 * KV head h / G); k'_{h,c} = sum_j p_j k_j and b'_{h,c} = -sum_j p_j log p_j.
 * The entropy is evaluated as (m + log Z) - sum_j p_j l_j, which is the same
 * quantity written without 0*log 0 terms.
 *   k     [B, Hkv, N, d]     q_lmk [B, Hq, C, d]
 *   k_sum [B, Hq, C, d]      b_sum [B, Hq, C]        (C = N / S)
 */
void hils_oracle_summaries(const hils_oracle_dims *dm, const float *k, const float *q_lmk,
                           double *k_sum, double *b_sum) {
  const int64_t C = n_chunks(dm), G = dm->Hq / dm->Hkv, d = dm->d, S = dm->S;
  const int64_t total = dm->B * dm->Hq * C;
#pragma omp parallel
  {
    double *l = (double *)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < total; ++t) {
      const int64_t c = t % C, h = (t / C) % dm->Hq, b = t / (C * dm->Hq);
      const float *ql = q_lmk + ((b * dm->Hq + h) * C + c) * d;
      const float *kc = k + ((b * dm->Hkv + h / G) * dm->N + c * S) * d;
      double m = -INFINITY;
      for (int64_t j = 0; j < S; ++j) {
        l[j] = dm->scale * dot_fd(ql, kc + j * d, d);
        if (l[j] > m) m = l[j];
      }
      double z = 0.0;
      for (int64_t j = 0; j < S; ++j) z += exp(l[j] - m);
      double *ks = k_sum + t * d;
      for (int64_t e = 0; e < d; ++e) ks[e] = 0.0;
      double pl = 0.0;
      for (int64_t j = 0; j < S; ++j) {
        const double p = exp(l[j] - m) / z;
        pl += p * l[j];
        for (int64_t e = 0; e < d; ++e) ks[e] += p * (double)kc[j * d + e];
      }
      b_sum[t] = (m + log(z)) - pl;
    }
    free(l);
  }
}

/*
 * Q-Cal scoring query ([M], second design choice): q~_i = q_i + W_up (W_down h_i),
 * with dq_i of width Hq*d reshaped to [Hq, d]. Used for scoring only.
 *   rows  [nrows, 2] = (b, position)     h [B, nq, Dm]
 *   w_down [r, Dm]   w_up [Hq*d, r]      qs (out) [nrows, Hq, d]
 */
void hils_oracle_qcal(const hils_oracle_dims *dm, int64_t Dm, int64_t r, const int64_t *rows,
                      int64_t nrows, const float *q, const float *h, const float *w_down,
                      const float *w_up, double *qs) {
  const int64_t d = dm->d, Hq = dm->Hq;
#pragma omp parallel
  {
    double *t = (double *)malloc(sizeof(double) * (size_t)r);
#pragma omp for schedule(static)
    for (int64_t n = 0; n < nrows; ++n) {
      const int64_t b = rows[2 * n], iq = rows[2 * n + 1] - dm->q_pos0;
      const float *hi = h + (b * dm->nq + iq) * Dm;
      for (int64_t a = 0; a < r; ++a) t[a] = dot_fd(w_down + a * Dm, hi, Dm);
      for (int64_t hh = 0; hh < Hq; ++hh)
        for (int64_t e = 0; e < d; ++e) {
          const float *wu = w_up + (hh * d + e) * r;
          double dq = 0.0;
          for (int64_t a = 0; a < r; ++a) dq += (double)wu[a] * t[a];
          qs[(n * Hq + hh) * d + e] = (double)q[((b * Hq + hh) * dm->nq + iq) * d + e] + dq;
        }
    }
    free(t);
  }
}

typedef struct { double g; int64_t c; } cand_t;

/* larger score first; equal scores: smaller chunk index first ([M], top-K; tie reading) */
static int cmp_cand(const void *x, const void *y) {
  const cand_t *a = (const cand_t *)x, *b = (const cand_t *)y;
  if (a->g > b->g) return -1;
  if (a->g < b->g) return 1;
  return (a->c > b->c) - (a->c < b->c);
}

static int cmp_i32(const void *x, const void *y) {
  const int32_t a = *(const int32_t *)x, b = *(const int32_t *)y;
  return (a > b) - (a < b);
}

/*
 * Chunk scoring and selection for a list of positions ([M], surrogate score,
 * GQA rule, top-K).  mode 0: s^_{h,i,c} = qs.k'_{h,c} * scale + b'_{h,c} with
 * qs = the scoring query (Q-Cal output, or q itself when qs is NULL).
 * mode 1 ("exact mass", the naive-BSA ranking of [M]): s^ is replaced by the
 * true chunk log-mass log Z_{i,c} = LSE_{j in c} (q_i.k_j * scale).
 * Per KV group the chunk score is the max over the group's heads; the K best
 * candidates are kept (ties: smaller c), stored ascending and -1 padded.
 *   rows  [nrows, 2]           idx   (out) [nrows, Hkv, K]
 *   s_sel (out) [nrows, Hq, K]  each head's own s^ of the chosen chunks, -inf padded
 *   s_all (out, optional) [nrows, Hq, C]   every head's s^ (-inf off-candidate)
 *   g_all (out, optional) [nrows, Hkv, C]  group scores (-inf off-candidate)
 */
void hils_oracle_select(const hils_oracle_dims *dm, int mode, const int64_t *rows, int64_t nrows,
                        const double *qs, const float *q, const float *k, const double *k_sum,
                        const double *b_sum, int32_t *idx, double *s_sel, double *s_all,
                        double *g_all) {
  const int64_t C = n_chunks(dm), G = dm->Hq / dm->Hkv, d = dm->d, S = dm->S, K = dm->K;
#pragma omp parallel
  {
    double *sh = (double *)malloc(sizeof(double) * (size_t)(G * (C > 0 ? C : 1)));
    cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(C > 0 ? C : 1));
    int32_t *chosen = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
    for (int64_t n = 0; n < nrows; ++n) {
      const int64_t b = rows[2 * n], i = rows[2 * n + 1], iq = i - dm->q_pos0;
      const int64_t nc = n_candidates(dm, i);
      for (int64_t grp = 0; grp < dm->Hkv; ++grp) {
        for (int64_t hg = 0; hg < G; ++hg) {
          const int64_t h = grp * G + hg;
          for (int64_t c = 0; c < nc; ++c) {
            double s;
            if (mode == 0) {
              const double *kp = k_sum + ((b * dm->Hq + h) * C + c) * d;
              double acc = 0.0;
              if (qs) {
                const double *qq = qs + (n * dm->Hq + h) * d;
                for (int64_t e = 0; e < d; ++e) acc += qq[e] * kp[e];
              } else {
                acc = dot_dd(kp, q + ((b * dm->Hq + h) * dm->nq + iq) * d, d);
              }
              s = acc * dm->scale + b_sum[(b * dm->Hq + h) * C + c];
            } else {
              const float *qi = q + ((b * dm->Hq + h) * dm->nq + iq) * d;
              const float *kc = k + ((b * dm->Hkv + grp) * dm->N + c * S) * d;
              double m = -INFINITY;
              for (int64_t j = 0; j < S; ++j) {
                const double l = dm->scale * dot_fd(qi, kc + j * d, d);
                if (l > m) m = l;
              }
              double z = 0.0;
              for (int64_t j = 0; j < S; ++j) z += exp(dm->scale * dot_fd(qi, kc + j * d, d) - m);
              s = m + log(z);
            }
            sh[hg * C + c] = s;
          }
          if (s_all)
            for (int64_t c = 0; c < C; ++c)
              s_all[(n * dm->Hq + h) * C + c] = c < nc ? sh[hg * C + c] : -INFINITY;
        }
        for (int64_t c = 0; c < nc; ++c) {
          double gm = -INFINITY;
          for (int64_t hg = 0; hg < G; ++hg) gm = sh[hg * C + c] > gm ? sh[hg * C + c] : gm;
          cand[c].g = gm;
          cand[c].c = c;
        }
        if (g_all)
          for (int64_t c = 0; c < C; ++c) g_all[(n * dm->Hkv + grp) * C + c] = c < nc ? cand[c].g : -INFINITY;
        qsort(cand, (size_t)nc, sizeof(cand_t), cmp_cand);
        const int64_t nsel = nc < K ? nc : K;
        for (int64_t s = 0; s < nsel; ++s) chosen[s] = (int32_t)cand[s].c;
        qsort(chosen, (size_t)nsel, sizeof(int32_t), cmp_i32);
        for (int64_t s = 0; s < K; ++s) {
          idx[(n * dm->Hkv + grp) * K + s] = s < nsel ? chosen[s] : -1;
          for (int64_t hg = 0; hg < G; ++hg)
            s_sel[(n * dm->Hq + grp * G + hg) * K + s] = s < nsel ? sh[hg * C + chosen[s]] : -INFINITY;
        }
      }
    }
    free(sh);
    free(cand);
    free(chosen);
  }
}

/*
 * Hierarchical-softmax sparse attention for a list of positions ([M], the
 * factorised weight w_{i,j} and Z^_i; [A], per-chunk attention fused by the
 * retrieval scores).  For each head h of the row:
 *   O_{i,c}  = sum_{j in c} softmax_{c}(s_ij) v_j        (own intra-chunk softmax)
 *   A_c      = s_sel (the chunk's surrogate log-mass for this head)
 *   A_swa    = LSE_{j in window} s_ij,  O_swa = window softmax . v
 *   O_i      = (sum_c e^{A_c} O_{i,c} + e^{A_swa} O_swa) / (sum_c e^{A_c} + e^{A_swa})
 * so a window key j has weight e^{s_ij}/Z^ and a key j of chunk c has weight
 * (e^{s_ij}/Z_{i,c}) (e^{s^_c}/Z^), Z^ = sum_c e^{s^_c} + Z_swa.  Evaluated with
 * all exponents shifted by their maximum.  Attention logits use the raw q
 * (Q-Cal only changes the scoring query).
 *   rows [nrows,2]  idx [nrows,Hkv,K]  s_sel [nrows,Hq,K]  out (out) [nrows,Hq,d]
 *   lse (out, optional) [nrows, Hq] = log Z^ (natural log, unshifted)
 */
void hils_oracle_attend(const hils_oracle_dims *dm, const int64_t *rows, int64_t nrows,
                        const float *q, const float *k, const float *v, const int32_t *idx,
                        const double *s_sel, double *out, double *lse) {
  const int64_t G = dm->Hq / dm->Hkv, d = dm->d, S = dm->S, K = dm->K;
  const int64_t total = nrows * dm->Hq;
#pragma omp parallel
  {
    double *sj = (double *)malloc(sizeof(double) * (size_t)(dm->W > S ? dm->W : S));
    double *oc = (double *)malloc(sizeof(double) * (size_t)d);
    double *osw = (double *)malloc(sizeof(double) * (size_t)d);
    double *ac = (double *)malloc(sizeof(double) * (size_t)K);
    double *ocs = (double *)malloc(sizeof(double) * (size_t)(K * d));
#pragma omp for schedule(dynamic, 4)
    for (int64_t t = 0; t < total; ++t) {
      const int64_t n = t / dm->Hq, h = t % dm->Hq, grp = h / G;
      const int64_t b = rows[2 * n], i = rows[2 * n + 1], iq = i - dm->q_pos0;
      const float *qi = q + ((b * dm->Hq + h) * dm->nq + iq) * d;
      const float *kb = k + (b * dm->Hkv + grp) * dm->N * d;
      const float *vb = v + (b * dm->Hkv + grp) * dm->N * d;
      /* window part: exact softmax over keys [w0, i] */
      const int64_t w0 = window_start(dm, i), nwin = i - w0 + 1;
      double mw = -INFINITY;
      for (int64_t j = 0; j < nwin; ++j) {
        sj[j] = dm->scale * dot_fd(qi, kb + (w0 + j) * d, d);
        if (sj[j] > mw) mw = sj[j];
      }
      double zw = 0.0;
      for (int64_t e = 0; e < d; ++e) osw[e] = 0.0;
      for (int64_t j = 0; j < nwin; ++j) {
        const double p = exp(sj[j] - mw);
        zw += p;
        for (int64_t e = 0; e < d; ++e) osw[e] += p * (double)vb[(w0 + j) * d + e];
      }
      for (int64_t e = 0; e < d; ++e) osw[e] /= zw;
      const double a_swa = mw + log(zw);
      /* selected chunks: each with its own softmax */
      int64_t nsel = 0;
      for (int64_t s = 0; s < K; ++s) {
        const int32_t c = idx[(n * dm->Hkv + grp) * K + s];
        if (c < 0) continue;
        double mc = -INFINITY;
        for (int64_t j = 0; j < S; ++j) {
          sj[j] = dm->scale * dot_fd(qi, kb + (c * S + j) * d, d);
          if (sj[j] > mc) mc = sj[j];
        }
        double zc = 0.0;
        for (int64_t e = 0; e < d; ++e) oc[e] = 0.0;
        for (int64_t j = 0; j < S; ++j) {
          const double p = exp(sj[j] - mc);
          zc += p;
          for (int64_t e = 0; e < d; ++e) oc[e] += p * (double)vb[(c * S + j) * d + e];
        }
        for (int64_t e = 0; e < d; ++e) ocs[nsel * d + e] = oc[e] / zc;
        ac[nsel] = s_sel[(n * dm->Hq + h) * K + s];
        ++nsel;
      }
      /* fusion: weights e^{A}/Z^ with a common shift */
      double m = a_swa;
      for (int64_t s = 0; s < nsel; ++s) m = ac[s] > m ? ac[s] : m;
      double zhat = exp(a_swa - m);
      double *o = out + t * d;
      for (int64_t e = 0; e < d; ++e) o[e] = exp(a_swa - m) * osw[e];
      for (int64_t s = 0; s < nsel; ++s) {
        const double w = exp(ac[s] - m);
        zhat += w;
        for (int64_t e = 0; e < d; ++e) o[e] += w * ocs[s * d + e];
      }
      for (int64_t e = 0; e < d; ++e) o[e] /= zhat;
      if (lse) lse[t] = m + log(zhat);
    }
    free(sj);
    free(oc);
    free(osw);
    free(ac);
    free(ocs);
  }
}

/* ------------------------------------------------------------- backward --- */
/*
 * Gradients of the forward pass above, with the chunk selection held fixed
 * (top-K is a discrete choice; gradients reach the chunk scores s^ because they
 * enter the output through the fusion weights exp(s^)/Z^: hyper.ai summary,
 * Method section, the factorised token weight w_ij and Z^_i; the wmrh.cn
 * article's point that the hierarchical softmax lets the language-model loss
 * train the summaries).  Plain serial loops: the gradient buffers accumulate
 * across rows, so no row-parallel split.  Every output is accumulated into
 * (callers zero it).
 */

/*
 * Attention backward for the listed rows.  With w_u = e^{A_u}/Z^ for the
 * window unit and every selected chunk, out = sum_u w_u O_u and D = dout.out:
 *   window token j:   omega_j = e^{s_ij}/Z^, ds_ij = omega_j (dout.v_j - D),
 *                     dv_j += omega_j dout;
 *   chunk c, token j: ds_ij = w_c p_j (dout.v_j - dout.O_c),
 *                     dv_j += w_c p_j dout,  dA_c = w_c (dout.O_c - D);
 *   dq_i += scale sum_j ds_ij k_j,  dk_j += scale ds_ij q_i.
 *   dout [nrows, Hq, d];  dq [B, Hq, nq, d];  dk, dv [B, Hkv, N, d];
 *   ds_sel [nrows, Hq, K] = dA_c per slot (0 for empty slots).
 */
void hils_oracle_attend_bwd(const hils_oracle_dims *dm, const int64_t *rows, int64_t nrows, const float *q,
                            const float *k, const float *v, const int32_t *idx, const double *s_sel,
                            const double *dout, double *dq, double *dk, double *dv, double *ds_sel) {
  const int64_t G = dm->Hq / dm->Hkv, d = dm->d, S = dm->S, K = dm->K;
  const int64_t span = dm->W > S ? dm->W : S;
  double *sj = (double *)malloc(sizeof(double) * (size_t)(K * S + span));
  double *ocs = (double *)malloc(sizeof(double) * (size_t)(K * d));
  double *ac = (double *)malloc(sizeof(double) * (size_t)K);
  double *out = (double *)malloc(sizeof(double) * (size_t)d);
  for (int64_t n = 0; n < nrows; ++n) {
    const int64_t b = rows[2 * n], i = rows[2 * n + 1], iq = i - dm->q_pos0;
    for (int64_t h = 0; h < dm->Hq; ++h) {
      const int64_t grp = h / G;
      const float *qi = q + ((b * dm->Hq + h) * dm->nq + iq) * d;
      const float *kb = k + (b * dm->Hkv + grp) * dm->N * d;
      const float *vb = v + (b * dm->Hkv + grp) * dm->N * d;
      const double *go = dout + (n * dm->Hq + h) * d;
      double *gq = dq + ((b * dm->Hq + h) * dm->nq + iq) * d;
      double *gk = dk + (b * dm->Hkv + grp) * dm->N * d;
      double *gv = dv + (b * dm->Hkv + grp) * dm->N * d;
      const int32_t *il = idx + (n * dm->Hkv + grp) * K;
      /* forward pieces: window logits, chunk logits and outputs, log-masses */
      const int64_t w0 = window_start(dm, i), nwin = i - w0 + 1;
      double *sw = sj + K * S;
      double mw = -INFINITY;
      for (int64_t j = 0; j < nwin; ++j) {
        sw[j] = dm->scale * dot_fd(qi, kb + (w0 + j) * d, d);
        if (sw[j] > mw) mw = sw[j];
      }
      double zw = 0.0;
      for (int64_t j = 0; j < nwin; ++j) zw += exp(sw[j] - mw);
      const double a_swa = mw + log(zw);
      double m = a_swa;
      for (int64_t s = 0; s < K; ++s) {
        const int32_t c = il[s];
        if (c < 0) continue;
        double mc = -INFINITY;
        for (int64_t j = 0; j < S; ++j) {
          sj[s * S + j] = dm->scale * dot_fd(qi, kb + (c * S + j) * d, d);
          if (sj[s * S + j] > mc) mc = sj[s * S + j];
        }
        double zc = 0.0;
        for (int64_t j = 0; j < S; ++j) zc += exp(sj[s * S + j] - mc);
        for (int64_t e = 0; e < d; ++e) ocs[s * d + e] = 0.0;
        for (int64_t j = 0; j < S; ++j) {
          const double p = exp(sj[s * S + j] - mc) / zc;
          sj[s * S + j] = p; /* keep the intra-chunk softmax */
          for (int64_t e = 0; e < d; ++e) ocs[s * d + e] += p * (double)vb[(c * S + j) * d + e];
        }
        ac[s] = s_sel[(n * dm->Hq + h) * K + s];
        if (ac[s] > m) m = ac[s];
      }
      double zhat = exp(a_swa - m);
      for (int64_t s = 0; s < K; ++s)
        if (il[s] >= 0) zhat += exp(ac[s] - m);
      for (int64_t e = 0; e < d; ++e) out[e] = 0.0;
      for (int64_t j = 0; j < nwin; ++j) {
        const double om = exp(sw[j] - m) / zhat;
        for (int64_t e = 0; e < d; ++e) out[e] += om * (double)vb[(w0 + j) * d + e];
      }
      for (int64_t s = 0; s < K; ++s) {
        if (il[s] < 0) continue;
        const double wc = exp(ac[s] - m) / zhat;
        for (int64_t e = 0; e < d; ++e) out[e] += wc * ocs[s * d + e];
      }
      double D = 0.0;
      for (int64_t e = 0; e < d; ++e) D += go[e] * out[e];
      /* window tokens */
      for (int64_t j = 0; j < nwin; ++j) {
        const int64_t t = w0 + j;
        const double om = exp(sw[j] - m) / zhat;
        const double gvj = dot_dd(go, vb + t * d, d);
        const double ds = om * (gvj - D);
        for (int64_t e = 0; e < d; ++e) {
          gv[t * d + e] += om * go[e];
          gq[e] += dm->scale * ds * (double)kb[t * d + e];
          gk[t * d + e] += dm->scale * ds * (double)qi[e];
        }
      }
      /* selected chunks */
      for (int64_t s = 0; s < K; ++s) {
        const int32_t c = il[s];
        if (c < 0) continue;
        const double wc = exp(ac[s] - m) / zhat;
        double go_oc = 0.0;
        for (int64_t e = 0; e < d; ++e) go_oc += go[e] * ocs[s * d + e];
        ds_sel[(n * dm->Hq + h) * K + s] += wc * (go_oc - D);
        for (int64_t j = 0; j < S; ++j) {
          const int64_t t = c * S + j;
          const double p = sj[s * S + j];
          const double gvj = dot_dd(go, vb + t * d, d);
          const double ds = wc * p * (gvj - go_oc);
          for (int64_t e = 0; e < d; ++e) {
            gv[t * d + e] += wc * p * go[e];
            gq[e] += dm->scale * ds * (double)kb[t * d + e];
            gk[t * d + e] += dm->scale * ds * (double)qi[e];
          }
        }
      }
    }
  }
  free(sj);
  free(ocs);
  free(ac);
  free(out);
}

/*
 * Chunk-score backward: s^_{h,i,c} = qs_{h,i}.k'_{h,c} * scale + b'_{h,c}
 * ([M], surrogate-score equation) for the chosen chunks, so
 *   dqs_{h,i} += scale sum_c dA_c k'_{h,c},  dk'_{h,c} += scale dA_c qs_{h,i},
 *   db'_{h,c} += dA_c.
 *   qs [nrows, Hq, d] (scoring queries, double), or NULL to read q;
 *   ds_sel [nrows, Hq, K];  dqs [nrows, Hq, d];  dk_sum [B,Hq,C,d];  db_sum [B,Hq,C].
 */
void hils_oracle_score_bwd(const hils_oracle_dims *dm, const int64_t *rows, int64_t nrows, const double *qs,
                           const float *q, const double *k_sum, const int32_t *idx, const double *ds_sel,
                           double *dqs, double *dk_sum, double *db_sum) {
  const int64_t C = n_chunks(dm), G = dm->Hq / dm->Hkv, d = dm->d, K = dm->K;
  for (int64_t n = 0; n < nrows; ++n) {
    const int64_t b = rows[2 * n], iq = rows[2 * n + 1] - dm->q_pos0;
    for (int64_t h = 0; h < dm->Hq; ++h) {
      const int32_t *il = idx + (n * dm->Hkv + h / G) * K;
      for (int64_t s = 0; s < K; ++s) {
        const int32_t c = il[s];
        if (c < 0) continue;
        const double g = ds_sel[(n * dm->Hq + h) * K + s];
        const double *kp = k_sum + ((b * dm->Hq + h) * C + c) * d;
        double *gkp = dk_sum + ((b * dm->Hq + h) * C + c) * d;
        for (int64_t e = 0; e < d; ++e) {
          const double qe = qs ? qs[(n * dm->Hq + h) * d + e] : (double)q[((b * dm->Hq + h) * dm->nq + iq) * d + e];
          dqs[(n * dm->Hq + h) * d + e] += dm->scale * g * kp[e];
          gkp[e] += dm->scale * g * qe;
        }
        db_sum[(b * dm->Hq + h) * C + c] += g;
      }
    }
  }
}

/*
 * Summary backward ([M], the landmark summary: p = softmax(q'.k_j * scale)
 * over the chunk's keys, k' = sum_j p_j k_j, b' = -sum_j p_j log p_j):
 *   dp_j = dk'.k_j - db' (log p_j + 1),  dl_j = p_j (dp_j - sum_m p_m dp_m),
 *   dk_j += p_j dk' + scale dl_j q',     dq' += scale sum_j dl_j k_j.
 *   dk_sum [B,Hq,C,d], db_sum [B,Hq,C];  dk [B,Hkv,N,d];  dq_lmk [B,Hq,C,d].
 */
void hils_oracle_summaries_bwd(const hils_oracle_dims *dm, const float *k, const float *q_lmk,
                               const double *dk_sum, const double *db_sum, double *dk, double *dq_lmk) {
  const int64_t C = n_chunks(dm), G = dm->Hq / dm->Hkv, d = dm->d, S = dm->S;
  double *p = (double *)malloc(sizeof(double) * (size_t)S);
  double *dl = (double *)malloc(sizeof(double) * (size_t)S);
  for (int64_t t = 0; t < dm->B * dm->Hq * C; ++t) {
    const int64_t c = t % C, h = (t / C) % dm->Hq, b = t / (C * dm->Hq);
    const float *ql = q_lmk + t * d;
    const float *kc = k + ((b * dm->Hkv + h / G) * dm->N + c * S) * d;
    double *gkc = dk + ((b * dm->Hkv + h / G) * dm->N + c * S) * d;
    const double *gks = dk_sum + t * d;
    const double gb = db_sum[t];
    double m = -INFINITY;
    for (int64_t j = 0; j < S; ++j) {
      p[j] = dm->scale * dot_fd(ql, kc + j * d, d);
      if (p[j] > m) m = p[j];
    }
    double z = 0.0;
    for (int64_t j = 0; j < S; ++j) z += exp(p[j] - m);
    const double lz = m + log(z);
    double pdp = 0.0;
    for (int64_t j = 0; j < S; ++j) {
      const double lp = p[j] - lz; /* log p_j */
      p[j] = exp(lp);
      dl[j] = dot_dd(gks, kc + j * d, d) - gb * (lp + 1.0); /* dp_j for now */
      pdp += p[j] * dl[j];
    }
    for (int64_t j = 0; j < S; ++j) {
      dl[j] = p[j] * (dl[j] - pdp);
      for (int64_t e = 0; e < d; ++e) {
        gkc[j * d + e] += p[j] * gks[e] + dm->scale * dl[j] * (double)ql[e];
        dq_lmk[t * d + e] += dm->scale * dl[j] * (double)kc[j * d + e];
      }
    }
  }
  free(p);
  free(dl);
}

/*
 * Q-Cal backward ([M], second design choice: q~ = q + W_up (W_down h)):
 *   t = W_down h,  dW_up += dq~ t^T,  dt = W_up^T dq~,  dW_down += dt h^T,
 *   dh += W_down^T dt  (and dq += dq~, added by the caller).
 *   rows [nrows,2]; h [B, nq, Dm]; w_down [r, Dm]; w_up [Hq d, r];
 *   dqs [nrows, Hq, d]; dh [B, nq, Dm]; dw_down [r, Dm]; dw_up [Hq d, r].
 */
void hils_oracle_qcal_bwd(const hils_oracle_dims *dm, int64_t Dm, int64_t r, const int64_t *rows, int64_t nrows,
                          const float *h, const float *w_down, const float *w_up, const double *dqs, double *dh,
                          double *dw_down, double *dw_up) {
  const int64_t E = dm->Hq * dm->d;
  double *t = (double *)malloc(sizeof(double) * (size_t)r);
  double *dt = (double *)malloc(sizeof(double) * (size_t)r);
  for (int64_t n = 0; n < nrows; ++n) {
    const int64_t b = rows[2 * n], iq = rows[2 * n + 1] - dm->q_pos0;
    const float *hi = h + (b * dm->nq + iq) * Dm;
    double *ghi = dh + (b * dm->nq + iq) * Dm;
    const double *g = dqs + n * E;
    for (int64_t a = 0; a < r; ++a) {
      t[a] = dot_fd(w_down + a * Dm, hi, Dm);
      dt[a] = 0.0;
    }
    for (int64_t e = 0; e < E; ++e)
      for (int64_t a = 0; a < r; ++a) {
        dw_up[e * r + a] += g[e] * t[a];
        dt[a] += (double)w_up[e * r + a] * g[e];
      }
    for (int64_t a = 0; a < r; ++a)
      for (int64_t mm = 0; mm < Dm; ++mm) {
        dw_down[a * Dm + mm] += dt[a] * (double)hi[mm];
        ghi[mm] += (double)w_down[a * Dm + mm] * dt[a];
      }
  }
  free(t);
  free(dt);
}
