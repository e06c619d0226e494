/*
 * oracle.c -- plain CPU float64 oracle of the windowed atom attention block.
 *
 * TEST INFRASTRUCTURE: see oracle.h. Straight loops in the order the pages state
 * the steps; no blocking, fusion or reordering. Every step cites its passage:
 *   [WAA n] = "Local atom attention, encoder pooling and decoder skip/readout",
 *             Required behavior, bullet n;
 *   [AF3 RB] / [ESM RB] = "AlphaFold 3 / ESMFold 2 Atom Attention Encoder",
 *             Required behavior.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* Built twice: plain (one thread) and with -fopenmp, where the per-atom loops run on
 * all host cores. Each atom's arithmetic is the same in both builds; every thread has
 * its own scratch rows, and the pooled sums are still accumulated serially in
 * ascending atom order. */
#ifdef _OPENMP
#include <omp.h>
static int orc_nthreads(void) { return omp_get_max_threads(); }
static int orc_tid(void) { return omp_get_thread_num(); }
#else
static int orc_nthreads(void) { return 1; }
static int orc_tid(void) { return 0; }
#endif

/* threads the per-atom loops of orc_forward use */
int orc_threads(void) { return orc_nthreads(); }

/* sigmoid(z) = 1 / (1 + e^-z); SiLU(z) = z * sigmoid(z)  [ESM RB, last-but-one item].
 * For z < 0 the same value is formed as e^z / (1 + e^z), so that a representable
 * subnormal tail is kept rather than flushed through an overflowing e^-z  [WAA 23] */
double orc_sigmoid(double z) {
  if (z >= 0.0) return 1.0 / (1.0 + exp(-z));
  double e = exp(z);
  return e / (1.0 + e);
}
double orc_silu(double z) { return z * orc_sigmoid(z); }

/* Population LayerNorm without affine, eps inside the root  [WAA 7] */
void orc_layer_norm(const double *v, int64_t n, double eps, double *out) {
  double mean = 0.0, var = 0.0;
  for (int64_t i = 0; i < n; ++i) mean += v[i];
  mean /= (double)n;
  for (int64_t i = 0; i < n; ++i) var += (v[i] - mean) * (v[i] - mean);
  var /= (double)n;
  double inv = 1.0 / sqrt(var + eps);
  for (int64_t i = 0; i < n; ++i) out[i] = (v[i] - mean) * inv;
}

/* RMS(z) = z / sqrt(mean(z^2) + eps), no affine  [WAA 12] */
void orc_rms_norm(const double *v, int64_t n, double eps, double *out) {
  double ms = 0.0;
  for (int64_t i = 0; i < n; ++i) ms += v[i] * v[i];
  ms /= (double)n;
  double inv = 1.0 / sqrt(ms + eps);
  for (int64_t i = 0; i < n; ++i) out[i] = v[i] * inv;
}

/* q * cos + rotate_half(q) * sin, rotate_half([q1, q2]) = [-q2, q1]  [WAA 13] */
void orc_rope_half_split(const double *q, const double *cosv, const double *sinv,
                         int64_t D, double *out) {
  int64_t h = D / 2;
  for (int64_t d = 0; d < D; ++d) {
    double rot = (d < h) ? -q[d + h] : q[d - h];
    out[d] = q[d] * cosv[d] + rot * sinv[d];
  }
}

/* Stabilised masked softmax; a row with no permitted entry is all zero  [WAA 15] */
void orc_masked_softmax(const double *logits, const uint8_t *permitted, int64_t K,
                        double *out) {
  int any = 0;
  double mx = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    if (!permitted[k]) continue;
    if (!any || logits[k] > mx) mx = logits[k];
    any = 1;
  }
  double sum = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    out[k] = permitted[k] ? exp(logits[k] - mx) : 0.0;
    sum += out[k];
  }
  if (any)
    for (int64_t k = 0; k < K; ++k) out[k] /= sum;
}

/* usable iff valid, 0 <= atom_to_token < T, and the mapped token is valid  [WAA 2] */
void orc_usable(const orc_dims *d, const orc_inputs *in, uint8_t *usable) {
  for (int64_t b = 0; b < d->B; ++b)
    for (int64_t a = 0; a < d->A; ++a) {
      int64_t i = b * d->A + a;
      int64_t t = in->atom_to_token[i];
      usable[i] = in->valid[i] && t >= 0 && t < d->T && in->token_valid[b * d->T + t];
    }
}

/* A slot is permitted iff 0 <= key id < A, query and key usable, window_mask,
 * and |key - query| <= radius when radius >= 0; ids are within one batch
 * element  [WAA 4, WAA 5] */
void orc_permitted(const orc_dims *d, const orc_inputs *in, const uint8_t *usable,
                   int64_t radius, uint8_t *permitted) {
  for (int64_t b = 0; b < d->B; ++b)
    for (int64_t a = 0; a < d->A; ++a)
      for (int64_t k = 0; k < d->K; ++k) {
        int64_t s = (b * d->A + a) * d->K + k;
        int64_t j = in->key_index[s];
        int ok = j >= 0 && j < d->A;
        ok = ok && usable[b * d->A + a] && usable[b * d->A + j];
        ok = ok && in->window_mask[s];
        if (ok && radius >= 0) {
          int64_t diff = j - a;
          if (diff < 0) diff = -diff;
          ok = diff <= radius;
        }
        permitted[s] = (uint8_t)ok;
      }
}

/* y[n_out] = x[n_in] @ W[n_in, n_out] (+ bias if given) */
static void vecmat(const double *x, const double *W, const double *bias, int64_t n_in,
                   int64_t n_out, double *y) {
  for (int64_t o = 0; o < n_out; ++o) y[o] = bias ? bias[o] : 0.0;
  for (int64_t i = 0; i < n_in; ++i) {
    double xi = x[i];
    const double *row = W + i * n_out;
    for (int64_t o = 0; o < n_out; ++o) y[o] += xi * row[o];
  }
}

typedef struct {
  double *buf[16];
  int n;
} arena;

static double *grab(arena *ar, int64_t n) {
  double *p = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
  if (p) ar->buf[ar->n++] = p;
  return p;
}

static void arena_free(arena *ar) {
  for (int i = 0; i < ar->n; ++i) free(ar->buf[i]);
  ar->n = 0;
}

/* scratch rows of the calling thread, carved from its slice of tmp */
#define ORC_SCRATCH_ROWS \
  double *r_c = tmp + scratch * orc_tid();              /* clean condition [S] */ \
  double *r_ln = r_c + S;         /* LN(c) or SiLU(c) [S] */ \
  double *r_cj = r_ln + S;        /* LN(c) * cond_scale[j] [S] */ \
  double *r_x = r_cj + S;         /* normalised x [C] */ \
  double *r_sc = r_x + C;         /* scale logits [C] */ \
  double *r_sh = r_sc + C;        /* shift [C] */ \
  double *r_f0 = r_sh + C;        /* query features / shared attention input [C] */ \
  double *r_f1 = r_f0 + C;        /* key/value features [C] */ \
  double *r_m = r_f1 + C;         /* ESMFold2 six vectors [6C] */ \
  double *r_q = r_m + 6 * C;      /* projection before head norm [HD] */ \
  double *r_h = r_q + HD;         /* one head [D] */ \
  double *r_o = r_h + D;          /* attention output [HD] */ \
  double *r_u = r_o + HD;         /* out-projection [C] */ \
  double *r_z = r_u + C;          /* transition input [C] */ \
  double *r_a = r_z + C;          /* z @ w_ff_gate [M] */ \
  double *r_b = r_a + M;          /* z @ w_ff_up [M] */ \
  double *r_ff = r_b + M;         /* transition update [C] */ \
  double *r_pool = r_ff + C;      /* hidden @ w_pool [U] */ \
  double *r_lg = r_pool + U;      /* logits of one row [K] */ \
  double *r_w = r_lg + K;         /* weights of one row [K] */ \
  double *r_pr = r_w + K;         /* LN(pair) [P] */ \
  double *r_tk = r_pr + P;        /* token @ w_token [C] */
#define ORC_SCRATCH_USED (void)r_c; (void)r_ln; (void)r_cj; (void)r_x; (void)r_sc; (void)r_sh; \
  (void)r_f0; (void)r_f1; (void)r_m; (void)r_q; (void)r_h; (void)r_o; (void)r_u; (void)r_z; \
  (void)r_a; (void)r_b; (void)r_ff; (void)r_pool; (void)r_lg; (void)r_w; (void)r_pr; (void)r_tk

int orc_forward(int style, int stage, const orc_dims *d, const orc_inputs *in,
                const orc_params *p, double eps, int64_t radius,
                const uint8_t *query_select, orc_outputs *out) {
  if (style != ORC_STYLE_AF3 && style != ORC_STYLE_ESMFOLD2) return ORC_ERR_ARG;
  if (stage != ORC_STAGE_DECODER && stage != ORC_STAGE_ENCODER) return ORC_ERR_ARG;
  const int af3 = style == ORC_STYLE_AF3, enc = stage == ORC_STAGE_ENCODER;
  const int64_t B = d->B, A = d->A, T = d->T, K = d->K, C = d->C, S = d->S, H = d->H,
                D = d->D, P = d->P, M = d->M, U = d->U, V = d->V, HD = H * D;
  /* dims >= 1, D even for ESMFold2, eps > 0, radius >= -1  [WAA 1, WAA 2, WAA 12] */
  if (B < 1 || A < 1 || T < 1 || K < 1 || C < 1 || S < 1 || H < 1 || D < 1 || M < 1)
    return ORC_ERR_DIM;
  if (enc && U < 1) return ORC_ERR_DIM;
  if (!enc && V < 1) return ORC_ERR_DIM;
  if (af3 && P < 1) return ORC_ERR_DIM;
  if (!af3 && (D % 2) != 0) return ORC_ERR_DIM;
  if (!(eps > 0.0) || !isfinite(eps)) return ORC_ERR_EPS;
  if (radius < -1) return ORC_ERR_RADIUS;
  if (!in->atom || !in->condition || !in->valid || !in->token_valid || !in->window_mask ||
      !in->key_index || !in->atom_to_token || !out->hidden || !out->attention)
    return ORC_ERR_ARG;
  if (af3 && (!in->pair || !p->cond_scale || !p->w_scale || !p->b_scale || !p->w_shift ||
              !p->w_residual_gate || !p->b_residual_gate || !p->b_q || !p->pair_scale ||
              !p->w_pair))
    return ORC_ERR_ARG;
  if (!af3 && (!p->w_mod || !in->rope_cos || !in->rope_sin)) return ORC_ERR_ARG;
  if (!p->w_q || !p->w_k || !p->w_v || !p->w_value_gate || !p->w_attention_out ||
      !p->w_ff_gate || !p->w_ff_up || !p->w_ff_out)
    return ORC_ERR_ARG;
  if (enc && (!p->w_pool || !out->token_output)) return ORC_ERR_ARG;
  if (!enc && (!in->token || !p->w_token || !p->readout_scale || !p->w_readout ||
               !out->position_update || (!af3 && !p->readout_bias)))
    return ORC_ERR_ARG;

  const double inv_sqrt_d = 1.0 / sqrt((double)D);
  const int64_t GW = p->value_gate_per_head ? H : HD; /* value-gate logit width */

  uint8_t *usable = (uint8_t *)malloc((size_t)(B * A));
  uint8_t *perm = (uint8_t *)malloc((size_t)(B * A * K));
  uint8_t *need = (uint8_t *)malloc((size_t)A);
  if (!usable || !perm || !need) {
    free(usable); free(perm); free(need);
    return ORC_ERR_NOMEM;
  }
  orc_usable(d, in, usable);
  orc_permitted(d, in, usable, radius, perm);

  arena ar = {{0}, 0};
  double *x = grab(&ar, A * C);        /* residual state per atom */
  double *Q = grab(&ar, A * HD), *Kf = grab(&ar, A * HD), *Vf = grab(&ar, A * HD);
  double *G = grab(&ar, A * GW);
  double *g0 = grab(&ar, A * C), *g1 = grab(&ar, A * C);    /* residual gates */
  double *tsc = grab(&ar, A * C), *tsh = grab(&ar, A * C);  /* transition scale/shift */
  const int nthr = orc_nthreads();
  /* per thread; covers every row carved below (3S + 15C + 2HD + D + 2M + U + 2K + P) */
  const int64_t scratch = 16 * (C + S + HD + D + M + U + V + P + K) + 64;
  double *tmp = grab(&ar, scratch * nthr);
  double *pooled = enc ? grab(&ar, T * U) : NULL;
  int64_t *count = enc ? (int64_t *)malloc((size_t)T * sizeof(int64_t)) : NULL;
  uint8_t *tok_ok = enc ? (uint8_t *)malloc((size_t)T) : NULL;
  int fail = (ar.n != 10 + (enc ? 1 : 0)) || (enc && (!count || !tok_ok));
  for (int i = 0; i < ar.n && !fail; ++i) fail = ar.buf[i] == NULL;
  if (fail) {
    arena_free(&ar); free(usable); free(perm); free(need); free(count); free(tok_ok);
    return ORC_ERR_NOMEM;
  }

  for (int64_t b = 0; b < B; ++b) {
    const uint8_t *use = usable + b * A;
    const uint8_t *sel = query_select ? query_select + b * A : NULL;
    const uint8_t *pm = perm + b * A * K;
    const int64_t *kid = in->key_index + b * A * K;
    const int64_t *att = in->atom_to_token + b * A;

    /* atoms whose features are needed: selected queries and their permitted keys */
    for (int64_t a = 0; a < A; ++a) need[a] = 0;
    for (int64_t a = 0; a < A; ++a) {
      if (sel && !sel[a]) continue;
      need[a] = 1;
      for (int64_t k = 0; k < K; ++k)
        if (pm[a * K + k]) need[kid[a * K + k]] = 1;
    }

    /* ---- residual start and conditioning for every needed usable atom ---- */
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t a = 0; a < A; ++a) {
      ORC_SCRATCH_ROWS
      ORC_SCRATCH_USED;
      if (!need[a] || !use[a]) continue;
      const int64_t ia = b * A + a;
      /* sanitised payloads: an unusable atom is never reached here, so the
       * select below is the usable branch  [WAA 3] */
      const double *atom_row = in->atom + ia * C;
      double *xa = x + a * C;
      if (enc) {
        for (int64_t c = 0; c < C; ++c) xa[c] = atom_row[c];          /* x = atom */
      } else {
        /* x = skip + gather(token @ w_token, atom_to_token), bias free  [WAA 3] */
        vecmat(in->token + (b * T + att[a]) * V, p->w_token, NULL, V, C, r_tk);
        for (int64_t c = 0; c < C; ++c) xa[c] = atom_row[c] + r_tk[c];
      }
      for (int64_t s = 0; s < S; ++s) r_c[s] = in->condition[ia * S + s];

      if (af3) {
        /* A_j(z, c) = LN(z) * sigmoid(c_j @ w_scale[j] + b_scale[j]) + c_j @ w_shift[j],
         * c_j = LN(c) * cond_scale[j]; j = 0 query, 1 key/value, 2 transition  [WAA 7] */
        orc_layer_norm(r_c, S, eps, r_ln);
        orc_layer_norm(xa, C, eps, r_x);
        for (int j = 0; j < 3; ++j) {
          for (int64_t s = 0; s < S; ++s) r_cj[s] = r_ln[s] * p->cond_scale[j * S + s];
          vecmat(r_cj, p->w_scale + j * S * C, p->b_scale + j * C, S, C, r_sc);
          vecmat(r_cj, p->w_shift + j * S * C, NULL, S, C, r_sh);
          if (j < 2) {
            double *f = j == 0 ? r_f0 : r_f1;
            for (int64_t c = 0; c < C; ++c) f[c] = r_x[c] * orc_sigmoid(r_sc[c]) + r_sh[c];
          } else {
            /* transition stage: kept as scale logits / shift, applied to x' later */
            for (int64_t c = 0; c < C; ++c) {
              tsc[a * C + c] = r_sc[c];
              tsh[a * C + c] = r_sh[c];
            }
          }
        }
        /* residual gates sigmoid(raw condition @ w_residual_gate[j] + b[j])  [WAA 9] */
        vecmat(r_c, p->w_residual_gate, p->b_residual_gate, S, C, g0 + a * C);
        vecmat(r_c, p->w_residual_gate + S * C, p->b_residual_gate + C, S, C, g1 + a * C);
        for (int64_t c = 0; c < C; ++c) {
          g0[a * C + c] = orc_sigmoid(g0[a * C + c]);
          g1[a * C + c] = orc_sigmoid(g1[a * C + c]);
        }
        /* Q from query features with b_q; K, V from key features, no bias; value
         * gate from query features  [WAA 8, WAA 16] */
        vecmat(r_f0, p->w_q, p->b_q, C, HD, Q + a * HD);
        vecmat(r_f1, p->w_k, NULL, C, HD, Kf + a * HD);
        vecmat(r_f1, p->w_v, NULL, C, HD, Vf + a * HD);
        vecmat(r_f0, p->w_value_gate, NULL, C, GW, G + a * GW);
      } else {
        /* six vectors SiLU(condition) @ w_mod[S,6,C], in the order attention shift,
         * scale, gate; transition shift, scale, gate  [WAA 10] */
        for (int64_t s = 0; s < S; ++s) r_ln[s] = orc_silu(r_c[s]);
        vecmat(r_ln, p->w_mod, NULL, S, 6 * C, r_m);
        const double *a_shift = r_m, *a_scale = r_m + C, *a_gate = r_m + 2 * C;
        const double *t_shift = r_m + 3 * C, *t_scale = r_m + 4 * C, *t_gate = r_m + 5 * C;
        /* attention input RMS(x) * (1 + attention_scale) + attention_shift  [WAA 11] */
        orc_rms_norm(xa, C, eps, r_x);
        for (int64_t c = 0; c < C; ++c) r_f0[c] = r_x[c] * (1.0 + a_scale[c]) + a_shift[c];
        /* raw gates, no sigmoid  [WAA 14] */
        for (int64_t c = 0; c < C; ++c) {
          g0[a * C + c] = a_gate[c];
          g1[a * C + c] = t_gate[c];
          tsc[a * C + c] = t_scale[c];
          tsh[a * C + c] = t_shift[c];
        }
        /* bias-free Q/K/V and value gate from the shared input  [ESM RB, WAA 11] */
        vecmat(r_f0, p->w_q, NULL, C, HD, Q + a * HD);
        vecmat(r_f0, p->w_k, NULL, C, HD, Kf + a * HD);
        vecmat(r_f0, p->w_v, NULL, C, HD, Vf + a * HD);
        vecmat(r_f0, p->w_value_gate, NULL, C, GW, G + a * GW);
        /* per-head RMS on Q and K, then half-split rotary before gathering
         * [WAA 12, WAA 13] */
        const double *cs = in->rope_cos + ia * D, *sn = in->rope_sin + ia * D;
        double *mats[2] = {Q + a * HD, Kf + a * HD};
        for (int m = 0; m < 2; ++m)
          for (int64_t h = 0; h < H; ++h) {
            double *vh = mats[m] + h * D;
            orc_rms_norm(vh, D, eps, r_h);
            orc_rope_half_split(r_h, cs, sn, D, vh);
          }
      }
    }

    /* ---- attention, residual, transition per selected query ---- */
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t a = 0; a < A; ++a) {
      ORC_SCRATCH_ROWS
      ORC_SCRATCH_USED;
      if (sel && !sel[a]) continue;
      const int64_t ia = b * A + a;
      for (int64_t h = 0; h < H; ++h) {
        double *arow = out->attention + ((b * H + h) * A + a) * K;
        for (int64_t k = 0; k < K; ++k) {
          r_lg[k] = 0.0;
          if (!pm[a * K + k]) continue;
          int64_t j = kid[a * K + k];
          /* dot(Q_query, K_key) / sqrt(D)  [WAA 15] */
          double dot = 0.0;
          for (int64_t e = 0; e < D; ++e) dot += Q[a * HD + h * D + e] * Kf[j * HD + h * D + e];
          double lg = dot * inv_sqrt_d;
          if (af3) {
            /* + (LN(pair) * pair_scale) @ w_pair, one value per head  [WAA 8] */
            orc_layer_norm(in->pair + (ia * K + k) * P, P, eps, r_pr);
            double beta = 0.0;
            for (int64_t q = 0; q < P; ++q) beta += r_pr[q] * p->pair_scale[q] * p->w_pair[q * H + h];
            lg += beta;
          }
          r_lg[k] = lg;
        }
        orc_masked_softmax(r_lg, pm + a * K, K, arow);
        /* weighted values; repeated slots are separate terms  [WAA 5, WAA 16] */
        for (int64_t e = 0; e < D; ++e) r_o[h * D + e] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          if (!pm[a * K + k]) continue;
          int64_t j = kid[a * K + k];
          for (int64_t e = 0; e < D; ++e) r_o[h * D + e] += arow[k] * Vf[j * HD + h * D + e];
        }
      }
      double *hid = out->hidden + ia * C;
      if (!use[a]) {
        /* hidden is masked to zero  [WAA 18] */
        for (int64_t c = 0; c < C; ++c) hid[c] = 0.0;
        if (!enc) for (int c = 0; c < 3; ++c) out->position_update[ia * 3 + c] = 0.0;
        continue;
      }
      /* value gate sigmoid(query features @ w_value_gate), flattened head-major
       * (index h*D + e), then w_attention_out without bias  [WAA 16] */
      for (int64_t h = 0; h < H; ++h)
        for (int64_t e = 0; e < D; ++e) {
          double gl = p->value_gate_per_head ? G[a * GW + h] : G[a * GW + h * D + e];
          r_o[h * D + e] *= orc_sigmoid(gl);
        }
      vecmat(r_o, p->w_attention_out, NULL, HD, C, r_u);
      double *xa = x + a * C;
      for (int64_t c = 0; c < C; ++c) hid[c] = xa[c] + g0[a * C + c] * r_u[c];   /* x' */

      /* transition norm on the NEW x: AF3 A_2(x', c); ESMFold2
       * RMS(x') * (1 + transition_scale) + transition_shift  [WAA 17] */
      if (af3) {
        orc_layer_norm(hid, C, eps, r_x);
        for (int64_t c = 0; c < C; ++c)
          r_z[c] = r_x[c] * orc_sigmoid(tsc[a * C + c]) + tsh[a * C + c];
      } else {
        orc_rms_norm(hid, C, eps, r_x);
        for (int64_t c = 0; c < C; ++c)
          r_z[c] = r_x[c] * (1.0 + tsc[a * C + c]) + tsh[a * C + c];
      }
      /* SiLU(z @ w_ff_gate) * (z @ w_ff_up), then w_ff_out, then gated residual  [WAA 17] */
      vecmat(r_z, p->w_ff_gate, NULL, C, M, r_a);
      vecmat(r_z, p->w_ff_up, NULL, C, M, r_b);
      for (int64_t m = 0; m < M; ++m) r_a[m] = orc_silu(r_a[m]) * r_b[m];
      vecmat(r_a, p->w_ff_out, NULL, M, C, r_ff);
      for (int64_t c = 0; c < C; ++c) hid[c] += g1[a * C + c] * r_ff[c];   /* hidden */

      if (!enc) {
        /* position_update = (LN(hidden) * readout_scale [+ readout_bias]) @ w_readout,
         * masked; an update, not coordinates  [WAA 18, WAA 19, WAA 20] */
        orc_layer_norm(hid, C, eps, r_x);
        for (int64_t c = 0; c < C; ++c)
          r_x[c] = r_x[c] * p->readout_scale[c] + (af3 ? 0.0 : p->readout_bias[c]);
        vecmat(r_x, p->w_readout, NULL, C, 3, out->position_update + ia * 3);
      }
    }

    /* ---- encoder pooling: exact per-token mean of ReLU(hidden @ w_pool) over the
     * usable atoms assigned to it; tokens without atoms give zero  [WAA 19] ---- */
    if (enc) {
      ORC_SCRATCH_ROWS
      ORC_SCRATCH_USED;
      for (int64_t t = 0; t < T; ++t) {
        count[t] = 0;
        tok_ok[t] = 1;
        for (int64_t u = 0; u < U; ++u) pooled[t * U + u] = 0.0;
      }
      for (int64_t a = 0; a < A; ++a) {   /* ascending atom order */
        if (!use[a]) continue;
        int64_t t = att[a];
        if (sel && !sel[a]) { tok_ok[t] = 0; continue; }
        vecmat(out->hidden + (b * A + a) * C, p->w_pool, NULL, C, U, r_pool);
        for (int64_t u = 0; u < U; ++u)
          pooled[t * U + u] += r_pool[u] > 0.0 ? r_pool[u] : 0.0;
        count[t] += 1;
      }
      for (int64_t t = 0; t < T; ++t) {
        if (!tok_ok[t]) continue;
        double *orow = out->token_output + (b * T + t) * U;
        for (int64_t u = 0; u < U; ++u)
          orow[u] = count[t] > 0 ? pooled[t * U + u] / (double)count[t] : 0.0;
      }
    }
  }

  arena_free(&ar);
  free(usable); free(perm); free(need); free(count); free(tok_ok);
  return ORC_OK;
}

/* ------------------------------------------------------------------ attention core */

/* permitted(a, k) of one batch element  [WAA 4, WAA 5] */
static int core_permitted(const orc_core_inputs *in, int64_t b, int64_t A, int64_t K,
                          int64_t a, int64_t k, int64_t radius, int64_t *j_out) {
  const int64_t s = (b * A + a) * K + k;
  const int64_t j = in->key_index[s];
  int ok = j >= 0 && j < A && in->usable[b * A + a] && in->usable[b * A + j] &&
           in->window_mask[s];
  if (ok && radius >= 0) ok = (j > a ? j - a : a - j) <= radius;
  *j_out = j;
  return ok;
}

/* the AF3 pair bias of slot row pr for every head: beta[h] = (LN(pr) * pair_scale)
 * @ w_pair[:, h]; y receives LN(pr)  [WAA 8] */
static void core_pair_bias(const double *pr, int64_t P, int64_t H, const double *ps,
                           const double *wp, double eps, double *y, double *beta) {
  orc_layer_norm(pr, P, eps, y);
  for (int64_t h = 0; h < H; ++h) {
    beta[h] = 0.0;
    for (int64_t p = 0; p < P; ++p) beta[h] += y[p] * ps[p] * wp[p * H + h];
  }
}

int orc_attention_core(int style, int64_t B, int64_t A, int64_t K, int64_t H, int64_t D,
                       int64_t P, const orc_core_inputs *in, double eps, int64_t radius,
                       double *attention, double *out) {
  const int af3 = style == ORC_STYLE_AF3;
  if (B < 1 || A < 1 || K < 1 || H < 1 || D < 1 || (af3 && P < 1)) return ORC_ERR_DIM;
  if (!(eps > 0.0) || !isfinite(eps)) return ORC_ERR_EPS;
  if (radius < -1) return ORC_ERR_RADIUS;
  const int64_t HD = H * D;
  const double inv_sqrt_d = 1.0 / sqrt((double)D);
  double *lg = (double *)malloc(sizeof(double) * (size_t)(K * H + K + P + H + 1));
  uint8_t *pm = (uint8_t *)malloc((size_t)K);
  if (!lg || !pm) { free(lg); free(pm); return ORC_ERR_NOMEM; }
  double *bias = lg + K, *y = bias + K * H, *beta = y + P;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t a = 0; a < A; ++a) {
      const int64_t ia = b * A + a;
      for (int64_t k = 0; k < K; ++k) {
        int64_t j;
        pm[k] = (uint8_t)core_permitted(in, b, A, K, a, k, radius, &j);
        for (int64_t h = 0; h < H; ++h) bias[k * H + h] = 0.0;
        if (af3 && pm[k]) {
          core_pair_bias(in->pair + (ia * K + k) * P, P, H, in->pair_scale, in->w_pair, eps, y, beta);
          for (int64_t h = 0; h < H; ++h) bias[k * H + h] = beta[h];
        }
      }
      for (int64_t h = 0; h < H; ++h) {
        double *arow = attention + ((b * H + h) * A + a) * K;
        for (int64_t k = 0; k < K; ++k) {
          lg[k] = 0.0;
          if (!pm[k]) continue;
          const int64_t j = in->key_index[ia * K + k];
          double dot = 0.0;
          for (int64_t e = 0; e < D; ++e) dot += in->q[ia * HD + h * D + e] * in->k[(b * A + j) * HD + h * D + e];
          lg[k] = dot * inv_sqrt_d + bias[k * H + h];
        }
        orc_masked_softmax(lg, pm, K, arow);
        for (int64_t e = 0; e < D; ++e) {
          double o = 0.0;
          for (int64_t k = 0; k < K; ++k) {
            if (!pm[k]) continue;
            const int64_t j = in->key_index[ia * K + k];
            o += arow[k] * in->v[(b * A + j) * HD + h * D + e];
          }
          out[ia * HD + h * D + e] = o * orc_sigmoid(in->g[ia * HD + h * D + e]);
        }
      }
    }
  free(lg);
  free(pm);
  return ORC_OK;
}

/* Reverse-mode derivative of orc_attention_core, step by step in reverse order of the
 * forward above (chain rule of the same definitions). */
int orc_attention_core_backward(int style, int64_t B, int64_t A, int64_t K, int64_t H,
                                int64_t D, int64_t P, const orc_core_inputs *in, double eps,
                                int64_t radius, const double *d_out,
                                const double *d_attention, double *d_q, double *d_k,
                                double *d_v, double *d_g, double *d_pair,
                                double *d_pair_scale, double *d_w_pair) {
  const int af3 = style == ORC_STYLE_AF3;
  if (B < 1 || A < 1 || K < 1 || H < 1 || D < 1 || (af3 && P < 1)) return ORC_ERR_DIM;
  if (!(eps > 0.0) || !isfinite(eps)) return ORC_ERR_EPS;
  if (radius < -1) return ORC_ERR_RADIUS;
  const int64_t HD = H * D;
  const double inv_sqrt_d = 1.0 / sqrt((double)D);
  for (int64_t i = 0; i < B * A * HD; ++i) d_q[i] = d_k[i] = d_v[i] = d_g[i] = 0.0;
  if (af3) {
    for (int64_t i = 0; i < B * A * K * P; ++i) d_pair[i] = 0.0;
    for (int64_t p = 0; p < P; ++p) d_pair_scale[p] = 0.0;
    for (int64_t i = 0; i < P * H; ++i) d_w_pair[i] = 0.0;
  }
  double *buf = (double *)malloc(sizeof(double) * (size_t)(3 * K + K * H + 2 * K * H + 3 * P + H + D + 1));
  uint8_t *pm = (uint8_t *)malloc((size_t)K);
  if (!buf || !pm) { free(buf); free(pm); return ORC_ERR_NOMEM; }
  double *lg = buf, *w = lg + K, *dw = w + K, *bias = dw + K, *dbeta = bias + K * H,
         *y = dbeta + K * H, *dy = y + P, *dx = dy + P, *beta = dx + P, *o = beta + H;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t a = 0; a < A; ++a) {
      const int64_t ia = b * A + a;
      for (int64_t k = 0; k < K; ++k) {
        int64_t j;
        pm[k] = (uint8_t)core_permitted(in, b, A, K, a, k, radius, &j);
        for (int64_t h = 0; h < H; ++h) {
          bias[k * H + h] = 0.0;
          dbeta[k * H + h] = 0.0;
        }
        if (af3 && pm[k]) {
          core_pair_bias(in->pair + (ia * K + k) * P, P, H, in->pair_scale, in->w_pair, eps, y, beta);
          for (int64_t h = 0; h < H; ++h) bias[k * H + h] = beta[h];
        }
      }
      for (int64_t h = 0; h < H; ++h) {
        /* forward of this row again: logits, weights, o */
        for (int64_t k = 0; k < K; ++k) {
          lg[k] = 0.0;
          if (!pm[k]) continue;
          const int64_t j = in->key_index[ia * K + k];
          double dot = 0.0;
          for (int64_t e = 0; e < D; ++e) dot += in->q[ia * HD + h * D + e] * in->k[(b * A + j) * HD + h * D + e];
          lg[k] = dot * inv_sqrt_d + bias[k * H + h];
        }
        orc_masked_softmax(lg, pm, K, w);
        for (int64_t e = 0; e < D; ++e) {
          o[e] = 0.0;
          for (int64_t k = 0; k < K; ++k) {
            if (!pm[k]) continue;
            o[e] += w[k] * in->v[(b * A + in->key_index[ia * K + k]) * HD + h * D + e];
          }
        }
        /* out = o * sigmoid(g): d_g = d_out * o * s (1 - s), d_o = d_out * s */
        for (int64_t e = 0; e < D; ++e) {
          const int64_t c = ia * HD + h * D + e;
          const double sg = orc_sigmoid(in->g[c]);
          d_g[c] = d_out[c] * o[e] * sg * (1.0 - sg);
          o[e] = d_out[c] * sg;   /* o now holds d_o */
        }
        /* o = sum_k w_k v_j: d_w_k = d_o . v_j (+ the weights' own gradient),
         * d_v_j += w_k d_o (each slot separately: repeated keys add up) */
        double sdw = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          dw[k] = 0.0;
          if (!pm[k]) continue;
          const int64_t j = in->key_index[ia * K + k];
          for (int64_t e = 0; e < D; ++e) {
            dw[k] += o[e] * in->v[(b * A + j) * HD + h * D + e];
            d_v[(b * A + j) * HD + h * D + e] += w[k] * o[e];
          }
          if (d_attention) dw[k] += d_attention[((b * H + h) * A + a) * K + k];
          sdw += w[k] * dw[k];
        }
        /* softmax over the permitted slots: d_logit_k = w_k (d_w_k - sum_k' w_k' d_w_k');
         * logit = q . k_j / sqrt(D) + beta */
        for (int64_t k = 0; k < K; ++k) {
          if (!pm[k]) continue;
          const int64_t j = in->key_index[ia * K + k];
          const double dl = w[k] * (dw[k] - sdw);
          for (int64_t e = 0; e < D; ++e) {
            d_q[ia * HD + h * D + e] += dl * in->k[(b * A + j) * HD + h * D + e] * inv_sqrt_d;
            d_k[(b * A + j) * HD + h * D + e] += dl * in->q[ia * HD + h * D + e] * inv_sqrt_d;
          }
          dbeta[k * H + h] = dl;
        }
      }
      if (!af3) continue;
      /* beta_h = sum_p y_p pair_scale_p w_pair[p,h], y = LN(pair row) */
      for (int64_t k = 0; k < K; ++k) {
        if (!pm[k]) continue;
        const double *pr = in->pair + (ia * K + k) * P;
        orc_layer_norm(pr, P, eps, y);
        for (int64_t p = 0; p < P; ++p) {
          dy[p] = 0.0;
          for (int64_t h = 0; h < H; ++h) {
            const double db = dbeta[k * H + h];
            d_w_pair[p * H + h] += db * y[p] * in->pair_scale[p];
            d_pair_scale[p] += db * y[p] * in->w_pair[p * H + h];
            dy[p] += db * in->pair_scale[p] * in->w_pair[p * H + h];
          }
        }
        /* y = (x - mean) / sqrt(var + eps) (population variance):
         * d_x = (d_y - mean(d_y) - y mean(d_y y)) / sqrt(var + eps) */
        double mean = 0.0, var = 0.0, mdy = 0.0, mdyy = 0.0;
        for (int64_t p = 0; p < P; ++p) mean += pr[p];
        mean /= (double)P;
        for (int64_t p = 0; p < P; ++p) var += (pr[p] - mean) * (pr[p] - mean);
        var /= (double)P;
        for (int64_t p = 0; p < P; ++p) {
          mdy += dy[p];
          mdyy += dy[p] * y[p];
        }
        mdy /= (double)P;
        mdyy /= (double)P;
        const double rstd = 1.0 / sqrt(var + eps);
        for (int64_t p = 0; p < P; ++p) dx[p] = (dy[p] - mdy - y[p] * mdyy) * rstd;
        for (int64_t p = 0; p < P; ++p) d_pair[(ia * K + k) * P + p] = dx[p];
      }
    }
  free(buf);
  free(pm);
  return ORC_OK;
}

/* ------------------------------------------------------------------ single to pair */

/* [S2P] one call: every step in the order the Required behavior lists it. */
int orc_single_to_pair(int64_t B, int64_t N, int64_t C, int64_t H, int64_t Dp,
                       const double *x, const uint8_t *mask, const double *norm_scale,
                       const double *norm_bias, const double *weight, const double *bias,
                       const double *out_weight, const double *out_bias,
                       const double *output_scale, const double *output_bias, double eps,
                       int output_norm, double *pair_features, double *output) {
  if (!x || !mask || !norm_scale || !norm_bias || !weight || !bias || !out_weight || !out_bias ||
      !pair_features || !output || (output_norm && (!output_scale || !output_bias)))
    return ORC_ERR_ARG;
  if (B < 1 || N < 1 || C < 1 || H < 1 || Dp < 1) return ORC_ERR_DIM;
  if (!(eps > 0.0) || !isfinite(eps)) return ORC_ERR_EPS;
  const int64_t H2 = 2 * H;
  double *qk = (double *)malloc(sizeof(double) * (size_t)(B * N * H2));
  double *row = (double *)malloc(sizeof(double) * (size_t)C);
  double *ln = (double *)malloc(sizeof(double) * (size_t)C);
  double *f = (double *)malloc(sizeof(double) * (size_t)H2);
  double *o = (double *)malloc(sizeof(double) * (size_t)Dp);
  double *on = (double *)malloc(sizeof(double) * (size_t)Dp);
  if (!qk || !row || !ln || !f || !o || !on) {
    free(qk); free(row); free(ln); free(f); free(o); free(on);
    return ORC_ERR_NOMEM;
  }
  for (int64_t bn = 0; bn < B * N; ++bn) {
    /* bullet 1: features of absent tokens are replaced by zero before normalisation */
    for (int64_t c = 0; c < C; ++c) row[c] = mask[bn] ? x[bn * C + c] : 0.0;
    /* bullet 2: affine population LayerNorm, then the projection */
    orc_layer_norm(row, C, eps, ln);
    for (int64_t c = 0; c < C; ++c) ln[c] = ln[c] * norm_scale[c] + norm_bias[c];
    for (int64_t e = 0; e < H2; ++e) {
      double acc = bias[e];
      for (int64_t c = 0; c < C; ++c) acc += ln[c] * weight[c * H2 + e];
      qk[bn * H2 + e] = acc;
    }
  }
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j) {
        const int64_t pij = (b * N + i) * N + j;
        const double *qi = qk + (b * N + i) * H2, *qj = qk + (b * N + j) * H2;
        const int both = mask[b * N + i] && mask[b * N + j];
        /* bullet 3: q then k; pair(i, j) = [k_i * q_j, q_j - k_i] */
        for (int64_t h = 0; h < H; ++h) {
          f[h] = qi[H + h] * qj[h];
          f[H + h] = qj[h] - qi[H + h];
        }
        /* bullet 4: the readout straight from the pair features */
        for (int64_t e = 0; e < Dp; ++e) {
          double acc = out_bias[e];
          for (int64_t h = 0; h < H2; ++h) acc += f[h] * out_weight[h * Dp + e];
          o[e] = acc;
        }
        /* bullet 5: optional affine LayerNorm of the output */
        if (output_norm) {
          orc_layer_norm(o, Dp, eps, on);
          for (int64_t e = 0; e < Dp; ++e) o[e] = on[e] * output_scale[e] + output_bias[e];
        }
        /* bullet 1: both returned tensors are zero unless both endpoints are present */
        for (int64_t h = 0; h < H2; ++h) pair_features[pij * H2 + h] = both ? f[h] : 0.0;
        for (int64_t e = 0; e < Dp; ++e) output[pij * Dp + e] = both ? o[e] : 0.0;
      }
  free(qk); free(row); free(ln); free(f); free(o); free(on);
  return ORC_OK;
}
