/*
 * oracle.h -- plain CPU float64 oracle of the windowed (slot-gathered) atom
 * attention block, AF3 and ESMFold2 styles, encoder and decoder stages.
 *
 * TEST INFRASTRUCTURE. This code exists only to check the CUDA library. Only the
 * test suite, the package smoke check and the benchmark's CPU-baseline leg may
 * load it. It shares no code, header, table or helper with the CUDA library, and
 * the CUDA library never calls it.
 *
 * Sources. Citations name the page title and the section on it:
 *   [WAA n]  "Local atom attention, encoder pooling and decoder skip/readout"
 *            (function windowed_atom_attention), Required behavior, bullet n
 *            (bullets counted from 1 in the order printed).
 *   [AF3 ...] "AlphaFold 3 Atom Attention Encoder", Required behavior / Worked example.
 *   [ESM ...] "ESMFold 2 Atom Attention Encoder", Required behavior / Worked example.
 *   [S2P n]  "ESMFold Single-to-Pair Features" (function esmfold_single_to_pair),
 *            Required behavior, bullet n (counted from 1).
 *
 * Readings taken where the pages are silent (dictionary keys and weight shapes are
 * not printed on any page): every weight is applied as x @ W with W stored
 * [in, out] row-major; the shapes are listed beside each field below.
 *
 * All arrays are dense row-major. Floating inputs are float64 (the caller widens
 * fp32 / bf16 values exactly); indices int64; masks one byte per element (0/1).
 */
#ifndef SWA_ORACLE_H
#define SWA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_STYLE_AF3 = 0, ORC_STYLE_ESMFOLD2 = 1 };
enum { ORC_STAGE_DECODER = 0, ORC_STAGE_ENCODER = 1 };

enum {
  ORC_OK = 0,
  ORC_ERR_ARG = -1,     /* null pointer that the style/stage needs, bad enum */
  ORC_ERR_DIM = -2,     /* a dimension < 1, or odd D in ESMFold2 style */
  ORC_ERR_EPS = -3,     /* eps not finite or not > 0 */
  ORC_ERR_RADIUS = -4,  /* radius < -1 */
  ORC_ERR_NOMEM = -5
};

typedef struct {
  int64_t B, A, T, K;   /* batch, atoms, tokens, key slots per query */
  int64_t C, S;         /* atom width, condition width */
  int64_t H, D;         /* heads, head width */
  int64_t P;            /* pair channels (AF3) */
  int64_t M, U, V;      /* transition hidden, pooled width (encoder), token width (decoder) */
} orc_dims;

typedef struct {
  const double *atom;        /* [B,A,C] encoder input / decoder skip */
  const double *condition;   /* [B,A,S] */
  const double *pair;        /* [B,A,K,P] AF3 only */
  const double *token;       /* [B,T,V] decoder only */
  const double *rope_cos;    /* [B,A,D] ESMFold2 only (broadcast over heads) */
  const double *rope_sin;    /* [B,A,D] */
  const uint8_t *valid;      /* [B,A] */
  const uint8_t *token_valid;/* [B,T] */
  const uint8_t *window_mask;/* [B,A,K] */
  const int64_t *key_index;  /* [B,A,K] within-batch atom ids; out of range = missing */
  const int64_t *atom_to_token; /* [B,A] */
} orc_inputs;

typedef struct {
  /* AF3 conditioning */
  const double *cond_scale;       /* [3,S] */
  const double *w_scale;          /* [3,S,C] */
  const double *b_scale;          /* [3,C] */
  const double *w_shift;          /* [3,S,C] */
  const double *w_residual_gate;  /* [2,S,C] */
  const double *b_residual_gate;  /* [2,C] */
  /* ESMFold2 conditioning */
  const double *w_mod;            /* [S,6,C] */
  /* attention */
  const double *w_q;              /* [C,H*D] */
  const double *b_q;              /* [H*D]  AF3 only */
  const double *w_k;              /* [C,H*D] */
  const double *w_v;              /* [C,H*D] */
  const double *w_value_gate;     /* [C,H*D], or [C,H] when value_gate_per_head */
  const double *pair_scale;       /* [P]   AF3 only */
  const double *w_pair;           /* [P,H] AF3 only */
  const double *w_attention_out;  /* [H*D,C] */
  /* transition */
  const double *w_ff_gate;        /* [C,M] */
  const double *w_ff_up;          /* [C,M] */
  const double *w_ff_out;         /* [M,C] */
  /* encoder boundary */
  const double *w_pool;           /* [C,U] */
  /* decoder boundary */
  const double *w_token;          /* [V,C] */
  const double *readout_scale;    /* [C] */
  const double *readout_bias;     /* [C] ESMFold2 only */
  const double *w_readout;        /* [C,3] */
  int32_t value_gate_per_head;    /* 1: w_value_gate is [C,H], one gate per head */
} orc_params;

typedef struct {
  double *hidden;           /* [B,A,C] */
  double *attention;        /* [B,H,A,K] */
  double *token_output;     /* [B,T,U] encoder */
  double *position_update;  /* [B,A,3] decoder */
} orc_outputs;

/* Scalar and row helpers, exported so that the tests can pin each one alone. */
double orc_sigmoid(double z);
double orc_silu(double z);
void orc_layer_norm(const double *v, int64_t n, double eps, double *out);
void orc_rms_norm(const double *v, int64_t n, double eps, double *out);
void orc_rope_half_split(const double *q, const double *cosv, const double *sinv,
                         int64_t D, double *out);
/* Masked softmax over one row of K logits: permitted[k] selects the entries. */
void orc_masked_softmax(const double *logits, const uint8_t *permitted, int64_t K,
                        double *out);
/* usable[B*A] (0/1) for every atom. */
void orc_usable(const orc_dims *d, const orc_inputs *in, uint8_t *usable);
/* permitted[B*A*K] (0/1) for every slot; needs usable from orc_usable. */
void orc_permitted(const orc_dims *d, const orc_inputs *in, const uint8_t *usable,
                   int64_t radius, uint8_t *permitted);

/*
 * Full forward pass. query_select (optional, [B,A] bytes): when non-null only the
 * selected query atoms get their attention rows, hidden rows and position updates
 * written, and a token's output row is written only when every usable atom mapped
 * to it is selected; every other output element is left untouched. The values
 * written do not depend on the selection.
 */
int orc_forward(int style, int stage, const orc_dims *d, const orc_inputs *in,
                const orc_params *p, double eps, int64_t radius,
                const uint8_t *query_select, orc_outputs *out);

/*
 * The attention core of the block on its own, given the projections (the gradient
 * check of the core runs through these two functions).
 *   [WAA 4, 5]   slot (a, k) of batch element b is permitted iff its key id j is in
 *                [0, A), usable[a] and usable[j], window_mask, and |j - a| <= radius
 *                when radius >= 0;
 *   [WAA 8, 15]  logit = q_a,h . k_j,h / sqrt(D) (+ AF3 pair bias
 *                (LN(pair[a,k]) * pair_scale) @ w_pair[:, h]); masked stable softmax
 *                over the permitted slots, a row without any is all zero; repeated
 *                slots are separate terms;
 *   [WAA 16]     o_a,h = sum_k w_k v_j,h, then out = o * sigmoid(g) per channel.
 * q, k, v, g [B,A,H*D] (head-major channels h*D + e; ESMFold2 q and k are the rows
 * after the per-head RMS and the rotary); pair [B,A,K,P], pair_scale [P], w_pair [P,H]
 * only for AF3 (style 0). Writes attention [B,H,A,K] and out [B,A,H*D].
 */
typedef struct {
  const double *q, *k, *v, *g;  /* [B,A,H*D] */
  const double *pair;           /* [B,A,K,P] AF3 */
  const double *pair_scale;     /* [P] AF3 */
  const double *w_pair;         /* [P,H] AF3 */
  const int64_t *key_index;     /* [B,A,K] */
  const uint8_t *window_mask;   /* [B,A,K] */
  const uint8_t *usable;        /* [B,A] */
} orc_core_inputs;

int orc_attention_core(int style, int64_t B, int64_t A, int64_t K, int64_t H, int64_t D,
                       int64_t P, const orc_core_inputs *in, double eps, int64_t radius,
                       double *attention, double *out);

/*
 * Gradient of the attention core: given d_out [B,A,H*D] (and, when not NULL,
 * d_attention [B,H,A,K], the gradient reaching the attention weights output), writes
 * d_q, d_k, d_v, d_g [B,A,H*D] and for AF3 d_pair [B,A,K,P], d_pair_scale [P],
 * d_w_pair [P,H] (all overwritten). A key selected by several slots, of one query or
 * of many, receives the sum of their contributions ([WAA 5]: repeated selection
 * accumulates gradients); slots that are not permitted contribute nothing and their
 * pair rows get zero gradient.
 */
int orc_attention_core_backward(int style, int64_t B, int64_t A, int64_t K, int64_t H,
                                int64_t D, int64_t P, const orc_core_inputs *in, double eps,
                                int64_t radius, const double *d_out,
                                const double *d_attention, double *d_q, double *d_k,
                                double *d_v, double *d_g, double *d_pair,
                                double *d_pair_scale, double *d_w_pair);

/*
 * Single-to-pair features [S2P 1-6]. x [B,N,C], mask [B,N] (1 = present);
 * norm_scale, norm_bias [C]; weight [C,2H], bias [2H] (columns 0..H-1 give q, H..2H-1
 * give k); out_weight [2H,Dp], out_bias [Dp]; output_scale, output_bias [Dp] (read only
 * when output_norm != 0). Writes pair_features [B,N,N,2H] = [k_i * q_j, q_j - k_i] and
 * output [B,N,N,Dp] = pair_features @ out_weight + out_bias (then the affine LayerNorm
 * when output_norm), both zero unless tokens i and j are present.
 */
int orc_single_to_pair(int64_t B, int64_t N, int64_t C, int64_t H, int64_t Dp,
                       const double *x, const uint8_t *mask, const double *norm_scale,
                       const double *norm_bias, const double *weight, const double *bias,
                       const double *out_weight, const double *out_bias,
                       const double *output_scale, const double *output_bias, double eps,
                       int output_norm, double *pair_features, double *output);

#ifdef __cplusplus
}
#endif
#endif
