/*
 * atomenc.h -- C ABI of the B200 (sm_100a) windowed atom attention library.
 *
 * One call runs the forward pass of one learned local atom block in AlphaFold3 or
 * ESMFold2 style, with its encoder (per-token pooled output) or decoder (coordinate
 * update) boundary, as defined on the page "Local atom attention, encoder pooling
 * and decoder skip/readout" (windowed_atom_attention), Required behavior; the two
 * encoder pages ("AlphaFold 3 Atom Attention Encoder", "ESMFold 2 Atom Attention
 * Encoder") are its encoder specialisations.
 *
 * Conventions
 *  - Every tensor is described by an atomenc_tensor: a DEVICE pointer, an element
 *    type, a rank and a shape. Strides are in elements; the library accepts only
 *    dense row-major tensors (stride[i] == product of shape[i+1..]) and returns
 *    ATOMENC_ERR_STRIDE otherwise.
 *  - All floating tensors of one call (activations, parameters, outputs) share one
 *    element type, ATOMENC_F32 or ATOMENC_BF16; arithmetic is float32 inside the
 *    kernels (bf16 values are widened exactly). Indices are ATOMENC_I64, masks
 *    ATOMENC_BOOL (one byte, 0 or 1).
 *  - A tensor that the chosen style/stage does not use may be left empty
 *    (data == NULL, ndim == 0); it is not read.
 *  - Ownership: the caller owns every buffer, including the workspace. The library
 *    never allocates device or pinned memory and never writes to an input.
 *  - Streams: atomenc_forward only enqueues work on `stream` and returns; it does
 *    not synchronise. All errors are decided on the host before the first launch,
 *    so a non-zero return means nothing was enqueued. Launch failures reported by
 *    the CUDA runtime are returned as ATOMENC_ERR_CUDA.
 *    Kernels are launched with programmatic stream serialization: the first kernel
 *    of a call may be scheduled while earlier work in the stream finishes, but it
 *    waits for that work before reading or writing memory, so stream order holds.
 *  - Inputs must not alias outputs or the workspace. Calls that share a workspace
 *    must be ordered on one stream.
 *  - Size limits (ATOMENC_ERR_UNSUPPORTED beyond them): D <= 64; S <= 256; AF3 P <= 32
 *    and H <= 32; K <= 8192; A <= 2^31 - 4097.
 *
 * Shapes (B batch, A atoms, T tokens, K key slots, C atom width, S condition width,
 * H heads, D head width, P pair channels, M transition width, U pooled width,
 * V token width). Every weight is applied as x @ W with W stored [in, out]; the
 * pages print no shape table, so these shapes are the reading the formulas give.
 */
#ifndef ATOMENC_H
#define ATOMENC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *atomenc_stream_t; /* a cudaStream_t; NULL = legacy default */

enum atomenc_dtype { ATOMENC_F32 = 0, ATOMENC_BF16 = 1, ATOMENC_I64 = 2, ATOMENC_BOOL = 3 };

/* style: "af3" (default on the windowed page) or "esmfold2" */
enum atomenc_style { ATOMENC_AF3 = 0, ATOMENC_ESMFOLD2 = 1 };
/* stage: "decoder" (default on the windowed page) or "encoder" */
enum atomenc_stage { ATOMENC_DECODER = 0, ATOMENC_ENCODER = 1 };

enum atomenc_status {
  ATOMENC_OK = 0,
  ATOMENC_ERR_NULL = -1,        /* a required tensor, pointer or struct is missing */
  ATOMENC_ERR_STYLE = -2,       /* unknown style or stage */
  ATOMENC_ERR_DTYPE = -3,       /* float types differ, index not int64, mask not bool */
  ATOMENC_ERR_SHAPE = -4,       /* ranks or sizes disagree, a dimension < 1 */
  ATOMENC_ERR_STRIDE = -5,      /* a tensor is not dense row-major */
  ATOMENC_ERR_EPS = -6,         /* eps not finite or not > 0 in the float type */
  ATOMENC_ERR_RADIUS = -7,      /* radius < -1 */
  ATOMENC_ERR_ODD_HEAD = -8,    /* ESMFold2 style with odd D (half-split rotary) */
  ATOMENC_ERR_UNSUPPORTED = -9, /* a size outside what the kernels are built for */
  ATOMENC_ERR_WORKSPACE = -10,  /* workspace NULL, too small or not 256-byte aligned */
  ATOMENC_ERR_CUDA = -11,       /* the CUDA runtime rejected a launch */
  ATOMENC_ERR_TOO_LARGE = -12   /* atomenc_forward_noalloc: the shapes need more scratch
                                   than its fixed device array holds */
};

typedef struct {
  void *data;         /* device pointer */
  int32_t dtype;      /* enum atomenc_dtype */
  int32_t ndim;       /* 0 = empty / not supplied */
  int64_t shape[5];
  int64_t stride[5];  /* elements */
} atomenc_tensor;

/* "activations", "masks" and "structure" dictionaries of the page signatures. */
typedef struct {
  atomenc_tensor atom;          /* [B,A,C] encoder input x / decoder skip */
  atomenc_tensor condition;     /* [B,A,S] per-atom condition */
  atomenc_tensor pair;          /* [B,A,K,P] pair descriptor per query slot (AF3) */
  atomenc_tensor token;         /* [B,T,V] token features (decoder) */
  atomenc_tensor rope_cos;      /* [B,A,D] full-width rotary cos (ESMFold2), shared by heads */
  atomenc_tensor rope_sin;      /* [B,A,D] */
  atomenc_tensor valid;         /* [B,A] bool */
  atomenc_tensor token_valid;   /* [B,T] bool */
  atomenc_tensor window_mask;   /* [B,A,K] bool, True permits the slot */
  atomenc_tensor key_index;     /* [B,A,K] int64 atom ids within the batch element;
                                   ids outside [0,A) are missing slots */
  atomenc_tensor atom_to_token; /* [B,A] int64, any order; out of range = unusable */
} atomenc_inputs;

/* "parameters" dictionary (names follow the page formulas). */
typedef struct {
  atomenc_tensor cond_scale;       /* [3,S]   AF3 */
  atomenc_tensor w_scale;          /* [3,S,C] AF3 */
  atomenc_tensor b_scale;          /* [3,C]   AF3 */
  atomenc_tensor w_shift;          /* [3,S,C] AF3 */
  atomenc_tensor w_residual_gate;  /* [2,S,C] AF3 */
  atomenc_tensor b_residual_gate;  /* [2,C]   AF3 */
  atomenc_tensor w_mod;            /* [S,6,C] ESMFold2 */
  atomenc_tensor w_q;              /* [C,H*D] */
  atomenc_tensor b_q;              /* [H*D]   AF3 */
  atomenc_tensor w_k;              /* [C,H*D] */
  atomenc_tensor w_v;              /* [C,H*D] */
  atomenc_tensor w_value_gate;     /* [C,H*D] */
  atomenc_tensor pair_scale;       /* [P]     AF3 */
  atomenc_tensor w_pair;           /* [P,H]   AF3 (gives H) */
  atomenc_tensor w_attention_out;  /* [H*D,C] */
  atomenc_tensor w_ff_gate;        /* [C,M] */
  atomenc_tensor w_ff_up;          /* [C,M] */
  atomenc_tensor w_ff_out;         /* [M,C] */
  atomenc_tensor w_pool;           /* [C,U]   encoder */
  atomenc_tensor w_token;          /* [V,C]   decoder */
  atomenc_tensor readout_scale;    /* [C]     decoder */
  atomenc_tensor readout_bias;     /* [C]     decoder, ESMFold2 */
  atomenc_tensor w_readout;        /* [C,3]   decoder */
} atomenc_params;

typedef struct {
  atomenc_tensor hidden;           /* [B,A,C]   always */
  atomenc_tensor attention;        /* [B,H,A,K] always; 0 on slots that are not permitted */
  atomenc_tensor token_output;     /* [B,T,U]   encoder only */
  atomenc_tensor position_update;  /* [B,A,3]   decoder only */
} atomenc_outputs;

/*
 * Bytes of device workspace atomenc_forward needs for these shapes (0 on a
 * validation error; the same checks as atomenc_forward, minus eps/radius).
 * The heads count H is taken from w_pair (AF3) or rope_cos's last dim D (ESMFold2).
 */
size_t atomenc_workspace_size(int style, int stage, const atomenc_inputs *in,
                              const atomenc_params *params, const atomenc_outputs *out);

/*
 * Enqueue the forward pass on `stream`.
 *   style, stage  enum atomenc_style / atomenc_stage
 *   eps           > 0; the one stabiliser added inside the square root of every
 *                 LayerNorm and RMS normalisation of the block (windowed page,
 *                 Required behavior, eps bullet)
 *   radius        -1 (no index window) or >= 0: a slot also needs |key - query| <= radius
 *   workspace     device buffer of at least atomenc_workspace_size() bytes, 256-byte
 *                 aligned; contents need not be initialised and are overwritten.
 * Writes every element of out->hidden and out->attention, and of out->token_output
 * (encoder) or out->position_update (decoder). Returns enum atomenc_status.
 */
int atomenc_forward(int style, int stage, const atomenc_inputs *in,
                    const atomenc_params *params, double eps, int64_t radius,
                    const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                    atomenc_stream_t stream);

/*
 * Prepared weights. A forward pass first converts the caller's weight tensors into the
 * layouts its kernels read (bf16 tensor-core images of every projection, hi and lo
 * parts for float32 storage; float32 panels of the small vectors); with weights that
 * stay fixed across calls that step can be done once:
 *   atomenc_weight_image_size        bytes of an image for these shapes (0 on a
 *                                    validation error)
 *   atomenc_prepare_weights          enqueue the conversion into `image` (device buffer
 *                                    of at least that many bytes, 256-byte aligned)
 *   atomenc_prepared_workspace_size  bytes of workspace atomenc_forward_prepared needs
 *                                    (the weight region lives in the image instead)
 *   atomenc_forward_prepared         atomenc_forward reading the weights from `image`;
 *                                    params still describe the weights (shapes are
 *                                    validated) but their data is not read.
 * The arguments are those of atomenc_forward; the image depends on style, stage, the
 * storage type and the weight shapes only, and starts with a key naming them: a pass
 * given an image built for anything else sets status bit 8 (outputs invalid) instead
 * of reading it. Results are bit-identical to atomenc_forward. Returns enum
 * atomenc_status; ATOMENC_ERR_WORKSPACE for a missing, short or unaligned image or
 * workspace.
 */
size_t atomenc_weight_image_size(int style, int stage, const atomenc_inputs *in,
                                 const atomenc_params *params, const atomenc_outputs *out);
size_t atomenc_prepared_workspace_size(int style, int stage, const atomenc_inputs *in,
                                       const atomenc_params *params, const atomenc_outputs *out);
int atomenc_prepare_weights(int style, int stage, const atomenc_inputs *in,
                            const atomenc_params *params, const atomenc_outputs *out,
                            void *image, size_t image_bytes, atomenc_stream_t stream);
int atomenc_forward_prepared(int style, int stage, const atomenc_inputs *in,
                             const atomenc_params *params, const void *image,
                             size_t image_bytes, double eps, int64_t radius,
                             const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                             atomenc_stream_t stream);

/* Phases of one forward pass, in launch order (for atomenc_forward_profiled). */
enum atomenc_phase {
  ATOMENC_PHASE_INPUTS = 0,        /* weight panels, usability, sanitisation, residual start */
  ATOMENC_PHASE_CONDITIONING = 1,  /* AF3 adaptive-norm / gate projections; ESMFold2 w_mod */
  ATOMENC_PHASE_PROJECTIONS = 2,   /* attention inputs, Q/K/V/value gate (+ head RMS, rotary) */
  ATOMENC_PHASE_ATTENTION = 3,     /* the slot-gathered attention kernel alone */
  ATOMENC_PHASE_TRANSITION = 4,    /* out-projection, residual, transition, hidden */
  ATOMENC_PHASE_BOUNDARY = 5,      /* encoder pooling / decoder readout */
  ATOMENC_NUM_PHASES = 6
};

/*
 * atomenc_forward with timing hooks: `events` holds n_events == ATOMENC_NUM_PHASES + 1
 * cudaEvent_t handles created by the caller; events[0] is recorded on `stream` before
 * the first launch and events[i + 1] after phase i, so cudaEventElapsedTime(events[i],
 * events[i + 1]) is the device time of phase i. *n_launches (if not NULL) receives the
 * number of kernels the call launched. Same results and errors as atomenc_forward.
 */
int atomenc_forward_profiled(int style, int stage, const atomenc_inputs *in,
                             const atomenc_params *params, double eps, int64_t radius,
                             const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                             atomenc_stream_t stream, void *const *events, int n_events,
                             int *n_launches);

/*
 * Kinds of kernel one forward pass launches (for atomenc_forward_traced).
 */
enum atomenc_kernel_kind {
  ATOMENC_KERNEL_PREP = 0,        /* weight images, panels, resets (CUDA cores) */
  ATOMENC_KERNEL_GEMM = 1,        /* a tcgen05 projection GEMM with its fused epilogue */
  ATOMENC_KERNEL_TRANSITION = 2,  /* the tcgen05 tail: out-projection .. hidden */
  ATOMENC_KERNEL_ATTENTION = 3,   /* the slot-gathered attention */
  ATOMENC_KERNEL_ROWS = 4,        /* a row kernel on CUDA cores (masking, norms, rotary, readout) */
  ATOMENC_KERNEL_POOL = 5         /* the per-token mean */
};

/*
 * atomenc_forward with an event per kernel: events[0] is recorded on `stream` before
 * the first launch and events[i + 1] right after launch i (these records serialise
 * the kernels: the pass is slightly slower than atomenc_forward); kinds[i] (if kinds
 * is not NULL) receives the enum atomenc_kernel_kind of launch i and *n_launches the
 * number of launches. n_events must exceed the number of launches (a pass launches at
 * most 16 kernels); ATOMENC_ERR_NULL otherwise. Same results as atomenc_forward.
 */
int atomenc_forward_traced(int style, int stage, const atomenc_inputs *in,
                           const atomenc_params *params, double eps, int64_t radius,
                           const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                           atomenc_stream_t stream, void *const *events, int n_events,
                           int *kinds, int *n_launches);

/*
 * Read the device status word that the last forward pass using `workspace` left
 * (waits for `stream`). Bits:
 *   1 = some query tile's keys spanned more rows than the shared-memory stage holds and
 *       were gathered from L2 instead. Not an error: same results, slower.
 *   4 = a bounded wait inside a kernel (a tensor-core completion, a bulk copy, or the
 *       partner CTA of the paired transition) reached its poll limit and gave up. AN
 *       ERROR: the kernel returned without finishing, and hidden, attention and the
 *       pooled / readout outputs of this pass are invalid.
 *   8 = (atomenc_forward_prepared) the weight image was built for another style, stage,
 *       storage type or weight shapes. AN ERROR: the outputs of this pass are invalid.
 * Returns enum atomenc_status (of the read, not of the pass).
 */
int atomenc_get_status(const void *workspace, int *device_status, atomenc_stream_t stream);

/*
 * Test hook of the bounded wait between the two CTAs of a row block in the paired
 * transition kernel (used when row blocks are few): poll_limit = polls of the
 * partner's flag before giving up (0 restores the default), withhold_flags != 0 makes
 * every CTA skip raising its own flag, so that the partner's wait runs out and the pass
 * sets status bit 4 instead of hanging. Process-wide; affects passes enqueued after
 * the call. Leave it at (0, 0) outside tests. Returns ATOMENC_OK. No counterpart on
 * the pages.
 */
int atomenc_debug_peer_wait(uint32_t poll_limit, int withhold_flags);

/*
 * Forward pass that allocates nothing and takes no workspace argument.
 *
 * For callers that cannot call cudaMalloc (or have the library do it): code running
 * inside a CUDA stream capture of another framework, where allocation calls are not
 * allowed; hosts whose memory pool owns all device memory and must not see memory
 * taken behind its back; latency-critical loops that cannot afford the implicit
 * synchronisation an allocation may bring. They pass inputs and outputs as for
 * atomenc_forward; the scratch the pass needs lives in one file-scope device array
 * of ATOMENC_NOALLOC_SCRATCH_BYTES (64 MiB) inside this library, which every GPU that
 * loads the library keeps until the process exits.
 *  - The first call on a device (with that device current) looks up the array's
 *    device address once (cudaGetSymbolAddress); make that first call before any
 *    stream capture. Later calls only enqueue work on `stream`.
 *  - Shapes whose atomenc_workspace_size() exceeds the array are rejected with
 *    ATOMENC_ERR_TOO_LARGE before anything is enqueued.
 *  - All calls share the one array and it keeps the last call's contents; each call
 *    clears what it needs zeroed itself. Two calls whose GPU work overlaps (different
 *    streams without ordering, or different host threads) race on the array: order
 *    them on one stream.
 * No counterpart on the pages; results and other errors are those of atomenc_forward,
 * and atomenc_noalloc_get_status reads the pass's status word.
 */
#define ATOMENC_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
int atomenc_forward_noalloc(int style, int stage, const atomenc_inputs *in,
                            const atomenc_params *params, double eps, int64_t radius,
                            const atomenc_outputs *out, atomenc_stream_t stream);

/*
 * The status word (bits as for atomenc_get_status) that the last atomenc_forward_noalloc
 * pass on the current device left in the library's scratch array; waits for `stream`.
 * Bit 4 means that pass's outputs are invalid. Returns enum atomenc_status.
 */
int atomenc_noalloc_get_status(int *device_status, atomenc_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Gradient of the attention core: the slot-gathered attention of the page "Local atom
 * attention, encoder pooling and decoder skip/readout", Required behavior (slot
 * permission and radius, bullets 4-5; logits q . k / sqrt(D) plus, in AF3 style, the
 * pair bias (LN(pair) * pair_scale) @ w_pair, bullets 8 and 15; masked stable softmax
 * over the permitted slots with repeated slots as separate entries, bullets 5, 6, 15;
 * out = (sum_k w_k v_key) * sigmoid(g), bullet 16), taken from its projections q, k,
 * v and the value-gate logits g. Given d_out (the gradient of out) and optionally
 * d_attention (the gradient of the attention weights), it writes d_q, d_k, d_v, d_g
 * and, in AF3 style, d_pair, d_pair_scale and d_w_pair. A key selected by several
 * slots, of one query or of many, receives the sum of their contributions (the slot
 * bullet: repeated selection accumulates gradients); the sums are formed in 64-bit
 * fixed point (2^-32 resolution, |sum| < 2^31), so the results do not depend on the
 * order of the GPU's work (deterministic).
 * Shapes: q, k, v, g, d_out, d_q, d_k, d_v, d_g [B,A,H*D] (heads = H given; channel
 * h*D + e, as the forward's Q/K/V/value-gate rows; ESMFold2 q and k after the per-head
 * RMS and the rotary); key_index [B,A,K] int64; window_mask [B,A,K] bool; usable [B,A]
 * bool (valid, mapped to a valid token); d_attention [B,H,A,K] (optional); AF3: pair
 * [B,A,K,P], pair_scale [P], w_pair [P,H] and d_pair, d_pair_scale, d_w_pair alike.
 * Float tensors share one type (F32 or BF16; arithmetic float32). Limits: K <= 128,
 * D <= 64, AF3 P <= 32 and H <= 32 (ATOMENC_ERR_UNSUPPORTED beyond). Errors are decided
 * on the host before anything is enqueued.
 */
typedef struct {
  atomenc_tensor q, k, v, g;        /* [B,A,H*D] */
  atomenc_tensor key_index;         /* [B,A,K] int64 */
  atomenc_tensor window_mask;       /* [B,A,K] bool */
  atomenc_tensor usable;            /* [B,A] bool */
  atomenc_tensor pair;              /* [B,A,K,P] AF3 */
  atomenc_tensor pair_scale;        /* [P] AF3 */
  atomenc_tensor w_pair;            /* [P,H] AF3 */
  atomenc_tensor d_out;             /* [B,A,H*D] */
  atomenc_tensor d_attention;       /* [B,H,A,K], optional (empty: zero) */
} atomenc_core_bwd_inputs;

typedef struct {
  atomenc_tensor d_q, d_k, d_v, d_g;              /* [B,A,H*D] */
  atomenc_tensor d_pair;                          /* [B,A,K,P] AF3 */
  atomenc_tensor d_pair_scale, d_w_pair;          /* [P], [P,H] AF3 */
} atomenc_core_bwd_outputs;

/* Workspace bytes (256-byte aligned buffer) for atomenc_attention_backward; 0 if the
 * arguments do not validate. */
size_t atomenc_attention_backward_workspace_size(int style, const atomenc_core_bwd_inputs *in,
                                                 int64_t heads,
                                                 const atomenc_core_bwd_outputs *out);

/* Enqueue the gradient on `stream` (eps and radius as for atomenc_forward); returns
 * ATOMENC_OK or an error code. */
int atomenc_attention_backward(int style, const atomenc_core_bwd_inputs *in, int64_t heads,
                               double eps, int64_t radius, const atomenc_core_bwd_outputs *out,
                               void *workspace, size_t workspace_bytes, atomenc_stream_t stream);

/* Static English text for an atomenc_status code. */
const char *atomenc_strerror(int code);

/* Library version, for the Python binding's load check. */
int atomenc_version(void);

/* ---------------------------------------------------------------------------------
 * Single-to-pair features: the page "ESMFold Single-to-Pair Features"
 * (esmfold_single_to_pair), Required behavior. For every ordered token pair (i, j):
 *   q, k = split(LN_affine(x_sanitised) @ weight + bias)          (q: first H columns)
 *   pair_features[b,i,j] = [k_i * q_j, q_j - k_i]                 [2H]
 *   output[b,i,j]        = pair_features[b,i,j] @ out_weight + out_bias, then (when
 *                          output_norm != 0) an affine LayerNorm with output_scale/bias
 * both zero unless mask[b,i] and mask[b,j]; rows of absent tokens are replaced by zero
 * before the normalisation. Every LayerNorm is the population one with eps inside the
 * square root. Shapes: x [B,N,C]; mask [B,N] bool; norm_scale, norm_bias [C];
 * weight [C,2H], bias [2H]; out_weight [2H,Dp], out_bias [Dp]; output_scale,
 * output_bias [Dp] (only read when output_norm != 0); pair_features [B,N,N,2H] and
 * output [B,N,N,Dp]. Float tensors share one type (F32 or BF16). Limits: C <= 256,
 * 2H <= 256, Dp <= 256, 2H * Dp <= 16384, C * 2H <= 49152
 * (ATOMENC_ERR_UNSUPPORTED beyond).
 * Errors are decided on the host before anything is enqueued, as for atomenc_forward.
 */
typedef struct {
  atomenc_tensor x;     /* [B,N,C] single (per-token) features */
  atomenc_tensor mask;  /* [B,N] bool, true = present */
} atomenc_s2p_inputs;

typedef struct {
  atomenc_tensor norm_scale, norm_bias;      /* [C] */
  atomenc_tensor weight, bias;               /* [C,2H], [2H] */
  atomenc_tensor out_weight, out_bias;       /* [2H,Dp], [Dp] */
  atomenc_tensor output_scale, output_bias;  /* [Dp], output_norm only */
} atomenc_s2p_params;

typedef struct {
  atomenc_tensor pair_features;  /* [B,N,N,2H] */
  atomenc_tensor output;         /* [B,N,N,Dp] */
} atomenc_s2p_outputs;

/* Workspace bytes (256-byte aligned) for atomenc_single_to_pair; 0 if the arguments do
 * not validate. */
size_t atomenc_s2p_workspace_size(const atomenc_s2p_inputs *in, const atomenc_s2p_params *params,
                                  int output_norm, const atomenc_s2p_outputs *out);

/* Enqueue the single-to-pair pass on `stream`; returns ATOMENC_OK or an error code. */
int atomenc_single_to_pair(const atomenc_s2p_inputs *in, const atomenc_s2p_params *params,
                           double eps, int output_norm, const atomenc_s2p_outputs *out,
                           void *workspace, size_t workspace_bytes, atomenc_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* ATOMENC_H */
