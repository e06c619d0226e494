// atomenc.cu -- host side of the C ABI declared in include/atomenc.h: argument checks,
// workspace plan and the launch sequence of the windowed atom attention block.
//
// Order of the steps (page "Local atom attention, encoder pooling and decoder
// skip/readout", Required behavior): usability + sanitisation + residual start
// (bullets 2-3), conditioning (AF3 bullets 7, 9; ESMFold2 bullet 10), attention inputs and
// Q/K/V/value-gate projections (bullets 8, 11-13), slot-gathered attention (bullets 4-6,
// 15-16), out-projection and gated residual (bullet 16), transition (bullet 17), hidden
// (bullet 18), encoder pooling or decoder readout (bullets 18-20).
#include <climits>
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>
#include <type_traits>
#include <utility>

#include "host.cuh"

using namespace atomenc;
using namespace atomenc::host;

namespace atomenc {
namespace host {

std::atomic<uint32_t> g_peer_spin_limit{kPeerSpinLimit};
std::atomic<int> g_peer_withhold{0};

struct SmemLimit {
  const void *fn;
  int dev, bytes;
};
constexpr int kMaxSmemLimits = 512;
SmemLimit g_smem_limits[kMaxSmemLimits];
int g_num_smem_limits = 0;
std::mutex g_smem_limits_mutex;

cudaError_t smem_limit_fn(const void *fn, size_t bytes) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  std::lock_guard<std::mutex> lock(g_smem_limits_mutex);
  int slot = -1;
  for (int i = 0; i < g_num_smem_limits; ++i)
    if (g_smem_limits[i].fn == fn && g_smem_limits[i].dev == dev) slot = i;
  if (slot >= 0 && (int)bytes <= g_smem_limits[slot].bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess || dev < 0) return e;
  if (slot < 0 && g_num_smem_limits < kMaxSmemLimits) {
    slot = g_num_smem_limits++;
    g_smem_limits[slot].fn = fn;
    g_smem_limits[slot].dev = dev;
  }
  if (slot >= 0) g_smem_limits[slot].bytes = (int)bytes;
  return e;
}

}  // namespace host
}  // namespace atomenc

namespace {

constexpr int kVersion = 1;

// Multiprocessors of the current device, looked up once per device.
int g_sm_count[kMaxDevices];
std::mutex g_sm_mutex;
int sm_count() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_sm_mutex);
  if (g_sm_count[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

bool present(const atomenc_tensor &t) { return t.data != nullptr && t.ndim > 0; }

int check_tensor(const atomenc_tensor &t, int dtype, int ndim, const int64_t *shape) {
  if (!present(t)) return ATOMENC_ERR_NULL;
  if (t.dtype != dtype) return ATOMENC_ERR_DTYPE;
  if (t.ndim != ndim) return ATOMENC_ERR_SHAPE;
  for (int i = 0; i < ndim; ++i)
    if (t.shape[i] != shape[i] || shape[i] < 1) return ATOMENC_ERR_SHAPE;
  int64_t st = 1;
  for (int i = ndim - 1; i >= 0; --i) {
    if (t.shape[i] > 1 && t.stride[i] != st) return ATOMENC_ERR_STRIDE;
    st *= t.shape[i];
  }
  return ATOMENC_OK;
}

#define CHECK(expr)                 \
  do {                              \
    int _rc = (expr);               \
    if (_rc != ATOMENC_OK) return _rc; \
  } while (0)

float bf16_round_host(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  std::memcpy(&f, &u, 4);
  return f;
}

size_t take(size_t &cur, size_t bytes) {
  size_t o = cur;
  cur += (bytes + 255) & ~size_t(255);
  return o;
}

// radius_hint: the pass's radius, when known (it only steers the attention tile size;
// the workspace size does not depend on it)
int validate(int style, int stage, const atomenc_inputs *in, const atomenc_params *p,
             const atomenc_outputs *out, Plan &pl, int64_t radius_hint = -1) {
  if (!in || !p || !out) return ATOMENC_ERR_NULL;
  if (style != ATOMENC_AF3 && style != ATOMENC_ESMFOLD2) return ATOMENC_ERR_STYLE;
  if (stage != ATOMENC_DECODER && stage != ATOMENC_ENCODER) return ATOMENC_ERR_STYLE;
  pl.style = style;
  pl.stage = stage;
  pl.af3 = style == ATOMENC_AF3;
  pl.enc = stage == ATOMENC_ENCODER;
  Dims &d = pl.d;
  if (!present(in->atom) || !present(in->condition) || !present(in->key_index) ||
      !present(in->token_valid))
    return ATOMENC_ERR_NULL;
  if (in->atom.ndim != 3 || in->condition.ndim != 3 || in->key_index.ndim != 3 ||
      in->token_valid.ndim != 2)
    return ATOMENC_ERR_SHAPE;
  const int fdt = in->atom.dtype;
  if (fdt != ATOMENC_F32 && fdt != ATOMENC_BF16) return ATOMENC_ERR_DTYPE;
  pl.fdt = fdt;
  d.B = in->atom.shape[0];
  d.A = in->atom.shape[1];
  d.C = in->atom.shape[2];
  d.S = in->condition.shape[2];
  d.K = in->key_index.shape[2];
  d.T = in->token_valid.shape[1];
  if (!present(p->w_q) || p->w_q.ndim != 2) return ATOMENC_ERR_NULL;
  const int64_t HD = p->w_q.shape[1];
  if (pl.af3) {
    if (!present(p->w_pair) || p->w_pair.ndim != 2 || !present(in->pair) || in->pair.ndim != 4)
      return ATOMENC_ERR_NULL;
    d.H = p->w_pair.shape[1];
    d.P = p->w_pair.shape[0];
    if (d.H < 1 || HD % d.H != 0) return ATOMENC_ERR_SHAPE;
    d.D = HD / d.H;
  } else {
    if (!present(in->rope_cos) || in->rope_cos.ndim != 3) return ATOMENC_ERR_NULL;
    d.D = in->rope_cos.shape[2];
    if (d.D < 1 || HD % d.D != 0) return ATOMENC_ERR_SHAPE;
    d.H = HD / d.D;
    if (d.D % 2 != 0) return ATOMENC_ERR_ODD_HEAD;
  }
  if (!present(p->w_ff_gate) || p->w_ff_gate.ndim != 2) return ATOMENC_ERR_NULL;
  d.M = p->w_ff_gate.shape[1];
  if (pl.enc) {
    if (!present(p->w_pool) || p->w_pool.ndim != 2) return ATOMENC_ERR_NULL;
    d.U = p->w_pool.shape[1];
  } else {
    if (!present(in->token) || in->token.ndim != 3) return ATOMENC_ERR_NULL;
    d.V = in->token.shape[2];
  }
  const int64_t B = d.B, A = d.A, T = d.T, K = d.K, C = d.C, S = d.S, H = d.H, D = d.D,
                P = d.P, M = d.M, U = d.U, V = d.V;
  {
    const int64_t s3[] = {B, A, C}, sc[] = {B, A, S}, sk[] = {B, A, K}, sa[] = {B, A},
                  st[] = {B, T};
    CHECK(check_tensor(in->atom, fdt, 3, s3));
    CHECK(check_tensor(in->condition, fdt, 3, sc));
    CHECK(check_tensor(in->key_index, ATOMENC_I64, 3, sk));
    CHECK(check_tensor(in->window_mask, ATOMENC_BOOL, 3, sk));
    CHECK(check_tensor(in->valid, ATOMENC_BOOL, 2, sa));
    CHECK(check_tensor(in->atom_to_token, ATOMENC_I64, 2, sa));
    CHECK(check_tensor(in->token_valid, ATOMENC_BOOL, 2, st));
  }
  {
    const int64_t cq[] = {C, HD}, oc[] = {HD, C}, cm[] = {C, M}, mc[] = {M, C};
    CHECK(check_tensor(p->w_q, fdt, 2, cq));
    CHECK(check_tensor(p->w_k, fdt, 2, cq));
    CHECK(check_tensor(p->w_v, fdt, 2, cq));
    CHECK(check_tensor(p->w_value_gate, fdt, 2, cq));
    CHECK(check_tensor(p->w_attention_out, fdt, 2, oc));
    CHECK(check_tensor(p->w_ff_gate, fdt, 2, cm));
    CHECK(check_tensor(p->w_ff_up, fdt, 2, cm));
    CHECK(check_tensor(p->w_ff_out, fdt, 2, mc));
  }
  if (pl.af3) {
    const int64_t pr[] = {B, A, K, P}, s3s[] = {3, S}, w3[] = {3, S, C}, b3[] = {3, C},
                  w2[] = {2, S, C}, b2[] = {2, C}, bq[] = {HD}, ps[] = {P}, wp[] = {P, H};
    CHECK(check_tensor(in->pair, fdt, 4, pr));
    CHECK(check_tensor(p->cond_scale, fdt, 2, s3s));
    CHECK(check_tensor(p->w_scale, fdt, 3, w3));
    CHECK(check_tensor(p->b_scale, fdt, 2, b3));
    CHECK(check_tensor(p->w_shift, fdt, 3, w3));
    CHECK(check_tensor(p->w_residual_gate, fdt, 3, w2));
    CHECK(check_tensor(p->b_residual_gate, fdt, 2, b2));
    CHECK(check_tensor(p->b_q, fdt, 1, bq));
    CHECK(check_tensor(p->pair_scale, fdt, 1, ps));
    CHECK(check_tensor(p->w_pair, fdt, 2, wp));
    if (P > kPairMax || H > kAttnHeadsMax) return ATOMENC_ERR_UNSUPPORTED;
  } else {
    const int64_t rp[] = {B, A, D}, wm[] = {S, 6, C};
    CHECK(check_tensor(in->rope_cos, fdt, 3, rp));
    CHECK(check_tensor(in->rope_sin, fdt, 3, rp));
    CHECK(check_tensor(p->w_mod, fdt, 3, wm));
  }
  if (pl.enc) {
    const int64_t cu[] = {C, U}, tu[] = {B, T, U};
    CHECK(check_tensor(p->w_pool, fdt, 2, cu));
    CHECK(check_tensor(out->token_output, fdt, 3, tu));
  } else {
    const int64_t tv[] = {B, T, V}, vc[] = {V, C}, c1[] = {C}, c3[] = {C, 3}, a3[] = {B, A, 3};
    CHECK(check_tensor(in->token, fdt, 3, tv));
    CHECK(check_tensor(p->w_token, fdt, 2, vc));
    CHECK(check_tensor(p->readout_scale, fdt, 1, c1));
    if (!pl.af3) CHECK(check_tensor(p->readout_bias, fdt, 1, c1));
    CHECK(check_tensor(p->w_readout, fdt, 2, c3));
    CHECK(check_tensor(out->position_update, fdt, 3, a3));
  }
  {
    const int64_t hc[] = {B, A, C}, at[] = {B, H, A, K};
    CHECK(check_tensor(out->hidden, fdt, 3, hc));
    CHECK(check_tensor(out->attention, fdt, 4, at));
  }
  if (D > kMaxD || A > INT_MAX - 4096 || K > 8192 || S > kRowsKMax) return ATOMENC_ERR_UNSUPPORTED;

  // ---- workspace plan
  const int64_t R = B * A;
  size_t cur = 0;
  pl.o_status = take(cur, 256);
  pl.o_usable = take(cur, R);
  // x, the conditioning vectors, the AF3 gates and the pooled rows are kept in the
  // storage type (bf16 workloads: bf16)
  const int64_t its = fdt == ATOMENC_BF16 ? 2 : 4;
  pl.o_xstats = take(cur, R * 2 * 4);
  pl.o_cstats = take(cur, pl.af3 ? R * 2 * 4 : 0);
  pl.o_first = take(cur, pl.enc ? B * T * 4 : 0);
  pl.o_last = take(cur, pl.enc ? B * T * 4 : 0);
  pl.o_tp = take(cur, pl.enc ? 0 : B * T * C * 4);
  pl.o_x = take(cur, R * C * its);
  pl.o_cond = take(cur, R * 6 * C * its);
  pl.o_gate = take(cur, pl.af3 ? R * 2 * C * its : 0);
  const bool fused = C <= kRowsKMax;
  pl.o_feat = take(cur, fused ? 0 : R * (pl.af3 ? 2 : 1) * C * 4);
  // row-gather attention: whole rows of all heads per quarter-warp (H*D == 128, a head
  // spans a whole number of lanes, at most 8 heads, K <= 128), for bf16 storage, and for
  // float32 storage only on small problems (above a few thousand atoms the per-(query,
  // head) kernel measured faster with float32 rows)
  {
    const int64_t lc = HD / 8;
    pl.rg = (fdt == ATOMENC_BF16 || B * A <= kRowAttnF32MaxAtoms) && HD == 128 && D >= lc && D % lc == 0 &&
            HD / D <= kRowAttnHeadsMax && K <= kRowAttnKMax && (!pl.af3 || P <= kRowAttnPairMax) &&
            B * A < INT_MAX;
    pl.ws_bf16 = pl.rg && fdt == ATOMENC_BF16;
  }
  const int64_t wsz = pl.ws_bf16 ? 2 : 4;   // bytes per Q/K/V/G/O element
  pl.o_q = take(cur, R * HD * wsz);
  pl.o_k = take(cur, R * HD * wsz);
  pl.o_v = take(cur, R * HD * wsz);
  pl.o_g = take(cur, R * HD * wsz);
  pl.o_o = take(cur, R * HD * wsz);
  // the fused tail (out-projection .. hidden in one kernel) keeps x', z and the SwiGLU
  // intermediate on chip
  pl.fuse_tail = C == 128 && (HD == 64 || HD == 128) && M % 128 == 0;
  // few row blocks: two CTAs per row block, each on half of the SwiGLU width (all CTAs
  // fit on the GPU at once, one per SM)
  const int64_t nrb = (R + kUmmaBM - 1) / kUmmaBM;
  pl.sms = sm_count();
  pl.tail_pair = pl.fuse_tail && 2 * nrb <= pl.sms;
  pl.o_xfer = take(cur, pl.tail_pair ? nrb * 2 * 128 * 64 * 4 : 0);
  pl.o_xflag = take(cur, pl.tail_pair ? nrb * 2 * 4 : 0);
  pl.o_xp = take(cur, pl.fuse_tail ? 0 : R * C * 4);
  pl.o_z = take(cur, pl.fuse_tail ? 0 : R * C * 4);
  pl.o_h = take(cur, pl.fuse_tail ? 0 : R * M * 4);
  pl.o_pool = take(cur, pl.enc ? R * U * its : 0);
  pl.o_wbase = cur;   // from here on: the weight region (panels and images)
  pl.o_wread = take(cur, pl.enc ? 0 : C * 3 * 4);
  pl.o_bscale = take(cur, pl.af3 ? 3 * C * 4 : 0);
  pl.o_brg = take(cur, pl.af3 ? 2 * C * 4 : 0);
  pl.o_bq = take(cur, pl.af3 ? HD * 4 : 0);
  pl.o_wpair = take(cur, pl.af3 ? P * H * 4 : 0);
  pl.o_rscale = take(cur, pl.enc ? 0 : C * 4);
  pl.o_rbias = take(cur, pl.enc ? 0 : C * 4);
  const bool split = fdt == ATOMENC_F32;
  pl.k_cond = take(cur, packed_bytes(S, 6 * C, split));
  pl.k_gate = take(cur, pl.af3 ? packed_bytes(S, 2 * C, split) : 0);
  pl.k_qkv0 = take(cur, packed_bytes(C, (pl.af3 ? 2 : 4) * HD, split));
  pl.k_qkv1 = take(cur, pl.af3 ? packed_bytes(C, 2 * HD, split) : 0);
  pl.k_out = take(cur, packed_bytes(HD, C, split));
  pl.k_ff1 = take(cur, packed_bytes(C, 2 * M, split));
  pl.k_ff2 = take(cur, packed_bytes(M, C, split));
  pl.k_pool = take(cur, pl.enc ? packed_bytes(C, U, split) : 0);
  pl.k_tok = take(cur, pl.enc ? 0 : packed_bytes(V, C, split));
  pl.bytes = cur;

  // ---- attention tile: QT queries per CTA (the grid should cover the SMs), a slot
  // plan, (AF3) the pair-bias table and the Q rows; the K/V stage gets the rest
  const int dmax = D <= 8 ? 8 : D <= 16 ? 16 : D <= 32 ? 32 : 64;
  pl.DP = dmax + 4;  // odd number of 16-byte chunks per staged row: no bank conflicts
  // AF3 tiles share an SM two at a time when their tables fit half the budget
  auto tile = [&](size_t budget, int per_sm) {
    int q = pl.af3 ? 32 : 64;
    const int64_t fill = (B * A + (int64_t)pl.sms * per_sm - 1) / ((int64_t)pl.sms * per_sm);
    if (fill < q) q = (int)(fill < 1 ? 1 : fill);
    while (q > 1 && attn_fixed_smem(q, (int)K, (int)H, (int)(H * D), pl.af3) > budget / 2) q /= 2;
    return q;
  };
  size_t budget = kAttnSmemBudget;
  int qt = tile(budget, 1);
  if (attn_ctas_per_sm(pl.af3) == 2) {
    const size_t half = kAttnSmemBudget / 2 - 1024;
    const int q2 = tile(half, 2);
    if (attn_fixed_smem(q2, (int)K, (int)H, (int)(H * D), pl.af3) + 8 * 1024 <= half) {
      budget = half;
      qt = q2;
    }
  }
  const size_t fixed = attn_fixed_smem(qt, (int)K, (int)H, (int)(H * D), pl.af3);
  if (fixed + 8 * 1024 > budget) return ATOMENC_ERR_UNSUPPORTED;
  pl.QT = qt;
  pl.kv_floats = (int)((budget - fixed) / 4);
  pl.attn_smem = fixed + (size_t)pl.kv_floats * 4;

  if (pl.rg) {
    // queries per tile: the largest power of two (<= 64, and small enough that there are
    // at least as many tiles as SMs) whose shared K/V ring holds the expected key span:
    // the tile plus 2 radius + 1 rows with an index window, the tile plus K otherwise
    const int es = (int)wsz, rb = (int)(HD * es);
    const int64_t fill = (B * A + pl.sms - 1) / pl.sms;
    auto rows_cap = [&](int qq, bool qg) -> int64_t {
      const size_t fx = rowattn_fixed_smem(qq, (int)K, (int)H, es, pl.af3, qg);
      return fx >= kRowAttnSmemBudget ? 0 : (int64_t)((kRowAttnSmemBudget - fx) / (2 * (size_t)rb));
    };
    auto need = [&](int qq) -> int64_t {
      return radius_hint >= 0 ? qq + 2 * radius_hint + 1 : qq + K;
    };
    auto pick = [&](bool qg) {
      int q = 64;
      while (q > 1 && q > fill) q /= 2;
      while (q > 1 && rows_cap(q, qg) < need(q)) q /= 2;
      return q;
    };
    // the tile's Q and value-gate rows go to shared memory too unless that would leave
    // fewer queries per tile than the CTA has warps
    const int q_qg = pick(true), q_plain = pick(false);
    const bool qg = q_qg >= std::min(q_plain, kRowAttnWarps);
    const int q = qg ? q_qg : q_plain;
    if (rows_cap(q, qg) < 1) return ATOMENC_ERR_UNSUPPORTED;
    pl.rg_qt = q;
    pl.rg_qg = qg;
    pl.rg_stage_rows = (int)rows_cap(q, qg);
    pl.rg_smem = rowattn_fixed_smem(q, (int)K, (int)H, es, pl.af3, qg) + 2 * (size_t)pl.rg_stage_rows * rb;
  }
  return ATOMENC_OK;
}

}  // namespace

extern "C" {

size_t atomenc_workspace_size(int style, int stage, const atomenc_inputs *in,
                              const atomenc_params *params, const atomenc_outputs *out) {
  Plan pl;
  if (validate(style, stage, in, params, out, pl) != ATOMENC_OK) return 0;
  return pl.bytes;
}

static int run_impl(int mode, int style, int stage, const atomenc_inputs *in,
                    const atomenc_params *params, double eps, int64_t radius,
                    const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                    void *image, size_t image_bytes, atomenc_stream_t stream, Hooks &hk) {
  Plan pl;
  CHECK(validate(style, stage, in, params, out, pl, radius));
  if (!std::isfinite(eps) || !(eps > 0.0)) return ATOMENC_ERR_EPS;
  float feps = (float)eps;
  if (!(feps > 0.f) || !std::isfinite(feps)) return ATOMENC_ERR_EPS;
  if (pl.fdt == ATOMENC_BF16 && !(bf16_round_host(feps) > 0.f)) return ATOMENC_ERR_EPS;
  if (radius < -1) return ATOMENC_ERR_RADIUS;
  if (mode != kPassPrepare) {
    const size_t need = mode == kPassFull ? pl.bytes : pl.o_wbase;
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
      return ATOMENC_ERR_WORKSPACE;
  }
  if (mode != kPassFull) {
    if (!image || image_bytes < kImageHeader + (pl.bytes - pl.o_wbase) ||
        (reinterpret_cast<uintptr_t>(image) & 255))
      return ATOMENC_ERR_WORKSPACE;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char *ws = static_cast<unsigned char *>(mode == kPassPrepare ? image : workspace);
  unsigned char *img = static_cast<unsigned char *>(image);
  hk.begin(st);
  if (pl.fdt == ATOMENC_F32)
    return launch_all<float>(pl, in, params, feps, radius, out, ws, st, hk, mode, img);
  return launch_all<__nv_bfloat16>(pl, in, params, feps, radius, out, ws, st, hk, mode, img);
}

static int forward_impl(int style, int stage, const atomenc_inputs *in,
                        const atomenc_params *params, double eps, int64_t radius,
                        const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                        atomenc_stream_t stream, Hooks &hk) {
  return run_impl(kPassFull, style, stage, in, params, eps, radius, out, workspace,
                  workspace_bytes, nullptr, 0, stream, hk);
}

size_t atomenc_weight_image_size(int style, int stage, const atomenc_inputs *in,
                                 const atomenc_params *params, const atomenc_outputs *out) {
  Plan pl;
  if (validate(style, stage, in, params, out, pl, -1) != ATOMENC_OK) return 0;
  return kImageHeader + (pl.bytes - pl.o_wbase);
}

size_t atomenc_prepared_workspace_size(int style, int stage, const atomenc_inputs *in,
                                       const atomenc_params *params, const atomenc_outputs *out) {
  Plan pl;
  if (validate(style, stage, in, params, out, pl, -1) != ATOMENC_OK) return 0;
  return pl.o_wbase;
}

int atomenc_prepare_weights(int style, int stage, const atomenc_inputs *in,
                            const atomenc_params *params, const atomenc_outputs *out,
                            void *image, size_t image_bytes, atomenc_stream_t stream) {
  Hooks hk;
  return run_impl(kPassPrepare, style, stage, in, params, 1.0, -1, out, nullptr, 0, image,
                  image_bytes, stream, hk);
}

int atomenc_forward_prepared(int style, int stage, const atomenc_inputs *in,
                             const atomenc_params *params, const void *image,
                             size_t image_bytes, double eps, int64_t radius,
                             const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                             atomenc_stream_t stream) {
  Hooks hk;
  return run_impl(kPassPrepared, style, stage, in, params, eps, radius, out, workspace,
                  workspace_bytes, const_cast<void *>(image), image_bytes, stream, hk);
}

int atomenc_forward(int style, int stage, const atomenc_inputs *in, const atomenc_params *params,
                    double eps, int64_t radius, const atomenc_outputs *out, void *workspace,
                    size_t workspace_bytes, atomenc_stream_t stream) {
  Hooks hk;
  return forward_impl(style, stage, in, params, eps, radius, out, workspace, workspace_bytes,
                      stream, hk);
}

int atomenc_forward_profiled(int style, int stage, const atomenc_inputs *in,
                             const atomenc_params *params, double eps, int64_t radius,
                             const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                             atomenc_stream_t stream, void *const *events, int n_events,
                             int *n_launches) {
  if (!events || n_events != ATOMENC_NUM_PHASES + 1) return ATOMENC_ERR_NULL;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return ATOMENC_ERR_NULL;
  Hooks hk;
  hk.ev = reinterpret_cast<cudaEvent_t const *>(events);
  int rc = forward_impl(style, stage, in, params, eps, radius, out, workspace, workspace_bytes,
                        stream, hk);
  if (n_launches) *n_launches = hk.launches;
  return rc;
}

int atomenc_forward_traced(int style, int stage, const atomenc_inputs *in,
                           const atomenc_params *params, double eps, int64_t radius,
                           const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                           atomenc_stream_t stream, void *const *events, int n_events,
                           int *kinds, int *n_launches) {
  if (!events || n_events < 2) return ATOMENC_ERR_NULL;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return ATOMENC_ERR_NULL;
  Hooks hk;
  hk.kev = reinterpret_cast<cudaEvent_t const *>(events);
  hk.n_kev = n_events;
  hk.kinds = kinds;
  int rc = forward_impl(style, stage, in, params, eps, radius, out, workspace, workspace_bytes,
                        stream, hk);
  if (n_launches) *n_launches = hk.launches;
  if (rc == ATOMENC_OK && hk.overflow) return ATOMENC_ERR_NULL;
  return rc;
}

int atomenc_debug_peer_wait(uint32_t poll_limit, int withhold_flags) {
  g_peer_spin_limit.store(poll_limit == 0 ? kPeerSpinLimit : poll_limit);
  g_peer_withhold.store(withhold_flags ? 1 : 0);
  return ATOMENC_OK;
}

// ---- no-allocation variant: scratch in a file-scope device array, address looked up
// once per device with that device current
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATOMENC_NOALLOC_SCRATCH_BYTES];
static void *g_noalloc_addr[kMaxDevices];
static std::mutex g_noalloc_mutex;

static int noalloc_scratch(void **ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATOMENC_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATOMENC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ATOMENC_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *ptr = g_noalloc_addr[dev];
  return ATOMENC_OK;
}

int atomenc_forward_noalloc(int style, int stage, const atomenc_inputs *in,
                            const atomenc_params *params, double eps, int64_t radius,
                            const atomenc_outputs *out, atomenc_stream_t stream) {
  Plan pl;
  CHECK(validate(style, stage, in, params, out, pl));
  if (pl.bytes > ATOMENC_NOALLOC_SCRATCH_BYTES) return ATOMENC_ERR_TOO_LARGE;
  void *scratch = nullptr;
  CHECK(noalloc_scratch(&scratch));
  Hooks hk;
  return forward_impl(style, stage, in, params, eps, radius, out, scratch,
                      ATOMENC_NOALLOC_SCRATCH_BYTES, stream, hk);
}

int atomenc_noalloc_get_status(int *device_status, atomenc_stream_t stream) {
  if (!device_status) return ATOMENC_ERR_NULL;
  void *scratch = nullptr;
  CHECK(noalloc_scratch(&scratch));
  return atomenc_get_status(scratch, device_status, stream);
}

int atomenc_get_status(const void *workspace, int *device_status, atomenc_stream_t stream) {
  if (!workspace || !device_status) return ATOMENC_ERR_NULL;
  unsigned v = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return ATOMENC_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATOMENC_ERR_CUDA;
  *device_status = (int)v;
  return ATOMENC_OK;
}

const char *atomenc_strerror(int code) {
  switch (code) {
    case ATOMENC_OK: return "ok";
    case ATOMENC_ERR_NULL: return "a required tensor, pointer or struct is missing";
    case ATOMENC_ERR_STYLE: return "unknown style or stage";
    case ATOMENC_ERR_DTYPE: return "element types disagree (floats must match; int64 indices; bool masks)";
    case ATOMENC_ERR_SHAPE: return "tensor ranks or sizes disagree, or a dimension is < 1";
    case ATOMENC_ERR_STRIDE: return "a tensor is not dense row-major";
    case ATOMENC_ERR_EPS: return "eps must be finite and > 0 in the float type";
    case ATOMENC_ERR_RADIUS: return "radius must be -1 or >= 0";
    case ATOMENC_ERR_ODD_HEAD: return "ESMFold2 style needs an even head width D";
    case ATOMENC_ERR_UNSUPPORTED: return "a size is outside what the kernels are built for";
    case ATOMENC_ERR_WORKSPACE: return "workspace is NULL, too small or not 256-byte aligned";
    case ATOMENC_ERR_CUDA: return "the CUDA runtime rejected a launch";
    case ATOMENC_ERR_TOO_LARGE:
      return "the shapes need more scratch than the no-allocation entry point's fixed 64 MiB array";
    default: return "unknown atomenc status";
  }
}

int atomenc_version(void) { return kVersion; }

}  // extern "C"
