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

#include "../../include/atomenc.h"
#include "attention.cuh"
#include "attn_rows.cuh"
#include "common.cuh"
#include "epilogues.cuh"
#include "gemm_umma.cuh"
#include "rows.cuh"
#include "transition.cuh"
#include "weights.cuh"

using namespace atomenc;

namespace {

constexpr int kVersion = 1;
constexpr int kMaxD = 64;
constexpr size_t kAttnSmemBudget = 210 * 1024;  // dynamic part: one CTA per SM, or per two (AF3) / 2 - 1 KB
constexpr size_t kRowAttnSmemBudget = 220 * 1024;  // dynamic part of the row-gather attention

struct Dims {
  int64_t B = 0, A = 0, T = 0, K = 0, C = 0, S = 0, H = 0, D = 0, P = 0, M = 0, U = 0, V = 0;
};

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

constexpr int kMaxDevices = 64;

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

struct Plan {
  int style = 0, stage = 0, fdt = 0;
  bool af3 = false, enc = false, fuse_tail = false, tail_pair = false;
  Dims d;
  // workspace layout (byte offsets)
  size_t o_status, o_usable, o_xstats, o_cstats, o_first, o_last, o_tp, o_x, o_cond, o_gate, o_feat,
      o_q, o_k, o_v, o_g, o_o, o_xp, o_z, o_h, o_pool, o_xfer, o_xflag;
  size_t o_wread, o_bscale, o_brg, o_bq, o_wpair, o_rscale, o_rbias;
  // tensor-core images of the weight panels (bf16, hi[/lo])
  size_t k_cond, k_gate, k_qkv0, k_qkv1, k_out, k_ff1, k_ff2, k_pool, k_tok;
  size_t bytes = 0;
  // attention launch
  int QT = 0, DP = 0, kv_floats = 0;
  size_t attn_smem = 0;
  int sms = 148;                    // multiprocessors of the device the pass runs on
  // row-gather attention (k_attn_rows): H*D in {64, 128} ... see attn_rows.cuh; Q, K, V,
  // value-gate logits and the gated output are then kept in the storage type
  bool rg = false;
  int rg_qt = 0, rg_stage_rows = 0;
  size_t rg_smem = 0;
  bool ws_bf16 = false;             // Q/K/V/G/O intermediates in bf16
};

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
  // spans a whole number of lanes, at most 8 heads, K <= 128)
  {
    const int64_t lc = HD / 8;
    pl.rg = HD == 128 && D >= lc && D % lc == 0 && HD / D <= kRowAttnHeadsMax &&
            K <= kRowAttnKMax && (!pl.af3 || P <= kRowAttnPairMax);
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
    // queries per CTA: the largest power of two (<= 64, and small enough that the grid
    // covers the SMs) whose shared K/V stage holds the expected key span: the tile plus
    // 2 radius + 1 rows with an index window, the tile plus K otherwise
    const int es = (int)wsz, rb = (int)(HD * es);
    const int64_t fill = (B * A + pl.sms - 1) / pl.sms;
    int q = 64;
    while (q > 1 && q > fill) q /= 2;
    auto rows_cap = [&](int qq) -> int64_t {
      const size_t fx = rowattn_fixed_smem(qq, (int)K, (int)H, es, pl.af3);
      return fx >= kRowAttnSmemBudget ? 0 : (int64_t)((kRowAttnSmemBudget - fx) / (2 * (size_t)rb));
    };
    auto need = [&](int qq) -> int64_t {
      return radius_hint >= 0 ? qq + 2 * radius_hint + 1 : qq + K;
    };
    while (q > 1 && rows_cap(q) < need(q)) q /= 2;
    if (rows_cap(q) < 1) return ATOMENC_ERR_UNSUPPORTED;
    pl.rg_qt = q;
    pl.rg_stage_rows = (int)rows_cap(q);
    pl.rg_smem = rowattn_fixed_smem(q, (int)K, (int)H, es, pl.af3) + 2 * (size_t)pl.rg_stage_rows * rb;
  }
  return ATOMENC_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), and again only
// if a larger size is asked for: the attribute outlives the call, so repeating it on
// every forward would only add host time.
struct SmemLimit {
  const void *fn;
  int dev, bytes;
};
constexpr int kMaxSmemLimits = 512;
SmemLimit g_smem_limits[kMaxSmemLimits];
int g_num_smem_limits = 0;
std::mutex g_smem_limits_mutex;

template <typename... KP>
cudaError_t smem_limit(void (*kern)(KP...), size_t bytes) {
  const void *fn = reinterpret_cast<const void *>(kern);
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

struct Hooks {
  cudaEvent_t const *ev = nullptr;  // ATOMENC_NUM_PHASES + 1 events, or null
  cudaEvent_t const *kev = nullptr; // traced: one event before the pass and one per launch
  int n_kev = 0;
  int *kinds = nullptr;             // traced: enum atomenc_kernel_kind per launch
  int launches = 0;
  cudaError_t err = cudaSuccess;    // first launch failure
  bool overflow = false;            // traced: more launches than events
  void mark(int i, cudaStream_t st) const {
    if (ev) cudaEventRecord(ev[i], st);
  }
  void begin(cudaStream_t st) {
    if (kev && n_kev > 0) cudaEventRecord(kev[0], st);
  }
  // Every kernel is launched here, with programmatic stream serialization: it may be
  // scheduled while its predecessor finishes and waits for it in pdl_enter(). A
  // cluster size of 2 launches the grid as CTA pairs that the hardware schedules
  // together.
  template <typename... KP, typename... Args>
  void launch(int kind, void (*kern)(KP...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
              Args &&...args) {
    launch_cluster(kind, 1, kern, grid, block, smem, st, std::forward<Args>(args)...);
  }
  template <typename... KP, typename... Args>
  void launch_cluster(int kind, int cluster, void (*kern)(KP...), dim3 grid, dim3 block,
                      size_t smem, cudaStream_t st, Args &&...args) {
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    int nat = 1;
    if (cluster > 1) {
      at[1].id = cudaLaunchAttributeClusterDimension;
      at[1].val.clusterDim.x = (unsigned)cluster;
      at[1].val.clusterDim.y = 1;
      at[1].val.clusterDim.z = 1;
      nat = 2;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = nat;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    if (kev) {
      if (launches + 1 < n_kev) {
        cudaEventRecord(kev[launches + 1], st);
        if (kinds) kinds[launches] = kind;
      } else {
        overflow = true;
      }
    }
    ++launches;
  }
};

// Test hook for the bounded wait of the paired transition CTAs (see
// atomenc_debug_peer_wait): poll limit, and whether the partials' flags are withheld.
std::atomic<uint32_t> g_peer_spin_limit{kPeerSpinLimit};
std::atomic<int> g_peer_withhold{0};

template <typename Elt>
int launch_all(const Plan &pl, const atomenc_inputs *in, const atomenc_params *p,
               float eps, int64_t radius, const atomenc_outputs *out, unsigned char *ws,
               cudaStream_t st, Hooks &hk) {
  const Dims &d = pl.d;
  const int64_t B = d.B, A = d.A, T = d.T, K = d.K, C = d.C, S = d.S, H = d.H, D = d.D,
                P = d.P, M = d.M, U = d.U, V = d.V, HD = H * D, R = B * A;
  auto F = [&](size_t off) { return reinterpret_cast<float *>(ws + off); };
  unsigned *status = reinterpret_cast<unsigned *>(ws + pl.o_status);
  uint8_t *usable = ws + pl.o_usable;
  int *first = reinterpret_cast<int *>(ws + pl.o_first);
  int *last = reinterpret_cast<int *>(ws + pl.o_last);

  hk.mark(0, st);

  // ---- one launch: tensor-core images of the projection weights (built from the
  // caller's tensors), small float32 panels, status and token-range resets
  WeightJobs wj;
  std::memset(&wj, 0, sizeof(wj));
  const size_t es = sizeof(Elt);
  auto elt = [&](const atomenc_tensor &t, size_t off) -> const void * {
    return t.data ? static_cast<const unsigned char *>(t.data) + off * es : nullptr;
  };
  auto copy = [&](const atomenc_tensor &src, size_t src_off, int64_t rows, int64_t cols, size_t dst_off,
                  int64_t dst_ld, int64_t col0, const atomenc_tensor *rowscale, size_t rs_off) {
    CopyJob &j = wj.copy[wj.ncopy++];
    j.src = elt(src, src_off);
    j.rowscale = rowscale ? elt(*rowscale, rs_off) : nullptr;
    j.dst = F(dst_off);
    j.rows = (int32_t)rows;
    j.cols = (int32_t)cols;
    j.dst_ld = (int32_t)dst_ld;
    j.dst_col0 = (int32_t)col0;
    j.dst_cstride = 1;
  };
  const bool split = pl.fdt == ATOMENC_F32;
  auto pack = [&](size_t dst, int64_t Kd, int64_t N) -> PackJob & {
    PackJob &j = wj.pack[wj.npack++];
    j.dst = ws + dst;
    j.K = (int32_t)Kd;
    j.N = (int32_t)N;
    j.split = split ? 1 : 0;
    return j;
  };
  auto seg = [&](PackJob &j, const atomenc_tensor &src, size_t src_off, int64_t cols, int64_t col0,
                 int cshift, const atomenc_tensor *rowscale, size_t rs_off) {
    PackSeg &g = j.seg[j.nseg++];
    g.src = elt(src, src_off);
    g.rowscale = rowscale ? elt(*rowscale, rs_off) : nullptr;
    g.cols = (int32_t)cols;
    g.col0 = (int32_t)col0;
    g.cshift = cshift;
  };
  if (pl.af3) {
    PackJob &jc = pack(pl.k_cond, S, 6 * C);
    for (int jj = 0; jj < 3; ++jj) {
      seg(jc, p->w_scale, (size_t)jj * S * C, C, 2 * jj * C, 0, &p->cond_scale, (size_t)jj * S);
      seg(jc, p->w_shift, (size_t)jj * S * C, C, 2 * jj * C + C, 0, &p->cond_scale, (size_t)jj * S);
    }
    PackJob &jg = pack(pl.k_gate, S, 2 * C);
    seg(jg, p->w_residual_gate, 0, C, 0, 0, nullptr, 0);
    seg(jg, p->w_residual_gate, (size_t)S * C, C, C, 0, nullptr, 0);
    PackJob &j0 = pack(pl.k_qkv0, C, 2 * HD);
    seg(j0, p->w_q, 0, HD, 0, 0, nullptr, 0);
    seg(j0, p->w_value_gate, 0, HD, HD, 0, nullptr, 0);
    PackJob &j1 = pack(pl.k_qkv1, C, 2 * HD);
    seg(j1, p->w_k, 0, HD, 0, 0, nullptr, 0);
    seg(j1, p->w_v, 0, HD, HD, 0, nullptr, 0);
    copy(p->b_scale, 0, 1, 3 * C, pl.o_bscale, 3 * C, 0, nullptr, 0);
    copy(p->b_residual_gate, 0, 1, 2 * C, pl.o_brg, 2 * C, 0, nullptr, 0);
    copy(p->b_q, 0, 1, HD, pl.o_bq, HD, 0, nullptr, 0);
    copy(p->w_pair, 0, P, H, pl.o_wpair, H, 0, &p->pair_scale, 0);
  } else {
    seg(pack(pl.k_cond, S, 6 * C), p->w_mod, 0, 6 * C, 0, 0, nullptr, 0);
    PackJob &j0 = pack(pl.k_qkv0, C, 4 * HD);
    seg(j0, p->w_q, 0, HD, 0, 0, nullptr, 0);
    seg(j0, p->w_k, 0, HD, HD, 0, nullptr, 0);
    seg(j0, p->w_v, 0, HD, 2 * HD, 0, nullptr, 0);
    seg(j0, p->w_value_gate, 0, HD, 3 * HD, 0, nullptr, 0);
  }
  seg(pack(pl.k_out, HD, C), p->w_attention_out, 0, C, 0, 0, nullptr, 0);
  PackJob &jf = pack(pl.k_ff1, C, 2 * M);
  seg(jf, p->w_ff_gate, 0, M, 0, 1, nullptr, 0);
  seg(jf, p->w_ff_up, 0, M, 1, 1, nullptr, 0);
  seg(pack(pl.k_ff2, M, C), p->w_ff_out, 0, C, 0, 0, nullptr, 0);
  if (pl.enc) {
    seg(pack(pl.k_pool, C, U), p->w_pool, 0, U, 0, 0, nullptr, 0);
  } else {
    seg(pack(pl.k_tok, V, C), p->w_token, 0, C, 0, 0, nullptr, 0);
    copy(p->readout_scale, 0, 1, C, pl.o_rscale, C, 0, nullptr, 0);
    if (!pl.af3) copy(p->readout_bias, 0, 1, C, pl.o_rbias, C, 0, nullptr, 0);
    copy(p->w_readout, 0, C, 3, pl.o_wread, 3, 0, nullptr, 0);
  }
  wj.fill[wj.nfill++] = FillJob{reinterpret_cast<int *>(status), 1, 0, 0};
  if (pl.tail_pair)
    wj.fill[wj.nfill++] = FillJob{reinterpret_cast<int *>(ws + pl.o_xflag), 2 * ((R + kUmmaBM - 1) / kUmmaBM), 0, 0};
  if (pl.enc) {
    wj.fill[wj.nfill++] = FillJob{first, B * T, INT_MAX, 0};
    wj.fill[wj.nfill++] = FillJob{last, B * T, -1, 0};
  }
  hk.launch(ATOMENC_KERNEL_PREP, (k_prep_weights<Elt>), dim3(64, wj.ncopy + wj.npack + wj.nfill), 256, 0, st, wj);

  // out = epi(A' @ W) on the tensor cores, W given by its packed image and A' produced by
  // `prod` (A itself, or a row normalisation fused into the operand); K <= 256
  auto gemm_rows = [&](auto prod, size_t wpk, int64_t Mr, int64_t N, int64_t Kd, auto epi) {
    using P = decltype(prod);
    using E = decltype(epi);
    const int64_t mt = (Mr + kUmmaBM - 1) / kUmmaBM, nt = (N + kUmmaBN - 1) / kUmmaBN;
    const int64_t want = (pl.sms + mt - 1) / mt;          // CTAs per row block to fill the GPU
    const int64_t sp = want < nt ? want : nt;
    const int per = (int)((nt + sp - 1) / sp);
    dim3 grid((unsigned)((nt + per - 1) / per), (unsigned)mt);
    const size_t smem = rows_smem_bytes(Kd, split);
    if (split) {
      smem_limit(k_gemm_rows<P, true, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_rows<P, true, E>), grid, kRowsThreads, smem, st, prod, ws + wpk, Mr, N, Kd, per, epi, status);
    } else {
      smem_limit(k_gemm_rows<P, false, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_rows<P, false, E>), grid, kRowsThreads, smem, st, prod, ws + wpk, Mr, N, Kd, per, epi, status);
    }
  };
  // out = epi(A @ W): the row-block kernel for K <= 256, else the streaming kernel
  auto gemm = [&](auto *A_, int64_t lda, size_t wpk, int64_t Mr, int64_t N, int64_t Kd, auto epi) {
    using TA = std::remove_cv_t<std::remove_pointer_t<decltype(A_)>>;
    using E = decltype(epi);
    if (Kd <= kRowsKMax) {
      gemm_rows(ProdPlain<TA>{A_, lda, Mr, Kd}, wpk, Mr, N, Kd, epi);
      return;
    }
    dim3 grid((unsigned)((N + kUmmaBN - 1) / kUmmaBN), (unsigned)((Mr + kUmmaBM - 1) / kUmmaBM));
    const size_t smem = umma_smem_bytes(split);
    if (split) {
      smem_limit(k_gemm_umma<TA, true, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_umma<TA, true, E>), grid, kUmmaThreads, smem, st, A_, lda, ws + wpk, Mr, N, Kd, epi, status);
    } else {
      smem_limit(k_gemm_umma<TA, false, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_umma<TA, false, E>), grid, kUmmaThreads, smem, st, A_, lda, ws + wpk, Mr, N, Kd, epi, status);
    }
  };
  // the conditioning-modulated row norm of x (or x') fused into a projection's operand
  const bool fuse_norm = C <= kRowsKMax;
  Elt *xb = reinterpret_cast<Elt *>(ws + pl.o_x), *condb = reinterpret_cast<Elt *>(ws + pl.o_cond),
      *gateb = reinterpret_cast<Elt *>(ws + pl.o_gate), *poolb = reinterpret_cast<Elt *>(ws + pl.o_pool);
  auto norm_prod = [&](int64_t sc_off, int64_t sh_off, bool plus1) {
    return ProdNormT<Elt>{xb, F(pl.o_xstats), condb, R, C, 6 * C, sc_off, sh_off, plus1 ? 1 : 0};
  };
  const int rows_per_block = 8;  // warps per 256-thread block for warp-per-row kernels
  const unsigned row_blocks = (unsigned)((R + rows_per_block - 1) / rows_per_block);

  // ---- decoder: token @ w_token, gathered per atom in the row pass
  if (!pl.enc)
    gemm(static_cast<const Elt *>(in->token.data), V, pl.k_tok, B * T, C, V,
         Quad<EpiStore>{{F(pl.o_tp), C}});

  // ---- usable, sanitised residual start, normalised condition
  RowsArgs ra;
  ra.B = B; ra.A = A; ra.T = T; ra.C = C; ra.S = S; ra.eps = eps;
  ra.af3 = pl.af3; ra.decoder = !pl.enc; ra.encoder = pl.enc;
  ra.atom = in->atom.data; ra.condition = in->condition.data;
  ra.valid = static_cast<const uint8_t *>(in->valid.data);
  ra.token_valid = static_cast<const uint8_t *>(in->token_valid.data);
  ra.att = static_cast<const int64_t *>(in->atom_to_token.data);
  ra.token_proj = F(pl.o_tp);
  ra.usable = usable; ra.x = xb; ra.xstats = F(pl.o_xstats); ra.cstats = F(pl.o_cstats);
  ra.tok_first = first; ra.tok_last = last;
  {
    const uintptr_t al = sizeof(Elt) == 4 ? 15 : 7;   // 4-element loads of atom / condition rows
    const bool reg = C % 4 == 0 && S % 4 == 0 && C <= 256 && S <= 256 &&
                     ((reinterpret_cast<uintptr_t>(in->atom.data) | reinterpret_cast<uintptr_t>(in->condition.data)) & al) == 0;
    if (reg)
      hk.launch(ATOMENC_KERNEL_ROWS, (k_rows_prep_reg<Elt>), row_blocks, 256, 0, st, ra);
    else
      hk.launch(ATOMENC_KERNEL_ROWS, (k_rows_prep<Elt>), row_blocks, 256, 0, st, ra);
  }
  hk.mark(1, st);

  // ---- conditioning: the operand (LN(c), raw c or SiLU(c) of the sanitised condition)
  // is formed from the caller's condition rows inside the product
  const Elt *cin = static_cast<const Elt *>(in->condition.data);
  if (pl.af3) {
    gemm_rows(ProdCond<Elt, 2>{cin, usable, F(pl.o_cstats), R, S}, pl.k_cond, R, 6 * C, S,
              EpiCondAF3<Elt>{condb, F(pl.o_bscale), C});
    gemm_rows(ProdCond<Elt, 0>{cin, usable, nullptr, R, S}, pl.k_gate, R, 2 * C, S,
              EpiGateAF3<Elt>{gateb, F(pl.o_brg), C});
  } else {
    gemm_rows(ProdCond<Elt, 1>{cin, usable, nullptr, R, S}, pl.k_cond, R, 6 * C, S,
              Quad<EpiStoreT<Elt>>{{condb, 6 * C}});
  }
  hk.mark(2, st);
  if (!fuse_norm) {
    FeatArgs fa{R, C, eps, pl.af3 ? 1 : 0, xb, condb, F(pl.o_feat)};
    hk.launch(ATOMENC_KERNEL_ROWS, (k_features<Elt>), row_blocks, 256, 0, st, fa);
  }

  // ---- projections .. transition; WT is the type of the Q/K/V/G/O intermediates
  // (bf16 for bf16 workloads on the row-gather attention, float32 otherwise)
  auto middle = [&](auto wt_tag) {
    using WT = decltype(wt_tag);
    WT *wq = reinterpret_cast<WT *>(ws + pl.o_q), *wk = reinterpret_cast<WT *>(ws + pl.o_k),
       *wv = reinterpret_cast<WT *>(ws + pl.o_v), *wg = reinterpret_cast<WT *>(ws + pl.o_g),
       *wo = reinterpret_cast<WT *>(ws + pl.o_o);
    // ---- projections (attention inputs fused into the operand when C <= 256)
    if (pl.af3) {
      EpiSplitT<WT> e0{{wq, wg, nullptr, nullptr}, {F(pl.o_bq), nullptr, nullptr, nullptr}, HD};
      EpiSplitT<WT> e1{{wk, wv, nullptr, nullptr}, {nullptr, nullptr, nullptr, nullptr}, HD};
      if (fuse_norm) {
        gemm_rows(norm_prod(0, C, false), pl.k_qkv0, R, 2 * HD, C, e0);
        gemm_rows(norm_prod(2 * C, 3 * C, false), pl.k_qkv1, R, 2 * HD, C, e1);
      } else {
        gemm(F(pl.o_feat), 2 * C, pl.k_qkv0, R, 2 * HD, C, e0);
        gemm(F(pl.o_feat) + C, 2 * C, pl.k_qkv1, R, 2 * HD, C, e1);
      }
    } else {
      EpiSplitT<WT> e{{wq, wk, wv, wg}, {nullptr, nullptr, nullptr, nullptr}, HD};
      if (fuse_norm)
        gemm_rows(norm_prod(C, 0, true), pl.k_qkv0, R, 4 * HD, C, e);
      else
        gemm(F(pl.o_feat), C, pl.k_qkv0, R, 4 * HD, C, e);
      RopeArgs rp{R, H, D, eps, usable, in->rope_cos.data, in->rope_sin.data, wq, wk};
      if (D >= 8 && D <= 128 && (D & (D - 1)) == 0) {
        const int64_t warps = R * 2;
        hk.launch(ATOMENC_KERNEL_ROWS, (k_qk_rope_warp<Elt, WT>), (unsigned)((warps + 7) / 8), 256, 0, st, rp);
      } else {
        const int64_t n = R * H * 2;
        hk.launch(ATOMENC_KERNEL_ROWS, (k_qk_rope<Elt>), (unsigned)((n + 255) / 256), 256, 0, st, rp);
      }
    }
    hk.mark(3, st);

    // ---- slot-gathered attention
    const int rad = radius < 0 ? -1 : (radius > INT_MAX ? INT_MAX : (int)radius);
    if (pl.rg) {
      RowAttnArgs ra2;
      ra2.B = (int)B; ra2.A = (int)A; ra2.K = (int)K; ra2.H = (int)H; ra2.D = (int)D; ra2.P = (int)P;
      ra2.radius = rad;
      ra2.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
      ra2.eps = eps;
      ra2.QT = pl.rg_qt;
      ra2.stage_rows = pl.rg_stage_rows;
      ra2.Q = wq; ra2.Kf = wk; ra2.Vf = wv; ra2.G = wg;
      ra2.key_index = static_cast<const int64_t *>(in->key_index.data);
      ra2.window = static_cast<const uint8_t *>(in->window_mask.data);
      ra2.usable = usable;
      ra2.pair = pl.af3 ? in->pair.data : nullptr;
      ra2.w_pair = F(pl.o_wpair);
      ra2.attention = out->attention.data;
      ra2.O = wo;
      ra2.status = status;
      ra2.pair_vec = pl.af3 && P == 16 && (reinterpret_cast<uintptr_t>(in->pair.data) & 15) == 0;
      ra2.att_vec = (reinterpret_cast<uintptr_t>(out->attention.data) & 15) == 0;
      dim3 grid((unsigned)((A + pl.rg_qt - 1) / pl.rg_qt), (unsigned)B);
      auto go = [&](auto kern) {
        smem_limit(kern, pl.rg_smem);
        hk.launch(ATOMENC_KERNEL_ATTENTION, kern, grid, kRowAttnThreads, pl.rg_smem, st, ra2);
      };
      // the attention weights are written in the storage type: WT == Elt here
      if constexpr (std::is_same<WT, Elt>::value) {
#define ROWATTN(DH)                                                 \
  if (D == DH) {                                                    \
    if (pl.af3) go(k_attn_rows<WT, 128, DH, true>);                 \
    else go(k_attn_rows<WT, 128, DH, false>);                       \
  }
        ROWATTN(16) ROWATTN(32) ROWATTN(64)
#undef ROWATTN
      }
    } else {
      AttnArgs ag;
      ag.B = (int)B; ag.A = (int)A; ag.K = (int)K; ag.H = (int)H; ag.D = (int)D; ag.P = (int)P;
      ag.radius = rad;
      ag.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
      ag.eps = eps;
      ag.QT = pl.QT; ag.DP = pl.DP; ag.kv_floats = pl.kv_floats;
      ag.kmagic = K > 1 ? (uint32_t)(((uint64_t)1 << 32) / (uint64_t)K + (((uint64_t)1 << 32) % (uint64_t)K != 0)) : 0u;
      ag.Q = F(pl.o_q); ag.Kf = F(pl.o_k); ag.Vf = F(pl.o_v); ag.G = F(pl.o_g);
      ag.key_index = static_cast<const int64_t *>(in->key_index.data);
      ag.window = static_cast<const uint8_t *>(in->window_mask.data);
      ag.usable = usable;
      ag.pair = pl.af3 ? in->pair.data : nullptr;
      ag.w_pair = F(pl.o_wpair);
      ag.attention = out->attention.data;
      ag.O = F(pl.o_o);
      ag.status = status;
      dim3 grid((unsigned)((A + pl.QT - 1) / pl.QT), (unsigned)B);
      auto go = [&](auto kern) {
        smem_limit(kern, pl.attn_smem);
        hk.launch(ATOMENC_KERNEL_ATTENTION, kern, grid, attn_threads(pl.af3), pl.attn_smem, st, ag);
      };
      const int dm = D <= 8 ? 8 : D <= 16 ? 16 : D <= 32 ? 32 : 64;
      const bool multi = K > kChunk;
#define ATTN_D(DM)                                                          \
  if (dm == DM) {                                                           \
    if (pl.af3)                                                             \
      multi ? go(k_slot_attention<Elt, DM, true, true>)                     \
            : go(k_slot_attention<Elt, DM, true, false>);                   \
    else                                                                    \
      multi ? go(k_slot_attention<Elt, DM, false, true>)                    \
            : go(k_slot_attention<Elt, DM, false, false>);                  \
  }
      ATTN_D(8) ATTN_D(16) ATTN_D(32) ATTN_D(64)
#undef ATTN_D
    }

    hk.mark(4, st);

    // ---- out-projection + gated residual, transition norm, SwiGLU, gated residual + mask
    const Elt *gbuf = pl.af3 ? gateb : condb;
    const int64_t gld = pl.af3 ? 2 * C : 6 * C;
    const int64_t g0off = pl.af3 ? 0 : 2 * C, g1off = pl.af3 ? C : 5 * C;
    if (pl.fuse_tail) {
      TransArgs ta;
      ta.R = R; ta.HD = (int)HD; ta.M = (int)M;
      ta.O = wo; ta.x = xb;
      ta.g0 = gbuf + g0off; ta.g1 = gbuf + g1off; ta.g_ld = gld;
      ta.sc = condb + 4 * C; ta.sh = condb + (pl.af3 ? 5 : 3) * C; ta.cond_ld = 6 * C;
      ta.rms = pl.af3 ? 0 : 1; ta.plus1 = pl.af3 ? 0 : 1; ta.eps = eps;
      ta.usable = usable;
      ta.w_out = ws + pl.k_out; ta.w_ff1 = ws + pl.k_ff1; ta.w_ff2 = ws + pl.k_ff2;
      ta.hidden = out->hidden.data; ta.status = status;
      ta.xfer = F(pl.o_xfer); ta.xflag = reinterpret_cast<int *>(ws + pl.o_xflag);
      ta.peer_spin_limit = g_peer_spin_limit.load();
      ta.withhold_flag = g_peer_withhold.load();
      const size_t smem = trans_smem_bytes(split);
      const dim3 grid((unsigned)(((R + kUmmaBM - 1) / kUmmaBM) * (pl.tail_pair ? 2 : 1)));
      // the two CTAs of a row block exchange partials: launched as a 2-CTA cluster, so
      // that they are always resident at the same time
      auto go = [&](auto kern) {
        smem_limit(kern, smem);
        hk.launch_cluster(ATOMENC_KERNEL_TRANSITION, pl.tail_pair ? 2 : 1, kern, grid, kTransThreads,
                          smem, st, ta);
      };
      if constexpr (std::is_same<Elt, float>::value) {
        pl.tail_pair ? go(k_transition<true, Elt, true, WT>) : go(k_transition<true, Elt, false, WT>);
      } else {
        pl.tail_pair ? go(k_transition<false, Elt, true, WT>) : go(k_transition<false, Elt, false, WT>);
      }
    } else {
      gemm(static_cast<const WT *>(wo), HD, pl.k_out, R, C, HD,
           Quad<EpiResidual<Elt>>{{xb, gbuf, gld, g0off, C, F(pl.o_xp)}});
      TNormArgs tn{R, C, eps, pl.af3 ? 1 : 0, F(pl.o_xp), condb, F(pl.o_z)};
      hk.launch(ATOMENC_KERNEL_ROWS, (k_transition_norm<Elt>), row_blocks, 256, 0, st, tn);
      gemm(F(pl.o_z), C, pl.k_ff1, R, 2 * M, C, EpiSwiGLU{F(pl.o_h), M});
      gemm(F(pl.o_h), M, pl.k_ff2, R, C, M,
           Quad<EpiHidden<Elt>>{{F(pl.o_xp), gbuf, gld, g1off, C, usable,
                                 static_cast<Elt *>(out->hidden.data)}});
    }
  };
  if constexpr (std::is_same<Elt, __nv_bfloat16>::value) {
    if (pl.ws_bf16)
      middle(__nv_bfloat16{});
    else
      middle(float{});
  } else {
    middle(float{});
  }

  hk.mark(5, st);

  // ---- boundary, read from the hidden output itself
  const Elt *hid = static_cast<const Elt *>(out->hidden.data);
  if (pl.enc) {
    gemm(hid, C, pl.k_pool, R, U, C, Quad<EpiRelu<Elt>>{{poolb, U}});
    PoolArgs pa{B, A, T, U, usable, static_cast<const int64_t *>(in->atom_to_token.data), first,
                last, poolb, out->token_output.data};
    hk.launch(ATOMENC_KERNEL_POOL, (k_token_mean<Elt>), (unsigned)(B * T), kPoolThreads, 0, st, pa);
  } else {
    ReadoutArgs rd{R, C, eps, pl.af3 ? 0 : 1, usable, hid, F(pl.o_rscale), F(pl.o_rbias),
                   F(pl.o_wread), out->position_update.data};
    hk.launch(ATOMENC_KERNEL_ROWS, (k_readout<Elt>), row_blocks, 256, 0, st, rd);
  }
  hk.mark(6, st);
  if (hk.err != cudaSuccess) return ATOMENC_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATOMENC_OK : ATOMENC_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t atomenc_workspace_size(int style, int stage, const atomenc_inputs *in,
                              const atomenc_params *params, const atomenc_outputs *out) {
  Plan pl;
  if (validate(style, stage, in, params, out, pl) != ATOMENC_OK) return 0;
  return pl.bytes;
}

static int forward_impl(int style, int stage, const atomenc_inputs *in,
                        const atomenc_params *params, double eps, int64_t radius,
                        const atomenc_outputs *out, void *workspace, size_t workspace_bytes,
                        atomenc_stream_t stream, Hooks &hk) {
  Plan pl;
  CHECK(validate(style, stage, in, params, out, pl, radius));
  if (!std::isfinite(eps) || !(eps > 0.0)) return ATOMENC_ERR_EPS;
  float feps = (float)eps;
  if (!(feps > 0.f) || !std::isfinite(feps)) return ATOMENC_ERR_EPS;
  if (pl.fdt == ATOMENC_BF16 && !(bf16_round_host(feps) > 0.f)) return ATOMENC_ERR_EPS;
  if (radius < -1) return ATOMENC_ERR_RADIUS;
  if (!workspace || workspace_bytes < pl.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return ATOMENC_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  hk.begin(st);
  if (pl.fdt == ATOMENC_F32) return launch_all<float>(pl, in, params, feps, radius, out, ws, st, hk);
  return launch_all<__nv_bfloat16>(pl, in, params, feps, radius, out, ws, st, hk);
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
