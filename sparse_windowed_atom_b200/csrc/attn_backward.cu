// attn_backward.cu -- host side of atomenc_attention_backward (include/atomenc.h): the
// gradient of the slot-gathered attention core (kernels in attn_backward.cuh).
#include <cmath>
#include <cstring>

#include "../../include/atomenc.h"
#include "attn_backward.cuh"

using namespace atomenc;

namespace {

bool present(const atomenc_tensor &t) { return t.data != nullptr && t.ndim > 0; }

int check(const atomenc_tensor &t, int dtype, int ndim, const int64_t *shape) {
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

#define CHECK(expr)                    \
  do {                                 \
    int _rc = (expr);                  \
    if (_rc != ATOMENC_OK) return _rc; \
  } while (0)

struct BwdPlan {
  int64_t B = 0, A = 0, K = 0, H = 0, D = 0, P = 0;
  int fdt = 0;
  bool af3 = false;
  size_t o_acc_k = 0, o_acc_v = 0, o_beta = 0, o_acc_ps = 0, o_acc_wp = 0, bytes = 0;
};

size_t take(size_t &cur, size_t bytes) {
  const size_t o = cur;
  cur += (bytes + 255) & ~size_t(255);
  return o;
}

int validate(int style, const atomenc_core_bwd_inputs *in, int64_t heads,
             const atomenc_core_bwd_outputs *out, BwdPlan &pl) {
  if (!in || !out) return ATOMENC_ERR_NULL;
  if (style != ATOMENC_AF3 && style != ATOMENC_ESMFOLD2) return ATOMENC_ERR_STYLE;
  pl.af3 = style == ATOMENC_AF3;
  if (!present(in->q) || !present(in->key_index)) return ATOMENC_ERR_NULL;
  if (in->q.ndim != 3 || in->key_index.ndim != 3) return ATOMENC_ERR_SHAPE;
  const int fdt = in->q.dtype;
  if (fdt != ATOMENC_F32 && fdt != ATOMENC_BF16) return ATOMENC_ERR_DTYPE;
  pl.fdt = fdt;
  pl.B = in->q.shape[0];
  pl.A = in->q.shape[1];
  const int64_t HD = in->q.shape[2];
  pl.K = in->key_index.shape[2];
  if (heads < 1 || HD % heads != 0) return ATOMENC_ERR_SHAPE;
  pl.H = heads;
  pl.D = HD / heads;
  const int64_t B = pl.B, A = pl.A, K = pl.K, H = pl.H;
  const int64_t shd[] = {B, A, HD}, sk[] = {B, A, K}, sa[] = {B, A}, sat[] = {B, H, A, K};
  CHECK(check(in->q, fdt, 3, shd));
  CHECK(check(in->k, fdt, 3, shd));
  CHECK(check(in->v, fdt, 3, shd));
  CHECK(check(in->g, fdt, 3, shd));
  CHECK(check(in->d_out, fdt, 3, shd));
  CHECK(check(in->key_index, ATOMENC_I64, 3, sk));
  CHECK(check(in->window_mask, ATOMENC_BOOL, 3, sk));
  CHECK(check(in->usable, ATOMENC_BOOL, 2, sa));
  if (present(in->d_attention)) CHECK(check(in->d_attention, fdt, 4, sat));
  CHECK(check(out->d_q, fdt, 3, shd));
  CHECK(check(out->d_k, fdt, 3, shd));
  CHECK(check(out->d_v, fdt, 3, shd));
  CHECK(check(out->d_g, fdt, 3, shd));
  if (pl.af3) {
    if (!present(in->pair) || in->pair.ndim != 4) return ATOMENC_ERR_NULL;
    pl.P = in->pair.shape[3];
    const int64_t P = pl.P, sp[] = {B, A, K, P}, s1[] = {P}, s2[] = {P, H};
    CHECK(check(in->pair, fdt, 4, sp));
    CHECK(check(in->pair_scale, fdt, 1, s1));
    CHECK(check(in->w_pair, fdt, 2, s2));
    CHECK(check(out->d_pair, fdt, 4, sp));
    CHECK(check(out->d_pair_scale, fdt, 1, s1));
    CHECK(check(out->d_w_pair, fdt, 2, s2));
    if (P > kBwdPairMax || H > kBwdHeadsMax) return ATOMENC_ERR_UNSUPPORTED;
  }
  if (K > kBwdKMax || pl.D > kBwdDMax || A > INT_MAX - 4096) return ATOMENC_ERR_UNSUPPORTED;
  size_t cur = 0;
  const int64_t R = B * A;
  pl.o_acc_k = take(cur, (size_t)R * HD * 8);
  pl.o_acc_v = take(cur, (size_t)R * HD * 8);
  pl.o_beta = take(cur, pl.af3 ? (size_t)R * K * H * 4 : 0);
  pl.o_acc_ps = take(cur, pl.af3 ? (size_t)pl.P * 8 : 0);
  pl.o_acc_wp = take(cur, pl.af3 ? (size_t)pl.P * H * 8 : 0);
  pl.bytes = cur;
  return ATOMENC_OK;
}

template <typename T>
int launch(const BwdPlan &pl, const atomenc_core_bwd_inputs *in, const atomenc_core_bwd_outputs *out,
           float eps, int64_t radius, unsigned char *ws, cudaStream_t st) {
  CoreBwdArgs g;
  std::memset(&g, 0, sizeof(g));
  g.B = (int)pl.B; g.A = (int)pl.A; g.K = (int)pl.K; g.H = (int)pl.H; g.D = (int)pl.D; g.P = (int)pl.P;
  g.radius = radius < 0 ? -1 : (radius > INT_MAX ? INT_MAX : (int)radius);
  g.scale = (float)(1.0 / std::sqrt((double)pl.D));
  g.eps = eps;
  g.q = in->q.data; g.k = in->k.data; g.v = in->v.data; g.g = in->g.data;
  g.key_index = static_cast<const int64_t *>(in->key_index.data);
  g.window = static_cast<const uint8_t *>(in->window_mask.data);
  g.usable = static_cast<const uint8_t *>(in->usable.data);
  g.d_out = in->d_out.data;
  g.d_att = present(in->d_attention) ? in->d_attention.data : nullptr;
  g.d_q = out->d_q.data; g.d_g = out->d_g.data;
  g.acc_k = reinterpret_cast<unsigned long long *>(ws + pl.o_acc_k);
  g.acc_v = reinterpret_cast<unsigned long long *>(ws + pl.o_acc_v);
  if (pl.af3) {
    g.pair = in->pair.data; g.pair_scale = in->pair_scale.data; g.w_pair = in->w_pair.data;
    g.d_beta = reinterpret_cast<float *>(ws + pl.o_beta);
    g.acc_ps = reinterpret_cast<unsigned long long *>(ws + pl.o_acc_ps);
    g.acc_wp = reinterpret_cast<unsigned long long *>(ws + pl.o_acc_wp);
    g.d_pair = out->d_pair.data;
  }
  const int64_t R = pl.B * pl.A, HD = pl.H * pl.D;
  // the fixed-point sums start at zero
  k_core_bwd_zero<<<296, 256, 0, st>>>(g.acc_k, R * HD);
  k_core_bwd_zero<<<296, 256, 0, st>>>(g.acc_v, R * HD);
  if (pl.af3) {
    k_core_bwd_zero<<<1, 256, 0, st>>>(g.acc_ps, pl.P);
    k_core_bwd_zero<<<1, 256, 0, st>>>(g.acc_wp, pl.P * pl.H);
  }
  const int64_t warps = R * pl.H;
  const unsigned blocks = (unsigned)((warps + kBwdThreads / 32 - 1) / (kBwdThreads / 32));
  const int dm = pl.D <= 16 ? 16 : pl.D <= 32 ? 32 : 64;
#define CORE_BWD(DM)                                                        \
  if (dm == DM) {                                                           \
    if (pl.af3) k_core_bwd<T, DM, true><<<blocks, kBwdThreads, 0, st>>>(g); \
    else k_core_bwd<T, DM, false><<<blocks, kBwdThreads, 0, st>>>(g);       \
  }
  CORE_BWD(16) CORE_BWD(32) CORE_BWD(64)
#undef CORE_BWD
  if (pl.af3) {
    const int64_t slots = R * pl.K;
    k_core_bwd_pair<T><<<(unsigned)((slots + kBwdThreads - 1) / kBwdThreads), kBwdThreads, 0, st>>>(g);
    k_core_bwd_finish<T><<<1, 256, 0, st>>>(g.acc_ps, out->d_pair_scale.data, pl.P);
    k_core_bwd_finish<T><<<1, 256, 0, st>>>(g.acc_wp, out->d_w_pair.data, pl.P * pl.H);
  }
  k_core_bwd_finish<T><<<296, 256, 0, st>>>(g.acc_k, out->d_k.data, R * HD);
  k_core_bwd_finish<T><<<296, 256, 0, st>>>(g.acc_v, out->d_v.data, R * HD);
  return cudaGetLastError() == cudaSuccess ? ATOMENC_OK : ATOMENC_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t atomenc_attention_backward_workspace_size(int style, const atomenc_core_bwd_inputs *in,
                                                 int64_t heads,
                                                 const atomenc_core_bwd_outputs *out) {
  BwdPlan pl;
  if (validate(style, in, heads, out, pl) != ATOMENC_OK) return 0;
  return pl.bytes;
}

int atomenc_attention_backward(int style, const atomenc_core_bwd_inputs *in, int64_t heads,
                               double eps, int64_t radius, const atomenc_core_bwd_outputs *out,
                               void *workspace, size_t workspace_bytes, atomenc_stream_t stream) {
  BwdPlan pl;
  CHECK(validate(style, in, heads, out, pl));
  if (!std::isfinite(eps) || !(eps > 0.0) || !((float)eps > 0.f)) return ATOMENC_ERR_EPS;
  if (radius < -1) return ATOMENC_ERR_RADIUS;
  if (!workspace || workspace_bytes < pl.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return ATOMENC_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  if (pl.fdt == ATOMENC_F32) return launch<float>(pl, in, out, (float)eps, radius, ws, st);
  return launch<__nv_bfloat16>(pl, in, out, (float)eps, radius, ws, st);
}

}  // extern "C"
