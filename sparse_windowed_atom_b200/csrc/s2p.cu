// s2p.cu -- single-to-pair features: page "ESMFold Single-to-Pair Features"
// (esmfold_single_to_pair), Required behavior bullets 1-6.
//
//   k_s2p_qk     one warp per token, the row held in registers and the weight staged in
//                shared memory: absent rows replaced by zero (bullet 1), affine population
//                LayerNorm (bullet 2), projection x @ weight + bias into q then k
//                (bullet 3); float32 [B*N, 2H] in the workspace.
//   k_s2p_pairs  one CTA per (b, i), warps over j: pair(i, j) = [k_i * q_j, q_j - k_i]
//                (bullet 3), its readout with out_weight held in shared memory (bullet 4),
//                the optional affine output LayerNorm (bullet 5); both returned tensors are
//                zero unless tokens i and j are present (bullet 1). The pass is bound by
//                writing the two [B,N,N,*] tensors.
#include <cmath>
#include <cstring>

#include "../../include/atomenc.h"
#include "common.cuh"

namespace atomenc {
namespace s2p {

constexpr int kMaxH2 = 256, kMaxDp = 256, kMaxWeight = 16384, kMaxC = 256;
constexpr int kPairThreads = 256;

struct QKArgs {
  int64_t rows;
  int C, H2;
  float eps;
  const void *x;
  const uint8_t *mask;
  const void *nsc, *nbi, *w, *bias;
  float *qk;  // [rows, 2H]
};

// rows per CTA of the projection pass; its weight [C, 2H] is staged once per CTA
constexpr int kQKRows = 16, kQKThreads = kQKRows * 32;

template <typename T>
__global__ void __launch_bounds__(kQKThreads) k_s2p_qk(QKArgs a) {
  extern __shared__ float sq[];  // weight [C][2H], then norm_scale [C], norm_bias [C]
  const int tid = threadIdx.x, lane = tid & 31;
  float *snsc = sq + a.C * a.H2, *snbi = snsc + a.C;
  for (int k = tid; k < a.C * a.H2; k += kQKThreads) sq[k] = ldf((const T *)a.w, k);
  for (int k = tid; k < a.C; k += kQKThreads) {
    snsc[k] = ldf((const T *)a.nsc, k);
    snbi[k] = ldf((const T *)a.nbi, k);
  }
  __syncthreads();
  const int64_t row = (int64_t)blockIdx.x * kQKRows + (tid >> 5);
  if (row >= a.rows) return;
  const bool use = a.mask[row] != 0;
  const T *x = (const T *)a.x + row * a.C;
  // the row in registers: lane holds channels lane + 32 u (C <= 32 * kMaxCU)
  constexpr int kMaxCU = kMaxC / kWarp;
  float v[kMaxCU];
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxCU; ++u) {
    const int c = lane + u * kWarp;
    v[u] = use && c < a.C ? ldf(x, c) : 0.f;
    s += v[u];
  }
  const float mean = warp_sum(s) / (float)a.C;
  float q = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxCU; ++u) {
    const int c = lane + u * kWarp;
    if (c < a.C) q = fmaf(v[u] - mean, v[u] - mean, q);
  }
  const float rstd = 1.f / sqrtf(warp_sum(q) / (float)a.C + a.eps);
#pragma unroll
  for (int u = 0; u < kMaxCU; ++u) {
    const int c = lane + u * kWarp;
    if (c < a.C) v[u] = (v[u] - mean) * rstd * snsc[c] + snbi[c];
  }
  float acc[kMaxH2 / kWarp];
#pragma unroll
  for (int t = 0; t < kMaxH2 / kWarp; ++t) {
    const int e = lane + t * kWarp;
    acc[t] = e < a.H2 ? ldf((const T *)a.bias, e) : 0.f;
  }
#pragma unroll
  for (int u = 0; u < kMaxCU; ++u) {
    if (u * kWarp >= a.C) break;
    const int lim = a.C - u * kWarp < kWarp ? a.C - u * kWarp : kWarp;
    for (int l = 0; l < lim; ++l) {
      const float vc = __shfl_sync(0xffffffffu, v[u], l);
      const float *wr = sq + (u * kWarp + l) * a.H2;
#pragma unroll
      for (int t = 0; t < kMaxH2 / kWarp; ++t) {
        const int e = lane + t * kWarp;
        if (e < a.H2) acc[t] = fmaf(vc, wr[e], acc[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kMaxH2 / kWarp; ++t) {
    const int e = lane + t * kWarp;
    if (e < a.H2) a.qk[row * a.H2 + e] = acc[t];
  }
}

struct PairArgs {
  int64_t N;
  int H, H2, Dp;
  float eps;
  int onorm;
  const uint8_t *mask;
  const float *qk;
  const void *ow, *ob, *osc, *obi;
  void *pf, *out;
};

template <typename T>
__global__ void __launch_bounds__(kPairThreads) k_s2p_pairs(PairArgs a) {
  extern __shared__ float sw[];  // out_weight [2H][Dp], then out_bias, output_scale, output_bias
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H2 = a.H2, Dp = a.Dp, H = a.H;
  float *sb = sw + H2 * Dp, *ssc = sb + Dp, *sbi = ssc + Dp;
  for (int k = tid; k < H2 * Dp; k += kPairThreads) sw[k] = ldf((const T *)a.ow, k);
  for (int k = tid; k < Dp; k += kPairThreads) {
    sb[k] = ldf((const T *)a.ob, k);
    ssc[k] = a.onorm ? ldf((const T *)a.osc, k) : 1.f;
    sbi[k] = a.onorm ? ldf((const T *)a.obi, k) : 0.f;
  }
  __syncthreads();

  const int64_t bi = blockIdx.x, b = bi / a.N;
  const bool mi = a.mask[bi] != 0;
  const float *ki = a.qk + bi * H2 + H;
  for (int64_t j = warp; j < a.N; j += kPairThreads / kWarp) {
    const int64_t bj = b * a.N + j, pij = bi * a.N + j;
    T *pf = (T *)a.pf + pij * H2;
    T *out = (T *)a.out + pij * Dp;
    if (!(mi && a.mask[bj] != 0)) {
      for (int h = lane; h < H2; h += kWarp) stf(pf, h, 0.f);
      for (int e = lane; e < Dp; e += kWarp) stf(out, e, 0.f);
      continue;
    }
    const float *qj = a.qk + bj * H2;
    float f[kMaxH2 / kWarp];
#pragma unroll
    for (int m = 0; m < kMaxH2 / kWarp; ++m) {
      const int h = lane + m * kWarp;
      f[m] = 0.f;
      if (h < H) f[m] = ki[h] * qj[h];
      else if (h < H2) f[m] = qj[h - H] - ki[h - H];
      if (h < H2) stf(pf, h, f[m]);
    }
    if ((Dp & 3) == 0) {
      // readout: lane owns columns 4 lane + 128 t .. +3 (Dp a multiple of 4)
      constexpr int kT = kMaxDp / 128;
      float4 o[kT];
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int e = 4 * lane + 128 * t;
        o[t] = e < Dp ? *reinterpret_cast<const float4 *>(sb + e) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int m = 0; m < kMaxH2 / kWarp; ++m) {
        if (m * kWarp >= H2) break;
        const int lim = H2 - m * kWarp < kWarp ? H2 - m * kWarp : kWarp;
        for (int l = 0; l < lim; ++l) {
          const float fv = __shfl_sync(0xffffffffu, f[m], l);
          const float *wr = sw + (m * kWarp + l) * Dp;
#pragma unroll
          for (int t = 0; t < kT; ++t) {
            const int e = 4 * lane + 128 * t;
            if (e < Dp) {
              const float4 w = *reinterpret_cast<const float4 *>(wr + e);
              o[t].x = fmaf(fv, w.x, o[t].x);
              o[t].y = fmaf(fv, w.y, o[t].y);
              o[t].z = fmaf(fv, w.z, o[t].z);
              o[t].w = fmaf(fv, w.w, o[t].w);
            }
          }
        }
      }
      if (a.onorm) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < kT; ++t)
          if (4 * lane + 128 * t < Dp) s += (o[t].x + o[t].y) + (o[t].z + o[t].w);
        const float mean = warp_sum(s) / (float)Dp;
        float q = 0.f;
#pragma unroll
        for (int t = 0; t < kT; ++t)
          if (4 * lane + 128 * t < Dp) {
            q = fmaf(o[t].x - mean, o[t].x - mean, q);
            q = fmaf(o[t].y - mean, o[t].y - mean, q);
            q = fmaf(o[t].z - mean, o[t].z - mean, q);
            q = fmaf(o[t].w - mean, o[t].w - mean, q);
          }
        const float rstd = 1.f / sqrtf(warp_sum(q) / (float)Dp + a.eps);
#pragma unroll
        for (int t = 0; t < kT; ++t) {
          const int e = 4 * lane + 128 * t;
          if (e < Dp) {
            o[t].x = fmaf((o[t].x - mean) * rstd, ssc[e], sbi[e]);
            o[t].y = fmaf((o[t].y - mean) * rstd, ssc[e + 1], sbi[e + 1]);
            o[t].z = fmaf((o[t].z - mean) * rstd, ssc[e + 2], sbi[e + 2]);
            o[t].w = fmaf((o[t].w - mean) * rstd, ssc[e + 3], sbi[e + 3]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int e = 4 * lane + 128 * t;
        if (e < Dp) {
          stf(out, e, o[t].x);
          stf(out, e + 1, o[t].y);
          stf(out, e + 2, o[t].z);
          stf(out, e + 3, o[t].w);
        }
      }
    } else {
      // readout: lane owns columns lane + 32 t (any Dp)
      float o[kMaxDp / kWarp];
#pragma unroll
      for (int t = 0; t < kMaxDp / kWarp; ++t) {
        const int e = lane + t * kWarp;
        o[t] = e < Dp ? sb[e] : 0.f;
      }
#pragma unroll
      for (int m = 0; m < kMaxH2 / kWarp; ++m) {
        if (m * kWarp >= H2) break;
        const int lim = H2 - m * kWarp < kWarp ? H2 - m * kWarp : kWarp;
        for (int l = 0; l < lim; ++l) {
          const float fv = __shfl_sync(0xffffffffu, f[m], l);
          const float *wr = sw + (m * kWarp + l) * Dp;
#pragma unroll
          for (int t = 0; t < kMaxDp / kWarp; ++t) {
            const int e = lane + t * kWarp;
            if (e < Dp) o[t] = fmaf(fv, wr[e], o[t]);
          }
        }
      }
      if (a.onorm) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < kMaxDp / kWarp; ++t)
          if (lane + t * kWarp < Dp) s += o[t];
        const float mean = warp_sum(s) / (float)Dp;
        float q = 0.f;
#pragma unroll
        for (int t = 0; t < kMaxDp / kWarp; ++t)
          if (lane + t * kWarp < Dp) q = fmaf(o[t] - mean, o[t] - mean, q);
        const float rstd = 1.f / sqrtf(warp_sum(q) / (float)Dp + a.eps);
#pragma unroll
        for (int t = 0; t < kMaxDp / kWarp; ++t) {
          const int e = lane + t * kWarp;
          if (e < Dp) o[t] = fmaf((o[t] - mean) * rstd, ssc[e], sbi[e]);
        }
      }
#pragma unroll
      for (int t = 0; t < kMaxDp / kWarp; ++t) {
        const int e = lane + t * kWarp;
        if (e < Dp) stf(out, e, o[t]);
      }
    }
  }
}

// ---------------------------------------------------------------- host side

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

struct Dims {
  int64_t B = 0, N = 0, C = 0, H2 = 0, Dp = 0;
  int fdt = 0;
};

#define S2P_CHECK(expr)                  \
  do {                                   \
    const int _rc = (expr);              \
    if (_rc != ATOMENC_OK) return _rc;   \
  } while (0)

int validate(const atomenc_s2p_inputs *in, const atomenc_s2p_params *p, int onorm,
             const atomenc_s2p_outputs *out, Dims &d) {
  if (!in || !p || !out) return ATOMENC_ERR_NULL;
  if (!present(in->x) || !present(p->weight) || !present(p->out_weight)) return ATOMENC_ERR_NULL;
  if (in->x.ndim != 3 || p->weight.ndim != 2 || p->out_weight.ndim != 2) return ATOMENC_ERR_SHAPE;
  d.fdt = in->x.dtype;
  if (d.fdt != ATOMENC_F32 && d.fdt != ATOMENC_BF16) return ATOMENC_ERR_DTYPE;
  d.B = in->x.shape[0];
  d.N = in->x.shape[1];
  d.C = in->x.shape[2];
  d.H2 = p->weight.shape[1];
  d.Dp = p->out_weight.shape[1];
  if (d.B < 1 || d.N < 1 || d.C < 1 || d.H2 < 1 || d.Dp < 1) return ATOMENC_ERR_SHAPE;
  if (d.H2 % 2) return ATOMENC_ERR_SHAPE;
  const int64_t sx[3] = {d.B, d.N, d.C}, sm[2] = {d.B, d.N}, sc[1] = {d.C};
  const int64_t sw[2] = {d.C, d.H2}, sb[1] = {d.H2}, so[2] = {d.H2, d.Dp}, sd[1] = {d.Dp};
  const int64_t spf[4] = {d.B, d.N, d.N, d.H2}, sout[4] = {d.B, d.N, d.N, d.Dp};
  S2P_CHECK(check(in->x, d.fdt, 3, sx));
  S2P_CHECK(check(in->mask, ATOMENC_BOOL, 2, sm));
  S2P_CHECK(check(p->norm_scale, d.fdt, 1, sc));
  S2P_CHECK(check(p->norm_bias, d.fdt, 1, sc));
  S2P_CHECK(check(p->weight, d.fdt, 2, sw));
  S2P_CHECK(check(p->bias, d.fdt, 1, sb));
  S2P_CHECK(check(p->out_weight, d.fdt, 2, so));
  S2P_CHECK(check(p->out_bias, d.fdt, 1, sd));
  if (onorm) {
    S2P_CHECK(check(p->output_scale, d.fdt, 1, sd));
    S2P_CHECK(check(p->output_bias, d.fdt, 1, sd));
  }
  S2P_CHECK(check(out->pair_features, d.fdt, 4, spf));
  S2P_CHECK(check(out->output, d.fdt, 4, sout));
  if (d.C > kMaxC || d.H2 > kMaxH2 || d.Dp > kMaxDp || d.H2 * d.Dp > kMaxWeight ||
      d.C * d.H2 > 3 * kMaxWeight)
    return ATOMENC_ERR_UNSUPPORTED;
  if (d.B * d.N >= (int64_t)1 << 31) return ATOMENC_ERR_UNSUPPORTED;
  return ATOMENC_OK;
}

size_t workspace_bytes(const Dims &d) {
  return ((size_t)(d.B * d.N * d.H2) * 4 + 255) / 256 * 256;
}

float bf16_round(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  std::memcpy(&f, &u, 4);
  return f;
}

template <typename T>
int launch(const Dims &d, const atomenc_s2p_inputs *in, const atomenc_s2p_params *p, float eps,
           int onorm, const atomenc_s2p_outputs *out, float *qk, cudaStream_t st) {
  QKArgs qa{d.B * d.N, (int)d.C, (int)d.H2, eps, in->x.data,
            static_cast<const uint8_t *>(in->mask.data), p->norm_scale.data, p->norm_bias.data,
            p->weight.data, p->bias.data, qk};
  const size_t qsmem = (size_t)(d.C * d.H2 + 2 * d.C) * 4;
  if (cudaFuncSetAttribute(k_s2p_qk<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qsmem) !=
      cudaSuccess)
    return ATOMENC_ERR_CUDA;
  k_s2p_qk<T><<<(unsigned)((d.B * d.N + kQKRows - 1) / kQKRows), kQKThreads, qsmem, st>>>(qa);
  PairArgs pa{d.N, (int)(d.H2 / 2), (int)d.H2, (int)d.Dp, eps, onorm ? 1 : 0,
              static_cast<const uint8_t *>(in->mask.data), qk, p->out_weight.data,
              p->out_bias.data, onorm ? p->output_scale.data : nullptr,
              onorm ? p->output_bias.data : nullptr, out->pair_features.data, out->output.data};
  const size_t smem = (size_t)(d.H2 * d.Dp + 3 * d.Dp) * 4;
  if (cudaFuncSetAttribute(k_s2p_pairs<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return ATOMENC_ERR_CUDA;
  k_s2p_pairs<T><<<(unsigned)(d.B * d.N), kPairThreads, smem, st>>>(pa);
  return cudaGetLastError() == cudaSuccess ? ATOMENC_OK : ATOMENC_ERR_CUDA;
}

}  // namespace s2p
}  // namespace atomenc

extern "C" {

size_t atomenc_s2p_workspace_size(const atomenc_s2p_inputs *in, const atomenc_s2p_params *params,
                                  int output_norm, const atomenc_s2p_outputs *out) {
  atomenc::s2p::Dims d;
  if (atomenc::s2p::validate(in, params, output_norm, out, d) != ATOMENC_OK) return 0;
  return atomenc::s2p::workspace_bytes(d);
}

int atomenc_single_to_pair(const atomenc_s2p_inputs *in, const atomenc_s2p_params *params,
                           double eps, int output_norm, const atomenc_s2p_outputs *out,
                           void *workspace, size_t workspace_bytes, atomenc_stream_t stream) {
  using namespace atomenc::s2p;
  Dims d;
  const int rc = validate(in, params, output_norm, out, d);
  if (rc != ATOMENC_OK) return rc;
  const float feps = (float)eps;
  if (!std::isfinite(eps) || !(feps > 0.f)) return ATOMENC_ERR_EPS;
  if (d.fdt == ATOMENC_BF16 && !(bf16_round(feps) > 0.f)) return ATOMENC_ERR_EPS;
  if (!workspace || workspace_bytes < atomenc::s2p::workspace_bytes(d) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return ATOMENC_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float *qk = static_cast<float *>(workspace);
  return d.fdt == ATOMENC_F32
             ? launch<float>(d, in, params, feps, output_norm, out, qk, st)
             : launch<__nv_bfloat16>(d, in, params, feps, output_norm, out, qk, st);
}

}  // extern "C"
