// rows.cuh -- per-row (atom / token) kernels: masking, sanitisation, normalisation,
// rotary, pooling and readout. Each kernel cites the passage of the page "Local atom
// attention, encoder pooling and decoder skip/readout" (Required behavior) it follows.
#pragma once

#include "common.cuh"

namespace atomenc {

// ------------------------------------------------------------------ row preparation
struct RowsArgs {
  int64_t B, A, T, C, S;
  float eps;
  int af3, decoder, encoder;
  const void *atom, *condition;
  const uint8_t *valid, *token_valid;
  const int64_t *att;
  const float *token_proj;  // [B*T, C] decoder: token @ w_token
  uint8_t *usable;          // [B*A]
  void *x;                  // [B*A, C] residual state start, in the storage type
  float *xstats;            // [B*A, 2] AF3: mean, 1/sqrt(var+eps); ESM: 0, 1/sqrt(mean sq+eps)
  float *cstats;            // [B*A, 2] AF3: mean, 1/sqrt(var+eps) of the sanitised condition
  int *tok_first, *tok_last;  // [B*T] encoder pooling ranges
};
// The conditioning products read the condition itself (sanitised, and SiLU'd or
// normalised with cstats, while their operand is formed); no copy of it is written.

// x / n, as a multiply by 1/n when n is a power of two (1/n is then exact, so the product
// is the same correctly rounded value as the quotient), else the IEEE division
__device__ __forceinline__ float div_n(float x, int n) {
  return (n & (n - 1)) == 0 ? x * __int_as_float((127 - (31 - __clz(n))) << 23) : x / (float)n;
}

// One warp per atom. usable = valid & 0 <= atom_to_token < T & token_valid  (bullet 2);
// payloads of unusable atoms are replaced by zero with a select before any arithmetic
// (bullet 3); encoder x = atom, decoder x = skip + gather(token @ w_token) (bullet 3).
template <typename T>
__global__ void k_rows_prep(RowsArgs r) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= r.B * r.A) return;
  const int64_t b = row / r.A, a = row % r.A;
  const bool use = atom_usable(r.valid, r.att, r.token_valid, b, a, r.A, r.T);
  const int64_t t = use ? r.att[row] : 0;
  if (lane == 0) {
    r.usable[row] = use ? 1 : 0;
    if (use && r.encoder) {
      atomicMin(r.tok_first + b * r.T + t, (int)a);
      atomicMax(r.tok_last + b * r.T + t, (int)a);
    }
  }
  const T *atom = (const T *)r.atom + row * r.C;
  T *xr = static_cast<T *>(r.x) + row * r.C;
  float s1 = 0.f;
  for (int64_t c = lane; c < r.C; c += kWarp) {
    float v = 0.f;
    if (use) {
      v = ldf(atom, c);
      if (r.decoder) v += r.token_proj[(b * r.T + t) * r.C + c];
    }
    stf(xr, c, v);
    s1 += ldf(xr, c);
  }
  // row statistics of x (as stored) for the attention inputs: AF3 population LayerNorm
  // (bullet 7), ESMFold2 RMS (bullet 11); the second pass re-reads the row just written
  __syncwarp();
  const float mean = r.af3 ? warp_sum(s1) / (float)r.C : 0.f;
  float s2 = 0.f;
  for (int64_t c = lane; c < r.C; c += kWarp) {
    const float d = ldf(xr, c) - mean;
    s2 = fmaf(d, d, s2);
  }
  s2 = warp_sum(s2);
  if (lane == 0) {
    r.xstats[2 * row] = mean;
    r.xstats[2 * row + 1] = 1.f / sqrtf(s2 / (float)r.C + r.eps);
  }
  if (r.af3) {
    // population LayerNorm statistics of the condition, eps inside the root (bullet 7)
    const T *cond = (const T *)r.condition + row * r.S;
    float s = 0.f;
    for (int64_t k = lane; k < r.S; k += kWarp) s += use ? ldf(cond, k) : 0.f;
    const float cm = warp_sum(s) / (float)r.S;
    float q = 0.f;
    for (int64_t k = lane; k < r.S; k += kWarp) {
      float d = (use ? ldf(cond, k) : 0.f) - cm;
      q += d * d;
    }
    const float rstd = 1.f / sqrtf(warp_sum(q) / (float)r.S + r.eps);
    if (lane == 0) {
      r.cstats[2 * row] = cm;
      r.cstats[2 * row + 1] = rstd;
    }
  }
}

// Four consecutive elements as floats (16-byte float32 / 8-byte bf16 loads), and four
// floats stored in the element type; the bf16 store rounds the values in place, so the
// caller's copy equals what was stored.
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
}
__device__ __forceinline__ void st4(float *p, float *v) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st4(__nv_bfloat16 *p, float *v) {
  uint32_t u[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    u[i] = bf16x2_bits(v[2 * i], v[2 * i + 1]);
    v[2 * i] = bf16_lo(u[i]);
    v[2 * i + 1] = bf16_hi(u[i]);
  }
  *reinterpret_cast<uint2 *>(p) = make_uint2(u[0], u[1]);
}

// k_rows_prep for C, S multiples of 4 up to 256 (aligned rows): the same arithmetic with
// the row held in registers (lane l owns channels 4l..4l+3 and 128+4l..128+4l+3). Every
// load of the caller's inputs is issued before the wait for the previous kernel, whose
// results (the reset token ranges; the token projection in the decoder) are used after.
// Grid: (ceil(A / 8), B), a warp per atom a of batch element b = blockIdx.y.
template <typename T>
__global__ void __launch_bounds__(256, 8) k_rows_prep_reg(RowsArgs r) {
  pdl_launch_next();
  const int lane = threadIdx.x & 31;
  const int64_t b = blockIdx.y, a = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const bool live = a < r.A;
  const int64_t row = b * r.A + a;
  const int C = (int)r.C, S = (int)r.S;
  // the payload rows are loaded whatever the flags say (they are readable memory) and
  // replaced by zero with a select below, so their loads overlap the flag loads
  float4 xl[2], cl[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = h * 128 + 4 * lane;
    xl[h] = cl[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live && c < C) xl[h] = ld4((const T *)r.atom + row * C + c);
    if (r.af3 && live && c < S) cl[h] = ld4((const T *)r.condition + row * S + c);
  }
  const bool use = live && atom_usable(r.valid, r.att, r.token_valid, b, a, r.A, r.T);
  const int64_t t = use ? r.att[row] : 0;
  float xv[8], cv[8];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float4 x = use ? xl[h] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 y = use ? cl[h] : make_float4(0.f, 0.f, 0.f, 0.f);
    xv[4 * h] = x.x; xv[4 * h + 1] = x.y; xv[4 * h + 2] = x.z; xv[4 * h + 3] = x.w;
    cv[4 * h] = y.x; cv[4 * h + 1] = y.y; cv[4 * h + 2] = y.z; cv[4 * h + 3] = y.w;
  }
  pdl_wait();
  if (!live) return;
  if (lane == 0) {
    r.usable[row] = use ? 1 : 0;
    if (use && r.encoder) {
      atomicMin(r.tok_first + b * r.T + t, (int)a);
      atomicMax(r.tok_last + b * r.T + t, (int)a);
    }
  }
  // x = atom, or skip + gathered token projection (bullet 3), stored in the storage type;
  // the row statistics of the stored values (AF3 population LayerNorm, bullet 7;
  // ESMFold2 RMS, bullet 11)
  float s1 = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = h * 128 + 4 * lane;
    if (c < C) {
      if (r.decoder && use) {
        const float4 tp = ld4(r.token_proj + (b * r.T + t) * C + c);
        xv[4 * h] += tp.x; xv[4 * h + 1] += tp.y; xv[4 * h + 2] += tp.z; xv[4 * h + 3] += tp.w;
      }
      st4(static_cast<T *>(r.x) + row * C + c, xv + 4 * h);
      s1 += (xv[4 * h] + xv[4 * h + 1]) + (xv[4 * h + 2] + xv[4 * h + 3]);
    }
  }
  const float mean = r.af3 ? div_n(warp_sum(s1), C) : 0.f;
  float s2 = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h)
    if (h * 128 + 4 * lane < C)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d = xv[4 * h + e] - mean;
        s2 = fmaf(d, d, s2);
      }
  s2 = warp_sum(s2);
  if (lane == 0) {
    r.xstats[2 * row] = mean;
    r.xstats[2 * row + 1] = 1.f / sqrtf(div_n(s2, C) + r.eps);
  }
  if (r.af3) {
    // population LayerNorm statistics of the condition, eps inside the root (bullet 7)
    float sc = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (h * 128 + 4 * lane < S) sc += (cv[4 * h] + cv[4 * h + 1]) + (cv[4 * h + 2] + cv[4 * h + 3]);
    const float cm = div_n(warp_sum(sc), S);
    float q = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (h * 128 + 4 * lane < S)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float d = cv[4 * h + e] - cm;
          q = fmaf(d, d, q);
        }
    const float rstd = 1.f / sqrtf(div_n(warp_sum(q), S) + r.eps);
    if (lane == 0) {
      r.cstats[2 * row] = cm;
      r.cstats[2 * row + 1] = rstd;
    }
  }
}

// ------------------------------------------------------------------ attention inputs
struct FeatArgs {
  int64_t rows, C;
  float eps;
  int af3;
  const void *x;      // [rows, C] storage type
  const void *cond;   // storage type; AF3 [rows, 6C] = (sig(scale_j + b), shift_j) j=0..2; ESM [rows, 6C] raw
  float *feat;        // AF3 [rows, 2C] = (A_0(x), A_1(x)); ESM [rows, C] attention input
};

// AF3: A_j(x) = LN(x) * sigmoid(c_j @ w_scale[j] + b_scale[j]) + c_j @ w_shift[j]  (bullet 7)
// ESM: attention input = RMS(x) * (1 + attention_scale) + attention_shift  (bullet 11)
template <typename IT>
__global__ void k_features(FeatArgs f) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= f.rows) return;
  const IT *x = static_cast<const IT *>(f.x) + row * f.C;
  const IT *cd = static_cast<const IT *>(f.cond) + row * 6 * f.C;
  if (f.af3) {
    float s = 0.f;
    for (int64_t c = lane; c < f.C; c += kWarp) s += ldf(x, c);
    const float mean = warp_sum(s) / (float)f.C;
    float q = 0.f;
    for (int64_t c = lane; c < f.C; c += kWarp) q += (ldf(x, c) - mean) * (ldf(x, c) - mean);
    const float rstd = 1.f / sqrtf(warp_sum(q) / (float)f.C + f.eps);
    for (int64_t c = lane; c < f.C; c += kWarp) {
      float ln = (ldf(x, c) - mean) * rstd;
      f.feat[row * 2 * f.C + c] = ln * ldf(cd, c) + ldf(cd, f.C + c);
      f.feat[row * 2 * f.C + f.C + c] = ln * ldf(cd, 2 * f.C + c) + ldf(cd, 3 * f.C + c);
    }
  } else {
    float q = 0.f;
    for (int64_t c = lane; c < f.C; c += kWarp) q += ldf(x, c) * ldf(x, c);
    const float rstd = 1.f / sqrtf(warp_sum(q) / (float)f.C + f.eps);
    for (int64_t c = lane; c < f.C; c += kWarp)
      f.feat[row * f.C + c] = ldf(x, c) * rstd * (1.f + ldf(cd, f.C + c)) + ldf(cd, c);
  }
}

// ------------------------------------------------------------------ ESMFold2 Q/K head norm + rotary
struct RopeArgs {
  int64_t rows, H, D;
  float eps;
  const uint8_t *usable;
  const void *cos, *sin;  // [rows, D]
  void *Q, *K;            // [rows, H*D], rewritten in place (float32; k_qk_rope_warp:
                          // its workspace type)
  int vec;                // k_qk_rope_warp: cos/sin rows are aligned for 4-value loads
};

// Per-head RMS of Q and K over D, then q * cos + rotate_half(q) * sin with
// rotate_half([q1, q2]) = [-q2, q1], before keys are gathered (bullets 12, 13).
// One thread per (atom, head, Q-or-K); D <= 128.
template <typename T>
__global__ void k_qk_rope(RopeArgs r) {
  pdl_enter();
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= r.rows * r.H * 2) return;
  const int which = (int)(id & 1);
  const int64_t rh = id >> 1;
  const int64_t row = rh / r.H, h = rh % r.H;
  float *v = static_cast<float *>(which ? r.K : r.Q) + row * r.H * r.D + h * r.D;
  const bool use = r.usable[row] != 0;
  float buf[128];
  float ss = 0.f;
  for (int d = 0; d < r.D; ++d) {
    buf[d] = v[d];
    ss += buf[d] * buf[d];
  }
  const float rstd = 1.f / sqrtf(ss / (float)r.D + r.eps);
  const T *cs = (const T *)r.cos + row * r.D;
  const T *sn = (const T *)r.sin + row * r.D;
  const int half = (int)(r.D / 2);
  for (int d = 0; d < r.D; ++d) {
    float qd = buf[d] * rstd;
    float rot = d < half ? -buf[d + half] * rstd : buf[d - half] * rstd;
    float c = use ? ldf(cs, d) : 0.f, s = use ? ldf(sn, d) : 0.f;
    v[d] = use ? qd * c + rot * s : 0.f;
  }
}

// four consecutive values of a Q / K row, read and written in the workspace type
__device__ __forceinline__ float4 ld4w(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4w(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
}
__device__ __forceinline__ void st4w(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void st4w(__nv_bfloat16 *p, float4 v) {
  *reinterpret_cast<uint2 *>(p) = make_uint2(bf16x2_bits(v.x, v.y), bf16x2_bits(v.z, v.w));
}

// Warp per atom for head widths D in {8, 16, 32, 64, 128}: lane l holds four consecutive
// channels of each 128-channel chunk of the Q row and of the K row, the D/4 lanes of one
// head reduce the sum of squares with xor-shuffles, and the half-split partner of
// channel d (d +- D/2) sits D/8 lanes away in the same head group. Every load (Q, K,
// cos, sin, the usable flag) is issued before any of them is used; an unusable atom's
// rows become zero by a select. Q and K are of type WT (float32, or bf16 when the
// attention reads bf16 rows); the arithmetic is float32. vec: cos/sin rows may be read
// four values at a time.
template <typename T, typename WT>
__global__ void __launch_bounds__(256, 8) k_qk_rope_warp(RopeArgs r) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= r.rows) return;
  const int D = (int)r.D, HD = (int)(r.H * r.D), glanes = D / 4, half = D / 2;
  WT *qv = static_cast<WT *>(r.Q) + row * HD;
  WT *kv = static_cast<WT *>(r.K) + row * HD;
  const T *cs = (const T *)r.cos + row * D;
  const T *sn = (const T *)r.sin + row * D;
  for (int c0 = 0; c0 < HD; c0 += 128) {
    const int c = c0 + lane * 4;
    const bool in = c < HD;
    const int d = c & (D - 1);   // D is a power of two
    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 xq = in ? ld4w(qv + c) : z4, xk = in ? ld4w(kv + c) : z4, co = z4, si = z4;
    if (in) {
      if (r.vec) {
        co = ld4(cs + d);
        si = ld4(sn + d);
      } else {
        co = make_float4(ldf(cs, d), ldf(cs, d + 1), ldf(cs, d + 2), ldf(cs, d + 3));
        si = make_float4(ldf(sn, d), ldf(sn, d + 1), ldf(sn, d + 2), ldf(sn, d + 3));
      }
    }
    const bool use = r.usable[row] != 0;
    const int po = D / 8;  // lanes between channel d and d +- D/2
    const float sg = d < half ? -1.f : 1.f;   // rotate_half: [-q2, q1]
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      float4 x = w ? xk : xq;
      float ss = x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
      for (int o = 1; o < glanes; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float rstd = 1.f / sqrtf(div_n(ss, D) + r.eps);
      x.x *= rstd; x.y *= rstd; x.z *= rstd; x.w *= rstd;
      float4 p;
      p.x = __shfl_xor_sync(0xffffffffu, x.x, po);
      p.y = __shfl_xor_sync(0xffffffffu, x.y, po);
      p.z = __shfl_xor_sync(0xffffffffu, x.z, po);
      p.w = __shfl_xor_sync(0xffffffffu, x.w, po);
      if (in) {
        float4 o = z4;
        if (use) {
          o.x = x.x * co.x + sg * p.x * si.x;
          o.y = x.y * co.y + sg * p.y * si.y;
          o.z = x.z * co.z + sg * p.z * si.z;
          o.w = x.w * co.w + sg * p.w * si.w;
        }
        st4w((w ? kv : qv) + c, o);
      }
    }
  }
}

// ------------------------------------------------------------------ transition norm
struct TNormArgs {
  int64_t rows, C;
  float eps;
  int af3;
  const float *xp;    // [rows, C] x' after the attention residual
  const void *cond;   // [rows, 6C] as in FeatArgs, storage type
  float *z;           // [rows, C]
};

// Normalise the NEW residual state: AF3 A_2(x'); ESMFold2
// RMS(x') * (1 + transition_scale) + transition_shift  (bullet 17)
template <typename IT>
__global__ void k_transition_norm(TNormArgs f) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= f.rows) return;
  const float *x = f.xp + row * f.C;
  const IT *cd = static_cast<const IT *>(f.cond) + row * 6 * f.C;
  if (f.af3) {
    float s = 0.f;
    for (int64_t c = lane; c < f.C; c += kWarp) s += x[c];
    const float mean = warp_sum(s) / (float)f.C;
    float q = 0.f;
    for (int64_t c = lane; c < f.C; c += kWarp) q += (x[c] - mean) * (x[c] - mean);
    const float rstd = 1.f / sqrtf(warp_sum(q) / (float)f.C + f.eps);
    for (int64_t c = lane; c < f.C; c += kWarp)
      f.z[row * f.C + c] = (x[c] - mean) * rstd * ldf(cd, 4 * f.C + c) + ldf(cd, 5 * f.C + c);
  } else {
    float q = 0.f;
    for (int64_t c = lane; c < f.C; c += kWarp) q += x[c] * x[c];
    const float rstd = 1.f / sqrtf(warp_sum(q) / (float)f.C + f.eps);
    for (int64_t c = lane; c < f.C; c += kWarp)
      f.z[row * f.C + c] = x[c] * rstd * (1.f + ldf(cd, 4 * f.C + c)) + ldf(cd, 3 * f.C + c);
  }
}

// ------------------------------------------------------------------ encoder pooling
struct PoolArgs {
  int64_t B, A, T, U;
  const uint8_t *usable;
  const int64_t *att;
  const int *tok_first, *tok_last;
  const void *pooled;   // [B*A, U] ReLU(hidden @ w_pool), storage type
  void *out;            // [B, T, U]
};

// token_output[t] = exact mean of ReLU(hidden @ w_pool) over the usable atoms mapped
// to t, summed in ascending atom order (deterministic); 0 for a token with none
// (bullet 19). One block of kPoolThreads per token: the atoms of the token's range are
// tested 128 at a time into a shared flag row, then each thread sums three output
// channels over the flagged rows with four rows' loads in flight.
constexpr int kPoolThreads = 128;
template <typename T>
__global__ void __launch_bounds__(kPoolThreads) k_token_mean(PoolArgs p) {
  pdl_enter();
  __shared__ uint8_t s_flag[kPoolThreads + 4];
  const int tid = threadIdx.x;
  const int64_t bt = blockIdx.x;
  const int64_t b = bt / p.T, t = bt % p.T;
  const int first = p.tok_first[bt], last = p.tok_last[bt];
  const int64_t U = p.U;
  for (int64_t u0 = 0; u0 < U; u0 += 3 * kPoolThreads) {
    float acc[3] = {0.f, 0.f, 0.f};
    int n = 0;
    for (int base = first; base <= last; base += kPoolThreads) {
      const int a = base + tid;
      bool f = false;
      if (a <= last) {
        const int64_t row = b * p.A + a;
        f = p.usable[row] != 0 && p.att[row] == t;
      }
      s_flag[tid] = f ? 1 : 0;
      if (tid < 4) s_flag[kPoolThreads + tid] = 0;
      n += __syncthreads_count(f);
      const int cnt = min(kPoolThreads, last - base + 1);
      const T *rows = static_cast<const T *>(p.pooled) + (b * p.A + base) * U + u0 + tid;
      for (int i = 0; i < cnt; i += 4) {
        float x[4][3];
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int c = 0; c < 3; ++c)
            x[e][c] = s_flag[i + e] && u0 + tid + c * kPoolThreads < U
                          ? ldf(rows, (int64_t)(i + e) * U + c * kPoolThreads)
                          : 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int c = 0; c < 3; ++c) acc[c] += x[e][c];
      }
      __syncthreads();
    }
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      const int64_t u = u0 + tid + c * kPoolThreads;
      if (u < U) stf((T *)p.out, bt * U + u, n > 0 ? acc[c] / (float)n : 0.f);
    }
  }
}

// The same mean with one warp per token, for U a multiple of 4 up to 512 (NCH chunks of
// 128 channels): lane l sums channels 4l..4l+3 of each chunk over the token's range in
// ascending atom order, four rows' loads in flight; the rows are loaded whatever the
// flags say (they lie inside the pooled buffer) and the flags (usable and mapped to
// this token, one per lane for 32 rows, by ballot) select what is added, so the sums
// are those of k_token_mean. vec_out: token_output rows may be written four values at
// a time.
// Grid: (ceil(T / 8), B), a warp per token t of batch element b = blockIdx.y.
template <typename T, int NCH>
__global__ void __launch_bounds__(256) k_token_mean_warp(PoolArgs p, int vec_out) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t b = blockIdx.y, t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const int64_t bt = b * p.T + t;
  const int first = p.tok_first[bt], last = p.tok_last[bt];
  const int U = (int)p.U;
  const T *base = static_cast<const T *>(p.pooled) + b * p.A * (int64_t)U;
  float acc[NCH][4];
#pragma unroll
  for (int k = 0; k < NCH; ++k) acc[k][0] = acc[k][1] = acc[k][2] = acc[k][3] = 0.f;
  int n = 0;
  for (int a0 = first; a0 <= last; a0 += 32) {
    const int cnt = min(32, last - a0 + 1);
    bool f = false;
    if (lane < cnt) {
      const int64_t row = b * p.A + a0 + lane;
      f = p.usable[row] != 0 && p.att[row] == t;
    }
    for (int i = 0; i < cnt; i += 4) {
      float4 x[4][NCH];
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          const int c = 128 * k + 4 * lane;
          x[e][k] = (i + e < cnt && c < U) ? ld4(base + (int64_t)(a0 + i + e) * U + c)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      const unsigned m = __ballot_sync(0xffffffffu, f);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool on = (m >> (i + e)) & 1u;
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          acc[k][0] += on ? x[e][k].x : 0.f;
          acc[k][1] += on ? x[e][k].y : 0.f;
          acc[k][2] += on ? x[e][k].z : 0.f;
          acc[k][3] += on ? x[e][k].w : 0.f;
        }
      }
    }
    n += __popc(__ballot_sync(0xffffffffu, f));
  }
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int c = 128 * k + 4 * lane;
    if (c >= U) continue;
    float o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = n > 0 ? acc[k][e] / (float)n : 0.f;
    T *dst = static_cast<T *>(p.out) + bt * U + c;
    if (vec_out) {
      st4(dst, o);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) stf(dst, e, o[e]);
    }
  }
}

// ------------------------------------------------------------------ decoder readout
struct ReadoutArgs {
  int64_t rows, C;
  float eps;
  int has_bias;
  const uint8_t *usable;
  const void *hid;         // [rows, C] hidden (the output tensor, storage type)
  const float *scale;      // [C]
  const float *bias;       // [C] ESMFold2
  const float *w_readout;  // [C, 3]
  void *out;               // [rows, 3]
};

// position_update = (LN(hidden) * readout_scale [+ readout_bias]) @ w_readout, masked
// to zero; an update, not coordinates (bullets 18-20). One warp per atom.
template <typename T>
__global__ void k_readout(ReadoutArgs r) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= r.rows) return;
  const T *x = static_cast<const T *>(r.hid) + row * r.C;
  float s = 0.f;
  for (int64_t c = lane; c < r.C; c += kWarp) s += ldf(x, c);
  const float mean = warp_sum(s) / (float)r.C;
  float q = 0.f;
  for (int64_t c = lane; c < r.C; c += kWarp) q += (ldf(x, c) - mean) * (ldf(x, c) - mean);
  const float rstd = 1.f / sqrtf(warp_sum(q) / (float)r.C + r.eps);
  float o0 = 0.f, o1 = 0.f, o2 = 0.f;
  for (int64_t c = lane; c < r.C; c += kWarp) {
    float y = (ldf(x, c) - mean) * rstd * r.scale[c] + (r.has_bias ? r.bias[c] : 0.f);
    o0 += y * r.w_readout[c * 3 + 0];
    o1 += y * r.w_readout[c * 3 + 1];
    o2 += y * r.w_readout[c * 3 + 2];
  }
  o0 = warp_sum(o0);
  o1 = warp_sum(o1);
  o2 = warp_sum(o2);
  if (lane == 0) {
    const bool use = r.usable[row] != 0;
    stf((T *)r.out, row * 3 + 0, use ? o0 : 0.f);
    stf((T *)r.out, row * 3 + 1, use ? o1 : 0.f);
    stf((T *)r.out, row * 3 + 2, use ? o2 : 0.f);
  }
}

}  // namespace atomenc
