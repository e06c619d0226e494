// attn_backward.cuh -- gradient of the slot-gathered attention core.
//
// Page "Local atom attention, encoder pooling and decoder skip/readout", Required
// behavior: the forward is the one of the block's attention (slot permission and radius,
// bullets 4-5; logits q . k / sqrt(D) plus the AF3 pair bias (LN(pair) * pair_scale) @
// w_pair, bullets 8 and 15; masked stable softmax with repeated slots as separate
// entries, bullets 5, 6 and 15; o * sigmoid(value gate), bullet 16), and a key selected
// by several slots, of one query or of many, receives the sum of their gradient
// contributions ("repeated selection accumulates gradients", the slot bullet).
//
// k_core_bwd: one warp per (query, head), lanes over the K slots (K <= 128, four per
// lane). It recomputes the permitted set, the logits and the softmax, then
//   o     = sum_k w_k v_j                      (folded across lanes)
//   d_g   = d_out * o * s (1 - s),  d_o = d_out * s,  s = sigmoid(g)
//   d_w_k = d_o . v_j (+ the weights' own gradient),  d_l_k = w_k (d_w_k - sum w d_w)
//   d_q   = sum_k d_l_k k_j / sqrt(D)          (written by the warp that owns the row)
//   d_k_j += d_l_k q / sqrt(D),  d_v_j += w_k d_o     (scattered)
//   d_beta[a, k, h] = d_l_k                    (AF3; float32 scratch)
// The scattered sums are accumulated as 64-bit fixed-point integers (value * 2^32,
// rounded to nearest) with integer reductions: integer addition is associative, so the
// result does not depend on the order in which contributions arrive (deterministic,
// no float atomics); |partial sums| must stay below 2^31.
// k_core_bwd_pair (AF3): one thread per slot, from d_beta: d_pair by the LayerNorm
// backward, and the CTA's contributions to d_pair_scale and d_w_pair summed in shared
// memory (fixed point) and added once per CTA.
// k_core_bwd_finish: fixed-point sums -> the output type.
#pragma once

#include <climits>

#include "common.cuh"

namespace atomenc {

constexpr int kBwdThreads = 256;        // 8 warps, one (query, head) each
constexpr int kBwdKMax = 128;
constexpr int kBwdDMax = 64;
constexpr int kBwdPairMax = 32;
constexpr int kBwdHeadsMax = 32;
constexpr double kFixScale = 4294967296.0;   // 2^32

struct CoreBwdArgs {
  int B, A, K, H, D, P;
  int radius;
  float scale;                 // 1 / sqrt(D)
  float eps;
  const void *q, *k, *v, *g;   // [B*A, HD] storage type
  const int64_t *key_index;    // [B, A, K]
  const uint8_t *window;       // [B, A, K]
  const uint8_t *usable;       // [B*A]
  const void *pair;            // [B, A, K, P] AF3
  const void *pair_scale;      // [P]
  const void *w_pair;          // [P, H]
  const void *d_out;           // [B*A, HD]
  const void *d_att;           // [B, H, A, K] or null
  void *d_q, *d_g;             // [B*A, HD]
  unsigned long long *acc_k, *acc_v;   // [B*A, HD] fixed point
  float *d_beta;               // [B, A, K, H] AF3
  unsigned long long *acc_ps, *acc_wp; // [P], [P*H] fixed point (AF3)
  void *d_pair;                // [B, A, K, P] AF3
};

__device__ __forceinline__ void red_fix(unsigned long long *p, float x) {
  const long long v = __float2ll_rn(x * 4294967296.f);
  atomicAdd(p, (unsigned long long)v);
}

// pair bias of one slot for head h (AF3): (LN(pair) * pair_scale) @ w_pair[:, h]
template <typename T>
__device__ __forceinline__ float core_beta(const T *pr, const T *ps, const T *wp, int P, int H,
                                           int h, float eps) {
  float mean = 0.f;
  for (int p = 0; p < P; ++p) mean += ldf(pr, p);
  mean /= (float)P;
  float var = 0.f;
  for (int p = 0; p < P; ++p) {
    const float d = ldf(pr, p) - mean;
    var = fmaf(d, d, var);
  }
  const float rstd = 1.f / sqrtf(var / (float)P + eps);
  float b = 0.f;
  for (int p = 0; p < P; ++p) b = fmaf((ldf(pr, p) - mean) * rstd * ldf(ps, p), ldf(wp, p * H + h), b);
  return b;
}

// DM: a compile-time bound on the head width D (16, 32 or 64), so that the query and d_o
// vectors stay in registers
template <typename T, int DM, bool AF3>
__global__ void __launch_bounds__(kBwdThreads) k_core_bwd(CoreBwdArgs g) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (kBwdThreads / 32) + (threadIdx.x >> 5);
  const int64_t R = (int64_t)g.B * g.A;
  if (item >= R * g.H) return;                 // warp-uniform
  const int64_t row = item / g.H;
  const int h = (int)(item - row * g.H);
  const int b = (int)(row / g.A), a = (int)(row - (int64_t)b * g.A);
  const int K = g.K, D = g.D, HD = g.H * g.D;
  const T *Q = static_cast<const T *>(g.q), *Kt = static_cast<const T *>(g.k);
  const T *V = static_cast<const T *>(g.v), *G = static_cast<const T *>(g.g);
  const T *dO = static_cast<const T *>(g.d_out);
  const int64_t rbase = (int64_t)b * g.A;
  const bool uq = g.usable[row] != 0;

  float qv[DM];
#pragma unroll
  for (int e = 0; e < DM; ++e) qv[e] = e < D ? ldf(Q, row * HD + h * D + e) : 0.f;

  // permitted slots and logits, four per lane
  int jj[4];
  float lg[4];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = i * 32 + lane;
    jj[i] = -1;
    lg[i] = -INFINITY;
    if (uq && k < K) {
      const int64_t s = row * K + k;
      const int64_t j = g.key_index[s];
      bool ok = g.window[s] != 0 && j >= 0 && j < g.A;
      if (ok && g.radius >= 0) ok = (j > a ? j - a : a - j) <= g.radius;
      if (ok) ok = g.usable[rbase + j] != 0;
      if (ok) {
        jj[i] = (int)j;
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < DM; ++e)
          if (e < D) dot = fmaf(qv[e], ldf(Kt, (rbase + j) * HD + h * D + e), dot);
        float l = dot * g.scale;
        if (AF3) {
          const T *pr = static_cast<const T *>(g.pair) + s * g.P;
          l += core_beta(pr, static_cast<const T *>(g.pair_scale), static_cast<const T *>(g.w_pair),
                         g.P, g.H, h, g.eps);
        }
        lg[i] = l;
        mx = fmaxf(mx, l);
      }
    }
  }
  mx = warp_max(mx);
  float w[4], sum = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = jj[i] >= 0 ? expf(lg[i] - mx) : 0.f;
    sum += w[i];
  }
  sum = warp_sum(sum);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] *= inv;

  // o = sum_k w_k v_j (every lane ends with the whole vector), then the value gate
  float dov[DM];
#pragma unroll
  for (int e = 0; e < DM; ++e) {
    float o = 0.f;
    if (e < D) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (jj[i] >= 0) o = fmaf(w[i], ldf(V, (rbase + jj[i]) * HD + h * D + e), o);
      o = warp_sum(o);
      const float sg = sigmoidf_(ldf(G, row * HD + h * D + e));
      const float d = ldf(dO, row * HD + h * D + e);
      if (lane == 0) stf(static_cast<T *>(g.d_g), row * HD + h * D + e, d * o * sg * (1.f - sg));
      dov[e] = d * sg;                         // d_o
    } else {
      dov[e] = 0.f;
    }
  }

  // d_w, the softmax backward, d_q
  float dl[4], sdw = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dl[i] = 0.f;
    if (jj[i] >= 0) {
      float dw = 0.f;
#pragma unroll
      for (int e = 0; e < DM; ++e)
        if (e < D) dw = fmaf(dov[e], ldf(V, (rbase + jj[i]) * HD + h * D + e), dw);
      if (g.d_att) dw += ldf(static_cast<const T *>(g.d_att), (((int64_t)b * g.H + h) * g.A + a) * K + i * 32 + lane);
      dl[i] = dw;
      sdw = fmaf(w[i], dw, sdw);
    }
  }
  sdw = warp_sum(sdw);
#pragma unroll
  for (int i = 0; i < 4; ++i) dl[i] = jj[i] >= 0 ? w[i] * (dl[i] - sdw) : 0.f;
#pragma unroll
  for (int e = 0; e < DM; ++e) {
    if (e >= D) break;
    float dq = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (jj[i] >= 0) dq = fmaf(dl[i], ldf(Kt, (rbase + jj[i]) * HD + h * D + e), dq);
    dq = warp_sum(dq);
    if (lane == 0) stf(static_cast<T *>(g.d_q), row * HD + h * D + e, dq * g.scale);
  }

  // scattered d_k, d_v (fixed point); AF3 d_beta
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (jj[i] < 0) continue;
    const int64_t kr = (rbase + jj[i]) * HD + h * D;
#pragma unroll
    for (int e = 0; e < DM; ++e) {
      if (e >= D) break;
      red_fix(g.acc_k + kr + e, dl[i] * qv[e] * g.scale);
      red_fix(g.acc_v + kr + e, w[i] * dov[e]);
    }
  }
  if (AF3) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = i * 32 + lane;
      if (k < K) g.d_beta[(row * K + k) * g.H + h] = dl[i];
    }
  }
}

// AF3: per slot, d_beta -> d_pair (LayerNorm backward), and this CTA's contributions to
// d_pair_scale and d_w_pair, summed in shared memory as fixed point, added once per CTA.
// beta_h = sum_p y_p ps_p W[p, h], y = (x - mean) rstd:
//   d_W[p, h] += d_beta_h y_p ps_p,  d_ps[p] += sum_h d_beta_h y_p W[p, h],
//   d_y_p = sum_h d_beta_h ps_p W[p, h],  d_x = rstd (d_y - mean(d_y) - y mean(d_y y))
template <typename T>
__global__ void __launch_bounds__(kBwdThreads) k_core_bwd_pair(CoreBwdArgs g) {
  pdl_enter();
  __shared__ unsigned long long s_ps[kBwdPairMax];
  __shared__ unsigned long long s_wp[kBwdPairMax * kBwdHeadsMax];
  const int P = g.P, H = g.H;
  for (int i = threadIdx.x; i < P; i += blockDim.x) s_ps[i] = 0ull;
  for (int i = threadIdx.x; i < P * H; i += blockDim.x) s_wp[i] = 0ull;
  __syncthreads();
  const int64_t slots = (int64_t)g.B * g.A * g.K;
  const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const T *ps = static_cast<const T *>(g.pair_scale), *wp = static_cast<const T *>(g.w_pair);
  if (s < slots) {
    const T *pr = static_cast<const T *>(g.pair) + s * P;
    T *dp = static_cast<T *>(g.d_pair) + s * P;
    const float *db = g.d_beta + s * H;
    bool any = false;
    for (int h = 0; h < H; ++h) any = any || db[h] != 0.f;
    if (!any) {
      for (int p = 0; p < P; ++p) stf(dp, p, 0.f);
    } else {
      float x[kBwdPairMax], dy[kBwdPairMax];
      float mean = 0.f;
      for (int p = 0; p < P; ++p) {
        x[p] = ldf(pr, p);
        mean += x[p];
      }
      mean /= (float)P;
      float var = 0.f;
      for (int p = 0; p < P; ++p) var = fmaf(x[p] - mean, x[p] - mean, var);
      const float rstd = 1.f / sqrtf(var / (float)P + g.eps);
      float mdy = 0.f, mdyy = 0.f;
      for (int p = 0; p < P; ++p) {
        const float y = (x[p] - mean) * rstd, psp = ldf(ps, p);
        float d = 0.f, dps = 0.f;
        for (int h = 0; h < H; ++h) {
          const float wph = ldf(wp, p * H + h);
          d = fmaf(db[h], psp * wph, d);
          dps = fmaf(db[h], y * wph, dps);
          atomicAdd(&s_wp[p * H + h], (unsigned long long)__float2ll_rn(db[h] * y * psp * 4294967296.f));
        }
        atomicAdd(&s_ps[p], (unsigned long long)__float2ll_rn(dps * 4294967296.f));
        dy[p] = d;
        x[p] = y;
        mdy += d;
        mdyy = fmaf(d, y, mdyy);
      }
      mdy /= (float)P;
      mdyy /= (float)P;
      for (int p = 0; p < P; ++p) stf(dp, p, (dy[p] - mdy - x[p] * mdyy) * rstd);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < P; i += blockDim.x)
    if (s_ps[i]) atomicAdd(g.acc_ps + i, s_ps[i]);
  for (int i = threadIdx.x; i < P * H; i += blockDim.x)
    if (s_wp[i]) atomicAdd(g.acc_wp + i, s_wp[i]);
}

// fixed-point sums -> output type
template <typename T>
__global__ void k_core_bwd_finish(const unsigned long long *acc, void *out, int64_t n) {
  pdl_enter();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    stf(static_cast<T *>(out), i, (float)((double)(long long)acc[i] / kFixScale));
}

// zero a fixed-point buffer
__global__ void k_core_bwd_zero(unsigned long long *p, int64_t n) {
  pdl_enter();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) p[i] = 0ull;
}

}  // namespace atomenc
