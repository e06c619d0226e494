// attention.cuh -- slot-gathered windowed attention (the HBM-bound core of the block).
//
// Page "Local atom attention, encoder pooling and decoder skip/readout", Required
// behavior: a slot (query a, slot k) is permitted iff its key id j is in [0, A), both
// atoms are usable, window_mask is set and, for radius >= 0, |j - a| <= radius (bullets
// 4, 5); logits are Q_a . K_j / sqrt(D) plus, in AF3 style, the pair bias
// (LN(pair) * pair_scale) @ w_pair (bullets 8, 15); a stabilised softmax runs over the
// permitted slots only, a row without any gets exact zeros, repeated slots are separate
// entries (bullets 5, 6, 15); the weighted values are multiplied by sigmoid of the value
// gate logits (bullet 16).
//
// One CTA owns QT consecutive queries of one batch element. Phase 1 reads key_index,
// window_mask and (AF3) the pair rows exactly once, builds the tile's slot plan (key id or
// -1) in shared memory and, for AF3, the pair bias of every (query, slot, head). Phase 2
// runs head by head: the K and V rows of the tile's key span are staged in shared memory
// (float32), then each warp takes one query at a time with its lanes over the slots.
#pragma once

#include "common.cuh"

namespace atomenc {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / kWarp;
constexpr int kPairMax = 32;

struct AttnArgs {
  int64_t B, A, K, H, D, P;
  int64_t radius;
  float inv_sqrt_d, eps;
  int QT, cap_rows, DP;
  const float *Q, *Kf, *Vf, *G;   // [B*A, H*D]
  const int64_t *key_index;       // [B, A, K]
  const uint8_t *window;          // [B, A, K]
  const uint8_t *usable;          // [B*A]
  const void *pair;               // [B, A, K, P] AF3
  const float *w_pair;            // [P, H] = pair_scale[p] * w_pair[p, h]
  void *attention;                // [B, H, A, K]
  float *O;                       // [B*A, H*D] gated attention output
  unsigned *status;
};

template <typename T, int DMAX, bool AF3>
__global__ void __launch_bounds__(kAttnThreads) k_slot_attention(AttnArgs g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b = blockIdx.y, a0 = (int64_t)blockIdx.x * g.QT;
  const int QT = g.QT;
  const int64_t K = g.K, H = g.H, D = g.D, A = g.A, HD = g.H * g.D;

  int *plan = reinterpret_cast<int *>(smem_raw);                       // [QT*K]
  float *beta = reinterpret_cast<float *>(plan + QT * K);              // [QT*K*H] (AF3)
  float *lgb = beta + (AF3 ? QT * K * H : 0);                          // [warps][K]
  float *ks = lgb + kAttnWarps * K;                                    // [cap][DP]
  float *vs = ks + (int64_t)g.cap_rows * g.DP;                         // [cap][DP]
  __shared__ int s_lo, s_hi;
  if (tid == 0) {
    s_lo = INT_MAX;
    s_hi = -1;
  }
  __syncthreads();

  // ---------------- phase 1: slot plan and pair bias, one pass over the tile's slots
  int lo = INT_MAX, hi = -1;
  for (int64_t idx = tid; idx < QT * K; idx += kAttnThreads) {
    const int64_t q = idx / K, k = idx % K, a = a0 + q;
    int jj = -1;
    if (a < A) {
      const int64_t s = (b * A + a) * K + k;
      const int64_t j = g.key_index[s];
      bool ok = j >= 0 && j < A && g.window[s] != 0 && g.usable[b * A + a] != 0;
      ok = ok && g.usable[b * A + j] != 0;
      if (ok && g.radius >= 0) ok = (j > a ? j - a : a - j) <= g.radius;
      if (ok) {
        jj = (int)j;
        lo = min(lo, jj);
        hi = max(hi, jj);
        if (AF3) {
          const T *pr = (const T *)g.pair + s * g.P;
          float v[kPairMax];
          float sum = 0.f;
#pragma unroll
          for (int p = 0; p < kPairMax; ++p)
            if (p < g.P) {
              v[p] = ldf(pr, p);
              sum += v[p];
            }
          const float mean = sum / (float)g.P;
          float var = 0.f;
#pragma unroll
          for (int p = 0; p < kPairMax; ++p)
            if (p < g.P) var += (v[p] - mean) * (v[p] - mean);
          const float rstd = 1.f / sqrtf(var / (float)g.P + g.eps);
          for (int64_t h = 0; h < H; ++h) {
            float bsum = 0.f;
#pragma unroll
            for (int p = 0; p < kPairMax; ++p)
              if (p < g.P) bsum += (v[p] - mean) * rstd * g.w_pair[p * H + h];
            beta[idx * H + h] = bsum;
          }
        }
      }
    }
    plan[idx] = jj;
  }
  if (lo <= hi) {
    atomicMin(&s_lo, lo);
    atomicMax(&s_hi, hi);
  }
  __syncthreads();
  const int klo = s_lo, khi = s_hi;
  const bool any = klo <= khi;
  const bool staged = any && (khi - klo + 1) <= g.cap_rows;
  if (any && !staged && tid == 0) atomicOr(g.status, 1u);
  float *lg = lgb + warp * K;

  // ---------------- phase 2: head by head
  for (int64_t h = 0; h < H; ++h) {
    if (staged) {
      const int rows = khi - klo + 1;
      for (int64_t idx = tid; idx < (int64_t)rows * D; idx += kAttnThreads) {
        const int64_t r = idx / D, d = idx % D;
        const int64_t src = (b * A + klo + r) * HD + h * D + d;
        ks[r * g.DP + d] = g.Kf[src];
        vs[r * g.DP + d] = g.Vf[src];
      }
    }
    __syncthreads();
    for (int q = warp; q < QT; q += kAttnWarps) {
      const int64_t a = a0 + q;
      if (a >= A) break;
      const int64_t arow = b * A + a;
      float qv[DMAX];
#pragma unroll
      for (int d = 0; d < DMAX; ++d) qv[d] = d < D ? g.Q[arow * HD + h * D + d] : 0.f;
      // logits of the lane's slots, and their maximum over permitted slots
      float mx = -INFINITY;
      for (int64_t k = lane; k < K; k += kWarp) {
        const int j = plan[q * K + k];
        float l = -INFINITY;
        if (j >= 0) {
          const float *kr = staged ? ks + (int64_t)(j - klo) * g.DP : g.Kf + (b * A + j) * HD + h * D;
          float dot = 0.f;
#pragma unroll
          for (int d = 0; d < DMAX; ++d)
            if (d < D) dot = fmaf(qv[d], kr[d], dot);
          l = dot * g.inv_sqrt_d;
          if (AF3) l += beta[(q * K + k) * H + h];
          mx = fmaxf(mx, l);
        }
        lg[k] = l;
      }
      mx = warp_max(mx);
      float sum = 0.f;
      for (int64_t k = lane; k < K; k += kWarp) {
        const float e = plan[q * K + k] >= 0 ? expf(lg[k] - mx) : 0.f;
        lg[k] = e;
        sum += e;
      }
      sum = warp_sum(sum);
      // normalised weights: exact zero off the permitted set and on empty rows
      float acc[DMAX];
#pragma unroll
      for (int d = 0; d < DMAX; ++d) acc[d] = 0.f;
      for (int64_t k = lane; k < K; k += kWarp) {
        const int j = plan[q * K + k];
        const float w = j >= 0 ? lg[k] / sum : 0.f;
        stf((T *)g.attention, ((b * H + h) * A + a) * K + k, w);
        if (j >= 0) {
          const float *vr = staged ? vs + (int64_t)(j - klo) * g.DP : g.Vf + (b * A + j) * HD + h * D;
#pragma unroll
          for (int d = 0; d < DMAX; ++d)
            if (d < D) acc[d] = fmaf(w, vr[d], acc[d]);
        }
      }
      // reduce the per-lane partial outputs; value gate; head-major store
      const bool has = sum > 0.f;
#pragma unroll
      for (int d = 0; d < DMAX; ++d) {
        if (d < D) {
          const float o = warp_sum(acc[d]);
          if ((d & 31) == lane) {
            const int64_t oi = arow * HD + h * D + d;
            g.O[oi] = has ? o * sigmoidf_(g.G[oi]) : 0.f;
          }
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace atomenc
