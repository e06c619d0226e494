// attention.cuh -- slot-gathered windowed attention (the HBM-bound core of the block).
//
// Page "Local atom attention, encoder pooling and decoder skip/readout", Required
// behavior: a slot (query a, slot k) is permitted iff its key id j is in [0, A), both
// atoms are usable, window_mask is set and, for radius >= 0, |j - a| <= radius (bullets
// 4, 5); logits are Q_a . K_j / sqrt(D) plus, in AF3 style, the pair bias
// (LN(pair) * pair_scale) @ w_pair (bullets 8, 15); a stabilised softmax runs over the
// permitted slots only, a row without any gets exact zeros, repeated slots are separate
// entries (bullets 5, 6, 15); the weighted values are multiplied by sigmoid of the value
// gate logits and stored head-major (bullet 16).
//
// One CTA owns QT consecutive queries of one batch element.
//  Phase 1 reads key_index and window_mask once and writes the tile's slot plan (key id
//  or -1) to shared memory, with the span [klo, khi] of the permitted key ids.
//  Phase 2 walks the heads in groups: as many heads as the shared-memory stage holds for
//  this span are staged (K and V rows of the span, float32), then each warp takes one
//  query at a time with its 32 lanes over the slots (4 slots per lane per 128-slot
//  chunk): logits, masked softmax (max / sum by warp shuffles), attention weights
//  written once, the weighted value sum kept per lane and folded across lanes by a
//  butterfly reduce-scatter (lane l ends with channel l), value gate, store.
//  AF3: the pair bias of the lane's slots is computed from the pair rows (read once per
//  head group, LayerNorm over P in registers) for every head of the group.
//  When even one head of the span does not fit, the tile reads K/V rows straight from
//  global memory (L2) instead and sets status bit 1; the results are the same.
#pragma once

#include <climits>

#include "common.cuh"

namespace atomenc {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / kWarp;
constexpr int kPairMax = 32;
constexpr int kSlotsPerLane = 4;                       // one chunk = 128 slots
constexpr int kChunk = kWarp * kSlotsPerLane;
constexpr int kAf3HeadsMax = 4;   // pair-bias heads held in registers per stage
constexpr int kAttnHeadsMax = 64;  // AF3 w_pair columns kept in shared memory

struct AttnArgs {
  int64_t B, A, K, H, D, P;
  int64_t radius;
  float inv_sqrt_d, eps;
  int QT, DP, kv_floats;          // queries per CTA, padded row width, K/V stage size
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

// Butterfly reduce-scatter of v[0..W) summed over the 32 lanes: afterwards v[0] holds
// the full sum of channel (lane & (W-1)). W is a power of two <= 32.
template <int W>
__device__ __forceinline__ float reduce_scatter(float (&v)[W], int lane) {
#pragma unroll
  for (int w = W / 2; w >= 1; w /= 2) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
#pragma unroll
  for (int s = W; s < 32; s *= 2) v[0] += __shfl_xor_sync(0xffffffffu, v[0], s);
  return v[0];
}

template <int DMAX>
__device__ __forceinline__ float dot_row(const float (&q)[DMAX], const float *r) {
  // r is 16-byte aligned and zero-padded to DMAX in shared memory
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int d = 0; d < DMAX; d += 4) {
    const float4 k = *reinterpret_cast<const float4 *>(r + d);
    s0 = fmaf(q[d], k.x, s0);
    s1 = fmaf(q[d + 1], k.y, s1);
    s2 = fmaf(q[d + 2], k.z, s2);
    s3 = fmaf(q[d + 3], k.w, s3);
  }
  return (s0 + s1) + (s2 + s3);
}

template <int DMAX>
__device__ __forceinline__ float dot_global(const float (&q)[DMAX], const float *r, int64_t D) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int d = 0; d < DMAX; d += 2) {
    if (d < D) s0 = fmaf(q[d], r[d], s0);
    if (d + 1 < D) s1 = fmaf(q[d + 1], r[d + 1], s1);
  }
  return s0 + s1;
}

// Pair bias of one slot for heads h0 .. h0+NB-1 (those < hg):
//   beta_h = sum_p LN(pair)_p * pair_scale_p * w_pair[p, h]
//          = rstd * (sum_p y_p W'[p, h] - m * sum_p W'[p, h]),
// with y_p = pair_p - pair_0 (a shift that keeps the one-pass variance well conditioned),
// m = mean(y), rstd = 1 / sqrt(mean(y^2) - m^2 + eps) (population variance, eps inside
// the root). W' = pair_scale * w_pair and its column sums live in shared memory.
template <typename T, int NB>
__device__ __forceinline__ void pair_bias(const T *pr, int P, float eps, const float *wp,
                                          const float *wsum, int H, int h0, int hg,
                                          float (&beta)[NB]) {
  const float x0 = ldf(pr, 0);
  float s1 = 0.f, s2 = 0.f, dot[NB];
#pragma unroll
  for (int x = 0; x < NB; ++x) dot[x] = 0.f;
  for (int p = 0; p < P; ++p) {
    const float y = ldf(pr, p) - x0;
    s1 += y;
    s2 = fmaf(y, y, s2);
#pragma unroll
    for (int x = 0; x < NB; ++x)
      if (x < hg) dot[x] = fmaf(y, wp[p * H + h0 + x], dot[x]);
  }
  const float m = s1 / (float)P;
  const float var = fmaxf(s2 / (float)P - m * m, 0.f);
  const float rstd = 1.f / sqrtf(var + eps);
#pragma unroll
  for (int x = 0; x < NB; ++x) beta[x] = x < hg ? rstd * (dot[x] - m * wsum[h0 + x]) : 0.f;
}

// MULTI = false: K <= 128, one chunk, logits kept in registers.
// MULTI = true:  any K; pass 1 finds the max and the sum chunk by chunk, pass 2
//                recomputes the logits to write the weights and accumulate the values.
template <typename T, int DMAX, bool AF3, bool MULTI>
__global__ void __launch_bounds__(kAttnThreads, 2) k_slot_attention(AttnArgs g) {
  extern __shared__ __align__(16) float smem[];
  constexpr int DW = DMAX < 32 ? DMAX : 32;            // channels per reduce-scatter
  constexpr int NB = AF3 ? kAf3HeadsMax : 1;            // pair-bias heads kept per slot
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b = blockIdx.y, a0 = (int64_t)blockIdx.x * g.QT;
  const int QT = g.QT;
  const int64_t K = g.K, A = g.A;
  const int H = (int)g.H, D = (int)g.D, HD = H * D;
  const int DP = g.DP, P = (int)g.P;

  int *plan = reinterpret_cast<int *>(smem);                           // [QT*K]
  float *kv = smem + (((int64_t)QT * K + 3) & ~int64_t(3));            // [kv_floats]
  __shared__ int s_lo, s_hi;
  __shared__ float s_wp[kPairMax * kAttnHeadsMax], s_wsum[kAttnHeadsMax];
  if (tid == 0) {
    s_lo = INT_MAX;
    s_hi = -1;
  }
  if (AF3) {
    for (int i = tid; i < P * H; i += kAttnThreads) s_wp[i] = g.w_pair[i];
    for (int h = tid; h < H; h += kAttnThreads) {
      float sw = 0.f;
      for (int p = 0; p < P; ++p) sw += g.w_pair[p * H + h];
      s_wsum[h] = sw;
    }
  }
  __syncthreads();

  // ---------------- phase 1: slot plan, one pass over the tile's key_index / window_mask
  int lo = INT_MAX, hi = -1;
  for (int q = warp; q < QT; q += kAttnWarps) {
    const int64_t a = a0 + q;
    const bool qok = a < A && g.usable[b * A + a] != 0;
    for (int k = lane; k < (int)K; k += kWarp) {
      int jj = -1;
      if (qok) {
        const int64_t s = (b * A + a) * K + k;
        const int64_t j = g.key_index[s];
        bool ok = j >= 0 && j < A && g.window[s] != 0;
        ok = ok && g.usable[b * A + j] != 0;
        if (ok && g.radius >= 0) ok = (j > a ? j - a : a - j) <= g.radius;
        if (ok) {
          jj = (int)j;
          lo = min(lo, jj);
          hi = max(hi, jj);
        }
      }
      plan[q * (int)K + k] = jj;
    }
  }
  if (lo <= hi) {
    atomicMin(&s_lo, lo);
    atomicMax(&s_hi, hi);
  }
  __syncthreads();
  const int klo = s_lo, khi = s_hi;
  const int span = khi >= klo ? khi - klo + 1 : 0;
  int HG = H;
  if (span > 0) {
    const int64_t fit = g.kv_floats / (2 * (int64_t)span * DP);
    HG = (int)(fit < H ? fit : H);
  }
  const bool staged = span > 0 && HG >= 1;
  if (!staged) HG = H;
  if (AF3) HG = min(HG, kAf3HeadsMax);
  if (span > 0 && !staged && tid == 0) atomicOr(g.status, 1u);
  const int nchunks = MULTI ? (int)((K + kChunk - 1) / kChunk) : 1;
  const float log2e = 1.4426950408889634f;

  // ---------------- phase 2: head groups
  for (int h0 = 0; h0 < H; h0 += HG) {
    const int hg = H - h0 < HG ? H - h0 : HG;
    float *ks = kv, *vs = kv + (int64_t)hg * span * DP;
    if (staged) {
      // one float4 chunk of one staged row per lane: rows_per_pass rows per warp pass
      const int CH = DP / 4, rpp = kWarp / CH, rsub = lane / CH, c4 = (lane - rsub * CH) * 4;
      const bool vec = (D & 3) == 0;
      for (int hl = 0; hl < hg; ++hl) {
        const int64_t col = (int64_t)(h0 + hl) * D + c4;
        for (int r0 = warp * rpp; r0 < span; r0 += kAttnWarps * rpp) {
          const int rr = r0 + rsub;
          if (rsub >= rpp || rr >= span) continue;
          float4 kx = make_float4(0.f, 0.f, 0.f, 0.f), vx = kx;
          const int64_t src = (b * A + klo + rr) * HD + col;
          if (vec) {
            if (c4 < D) {
              kx = *reinterpret_cast<const float4 *>(g.Kf + src);
              vx = *reinterpret_cast<const float4 *>(g.Vf + src);
            }
          } else {
            float kk[4] = {0.f, 0.f, 0.f, 0.f}, vv[4] = {0.f, 0.f, 0.f, 0.f};
            for (int e = 0; e < 4; ++e)
              if (c4 + e < D) {
                kk[e] = g.Kf[src + e];
                vv[e] = g.Vf[src + e];
              }
            kx = make_float4(kk[0], kk[1], kk[2], kk[3]);
            vx = make_float4(vv[0], vv[1], vv[2], vv[3]);
          }
          const int64_t dst = ((int64_t)hl * span + rr) * DP + c4;
          *reinterpret_cast<float4 *>(ks + dst) = kx;
          *reinterpret_cast<float4 *>(vs + dst) = vx;
        }
      }
    }
    __syncthreads();

    for (int q = warp; q < QT; q += kAttnWarps) {
      const int64_t a = a0 + q;
      if (a >= A) break;
      const int64_t arow = b * A + a;
      const T *prow = AF3 ? (const T *)g.pair + arow * K * P : nullptr;

      int jr[kSlotsPerLane];
      float beta[kSlotsPerLane][NB];
      if (!MULTI) {
#pragma unroll
        for (int i = 0; i < kSlotsPerLane; ++i) {
          const int k = i * kWarp + lane;
          jr[i] = k < K ? plan[q * K + k] : -1;
          if (AF3) {
            if (jr[i] >= 0)
              pair_bias<T, NB>(prow + (int64_t)k * P, P, g.eps, s_wp, s_wsum, H, h0, hg, beta[i]);
            else
#pragma unroll
              for (int x = 0; x < NB; ++x) beta[i][x] = 0.f;
          }
        }
      }

      for (int hl = 0; hl < hg; ++hl) {
        const int h = h0 + hl;
        float qv[DMAX];
        const float *qsrc = g.Q + arow * HD + h * D;
        if ((D & 3) == 0) {
#pragma unroll
          for (int d = 0; d < DMAX; d += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (d < D) x = *reinterpret_cast<const float4 *>(qsrc + d);
            qv[d] = x.x;
            qv[d + 1] = x.y;
            qv[d + 2] = x.z;
            qv[d + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int d = 0; d < DMAX; ++d) qv[d] = d < D ? qsrc[d] : 0.f;
        }
        const float *kbase = staged ? ks + (int64_t)hl * span * DP : nullptr;
        const float *vbase = staged ? vs + (int64_t)hl * span * DP : nullptr;

        // logit in log2 units (exp2 of a difference of them = e^difference)
        auto logit = [&](int64_t k, int i, int j) -> float {
          float dot = staged ? dot_row<DMAX>(qv, kbase + (int64_t)(j - klo) * DP)
                             : dot_global<DMAX>(qv, g.Kf + (b * A + j) * HD + h * D, D);
          float l = dot * g.inv_sqrt_d;
          if (AF3) {
            if (!MULTI) {
              float bsel = 0.f;
#pragma unroll
              for (int x = 0; x < NB; ++x)
                if (x == hl) bsel = beta[i][x];
              l += bsel;
            } else {
              float b1[1];
              pair_bias<T, 1>(prow + k * P, P, g.eps, s_wp, s_wsum, H, h, 1, b1);
              l += b1[0];
            }
          }
          return l * log2e;
        };

        float mx = -INFINITY, sum = 0.f;
        float l2[kSlotsPerLane];
        for (int c = 0; c < nchunks; ++c) {
          float cmx = -INFINITY;
#pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            const int64_t k = (int64_t)c * kChunk + i * kWarp + lane;
            if (MULTI) jr[i] = k < K ? plan[q * K + k] : -1;
            l2[i] = jr[i] >= 0 ? logit(k, i, jr[i]) : -INFINITY;
            cmx = fmaxf(cmx, l2[i]);
          }
          cmx = warp_max(cmx);
          if (cmx > -INFINITY) {
            const float nm = fmaxf(mx, cmx);
            float cs = 0.f;
#pragma unroll
            for (int i = 0; i < kSlotsPerLane; ++i)
              if (jr[i] >= 0) cs += exp2f(l2[i] - nm);
            sum = sum * exp2f(mx - nm) + warp_sum(cs);
            mx = nm;
          }
        }
        const float inv = sum > 0.f ? 1.f / sum : 0.f;

        float acc[DMAX];
#pragma unroll
        for (int d = 0; d < DMAX; ++d) acc[d] = 0.f;
        for (int c = 0; c < nchunks; ++c) {
#pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            const int64_t k = (int64_t)c * kChunk + i * kWarp + lane;
            if (MULTI) {
              jr[i] = k < K ? plan[q * K + k] : -1;
              l2[i] = jr[i] >= 0 ? logit(k, i, jr[i]) : -INFINITY;
            }
            const int j = jr[i];
            const float wgt = j >= 0 ? exp2f(l2[i] - mx) * inv : 0.f;
            if (k < K) stf((T *)g.attention, ((b * H + h) * A + a) * K + k, wgt);
            if (j >= 0) {
              if (staged) {
                const float *vr = vbase + (int64_t)(j - klo) * DP;
#pragma unroll
                for (int d = 0; d < DMAX; d += 4) {
                  const float4 v = *reinterpret_cast<const float4 *>(vr + d);
                  acc[d] = fmaf(wgt, v.x, acc[d]);
                  acc[d + 1] = fmaf(wgt, v.y, acc[d + 1]);
                  acc[d + 2] = fmaf(wgt, v.z, acc[d + 2]);
                  acc[d + 3] = fmaf(wgt, v.w, acc[d + 3]);
                }
              } else {
                const float *vr = g.Vf + (b * A + j) * HD + h * D;
#pragma unroll
                for (int d = 0; d < DMAX; ++d)
                  if (d < D) acc[d] = fmaf(wgt, vr[d], acc[d]);
              }
            }
          }
        }

        // fold the lanes' partial outputs: lane l ends with channel l (and l + 32)
        const bool has = sum > 0.f;
#pragma unroll
        for (int part = 0; part < DMAX; part += DW) {
          float v[DW];
#pragma unroll
          for (int i = 0; i < DW; ++i) v[i] = acc[part + i];
          const float o = reduce_scatter<DW>(v, lane);
          const int d = part + (lane & (DW - 1));
          if (lane < DW && d < D) {
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
