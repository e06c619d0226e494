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
// One CTA (512 threads, one per SM; AF3: 256 threads, two per SM) owns QT consecutive
// queries of one batch element.
//  Phase 1  (may run while the projections finish) one slot per thread per round, eight
//           rounds in flight: key_index and window_mask are read once (coalesced),
//           eligibility decided and the slot plan written with the span [klo, khi] of
//           the permitted ids; AF3: the pair bias of every permitted (slot, head) is
//           computed from its pair row (16-byte loads, LayerNorm over P in one shifted
//           pass) and kept in shared memory as float32 [head][slot].
//  Phase 0  (after the wait for the projections) the tile's Q rows are copied to shared
//           memory with cp.async.
//  Phase 2  head groups: the K and V rows of the span for as many heads as fit are staged
//           (float32, cp.async); the warps share the (query, head) pairs, lanes over the
//           slots (4 per lane per 128-slot chunk): logits, max, one exp2 per entry, sum,
//           weights written once (bf16 rounded with integer ops), the weighted value sum
//           per lane with packed f32x2 FMAs, folded across lanes by a butterfly
//           reduce-scatter, value gate, store. Queries that read the same key rows may be
//           processed two at a time (each row read once for both).
// A tile whose span does not fit even one head reads K/V rows from global memory (L2)
// instead and sets status bit 1; the results are the same.
#pragma once

#include <climits>

#include "common.cuh"

namespace atomenc {

// block size: ESMFold2 one 512-thread CTA per SM; AF3 two 256-thread CTAs per SM, so that
// one CTA's pair-bias phase (its pair rows are the largest input) overlaps the other's
// attention
__host__ __device__ constexpr int attn_threads(bool af3) { return af3 ? 256 : 512; }
__host__ __device__ constexpr int attn_ctas_per_sm(bool af3) { return af3 ? 2 : 1; }
constexpr int kPairMax = 32;
constexpr int kSlotsPerLane = 4;                       // one chunk = 128 slots
constexpr int kChunk = kWarp * kSlotsPerLane;
constexpr int kAttnHeadsMax = 32;                      // AF3 w_pair columns in shared memory
constexpr int kMaxQT = 64;                             // queries per CTA at most

struct AttnArgs {
  int B, A, K, H, D, P;
  int radius;                     // -1 = no index window
  float scale_log2;               // log2(e) / sqrt(D)
  float eps;
  int QT, DP, kv_floats;          // queries per CTA, padded row width, K/V stage size
  uint32_t kmagic;                // ceil(2^32 / K) for K > 1: s / K == umulhi(s, kmagic), s < QT*K
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

// float counts of the shared regions, each rounded to 4 floats (16-byte aligned regions)
__host__ __device__ inline size_t ru4(size_t n) { return (n + 3) & ~size_t(3); }
__host__ __device__ inline size_t attn_fixed_smem(int QT, int K, int H, int HD, bool af3) {
  const size_t slots = (size_t)QT * K;
  return 4 * (ru4(slots) + (af3 ? ru4((size_t)H * slots) : 0) + ru4((size_t)QT * HD));
}


// 16-byte / 4-byte shared-memory loads by 32-bit shared address
__device__ __forceinline__ ulonglong2 lds128(uint32_t addr) {
  ulonglong2 v;
  asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ float lds32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// 2^x on the special-function unit (the exponent of the softmax is always <= 0 here)
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// float -> bf16 bits, round to nearest even, by integer arithmetic (finite inputs)
__device__ __forceinline__ uint16_t bf16_rne(float x) {
  const uint32_t u = __float_as_uint(x);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

template <typename T>
__device__ __forceinline__ void store_weight(T *p, int64_t i, float w);
template <>
__device__ __forceinline__ void store_weight<float>(float *p, int64_t i, float w) { p[i] = w; }
template <>
__device__ __forceinline__ void store_weight<__nv_bfloat16>(__nv_bfloat16 *p, int64_t i, float w) {
  reinterpret_cast<uint16_t *>(p)[i] = bf16_rne(w);
}

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

// Pair bias of one slot for every head:
//   beta_h = sum_p LN(pair)_p * pair_scale_p * w_pair[p, h]
//          = rstd * (sum_p y_p W'[p, h] - m * sum_p W'[p, h]),
// y_p = pair_p - pair_0 (a shift that keeps the one-pass variance well conditioned),
// m = mean(y), rstd = 1 / sqrt(mean(y^2) - m^2 + eps); W' = pair_scale * w_pair and its
// column sums are in shared memory ([P][H] and [H]).
template <int NP>
__device__ __forceinline__ void pair_bias_from(const float (&x)[NP], int P, int H, float eps,
                                               const float *wp, const float *wsum, float *out,
                                               int out_stride) {
  float y[NP];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    y[p] = x[p] - x[0];
    s1 += y[p];
    s2 = fmaf(y[p], y[p], s2);
  }
  const float invP = 1.f / (float)NP;
  const float m = s1 * invP;
  const float var = fmaxf(s2 * invP - m * m, 0.f);
  const float rstd = rsqrtf(var + eps);
  int h = 0;
  if ((H & 3) == 0) {
    for (; h < H; h += 4) {
      float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float4 w = *reinterpret_cast<const float4 *>(wp + p * H + h);
        d0 = fmaf(y[p], w.x, d0);
        d1 = fmaf(y[p], w.y, d1);
        d2 = fmaf(y[p], w.z, d2);
        d3 = fmaf(y[p], w.w, d3);
      }
      out[(h + 0) * out_stride] = rstd * (d0 - m * wsum[h + 0]);
      out[(h + 1) * out_stride] = rstd * (d1 - m * wsum[h + 1]);
      out[(h + 2) * out_stride] = rstd * (d2 - m * wsum[h + 2]);
      out[(h + 3) * out_stride] = rstd * (d3 - m * wsum[h + 3]);
    }
  }
  for (; h < H; ++h) {
    float d = 0.f;
#pragma unroll
    for (int p = 0; p < NP; ++p) d = fmaf(y[p], wp[p * H + h], d);
    out[h * out_stride] = rstd * (d - m * wsum[h]);
  }
}

// 16 channels of a pair row by 16-byte loads (bf16: 2 loads, float32: 4 loads)
__device__ __forceinline__ void load_pair16(const __nv_bfloat16 *pr, float (&x)[16]) {
  const uint4 a = *reinterpret_cast<const uint4 *>(pr);
  const uint4 b = *reinterpret_cast<const uint4 *>(pr + 8);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load_pair16(const float *pr, float (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = *reinterpret_cast<const float4 *>(pr + 4 * i);
    x[4 * i] = v.x;
    x[4 * i + 1] = v.y;
    x[4 * i + 2] = v.z;
    x[4 * i + 3] = v.w;
  }
}

// generic P (any width up to kPairMax): scalar loads
template <typename T>
__device__ __forceinline__ void pair_bias_generic(const T *pr, int P, int H, float eps,
                                                  const float *wp, const float *wsum, float *out,
                                                  int out_stride) {
  const float x0 = ldf(pr, 0);
  float s1 = 0.f, s2 = 0.f;
  for (int p = 0; p < P; ++p) {
    const float y = ldf(pr, p) - x0;
    s1 += y;
    s2 = fmaf(y, y, s2);
  }
  const float m = s1 / (float)P;
  const float var = fmaxf(s2 / (float)P - m * m, 0.f);
  const float rstd = rsqrtf(var + eps);
  for (int h = 0; h < H; ++h) {
    float d = 0.f;
    for (int p = 0; p < P; ++p) d = fmaf(ldf(pr, p) - x0, wp[p * H + h], d);
    out[h * out_stride] = rstd * (d - m * wsum[h]);
  }
}

// q . r with the query already packed in registers (zero beyond D) and the key row in
// shared memory (16-byte aligned, zero-padded to DMAX)
template <int DMAX>
__device__ __forceinline__ float dot_q2(const f32x2 (&q2)[DMAX / 2], const float *r) {
  f32x2 s0 = 0ull, s1 = 0ull;
#pragma unroll
  for (int d = 0; d < DMAX; d += 4) {
    const ulonglong2 k = *reinterpret_cast<const ulonglong2 *>(r + d);
    s0 = ffma2(q2[d / 2], k.x, s0);
    s1 = ffma2(q2[d / 2 + 1], k.y, s1);
  }
  const float2 x = unpack2(s0), y = unpack2(s1);
  return (x.x + x.y) + (y.x + y.y);
}
// the same with the key row read from global memory (D floats, any alignment)
template <int DMAX>
__device__ __forceinline__ float dot_q2_global(const f32x2 (&q2)[DMAX / 2], const float *r, int D) {
  f32x2 s = 0ull;
#pragma unroll
  for (int d = 0; d < DMAX; d += 2) {
    if (d < D) s = ffma2(q2[d / 2], pack2(r[d], d + 1 < D ? r[d + 1] : 0.f), s);
  }
  const float2 x = unpack2(s);
  return x.x + x.y;
}

// MULTI = false: K <= 128, one chunk, logits and exponentials kept in registers.
// MULTI = true:  any K; pass 1 finds the max and the sum chunk by chunk, pass 2
//                recomputes the logits to write the weights and accumulate the values.
template <typename T, int DMAX, bool AF3, bool MULTI>
__global__ void __launch_bounds__(attn_threads(AF3), attn_ctas_per_sm(AF3)) k_slot_attention(AttnArgs g) {
  // the slot plan and the pair bias read only the caller's inputs, the usable flags and
  // the folded pair weights (all from kernels at least two places earlier), so they run
  // before the wait for the projections; Q, K, V, G are read after it
  pdl_launch_next();
  constexpr int kAttnThreads = attn_threads(AF3), kAttnWarps = kAttnThreads / kWarp;
  extern __shared__ __align__(16) float smem[];
  constexpr int DW = DMAX < 32 ? DMAX : 32;            // channels per reduce-scatter
  // Query pairs sharing their key rows are processed jointly in the 128-slot path; built
  // for the ESMFold2 style at 16 < D <= 32 only (with the AF3 pair-bias reads, or at
  // D <= 16, the joint path's registers were measured to cost more than the halved row
  // reads save).
  constexpr bool kPairs = !MULTI && !AF3 && DMAX == 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y, a0 = blockIdx.x * g.QT;
  const int QT = g.QT, K = g.K, H = g.H, D = g.D, A = g.A, HD = H * D, DP = g.DP, P = g.P;
  const int nq = min(QT, A - a0);                      // queries of this tile
  const int slots = QT * K;
  const bool vecD = (D & 3) == 0;                      // 16-byte rows of Q, K, V
  const bool fullD = D == DMAX;                        // shared Q rows cover DMAX exactly

  int *plan = reinterpret_cast<int *>(smem);                          // [QT*K]
  float *beta = smem + ru4(slots);                                    // [H][QT*K] (AF3)
  float *qs = beta + (AF3 ? ru4((size_t)H * slots) : 0);              // [QT][HD]
  float *kv = qs + ru4((size_t)QT * HD);                              // [kv_floats]
  __shared__ int s_lo, s_hi;
  __shared__ int s_pairs_differ;                    // some pair (2p, 2p + 1) reads different rows
  __shared__ __align__(16) float s_wp[AF3 ? kPairMax * kAttnHeadsMax : 4];  // float4 rows
  __shared__ __align__(16) float s_wsum[AF3 ? kAttnHeadsMax : 4];
  if (tid == 0) {
    s_lo = INT_MAX;
    s_hi = -1;
  }

  // ---------------- pair weights
  if (AF3) {
    for (int i = tid; i < P * H; i += kAttnThreads) s_wp[i] = g.w_pair[i];
    for (int h = tid; h < H; h += kAttnThreads) {
      float sw = 0.f;
      for (int p = 0; p < P; ++p) sw += g.w_pair[p * H + h];
      s_wsum[h] = sw;
    }
  }
  __syncthreads();

  // ---------------- phase 1a: slot plan, one slot per thread per round (coalesced
  // 8-byte key_index loads, consecutive shared stores), eight rounds in flight
  int lo = INT_MAX, hi = -1;
  const int64_t sbase = ((int64_t)b * A + a0) * K;     // first slot of the tile
  const int vslots = nq * K;
  constexpr int R = 8;
  for (int s0 = tid; s0 < slots; s0 += kAttnThreads * R) {
    int64_t kid[R];
    uint8_t win[R];
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int s = s0 + u * kAttnThreads;
      const bool in = s < vslots;
      kid[u] = in ? g.key_index[sbase + s] : -1;
      win[u] = in ? g.window[sbase + s] : 0;
    }
    int jj[R], raw[R];
    bool qu[R];
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int s = s0 + u * kAttnThreads;
      const int q = K == 1 ? s : (int)__umulhi((uint32_t)s, g.kmagic);
      const int a = a0 + q;
      const int64_t j = kid[u];
      bool ok = s < vslots && win[u] != 0 && j >= 0 && j < A;
      raw[u] = kPairs && s < vslots && j >= 0 && j < A ? (int)j : -1;
      if (ok && g.radius >= 0) ok = (j > a ? j - a : a - j) <= g.radius;
      jj[u] = ok ? (int)j : -1;
      qu[u] = s < vslots && g.usable[(int64_t)b * A + a] != 0;
    }
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int s = s0 + u * kAttnThreads;
      if (jj[u] >= 0 && (!qu[u] || g.usable[(int64_t)b * A + jj[u]] == 0)) jj[u] = -1;
      // plan: key id of a permitted slot; -2 - id for a slot that names a key in [0, A)
      // but is not permitted (its row may still be read, with weight 0); -1 otherwise
      if (s < slots) plan[s] = jj[u] >= 0 ? jj[u] : (kPairs && raw[u] >= 0 ? -2 - raw[u] : -1);
      if (jj[u] >= 0) {
        lo = min(lo, jj[u]);
        hi = max(hi, jj[u]);
      }
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0 && lo <= hi) {
    atomicMin(&s_lo, lo);
    atomicMax(&s_hi, hi);
  }
  // ---------------- phase 1b (AF3): pair bias of every permitted (slot, head), one slot
  // per thread per round, rows read with 16-byte loads, two rows in flight
  if (AF3) {
    __syncthreads();
    const T *pbase = (const T *)g.pair + sbase * P;
    const bool p16 = P == 16 && (reinterpret_cast<uintptr_t>(g.pair) & 15) == 0;
    for (int s0 = tid; s0 < vslots; s0 += 2 * kAttnThreads) {
      const int s1 = s0 + kAttnThreads;
      const bool on0 = plan[s0] >= 0, on1 = s1 < vslots && plan[s1] >= 0;
      if (p16) {
        float x0[16], x1[16];
        if (on0) load_pair16(pbase + (int64_t)s0 * 16, x0);
        if (on1) load_pair16(pbase + (int64_t)s1 * 16, x1);
        if (on0) pair_bias_from<16>(x0, P, H, g.eps, s_wp, s_wsum, beta + s0, slots);
        if (on1) pair_bias_from<16>(x1, P, H, g.eps, s_wp, s_wsum, beta + s1, slots);
      } else {
        if (on0) pair_bias_generic<T>(pbase + (int64_t)s0 * P, P, H, g.eps, s_wp, s_wsum, beta + s0, slots);
        if (on1) pair_bias_generic<T>(pbase + (int64_t)s1 * P, P, H, g.eps, s_wp, s_wsum, beta + s1, slots);
      }
    }
  }

  // ---------------- phase 0 (after the wait for the projections): the tile's Q rows
  pdl_wait();
  const int64_t qbase = ((int64_t)b * A + a0) * HD;
  if (vecD) {
    for (int i = tid; i < nq * HD / 4; i += kAttnThreads) {
      const uint32_t dst = (uint32_t)__cvta_generic_to_shared(qs + 4 * i);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(g.Q + qbase + 4 * i)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  } else {
    for (int i = tid; i < nq * HD; i += kAttnThreads) qs[i] = g.Q[qbase + i];
  }
  __syncthreads();
  const int klo = s_lo, khi = s_hi;
  const int span = khi >= klo ? khi - klo + 1 : 0;
  int HG = H;
  if (span > 0) {
    const int fit = g.kv_floats / (2 * span * DP);
    HG = fit < H ? fit : H;
  }
  const bool staged = span > 0 && HG >= 1;
  if (!staged) HG = H;
  if (span > 0 && !staged && tid == 0) atomicOr(g.status, 1u);
  const int nchunks = MULTI ? (K + kChunk - 1) / kChunk : 1;

  // the staged row a slot reads: its key if permitted, else its named key when that is in
  // the span, else the span's first row (weight 0 either way)
  auto row_of = [&](int p) -> int {
    const int r = p >= 0 ? p : -2 - p;
    return p >= 0 || (p <= -2 && r >= klo && r <= khi) ? r : klo;
  };
  // 128-slot path: does every pair of queries (2p, 2p + 1) of the tile read the same row
  // in every slot (blocked windows)? Then each pair is processed by one warp with every
  // K/V row read once for both queries.
  const bool fast = !MULTI && staged && K == kChunk;
  if (kPairs && fast) {
    if (tid == 0) s_pairs_differ = 0;
    __syncthreads();
    bool differ = false;
    for (int q = 2 * warp; q + 1 < nq; q += 2 * kAttnWarps) {
#pragma unroll
      for (int i = 0; i < kSlotsPerLane; ++i) {
        const int k = i * kWarp + lane;
        differ = differ || row_of(plan[q * K + k]) != row_of(plan[(q + 1) * K + k]);
      }
    }
    if (__any_sync(0xffffffffu, differ) && lane == 0) s_pairs_differ = 1;
    __syncthreads();
  }
  const bool all_pairs = kPairs && fast && s_pairs_differ == 0;

  // ---------------- phase 2: head groups
  for (int h0 = 0; h0 < H; h0 += HG) {
    const int hg = H - h0 < HG ? H - h0 : HG;
    float *ks = kv, *vs = kv + hg * span * DP;
    if (staged) {
      // one 16-byte chunk of one staged row per lane; only the DMAX columns that are read
      // (zero-filled beyond D when D < DMAX), so every lane of a pass does the same work
      constexpr int CH = DMAX / 4, rpp = kWarp / CH;
      const int rsub = lane / CH, c4 = (lane - rsub * CH) * 4;
      for (int hl = 0; hl < hg; ++hl) {
        const int col = (h0 + hl) * D + c4;
        for (int r0 = warp * rpp; r0 < span; r0 += kAttnWarps * rpp) {
          const int rr = r0 + rsub;
          if (rr >= span) continue;
          const int64_t src = ((int64_t)b * A + klo + rr) * HD + col;
          float *kd = ks + (hl * span + rr) * DP + c4, *vd = vs + (hl * span + rr) * DP + c4;
          if (vecD && c4 < D) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                             (uint32_t)__cvta_generic_to_shared(kd)),
                         "l"(g.Kf + src)
                         : "memory");
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                             (uint32_t)__cvta_generic_to_shared(vd)),
                         "l"(g.Vf + src)
                         : "memory");
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              kd[e] = c4 + e < D ? g.Kf[src + e] : 0.f;
              vd[e] = c4 + e < D ? g.Vf[src + e] : 0.f;
            }
          }
        }
      }
      asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();

    if (fast) {
      if constexpr (kPairs) {
        // ---- fast path: 128 slots, staged K/V, 32-bit shared addresses, no slot guards.
        // Work items are (query pair, head); a pair whose queries read the same rows is
        // done jointly, otherwise its queries one after the other.
        const uint32_t rowb = (uint32_t)DP * 4u;
        const uint32_t kbase = (uint32_t)__cvta_generic_to_shared(ks);
        const uint32_t vbase = (uint32_t)__cvta_generic_to_shared(vs);
        const uint32_t qbase_s = (uint32_t)__cvta_generic_to_shared(qs);
        const uint32_t bbase = AF3 ? (uint32_t)__cvta_generic_to_shared(beta) : 0u;

        // q2 <- the query row (zero beyond D) from shared memory
        auto load_q = [&](uint32_t qa, f32x2 (&q2)[DMAX / 2]) {
          if (fullD) {
  #pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 x = lds128(qa + 4u * d);
              q2[d / 2] = x.x;
              q2[d / 2 + 1] = x.y;
            }
          } else {
  #pragma unroll
            for (int d = 0; d < DMAX; d += 2)
              q2[d / 2] = pack2(d < D ? lds32(qa + 4u * d) : 0.f, d + 1 < D ? lds32(qa + 4u * d + 4u) : 0.f);
          }
        };
        // ev <- exp2(l - max) of the permitted slots (0 elsewhere); returns 1/sum (0: none)
        auto softmax = [&](float (&ev)[kSlotsPerLane], const int (&jr)[kSlotsPerLane]) -> float {
          float mx = -INFINITY;
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) mx = fmaxf(mx, ev[i]);
          mx = warp_max(mx);
          float sum = 0.f;
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            ev[i] = jr[i] >= 0 ? exp2_approx(ev[i] - mx) : 0.f;
            sum += ev[i];
          }
          sum = warp_sum(sum);
          float inv = 0.f;
          if (sum > 0.f) asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(sum));
          return inv;
        };
        // fold the lanes' partial outputs, gate, store (lane l ends with channel l)
        auto finish = [&](f32x2 (&acc2)[DMAX / 2], const float (&gv)[DMAX / DW], bool has,
                          int64_t obase) {
          float acc[DMAX];
  #pragma unroll
          for (int d = 0; d < DMAX; d += 2) {
            const float2 p2 = unpack2(acc2[d / 2]);
            acc[d] = p2.x;
            acc[d + 1] = p2.y;
          }
  #pragma unroll
          for (int part = 0; part < DMAX; part += DW) {
            float v[DW];
  #pragma unroll
            for (int i = 0; i < DW; ++i) v[i] = acc[part + i];
            const float o = reduce_scatter<DW>(v, lane);
            const int d = part + (lane & (DW - 1));
            if (lane < DW && d < D) g.O[obase + d] = has ? o * sigmoid_fast(gv[part / DW]) : 0.f;
          }
        };
        auto gates = [&](int64_t obase, float (&gv)[DMAX / DW]) {
  #pragma unroll
          for (int part = 0; part < DMAX; part += DW) {
            const int d = part + (lane & (DW - 1));
            gv[part / DW] = lane < DW && d < D ? g.G[obase + d] : 0.f;
          }
        };

        // one query, one head
        auto single = [&](int q, int hl) {
          const int h = h0 + hl, a = a0 + q;
          const int64_t obase = ((int64_t)b * A + a) * HD + h * D;
          float gv[DMAX / DW];
          gates(obase, gv);
          int jr[kSlotsPerLane];
          uint32_t ja[kSlotsPerLane];
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            jr[i] = plan[q * K + i * kWarp + lane];
            ja[i] = (uint32_t)(jr[i] >= 0 ? jr[i] : klo) * rowb;
          }
          const uint32_t kb = kbase + (uint32_t)(hl * span - klo) * rowb;
          const uint32_t vb = vbase + (uint32_t)(hl * span - klo) * rowb;
          f32x2 q2[DMAX / 2];
          load_q(qbase_s + (uint32_t)(q * HD + h * D) * 4u, q2);
          const uint32_t ba = bbase + (uint32_t)(h * slots + q * K + lane) * 4u;
          float ev[kSlotsPerLane];
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            f32x2 s0 = 0ull, s1 = 0ull;
  #pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 k = lds128(kb + ja[i] + 4u * d);
              s0 = ffma2(q2[d / 2], k.x, s0);
              s1 = ffma2(q2[d / 2 + 1], k.y, s1);
            }
            const float2 x = unpack2(s0), y = unpack2(s1);
            float l = ((x.x + x.y) + (y.x + y.y)) * g.scale_log2;
            if (AF3) l = fmaf(lds32(ba + 128u * i), 1.4426950408889634f, l);
            ev[i] = jr[i] >= 0 ? l : -INFINITY;
          }
          const float inv = softmax(ev, jr);
          T *wout = (T *)g.attention + (((int64_t)b * H + h) * A + a) * K + lane;
          f32x2 acc2[DMAX / 2];
  #pragma unroll
          for (int d = 0; d < DMAX / 2; ++d) acc2[d] = 0ull;
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            const float wgt = ev[i] * inv;
            store_weight<T>(wout, i * kWarp, wgt);
            const f32x2 w2 = pack2(wgt, wgt);
  #pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 v = lds128(vb + ja[i] + 4u * d);
              acc2[d / 2] = ffma2(w2, v.x, acc2[d / 2]);
              acc2[d / 2 + 1] = ffma2(w2, v.y, acc2[d / 2 + 1]);
            }
          }
          finish(acc2, gv, inv > 0.f, obase);
        };

        // queries q and q + 1, one head, every K/V row read once for both
        auto joint = [&](int q, int hl) {
          const int h = h0 + hl, a = a0 + q;
          const int64_t obase = ((int64_t)b * A + a) * HD + h * D;
          float gv0[DMAX / DW], gv1[DMAX / DW];
          gates(obase, gv0);
          gates(obase + HD, gv1);
          int j0[kSlotsPerLane], j1[kSlotsPerLane];
          uint32_t ja[kSlotsPerLane];
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            j0[i] = plan[q * K + i * kWarp + lane];
            j1[i] = plan[(q + 1) * K + i * kWarp + lane];
            ja[i] = (uint32_t)row_of(j0[i]) * rowb;
          }
          const uint32_t kb = kbase + (uint32_t)(hl * span - klo) * rowb;
          const uint32_t vb = vbase + (uint32_t)(hl * span - klo) * rowb;
          float e0[kSlotsPerLane], e1[kSlotsPerLane];
          {
            f32x2 qa[DMAX / 2], qb[DMAX / 2];
            load_q(qbase_s + (uint32_t)(q * HD + h * D) * 4u, qa);
            load_q(qbase_s + (uint32_t)((q + 1) * HD + h * D) * 4u, qb);
            const uint32_t ba = bbase + (uint32_t)(h * slots + q * K + lane) * 4u;
  #pragma unroll
            for (int i = 0; i < kSlotsPerLane; ++i) {
              f32x2 sa = 0ull, sb = 0ull, ta = 0ull, tb = 0ull;
  #pragma unroll
              for (int d = 0; d < DMAX; d += 4) {
                const ulonglong2 k = lds128(kb + ja[i] + 4u * d);
                sa = ffma2(qa[d / 2], k.x, sa);
                ta = ffma2(qa[d / 2 + 1], k.y, ta);
                sb = ffma2(qb[d / 2], k.x, sb);
                tb = ffma2(qb[d / 2 + 1], k.y, tb);
              }
              const float2 xa = unpack2(sa), ya = unpack2(ta), xb = unpack2(sb), yb = unpack2(tb);
              float la = ((xa.x + xa.y) + (ya.x + ya.y)) * g.scale_log2;
              float lb = ((xb.x + xb.y) + (yb.x + yb.y)) * g.scale_log2;
              if (AF3) {
                la = fmaf(lds32(ba + 128u * i), 1.4426950408889634f, la);
                lb = fmaf(lds32(ba + 128u * i + 4u * K), 1.4426950408889634f, lb);
              }
              e0[i] = j0[i] >= 0 ? la : -INFINITY;
              e1[i] = j1[i] >= 0 ? lb : -INFINITY;
            }
          }
          const float inv0 = softmax(e0, j0), inv1 = softmax(e1, j1);
          T *w0 = (T *)g.attention + (((int64_t)b * H + h) * A + a) * K + lane;
          f32x2 acca[DMAX / 2], accb[DMAX / 2];
  #pragma unroll
          for (int d = 0; d < DMAX / 2; ++d) acca[d] = accb[d] = 0ull;
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            const float wa = e0[i] * inv0, wb = e1[i] * inv1;
            store_weight<T>(w0, i * kWarp, wa);
            store_weight<T>(w0, K + i * kWarp, wb);
            const f32x2 wa2 = pack2(wa, wa), wb2 = pack2(wb, wb);
  #pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 v = lds128(vb + ja[i] + 4u * d);
              acca[d / 2] = ffma2(wa2, v.x, acca[d / 2]);
              acca[d / 2 + 1] = ffma2(wa2, v.y, acca[d / 2 + 1]);
              accb[d / 2] = ffma2(wb2, v.x, accb[d / 2]);
              accb[d / 2 + 1] = ffma2(wb2, v.y, accb[d / 2 + 1]);
            }
          }
          finish(acca, gv0, inv0 > 0.f, obase);
          finish(accb, gv1, inv1 > 0.f, obase + HD);
        };

        const uint32_t hmagic = hg > 1 ? (uint32_t)(0xFFFFFFFFu / (uint32_t)hg + 1u) : 0u;  // ceil(2^32/hg)
        if (kPairs && all_pairs) {
          for (int pr = warp; pr < (nq >> 1) * hg; pr += kAttnWarps) {
            const int qp = hg > 1 ? (int)__umulhi((uint32_t)pr, hmagic) : pr;
            joint(2 * qp, pr - qp * hg);
          }
          if (nq & 1)
            for (int hl = warp; hl < hg; hl += kAttnWarps) single(nq - 1, hl);
        } else {
          for (int pr = warp; pr < nq * hg; pr += kAttnWarps) {
            const int q = hg > 1 ? (int)__umulhi((uint32_t)pr, hmagic) : pr;
            single(q, pr - q * hg);
          }
        }
      } else {
        // ---- fast path: 128 slots, staged K/V, 32-bit shared addresses, no slot guards;
        // the warps share the tile's (query, head) pairs evenly
        const uint32_t rowb = (uint32_t)DP * 4u;
        const uint32_t hmagic = hg > 1 ? (uint32_t)(0xFFFFFFFFu / (uint32_t)hg + 1u) : 0u;  // ceil(2^32/hg)
        for (int pr = warp; pr < nq * hg; pr += kAttnWarps) {
          const int q = hg > 1 ? (int)__umulhi((uint32_t)pr, hmagic) : pr;
          const int hl = pr - q * hg, h = h0 + hl;
          const int a = a0 + q;
          const int64_t arow = (int64_t)b * A + a;
          // the value-gate logits of this (query, head), fetched early
          float gv[DMAX / DW];
  #pragma unroll
          for (int part = 0; part < DMAX; part += DW) {
            const int d = part + (lane & (DW - 1));
            gv[part / DW] = lane < DW && d < D ? g.G[arow * HD + h * D + d] : 0.f;
          }
          int jr[kSlotsPerLane];
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) jr[i] = plan[q * K + i * kWarp + lane];
          const uint32_t kb = (uint32_t)__cvta_generic_to_shared(ks) + (uint32_t)(hl * span - klo) * rowb;
          const uint32_t vb = (uint32_t)__cvta_generic_to_shared(vs) + (uint32_t)(hl * span - klo) * rowb;
          const uint32_t qa = (uint32_t)__cvta_generic_to_shared(qs) + (uint32_t)(q * HD + h * D) * 4u;
          f32x2 q2[DMAX / 2];
          if (fullD) {
  #pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 x = lds128(qa + 4u * d);
              q2[d / 2] = x.x;
              q2[d / 2 + 1] = x.y;
            }
          } else {
  #pragma unroll
            for (int d = 0; d < DMAX; d += 2)
              q2[d / 2] = pack2(d < D ? lds32(qa + 4u * d) : 0.f, d + 1 < D ? lds32(qa + 4u * d + 4u) : 0.f);
          }
          const uint32_t ba = AF3 ? (uint32_t)__cvta_generic_to_shared(beta) +
                                        (uint32_t)(h * slots + q * K + lane) * 4u
                                  : 0u;
          float ev[kSlotsPerLane];
          uint32_t ja[kSlotsPerLane];
          float mx = -INFINITY;
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            ja[i] = (uint32_t)(jr[i] >= 0 ? jr[i] : klo) * rowb;
            f32x2 s0 = 0ull, s1 = 0ull;
  #pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 k = lds128(kb + ja[i] + 4u * d);
              s0 = ffma2(q2[d / 2], k.x, s0);
              s1 = ffma2(q2[d / 2 + 1], k.y, s1);
            }
            const float2 x = unpack2(s0), y = unpack2(s1);
            float l = ((x.x + x.y) + (y.x + y.y)) * g.scale_log2;
            if (AF3) l = fmaf(lds32(ba + 128u * i), 1.4426950408889634f, l);
            ev[i] = jr[i] >= 0 ? l : -INFINITY;
            mx = fmaxf(mx, ev[i]);
          }
          mx = warp_max(mx);
          float sum = 0.f;
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            ev[i] = jr[i] >= 0 ? exp2_approx(ev[i] - mx) : 0.f;
            sum += ev[i];
          }
          sum = warp_sum(sum);
          float inv = 0.f;
          if (sum > 0.f) asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(sum));
          T *wout = (T *)g.attention + (((int64_t)b * H + h) * A + a) * K + lane;
          f32x2 acc2[DMAX / 2];
  #pragma unroll
          for (int d = 0; d < DMAX / 2; ++d) acc2[d] = 0ull;
  #pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            const float wgt = ev[i] * inv;
            store_weight<T>(wout, i * kWarp, wgt);
            const f32x2 w2 = pack2(wgt, wgt);
  #pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 v = lds128(vb + ja[i] + 4u * d);
              acc2[d / 2] = ffma2(w2, v.x, acc2[d / 2]);
              acc2[d / 2 + 1] = ffma2(w2, v.y, acc2[d / 2 + 1]);
            }
          }
          const bool has = sum > 0.f;
          float acc[DMAX];
  #pragma unroll
          for (int d = 0; d < DMAX; d += 2) {
            const float2 p2 = unpack2(acc2[d / 2]);
            acc[d] = p2.x;
            acc[d + 1] = p2.y;
          }
  #pragma unroll
          for (int part = 0; part < DMAX; part += DW) {
            float v[DW];
  #pragma unroll
            for (int i = 0; i < DW; ++i) v[i] = acc[part + i];
            const float o = reduce_scatter<DW>(v, lane);
            const int d = part + (lane & (DW - 1));
            if (lane < DW && d < D)
              g.O[arow * HD + h * D + d] = has ? o * sigmoid_fast(gv[part / DW]) : 0.f;
          }
        }
      }
    } else {
      for (int q = warp; q < nq; q += kAttnWarps) {
        const int a = a0 + q;
        const int64_t arow = (int64_t)b * A + a;
        int jr[kSlotsPerLane];
        if (!MULTI) {
#pragma unroll
          for (int i = 0; i < kSlotsPerLane; ++i) {
            const int k = i * kWarp + lane;
            jr[i] = k < K ? plan[q * K + k] : -1;
          }
        }
        for (int hl = 0; hl < hg; ++hl) {
          const int h = h0 + hl;
          const float *qv = qs + q * HD + h * D;
          const float *kbase = staged ? ks + (hl * span - klo) * DP : nullptr;
          const float *vbase = staged ? vs + (hl * span - klo) * DP : nullptr;
          const float *bh = AF3 ? beta + h * slots + q * K : nullptr;
          // the query, packed once per (query, head), zero beyond D
          f32x2 q2[DMAX / 2];
          if (fullD) {
#pragma unroll
            for (int d = 0; d < DMAX; d += 4) {
              const ulonglong2 x = *reinterpret_cast<const ulonglong2 *>(qv + d);
              q2[d / 2] = x.x;
              q2[d / 2 + 1] = x.y;
            }
          } else {
#pragma unroll
            for (int d = 0; d < DMAX; d += 2)
              q2[d / 2] = pack2(d < D ? qv[d] : 0.f, d + 1 < D ? qv[d + 1] : 0.f);
          }

          // logit of slot k (key j, clamped to a readable row when the slot is not
          // permitted; the caller masks that value) in log2 units
          auto logit = [&](int k, int j) -> float {
            const float dot = staged ? dot_q2<DMAX>(q2, kbase + j * DP)
                                     : dot_q2_global<DMAX>(q2, g.Kf + ((int64_t)b * A + j) * HD + h * D, D);
            float l = dot * g.scale_log2;
            if (AF3) l = fmaf(bh[k], 1.4426950408889634f, l);
            return l;
          };
          const int jsafe = staged ? klo : 0;

          float mx = -INFINITY, sum = 0.f;
          float ev[kSlotsPerLane];
          if (!MULTI) {
#pragma unroll
            for (int i = 0; i < kSlotsPerLane; ++i) {
              const int k = i * kWarp + lane;
              const float l = logit(k < K ? k : 0, jr[i] >= 0 ? jr[i] : jsafe);
              ev[i] = jr[i] >= 0 ? l : -INFINITY;
              mx = fmaxf(mx, ev[i]);
            }
            mx = warp_max(mx);
#pragma unroll
            for (int i = 0; i < kSlotsPerLane; ++i) {
              ev[i] = jr[i] >= 0 ? exp2_approx(ev[i] - mx) : 0.f;
              sum += ev[i];
            }
            sum = warp_sum(sum);
          } else {
            for (int c = 0; c < nchunks; ++c) {
              float cmx = -INFINITY;
#pragma unroll
              for (int i = 0; i < kSlotsPerLane; ++i) {
                const int k = c * kChunk + i * kWarp + lane;
                jr[i] = k < K ? plan[q * K + k] : -1;
                ev[i] = jr[i] >= 0 ? logit(k, jr[i]) : -INFINITY;
                cmx = fmaxf(cmx, ev[i]);
              }
              cmx = warp_max(cmx);
              if (cmx > -INFINITY) {
                const float nm = fmaxf(mx, cmx);
                float cs = 0.f;
#pragma unroll
                for (int i = 0; i < kSlotsPerLane; ++i)
                  if (jr[i] >= 0) cs += exp2_approx(ev[i] - nm);
                sum = sum * exp2_approx(mx - nm) + warp_sum(cs);
                mx = nm;
              }
            }
          }
          float inv = 0.f;
          if (sum > 0.f) asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(sum));

          f32x2 acc2[DMAX / 2];
#pragma unroll
          for (int d = 0; d < DMAX / 2; ++d) acc2[d] = 0ull;
          T *arow_out = (T *)g.attention + (((int64_t)b * H + h) * A + a) * K;
          for (int c = 0; c < nchunks; ++c) {
#pragma unroll
            for (int i = 0; i < kSlotsPerLane; ++i) {
              const int k = c * kChunk + i * kWarp + lane;
              if (MULTI) {
                jr[i] = k < K ? plan[q * K + k] : -1;
                ev[i] = jr[i] >= 0 ? exp2_approx(logit(k, jr[i]) - mx) : 0.f;
              }
              const int j = jr[i] >= 0 ? jr[i] : jsafe;   // weight 0 on a readable row
              const float wgt = ev[i] * inv;
              if (k < K) store_weight<T>(arow_out, k, wgt);
              if (sum > 0.f) {
                if (staged) {
                  const float *vr = vbase + j * DP;
                  const f32x2 w2 = pack2(wgt, wgt);
#pragma unroll
                  for (int d = 0; d < DMAX; d += 4) {
                    const ulonglong2 v = *reinterpret_cast<const ulonglong2 *>(vr + d);
                    acc2[d / 2] = ffma2(w2, v.x, acc2[d / 2]);
                    acc2[d / 2 + 1] = ffma2(w2, v.y, acc2[d / 2 + 1]);
                  }
                } else {
                  const float *vr =
                      staged ? vbase + j * DP : g.Vf + ((int64_t)b * A + j) * HD + h * D;
#pragma unroll
                  for (int d = 0; d < DMAX; d += 2) {
                    const float v0 = d < D ? vr[d] : 0.f, v1 = d + 1 < D ? vr[d + 1] : 0.f;
                    acc2[d / 2] = ffma2(pack2(wgt, wgt), pack2(v0, v1), acc2[d / 2]);
                  }
                }
              }
            }
          }

          // fold the lanes' partial outputs: lane l ends with channel l (and l + 32)
          const bool has = sum > 0.f;
          float acc[DMAX];
#pragma unroll
          for (int d = 0; d < DMAX; d += 2) {
            const float2 p = unpack2(acc2[d / 2]);
            acc[d] = p.x;
            acc[d + 1] = p.y;
          }
#pragma unroll
          for (int part = 0; part < DMAX; part += DW) {
            float v[DW];
#pragma unroll
            for (int i = 0; i < DW; ++i) v[i] = acc[part + i];
            const float o = reduce_scatter<DW>(v, lane);
            const int d = part + (lane & (DW - 1));
            if (lane < DW && d < D) {
              const int64_t oi = arow * HD + h * D + d;
              g.O[oi] = has ? o * sigmoid_fast(g.G[oi]) : 0.f;
            }
          }
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace atomenc
