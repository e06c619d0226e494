// attn_rows.cuh -- slot-gathered windowed attention, one warp per query over all heads.
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
// Layout and work split (H*D = HD in {64, 128}, D a multiple of HD / 8, K <= 128):
//  * Persistent CTAs (512 threads, one per SM): CTA c walks a contiguous range of query
//    tiles (QT consecutive queries of one batch element each), in order.
//  * Per tile, warp w builds, for each of its queries, the compacted list of permitted
//    slots (key id, slot index) with ballots, and the tile's key span [klo, khi]; AF3:
//    the pair bias of every listed slot for every head (LayerNorm over P in one shifted
//    pass, folded pair_scale * w_pair) into a float32 table in list order. The first
//    tile's lists are built before the wait for the projections (the inputs and the
//    usable flags come from kernels at least two places earlier).
//  * The K and V rows live in a shared ring of R rows: key j sits in row j mod R. A tile
//    copies in only the rows of its span that the previous tile's span did not hold
//    (consecutive tiles of a batch element share most of their span), together with its
//    own Q and value-gate rows. Rows are whole (all heads, storage type), each 16-byte
//    chunk placed so that the eight lanes of a quarter-warp read one 128-byte segment
//    of a row per load: lane i of every quarter-warp owns channels [HD/8 i, HD/8 (i+1))
//    of the row (the same head for HD/8 / D of the lanes), so a gathered row never
//    meets a bank conflict.
//  * A warp takes one query: quarter-warp g takes list entries g, g + 4, ...; lane i
//    forms the partial dot product of its channels, the lanes of a head combine theirs
//    with xor-shuffles; logits stay in registers (log2 units), max and sum across the
//    quarter-warps by shuffles, one exp2 per entry; weights go to a per-warp shared row
//    buffer (zeros for slots that are not permitted) that is written out with 16-byte
//    coalesced stores; the weighted value sum per lane, folded across the four
//    quarter-warps by a reduce-scatter, is gated by sigmoid(value gate) and stored.
// A span too wide for the shared stage is read from global memory (L2) instead with the
// same lane mapping and sets status bit 1; the results are the same.
#pragma once

#include <climits>
#include <type_traits>

#include "common.cuh"

namespace atomenc {

constexpr int kRowAttnThreads = 512;
constexpr int kRowAttnWarps = kRowAttnThreads / kWarp;
constexpr int kRowAttnKMax = 128;                  // slots per query (list entries <= K)
constexpr int kRowAttnIters = kRowAttnKMax / 4;     // list entries per quarter-warp
constexpr int kRowAttnPairMax = 32;
constexpr int kRowAttnHeadsMax = 8;
constexpr int kRowAttnF32MaxAtoms = 1024;   // float32 storage: problems up to this many atoms

struct RowAttnArgs {
  int B, A, K, H, D, P;
  int radius;                     // -1 = no index window
  float scale_log2;               // log2(e) / sqrt(D)
  float eps;
  int QT;                         // queries per tile
  int tiles_per_b;                // ceil(A / QT)
  int ntiles;                     // B * tiles_per_b
  int stage_rows;                 // R: rows of K (and of V) the shared ring holds
  int qg_staged;                  // the tile's Q and value-gate rows are copied to shared memory
  const void *Q, *Kf, *Vf, *G;    // [B*A, HD] storage type
  const int64_t *key_index;       // [B, A, K]
  const uint8_t *window;          // [B, A, K]
  const uint8_t *usable;          // [B*A]
  const void *pair;               // [B, A, K, P] AF3
  const float *w_pair;            // [P, H] = pair_scale[p] * w_pair[p, h]
  void *attention;                // [B, H, A, K]
  void *O;                        // [B*A, HD] gated attention output, storage type
  unsigned *status;
  int pair_vec;                   // pair rows may be read with 16-byte loads (P = 16, aligned)
  int att_vec;                    // weight rows may be written with 16-byte stores (aligned)
};

// bytes of one per-warp weight row (K weights, 16-byte multiple, + 16 to spread banks)
__host__ __device__ inline int rowattn_wrow_bytes(int K, int es) {
  return ((K * es + 15) & ~15) + 16;
}
// shared bytes before the K/V ring: list keys, list slots, counts, (AF3) bias table,
// per-warp weight rows, the tile's Q and value-gate rows; each region 128-byte aligned
__host__ __device__ inline size_t rowattn_fixed_smem(int QT, int K, int H, int es, bool af3, bool qg) {
  auto r128 = [](size_t n) { return (n + 127) & ~size_t(127); };
  size_t b = r128((size_t)QT * K * 4) + r128((size_t)QT * K) + r128((size_t)QT * 4);
  if (af3) b += r128((size_t)QT * K * H * 4);
  b += r128((size_t)kRowAttnWarps * H * rowattn_wrow_bytes(K, es));
  if (qg) b += 2 * (size_t)QT * 128 * es;   // the tile's Q and value-gate rows (H*D = 128)
  return b;
}

namespace rowattn {

// 16 bytes of a row -> floats (CH = 8 bf16 or 4 float32)
__device__ __forceinline__ void unpack(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void unpack(const uint4 v, float (&f)[4]) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T>
__device__ __forceinline__ void store_w(T *p, float w);
template <>
__device__ __forceinline__ void store_w<float>(float *p, float w) { *p = w; }
template <>
__device__ __forceinline__ void store_w<__nv_bfloat16>(__nv_bfloat16 *p, float w) {
  const uint32_t u = __float_as_uint(w);
  *reinterpret_cast<uint16_t *>(p) = (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// N consecutive channels of one row as floats, and the gated output store
template <int N>
__device__ __forceinline__ void ldn(const float *p, float (&v)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int c = 0; c < N; c += 4) {
      const float4 x = *reinterpret_cast<const float4 *>(p + c);
      v[c] = x.x; v[c + 1] = x.y; v[c + 2] = x.z; v[c + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < N; c += 2) {
      const float2 x = *reinterpret_cast<const float2 *>(p + c);
      v[c] = x.x; v[c + 1] = x.y;
    }
  }
}
template <int N>
__device__ __forceinline__ void ldn(const __nv_bfloat16 *p, float (&v)[N]) {
  static_assert(N % 2 == 0, "pairs");
  if constexpr (N >= 8) {
#pragma unroll
    for (int c = 0; c < N; c += 8) {
      float f[8];
      unpack(*reinterpret_cast<const uint4 *>(p + c), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[c + e] = f[e];
    }
  } else {
#pragma unroll
    for (int c = 0; c < N; c += 2) {
      const uint32_t u = *reinterpret_cast<const uint32_t *>(p + c);
      v[c] = __uint_as_float(u << 16);
      v[c + 1] = __uint_as_float(u & 0xFFFF0000u);
    }
  }
}
template <int N>
__device__ __forceinline__ void stn(float *p, const float (&v)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int c = 0; c < N; c += 4) *reinterpret_cast<float4 *>(p + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < N; c += 2) *reinterpret_cast<float2 *>(p + c) = make_float2(v[c], v[c + 1]);
  }
}
template <int N>
__device__ __forceinline__ void stn(__nv_bfloat16 *p, const float (&v)[N]) {
  uint32_t u[N / 2];
#pragma unroll
  for (int c = 0; c < N; c += 2) {
    const uint32_t a = __float_as_uint(v[c]), b = __float_as_uint(v[c + 1]);
    const uint32_t ha = (a + 0x7FFFu + ((a >> 16) & 1u)) >> 16;
    const uint32_t hb = (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
    u[c / 2] = ha | (hb << 16);
  }
  if constexpr (N == 4) {
    *reinterpret_cast<uint2 *>(p) = make_uint2(u[0], u[1]);
  } else if constexpr (N == 2) {
    *reinterpret_cast<uint32_t *>(p) = u[0];
  } else {
#pragma unroll
    for (int c = 0; c < N / 2; c += 4) *reinterpret_cast<uint4 *>(p + 2 * c) = make_uint4(u[c], u[c + 1], u[c + 2], u[c + 3]);
  }
}

// 16 pair channels of one slot by 16-byte loads (bf16: 2 loads, float32: 4 loads)
__device__ __forceinline__ void ldpair16(const __nv_bfloat16 *pr, float (&x)[16]) {
  float a[8], b[8];
  unpack(*reinterpret_cast<const uint4 *>(pr), a);
  unpack(*reinterpret_cast<const uint4 *>(pr + 8), b);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    x[e] = a[e];
    x[8 + e] = b[e];
  }
}
__device__ __forceinline__ void ldpair16(const float *pr, float (&x)[16]) { ldn<16>(pr, x); }

// Pair bias of one slot for heads 0..H-1 from its 16 pair channels x (in registers):
// one shifted pass for the LayerNorm statistics, then the folded head sums
template <int H>
__device__ __forceinline__ void pair_bias16(float (&x)[16], float eps, const float *wp,
                                            const float *wsum, float *out) {
  const float x0 = x[0];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    x[p] -= x0;
    s1 += x[p];
    s2 = fmaf(x[p], x[p], s2);
  }
  const float m = s1 * (1.f / 16.f);
  const float rstd = rsqrtf(fmaxf(s2 * (1.f / 16.f) - m * m, 0.f) + eps);
#pragma unroll
  for (int h = 0; h < H; ++h) {
    float d = 0.f;
#pragma unroll
    for (int p = 0; p < 16; ++p) d = fmaf(x[p], wp[p * H + h], d);
    out[h] = rstd * (d - m * wsum[h]);
  }
}

// Pair bias of one slot for heads 0..H-1 (H <= 8):
//   beta_h = sum_p LN(pair)_p * pair_scale_p * w_pair[p, h]
//          = rstd * (sum_p y_p W'[p, h] - m * sum_p W'[p, h]),
// y_p = pair_p - pair_0 (a shift that keeps the one-pass variance well conditioned),
// m = mean(y), rstd = 1 / sqrt(mean(y^2) - m^2 + eps); W' = pair_scale * w_pair ([P][H]
// in shared memory) and its column sums wsum.
template <typename T, int H>
__device__ __forceinline__ void pair_bias(const T *pr, int P, bool vec16, float eps,
                                          const float *wp, const float *wsum, float *out) {
  if (vec16) {
    float x[16];
    ldpair16(pr, x);
    const float x0 = x[0];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      x[p] -= x0;
      s1 += x[p];
      s2 = fmaf(x[p], x[p], s2);
    }
    const float m = s1 * (1.f / 16.f);
    const float rstd = rsqrtf(fmaxf(s2 * (1.f / 16.f) - m * m, 0.f) + eps);
#pragma unroll
    for (int h = 0; h < H; ++h) {
      float d = 0.f;
#pragma unroll
      for (int p = 0; p < 16; ++p) d = fmaf(x[p], wp[p * H + h], d);
      out[h] = rstd * (d - m * wsum[h]);
    }
    return;
  }
  // any P <= 32: statistics first, then the head sums with the channels read again
  const float x0 = ldf(pr, 0);
  float s1 = 0.f, s2 = 0.f;
  for (int p = 0; p < P; ++p) {
    const float y = ldf(pr, p) - x0;
    s1 += y;
    s2 = fmaf(y, y, s2);
  }
  const float m = s1 / (float)P;
  const float rstd = rsqrtf(fmaxf(s2 / (float)P - m * m, 0.f) + eps);
  float d[H];
#pragma unroll
  for (int h = 0; h < H; ++h) d[h] = 0.f;
  for (int p = 0; p < P; ++p) {
    const float y = ldf(pr, p) - x0;
#pragma unroll
    for (int h = 0; h < H; ++h) d[h] = fmaf(y, wp[p * H + h], d[h]);
  }
#pragma unroll
  for (int h = 0; h < H; ++h) out[h] = rstd * (d[h] - m * wsum[h]);
}

}  // namespace rowattn

template <typename T, int HD, int DH, bool AF3>
__global__ void __launch_bounds__(kRowAttnThreads, 1) k_attn_rows(RowAttnArgs g) {
  pdl_launch_next();
  constexpr int ES = sizeof(T);
  constexpr int LC = HD / 8;            // channels per lane; a quarter-warp covers a row
  constexpr int CH = 16 / ES;           // channels per 16-byte chunk
  constexpr int NSEG = LC / CH;         // 16-byte chunks per lane = 128-byte segments per row
  constexpr int RB = HD * ES;           // bytes per staged row
  constexpr int LPH = DH / LC;          // lanes of a quarter-warp per head
  constexpr int H = HD / DH;
  constexpr int OC = LC / 4;            // output channels per lane after the fold
  static_assert(LC % CH == 0 && DH % LC == 0 && H <= kRowAttnHeadsMax, "row attention shape");
  constexpr int NIT = kRowAttnIters;

  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  __shared__ int s_lo, s_hi;
  __shared__ __align__(16) float s_wp[AF3 ? kRowAttnPairMax * kRowAttnHeadsMax : 4];
  __shared__ __align__(16) float s_wsum[AF3 ? kRowAttnHeadsMax : 4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g4 = lane >> 3, li = lane & 7;            // quarter-warp, lane in it
  const int QT = g.QT, K = g.K, A = g.A, P = g.P, R = g.stage_rows;

  auto r128 = [](size_t n) { return (n + 127) & ~size_t(127); };
  uint8_t *cur = smem_dyn;
  int *ckey = reinterpret_cast<int *>(cur);           cur += r128((size_t)QT * K * 4);
  uint8_t *cks = cur;                                  cur += r128((size_t)QT * K);
  int *cnt = reinterpret_cast<int *>(cur);            cur += r128((size_t)QT * 4);
  float *beta = reinterpret_cast<float *>(cur);       if (AF3) cur += r128((size_t)QT * K * H * 4);
  const int WB = rowattn_wrow_bytes(K, ES);
  uint8_t *wbuf_all = cur;                             cur += r128((size_t)kRowAttnWarps * H * WB);
  const bool qg_st = g.qg_staged != 0;
  uint8_t *sQ = cur;                                   if (qg_st) cur += (size_t)QT * RB;
  uint8_t *sG = cur;                                   if (qg_st) cur += (size_t)QT * RB;
  uint8_t *kstage = cur;
  uint8_t *vstage = cur + (size_t)R * RB;

  if (tid == 0) {
    s_lo = INT_MAX;
    s_hi = -1;
  }
  if (AF3) {
    for (int i = tid; i < P * H; i += kRowAttnThreads) s_wp[i] = g.w_pair[i];
    for (int h = tid; h < H; h += kRowAttnThreads) {
      float sw = 0.f;
      for (int p = 0; p < P; ++p) sw += g.w_pair[p * H + h];
      s_wsum[h] = sw;
    }
  }
  __syncthreads();

  // per-thread constants of the query phase
  const T *Qg = static_cast<const T *>(g.Q);
  const T *Gg = static_cast<const T *>(g.G);
  T *Og = static_cast<T *>(g.O);
  T *Wg = static_cast<T *>(g.attention);
  const uint8_t *Kg = static_cast<const uint8_t *>(g.Kf);
  const uint8_t *Vg = static_cast<const uint8_t *>(g.Vf);
  uint8_t *wbuf = wbuf_all + (size_t)warp * H * WB;
  const int hd_lane = (li * LC) / DH;                 // this lane's head
  const bool head_writer = (li % LPH) == 0;
  T *wrow = reinterpret_cast<T *>(wbuf + hd_lane * WB);
  const uint32_t kbase = (uint32_t)__cvta_generic_to_shared(kstage) + (uint32_t)li * 16u;
  const uint32_t vbase = (uint32_t)__cvta_generic_to_shared(vstage) + (uint32_t)li * 16u;
  const int oc0 = li * LC + OC * g4;                  // first output channel of this lane
  // the per-warp weight rows are zeroed and written out in 16-byte chunks: lane l takes
  // chunk l % cpr of rows l / cpr, l / cpr + 32 / cpr, ... (a row has cpr <= 32 chunks)
  const int cpr = (K * ES + 15) / 16;
  const int rpp = 32 / cpr, wr_row = lane / cpr, wr_chunk = lane - wr_row * cpr;
  const bool vecw = ((K * ES) & 15) == 0 && g.att_vec;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr int CPR = RB / 16;                        // 16-byte chunks per row (a power of two)

  // the ring holds the rows [ring_lo, ring_hi] of batch element ring_b (uniform over the CTA)
  int ring_b = -1, ring_lo = 0, ring_hi = -1;
  const int t_begin = (int)((int64_t)blockIdx.x * g.ntiles / gridDim.x);
  const int t_end = (int)((int64_t)(blockIdx.x + 1) * g.ntiles / gridDim.x);
  for (int tile = t_begin; tile < t_end; ++tile) {
  const int b = tile / g.tiles_per_b, a0 = (tile - b * g.tiles_per_b) * QT;
  const int nq = min(QT, A - a0);

  // ---------------- list of permitted slots per query
  const int64_t rbase = (int64_t)b * A;
  int lo = INT_MAX, hi = -1;
  for (int q = warp; q < QT; q += kRowAttnWarps) {
    const int a = a0 + q;
    const bool uq = q < nq && g.usable[rbase + a] != 0;
    const int64_t sb = (rbase + a) * K;
    int64_t kid[4];
    uint8_t win[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int k = r * 32 + lane;
      const bool in = uq && k < K;
      kid[r] = in ? g.key_index[sb + k] : -1;
      win[r] = in ? g.window[sb + k] : 0;
    }
    bool ok[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t j = kid[r];
      bool o = win[r] != 0 && j >= 0 && j < A;
      if (o && g.radius >= 0) o = (j > a ? j - a : a - j) <= g.radius;
      ok[r] = o;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
      if (ok[r]) ok[r] = g.usable[rbase + kid[r]] != 0;
    int base = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const unsigned bal = __ballot_sync(0xffffffffu, ok[r]);
      if (ok[r]) {
        const int pos = base + __popc(bal & ((1u << lane) - 1u));
        ckey[q * K + pos] = (int)kid[r];
        cks[q * K + pos] = (uint8_t)(r * 32 + lane);
        lo = min(lo, (int)kid[r]);
        hi = max(hi, (int)kid[r]);
      }
      base += __popc(bal);
    }
    if (lane == 0) cnt[q] = base;
    if (AF3) {
      // pair bias of every listed slot for every head, in list order
      __syncwarp();
      const T *prow = static_cast<const T *>(g.pair) + sb * P;
      if constexpr (ES == 2) {
        if (g.pair_vec) {
          // 16 bf16 channels a slot: the rows of all of this lane's slots (at most 4) are
          // loaded before any is used
          uint4 raw[4][2];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = lane + 32 * u;
            if (e < base) {
              const uint4 *pr = reinterpret_cast<const uint4 *>(prow + (int64_t)cks[q * K + e] * P);
              raw[u][0] = pr[0];
              raw[u][1] = pr[1];
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = lane + 32 * u;
            if (e < base) {
              float x[16], lo8[8], hi8[8];
              rowattn::unpack(raw[u][0], lo8);
              rowattn::unpack(raw[u][1], hi8);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                x[c] = lo8[c];
                x[8 + c] = hi8[c];
              }
              rowattn::pair_bias16<H>(x, g.eps, s_wp, s_wsum, beta + ((size_t)q * K + e) * H);
            }
          }
          continue;
        }
      }
      for (int e = lane; e < base; e += 32)
        rowattn::pair_bias<T, H>(prow + (int64_t)cks[q * K + e] * P, P, g.pair_vec != 0, g.eps,
                                 s_wp, s_wsum, beta + ((size_t)q * K + e) * H);
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0 && lo <= hi) {
    atomicMin(&s_lo, lo);
    atomicMax(&s_hi, hi);
  }

  // ---------------- the ring: rows of the span the ring does not hold yet, and the
  // tile's Q and value-gate rows (the first tile waits for the projections here)
  if (tile == t_begin) pdl_wait();
  __syncthreads();
  const int klo = s_lo, khi = s_hi;
  const int span = khi >= klo ? khi - klo + 1 : 0;
  const bool staged = span > 0 && span <= R;
  if (span > 0 && !staged && tid == 0) atomicOr(g.status, 1u);
  {
    const uint32_t ks = (uint32_t)__cvta_generic_to_shared(kstage);
    const uint32_t vs = (uint32_t)__cvta_generic_to_shared(vstage);
    if (staged) {
      // key j lives in ring row j mod R = (j - klo + ph) mod R
      const int ph = klo % R;
      // rows to copy: [klo, khi] less what the ring holds (one or two intervals)
      int l0 = klo, l1 = khi, m0 = 1, m1 = 0;
      if (ring_b == b) {
        const int i0 = max(klo, ring_lo), i1 = min(khi, ring_hi);
        if (i0 <= i1) {
          l1 = i0 - 1;
          m0 = i1 + 1;
          m1 = khi;
        }
      }
      const int n1 = max(l1 - l0 + 1, 0), n2 = max(m1 - m0 + 1, 0);
      const int total = (n1 + n2) * CPR;
      for (int i = tid; i < total; i += kRowAttnThreads) {
        const int rr = i / CPR, c = i - rr * CPR;
        const int j = rr < n1 ? l0 + rr : m0 + (rr - n1);
        int pr = j - klo + ph;
        pr -= pr >= R ? R : 0;
        // logical 16-byte chunk c of a row goes to position (c % NSEG) * 8 + c / NSEG
        const int p = (c % NSEG) * 8 + c / NSEG;
        const size_t src = (size_t)(rbase + j) * RB + (size_t)c * 16;
        const uint32_t dst = (uint32_t)(pr * RB + p * 16);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ks + dst), "l"(Kg + src) : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(vs + dst), "l"(Vg + src) : "memory");
      }
      ring_b = b;
      ring_lo = klo;
      ring_hi = khi;
      // list entries name ring rows from here on
      for (int q = warp; q < nq; q += kRowAttnWarps) {
        const int n = cnt[q];
        for (int e = lane; e < n; e += 32) {
          int pr = ckey[q * K + e] - klo + ph;
          pr -= pr >= R ? R : 0;
          ckey[q * K + e] = pr;
        }
      }
    }
    // the tile's Q and value-gate rows (contiguous in global memory), when they fit
    const uint32_t qs = (uint32_t)__cvta_generic_to_shared(sQ);
    const uint32_t gs = (uint32_t)__cvta_generic_to_shared(sG);
    const uint8_t *Qb = reinterpret_cast<const uint8_t *>(Qg) + (size_t)(rbase + a0) * RB;
    const uint8_t *Gb = reinterpret_cast<const uint8_t *>(Gg) + (size_t)(rbase + a0) * RB;
    for (int i = tid; qg_st && i < nq * CPR; i += kRowAttnThreads) {
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(qs + 16u * i), "l"(Qb + 16 * (size_t)i) : "memory");
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(gs + 16u * i), "l"(Gb + 16 * (size_t)i) : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  }
  __syncthreads();

  // ---------------- while this tile computes: bring the next tile's inputs into L2 (its
  // slot rows and AF3 pair rows, the Q and value-gate rows, and the rows its key span
  // most likely adds, the QT after the ring's last), so that its lists and copies find
  // them there
  if (tile + 1 < t_end) {
    const int nb = (tile + 1) / g.tiles_per_b, na0 = (tile + 1 - nb * g.tiles_per_b) * QT;
    const int nnq = min(QT, A - na0);
    const int64_t nrow = (int64_t)nb * A + na0;
    const char *kb = reinterpret_cast<const char *>(g.key_index + nrow * K);
    const char *wbp = reinterpret_cast<const char *>(g.window + nrow * K);
    const int64_t kbytes = (int64_t)nnq * K * 8, wbytes = (int64_t)nnq * K, qbytes = (int64_t)nnq * RB;
    const int nk = (int)((kbytes + 127) >> 7), nw = (int)((wbytes + 127) >> 7), nqr = (int)((qbytes + 127) >> 7);
    int s0 = 0, ns = 0;
    if (ring_b == nb && ring_lo <= ring_hi) {
      s0 = ring_hi + 1;
      ns = max(0, min(QT, A - s0));
    }
    const int nkv = (int)(((int64_t)ns * RB + 127) >> 7);
    const int np = AF3 ? (int)(((int64_t)nnq * K * P * ES + 127) >> 7) : 0;
    const char *pb = AF3 ? static_cast<const char *>(g.pair) + nrow * K * P * ES : nullptr;
    const int total = nk + nw + 2 * nqr + 2 * nkv + np;
    for (int i = tid; i < total; i += kRowAttnThreads) {
      const char *ptr;
      int j = i;
      if (j < nk) ptr = kb + ((int64_t)j << 7);
      else if ((j -= nk) < nw) ptr = wbp + ((int64_t)j << 7);
      else if ((j -= nw) < nqr) ptr = reinterpret_cast<const char *>(Qg) + nrow * RB + ((int64_t)j << 7);
      else if ((j -= nqr) < nqr) ptr = reinterpret_cast<const char *>(Gg) + nrow * RB + ((int64_t)j << 7);
      else if ((j -= nqr) < nkv) ptr = reinterpret_cast<const char *>(Kg) + ((int64_t)nb * A + s0) * RB + ((int64_t)j << 7);
      else if ((j -= nkv) < nkv) ptr = reinterpret_cast<const char *>(Vg) + ((int64_t)nb * A + s0) * RB + ((int64_t)j << 7);
      else ptr = pb + ((int64_t)(j - nkv) << 7);
      asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    }
  }

  // One query: NIT list iterations at most (4 entries each), the K/V rows staged in
  // shared memory or read from global memory.
  auto run_query = [&](auto nit_c, auto staged_c, int q) {
    constexpr int NI = decltype(nit_c)::value;
    constexpr bool ST = decltype(staged_c)::value;
    const int a = a0 + q;
    const int64_t arow = rbase + a;
    const int n = cnt[q];
    const int niter = (n + 3) >> 2;
    const int *ck = ckey + q * K;
    const uint8_t *cs = cks + q * K;
    // the query's channels of this lane (bf16 pairs, or float32 pairs) and the value-gate
    // logits of its output channels
    uint32_t qb[LC / 2];
    f32x2 qf[LC / 2];
    const T *qrow = qg_st ? reinterpret_cast<const T *>(sQ + (size_t)q * RB) : Qg + arow * HD;
    const T *grow = qg_st ? reinterpret_cast<const T *>(sG + (size_t)q * RB) : Gg + arow * HD;
    if constexpr (ES == 2) {
#pragma unroll
      for (int c = 0; c < LC; c += 8) {
        const uint4 v = *reinterpret_cast<const uint4 *>(qrow + li * LC + c);
        qb[c / 2] = v.x; qb[c / 2 + 1] = v.y; qb[c / 2 + 2] = v.z; qb[c / 2 + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < LC; c += 4) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2 *>(qrow + li * LC + c);
        qf[c / 2] = v.x;
        qf[c / 2 + 1] = v.y;
      }
    }
    float gv[OC];
    rowattn::ldn<OC>(grow + oc0, gv);
    // zero this warp's weight rows
    if (wr_row < rpp)
      for (int h = wr_row; h < H; h += rpp)
        *reinterpret_cast<uint4 *>(wbuf + h * WB + wr_chunk * 16) = make_uint4(0u, 0u, 0u, 0u);

    // the row of list entry e (a readable row with weight 0 past the list's end): a ring
    // row when staged, a key id otherwise
    auto row_of = [&](int e) -> int { return e < n ? ck[e] : ck[0]; };
    // 16-byte chunk s of the K or V row j for this lane
    auto chunk = [&](uint32_t sbase, const uint8_t *gbase, int j, int s) -> uint4 {
      if constexpr (ST)
        return rowattn::lds128(sbase + (uint32_t)(j * RB + s * 128));
      else
        return *reinterpret_cast<const uint4 *>(gbase + (size_t)(rbase + j) * RB + (size_t)(NSEG * li + s) * 16);
    };

    // ---- logits of the listed slots (log2 units)
    // (the loops over list iterations leave at the query's own count: no predicated
    // iterations past it)
    float lt[NI];
    float mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < NI; ++t) lt[t] = -INFINITY;
#pragma unroll
    for (int t = 0; t < NI; ++t) {
      if (t >= niter) break;
      {
        const int e = 4 * t + g4;
        const int j = row_of(e);
        float part;
        if constexpr (ES == 2) {
          float p0 = 0.f, p1 = 0.f;
#pragma unroll
          for (int s = 0; s < NSEG; ++s) {
            const uint4 raw = chunk(kbase, Kg, j, s);
            p0 = fma_bf16x2(qb[4 * s], raw.x, p0);
            p1 = fma_bf16x2(qb[4 * s + 1], raw.y, p1);
            p0 = fma_bf16x2(qb[4 * s + 2], raw.z, p0);
            p1 = fma_bf16x2(qb[4 * s + 3], raw.w, p1);
          }
          part = p0 + p1;
        } else {
          f32x2 s0 = 0ull, s1 = 0ull;
#pragma unroll
          for (int s = 0; s < NSEG; ++s) {
            const uint4 raw = chunk(kbase, Kg, j, s);
            s0 = ffma2(qf[2 * s], ((f32x2)raw.y << 32) | raw.x, s0);
            s1 = ffma2(qf[2 * s + 1], ((f32x2)raw.w << 32) | raw.z, s1);
          }
          const float2 x = unpack2(s0), y = unpack2(s1);
          part = (x.x + x.y) + (y.x + y.y);
        }
#pragma unroll
        for (int w = 1; w < LPH; w <<= 1) part += __shfl_xor_sync(0xffffffffu, part, w);
        float l = part * g.scale_log2;
        if (AF3 && e < n) l = fmaf(beta[((size_t)q * K + e) * H + hd_lane], kLog2e, l);
        lt[t] = e < n ? l : -INFINITY;
        mx = fmaxf(mx, lt[t]);
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    float sum = 0.f;
#pragma unroll
    for (int t = 0; t < NI; ++t) {
      if (t >= niter) break;
      lt[t] = lt[t] > -INFINITY ? rowattn::ex2(lt[t] - mx) : 0.f;
      sum += lt[t];
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 8);
    sum += __shfl_xor_sync(0xffffffffu, sum, 16);
    float inv = 0.f;
    if (sum > 0.f) asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(sum));
    __syncwarp();

    // ---- weights out (per-warp rows), weighted values
    float acc[LC];
    f32x2 acc2[LC / 2];
#pragma unroll
    for (int c = 0; c < LC; ++c) acc[c] = 0.f;
#pragma unroll
    for (int c = 0; c < LC / 2; ++c) acc2[c] = 0ull;
#pragma unroll
    for (int t = 0; t < NI; ++t) {
      if (t >= niter) break;
      {
        const int e = 4 * t + g4;
        const float w = lt[t] * inv;
        const int j = row_of(e);
        if constexpr (ES == 2) {
          // the weight rounded to bf16 once: the stored weight and the one that scales V
          const uint16_t wb = __bfloat16_as_ushort(__float2bfloat16_rn(w));
          if (e < n && head_writer) *reinterpret_cast<uint16_t *>(wrow + cs[e]) = wb;
#pragma unroll
          for (int s = 0; s < NSEG; ++s) {
            const uint4 raw = chunk(vbase, Vg, j, s);
            axpy_bf16x2(wb, raw.x, acc[8 * s], acc[8 * s + 1]);
            axpy_bf16x2(wb, raw.y, acc[8 * s + 2], acc[8 * s + 3]);
            axpy_bf16x2(wb, raw.z, acc[8 * s + 4], acc[8 * s + 5]);
            axpy_bf16x2(wb, raw.w, acc[8 * s + 6], acc[8 * s + 7]);
          }
        } else {
          if (e < n && head_writer) rowattn::store_w<T>(wrow + cs[e], w);
          const f32x2 w2 = pack2(w, w);
#pragma unroll
          for (int s = 0; s < NSEG; ++s) {
            const uint4 raw = chunk(vbase, Vg, j, s);
            acc2[2 * s] = ffma2(w2, ((f32x2)raw.y << 32) | raw.x, acc2[2 * s]);
            acc2[2 * s + 1] = ffma2(w2, ((f32x2)raw.w << 32) | raw.z, acc2[2 * s + 1]);
          }
        }
      }
    }
    if constexpr (ES == 4) {
#pragma unroll
      for (int c = 0; c < LC / 2; ++c) {
        const float2 v = unpack2(acc2[c]);
        acc[2 * c] = v.x;
        acc[2 * c + 1] = v.y;
      }
    }
    // fold the four quarter-warps: lane (g4, li) ends with channels oc0 .. oc0 + OC
#pragma unroll
    for (int w = 16, h = LC / 2; w >= 8; w >>= 1, h >>= 1) {
      const bool up = (lane & w) != 0;
#pragma unroll
      for (int c = 0; c < LC / 2; ++c) {
        if (c < h) {
          const float send = up ? acc[c] : acc[c + h];
          const float keep = up ? acc[c + h] : acc[c];
          acc[c] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
      }
    }
    float ov[OC];
#pragma unroll
    for (int c = 0; c < OC; ++c) ov[c] = sum > 0.f ? acc[c] * sigmoid_fast(gv[c]) : 0.f;
    rowattn::stn<OC>(Og + arow * HD + oc0, ov);

    // ---- the query's weight rows to attention[b, h, a, :]
    __syncwarp();
    if (vecw) {
      if (wr_row < rpp)
        for (int h = wr_row; h < H; h += rpp) {
          const uint4 v = *reinterpret_cast<const uint4 *>(wbuf + h * WB + wr_chunk * 16);
          *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(Wg + (((int64_t)b * H + h) * A + a) * K) + wr_chunk * 16) = v;
        }
    } else {
      for (int h = 0; h < H; ++h)
        for (int k = lane; k < K; k += 32)
          Wg[(((int64_t)b * H + h) * A + a) * K + k] = reinterpret_cast<const T *>(wbuf + h * WB)[k];
    }
    __syncwarp();
  };

  using I8 = std::integral_constant<int, 8>;
  using I16 = std::integral_constant<int, 16>;
  using I32 = std::integral_constant<int, 32>;
  for (int q = warp; q < nq; q += kRowAttnWarps) {
    const int niter = (cnt[q] + 3) >> 2;
    if (staged) {
      if (niter <= 8) run_query(I8{}, std::true_type{}, q);
      else if (niter <= 16) run_query(I16{}, std::true_type{}, q);
      else run_query(I32{}, std::true_type{}, q);
    } else {
      run_query(I32{}, std::false_type{}, q);
    }
  }
  if (tid == 0) {
    s_lo = INT_MAX;
    s_hi = -1;
  }
  __syncthreads();
  }  // tiles
}

}  // namespace atomenc
