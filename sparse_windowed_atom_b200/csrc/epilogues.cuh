// epilogues.cuh -- per-element epilogues of the projection GEMMs. Each functor ends one
// step of the block; the GEMM hands it four consecutive columns of one output row.
#pragma once

#include "common.cuh"

namespace atomenc {

// Per-element epilogues get the four consecutive columns of one thread through this.
template <class E>
struct Quad {
  E e;
  __device__ void quad(int64_t r, int64_t c0, const float (&v)[4], int64_t N) const {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (c0 + j < N) e(r, c0 + j, v[j]);
  }
};

// ---- epilogues (each a small functor; names say which step of the block they end)

template <typename IT>
struct EpiStoreT {  // plain store in the intermediate type
  IT *out;
  int64_t ld;
  __device__ void operator()(int64_t r, int64_t c, float v) const { stf(out, r * ld + c, v); }
};
using EpiStore = EpiStoreT<float>;

// four consecutive values in the intermediate type (16-byte float32 / 8-byte bf16)
__device__ __forceinline__ void st4i(float *d, float4 o) { *reinterpret_cast<float4 *>(d) = o; }
__device__ __forceinline__ void st4i(__nv_bfloat16 *d, float4 o) {
  *reinterpret_cast<uint2 *>(d) = make_uint2(bf16x2_bits(o.x, o.y), bf16x2_bits(o.z, o.w));
}

// eight consecutive values in the intermediate type (two 16-byte float32 stores / one
// 16-byte bf16 store); the caller checks 16-byte alignment
__device__ __forceinline__ void st8i(float *d, const float (&v)[8]) {
  *reinterpret_cast<float4 *>(d) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4 *>(d + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void st8i(__nv_bfloat16 *d, const float (&v)[8]) {
  *reinterpret_cast<uint4 *>(d) = make_uint4(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]),
                                             bf16x2_bits(v[4], v[5]), bf16x2_bits(v[6], v[7]));
}
template <typename T>
__device__ __forceinline__ bool aligned16(const T *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Plain store of four consecutive columns (one 16-byte / 8-byte store when the row
// stride and the column keep them aligned); oct: eight columns, one 16-byte bf16 store.
template <typename IT>
struct QuadStore {
  static constexpr bool kOct = true;   // takes eight columns per lane
  IT *out;
  int64_t ld;
  __device__ void quad(int64_t r, int64_t c0, const float (&v)[4], int64_t N) const {
    if (c0 + 4 <= N && ((ld | c0) & 3) == 0) {
      st4i(out + r * ld + c0, make_float4(v[0], v[1], v[2], v[3]));
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (c0 + j < N) stf(out, r * ld + c0 + j, v[j]);
    }
  }
  __device__ void oct(int64_t r, int64_t c0, const float (&v)[8], int64_t N) const {
    if (c0 + 8 <= N && ((ld | c0) & 7) == 0 && aligned16(out)) {
      st8i(out + r * ld + c0, v);
    } else {
      quad(r, c0, {v[0], v[1], v[2], v[3]}, N);
      if (c0 + 4 < N) quad(r, c0 + 4, {v[4], v[5], v[6], v[7]}, N);   // quads store unchecked
    }
  }
};

// ReLU(hidden @ w_pool) before the per-token mean (bullet 19), four columns at a time
template <typename IT>
struct QuadRelu {
  static constexpr bool kOct = true;   // takes eight columns per lane
  IT *out;
  int64_t ld;
  __device__ void quad(int64_t r, int64_t c0, const float (&v)[4], int64_t N) const {
    const float4 o = make_float4(fmaxf(v[0], 0.f), fmaxf(v[1], 0.f), fmaxf(v[2], 0.f), fmaxf(v[3], 0.f));
    if (c0 + 4 <= N && ((ld | c0) & 3) == 0) {
      st4i(out + r * ld + c0, o);
    } else {
      const float w[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (c0 + j < N) stf(out, r * ld + c0 + j, w[j]);
    }
  }
  __device__ void oct(int64_t r, int64_t c0, const float (&v)[8], int64_t N) const {
    if (c0 + 8 <= N && ((ld | c0) & 7) == 0 && aligned16(out)) {
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = fmaxf(v[e], 0.f);
      st8i(out + r * ld + c0, o);
    } else {
      quad(r, c0, {v[0], v[1], v[2], v[3]}, N);
      if (c0 + 4 < N) quad(r, c0 + 4, {v[4], v[5], v[6], v[7]}, N);   // quads store unchecked
    }
  }
};

// AF3 conditioning: columns (scale_0, shift_0, scale_1, shift_1, scale_2, shift_2), C each;
// scale columns become sigmoid(c_j @ w_scale[j] + b_scale[j])  (bullet 7)
// Index math is done once per four columns, in 32 bits (C is a multiple of 4).
template <typename IT>
struct EpiCondAF3 {
  static constexpr bool kOct = true;   // takes eight columns per lane
  IT *out;     // [M, 6C]
  const float *b_scale;  // [3, C]
  int64_t C;
  __device__ void quad(int64_t r, int64_t c0, const float (&v)[4], int64_t N) const {
    const int c = (int)c0, Ci = (int)C;
    if (Ci & 3) {  // a quad may straddle two blocks
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ce = c + e;
        if (ce >= N) break;
        const int be = ce / Ci, he = ce - be * Ci;
        stf(out, r * 6 * C + ce, (be & 1) ? v[e] : sigmoid_fast(v[e] + b_scale[(be >> 1) * Ci + he]));
      }
      return;
    }
    // blk = c / C without a division (six blocks)
    const int blk = (c >= Ci) + (c >= 2 * Ci) + (c >= 3 * Ci) + (c >= 4 * Ci) + (c >= 5 * Ci);
    const int ch = c - blk * Ci;
    float4 o = make_float4(v[0], v[1], v[2], v[3]);
    if ((blk & 1) == 0) {  // scale block j = blk / 2
      const float *bs = b_scale + (blk >> 1) * Ci + ch;
      o.x = sigmoid_fast(v[0] + bs[0]);
      o.y = sigmoid_fast(v[1] + bs[1]);
      o.z = sigmoid_fast(v[2] + bs[2]);
      o.w = sigmoid_fast(v[3] + bs[3]);
    }
    st4i(out + r * 6 * C + c0, o);
  }
  // eight columns of one block when C is a multiple of 8 (one 16-byte bf16 store)
  __device__ void oct(int64_t r, int64_t c0, const float (&v)[8], int64_t N) const {
    const int c = (int)c0, Ci = (int)C;
    if ((Ci & 7) == 0 && c0 + 8 <= N && aligned16(out)) {
      const int blk = (c >= Ci) + (c >= 2 * Ci) + (c >= 3 * Ci) + (c >= 4 * Ci) + (c >= 5 * Ci);
      const int ch = c - blk * Ci;
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = v[e];
      if ((blk & 1) == 0) {
        const float *bs = b_scale + (blk >> 1) * Ci + ch;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = sigmoid_fast(v[e] + bs[e]);
      }
      st8i(out + r * 6 * C + c0, o);
    } else {
      quad(r, c0, {v[0], v[1], v[2], v[3]}, N);
      if (c0 + 4 < N) quad(r, c0 + 4, {v[4], v[5], v[6], v[7]}, N);   // quads store unchecked
    }
  }
};

// AF3 residual gates sigmoid(raw condition @ w_residual_gate[j] + b_residual_gate[j])  (bullet 9)
template <typename IT>
struct EpiGateAF3 {
  static constexpr bool kOct = true;   // takes eight columns per lane
  IT *out;     // [M, 2C]
  const float *b_rg;  // [2, C]
  int64_t C;
  __device__ void quad(int64_t r, int64_t c0, const float (&v)[4], int64_t N) const {
    const float *b = b_rg + c0;
    if (C & 1) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c0 + e < N) stf(out, r * 2 * C + c0 + e, sigmoid_fast(v[e] + b[e]));
      return;
    }
    st4i(out + r * 2 * C + c0,
         make_float4(sigmoid_fast(v[0] + b[0]), sigmoid_fast(v[1] + b[1]), sigmoid_fast(v[2] + b[2]),
                     sigmoid_fast(v[3] + b[3])));
  }
  __device__ void oct(int64_t r, int64_t c0, const float (&v)[8], int64_t N) const {
    if ((C & 3) == 0 && c0 + 8 <= N && aligned16(out)) {
      const float *b = b_rg + c0;
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = sigmoid_fast(v[e] + b[e]);
      st8i(out + r * 2 * C + c0, o);
    } else {
      quad(r, c0, {v[0], v[1], v[2], v[3]}, N);
      if (c0 + 4 < N) quad(r, c0 + 4, {v[4], v[5], v[6], v[7]}, N);   // quads store unchecked
    }
  }
};

// four consecutive values of a [rows, HD] intermediate in its workspace type
__device__ __forceinline__ void st4w(float *d, const float (&o)[4]) {
  *reinterpret_cast<float4 *>(d) = make_float4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ void st4w(__nv_bfloat16 *d, const float (&o)[4]) {
  *reinterpret_cast<uint2 *>(d) = make_uint2(bf16x2_bits(o[0], o[1]), bf16x2_bits(o[2], o[3]));
}

// Q/K/V/value-gate projections: the N columns are `nparts` blocks of HD written to
// separate [M, HD] buffers of type WT (float32, or bf16 for bf16 workloads whose
// attention reads bf16 rows); only Q takes a bias (AF3 b_q, bullet 8)
template <typename WT>
struct EpiSplitT {
  static constexpr bool kOct = true;   // takes eight columns per lane
  WT *dst[4];
  const float *bias[4];
  int64_t HD;
  __device__ void quad(int64_t r, int64_t c0, const float (&v)[4], int64_t N) const {
    // part = c / HD without a division (at most four parts)
    const int HDi = (int)HD, c = (int)c0;
    const int part = (c >= HDi) + (c >= 2 * HDi) + (c >= 3 * HDi), ch = c - part * HDi;
    float o[4] = {v[0], v[1], v[2], v[3]};
    // selects, not an indexed read: an indexed read of the functor's arrays would copy
    // the functor to local memory
    auto bias_of = [&](int p) { return p == 0 ? bias[0] : p == 1 ? bias[1] : p == 2 ? bias[2] : bias[3]; };
    auto dst_of = [&](int p) { return p == 0 ? dst[0] : p == 1 ? dst[1] : p == 2 ? dst[2] : dst[3]; };
    if ((HDi & 3) == 0) {
      const float *b = bias_of(part);
      if (b) {
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] += b[ch + e];
      }
      st4w(dst_of(part) + r * HD + ch, o);
    } else {  // a quad may straddle two parts when HD is not a multiple of 4
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ce = c + e;
        if (ce >= N) break;
        const int pe = (ce >= HDi) + (ce >= 2 * HDi) + (ce >= 3 * HDi), he = ce - pe * HDi;
        const float *b = bias_of(pe);
        stf(dst_of(pe), r * HD + he, b ? v[e] + b[he] : v[e]);
      }
    }
  }
  // eight columns: one part when HD is a multiple of 8 (one 16-byte bf16 store)
  __device__ void oct(int64_t r, int64_t c0, const float (&v)[8], int64_t N) const {
    const int HDi = (int)HD, c = (int)c0;
    const int part = (c >= HDi) + (c >= 2 * HDi) + (c >= 3 * HDi), ch = c - part * HDi;
    WT *d = part == 0 ? dst[0] : part == 1 ? dst[1] : part == 2 ? dst[2] : dst[3];
    const float *b = part == 0 ? bias[0] : part == 1 ? bias[1] : part == 2 ? bias[2] : bias[3];
    if ((HDi & 7) == 0 && c0 + 8 <= N && aligned16(d)) {
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = b ? v[e] + b[ch + e] : v[e];
      st8i(d + r * HD + ch, o);
    } else {
      quad(r, c0, {v[0], v[1], v[2], v[3]}, N);
      if (c0 + 4 < N) quad(r, c0 + 4, {v[4], v[5], v[6], v[7]}, N);   // quads store unchecked
    }
  }
};
using EpiSplit = EpiSplitT<float>;

// x' = x + g_attn * (o @ w_attention_out)  (bullet 16); x and the gates in the
// intermediate type, x' in float32
template <typename IT>
struct EpiResidual {
  const IT *x;
  const IT *gate;  // gate[r * gate_ld + gate_off + c]
  int64_t gate_ld, gate_off, C;
  float *out;
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    out[r * C + c] = ldf(x, r * C + c) + ldf(gate, r * gate_ld + gate_off + c) * v;
  }
};

// SwiGLU with gate/up interleaved column-wise: h[m] = SiLU(z @ w_ff_gate)[m] * (z @ w_ff_up)[m]
// (bullet 17). Column 2m holds the gate, 2m+1 the up projection; a thread's four columns
// start at an even column, so both halves of a pair are in its hands.
struct EpiSwiGLU {
  float *h;  // [M, Mh]
  int64_t Mh;
  __device__ void quad(int64_t r, int64_t c0, const float (&v)[4], int64_t N) const {
#pragma unroll
    for (int p = 0; p < 2; ++p)
      if (c0 + 2 * p + 1 < N) h[r * Mh + c0 / 2 + p] = silu_fast(v[2 * p]) * v[2 * p + 1];
  }
};

// hidden = usable * (x' + g_trans * ((...) @ w_ff_out))  (bullet 18); the gates in the
// storage type T of the output
template <typename T>
struct EpiHidden {
  const float *xp;
  const T *gate;
  int64_t gate_ld, gate_off, C;
  const uint8_t *usable;
  T *hid;        // output
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    const float h = usable[r] ? xp[r * C + c] + ldf(gate, r * gate_ld + gate_off + c) * v : 0.f;
    stf(hid, r * C + c, h);
  }
};

// ReLU(hidden @ w_pool) before the per-token mean (bullet 19), in the intermediate type
template <typename IT>
struct EpiRelu {
  IT *out;
  int64_t ld;
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    stf(out, r * ld + c, v > 0.f ? v : 0.f);
  }
};

}  // namespace atomenc
