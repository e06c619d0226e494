// gemm_simt.cuh -- CUDA-core float32 GEMM with fused epilogues: out = epi(A @ W).
// A [M, K] (float32 or the storage type), W [K, N] float32, both row-major.
// 64x64 tile, 16-deep k step, 256 threads, 4x4 outputs per thread.
#pragma once

#include "common.cuh"

namespace atomenc {

constexpr int kGemmBM = 64, kGemmBN = 64, kGemmBK = 16, kGemmThreads = 256;

template <typename TA, class Epi>
__global__ void __launch_bounds__(kGemmThreads)
    k_gemm_simt(const TA *__restrict__ A, int64_t lda, const float *__restrict__ W,
                int64_t ldw, int64_t M, int64_t N, int64_t K, Epi epi) {
  __shared__ __align__(16) float As[kGemmBK][kGemmBM + 4];
  __shared__ __align__(16) float Ws[kGemmBK][kGemmBN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.y * kGemmBM, n0 = (int64_t)blockIdx.x * kGemmBN;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += kGemmBK) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + e * kGemmThreads;
      const int m = idx >> 4, k = idx & 15;
      const int64_t gm = m0 + m, gk = k0 + k;
      As[k][m] = (gm < M && gk < K) ? ldf(A, gm * lda + gk) : 0.f;
      const int kk = idx >> 6, n = idx & 63;
      const int64_t wk = k0 + kk, wn = n0 + n;
      Ws[kk][n] = (wk < K && wn < N) ? W[wk * ldw + wn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kGemmBK; ++k) {
      const float4 a = *reinterpret_cast<const float4 *>(&As[k][ty * 4]);
      const float4 w = *reinterpret_cast<const float4 *>(&Ws[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = m0 + ty * 4 + i;
    if (row < M && n0 + tx * 4 < N) epi.quad(row, n0 + tx * 4, acc[i], N);
  }
}

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

struct EpiStore {  // plain float32 store
  float *out;
  int64_t ld;
  __device__ void operator()(int64_t r, int64_t c, float v) const { out[r * ld + c] = v; }
};

// AF3 conditioning: columns (scale_0, shift_0, scale_1, shift_1, scale_2, shift_2), C each;
// scale columns become sigmoid(c_j @ w_scale[j] + b_scale[j])  (bullet 7)
struct EpiCondAF3 {
  float *out;  // [M, 6C]
  const float *b_scale;  // [3, C]
  int64_t C;
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    const int64_t j = c / (2 * C), part = (c / C) & 1, ch = c % C;
    out[r * 6 * C + c] = part == 0 ? sigmoidf_(v + b_scale[j * C + ch]) : v;
  }
};

// AF3 residual gates sigmoid(raw condition @ w_residual_gate[j] + b_residual_gate[j])  (bullet 9)
struct EpiGateAF3 {
  float *out;  // [M, 2C]
  const float *b_rg;  // [2, C]
  int64_t C;
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    out[r * 2 * C + c] = sigmoidf_(v + b_rg[c]);
  }
};

// Q/K/V/value-gate projections: the N columns are `nparts` blocks of HD written to
// separate [M, HD] buffers; only Q takes a bias (AF3 b_q, bullet 8)
struct EpiSplit {
  float *dst[4];
  const float *bias[4];
  int64_t HD;
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    const int64_t part = c / HD, ch = c % HD;
    if (bias[part]) v += bias[part][ch];
    dst[part][r * HD + ch] = v;
  }
};

// x' = x + g_attn * (o @ w_attention_out)  (bullet 16)
struct EpiResidual {
  const float *x;
  const float *gate;  // gate[r * gate_ld + gate_off + c]
  int64_t gate_ld, gate_off, C;
  float *out;
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    out[r * C + c] = x[r * C + c] + gate[r * gate_ld + gate_off + c] * v;
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
      if (c0 + 2 * p + 1 < N) h[r * Mh + c0 / 2 + p] = siluf_(v[2 * p]) * v[2 * p + 1];
  }
};

// hidden = usable * (x' + g_trans * ((...) @ w_ff_out))  (bullet 18)
template <typename T>
struct EpiHidden {
  const float *xp;
  const float *gate;
  int64_t gate_ld, gate_off, C;
  const uint8_t *usable;
  float *hid32;  // float32 copy for pooling / readout
  T *hid;        // output
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    const float h = usable[r] ? xp[r * C + c] + gate[r * gate_ld + gate_off + c] * v : 0.f;
    hid32[r * C + c] = h;
    stf(hid, r * C + c, h);
  }
};

// ReLU(hidden @ w_pool) before the per-token mean (bullet 19)
struct EpiRelu {
  float *out;
  int64_t ld;
  __device__ void operator()(int64_t r, int64_t c, float v) const {
    out[r * ld + c] = v > 0.f ? v : 0.f;
  }
};

}  // namespace atomenc
