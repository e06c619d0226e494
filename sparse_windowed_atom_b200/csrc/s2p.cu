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
//                zero unless tokens i and j are present (bullet 1).
//   k_s2p_pairs_tc  the same pass with the readout on the tensor cores, for 2H and D
//                multiples of 32 up to 128 and 256: one CTA per (b, i, 128 pairs j); each
//                thread forms its pair's features (written out, and into the bf16 MMA
//                operand as hi + lo parts), tcgen05.mma multiplies them by the out_weight
//                image (bf16 hi [+ lo] blocks, built once per call by k_s2p_pack) into TMEM,
//                and each thread reads its pair's row back for the bias, the output
//                LayerNorm and the store. Products: hi·hi + lo·hi (+ hi·lo for float32
//                weights), float32 accumulation. The pass is bound by writing the two
//                [B,N,N,*] tensors.
#include <cmath>
#include <cstring>

#include "../../include/atomenc.h"
#include "common.cuh"
#include "umma.cuh"

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
constexpr int kQKRows = 4, kQKThreads = kQKRows * 32;

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


// ---------------------------------------------------------------- tensor-core readout
constexpr int kTcRows = 128;                 // pairs per CTA (TMEM lanes)

// four consecutive values in the storage type (16-byte float32 / 8-byte bf16 store)
__device__ __forceinline__ void st4(float *p, const float (&v)[4]) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st4(__nv_bfloat16 *p, const float (&v)[4]) {
  *reinterpret_cast<uint2 *>(p) = make_uint2(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]));
}
constexpr uint32_t kTcBlk = 128 * 64 * 2;    // one bf16 [128 x 64] swizzled block
constexpr int kTcMaxH2 = 128, kTcMaxDp = 256;

// out_weight [2H, D] (x @ W) -> image: for output tile t (128 columns) and k chunk c (64),
// a [128 n x 64 k] bf16 block, hi then (float32 weights) lo
template <typename T>
__global__ void k_s2p_pack(const T *w, int H2, int Dp, uint8_t *img, int parts) {
  const int nt = (Dp + 127) / 128, kc = (H2 + 63) / 64;
  const int64_t total = (int64_t)nt * 128 * kc * 8;     // 16-byte chunks of one part
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(i % (nt * 128)), k0 = (int)(i / (nt * 128)) * 8;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = (n < Dp && k0 + e < H2) ? ldf(w, (int64_t)(k0 + e) * Dp + n) : 0.f;
    uint32_t hi[4], lo[4];
    umma::split8<true>(v, hi, lo);
    const int t = n / 128, c = k0 / 64;
    uint8_t *blk = img + ((size_t)t * kc + c) * parts * kTcBlk;
    const uint32_t off = umma::swz_offset(n % 128, k0 % 64, 128);
    *reinterpret_cast<uint4 *>(blk + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    if (parts == 2) *reinterpret_cast<uint4 *>(blk + kTcBlk + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

struct PairTcArgs {
  int64_t N;
  int H, H2, Dp;
  float eps;
  int onorm, bparts, vec_pf, vec_out;
  const uint8_t *mask;
  const float *qk;
  const uint8_t *img;                    // out_weight image, bparts parts per block
  const void *ob, *osc, *obi;
  void *pf, *out;
};

template <typename T>
__global__ void __launch_bounds__(kTcRows) k_s2p_pairs_tc(PairTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const int H = a.H, H2 = a.H2, Dp = a.Dp;
  const int kc = (H2 + 63) / 64, nt = (Dp + 127) / 128;
  uint8_t *sA = sm;                                   // [kc][2] blocks: hi, lo
  uint8_t *sB = sA + (size_t)kc * 2 * kTcBlk;         // [nt][kc][bparts] blocks
  float *sk = reinterpret_cast<float *>(sB + (size_t)nt * kc * a.bparts * kTcBlk);   // k_i [H]
  float *sbias = sk + kTcMaxH2;                       // out_bias, output_scale, output_bias [Dp]
  float *ssc = sbias + kTcMaxDp, *sbi = ssc + kTcMaxDp;
  float *sT = sbi + kTcMaxDp;                         // [4 warps][32 rows][32 floats]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sT + 4 * 32 * 32);   // [0] image, [1] MMAs
  uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 2);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float *tile = sT + warp * 32 * 32;
  const int64_t bi = blockIdx.y, b = bi / a.N;
  const int64_t j = (int64_t)blockIdx.x * kTcRows + tid;   // this thread's pair (i, j)
  const bool live = j < a.N;
  const bool mi = a.mask[bi] != 0;
  const bool use = live && mi && a.mask[b * a.N + j] != 0;
  const uint32_t img_bytes = (uint32_t)((size_t)nt * kc * a.bparts * kTcBlk);
  // 32 columns of this warp's 32 pairs (each thread holds its own pair's) through the
  // warp's shared tile (16-byte chunk q of row r at q ^ (r & 7): conflict-free both ways),
  // stored with 8 lanes per row segment into rows (b, i, j) of a [B, N, N, ld] tensor at
  // column c0 (ncol of the 32 are real). Warp-collective.
  auto store_rows = [&](const float (&v)[32], T *dst, int64_t ld, int c0, int ncol, bool vec) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *reinterpret_cast<float4 *>(tile + lane * 32 + 4 * (q ^ (lane & 7))) =
          make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rl = i * 4 + (lane >> 3), q = lane & 7;
      const int64_t jr = (int64_t)blockIdx.x * kTcRows + warp * 32 + rl;
      if (jr < a.N && 4 * q < ncol) {
        const float4 t4 = *reinterpret_cast<const float4 *>(tile + rl * 32 + 4 * (q ^ (rl & 7)));
        const float o[4] = {t4.x, t4.y, t4.z, t4.w};
        T *d = dst + (bi * a.N + jr) * ld + c0 + 4 * q;
        if (vec && 4 * q + 4 <= ncol) {
          st4(d, o);
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (4 * q + u < ncol) stf(d, u, o[u]);
        }
      }
    }
    __syncwarp();
  };

  if (tid == 0) {
    umma::mbar_init(bar, 1);
    umma::mbar_init(bar + 1, 1);
    umma::fence_mbar_init();
  }
  if (warp == 0) umma::tmem_alloc(tslot, Dp <= 128 ? 128 : 256);
  for (int h = tid; h < H; h += kTcRows) sk[h] = a.qk[bi * H2 + H + h];
  for (int e = tid; e < Dp; e += kTcRows) {
    sbias[e] = ldf((const T *)a.ob, e);
    ssc[e] = a.onorm ? ldf((const T *)a.osc, e) : 1.f;
    sbi[e] = a.onorm ? ldf((const T *)a.obi, e) : 0.f;
  }
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tslot;
  if (tid == 0) {
    umma::mbar_arrive_expect_tx(bar, img_bytes);
    umma::bulk_g2s(sB, a.img, img_bytes, bar);
  }

  // ---- the pair's features, 32 at a time: into the MMA operand (row tid) and out
  const float *qj = a.qk + (b * a.N + (live ? j : 0)) * H2;
  for (int hc = 0; hc < kc * 64; hc += 32) {
    float f[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int h = hc + e;
      float v = 0.f;
      if (use && h < H) v = sk[h] * qj[h];
      else if (use && h < H2) v = qj[h - H] - sk[h - H];
      f[e] = v;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f8[e] = f[8 * u + e];
      uint32_t hi[4], lo[4];
      umma::split8<true>(f8, hi, lo);
      const int h0 = hc + 8 * u;
      uint8_t *blk = sA + (size_t)(h0 / 64) * 2 * kTcBlk;
      const uint32_t off = umma::swz_offset(tid, h0 % 64, kTcRows);
      *reinterpret_cast<uint4 *>(blk + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4 *>(blk + kTcBlk + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (hc < H2) store_rows(f, static_cast<T *>(a.pf), H2, hc, min(32, H2 - hc), a.vec_pf != 0);
  }
  umma::fence_async_smem();
  __syncthreads();

  // ---- readout products into TMEM columns [128 t, 128 t + 128)
  bool ok = true;
  if (tid == 0) {
    ok = umma::mbar_wait(bar, 0);
    umma::tc_fence_after();
    constexpr uint32_t idesc = umma::idesc_bf16(128, 128);
    for (int t = 0; t < nt && ok; ++t) {
      for (int c = 0; c < kc; ++c) {
        const uint32_t a0 = umma::smem_u32(sA + (size_t)c * 2 * kTcBlk);
        const uint32_t b0 = umma::smem_u32(sB + ((size_t)t * kc + c) * a.bparts * kTcBlk);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t dah = umma::sw128_desc(a0 + kk * 32), dal = umma::sw128_desc(a0 + kTcBlk + kk * 32);
          const uint64_t dbh = umma::sw128_desc(b0 + kk * 32);
          umma::mma_bf16(tmem + t * 128, dah, dbh, idesc, (c | kk) != 0);
          umma::mma_bf16(tmem + t * 128, dal, dbh, idesc, 1);
          if (a.bparts == 2)
            umma::mma_bf16(tmem + t * 128, dah, umma::sw128_desc(b0 + kTcBlk + kk * 32), idesc, 1);
        }
      }
    }
    umma::mma_commit(bar + 1);
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;    // warp 0's view; the others wait below
  __syncwarp();
  {
    int done = 1;
    if (lane == 0) done = umma::mbar_wait(bar + 1, 0) ? 1 : 0;
    done = __shfl_sync(0xffffffffu, done, 0);
    ok = ok && done != 0;
  }
  __syncthreads();
  umma::tc_fence_after();

  // ---- epilogue: thread tid owns TMEM lane tid (warp w reads lanes 32w..32w+31)
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  float mean = 0.f, rstd = 1.f;
  if (a.onorm) {
    // statistics over the row (+ bias), shifted by its first value
    float s1 = 0.f, s2 = 0.f, sh = 0.f;
    for (int c0 = 0; c0 < Dp; c0 += 32) {
      float v[32];
      umma::tmem_ld32(trow + c0, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float x = v[e] + sbias[c0 + e];
        if (c0 == 0 && e == 0) sh = x;
        const float d = x - sh;
        s1 += d;
        s2 = fmaf(d, d, s2);
      }
    }
    const float m = s1 / (float)Dp;
    mean = sh + m;
    rstd = 1.f / sqrtf(fmaxf(s2 / (float)Dp - m * m, 0.f) + a.eps);
  }
  for (int c0 = 0; c0 < Dp; c0 += 32) {
    float v[32];
    umma::tmem_ld32(trow + c0, v);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float x = v[e] + sbias[c0 + e];
      if (a.onorm) x = fmaf((x - mean) * rstd, ssc[c0 + e], sbi[c0 + e]);
      v[e] = !ok ? __int_as_float(0x7fc00000) : (use ? x : 0.f);
    }
    store_rows(v, static_cast<T *>(a.out), Dp, c0, min(32, Dp - c0), a.vec_out != 0);
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, Dp <= 128 ? 128 : 256);
}

size_t tc_smem_bytes(int H2, int Dp, int bparts) {
  const size_t kc = (size_t)(H2 + 63) / 64, nt = (size_t)(Dp + 127) / 128;
  return 1024 + kc * 2 * kTcBlk + nt * kc * bparts * kTcBlk +
         (size_t)(kTcMaxH2 + 3 * kTcMaxDp + 4 * 32 * 32) * 4 + 64;
}
size_t tc_image_bytes(int H2, int Dp, int bparts) {
  return (size_t)((Dp + 127) / 128) * ((H2 + 63) / 64) * bparts * kTcBlk;
}
bool tc_shape(int64_t H2, int64_t Dp) {
  return H2 % 32 == 0 && H2 <= kTcMaxH2 && Dp % 32 == 0 && Dp <= kTcMaxDp;
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

// q/k rows [B*N, 2H] float32, then (tensor-core readout) the out_weight image
size_t qk_bytes(const Dims &d) { return ((size_t)(d.B * d.N * d.H2) * 4 + 255) / 256 * 256; }
size_t workspace_bytes(const Dims &d) {
  size_t b = qk_bytes(d);
  if (tc_shape(d.H2, d.Dp)) b += tc_image_bytes((int)d.H2, (int)d.Dp, d.fdt == ATOMENC_F32 ? 2 : 1);
  return b;
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
  if (tc_shape(d.H2, d.Dp)) {
    const int bparts = d.fdt == ATOMENC_F32 ? 2 : 1;
    uint8_t *img = reinterpret_cast<uint8_t *>(qk) + qk_bytes(d);
    k_s2p_pack<T><<<64, 256, 0, st>>>(static_cast<const T *>(p->out_weight.data), (int)d.H2, (int)d.Dp, img, bparts);
    const size_t es = sizeof(T);
    PairTcArgs ta;
    ta.N = d.N; ta.H = (int)(d.H2 / 2); ta.H2 = (int)d.H2; ta.Dp = (int)d.Dp; ta.eps = eps;
    ta.onorm = onorm ? 1 : 0; ta.bparts = bparts;
    ta.vec_pf = (reinterpret_cast<uintptr_t>(out->pair_features.data) & (4 * es - 1)) == 0;
    ta.vec_out = (reinterpret_cast<uintptr_t>(out->output.data) & (4 * es - 1)) == 0;
    ta.mask = static_cast<const uint8_t *>(in->mask.data);
    ta.qk = qk;
    ta.img = img;
    ta.ob = p->out_bias.data;
    ta.osc = onorm ? p->output_scale.data : nullptr;
    ta.obi = onorm ? p->output_bias.data : nullptr;
    ta.pf = out->pair_features.data;
    ta.out = out->output.data;
    const size_t tsmem = tc_smem_bytes((int)d.H2, (int)d.Dp, bparts);
    if (cudaFuncSetAttribute(k_s2p_pairs_tc<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsmem) !=
        cudaSuccess)
      return ATOMENC_ERR_CUDA;
    k_s2p_pairs_tc<T><<<dim3((unsigned)((d.N + kTcRows - 1) / kTcRows), (unsigned)(d.B * d.N)), kTcRows, tsmem, st>>>(ta);
    return cudaGetLastError() == cudaSuccess ? ATOMENC_OK : ATOMENC_ERR_CUDA;
  }
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
