// transition.cuh -- one kernel for the tail of the block, per 128-row block:
//   x'     = x + g_attn * (o @ w_attention_out)                           (bullet 16)
//   z      = AF3: LN(x') * sigmoid(scale_2) + shift_2;
//            ESMFold2: RMS(x') * (1 + transition_scale) + transition_shift (bullet 17)
//   hidden = usable * (x' + g_trans * ((SiLU(z @ w_ff_gate) * (z @ w_ff_up)) @ w_ff_out))
//                                                                          (bullets 17, 18)
// (page "Local atom attention, encoder pooling and decoder skip/readout", Required
// behavior). The three products run on tcgen05 with their operands chained through
// shared memory and TMEM accumulators: out-projection (128 columns), the SwiGLU hidden
// width in 64-wide chunks (128 interleaved gate/up columns each, two TMEM buffers and two
// shared operand buffers, so the products of chunk i+1 overlap the SiLU of chunk i) and
// w_ff_out (128 columns), 512 TMEM columns in all; x', z and the SwiGLU intermediate
// never go to HBM.
//
// Warp roles: warps 0-7 convert the o rows into the first operand, then work one output
// row per thread (warp w: TMEM lanes 32 (w % 4).. and the column half w / 4 of every
// 128-column matrix): residual x' (stored back into TMEM over the out-projection
// accumulator), row statistics (the two halves combined through shared memory) and z
// (written as the next operand), SiLU(gate) * up per chunk (written as the last
// operand), and the final gated residual; warp 8 lane 0 issues the MMAs; warp 9 lane 0
// streams the packed weight
// blocks through a ring of bulk async copies in the order the MMAs consume them. Every
// wait is bounded (status bit 4 on timeout). Needs C == 128, H*D in {64, 128}, M a
// multiple of 128.
#pragma once

#include "common.cuh"
#include "gemm_umma.cuh"
#include "umma.cuh"

namespace atomenc {

constexpr int kTransEpiWarps = 8;                       // two per TMEM lane quadrant
constexpr int kTransThreads = (kTransEpiWarps + 2) * 32;   // + MMA issuer + weight loader

struct TransArgs {
  int64_t R;
  int HD, M;                   // C is 128
  const void *O;               // [R, HD] gated attention output (float32, or bf16 when
                               // the attention wrote bf16 rows)
  // x, the gates and the transition norm vectors are in the output's storage type
  const void *x;               // [R, 128] residual state start
  const void *g0, *g1;         // attention / transition residual gates (row stride g_ld)
  int64_t g_ld;
  const void *sc, *sh;         // transition norm scale / shift (row stride cond_ld)
  int64_t cond_ld;
  int rms, plus1;
  float eps;
  const uint8_t *usable;
  const uint8_t *w_out, *w_ff1, *w_ff2;   // packed tensor-core images
  void *hidden;                // [R, 128] output
  unsigned *status;
  // PAIR mode: two CTAs per row block, each on half of the SwiGLU width; w_ff_out partials
  // of the half of the columns the other CTA finishes go through global scratch
  float *xfer;                 // [row blocks][2][128][64] partial columns
  int *xflag;                  // [row blocks][2], zero at entry
  uint32_t peer_spin_limit;    // polls of the peer's flag before giving up (status bit 4)
  int withhold_flag;           // test hook: never raise this CTA's flag (the peer's wait
                               // then runs out); 0 in normal use
};

constexpr int kTransSlotsSplit = 3, kTransSlotsPlain = 6;   // weight ring depth
__host__ __device__ inline size_t trans_smem_bytes(bool split) {
  const size_t parts = split ? 2 : 1, slots = split ? kTransSlotsSplit : kTransSlotsPlain;
  return 1024 + (2 + 2 + slots) * parts * kUmmaBlockBytes + 256;
}

// eight floats of one row into an operand block pair (hi, and lo when split) at column k
template <bool SPLIT>
__device__ __forceinline__ void put8(uint8_t *blk, int r, int k, const float (&v)[8]) {
  uint32_t hi[4], lo[4];
  umma::split8<SPLIT>(v, hi, lo);
  const uint32_t off = umma::swz_offset(r, k, kUmmaBM);
  *reinterpret_cast<uint4 *>(blk + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  if (SPLIT)
    *reinterpret_cast<uint4 *>(blk + kUmmaBlockBytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

// 32 consecutive values of row r from global memory as floats (zeros when r is out of
// range): float32 rows by 16-byte loads, bf16 rows by 16-byte loads of 8 values
__device__ __forceinline__ void row32(const float *p, int64_t ld, int64_t r, bool ok, int c0,
                                      float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ok) x = *reinterpret_cast<const float4 *>(p + r * ld + c0 + i);
    v[i] = x.x;
    v[i + 1] = x.y;
    v[i + 2] = x.z;
    v[i + 3] = x.w;
  }
}
__device__ __forceinline__ void row32(const __nv_bfloat16 *p, int64_t ld, int64_t r, bool ok, int c0,
                                      float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (ok) x = *reinterpret_cast<const uint4 *>(p + r * ld + c0 + i);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[i + 2 * e] = __uint_as_float(w[e] << 16);
      v[i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
}

template <typename T>
__device__ __forceinline__ void store4(T *p, int64_t i, float4 v);
// (the output is the caller's tensor: vector stores only at aligned addresses)
template <>
__device__ __forceinline__ void store4<float>(float *p, int64_t i, float4 v) {
  if ((reinterpret_cast<uintptr_t>(p + i) & 15) == 0) {
    *reinterpret_cast<float4 *>(p + i) = v;
  } else {
    p[i] = v.x; p[i + 1] = v.y; p[i + 2] = v.z; p[i + 3] = v.w;
  }
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *p, int64_t i, float4 v) {
  const uint32_t lo = bf16x2_bits(v.x, v.y), hi = bf16x2_bits(v.z, v.w);
  if ((reinterpret_cast<uintptr_t>(p + i) & 7) == 0) {
    *reinterpret_cast<uint2 *>(p + i) = make_uint2(lo, hi);
  } else {
    const uint16_t b[4] = {(uint16_t)lo, (uint16_t)(lo >> 16), (uint16_t)hi, (uint16_t)(hi >> 16)};
#pragma unroll
    for (int e = 0; e < 4; ++e) reinterpret_cast<uint16_t *>(p)[i + e] = b[e];
  }
}

// eight consecutive values: one 16-byte store of bf16 (two of float32) where the address
// allows it, else two four-value stores
template <typename T>
__device__ __forceinline__ void store8(T *p, int64_t i, const float (&v)[8]) {
  if ((reinterpret_cast<uintptr_t>(p + i) & 15) == 0) {
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint4 *>(p + i) = make_uint4(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]),
                                                     bf16x2_bits(v[4], v[5]), bf16x2_bits(v[6], v[7]));
    } else {
      *reinterpret_cast<float4 *>(p + i) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4 *>(p + i + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
  } else {
    store4<T>(p, i, make_float4(v[0], v[1], v[2], v[3]));
    store4<T>(p, i + 4, make_float4(v[4], v[5], v[6], v[7]));
  }
}

// the CTA pair's flags (global memory, GPU scope); the pair is launched as a 2-CTA
// cluster, so both CTAs are resident together, and a poll still gives up after
// peer_spin_limit reads (default kPeerSpinLimit; status bit 4), so a missing peer cannot
// hang the kernel
constexpr uint32_t kPeerSpinLimit = 1u << 22;
__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <bool SPLIT, typename TOut, bool PAIR, typename TO = float>
__global__ void __launch_bounds__(kTransThreads, 1) k_transition(TransArgs t) {
  pdl_enter();
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  constexpr int P = SPLIT ? 2 : 1, NSLOT = SPLIT ? kTransSlotsSplit : kTransSlotsPlain, C = 128;
  constexpr uint32_t BLK = kUmmaBlockBytes;
  constexpr uint32_t idesc = umma::idesc_bf16(kUmmaBM, kUmmaBN);
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = sm;                        // [2][P]: o operand, later z
  uint8_t *sH = sA + 2 * P * BLK;          // [2][P]: SwiGLU chunk
  uint8_t *sR = sH + 2 * P * BLK;          // weight ring [NSLOT][P]
  uint64_t *full = reinterpret_cast<uint64_t *>(sR + NSLOT * P * BLK);
  uint64_t *empty = full + NSLOT, *a_ready = empty + NSLOT, *acc0_done = a_ready + 1,
           *z_ready = acc0_done + 1, *acc1_full = z_ready + 1, *h_ready = acc1_full + 2,
           *h_free = h_ready + 2, *acc2_done = h_free + 2;                 // [2] = per buffer
  uint32_t *tslot = reinterpret_cast<uint32_t *>(acc2_done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const TOut *tx = static_cast<const TOut *>(t.x);
  const TOut *tg0 = static_cast<const TOut *>(t.g0), *tg1 = static_cast<const TOut *>(t.g1);
  const TOut *tsc = static_cast<const TOut *>(t.sc), *tsh = static_cast<const TOut *>(t.sh);
  // PAIR: CTAs 2p and 2p+1 share row block p; rank k runs SwiGLU chunks [k nL, (k+1) nL)
  // and finishes output columns [64k, 64k + 64)
  const int pb = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x, rank = PAIR ? (int)(blockIdx.x & 1) : 0;
  const int64_t m0 = (int64_t)pb * kUmmaBM;
  const int nkc_out = t.HD / kUmmaBK, nCall = t.M / 64;   // 64-wide hidden chunks
  const int nC = PAIR ? nCall / 2 : nCall, ch0 = rank * nC;   // this CTA's chunks

  if (tid == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      umma::mbar_init(full + s, 1);
      umma::mbar_init(empty + s, 1);
    }
    umma::mbar_init(a_ready, kTransEpiWarps);          // one arrival per epilogue warp
    umma::mbar_init(acc0_done, 1);
    umma::mbar_init(z_ready, kTransEpiWarps);
    for (int b = 0; b < 2; ++b) {
      umma::mbar_init(acc1_full + b, 1);
      umma::mbar_init(h_ready + b, kTransEpiWarps);
      umma::mbar_init(h_free + b, 1);
    }
    umma::mbar_init(acc2_done, 1);
    *abort_flag = 0;
    umma::fence_mbar_init();
  }
  if (warp == 0) umma::tmem_alloc(tslot, 512);
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t acc0 = tmem, acc1 = tmem + 128, acc2 = tmem + 384;   // acc1: two 128-col buffers
  bool ok = true;

  if (warp < kTransEpiWarps) {
    // warp w: TMEM lane quadrant w % 4 (rows 32 (w % 4) ..), column half w / 4 of every
    // 128-column matrix
    const int qd = warp & 3, hf = warp >> 2, cb = hf * 64;
    const int rl = qd * 32 + lane;
    const int64_t r = m0 + rl;
    const bool rok = r < t.R;
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    auto epi_sync = []() { asm volatile("bar.sync 1, %0;" ::"n"(kTransEpiWarps * 32) : "memory"); };

    // ---- o rows -> first operand (warp w converts rows 16w..16w+15; 8 lanes per row
    // segment, coalesced; the next chunk's loads in flight while one is converted)
    {
      const ProdPlain<TO> po{static_cast<const TO *>(t.O), (int64_t)t.HD, t.R, (int64_t)t.HD};
      if (po.vec_ok()) {
        form_rows_pipelined<SPLIT, 1, 1>(po, sA, m0, warp * 16, nkc_out, lane);
      } else {
        for (int kc = 0; kc < nkc_out; ++kc) {
          float v[4][8];
#pragma unroll
          for (int it = 0; it < 4; ++it)
            po.load8(m0 + warp * 16 + it * 4 + (lane >> 3), (int64_t)kc * kUmmaBK + (lane & 7) * 8, v[it]);
#pragma unroll
          for (int it = 0; it < 4; ++it)
            put8<SPLIT>(sA + kc * P * BLK, warp * 16 + it * 4 + (lane >> 3), (lane & 7) * 8, v[it]);
        }
      }
    }
    umma::fence_async_smem();
    __syncwarp();
    if (lane == 0) umma::mbar_arrive(a_ready);

    // ---- x' = x + g0 * acc0 on this warp's 64 columns, kept in TMEM in place of acc0;
    // partial statistics (shifted by the half's first x'), combined with the other half
    // through shared memory; then z -> operand
    float xv[32], gv[32];                       // chunk 0 fetched before the wait
    row32(tx, C, r, rok, cb, xv);
    row32(tg0, t.g_ld, r, rok, cb, gv);
    if (ok) ok = umma::mbar_wait_warp(acc0_done, 0, abort_flag, lane);
    umma::tc_fence_after();
    float shift = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll 1
    for (int c0 = cb; c0 < cb + 64; c0 += 32) {
      float a[32];
      if (c0 > cb) {
        row32(tx, C, r, rok, c0, xv);
        row32(tg0, t.g_ld, r, rok, c0, gv);
      }
      umma::tmem_ld32(tl + c0, a);
#pragma unroll
      for (int i = 0; i < 32; ++i) a[i] = fmaf(gv[i], a[i], xv[i]);
      if (c0 == cb) shift = t.rms ? 0.f : a[0];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float d = a[i] - shift;
        s1 += d;
        s2 = fmaf(d, d, s2);
      }
      umma::tmem_st32(tl + c0, a);
    }
    umma::tmem_wait_st();
    // the SwiGLU operand buffer is free until the first SwiGLU chunk: partials go there
    float *part = reinterpret_cast<float *>(sH);      // [2][128][3]
    part[(hf * 128 + rl) * 3 + 0] = s1;
    part[(hf * 128 + rl) * 3 + 1] = s2;
    part[(hf * 128 + rl) * 3 + 2] = shift;
    epi_sync();
    float mean = 0.f, ssd = 0.f;                // sum of squared deviations from mean
    {
      const float* p0 = part + rl * 3, *p1 = part + (128 + rl) * 3;
      if (t.rms) {
        ssd = p0[1] + p1[1];
      } else {
        mean = ((p0[0] + 64.f * p0[2]) + (p1[0] + 64.f * p1[2])) / (float)C;
        const float d0 = p0[2] - mean, d1 = p1[2] - mean;
        ssd = (p0[1] + 2.f * d0 * p0[0] + 64.f * d0 * d0) + (p1[1] + 2.f * d1 * p1[0] + 64.f * d1 * d1);
      }
    }
    const float rstd = 1.f / sqrtf(fmaxf(ssd, 0.f) / (float)C + t.eps);
#pragma unroll 1
    for (int c0 = cb; c0 < cb + 64; c0 += 32) {
      float a[32], sv[32], hv[32];
      row32(tsc, t.cond_ld, r, rok, c0, sv);
      row32(tsh, t.cond_ld, r, rok, c0, hv);
      umma::tmem_ld32(tl + c0, a);
#pragma unroll
      for (int s8 = 0; s8 < 4; ++s8) {
        float z[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = s8 * 8 + e;
          const float sc = t.plus1 ? 1.f + sv[i] : sv[i];
          z[e] = rok ? fmaf((a[i] - mean) * rstd, sc, hv[i]) : 0.f;
        }
        const int k = c0 + s8 * 8;
        put8<SPLIT>(sA + (k / kUmmaBK) * P * BLK, rl, k % kUmmaBK, z);
      }
    }
    umma::tc_fence_before();
    umma::fence_async_smem();
    __syncwarp();
    if (lane == 0) umma::mbar_arrive(z_ready);

    // ---- SwiGLU, one 64-wide chunk i of the hidden width at a time: TMEM buffer i % 2
    // (128 interleaved gate/up columns, this warp's 64) -> shared operand buffer i % 2
    for (int ch = 0; ch < nC; ++ch) {
      const int bf = ch & 1;
      if (ok) ok = umma::mbar_wait_warp(acc1_full + bf, (ch >> 1) & 1, abort_flag, lane);
      if (ch >= 2 && ok) ok = umma::mbar_wait_warp(h_free + bf, ((ch - 2) >> 1) & 1, abort_flag, lane);
      umma::tc_fence_after();
#pragma unroll 1
      for (int c0 = cb; c0 < cb + 64; c0 += 32) {
        float a[32];
        umma::tmem_ld32(tl + 128 + bf * 128 + c0, a);
#pragma unroll
        for (int s8 = 0; s8 < 2; ++s8) {
          float h[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = s8 * 16 + 2 * e;
            h[e] = silu_fast(a[j]) * a[j + 1];
          }
          put8<SPLIT>(sH + bf * P * BLK, rl, c0 / 2 + s8 * 8, h);
        }
      }
      umma::tc_fence_before();
      umma::fence_async_smem();
      __syncwarp();
      if (lane == 0) umma::mbar_arrive(h_ready + bf);
    }

    // ---- hidden = usable * (x' + g1 * acc2)
    // PAIR: the warps of the column half the other CTA finishes send their w_ff_out
    // partial through global scratch; the other warps add the peer's partial to theirs
    const bool sender = PAIR && hf != rank;
    const int64_t xrow = ((int64_t)pb * 2 + rank) * 128 + rl;        // this CTA's scratch row
    const int64_t prow = ((int64_t)pb * 2 + (1 - rank)) * 128 + rl;  // the peer's
    float g1v[32];                              // chunk 0 fetched before the wait
    if (!sender) row32(tg1, t.g_ld, r, rok, cb, g1v);
    const bool use_row = rok && t.usable[r] != 0;
    if (ok) ok = umma::mbar_wait_warp(acc2_done, 0, abort_flag, lane);
    umma::tc_fence_after();
    if (PAIR) {
      if (sender) {
#pragma unroll 1
        for (int c0 = cb; c0 < cb + 64; c0 += 32) {
          float f[32];
          umma::tmem_ld32(tl + 384 + c0, f);
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(t.xfer + xrow * 64 + (c0 - cb) + i) =
                make_float4(f[i], f[i + 1], f[i + 2], f[i + 3]);
        }
      }
      epi_sync();
      if (warp == 0 && lane == 0 && !t.withhold_flag) {
        __threadfence();
        atomicExch(t.xflag + pb * 2 + rank, 1);
      }
      if (!sender) {   // wait (bounded) for the peer's partial
        int got = 1;
        if (lane == 0) {
          got = 0;
          for (uint32_t it = 0; it < t.peer_spin_limit && !got; ++it)
            got = ld_acquire(t.xflag + pb * 2 + (1 - rank));
        }
        got = __shfl_sync(0xffffffffu, got, 0);
        __syncwarp();
        if (!got) ok = false;
      }
    }
    const bool use = ok && use_row;
    if (!sender) {
#pragma unroll 1
      for (int c0 = cb; c0 < cb + 64; c0 += 32) {
        float a[32], f[32];
        if (c0 > cb) row32(tg1, t.g_ld, r, rok, c0, g1v);
        umma::tmem_ld32(tl + c0, a);
        umma::tmem_ld32(tl + 384 + c0, f);
        if (PAIR) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 q = ok ? __ldcg(reinterpret_cast<const float4 *>(t.xfer + prow * 64 + (c0 - cb) + i))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            f[i] += q.x; f[i + 1] += q.y; f[i + 2] += q.z; f[i + 3] += q.w;
          }
        }
        if (rok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = use ? fmaf(g1v[i + e], f[i + e], a[i + e]) : 0.f;
            store8<TOut>((TOut *)t.hidden, r * C + c0 + i, o);
          }
        }
      }
    }
  } else if (warp == kTransEpiWarps) {
    if (lane == 0) {
      int i = 0;
      auto mma_block = [&](uint32_t dtm, const uint8_t *a_blk, bool first) {
        const int slot = i % NSLOT;
        if (ok) ok = umma::mbar_wait(full + slot, (i / NSLOT) & 1, abort_flag);
        umma::tc_fence_after();
        const uint32_t a0 = umma::smem_u32(a_blk), b0 = umma::smem_u32(sR + slot * P * BLK);
#pragma unroll
        for (int kk = 0; kk < kUmmaBK / 16; ++kk) {
          const uint64_t da = umma::sw128_desc(a0 + kk * 32), db = umma::sw128_desc(b0 + kk * 32);
          umma::mma_bf16(dtm, da, db, idesc, (!first || kk > 0) ? 1u : 0u);
          if (SPLIT) {
            umma::mma_bf16(dtm, da, umma::sw128_desc(b0 + BLK + kk * 32), idesc, 1);
            umma::mma_bf16(dtm, umma::sw128_desc(a0 + BLK + kk * 32), db, idesc, 1);
          }
        }
        umma::mma_commit(empty + slot);
        ++i;
      };
      if (ok) ok = umma::mbar_wait(a_ready, 0, abort_flag);
      umma::tc_fence_after();
      for (int kc = 0; kc < nkc_out; ++kc) mma_block(acc0, sA + kc * P * BLK, kc == 0);
      umma::mma_commit(acc0_done);
      if (ok) ok = umma::mbar_wait(z_ready, 0, abort_flag);
      umma::tc_fence_after();
      auto ff1 = [&](int ch) {   // hidden chunk ch (n-tile ch of w_ff1) -> acc1 buffer ch % 2
        for (int kc = 0; kc < 2; ++kc) mma_block(acc1 + (ch & 1) * 128, sA + kc * P * BLK, kc == 0);
        umma::mma_commit(acc1_full + (ch & 1));
      };
      ff1(0);
      if (nC > 1) ff1(1);
      for (int ch = 0; ch < nC && ok; ++ch) {
        if (ok) ok = umma::mbar_wait(h_ready + (ch & 1), (ch >> 1) & 1, abort_flag);
        umma::tc_fence_after();
        mma_block(acc2, sH + (ch & 1) * P * BLK, ch == 0);
        umma::mma_commit(h_free + (ch & 1));
        if (ch + 2 < nC) ff1(ch + 2);
      }
      umma::mma_commit(acc2_done);
    }
  } else {
    if (lane == 0) {
      int i = 0;
      auto put = [&](const uint8_t *W, int nkcW, int tile, int kc) {
        const int slot = i % NSLOT;
        if (i >= NSLOT && ok) ok = umma::mbar_wait(empty + slot, ((i - NSLOT) / NSLOT) & 1, abort_flag);
        umma::mbar_arrive_expect_tx(full + slot, P * BLK);
        umma::bulk_g2s(sR + slot * P * BLK, W + ((size_t)tile * nkcW + kc) * P * BLK, P * BLK,
                       full + slot);
        ++i;
      };
      for (int kc = 0; kc < nkc_out && ok; ++kc) put(t.w_out, nkc_out, 0, kc);
      // same order as the MMAs consume them
      auto ld_ff1 = [&](int ch) {
        for (int kc = 0; kc < 2; ++kc) put(t.w_ff1, 2, ch0 + ch, kc);
      };
      ld_ff1(0);
      if (nC > 1) ld_ff1(1);
      for (int ch = 0; ch < nC && ok; ++ch) {
        put(t.w_ff2, nCall, 0, ch0 + ch);
        if (ch + 2 < nC) ld_ff1(ch + 2);
      }
    }
  }
  if (!ok) {
    *abort_flag = 1;
    atomicOr(t.status, kStatusMmaTimeout);
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, 512);
}

}  // namespace atomenc
