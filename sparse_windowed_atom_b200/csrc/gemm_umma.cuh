// gemm_umma.cuh -- tcgen05 (5th-generation tensor core) GEMM with fused epilogues:
//   out = epi(A @ W),  A [M, K] float32 or bf16 in global memory, W [K, N] prepacked.
//
// One CTA computes a 128 x 128 output tile; 128 threads (4 warps).
//  * W is prepacked (k_prep_weights) as bf16 blocks of 128 output columns x 64 k in the
//    exact 128B-swizzled shared-memory image, so a block arrives with one bulk async
//    copy (mbarrier transaction count).
//  * The CTA's threads convert their A chunk (128 rows x 64 k) to bf16 and store it
//    swizzled; with SPLIT (float32 workloads) A and W are each split into bf16 high and
//    low parts and the product is hi*hi + hi*lo + lo*hi (three MMAs per k step), which
//    carries about 16 significant bits per operand into the float32 accumulator.
//  * Two shared-memory stages: the conversion of chunk c+1 overlaps the MMAs of chunk c.
//  * One thread issues tcgen05.mma (M=128, N=128, K=16) into a 128-column TMEM
//    accumulator and commits to mbarriers; every wait is bounded (status bit 4 on
//    timeout, never a hang).
//  * Epilogue: warp w reads TMEM lanes 32w..32w+31 (one output row per thread) with
//    tcgen05.ld and hands four consecutive columns at a time to the epilogue functor.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "umma.cuh"

namespace atomenc {

constexpr int kUmmaBM = 128, kUmmaBN = 128, kUmmaBK = 64, kUmmaThreads = 128, kUmmaStages = 2;
constexpr uint32_t kUmmaBlockBytes = kUmmaBN * kUmmaBK * 2;   // one bf16 [128 x 64] block
constexpr unsigned kStatusMmaTimeout = 4u;

__host__ __device__ constexpr size_t umma_smem_bytes(bool split) {
  // per stage: A (hi[, lo]) + B (hi[, lo]); + 1 KB for alignment and barriers
  return (size_t)kUmmaStages * (split ? 4 : 2) * kUmmaBlockBytes + 2048;
}

// Bytes of the packed image of a [K, N] weight.
__host__ __device__ inline size_t packed_bytes(int64_t K, int64_t N, bool split) {
  return (size_t)((N + kUmmaBN - 1) / kUmmaBN) * ((K + kUmmaBK - 1) / kUmmaBK) *
         kUmmaBlockBytes * (split ? 2 : 1);
}

template <typename TA>
__device__ __forceinline__ void load8_t(const TA *A, int64_t lda, int64_t M, int64_t K, int64_t r,
                                        int64_t k, float (&v)[8]);

template <>
__device__ __forceinline__ void load8_t<float>(const float *A, int64_t lda, int64_t M, int64_t K,
                                             int64_t r, int64_t k, float (&v)[8]) {
  // 16-byte loads only at 16-byte aligned addresses (callers' tensors may start anywhere)
  if (r < M && k + 8 <= K && (reinterpret_cast<uintptr_t>(A + r * lda + k) & 15) == 0) {
    const float4 x = *reinterpret_cast<const float4 *>(A + r * lda + k);
    const float4 y = *reinterpret_cast<const float4 *>(A + r * lda + k + 4);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = (r < M && k + e < K) ? A[r * lda + k + e] : 0.f;
  }
}

template <>
__device__ __forceinline__ void load8_t<__nv_bfloat16>(const __nv_bfloat16 *A, int64_t lda,
                                                     int64_t M, int64_t K, int64_t r, int64_t k,
                                                     float (&v)[8]) {
  if (r < M && k + 8 <= K && (reinterpret_cast<uintptr_t>(A + r * lda + k) & 15) == 0) {
    const uint4 x = *reinterpret_cast<const uint4 *>(A + r * lda + k);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(w[e] << 16);
      v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = (r < M && k + e < K) ? ldf(A, r * lda + k + e) : 0.f;
  }
}

// Eight consecutive elements of a row as loaded (one 16-byte load for bf16, two for
// float32), and their values.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> { uint4 u; };
template <> struct Raw8<float> { float4 a, b; };
__device__ __forceinline__ void raw8_load(const __nv_bfloat16 *p, Raw8<__nv_bfloat16> &w) {
  w.u = *reinterpret_cast<const uint4 *>(p);
}
__device__ __forceinline__ void raw8_load(const float *p, Raw8<float> &w) {
  w.a = *reinterpret_cast<const float4 *>(p);
  w.b = *reinterpret_cast<const float4 *>(p + 4);
}
__device__ __forceinline__ void raw8_get(const Raw8<__nv_bfloat16> &w, float (&v)[8]) {
  const uint32_t u[4] = {w.u.x, w.u.y, w.u.z, w.u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = __uint_as_float(u[e] << 16);
    v[2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void raw8_get(const Raw8<float> &w, float (&v)[8]) {
  v[0] = w.a.x; v[1] = w.a.y; v[2] = w.a.z; v[3] = w.a.w;
  v[4] = w.b.x; v[5] = w.b.y; v[6] = w.b.z; v[7] = w.b.w;
}
// rows of a [*, ld] tensor can be read as aligned groups of eight from column 8j
template <typename T>
__device__ __forceinline__ bool rows_vec_ok(const T *p, int64_t ld) {
  return (reinterpret_cast<uintptr_t>(p) & 15) == 0 && (ld & 7) == 0;
}

// ---- A producers of the row-block GEMM: what the CTA converts into its A operand.
// Each has two ways of delivering eight consecutive k of one row:
//   load8(r, k, v)        loads and converts at once, any shape or alignment;
//   row(r, rw), issue(r, k, w) and finish(rw, w, r, k, v)
//                         the loads alone (no branch: the row and k are clamped into the
//                         tensor, so every address is readable): the row's own values
//                         (flag, statistics) once per row, the eight payload values per k
//                         chunk; later the conversion, with rows >= M and k >= K set to
//                         zero. The operand loops keep kPipe chunks of payload loads in
//                         flight. Usable when vec_ok() (K a multiple of 8, rows 16-byte
//                         aligned); kPipe = 0 keeps a producer on load8 (its raw loads
//                         would not fit in registers).
// ProdPlain: A itself. ProdNorm: a row normalisation fused into the operand,
//   (x - mean) * rstd * scale + shift      (AF3 adaptive LN; the scale column already
//                                           holds sigmoid(...))
//   x * rstd * (1 + scale) + shift         (ESMFold2 modulation; mean = 0 for RMS)
// with the per-row mean/rstd computed where x is produced and scale/shift read from the
// conditioning rows.
template <typename TA>
struct ProdPlain {
  static constexpr bool kLight = true;   // a copy: four warps keep up with the epilogues
  static constexpr int kEpiWarps = 8;
  static constexpr int kPipe = 1;
  const TA *A;
  int64_t lda, M, K;
  __device__ void load8(int64_t r, int64_t k, float (&v)[8]) const {
    load8_t(A, lda, M, K, r, k, v);
  }
  struct Raw { Raw8<TA> a; };
  struct RowRaw {};
  __device__ bool vec_ok() const { return M > 0 && K > 0 && (K & 7) == 0 && rows_vec_ok(A, lda); }
  __device__ void row(int64_t, RowRaw &) const {}
  __device__ void issue(int64_t r, int64_t k, Raw &w) const {
    raw8_load(A + (r < M ? r : M - 1) * lda + (k < K ? k : K - 8), w.a);
  }
  __device__ void finish(const RowRaw &, const Raw &w, int64_t r, int64_t k, float (&v)[8]) const {
    float a[8];
    raw8_get(w.a, a);
    const bool in = r < M && k < K;
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = in ? a[e] : 0.f;
  }
};

template <typename IT>
struct ProdNormT {
  static constexpr bool kLight = false;
  // bf16: the pipelined loads let four producer warps keep up with eight epilogue warps
  static constexpr int kEpiWarps = sizeof(IT) == 2 ? 8 : 4;
  const IT *x;           // [M, K] residual state, storage type
  const float *stats;    // [M, 2]: mean (0 for RMS) and rstd of each row of x
  const IT *cond;        // rows of cond_ld values, storage type
  int64_t M, K, cond_ld, sc_off, sh_off;
  int plus1;
  static constexpr int kPipe = sizeof(IT) == 2 ? 1 : 0;
  __device__ void load8(int64_t r, int64_t k, float (&v)[8]) const {
    float xv[8], sc[8], sh[8];
    load8_t(x, K, M, K, r, k, xv);
    load8_t(cond + sc_off, cond_ld, M, K, r, k, sc);
    load8_t(cond + sh_off, cond_ld, M, K, r, k, sh);
    const float2 ms = r < M ? *reinterpret_cast<const float2 *>(stats + 2 * r) : make_float2(0.f, 0.f);
    combine(xv, sc, sh, ms, r < M, k, v);
  }
  __device__ void combine(const float (&xv)[8], const float (&sc)[8], const float (&sh)[8], float2 ms,
                          bool row_in, int64_t k, float (&v)[8]) const {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float s = plus1 ? 1.f + sc[e] : sc[e];
      v[e] = (row_in && k + e < K) ? fmaf((xv[e] - ms.x) * ms.y, s, sh[e]) : 0.f;
    }
  }
  struct Raw { Raw8<IT> x, sc, sh; };
  struct RowRaw { float2 ms; };
  __device__ bool vec_ok() const {
    return M > 0 && K > 0 && (K & 7) == 0 && rows_vec_ok(x, K) && rows_vec_ok(cond + sc_off, cond_ld) &&
           rows_vec_ok(cond + sh_off, cond_ld) && (reinterpret_cast<uintptr_t>(stats) & 7) == 0;
  }
  __device__ void row(int64_t r, RowRaw &rw) const {
    rw.ms = *reinterpret_cast<const float2 *>(stats + 2 * (r < M ? r : M - 1));
  }
  __device__ void issue(int64_t r, int64_t k, Raw &w) const {
    const int64_t rc = r < M ? r : M - 1, kc = k < K ? k : K - 8;
    raw8_load(x + rc * K + kc, w.x);
    raw8_load(cond + sc_off + rc * cond_ld + kc, w.sc);
    raw8_load(cond + sh_off + rc * cond_ld + kc, w.sh);
  }
  __device__ void finish(const RowRaw &rw, const Raw &w, int64_t r, int64_t k, float (&v)[8]) const {
    float xv[8], sc[8], sh[8];
    raw8_get(w.x, xv);
    raw8_get(w.sc, sc);
    raw8_get(w.sh, sh);
    combine(xv, sc, sh, rw.ms, r < M, k, v);
  }
};
using ProdNorm = ProdNormT<float>;

// The condition operand of the conditioning products, formed from the caller's
// condition rows: zero for an unusable atom (a select, so NaN / Inf payloads never
// enter), else MODE 0 the raw value (AF3 residual gates, bullet 9), MODE 1 SiLU
// (ESMFold2 w_mod, bullet 10), MODE 2 (c - mean) * rstd with the row's population
// LayerNorm statistics (AF3 c_j, bullet 7; cond_scale[j] is folded into the weights).
template <typename T, int MODE>
struct ProdCond {
  static constexpr bool kLight = false;
  // SiLU / LayerNorm operands over K up to 256: eight producer warps (four, even with
  // two chunks of loads in flight, fell behind eight epilogue warps)
  static constexpr int kEpiWarps = 4;
  const T *c;            // [M, K] condition rows
  const uint8_t *usable; // [M]
  const float *stats;    // [M, 2] (MODE 2)
  int64_t M, K;
  static constexpr int kPipe = 1;
  __device__ void load8(int64_t r, int64_t k, float (&v)[8]) const {
    // the loads do not wait for the usable flag (every row in range is readable memory;
    // what an unusable row holds is dropped by the select below)
    float cv[8];
    load8_t(c, K, M, K, r, k, cv);
    float2 ms = make_float2(0.f, 1.f);
    if (MODE == 2 && r < M) ms = *reinterpret_cast<const float2 *>(stats + 2 * r);
    combine(cv, ms, r < M && usable[r] != 0, k, v);
  }
  __device__ void combine(const float (&cv)[8], float2 ms, bool use, int64_t k, float (&v)[8]) const {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float y = cv[e];
      if (MODE == 1) y = silu_fast(y);
      if (MODE == 2) y = (y - ms.x) * ms.y;
      v[e] = (use && k + e < K) ? y : 0.f;
    }
  }
  struct Raw { Raw8<T> c; };
  struct RowRaw { float2 ms; uint32_t use; };
  __device__ bool vec_ok() const {
    return M > 0 && K > 0 && (K & 7) == 0 && rows_vec_ok(c, K) &&
           (MODE != 2 || (reinterpret_cast<uintptr_t>(stats) & 7) == 0);
  }
  __device__ void row(int64_t r, RowRaw &rw) const {
    const int64_t rc = r < M ? r : M - 1;
    rw.use = usable[rc];
    rw.ms = make_float2(0.f, 1.f);
    if (MODE == 2) rw.ms = *reinterpret_cast<const float2 *>(stats + 2 * rc);
  }
  __device__ void issue(int64_t r, int64_t k, Raw &w) const {
    raw8_load(c + (r < M ? r : M - 1) * K + (k < K ? k : K - 8), w.c);
  }
  __device__ void finish(const RowRaw &rw, const Raw &w, int64_t r, int64_t k, float (&v)[8]) const {
    float cv[8];
    raw8_get(w.c, cv);
    combine(cv, rw.ms, r < M && rw.use != 0, k, v);
  }
};

template <typename TA, bool SPLIT, class Epi>
__global__ void __launch_bounds__(kUmmaThreads)
    k_gemm_umma(const TA *__restrict__ A, int64_t lda, const uint8_t *__restrict__ Wpk, int64_t M,
                int64_t N, int64_t K, Epi epi, unsigned *status) {
  pdl_enter();
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  // 1024-byte alignment of the operand blocks (swizzle atoms)
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  constexpr int PARTS = SPLIT ? 2 : 1;
  uint8_t *sA = sm;                                                  // [stage][part] blocks
  uint8_t *sB = sm + kUmmaStages * PARTS * kUmmaBlockBytes;          // [stage][part] blocks
  uint64_t *bar = reinterpret_cast<uint64_t *>(sB + kUmmaStages * PARTS * kUmmaBlockBytes);
  uint64_t *bar_b = bar, *bar_mma = bar + kUmmaStages, *bar_done = bar + 2 * kUmmaStages;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 2 * kUmmaStages + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tile = blockIdx.x, m0 = (int64_t)blockIdx.y * kUmmaBM, n0 = n_tile * kUmmaBN;
  const int nkc = (int)((K + kUmmaBK - 1) / kUmmaBK);
  constexpr uint32_t idesc = umma::idesc_bf16(kUmmaBM, kUmmaBN);

  if (tid == 0) {
    for (int s = 0; s < kUmmaStages; ++s) {
      umma::mbar_init(bar_b + s, 1);
      umma::mbar_init(bar_mma + s, 1);
    }
    umma::mbar_init(bar_done, 1);
    umma::fence_mbar_init();
  }
  if (warp == 0) umma::tmem_alloc(tslot, kUmmaBN);
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = true;

  for (int c = 0; c < nkc; ++c) {
    const int s = c % kUmmaStages;
    if (c >= kUmmaStages && ok)  // the MMAs that read this stage two chunks ago are done
      ok = umma::mbar_wait(bar_mma + s, ((c - kUmmaStages) / kUmmaStages) & 1);
    uint8_t *a_s = sA + s * PARTS * kUmmaBlockBytes;
    uint8_t *b_s = sB + s * PARTS * kUmmaBlockBytes;
    if (tid == 0) {
      umma::mbar_arrive_expect_tx(bar_b + s, PARTS * kUmmaBlockBytes);
      umma::bulk_g2s(b_s, Wpk + ((n_tile * nkc + c) * PARTS) * (size_t)kUmmaBlockBytes,
                     PARTS * kUmmaBlockBytes, bar_b + s);
    }
    // A chunk: warp w converts rows 32w..32w+31; 8 lanes per row, 8 k each
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int r = warp * 32 + it * 4 + (lane >> 3), seg = lane & 7;
      float v[8];
      load8_t<TA>(A, lda, M, K, m0 + r, (int64_t)c * kUmmaBK + seg * 8, v);
      uint32_t hi[4], lo[4];
      umma::split8<SPLIT>(v, hi, lo);
      const uint32_t off = umma::swz_offset(r, seg * 8, kUmmaBM);
      *reinterpret_cast<uint4 *>(a_s + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      if (SPLIT)
        *reinterpret_cast<uint4 *>(a_s + kUmmaBlockBytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    umma::fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      if (ok) ok = umma::mbar_wait(bar_b + s, (c / kUmmaStages) & 1);
      umma::tc_fence_after();
      const uint32_t a0 = umma::smem_u32(a_s), b0 = umma::smem_u32(b_s);
#pragma unroll
      for (int kk = 0; kk < kUmmaBK / 16; ++kk) {
        const uint64_t da = umma::sw128_desc(a0 + kk * 32), db = umma::sw128_desc(b0 + kk * 32);
        umma::mma_bf16(tmem, da, db, idesc, (c | kk) != 0);
        if (SPLIT) {
          umma::mma_bf16(tmem, da, umma::sw128_desc(b0 + kUmmaBlockBytes + kk * 32), idesc, 1);
          umma::mma_bf16(tmem, umma::sw128_desc(a0 + kUmmaBlockBytes + kk * 32), db, idesc, 1);
        }
      }
      umma::mma_commit(bar_mma + s);
    }
  }
  if (tid == 0) umma::mma_commit(bar_done);
  if (ok) ok = umma::mbar_wait(bar_done, 0);
  if (!ok && lane == 0) atomicOr(status, kStatusMmaTimeout);
  umma::tc_fence_after();

  // epilogue: thread (warp w, lane l) owns output row m0 + 32w + l
  const int64_t row = m0 + warp * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
  for (int c0 = 0; c0 < kUmmaBN; c0 += 32) {
    if (n0 + c0 >= N) break;
    float v[32];
    umma::tmem_ld32(trow + c0, v);
    if (row < M && ok) {
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        if (n0 + c0 + j < N) {
          const float q[4] = {v[j], v[j + 1], v[j + 2], v[j + 3]};
          epi.quad(row, n0 + c0 + j, q, N);
        }
    }
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, kUmmaBN);
}

// ----------------------------------------------------------------------------------
// Row-block GEMM: one CTA owns 128 rows of A (all of K resident in shared memory,
// converted once) and a contiguous range of 128-column output tiles. Warp roles:
//   warps 0-7  convert A (warp w: rows 16w..16w+15), then run the epilogue of each tile
//              (warp w: TMEM lanes 32 (w % 4).. and the column half w / 4); the
//              accumulator chunk is transposed through a per-warp shared tile so that
//              the epilogue functor sees 8 lanes per 128-byte row segment (coalesced
//              global reads and writes);
//   warp 8     lane 0 issues the MMAs: two 128-column TMEM accumulators, so the MMAs of
//              tile t+1 run while the epilogue drains tile t;
//   warp 9     lane 0 streams the packed weight blocks through a ring of nslot shared
//              buffers with bulk async copies (nslot is sized on the host to what shared
//              memory holds, up to every block the CTA needs, so the copies of all of a
//              CTA's weight blocks can be in flight at once).
// Requires K <= kRowsKMax; every wait is bounded (status bit 4 on timeout).
constexpr int kRowsEpiWarps = 8;                        // two per TMEM lane quadrant
constexpr int kRowsTPitch = 32;                         // floats per row of a transpose tile
// shared loads per batch in the row-block GEMMs' epilogue chunks (measured: 2 beats 1, 4
// and 8 in both the one-CTA-per-row-block and the persistent kernel)
constexpr int kRowsEpiBatch = 2;
constexpr int kRowsThreads = (kRowsEpiWarps + 2) * 32;  // + MMA issuer + weight loader
constexpr int kRowsKMax = 256;
constexpr int kRowsMaxSlots = 4;   // deeper rings were measured slower (every CTA fetches
                                   // the same weight blocks)
constexpr size_t kRowsSmemBudget = 225 * 1024;

// shared bytes of the row-block GEMM with nslot weight slots
__host__ __device__ inline size_t rows_smem_bytes(int64_t K, bool split, int nslot) {
  const int parts = split ? 2 : 1;
  const size_t nkc = (size_t)((K + kUmmaBK - 1) / kUmmaBK);
  return 1024 + (nkc + (size_t)nslot) * parts * kUmmaBlockBytes +
         (size_t)kRowsEpiWarps * 32 * kRowsTPitch * 4 + 512;
}
// weight slots: every block one CTA consumes (blocks_per_cta) if they fit, else as many
// as shared memory holds, at least 2
__host__ __device__ inline int rows_slots(int64_t K, bool split, int blocks_per_cta) {
  int n = blocks_per_cta < kRowsMaxSlots ? blocks_per_cta : kRowsMaxSlots;
  while (n > 2 && rows_smem_bytes(K, split, n) > kRowsSmemBudget) --n;
  return n < 2 ? 2 : n;
}

// The epilogue of one 32 x 32 chunk of accumulator rows: v holds this lane's row (TMEM
// lane = row) at 32 consecutive columns. The chunk is transposed through the warp's shared
// tile T so that each store instruction covers 64 contiguous bytes of four rows: lane
// (rr = lane / 8, q = lane % 8) hands columns col0 + 4q .. + 3 of rows row0 + rr, + 4, ...
// to the epilogue functor. 16-byte chunk j of tile row r sits at chunk j ^ (r & 7), so the
// eight lanes of a store phase (eight rows, one chunk) and of a load phase (one row, eight
// chunks) each cover all 32 banks once. The shared loads are issued NB at a time and a
// whole in-range chunk takes one bounds check.
// Epilogue functors whose kOct is true (with an oct(row, col, v[8], N) member) take eight
// consecutive columns per lane: one 16-byte store of bf16 (two of float32), eight rows
// per store instruction instead of four; the others take quads.
template <class E, class = void> struct EpiOct : std::false_type {};
template <class E>
struct EpiOct<E, std::void_t<decltype(E::kOct)>> : std::bool_constant<E::kOct> {};

template <int NB, class Epi>
__device__ __forceinline__ void epi_chunk(const Epi &epi, float *T, const float (&v)[32], int lane,
                                          int64_t row0, int64_t col0, int64_t M, int64_t N, bool ok) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4 *>(T + lane * kRowsTPitch + 4 * (j ^ (lane & 7))) =
        make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  __syncwarp();
  const bool whole = row0 + 32 <= M && col0 + 32 <= N;
  if constexpr (EpiOct<Epi>::value) {
    // lane (g = lane / 8, h = lane / 4 % 2, q = lane % 4) takes columns 8q .. 8q + 7 of row
    // 8i + 2g + h: each store instruction covers eight rows, 64 contiguous bytes of bf16
    // each; the eight lanes of a load phase read two rows of opposite parity, whose four
    // chunks each land on distinct swizzled positions (all 32 banks once). An oct whose
    // eight columns cannot go in one aligned store falls back to quads, the second only
    // where it starts inside the row (quads store without a column check).
    const int q = lane & 3, rr = 2 * (lane >> 3) + ((lane >> 2) & 1);
    const int64_t col = col0 + 8 * q;
#pragma unroll
    for (int i0 = 0; i0 < 4; i0 += NB) {
      float4 t[NB][2];
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        const int rl = (i0 + i) * 8 + rr;
        t[i][0] = *reinterpret_cast<const float4 *>(T + rl * kRowsTPitch + 4 * ((2 * q) ^ (rl & 7)));
        t[i][1] = *reinterpret_cast<const float4 *>(T + rl * kRowsTPitch + 4 * ((2 * q + 1) ^ (rl & 7)));
      }
      if (ok) {
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          const int64_t row = row0 + (i0 + i) * 8 + rr;
          const float x[8] = {t[i][0].x, t[i][0].y, t[i][0].z, t[i][0].w,
                              t[i][1].x, t[i][1].y, t[i][1].z, t[i][1].w};
          if (whole || (row < M && col < N)) epi.oct(row, col, x, N);
        }
      }
    }
  } else {
    const int q = lane & 7, rr = lane >> 3;
    const int64_t col = col0 + 4 * q;
#pragma unroll
    for (int i0 = 0; i0 < 8; i0 += NB) {
      float4 t[NB];
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        const int rl = (i0 + i) * 4 + rr;
        t[i] = *reinterpret_cast<const float4 *>(T + rl * kRowsTPitch + 4 * (q ^ (rl & 7)));
      }
      if (ok) {
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          const int64_t row = row0 + (i0 + i) * 4 + rr;
          const float x[4] = {t[i].x, t[i].y, t[i].z, t[i].w};
          if (whole || (row < M && col < N)) epi.quad(row, col, x, N);
        }
      }
    }
  }
  __syncwarp();   // T is free for the next chunk
}

template <bool SPLIT, int P, int HALVES, class Prod>
__device__ __forceinline__ void form_rows_pipelined(const Prod &prod, uint8_t *aB, int64_t m0, int row_first,
                                                    int nkc, int lane) {
  constexpr int PARTS = SPLIT ? 2 : 1;
  constexpr uint32_t BLK = kUmmaBlockBytes;
  const int nst = HALVES * nkc, seg = lane & 7;
  auto row_of = [&](int st, int it) { return row_first + (st / nkc) * 16 + it * 4 + (lane >> 3); };
  auto k_of = [&](int st) { return (int64_t)(st % nkc) * kUmmaBK + seg * 8; };
  typename Prod::RowRaw rw[HALVES][4];
#pragma unroll
  for (int h = 0; h < HALVES; ++h)
#pragma unroll
    for (int it = 0; it < 4; ++it) prod.row(m0 + row_first + h * 16 + it * 4 + (lane >> 3), rw[h][it]);
  typename Prod::Raw w[P][4];
#pragma unroll
  for (int p = 0; p < P; ++p)
    if (p < nst) {
#pragma unroll
      for (int it = 0; it < 4; ++it) prod.issue(m0 + row_of(p, it), k_of(p), w[p][it]);
    }
  for (int s0 = 0; s0 < nst; s0 += P) {
#pragma unroll
    for (int p = 0; p < P; ++p) {
      const int st = s0 + p;
      if (st < nst) {
        uint8_t *a_c = aB + (size_t)(st % nkc) * PARTS * BLK;
        const int64_t k = k_of(st);
        const int h = st / nkc;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int r = row_of(st, it);
          float v[8];
          // rw is indexed by the half through a select (HALVES <= 2), not a dynamic index
          prod.finish(HALVES == 1 || h == 0 ? rw[0][it] : rw[HALVES - 1][it], w[p][it], m0 + r, k, v);
          if (st + P < nst) prod.issue(m0 + row_of(st + P, it), k_of(st + P), w[p][it]);
          uint32_t hi[4], lo[4];
          umma::split8<SPLIT>(v, hi, lo);
          const uint32_t off = umma::swz_offset(r, seg * 8, kUmmaBM);
          *reinterpret_cast<uint4 *>(a_c + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          if (SPLIT) *reinterpret_cast<uint4 *>(a_c + BLK + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
  }
}

template <class Prod, bool SPLIT, class Epi>
__global__ void __launch_bounds__(kRowsThreads, 1)
    k_gemm_rows(Prod prod, const uint8_t *__restrict__ Wpk, int64_t M, int64_t N, int64_t K,
                int tiles_per_cta, int NSLOT, Epi epi, unsigned *status) {
  pdl_enter();
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  constexpr int PARTS = SPLIT ? 2 : 1;
  constexpr uint32_t BLK = kUmmaBlockBytes;
  constexpr uint32_t idesc = umma::idesc_bf16(kUmmaBM, kUmmaBN);
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const int nkc = (int)((K + kUmmaBK - 1) / kUmmaBK);
  uint8_t *sA = sm;                                       // [nkc][PARTS] blocks
  uint8_t *sR = sA + (size_t)nkc * PARTS * BLK;           // [NSLOT][PARTS] blocks
  float *sT = reinterpret_cast<float *>(sR + (size_t)NSLOT * PARTS * BLK);   // [warps][32][pitch]
  uint64_t *full = reinterpret_cast<uint64_t *>(sT + kRowsEpiWarps * 32 * kRowsTPitch);
  uint64_t *empty = full + NSLOT, *accf = empty + NSLOT, *acce = accf + 2, *aready = acce + 2;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(aready + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = (int)((N + kUmmaBN - 1) / kUmmaBN);
  const int t_begin = blockIdx.x * tiles_per_cta;
  const int ntl = min(nt, t_begin + tiles_per_cta) - t_begin;
  if (ntl <= 0) return;  // uniform over the CTA
  const int64_t m0 = (int64_t)blockIdx.y * kUmmaBM;

  if (tid == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      umma::mbar_init(full + s, 1);
      umma::mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      umma::mbar_init(accf + b, 1);
      umma::mbar_init(acce + b, kRowsEpiWarps);        // one arrival per epilogue warp
    }
    umma::mbar_init(aready, kRowsEpiWarps);
    *abort_flag = 0;
    umma::fence_mbar_init();
  }
  if (warp == 0) umma::tmem_alloc(tslot, 2 * kUmmaBN);
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = true;

  if (warp < kRowsEpiWarps) {
    // ---- A: rows 16w..16w+15 of the tile, every k chunk, bf16 (hi[, lo]) swizzled;
    // the loads of chunk c + 1 are issued before chunk c is converted
    bool piped = false;
    if constexpr (Prod::kPipe > 0) {
      if (prod.vec_ok()) {
        form_rows_pipelined<SPLIT, Prod::kPipe, 1>(prod, sA, m0, warp * 16, nkc, lane);
        piped = true;
      }
    }
    if (!piped) {
    float vb[2][4][8];
    auto load_chunk = [&](int c, float (&v)[4][8]) {
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int rl = warp * 16 + it * 4 + (lane >> 3);
        prod.load8(m0 + rl, (int64_t)c * kUmmaBK + (lane & 7) * 8, v[it]);
      }
    };
    auto store_chunk = [&](int c, float (&v)[4][8]) {
      uint8_t *a_c = sA + (size_t)c * PARTS * BLK;
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int r = warp * 16 + it * 4 + (lane >> 3), seg = lane & 7;
        uint32_t hi[4], lo[4];
        umma::split8<SPLIT>(v[it], hi, lo);
        const uint32_t off = umma::swz_offset(r, seg * 8, kUmmaBM);
        *reinterpret_cast<uint4 *>(a_c + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if (SPLIT)
          *reinterpret_cast<uint4 *>(a_c + BLK + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    };
    load_chunk(0, vb[0]);
    for (int c = 0; c < nkc; c += 2) {
      if (c + 1 < nkc) load_chunk(c + 1, vb[1]);
      store_chunk(c, vb[0]);
      if (c + 1 < nkc) {
        if (c + 2 < nkc) load_chunk(c + 2, vb[0]);
        store_chunk(c + 1, vb[1]);
      }
    }
    }
    umma::fence_async_smem();
    __syncwarp();
    if (lane == 0) umma::mbar_arrive(aready);

    // ---- epilogue of each output tile: warp w reads TMEM lane quadrant w % 4 and the
    // column half w / 4 of the tile
    const int qd = warp & 3, cb = (warp >> 2) * (kUmmaBN / 2);
    float *T = sT + warp * 32 * kRowsTPitch;
    const uint32_t tlane = tmem + ((uint32_t)(qd * 32) << 16);
    for (int tl = 0; tl < ntl; ++tl) {
      const int buf = tl & 1;
      if (ok) ok = umma::mbar_wait_warp(accf + buf, (tl >> 1) & 1, abort_flag, lane);
      umma::tc_fence_after();
      const int64_t n0 = (int64_t)(t_begin + tl) * kUmmaBN;
#pragma unroll 1
      for (int c0 = cb; c0 < cb + kUmmaBN / 2; c0 += 32) {
        if (n0 + c0 >= N) break;
        float v[32];
        umma::tmem_ld32(tlane + buf * kUmmaBN + c0, v);
        epi_chunk<kRowsEpiBatch>(epi, T, v, lane, m0 + qd * 32, n0 + c0, M, N, ok);
      }
      umma::tc_fence_before();
      __syncwarp();
      if (lane == 0) umma::mbar_arrive(acce + buf);
    }
  } else if (warp == kRowsEpiWarps) {
    if (lane == 0) {
      // ---- MMA issue
      ok = umma::mbar_wait(aready, 0, abort_flag);
      umma::tc_fence_after();
      for (int tl = 0; tl < ntl && ok; ++tl) {
        const int buf = tl & 1;
        if (tl >= 2) {
          ok = umma::mbar_wait(acce + buf, ((tl - 2) >> 1) & 1, abort_flag);
          umma::tc_fence_after();
        }
        const uint32_t dtm = tmem + buf * kUmmaBN;
        for (int c = 0; c < nkc && ok; ++c) {
          const int i = tl * nkc + c, slot = i % NSLOT;
          ok = umma::mbar_wait(full + slot, (i / NSLOT) & 1, abort_flag);
          umma::tc_fence_after();
          const uint32_t a0 = umma::smem_u32(sA + (size_t)c * PARTS * BLK);
          const uint32_t b0 = umma::smem_u32(sR + (size_t)slot * PARTS * BLK);
#pragma unroll
          for (int kk = 0; kk < kUmmaBK / 16; ++kk) {
            const uint64_t da = umma::sw128_desc(a0 + kk * 32), db = umma::sw128_desc(b0 + kk * 32);
            umma::mma_bf16(dtm, da, db, idesc, (c | kk) != 0);
            if (SPLIT) {
              umma::mma_bf16(dtm, da, umma::sw128_desc(b0 + BLK + kk * 32), idesc, 1);
              umma::mma_bf16(dtm, umma::sw128_desc(a0 + BLK + kk * 32), db, idesc, 1);
            }
          }
          umma::mma_commit(empty + slot);
        }
        umma::mma_commit(accf + buf);
      }
    }
  } else {
    if (lane == 0) {
      // ---- weight blocks, ring of NSLOT buffers
      const int total = ntl * nkc;
      for (int i = 0; i < total && ok; ++i) {
        const int slot = i % NSLOT;
        if (i >= NSLOT) ok = umma::mbar_wait(empty + slot, ((i - NSLOT) / NSLOT) & 1, abort_flag);
        const int tl = i / nkc, c = i - tl * nkc;
        umma::mbar_arrive_expect_tx(full + slot, PARTS * BLK);
        umma::bulk_g2s(sR + (size_t)slot * PARTS * BLK,
                       Wpk + ((size_t)(t_begin + tl) * nkc + c) * PARTS * BLK, PARTS * BLK,
                       full + slot);
      }
    }
  }
  if (!ok) {
    *abort_flag = 1;
    atomicOr(status, kStatusMmaTimeout);
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, 2 * kUmmaBN);
}

// ----------------------------------------------------------------------------------
// Persistent row-block GEMM (bf16 operands, no hi/lo split): one CTA per SM walks the
// row blocks blockIdx.x, blockIdx.x + gridDim.x, ... and all output tiles of each, with
// the A operand double-buffered so that the operand of the next row block is formed
// while the current one's MMAs and epilogues run. Fourteen warps (four per SM
// sub-partition at most, so 128 registers a thread); roles:
//   warps 0..EW-1      epilogue of each tile (TMEM lane quadrant w % 4, a 512/EW-column
//                      share of the tile, transposed through a per-warp shared tile);
//   warps EW..11       form the A operand (128/(12-EW) rows each) into the free buffer,
//                      then arrive on its "full" barrier;
//   warp 12            lane 0 issues the MMAs: two 128-column TMEM accumulators alternate
//                      over the CTA's tiles; after a block's last tile a commit frees its A
//                      buffer;
//   warp 13            lane 0 streams the weight blocks through the ring (every block of
//                      every tile, in the MMA's order).
// EW is the producer's kEpiWarps: 8 for a plain copy and for the bf16 modulated norm of
// the projections (four producer warps with pipelined loads keep up), 4 for the condition
// operands (SiLU / LayerNorm over K up to 256 need eight producer warps).
// Every wait is bounded (status bit 4 on timeout; the other roles then stop too).
constexpr int kRowsPThreads = 14 * 32;

__host__ __device__ inline size_t rows_p_smem_bytes(int64_t K, int nslot, int ew) {
  const size_t nkc = (size_t)((K + kUmmaBK - 1) / kUmmaBK);
  return 1024 + (2 * nkc + (size_t)nslot) * kUmmaBlockBytes + (size_t)ew * 32 * kRowsTPitch * 4 + 512;
}
// weight slots of the persistent kernel: up to kRowsMaxSlots, at least 2, within the budget
__host__ __device__ inline int rows_p_slots(int64_t K, int ew) {
  int n = kRowsMaxSlots;
  while (n > 2 && rows_p_smem_bytes(K, n, ew) > kRowsSmemBudget) --n;
  return n;
}

template <class Prod, class Epi, int EW>
__global__ void __launch_bounds__(kRowsPThreads, 1)
    k_gemm_rows_p(Prod prod, const uint8_t *__restrict__ Wpk, int64_t M, int64_t N, int64_t K,
                  int NSLOT, Epi epi, unsigned *status) {
  constexpr int PW = 12 - EW;               // producer warps
  constexpr int RPW = kUmmaBM / PW;         // operand rows per producer warp
  constexpr int CPW = kUmmaBN * 4 / EW;     // tile columns per epilogue warp
  static_assert(EW == 4 || EW == 8, "epilogue warps");
  pdl_enter();
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  constexpr uint32_t BLK = kUmmaBlockBytes;
  constexpr uint32_t idesc = umma::idesc_bf16(kUmmaBM, kUmmaBN);
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  const int nkc = (int)((K + kUmmaBK - 1) / kUmmaBK);
  uint8_t *sA = sm;                                       // [2][nkc] blocks
  uint8_t *sR = sA + (size_t)2 * nkc * BLK;               // [NSLOT] blocks
  float *sT = reinterpret_cast<float *>(sR + (size_t)NSLOT * BLK);   // [warps][32][pitch]
  uint64_t *full = reinterpret_cast<uint64_t *>(sT + EW * 32 * kRowsTPitch);
  uint64_t *empty = full + NSLOT, *accf = empty + NSLOT, *acce = accf + 2;
  uint64_t *afull = acce + 2, *aempty = afull + 2;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(aempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = (int)((N + kUmmaBN - 1) / kUmmaBN);
  const int64_t mb = (M + kUmmaBM - 1) / kUmmaBM;
  const int nblk = (int)((mb - blockIdx.x + gridDim.x - 1) / gridDim.x);   // my row blocks
  if (nblk <= 0) return;  // uniform over the CTA

  if (tid == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      umma::mbar_init(full + s, 1);
      umma::mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      umma::mbar_init(accf + b, 1);
      umma::mbar_init(acce + b, EW);
      umma::mbar_init(afull + b, PW);
      umma::mbar_init(aempty + b, 1);
    }
    *abort_flag = 0;
    umma::fence_mbar_init();
  }
  if (warp == 0) umma::tmem_alloc(tslot, 2 * kUmmaBN);
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = true;

  if (warp < EW) {
    // ---- epilogues: tile g of the CTA (block bi, tile tl) reads accumulator g % 2
    const int qd = warp & 3, cb = (warp >> 2) * CPW;
    float *T = sT + warp * 32 * kRowsTPitch;
    const uint32_t tlane = tmem + ((uint32_t)(qd * 32) << 16);
    int g = 0;
    for (int bi = 0; bi < nblk && ok; ++bi) {
      const int64_t m0 = ((int64_t)blockIdx.x + (int64_t)bi * gridDim.x) * kUmmaBM;
      for (int tl = 0; tl < nt && ok; ++tl, ++g) {
        const int buf = g & 1;
        ok = umma::mbar_wait_warp(accf + buf, (g >> 1) & 1, abort_flag, lane);
        umma::tc_fence_after();
        const int64_t n0 = (int64_t)tl * kUmmaBN;
#pragma unroll 1
        for (int c0 = cb; c0 < cb + CPW; c0 += 32) {
          if (n0 + c0 >= N) break;
          float v[32];
          umma::tmem_ld32(tlane + buf * kUmmaBN + c0, v);
          epi_chunk<kRowsEpiBatch>(epi, T, v, lane, m0 + qd * 32, n0 + c0, M, N, ok);
        }
        umma::tc_fence_before();
        __syncwarp();
        if (lane == 0) umma::mbar_arrive(acce + buf);
      }
    }
  } else if (warp < EW + PW) {
    // ---- A operand of each of the CTA's row blocks into buffer bi % 2: producer warp p
    // forms rows RPW p .. RPW (p + 1) - 1 in groups of 16, the loads of chunk c + 1 in
    // flight while chunk c is converted
    const int pw = warp - EW;
    bool pipe_ok = false;
    if constexpr (Prod::kPipe > 0) pipe_ok = prod.vec_ok();
    for (int bi = 0; bi < nblk && ok; ++bi) {
      const int buf = bi & 1;
      if (bi >= 2) {
        ok = umma::mbar_wait_warp(aempty + buf, ((bi - 2) >> 1) & 1, abort_flag, lane);
        umma::tc_fence_after();
        if (!ok) break;
      }
      const int64_t m0 = ((int64_t)blockIdx.x + (int64_t)bi * gridDim.x) * kUmmaBM;
      uint8_t *aB = sA + (size_t)buf * nkc * BLK;
      if constexpr (Prod::kPipe > 0) {
        if (pipe_ok) {
          form_rows_pipelined<false, Prod::kPipe, RPW / 16>(prod, aB, m0, pw * RPW, nkc, lane);
          umma::fence_async_smem();
          __syncwarp();
          if (lane == 0) umma::mbar_arrive(afull + buf);
          continue;
        }
      }
      for (int half = 0; half < RPW / 16; ++half) {
        const int r0 = pw * RPW + half * 16;
        float vb[2][4][8];
        auto load_chunk = [&](int c, float (&v)[4][8]) {
#pragma unroll
          for (int it = 0; it < 4; ++it)
            prod.load8(m0 + r0 + it * 4 + (lane >> 3), (int64_t)c * kUmmaBK + (lane & 7) * 8, v[it]);
        };
        auto store_chunk = [&](int c, float (&v)[4][8]) {
          uint8_t *a_c = aB + (size_t)c * BLK;
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int r = r0 + it * 4 + (lane >> 3), seg = lane & 7;
            uint32_t hi[4], lo[4];
            umma::split8<false>(v[it], hi, lo);
            *reinterpret_cast<uint4 *>(a_c + umma::swz_offset(r, seg * 8, kUmmaBM)) =
                make_uint4(hi[0], hi[1], hi[2], hi[3]);
          }
        };
        load_chunk(0, vb[0]);
        for (int c = 0; c < nkc; c += 2) {
          if (c + 1 < nkc) load_chunk(c + 1, vb[1]);
          store_chunk(c, vb[0]);
          if (c + 1 < nkc) {
            if (c + 2 < nkc) load_chunk(c + 2, vb[0]);
            store_chunk(c + 1, vb[1]);
          }
        }
      }
      umma::fence_async_smem();
      __syncwarp();
      if (lane == 0) umma::mbar_arrive(afull + buf);
    }
  } else if (warp == EW + PW) {
    if (lane == 0) {
      // ---- MMA issue
      int g = 0;
      for (int bi = 0; bi < nblk && ok; ++bi) {
        const int ab = bi & 1;
        ok = umma::mbar_wait(afull + ab, (bi >> 1) & 1, abort_flag);
        umma::tc_fence_after();
        for (int tl = 0; tl < nt && ok; ++tl, ++g) {
          const int buf = g & 1;
          if (g >= 2) {
            ok = umma::mbar_wait(acce + buf, ((g - 2) >> 1) & 1, abort_flag);
            umma::tc_fence_after();
          }
          const uint32_t dtm = tmem + buf * kUmmaBN;
          for (int c = 0; c < nkc && ok; ++c) {
            const int i = g * nkc + c, slot = i % NSLOT;
            ok = umma::mbar_wait(full + slot, (i / NSLOT) & 1, abort_flag);
            umma::tc_fence_after();
            const uint32_t a0 = umma::smem_u32(sA + ((size_t)ab * nkc + c) * BLK);
            const uint32_t b0 = umma::smem_u32(sR + (size_t)slot * BLK);
#pragma unroll
            for (int kk = 0; kk < kUmmaBK / 16; ++kk)
              umma::mma_bf16(dtm, umma::sw128_desc(a0 + kk * 32), umma::sw128_desc(b0 + kk * 32), idesc,
                             (c | kk) != 0);
            umma::mma_commit(empty + slot);
          }
          umma::mma_commit(accf + buf);
        }
        umma::mma_commit(aempty + ab);   // the block's A buffer is free once these MMAs are done
      }
      // the last blocks' "A free" arrivals land before the CTA leaves
      for (int bi = (nblk > 2 ? nblk - 2 : 0); bi < nblk && ok; ++bi)
        ok = umma::mbar_wait(aempty + (bi & 1), (bi >> 1) & 1, abort_flag);
    }
  } else {
    if (lane == 0) {
      // ---- weight blocks of every tile of every block, ring of NSLOT buffers
      const int total = nblk * nt * nkc;
      for (int i = 0; i < total && ok; ++i) {
        const int slot = i % NSLOT;
        if (i >= NSLOT) ok = umma::mbar_wait(empty + slot, ((i - NSLOT) / NSLOT) & 1, abort_flag);
        const int c = i % nkc, tl = (i / nkc) % nt;
        umma::mbar_arrive_expect_tx(full + slot, BLK);
        umma::bulk_g2s(sR + (size_t)slot * BLK, Wpk + ((size_t)tl * nkc + c) * BLK, BLK, full + slot);
      }
    }
  }
  if (!ok) {
    *abort_flag = 1;
    atomicOr(status, kStatusMmaTimeout);
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, 2 * kUmmaBN);
}

}  // namespace atomenc
