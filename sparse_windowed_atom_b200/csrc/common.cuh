// common.cuh -- device helpers shared by the atomenc kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace atomenc {

constexpr int kWarp = 32;

// ---- element access: every float tensor is float32 or bf16 in memory, float32 in math
// Programmatic dependent launch. Every kernel of a forward pass is launched so that it
// may be scheduled while its predecessor in the stream is still running. Its first act
// is to wait until that predecessor grid has completed and its writes are visible
// (before any global or tensor memory is touched, so chains of such kernels stay in
// stream order); then it lets its own successor begin launching.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_launch_next();
}
// A kernel may read before pdl_wait() what the kernels two or more places earlier in the
// stream wrote: its predecessor only launches it after passing its own pdl_wait(), so
// those kernels have completed and their writes are visible. The caller's inputs count
// as such (the first kernel of a pass waits for everything before it). Writes, and reads
// of the immediate predecessor's results, come after pdl_wait().

__device__ __forceinline__ float ldf(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void stf(float *p, int64_t i, float v) { p[i] = v; }
// two floats rounded to nearest-even bf16 by one packed conversion; lo in bits 0-15
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  uint32_t u;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(hi), "f"(lo));
  return u;
}
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

// ---- activations (no fast-math: IEEE division, expf, subnormals kept)
// sigmoid(z) = 1 / (1 + e^-z); for z < 0 the same value as e^z / (1 + e^z) so that a
// representable subnormal tail is not flushed by an overflowing e^-z.
__device__ __forceinline__ float sigmoidf_(float z) {
  if (z >= 0.f) return 1.f / (1.f + expf(-z));
  float e = expf(z);
  return e / (1.f + e);
}
__device__ __forceinline__ float siluf_(float z) { return z * sigmoidf_(z); }

// The same sigmoid on the special-function unit: e = 2^(-|z| log2 e) = e^-|z| with the
// hardware exp2, one hardware reciprocal; z >= 0 -> 1 / (1 + e), z < 0 -> e / (1 + e).
// About 3e-7 relative error; the exp2 keeps subnormal results.
__device__ __forceinline__ float sigmoid_fast(float z) {
  float e, r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(e) : "f"(-fabsf(z) * 1.4426950408889634f));
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
  return z >= 0.f ? r : e * r;
}
__device__ __forceinline__ float silu_fast(float z) { return z * sigmoid_fast(z); }

// Two floats packed in one 64-bit register, and the sm_100 packed FMA on them.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 ffma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 pack2(float x, float y) {
  f32x2 d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(x), "f"(y));
  return d;
}
__device__ __forceinline__ float2 unpack2(f32x2 v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}

// c + a.lo * b.lo + a.hi * b.hi for two pairs of bf16 values (each product is exact in
// float32; two float32-accumulating fused multiply-adds with bf16 sources)
__device__ __forceinline__ float fma_bf16x2(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %3;\n\tfma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "=f"(d)
      : "r"(a), "r"(b), "f"(c));
  return d;
}
// a0 += w * v.lo, a1 += w * v.hi with w and v bf16 (float32 accumulation)
__device__ __forceinline__ void axpy_bf16x2(uint16_t w, uint32_t v, float &a0, float &a1) {
  asm("{\n\t.reg .b16 vl, vh;\n\tmov.b32 {vl, vh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, %3, vl, %0;\n\tfma.rn.f32.bf16 %1, %3, vh, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(v), "h"(w));
}

// ---- warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// usable iff valid, 0 <= atom_to_token < T and the mapped token is valid
__device__ __forceinline__ bool atom_usable(const uint8_t *valid, const int64_t *att,
                                            const uint8_t *token_valid, int64_t b,
                                            int64_t a, int64_t A, int64_t T) {
  int64_t i = b * A + a;
  int64_t t = att[i];
  return valid[i] != 0 && t >= 0 && t < T && token_valid[b * T + t] != 0;
}

}  // namespace atomenc
