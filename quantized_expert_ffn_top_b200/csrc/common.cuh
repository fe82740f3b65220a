// Shared device helpers of the B200 MoE layer: status word, bf16 bits, the
// e2m1 / e4m3 / e8m0 codecs on top of the sm_100a conversion instructions,
// and the block quantisers the layer applies to activations.
//
// Formats: e2m1 and e8m0 per the OCP Microscaling Formats (MX) v1.0
// specification, e4m3 per the OCP 8-bit floating point specification; NVFP4
// (e2m1 + e4m3 scale per 16 + fp32 global scale) and MXFP4 (e2m1 + e8m0 scale
// per 32) as named by the FreeToken upstream README ("About").  Every
// quantisation decision is an fp32 operation with round-to-nearest-even,
// spelled out with the _rn intrinsics so that no contraction or fast-math
// rewrite can change a code.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

constexpr int kWarp = 32;

// ----------------------------------------------------------- status word --
// The first 4 bytes of every workspace.  0 = OK, otherwise a moe_status.
// Programmatic dependent launch (sm_90 and later).  A kernel launched with
// the programmatic-serialisation attribute may start while the kernel before
// it in the stream is still running; pdl_wait() returns once that kernel (and
// so every earlier one) has completed and its memory is visible, so it comes
// before the first read of anything they wrote.  pdl_trigger() lets the next
// kernel start launching.  Both are no-ops for a kernel launched without the
// attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void raise_status(int32_t* st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

// ------------------------------------------------------------------ bf16 --
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  uint16_t r;
  asm("{ .reg .b16 t; cvt.rn.bf16.f32 t, %1; mov.b16 %0, t; }" : "=h"(r) : "f"(f));
  return r;
}

// ------------------------------------------------------------------ codecs --
// Two fp32 values -> one byte of e2m1 codes (lo in bits 3..0, hi in 7..4),
// round to nearest even, saturating.  The instruction puts its first source
// operand in the upper nibble.
__device__ __forceinline__ uint32_t e2m1x2_encode(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 b0, b1, b2, b3; cvt.rn.satfinite.e2m1x2.f32 b0, %1, %2; mov.b32 %0, {b0, b1, b2, b3}; }"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// Two fp32 values -> two e4m3 codes (lo in bits 7..0), RNE, saturating.
__device__ __forceinline__ uint32_t e4m3x2_encode(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}

__device__ __forceinline__ uint32_t e4m3_encode(float v) { return e4m3x2_encode(v, 0.0f) & 0xFFu; }

// e4m3 code -> fp32 (exact: every e4m3 value is an fp16 value).
__device__ __forceinline__ float e4m3_decode(uint32_t code) {
  uint32_t h2;
  uint16_t c = (uint16_t)(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  uint16_t lo = (uint16_t)(h2 & 0xFFFFu);
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(lo));
  return f;
}

// Byte of two e2m1 codes -> two fp32 values (exact).
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t byte) {
  uint32_t h2;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(h2) : "r"(byte & 0xFFu));
  float lo, hi;
  uint16_t l = (uint16_t)(h2 & 0xFFFFu), h = (uint16_t)(h2 >> 16);
  asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(l));
  asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(h));
  return make_float2(lo, hi);
}

// e8m0 code -> 2^(c-127) (c = 0 is the subnormal 2^-127; 255 is not a scale
// the quantisers produce).
__device__ __forceinline__ float e8m0_decode(uint32_t c) {
  c &= 0xFFu;
  return c == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(c << 23);
}

// ------------------------------------------------------------- scales ----
// Tensor scale from an amax: NVFP4 g = amax / (448 * 6), FP8 s = amax / 448,
// 1 when the amax is 0.
__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}
__device__ __forceinline__ float fp8_tensor_scale(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// NVFP4 block: scale code sc = e4m3(bmax / (6 g)) and the element multiplier
// r = 1 / (dec(sc) g); r = 0 marks an all-zero block.
__device__ __forceinline__ uint32_t nvfp4_scale_code(float bmax, float g) {
  return e4m3_encode(__fdiv_rn(bmax, __fmul_rn(6.0f, g)));
}
__device__ __forceinline__ float nvfp4_multiplier(uint32_t sc, float g) {
  const float dec = e4m3_decode(sc);
  return dec != 0.0f ? __frcp_rn(__fmul_rn(dec, g)) : 0.0f;
}
__device__ __forceinline__ void nvfp4_block_scale(float bmax, float g, uint32_t& sc, float& r) {
  sc = nvfp4_scale_code(bmax, g);
  r = nvfp4_multiplier(sc, g);
}

// SiLU(x) = x / (1 + e^-x) = (x/2)(1 + tanh(x/2)), with the hardware tanh
// approximation (relative error about 2^-11, far below one e2m1 step).
__device__ __forceinline__ float silu_fast(float x) {
  const float hx = 0.5f * x;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hx));
  return fmaf(hx, t, hx);
}

// MXFP4 block (OCP MX v1.0 conversion): c = clamp(floor(log2 bmax) - 2 + 127,
// 0, 254), 0 for a zero or subnormal maximum; multiplier 2^(127 - c).
__device__ __forceinline__ void mxfp4_block_scale(float bmax, uint32_t& c, float& inv) {
  const int be = (int)((__float_as_uint(bmax) >> 23) & 0xFFu);   // biased exponent
  int cc = be == 0 ? 0 : be - 2;
  cc = cc < 0 ? 0 : (cc > 254 ? 254 : cc);
  c = (uint32_t)cc;
  inv = __uint_as_float((uint32_t)(254 - cc) << 23);              // 2^(127-c), c <= 252 here
}

// 16 values -> 8 bytes of NVFP4 codes (uint2), given the multiplier r.
__device__ __forceinline__ uint2 nvfp4_encode16(const float* v, float r) {
  uint32_t w[2] = {0u, 0u};
  if (r != 0.0f) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i >> 2] |= e2m1x2_encode(__fmul_rn(v[2 * i], r), __fmul_rn(v[2 * i + 1], r)) << (8 * (i & 3));
  }
  return make_uint2(w[0], w[1]);
}

// n values (n % 8 == 0) -> n/2 bytes of e2m1 codes with an exact multiplier.
__device__ __forceinline__ uint32_t e2m1_encode8(const float* v, float m) {
  uint32_t w = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) w |= e2m1x2_encode(__fmul_rn(v[2 * i], m), __fmul_rn(v[2 * i + 1], m)) << (8 * i);
  return w;
}

// ------------------------------------------------------ small utilities --
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Non-negative float max through integer atomics (bit order = value order).
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
  atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
}

// Index of the expert segment containing position p: offsets is [E+1],
// non-decreasing, offsets[0] = 0.
__device__ __forceinline__ int segment_of(const int32_t* offsets, int E, int p) {
  int lo = 0, hi = E;  // invariant: offsets[lo] <= p < offsets[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(offsets + mid) <= p) lo = mid; else hi = mid;
  }
  return lo;
}

}  // namespace moe
