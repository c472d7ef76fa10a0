// Activation-quantization arithmetic shared by the quantization kernels and
// the fused quantize + GEMM kernel, so that both produce the same codes and
// scales bit for bit:
//
//   s = max(fp32(amax / Q), 2^-126),   q = encode(fp32(x / s))
//
// Q = 448 (e4m3: round to nearest even, saturating) or 127 (int8: round half
// to even, clamped to +-127); both divisions are correctly rounded (the
// scale by __fdiv_rn, x / s as described at Divisor below).  (Formats:
// PyTorch blog "Building a High-Performance and Portable vLLM Linear Backend
// with Helion", "Helion Linear Backend > Scope".)
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cfloat>
#include <cstdint>

namespace lq {

constexpr float kE4m3Max = 448.0f;
constexpr float kInt8Max = 127.0f;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float amax8(const float (&f)[8]) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
  return a;
}

__device__ __forceinline__ float scale_from_amax(float amax, float qmax) {
  return fmaxf(__fdiv_rn(amax, qmax), FLT_MIN);
}

// Division by a row's scale s, correctly rounded (fp32(x / s) decides the
// code).  With y = RN(1/s), q0 = RN(x y), r = x - s q0 (exact in one FMA) and
// q1 = RN(q0 + r y), q1 = RN(x / s) when nothing underflows: Markstein's
// correction (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990); when r = 0, q0
// is already exact and is kept (so x = -0 gives -0).  Two roundings and one
// reciprocal per row instead of a full division per element; checked bit for
// bit on the host against IEEE division for every bf16 significand of x
// (and +-0, subnormal x) and every fp32 significand of s.  Rows with amax >= 2^-80 (finite) take it: an x
// there with |x| < 2^-103, where r could lose bits, has |x / s| < 2^-14 and
// gets the code 0 either way; other rows (all zero, tiny, inf or NaN) divide.
struct Divisor {
  float s;
  float y;   // RN(1 / s), or 0: divide
};

__device__ __forceinline__ Divisor make_divisor(float amax, float s) {
  const bool fast = amax >= 0x1p-80f && amax <= FLT_MAX;
  return Divisor{s, fast ? __frcp_rn(s) : 0.f};
}

// q[i] = RN(f[i] / s) for 8 values.  The test of the row's path is made
// once per 8 values: with the division's code inside the per-value loop the
// compiler cannot interleave the 8 independent corrections.
__device__ __forceinline__ void quotient8(const float (&f)[8], const Divisor& d, float (&q)[8]) {
  if (d.y != 0.f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float q0 = __fmul_rn(f[i], d.y);
      const float r = __fmaf_rn(-d.s, q0, f[i]);
      // r = 0: q0 is exact (and keeps the sign of x = -0, which the FMA would not)
      q[i] = r == 0.f ? q0 : __fmaf_rn(r, d.y, q0);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], d.s);
  }
}

// 8 values -> 8 e4m3 bytes (lowest address first).
__device__ __forceinline__ uint2 encode8_e4m3(const float (&f)[8], const Divisor& d) {
  float q[8];
  quotient8(f, d, q);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = static_cast<uint32_t>(
        __nv_cvt_float2_to_fp8x2(make_float2(q[2 * i], q[2 * i + 1]), __NV_SATFINITE, __NV_E4M3));
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// 8 values -> 8 int8 bytes.
__device__ __forceinline__ uint2 encode8_int8(const float (&f)[8], const Divisor& d) {
  float q[8];
  quotient8(f, d, q);
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int v = __float2int_rn(q[i]);
    v = v > 127 ? 127 : (v < -127 ? -127 : v);
    b[i] = static_cast<uint32_t>(v) & 0xFFu;
  }
  return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                    b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}

}  // namespace lq
