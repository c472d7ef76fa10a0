// Activation-quantization arithmetic shared by the quantization kernels and
// the fused quantize + GEMM kernel, so that both produce the same codes and
// scales bit for bit:
//
//   s = max(fp32(amax / Q), 2^-126),   q = encode(fp32(x / s))
//
// Q = 448 (e4m3: round to nearest even, saturating) or 127 (int8: round half
// to even, clamped to +-127); the divisions are the correctly rounded
// __fdiv_rn.  (Formats: PyTorch blog "Building a High-Performance and
// Portable vLLM Linear Backend with Helion", "Helion Linear Backend > Scope".)
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

// 8 values -> 8 e4m3 bytes (lowest address first).
__device__ __forceinline__ uint2 encode8_e4m3(const float (&f)[8], float s) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 pr = make_float2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s));
    w[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3));
  }
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// 8 values -> 8 int8 bytes.
__device__ __forceinline__ uint2 encode8_int8(const float (&f)[8], float s) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int v = __float2int_rn(__fdiv_rn(f[i], s));
    v = v > 127 ? 127 : (v < -127 ? -127 : v);
    b[i] = static_cast<uint32_t>(v) & 0xFFu;
  }
  return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                    b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}


}  // namespace lq
