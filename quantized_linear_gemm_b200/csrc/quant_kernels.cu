// Dynamic activation quantizers and the offline weight quantizer.
//
// Rule (formats of the PyTorch blog "Building a High-Performance and Portable
// vLLM Linear Backend with Helion", "Helion Linear Backend > Scope"; kernels
// dynamic_per_token_scaled_fp8_quant and per_token_group_fp8_quant of the
// 24-ai.news report, "kernels integrated into vLLM"):
//
//   s = max(fp32(amax / Q), 2^-126),   q = encode(fp32(x / s))
//
// with Q = 448 (e4m3, round to nearest even, saturating) or 127 (int8,
// round half to even, clamped to +-127).  x / s is the correctly rounded
// quotient (quant_common.cuh: reciprocal plus one FMA correction, or a
// division), so codes and scales are reproducible bit for bit.
//
// These kernels are bandwidth / launch bound: each reads bf16 once per pass
// with 16-byte loads and writes 8-byte code chunks.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cfloat>
#include <cstdint>

#include "lq_kernels.h"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace lq {

// Programmatic dependent launch: every kernel here lets the next kernel on the
// stream launch before it waits for its own predecessor.
// The next kernel (normally the GEMM that reads these codes) can then become
// resident and start streaming its weights while this kernel's predecessor
// finishes; its griddepcontrol.wait still waits for this whole grid, which
// completes only after its own predecessor did.  A dependent grid launches
// only once every CTA of this grid has triggered, so it never takes the
// place of a CTA of this grid that has not started.
namespace {

template <int kThreadsPerRow>
__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kThreadsPerRow / 32 ? red[lane] : 0.f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// One CTA per row, the row held in registers (VPT 16-byte vectors per
// thread): one global read, a block-wide amax, then quantization.
template <bool kInt8, int VPT>
__global__ void __launch_bounds__(256) quant_per_token_reg_kernel(const __nv_bfloat16* __restrict__ x,
                                                                   uint8_t* __restrict__ q,
                                                                   float* __restrict__ scales, int64_t K) {
  __shared__ float red[32];
  grid_launch_dependents();   // before the wait: see the note at the top of the namespace
  grid_dependency_wait();
  const int64_t row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * K);
  const int nvec = static_cast<int>(K / 8);
  uint4 v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * 256;
    v[i] = idx < nvec ? __ldg(xr + idx) : make_uint4(0u, 0u, 0u, 0u);
  }
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    float f[8];
    bf16x8_to_f32(v[i], f);
    a = fmaxf(a, amax8(f));
  }
  const float amax = block_max<256>(a, red);
  const float s = scale_from_amax(amax, kInt8 ? kInt8Max : kE4m3Max);
  const Divisor d = make_divisor(amax, s);
  if (threadIdx.x == 0) scales[row] = s;
  uint2* qr = reinterpret_cast<uint2*>(q + row * K);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * 256;
    if (idx < nvec) {
      float f[8];
      bf16x8_to_f32(v[i], f);
      qr[idx] = kInt8 ? encode8_int8(f, d) : encode8_e4m3(f, d);
    }
  }
}

// One CTA per row.  Two passes over the row (the second hits L1/L2); used
// for rows longer than the register-resident kernel holds.
template <bool kInt8>
__global__ void __launch_bounds__(256) quant_per_token_kernel(const __nv_bfloat16* __restrict__ x,
                                                               uint8_t* __restrict__ q, float* __restrict__ scales,
                                                               int64_t K) {
  __shared__ float red[32];
  grid_launch_dependents();   // before the wait: see the note at the top of the namespace
  grid_dependency_wait();
  const int64_t row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * K);
  const int64_t nvec = K / 8;
  float a = 0.f;
  for (int64_t i = threadIdx.x; i < nvec; i += blockDim.x) {
    float f[8];
    bf16x8_to_f32(__ldg(xr + i), f);
    a = fmaxf(a, amax8(f));
  }
  const float amax = block_max<256>(a, red);
  const float s = scale_from_amax(amax, kInt8 ? kInt8Max : kE4m3Max);
  const Divisor d = make_divisor(amax, s);
  if (threadIdx.x == 0) scales[row] = s;
  uint2* qr = reinterpret_cast<uint2*>(q + row * K);
  for (int64_t i = threadIdx.x; i < nvec; i += blockDim.x) {
    float f[8];
    bf16x8_to_f32(__ldg(xr + i), f);
    qr[i] = kInt8 ? encode8_int8(f, d) : encode8_e4m3(f, d);
  }
}

// UE8M0 scale of a group: the smallest power of two 2^e with amax <= 448 2^e,
// e clamped to [-127, 127], decided exactly on the bits of amax (448 =
// 1.75 2^8): for amax = m 2^E (m in [1, 2)), e = E - 8, plus one when
// m > 1.75.  Zero and subnormal amax give e = -127 (byte 0).
__device__ __forceinline__ int ue8m0_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int biased = static_cast<int>(bits >> 23);
  if (biased == 0) return -127;
  const int e = (biased - 127) - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : e;
}

// 2^-e as a float; for e in [-127, 120] (finite amax) a normal number.
__device__ __forceinline__ float pow2_neg(int e) { return __uint_as_float(static_cast<uint32_t>(127 - e) << 23); }

// 8 values times 2^-e (exact) -> 8 e4m3 bytes.
__device__ __forceinline__ uint2 encode8_e4m3_pow2(const float (&f)[8], int e) {
  const float r = pow2_neg(e);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f[2 * i], r), __fmul_rn(f[2 * i + 1], r)),
                                                          __NV_SATFINITE, __NV_E4M3));
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// 16 threads per 128-element group, 8 elements each; 16 groups per CTA.
// kE8m0: UE8M0 scale bytes (power-of-two scales) instead of fp32 scales.
template <bool kE8m0>
__global__ void __launch_bounds__(256) quant_group128_kernel(const __nv_bfloat16* __restrict__ x,
                                                              uint8_t* __restrict__ q, void* __restrict__ scales,
                                                              int64_t M, int64_t K) {
  grid_launch_dependents();   // before the wait: see the note at the top of the namespace
  grid_dependency_wait();
  const int64_t KB = K / 128;
  const int64_t g = blockIdx.x * 16ll + (threadIdx.x >> 4);
  const int sub = threadIdx.x & 15;
  const bool valid = g < M * KB;
  const int64_t row = valid ? g / KB : 0;
  const int64_t kb = valid ? g - row * KB : 0;
  const int64_t off = row * K + kb * 128 + sub * 8;
  float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (valid) bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(x + off)), f);
  float a = amax8(f);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));   // within 16 lanes
  if constexpr (kE8m0) {
    const int e = ue8m0_exponent(a);
    if (valid) {
      if (sub == 0) static_cast<uint8_t*>(scales)[row * KB + kb] = static_cast<uint8_t>(e + 127);
      *reinterpret_cast<uint2*>(q + off) = encode8_e4m3_pow2(f, e);
    }
  } else {
    const float s = scale_from_amax(a, kE4m3Max);
    if (valid) {
      if (sub == 0) static_cast<float*>(scales)[row * KB + kb] = s;
      *reinterpret_cast<uint2*>(q + off) = encode8_e4m3(f, make_divisor(a, s));
    }
  }
}

// One CTA per 128x128 block of W[N, K]; thread t covers row t/2, 64 columns.
template <bool kE8m0>
__global__ void __launch_bounds__(256) quant_weight_block128_kernel(const __nv_bfloat16* __restrict__ w,
                                                                     uint8_t* __restrict__ q,
                                                                     void* __restrict__ scales, int64_t K) {
  __shared__ float red[32];
  const int64_t KB = K / 128;
  const int64_t nb = blockIdx.y, kb = blockIdx.x;
  const int64_t row = nb * 128 + (threadIdx.x >> 1);
  const int64_t col = kb * 128 + (threadIdx.x & 1) * 64;
  const uint4* src = reinterpret_cast<const uint4*>(w + row * K + col);
  float f[8][8];
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    bf16x8_to_f32(__ldg(src + i), f[i]);
    a = fmaxf(a, amax8(f[i]));
  }
  const float amax = block_max<256>(a, red);
  uint2* dst = reinterpret_cast<uint2*>(q + row * K + col);
  if constexpr (kE8m0) {
    const int e = ue8m0_exponent(amax);
    if (threadIdx.x == 0) static_cast<uint8_t*>(scales)[nb * KB + kb] = static_cast<uint8_t>(e + 127);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = encode8_e4m3_pow2(f[i], e);
  } else {
    const float s = scale_from_amax(amax, kE4m3Max);
    const Divisor d = make_divisor(amax, s);
    if (threadIdx.x == 0) static_cast<float*>(scales)[nb * KB + kb] = s;
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = encode8_e4m3(f[i], d);
  }
}

__global__ void fill_zero_bf16_kernel(__nv_bfloat16* __restrict__ C, int64_t count) {
  grid_launch_dependents();   // before the wait: see the note at the top of the namespace
  grid_dependency_wait();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    C[i] = __float2bfloat16_rn(0.f);
}

cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

}  // namespace

cudaError_t launch_quant_per_token(int fmt, const void* x, void* q, float* scales, int64_t M, int64_t K,
                                   cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(static_cast<unsigned>(M)), dim3(256), stream, attr);
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  auto* qp = static_cast<uint8_t*>(q);
  const bool i8 = fmt == kFmtInt8;
  const int64_t nvec = K / 8;
#define LQ_QROW(V)                                                                                     \
  if (nvec <= 256 * (V))                                                                               \
    return i8 ? cudaLaunchKernelEx(&cfg, quant_per_token_reg_kernel<true, V>, xp, qp, scales, K)       \
              : cudaLaunchKernelEx(&cfg, quant_per_token_reg_kernel<false, V>, xp, qp, scales, K);
  LQ_QROW(1)
  LQ_QROW(2)
  LQ_QROW(4)
  LQ_QROW(8)
  LQ_QROW(16)
#undef LQ_QROW
  if (i8) return cudaLaunchKernelEx(&cfg, quant_per_token_kernel<true>, xp, qp, scales, K);
  return cudaLaunchKernelEx(&cfg, quant_per_token_kernel<false>, xp, qp, scales, K);
}

cudaError_t launch_quant_group128(const void* x, void* q, void* scales, int64_t M, int64_t K, bool e8m0,
                                  cudaStream_t stream) {
  const int64_t groups = M * (K / 128);
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(static_cast<unsigned>((groups + 15) / 16)), dim3(256), stream, attr);
  if (e8m0)
    return cudaLaunchKernelEx(&cfg, quant_group128_kernel<true>, static_cast<const __nv_bfloat16*>(x),
                              static_cast<uint8_t*>(q), scales, M, K);
  return cudaLaunchKernelEx(&cfg, quant_group128_kernel<false>, static_cast<const __nv_bfloat16*>(x),
                            static_cast<uint8_t*>(q), scales, M, K);
}

cudaError_t launch_quant_weight_block128(const void* w, void* q, void* scales, int64_t N, int64_t K, bool e8m0,
                                         cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(K / 128), static_cast<unsigned>(N / 128));
  if (e8m0)
    quant_weight_block128_kernel<true><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w),
                                                                 static_cast<uint8_t*>(q), scales, K);
  else
    quant_weight_block128_kernel<false><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w),
                                                                  static_cast<uint8_t*>(q), scales, K);
  return cudaGetLastError();
}

cudaError_t launch_fill_zero_bf16(__nv_bfloat16* C, int64_t count, cudaStream_t stream) {
  int64_t blocks = (count + 255) / 256;
  if (blocks > 148 * 4) blocks = 148 * 4;
  if (blocks < 1) blocks = 1;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(static_cast<unsigned>(blocks)), dim3(256), stream, attr);
  return cudaLaunchKernelEx(&cfg, fill_zero_bf16_kernel, C, count);
}

}  // namespace lq
