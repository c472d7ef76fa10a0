// Producer-side fused quantizers: the kernel that makes a GEMM's activations
// (RMSNorm, or SiLU-and-multiply of the gate/up projection) quantizes them in
// the same pass, per token (FP8 e4m3 or INT8) or per 1 x 128 group (FP8).
// Kernels rms_norm_dynamic_per_token_quant, rms_norm_per_block_quant,
// silu_and_mul_dynamic_per_token_quant and silu_and_mul_per_block_quant of
// the 24-ai.news report "HelionがvLLMに統合：PyTorchネイティブDSLがCUDAカーネルを
// 代替し、Qwen3モデルのFP8推論を高速化", section "vLLMに統合されたカーネル".
//
// The bf16 value y that is quantized, with every rounding written out:
//
//   RMSNorm:  h = bf16(fp32(x + residual)) (the new residual; h = x without one)
//             v = sum(h^2) / K + eps in fp64;  r = fp32(1 / sqrt(v)) (fp64 ops)
//             y = bf16(fp32(bf16(fp32(h r)) w))
//   SiLU-mul: y = bf16(fp32(bf16(g / (1 + exp(-g))) u)), the silu rounded once
//             from its exact value
//
// then s = max(fp32(amax / Q), 2^-126) and q = encode(fp32(y / s)) over the
// row or the group, as in quant_common.cuh.
//
// One CTA of 256 threads per row; the row stays in registers (8 values per
// 16-byte chunk, up to 16 chunks per thread: rows of up to 32768 outputs).
// HBM / latency bound: the row is read once and the codes written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cfloat>
#include <cstdint>

#include "lq_kernels.h"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace lq {
namespace {

constexpr int kRowThreads = 256;

__device__ __forceinline__ float bf(uint32_t w, int hi) {
  return __uint_as_float(hi ? (w & 0xFFFF0000u) : (w << 16));
}

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

// silu(g) rounded once to bf16.  The fp32 evaluation g / (1 + expf(-g)) is
// within 8 fp32 units in the last place of the exact value (expf: at most 2
// ulp; the add and the divide: half an ulp each).  Unless the fp32 result is
// that close to a midpoint between two bf16 values (its low 16 bits within 64
// of 0x8000), rounding it gives the rounding of the exact value (Ziv's
// rounding test).  Otherwise, and where expf could overflow or the result
// leave the fp32 normal range (g <= -80), the value is recomputed in fp64.
__device__ __forceinline__ __nv_bfloat16 silu_bf16(float g) {
  if (g > -80.f) {
    const float s = __fdiv_rn(g, __fadd_rn(1.f, expf(-g)));
    const uint32_t low = __float_as_uint(s) & 0xFFFFu;
    const uint32_t dist = low > 0x8000u ? low - 0x8000u : 0x8000u - low;
    if (dist > 64u && fabsf(s) >= 0x1p-100f) return __float2bfloat16_rn(s);
    if (s == 0.f) return __float2bfloat16_rn(s);   // g = +-0
  }
  const double gd = static_cast<double>(g);
  return __double2bfloat16(__ddiv_rn(gd, __dadd_rn(1.0, exp(-gd))));
}

template <int kThreads>
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kThreads / 32 ? red[lane] : 0.0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  const double t = red[0];
  __syncthreads();   // red is reused by the next reduction
  return t;
}

template <int kThreads>
__device__ __forceinline__ float block_max_f32(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kThreads / 32 ? red[lane] : 0.f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

enum : int { kOpRmsNorm = 0, kOpSiluMul = 1 };

// GROUP = 0: one scale per row (FP8 or INT8); GROUP = 128: one FP8 scale per
// 128 outputs (16 consecutive chunks, held by 16 consecutive threads).
template <int OP, int GROUP, bool kInt8, int VPT>
__global__ void __launch_bounds__(kRowThreads) producer_quant_kernel(const __nv_bfloat16* __restrict__ in,
                                                                     __nv_bfloat16* __restrict__ residual,
                                                                     const __nv_bfloat16* __restrict__ weight,
                                                                     float eps, uint8_t* __restrict__ q,
                                                                     float* __restrict__ scales, int64_t Kout) {
  static_assert(GROUP == 0 || !kInt8, "1 x 128 groups are FP8");
  __shared__ double red_d[kRowThreads / 32];
  __shared__ float red_f[kRowThreads / 32];
  grid_launch_dependents();   // as the other quantization kernels: before the wait
  grid_dependency_wait();
  const int64_t row = blockIdx.x;
  const int nvec = static_cast<int>(Kout / 8);
  uint4 y[VPT];

  if constexpr (OP == kOpRmsNorm) {
    const uint4* xr = reinterpret_cast<const uint4*>(in + row * Kout);
    uint4* rr = residual ? reinterpret_cast<uint4*>(residual + row * Kout) : nullptr;
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;
      y[i] = make_uint4(0u, 0u, 0u, 0u);
      if (idx < nvec) {
        uint4 h = __ldg(xr + idx);
        if (rr) {
          const uint4 rv = rr[idx];
          const uint32_t xw[4] = {h.x, h.y, h.z, h.w}, rw[4] = {rv.x, rv.y, rv.z, rv.w};
          uint32_t hw[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            hw[j] = pack_bf16x2(__float2bfloat16_rn(__fadd_rn(bf(xw[j], 0), bf(rw[j], 0))),
                                __float2bfloat16_rn(__fadd_rn(bf(xw[j], 1), bf(rw[j], 1))));
          h = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          rr[idx] = h;
        }
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const double d = static_cast<double>(bf(hw[j >> 1], j & 1));
          ss = __fma_rn(d, d, ss);   // d * d is exact (8-bit significands)
        }
        y[i] = h;
      }
    }
    const double total = block_sum_f64<kRowThreads>(ss, red_d);
    const double v = __dadd_rn(__ddiv_rn(total, static_cast<double>(Kout)), static_cast<double>(eps));
    const float r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(v)));
    const uint4* wr = reinterpret_cast<const uint4*>(weight);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;
      if (idx < nvec) {
        const uint4 wv = __ldg(wr + idx);
        const uint32_t hw[4] = {y[i].x, y[i].y, y[i].z, y[i].w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __nv_bfloat16 o[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const __nv_bfloat16 n = __float2bfloat16_rn(__fmul_rn(bf(hw[j], k), r));
            o[k] = __float2bfloat16_rn(__fmul_rn(__bfloat162float(n), bf(ww[j], k)));
          }
          out[j] = pack_bf16x2(o[0], o[1]);
        }
        y[i] = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
  } else {
    const uint4* gr = reinterpret_cast<const uint4*>(in + row * 2 * Kout);
    const uint4* ur = gr + nvec;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;
      y[i] = make_uint4(0u, 0u, 0u, 0u);
      if (idx < nvec) {
        const uint4 gv = __ldg(gr + idx), uv = __ldg(ur + idx);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __nv_bfloat16 o[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const __nv_bfloat16 a = silu_bf16(bf(gw[j], k));
            o[k] = __float2bfloat16_rn(__fmul_rn(__bfloat162float(a), bf(uw[j], k)));   // exact product
          }
          out[j] = pack_bf16x2(o[0], o[1]);
        }
        y[i] = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
  }

  // ---------------------------------------------------------------- quantize
  const float qmax = kInt8 ? kInt8Max : kE4m3Max;
  uint2* qr = reinterpret_cast<uint2*>(q + row * Kout);
  if constexpr (GROUP == 0) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      float f[8];
      bf16x8_to_f32(y[i], f);
      a = fmaxf(a, amax8(f));   // chunks past the row are zero
    }
    const float amax = block_max_f32<kRowThreads>(a, red_f);
    const float s = scale_from_amax(amax, qmax);
    const Divisor d = make_divisor(amax, s);
    if (threadIdx.x == 0) scales[row] = s;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;
      if (idx < nvec) {
        float f[8];
        bf16x8_to_f32(y[i], f);
        qr[idx] = kInt8 ? encode8_int8(f, d) : encode8_e4m3(f, d);
      }
    }
  } else {
    const int64_t groups = Kout / 128;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;   // 16 threads share idx / 16 (256 % 16 == 0)
      float f[8];
      bf16x8_to_f32(y[i], f);
      float a = amax8(f);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (idx < nvec) {
        const float s = scale_from_amax(a, qmax);
        if ((idx & 15) == 0) scales[row * groups + idx / 16] = s;
        qr[idx] = encode8_e4m3(f, make_divisor(a, s));
      }
    }
  }
}

cudaLaunchConfig_t row_config(int64_t M, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  cfg.blockDim = dim3(kRowThreads);
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int OP, int GROUP, bool kInt8>
cudaError_t launch_rows(const void* in, void* residual, const void* weight, float eps, void* q, float* scales,
                        int64_t M, int64_t Kout, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = row_config(M, stream, attr);
  const auto* ip = static_cast<const __nv_bfloat16*>(in);
  auto* rp = static_cast<__nv_bfloat16*>(residual);
  const auto* wp = static_cast<const __nv_bfloat16*>(weight);
  auto* qp = static_cast<uint8_t*>(q);
  const int64_t nvec = Kout / 8;
#define LQ_PROW(V) \
  if (nvec <= kRowThreads * (V)) \
    return cudaLaunchKernelEx(&cfg, producer_quant_kernel<OP, GROUP, kInt8, V>, ip, rp, wp, eps, qp, scales, Kout);
  LQ_PROW(1)
  LQ_PROW(2)
  LQ_PROW(4)
  LQ_PROW(8)
  LQ_PROW(16)
#undef LQ_PROW
  return cudaErrorInvalidValue;
}

}  // namespace

int64_t producer_max_row() { return static_cast<int64_t>(kRowThreads) * 16 * 8; }

cudaError_t launch_rms_norm_quant(int fmt, bool per_block, const void* x, void* residual, const void* weight,
                                  float eps, void* q, float* scales, int64_t M, int64_t K, cudaStream_t stream) {
  if (per_block) return launch_rows<kOpRmsNorm, 128, false>(x, residual, weight, eps, q, scales, M, K, stream);
  if (fmt == kFmtInt8) return launch_rows<kOpRmsNorm, 0, true>(x, residual, weight, eps, q, scales, M, K, stream);
  return launch_rows<kOpRmsNorm, 0, false>(x, residual, weight, eps, q, scales, M, K, stream);
}

cudaError_t launch_silu_mul_quant(int fmt, bool per_block, const void* gate_up, void* q, float* scales, int64_t M,
                                  int64_t I, cudaStream_t stream) {
  if (per_block) return launch_rows<kOpSiluMul, 128, false>(gate_up, nullptr, nullptr, 0.f, q, scales, M, I, stream);
  if (fmt == kFmtInt8) return launch_rows<kOpSiluMul, 0, true>(gate_up, nullptr, nullptr, 0.f, q, scales, M, I, stream);
  return launch_rows<kOpSiluMul, 0, false>(gate_up, nullptr, nullptr, 0.f, q, scales, M, I, stream);
}

}  // namespace lq
