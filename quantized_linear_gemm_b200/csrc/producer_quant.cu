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
// One CTA per row; the row stays in registers (8 values per 16-byte chunk,
// at most 32768 outputs per row).  CTAs of 256 threads for short rows when
// there are many; with few rows (decode) or long rows 1024 threads share a
// row, more warps per SM to hide the latency of the arithmetic.  The row is
// read once and the codes written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cfloat>
#include <cstdint>

#include "lq_kernels.h"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace lq {
namespace {

constexpr int kMaxRow = 32768;
constexpr int kMaxStagedSmem = 200 * 1024;   // two row buffers at most

__device__ __forceinline__ float bf(uint32_t w, int hi) {
  return __uint_as_float(hi ? (w & 0xFFFF0000u) : (w << 16));
}

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

// Two fp32 values rounded to bf16 (to nearest, ties to even) by one
// conversion instruction; a in the low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return static_cast<uint32_t>(__bfloat16_as_ushort(v.x)) | (static_cast<uint32_t>(__bfloat16_as_ushort(v.y)) << 16);
}

// silu(g) rounded once to bf16, in three tiers: each returns a bf16 value
// and clears *ok where it cannot vouch for it; the next tier then recomputes.
// Every finite bf16 gate is checked against the exactly rounded value on the
// device (lq_test_silu_bf16 runs the tiers the producer kernels run).
//
// Tier 1, the hot loop's: e^-g = 2^(-g log2 e) with log2 e split as
// Lh + Ll, Lh = 47274 / 2^15: g Lh is exact in fp32 (a bf16 gate has 8
// significant bits, Lh 16), 2^(-g Lh) comes from ex2.approx, and the factor
// 2^(-g Ll) = 1 - g Ll ln2 + ... from one fma (the next term is below
// 2^-23.5 for |g| < 80).  The quotient uses the approximate reciprocal
// (__fdividef).  The estimate is then within a few units of 2^-23 of the
// exact quotient (the argument's rounding, which grows with |g| in the plain
// ex2(g log2 e), is gone), and the Ziv test keeps its rounding unless its
// low 16 bits lie within 16 of a bf16 midpoint.  Returns the fp32 estimate;
// its bf16 rounding is the result where *ok.
__device__ __forceinline__ float silu_est_ex2(float g, bool* ok) {
  float eh;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(eh) : "f"(g * -1.44268798828125f));
  const float e = __fmaf_rn(eh, g * -4.8884952e-6f, eh);   // times 2^(-g Ll), Ll ln2 = 4.8885e-6
  const float s = __fdividef(g, 1.f + e);
  const uint32_t low = __float_as_uint(s) & 0xFFFFu;
  *ok = g > -80.f && low + 16u - 0x8000u > 32u && fabsf(s) >= 0x1p-100f;
  return s;
}

// Tier 2.  The fp32 estimate g / (1 + expf(-g)) has a
// relative error of at most about 2.25 * 2^-22: expf is within 2 ulp (2^-22
// relative), the add within half an ulp, and __fdividef within 2 ulp for a
// divisor in [2^-126, 2^126] (here 1 + e^-g lies in [1, e^80]).  That is at
// most 9 ulp of the estimate.  Unless the estimate is within 32 ulp of a
// midpoint between two bf16 values (its low 16 bits within 32 of 0x8000),
// rounding it gives the rounding of the exact value (Ziv's rounding test).
// Otherwise, and where the result could leave the fp32 normal range
// (g <= -80), *ok is cleared and the caller recomputes the value with
// silu_bf16_f64, outside its hot loop.
__device__ __forceinline__ __nv_bfloat16 silu_bf16_fast(float g, bool* ok) {
  const float s = __fdividef(g, __fadd_rn(1.f, expf(-g)));
  const uint32_t low = __float_as_uint(s) & 0xFFFFu;
  const uint32_t dist = low > 0x8000u ? low - 0x8000u : 0x8000u - low;
  *ok = g > -80.f && ((dist > 32u && fabsf(s) >= 0x1p-100f) || s == 0.f);   // s = 0 only for g = +-0
  return __float2bfloat16_rn(s);
}

// silu(g) from fp64, rounded once to bf16.  Over all bf16 inputs the fp64
// quotient (within a few units of 2^-52 of the exact value) decides the
// rounding, except where it is exactly g / 2: for 0 < |g| < 2^-125, where
// 1 + e^-g rounds to 2.  For half of those gates g / 2 is a midpoint between
// two bf16 values, and the exact value lies above it (silu(g) - g / 2 =
// g (sigma(g) - 1/2) > 0 for every g != 0).  There g / 2 is rounded with a
// positive excess of |g| 2^-20, far below half a bf16 unit: the rounding of
// a value just above g / 2, like the exact one.
__device__ __forceinline__ __nv_bfloat16 silu_bf16_f64(float g) {
  const double gd = static_cast<double>(g);
  if (gd != 0.0 && fabs(gd) < 0x1p-60) return __double2bfloat16(fma(fabs(gd), 0x1p-20, gd * 0.5));
  return __double2bfloat16(__ddiv_rn(gd, __dadd_rn(1.0, exp(-gd))));
}

// Tiers 2 and 3, for a gate that tier 1 could not vouch for.
__device__ __noinline__ __nv_bfloat16 silu_bf16_slow(float g) {
  bool ok;
  const __nv_bfloat16 a = silu_bf16_fast(g, &ok);
  return ok ? a : silu_bf16_f64(g);
}

// All three tiers.
__device__ __forceinline__ __nv_bfloat16 silu_bf16(float g) {
  bool ok;
  const float s = silu_est_ex2(g, &ok);
  return ok ? __float2bfloat16_rn(s) : silu_bf16_slow(g);
}

// Block reductions with one barrier: every warp reduces the per-warp values
// itself.  An xor butterfly pairs each lane with a partner that adds the
// same two values, so all lanes (and all warps) hold the same bits.  `red`
// is written again only by the next row, after the next barrier of the
// caller's row loop (one row per CTA in the one-shot kernel).
template <int kThreads>
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = lane < kThreads / 32 ? red[lane] : 0.0;
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

template <int kThreads>
__device__ __forceinline__ float block_max_f32(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = lane < kThreads / 32 ? red[lane] : 0.f;
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

enum : int { kOpRmsNorm = 0, kOpSiluMul = 1 };

template <bool kGlobal>
__device__ __forceinline__ uint4 ld16(const uint4* p) {
  if constexpr (kGlobal) return __ldg(p);
  return *p;   // shared memory (staged rows)
}

// One row: y (bf16, in registers), then its quantization.  Inputs come from
// global memory (kGlobal) or from a row staged in shared memory; `res_in`
// (may be null) is the residual row, `res_out` (global, may be null) where h
// goes; `wv` the RMSNorm gain chunks of this thread.
// GROUP = 0: one scale per row (FP8 or INT8); GROUP = 128: one FP8 scale per
// 128 outputs (16 consecutive chunks, held by 16 consecutive threads).
template <int OP, int GROUP, bool kInt8, int kRowThreads, int VPT, bool kGlobal>
__device__ __forceinline__ void quantize_row(int64_t row, const uint4* in_row, const uint4* res_in, uint4* res_out,
                                             const uint4 (&wv)[VPT], float eps, uint8_t* __restrict__ q,
                                             float* __restrict__ scales, int64_t Kout, double* red_d, float* red_f) {
  const int nvec = static_cast<int>(Kout / 8);
  uint4 y[VPT];

  if constexpr (OP == kOpRmsNorm) {
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;
      y[i] = make_uint4(0u, 0u, 0u, 0u);
      if (idx < nvec) {
        uint4 h = ld16<kGlobal>(in_row + idx);
        if (res_in) {
          const uint4 rv = kGlobal ? res_in[idx] : ld16<false>(res_in + idx);   // not __ldg: written below
          const uint32_t xw[4] = {h.x, h.y, h.z, h.w}, rw[4] = {rv.x, rv.y, rv.z, rv.w};
          uint32_t hw[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            hw[j] = bf16x2_rn(__fadd_rn(bf(xw[j], 0), bf(rw[j], 0)), __fadd_rn(bf(xw[j], 1), bf(rw[j], 1)));
          h = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          res_out[idx] = h;
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
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;
      if (idx < nvec) {
        const uint32_t hw[4] = {y[i].x, y[i].y, y[i].z, y[i].w}, ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t n = bf16x2_rn(__fmul_rn(bf(hw[j], 0), r), __fmul_rn(bf(hw[j], 1), r));
          out[j] = bf16x2_rn(__fmul_rn(bf(n, 0), bf(ww[j], 0)), __fmul_rn(bf(n, 1), bf(ww[j], 1)));
        }
        y[i] = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
  } else {
    static_assert(OP != kOpSiluMul || VPT <= 4, "one bit per element of the thread's chunks");
    const uint4* gr = in_row;
    const uint4* ur = in_row + nvec;
    uint32_t redo = 0;   // bit 8 i + e: element e of chunk i needs the fp64 silu
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;
      y[i] = make_uint4(0u, 0u, 0u, 0u);
      if (idx < nvec) {
        const uint4 gv = ld16<kGlobal>(gr + idx), uv = ld16<kGlobal>(ur + idx);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bool ok0, ok1;
          const float s0 = silu_est_ex2(bf(gw[j], 0), &ok0), s1 = silu_est_ex2(bf(gw[j], 1), &ok1);
          if (!ok0) redo |= 1u << (8 * i + 2 * j);
          if (!ok1) redo |= 1u << (8 * i + 2 * j + 1);
          const uint32_t a = bf16x2_rn(s0, s1);   // the two SiLUs in bf16
          // products of two bf16 values are exact in fp32
          out[j] = bf16x2_rn(__fmul_rn(bf(a, 0), bf(uw[j], 0)), __fmul_rn(bf(a, 1), bf(uw[j], 1)));
        }
        y[i] = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
    // Cold pass: the few elements whose tier-1 estimate could round the wrong
    // way are recomputed from their inputs by the later tiers.
    if (redo) {
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        if ((redo >> (8 * i)) & 0xFFu) {
          const int idx = threadIdx.x + i * kRowThreads;
          const uint4 gv = ld16<kGlobal>(gr + idx), uv = ld16<kGlobal>(ur + idx);
          const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
          uint32_t yw[4] = {y[i].x, y[i].y, y[i].z, y[i].w};
#pragma unroll 1
          for (int e = 0; e < 8; ++e) {
            if ((redo >> (8 * i + e)) & 1u) {
              const int j = e >> 1, k = e & 1;
              const __nv_bfloat16 a = silu_bf16_slow(bf(gw[j], k));
              const uint32_t v =
                  __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__bfloat162float(a), bf(uw[j], k))));
              yw[j] = k ? ((yw[j] & 0x0000FFFFu) | (v << 16)) : ((yw[j] & 0xFFFF0000u) | v);
            }
          }
          y[i] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
        }
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
    static_assert(GROUP == 0 || !kInt8, "1 x 128 groups are FP8");
    const int64_t groups = Kout / 128;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * kRowThreads;   // 16 threads share idx / 16 (kRowThreads % 16 == 0)
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

template <int kRowThreads, int VPT>
__device__ __forceinline__ void load_gain(const __nv_bfloat16* weight, int nvec, uint4 (&wv)[VPT]) {
  const uint4* wr = reinterpret_cast<const uint4*>(weight);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * kRowThreads;
    wv[i] = (weight && idx < nvec) ? __ldg(wr + idx) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// One row per CTA, read straight from global memory into registers (few
// rows, or rows too long to double-buffer in shared memory).
template <int OP, int GROUP, bool kInt8, int kRowThreads, int VPT>
__global__ void __launch_bounds__(kRowThreads) producer_quant_kernel(const __nv_bfloat16* __restrict__ in,
                                                                     __nv_bfloat16* __restrict__ residual,
                                                                     const __nv_bfloat16* __restrict__ weight,
                                                                     float eps, uint8_t* __restrict__ q,
                                                                     float* __restrict__ scales, int64_t Kout) {
  static_assert(kRowThreads * VPT * 8 <= kMaxRow || VPT == 1, "row longer than the ABI allows");
  __shared__ double red_d[kRowThreads / 32];
  __shared__ float red_f[kRowThreads / 32];
  grid_launch_dependents();   // as the other quantization kernels: before the wait
  grid_dependency_wait();
  const int64_t row = blockIdx.x;
  const int nvec = static_cast<int>(Kout / 8);
  uint4 wv[VPT];   // the gain, loaded with the row rather than after the reduction
  load_gain<kRowThreads, VPT>(OP == kOpRmsNorm ? weight : nullptr, nvec, wv);
  const int64_t in_len = OP == kOpRmsNorm ? Kout : 2 * Kout;
  uint4* rrow = residual ? reinterpret_cast<uint4*>(residual + row * Kout) : nullptr;
  quantize_row<OP, GROUP, kInt8, kRowThreads, VPT, true>(row, reinterpret_cast<const uint4*>(in + row * in_len),
                                                         rrow, rrow, wv, eps, q, scales, Kout, red_d, red_f);
}

// Many rows: a persistent CTA walks rows blockIdx.x, + gridDim.x, ...; one
// thread copies each row (and its residual) into one of two shared-memory
// buffers with the bulk-copy engine while the CTA works on the other, so
// the next row's load overlaps this row's arithmetic and stores.  Every
// wait is bounded; a timeout sets bit 12 of the status word and the CTA
// stops after waiting (bounded) for its copies still in flight.
template <int OP, int GROUP, bool kInt8, int kRowThreads, int VPT>
__global__ void __launch_bounds__(kRowThreads) producer_quant_staged_kernel(
    const __nv_bfloat16* __restrict__ in, __nv_bfloat16* __restrict__ residual,
    const __nv_bfloat16* __restrict__ weight, float eps, uint8_t* __restrict__ q, float* __restrict__ scales,
    int64_t M, int64_t Kout, int* status, uint64_t wait_limit_ns) {
  extern __shared__ __align__(128) uint8_t rows[];   // two buffers of row_bytes
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ double red_d[kRowThreads / 32];
  __shared__ float red_f[kRowThreads / 32];
  const int nvec = static_cast<int>(Kout / 8);
  const int64_t in_len = OP == kOpRmsNorm ? Kout : 2 * Kout;    // bf16 input values per row
  const uint32_t in_bytes = static_cast<uint32_t>(in_len * 2);
  const uint32_t row_bytes = in_bytes + (residual ? static_cast<uint32_t>(Kout * 2) : 0u);
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  grid_launch_dependents();
  grid_dependency_wait();
  uint4 wv[VPT];
  load_gain<kRowThreads, VPT>(OP == kOpRmsNorm ? weight : nullptr, nvec, wv);

  auto issue = [&](int64_t r, int b) {   // thread 0 only
    uint8_t* dst = rows + static_cast<size_t>(b) * row_bytes;
    mbar_arrive_expect_tx(&bar[b], row_bytes);
    bulk_copy_g2s(dst, in + r * in_len, in_bytes, &bar[b]);
    if (residual) bulk_copy_g2s(dst + in_bytes, residual + r * Kout, static_cast<uint32_t>(Kout * 2), &bar[b]);
  };
  // Rows it and it + 1 are in flight while row it is worked on: both
  // buffers are filled up front, and the copy of row it + 1 into buffer
  // (it + 1) & 1 is issued once every thread has passed iteration it's
  // barrier, i.e. has left iteration it - 1, the last reader of that buffer.
  if (threadIdx.x == 0 && blockIdx.x < M) issue(blockIdx.x, 0);
  if (threadIdx.x == 0 && blockIdx.x + gridDim.x < M) issue(blockIdx.x + gridDim.x, 1);
  int it = 0;
  int issued = 2;   // copies issued (for the drain after a timeout)
  bool failed = false;
  for (int64_t row = blockIdx.x; row < M; row += gridDim.x, ++it) {
    const int b = it & 1;
    const bool landed = mbar_wait(&bar[b], static_cast<uint32_t>(it >> 1) & 1u, wait_limit_ns);
    if (!__syncthreads_and(landed)) {
      failed = true;
      break;
    }
    if (it > 0) {
      if (threadIdx.x == 0 && row + gridDim.x < M) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(row + gridDim.x, b ^ 1);
      }
      issued = it + 2;
    }
    const uint8_t* buf = rows + static_cast<size_t>(b) * row_bytes;
    uint4* rout = residual ? reinterpret_cast<uint4*>(residual + row * Kout) : nullptr;
    quantize_row<OP, GROUP, kInt8, kRowThreads, VPT, false>(
        row, reinterpret_cast<const uint4*>(buf),
        residual ? reinterpret_cast<const uint4*>(buf + in_bytes) : nullptr, rout, wv, eps, q, scales, Kout, red_d,
        red_f);
  }
  if (failed && threadIdx.x == 0) {
    if (status) atomicOr(status, 1 << 12);
    // wait (bounded) for the copies this CTA may still have in flight
    for (int jt = it; jt < issued; ++jt) {
      const int64_t r = blockIdx.x + static_cast<int64_t>(jt) * gridDim.x;
      if (r < M) mbar_wait(&bar[jt & 1], static_cast<uint32_t>(jt >> 1) & 1u, wait_limit_ns);
    }
  }
}

cudaLaunchConfig_t row_config(int64_t M, int threads, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int OP, int GROUP, bool kInt8, int T, int V>
cudaError_t launch_staged(const __nv_bfloat16* ip, __nv_bfloat16* rp, const __nv_bfloat16* wp, float eps,
                          uint8_t* qp, float* scales, int64_t M, int64_t Kout, int smem, int* status,
                          uint64_t wait_limit_ns, cudaStream_t stream) {
  auto kern = producer_quant_staged_kernel<OP, GROUP, kInt8, T, V>;
  static int configured = 0;   // dynamic shared memory opted in once per instantiation and process
  if (configured < smem) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxStagedSmem);
    if (e != cudaSuccess) return e;
    configured = kMaxStagedSmem;
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, T, smem);
  if (e != cudaSuccess) return e;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ctas = M < static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1) ? M
                                                                                 : static_cast<int64_t>(sms) * per_sm;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = row_config(ctas, T, stream, attr);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  return cudaLaunchKernelEx(&cfg, kern, ip, rp, wp, eps, qp, scales, M, Kout, status, wait_limit_ns);
}

template <int OP, int GROUP, bool kInt8>
cudaError_t launch_rows(const void* in, void* residual, const void* weight, float eps, void* q, float* scales,
                        int64_t M, int64_t Kout, int* status, uint64_t wait_limit_ns, cudaStream_t stream) {
  const auto* ip = static_cast<const __nv_bfloat16*>(in);
  auto* rp = static_cast<__nv_bfloat16*>(residual);
  const auto* wp = static_cast<const __nv_bfloat16*>(weight);
  auto* qp = static_cast<uint8_t*>(q);
  const int64_t nvec = Kout / 8;
  // Many rows of at least 16 KB whose two copies fit in shared memory:
  // persistent CTAs that double-buffer rows (256 / 512 / 1024 threads as the
  // row grows).  Shorter rows keep more one-shot CTAs per SM in flight.
  const int64_t row_bytes = (OP == kOpRmsNorm ? 2 * Kout : 4 * Kout) + (residual ? 2 * Kout : 0);
  const int64_t in_row_bytes = OP == kOpRmsNorm ? 2 * Kout : 4 * Kout;
  if (M >= 2 * 148 && in_row_bytes >= 16 * 1024 && 2 * row_bytes <= kMaxStagedSmem) {
    const int smem = static_cast<int>(2 * row_bytes);
#define LQ_SROW(T, V)                                                                                         \
  if (nvec <= (T) * (V))                                                                                      \
    return launch_staged<OP, GROUP, kInt8, T, V>(ip, rp, wp, eps, qp, scales, M, Kout, smem, status,           \
                                                 wait_limit_ns, stream);
    if (nvec <= 512) {
      LQ_SROW(256, 1)
      LQ_SROW(256, 2)
    }
    if (nvec <= 2048) {
      LQ_SROW(512, 1)
      LQ_SROW(512, 2)
      LQ_SROW(512, 4)
    }
    LQ_SROW(1024, 2)
    LQ_SROW(1024, 4)
#undef LQ_SROW
    return cudaErrorInvalidValue;
  }
  cudaLaunchAttribute attr[1];
  // Fewer rows than two per SM, or rows longer than 8192 outputs: a row per
  // 1024-thread CTA (more warps per SM to hide the arithmetic's latency).
  if ((M < 2 * 148 && nvec > 256) || nvec > 1024) {
    cudaLaunchConfig_t cfg = row_config(M, 1024, stream, attr);
#define LQ_PROW(T, V) \
  if (nvec <= (T) * (V)) \
    return cudaLaunchKernelEx(&cfg, producer_quant_kernel<OP, GROUP, kInt8, T, V>, ip, rp, wp, eps, qp, scales, Kout);
    LQ_PROW(1024, 1)
    LQ_PROW(1024, 2)
    LQ_PROW(1024, 4)
    return cudaErrorInvalidValue;
  }
  cudaLaunchConfig_t cfg = row_config(M, 256, stream, attr);
  LQ_PROW(256, 1)
  LQ_PROW(256, 2)
  LQ_PROW(256, 4)
  if constexpr (OP == kOpRmsNorm) {   // SiLU rows this long take the 1024-thread CTAs above
    LQ_PROW(256, 8)
    LQ_PROW(256, 16)
  }
#undef LQ_PROW
  return cudaErrorInvalidValue;
}

// The SiLU of the producer kernels, element by element (a test hook).
__global__ void __launch_bounds__(256) silu_bf16_kernel(const __nv_bfloat16* __restrict__ g,
                                                        __nv_bfloat16* __restrict__ out, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = silu_bf16(__bfloat162float(g[i]));
}

}  // namespace

int64_t producer_max_row() { return kMaxRow; }

cudaError_t launch_silu_bf16(const void* g, void* out, int64_t n, cudaStream_t stream) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  silu_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(g),
                                                                       static_cast<__nv_bfloat16*>(out), n);
  return cudaGetLastError();
}

cudaError_t launch_rms_norm_quant(int fmt, bool per_block, const void* x, void* residual, const void* weight,
                                  float eps, void* q, float* scales, int64_t M, int64_t K, int* status,
                                  uint64_t wait_limit_ns, cudaStream_t stream) {
  if (per_block)
    return launch_rows<kOpRmsNorm, 128, false>(x, residual, weight, eps, q, scales, M, K, status, wait_limit_ns,
                                               stream);
  if (fmt == kFmtInt8)
    return launch_rows<kOpRmsNorm, 0, true>(x, residual, weight, eps, q, scales, M, K, status, wait_limit_ns,
                                            stream);
  return launch_rows<kOpRmsNorm, 0, false>(x, residual, weight, eps, q, scales, M, K, status, wait_limit_ns, stream);
}

cudaError_t launch_silu_mul_quant(int fmt, bool per_block, const void* gate_up, void* q, float* scales, int64_t M,
                                  int64_t I, int* status, uint64_t wait_limit_ns, cudaStream_t stream) {
  if (per_block)
    return launch_rows<kOpSiluMul, 128, false>(gate_up, nullptr, nullptr, 0.f, q, scales, M, I, status,
                                               wait_limit_ns, stream);
  if (fmt == kFmtInt8)
    return launch_rows<kOpSiluMul, 0, true>(gate_up, nullptr, nullptr, 0.f, q, scales, M, I, status, wait_limit_ns,
                                            stream);
  return launch_rows<kOpSiluMul, 0, false>(gate_up, nullptr, nullptr, 0.f, q, scales, M, I, status, wait_limit_ns,
                                           stream);
}

}  // namespace lq
