// Internal interface between the host library (lq_host.cu) and the kernel
// translation units.  Not part of the public C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace lq {

constexpr int kFmtFp8 = 0;    // LQ_FP8_DYNAMIC
constexpr int kFmtInt8 = 1;   // LQ_W8A8_INT8
constexpr int kFmtBlock = 2;  // LQ_BLOCK_FP8
constexpr int kFmtBlockE8m0 = 3;  // LQ_BLOCK_FP8_UE8M0: Block_FP8 with power-of-two (e8m0 byte) scales
__host__ __device__ constexpr bool is_block_fmt(int fmt) { return fmt == kFmtBlock || fmt == kFmtBlockE8m0; }

struct GemmParams {
  int64_t M, N, K;
  int T;               // number of 128-wide K tiles, ceil(K / 128)
  int KB;              // K / 128 (Block_FP8 scale row length)
  int S;               // split_k
  int stages;          // shared-memory ring depth
  int reduce_mode;     // S > 1: 0 separate kernel, 1 last-arriver (global), 2 cluster (DSMEM)
  int early_weights;   // stream weight tiles before the grid dependency wait
  const float* a_s;
  const float* b_s;
  __nv_bfloat16* C;
  void* ws;            // Split-K partials [S, M, N] (f32, or s32 for INT8)
  int* counters;       // Split-K arrival counters, one per output tile
  int32_t* acc_out;    // optional exact INT8 accumulators [M, N]
  int* status;         // device status word (bit set per timed-out wait site)
  uint64_t wait_limit_ns;
  uint64_t* trace;     // optional: kTraceSlots globaltimer stamps per CTA
  int skip_stage;      // test hook: >= 0 = the producer never fills this K tile (a wait runs out)
  // fused activation quantization (Swap-AB, FP8_Dynamic / W8A8_INT8)
  const __nv_bfloat16* x;   // bf16 activations [M, K]
  uint8_t* a_codes_out;     // [M, K] codes written by the first n-tile's CTAs
  float* a_scales_out;      // [M] per-token scales
  // grouped (mixture-of-experts) launch, Swap-AB: M = tokens T, N = rows per expert
  const int* expert_offsets;   // device [num_experts + 1]; null = one GEMM
  int num_experts;
  const __nv_bfloat16* bias;   // optional bf16 [N], added before the rounding to bf16
};

constexpr int kTraceSlots = 12;

// Launch description filled by the host library.
struct GemmLaunch {
  CUtensorMap tmX;     // operand on the MMA M side (128-row tiles)
  CUtensorMap tmY;     // operand on the MMA N side (tile_n-row tiles)
  GemmParams p;
  dim3 grid;
  int smem_bytes;
  int pdl;
  int cluster_z;       // > 1: launch clusters of (1, 1, cluster_z) CTAs
  int fuse;            // fused activation quantization (Swap-AB only)
  int grouped;         // grouped (mixture-of-experts) launch (Swap-AB only; p.expert_offsets set)
  int persistent;      // 1: persistent CTAs looping over output tiles (Standard, split_k 1, FP8 / INT8);
                       // 2: the same on CTA pairs (cta_group::2, 256-row tiles, clusters of two);
                       // 3: stream-K (equal shares of tiles x K blocks; p.ws slots, p.counters flags)
  cudaStream_t stream;
};

// Implemented in scaled_mm_{fp8,int8,block}.cu: launches the instantiation
// (swap_ab, tile_n) of the format.  Returns cudaErrorInvalidValue for a
// (swap_ab, tile_n) pair that is not instantiated.
cudaError_t launch_scaled_mm_fp8(const GemmLaunch& l, int swap_ab, int tile_n);
cudaError_t launch_scaled_mm_int8(const GemmLaunch& l, int swap_ab, int tile_n);
cudaError_t launch_scaled_mm_block(const GemmLaunch& l, int swap_ab, int tile_n);
cudaError_t launch_scaled_mm_block_e8m0(const GemmLaunch& l, int swap_ab, int tile_n);
cudaError_t launch_splitk_reduce(int fmt, const GemmParams& p, int pdl, cudaStream_t stream);

// Dynamic shared memory of the GEMM kernel for (tile_n, stages), with or
// without the cluster Split-K reduction (reduce mode 2 with split_k > 1).
// Dynamic shared memory of the GEMM kernel; `fuse`: the fused-quantization
// instantiation (each ring slot also stages a bf16 activation tile).
int gemm_smem_bytes_for(int tile_n, int stages, bool cluster_reduce, bool fuse = false);
// Dynamic shared memory of the persistent kernel for (tile_n, stages).
int persistent_smem_bytes_for(int tile_n, int stages);
// ... and of the CTA-pair kernel (tile_n 128 or 256; -1 otherwise).
int pair_smem_bytes_for(int tile_n, int stages);
// Largest number of co-resident CTA pairs of the pair kernel (0 if unknown).
int pair_capacity_fp8(int tile_n, bool bias, int smem_bytes);
int pair_capacity_int8(int tile_n, bool bias, int smem_bytes);
int pair_capacity_block(int tile_n, bool bias, int smem_bytes);        // tile_n 128
// Tensor-memory columns one CTA allocates: the one-SM kernel (persistent 0),
// the persistent and stream-K kernels (1, 3), CTA pairs (2: all 512).
int tmem_cols_per_cta(int fmt, int tile_n, int persistent);
int pair_capacity_block_e8m0(int tile_n, bool bias, int smem_bytes);   // tile_n 128

// Quantization kernels (quant_kernels.cu).
cudaError_t launch_quant_per_token(int fmt, const void* x, void* q, float* scales, int64_t M, int64_t K,
                                   cudaStream_t stream);
cudaError_t launch_quant_group128(const void* x, void* q, void* scales, int64_t M, int64_t K, bool e8m0,
                                  cudaStream_t stream);
// Producer-side fused quantizers (producer_quant.cu); rows of at most
// producer_max_row() outputs.
int64_t producer_max_row();
// bf16(silu(g)) of n bf16 gates, by the producer kernels' own tiers (a test hook).
cudaError_t launch_silu_bf16(const void* g, void* out, int64_t n, cudaStream_t stream);
cudaError_t launch_rms_norm_quant(int fmt, bool per_block, const void* x, void* residual, const void* weight,
                                  float eps, void* q, float* scales, int64_t M, int64_t K, int* status,
                                  uint64_t wait_limit_ns, cudaStream_t stream);
cudaError_t launch_silu_mul_quant(int fmt, bool per_block, const void* gate_up, void* q, float* scales, int64_t M,
                                  int64_t I, int* status, uint64_t wait_limit_ns, cudaStream_t stream);
cudaError_t launch_quant_weight_block128(const void* w, void* q, void* scales, int64_t N, int64_t K, bool e8m0,
                                         cudaStream_t stream);
cudaError_t launch_fill_zero_bf16(__nv_bfloat16* C, int64_t count, cudaStream_t stream);

}  // namespace lq
