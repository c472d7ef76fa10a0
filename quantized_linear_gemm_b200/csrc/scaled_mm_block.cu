// Block_FP8 instantiations of the scaled_mm kernel and the Split-K reduction.
#include <type_traits>

#include "scaled_mm_launch.cuh"
namespace lq {
cudaError_t launch_scaled_mm_block(const GemmLaunch& l, int swap_ab, int tile_n) {
  return launch_format<kFmtBlock>(l, swap_ab, tile_n);
}
int tmem_cols_per_cta(int fmt, int tile_n, int persistent) {
  if (persistent == 1 || persistent == 3) return tmem_cols_for(2 * tile_n);   // two accumulators
  if (persistent == 2) return (is_block_fmt(fmt) || tile_n == 256) ? 512 : 2 * tile_n;   // CTA pairs
  auto one = [&](auto fmt_c) -> int {
    constexpr int F = decltype(fmt_c)::value;
    switch (tile_n) {
      case 16: return tc_tmem_cols<F, 16>();
      case 32: return tc_tmem_cols<F, 32>();
      case 64: return tc_tmem_cols<F, 64>();
      case 128: return tc_tmem_cols<F, 128>();
      case 256: return tc_tmem_cols<F, 256>();
      default: return 512;
    }
  };
  switch (fmt) {
    case kFmtFp8: return one(std::integral_constant<int, kFmtFp8>{});
    case kFmtInt8: return one(std::integral_constant<int, kFmtInt8>{});
    case kFmtBlock: return one(std::integral_constant<int, kFmtBlock>{});
    default: return one(std::integral_constant<int, kFmtBlockE8m0>{});
  }
}

int pair_capacity_block(int tile_n, bool bias, int smem_bytes) {
  return pair_capacity<kFmtBlock>(tile_n, bias, smem_bytes);
}

int gemm_smem_bytes_for(int tile_n, int stages, bool cluster_reduce, bool fuse) {
  if (fuse) {
    switch (tile_n) {
      case 16: return gemm_smem_bytes<16, true>(stages, cluster_reduce);
      case 32: return gemm_smem_bytes<32, true>(stages, cluster_reduce);
      case 64: return gemm_smem_bytes<64, true>(stages, cluster_reduce);
      default: return -1;
    }
  }
  switch (tile_n) {
    case 16: return gemm_smem_bytes<16>(stages, cluster_reduce);
    case 32: return gemm_smem_bytes<32>(stages, cluster_reduce);
    case 64: return gemm_smem_bytes<64>(stages, cluster_reduce);
    case 128: return gemm_smem_bytes<128>(stages, cluster_reduce);
    case 256: return gemm_smem_bytes<256>(stages, cluster_reduce);
    default: return -1;
  }
}

int pair_smem_bytes_for(int tile_n, int stages) {
  switch (tile_n) {
    case 128: return pair_smem_bytes<128>(stages);
    case 256: return pair_smem_bytes<256>(stages);
    default: return -1;
  }
}

int persistent_smem_bytes_for(int tile_n, int stages) {
  switch (tile_n) {
    case 64: return persistent_smem_bytes<64>(stages);
    case 128: return persistent_smem_bytes<128>(stages);
    case 256: return persistent_smem_bytes<256>(stages);
    default: return -1;
  }
}

cudaError_t launch_splitk_reduce(int fmt, const GemmParams& p, int pdl, cudaStream_t stream) {
  const int64_t work = p.M * p.N / 4;
  int64_t blocks = (work + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  switch (fmt) {
    case kFmtFp8: return cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<kFmtFp8>, p);
    case kFmtInt8: return cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<kFmtInt8>, p);
    case kFmtBlock:
    case kFmtBlockE8m0:   // the partials already carry their block scales
      return cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<kFmtBlock>, p);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace lq
