// FP8_Dynamic instantiations of the scaled_mm kernel.
#include "scaled_mm_launch.cuh"
namespace lq {
cudaError_t launch_scaled_mm_fp8(const GemmLaunch& l, int swap_ab, int tile_n) {
  return launch_format<kFmtFp8>(l, swap_ab, tile_n);
}
int pair_capacity_fp8(int tile_n, bool bias, int smem_bytes) { return pair_capacity<kFmtFp8>(tile_n, bias, smem_bytes); }
}  // namespace lq
