// Block_FP8 instantiations with UE8M0 (power-of-two) scales.
#include "scaled_mm_launch.cuh"
namespace lq {
cudaError_t launch_scaled_mm_block_e8m0(const GemmLaunch& l, int swap_ab, int tile_n) {
  return launch_format<kFmtBlockE8m0>(l, swap_ab, tile_n);
}
int pair_capacity_block_e8m0(int tile_n, bool bias, int smem_bytes) {
  return pair_capacity<kFmtBlockE8m0>(tile_n, bias, smem_bytes);
}
}  // namespace lq
