// Block_FP8 instantiations with UE8M0 (e8m0 byte) scales.
#include "scaled_mm_launch.cuh"
namespace lq {
cudaError_t launch_scaled_mm_block_e8m0(const GemmLaunch& l, int swap_ab, int tile_n) {
  return launch_format<kFmtBlockE8m0>(l, swap_ab, tile_n);
}
}  // namespace lq
