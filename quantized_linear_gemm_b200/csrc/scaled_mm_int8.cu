// W8A8_INT8 instantiations of the scaled_mm kernel.
#include "scaled_mm_launch.cuh"
namespace lq {
cudaError_t launch_scaled_mm_int8(const GemmLaunch& l, int swap_ab, int tile_n) {
  return launch_format<kFmtInt8>(l, swap_ab, tile_n);
}
int pair_capacity_int8(int tile_n, bool bias, int smem_bytes) { return pair_capacity<kFmtInt8>(tile_n, bias, smem_bytes); }
}  // namespace lq
