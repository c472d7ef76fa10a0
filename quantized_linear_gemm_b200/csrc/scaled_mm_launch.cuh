// Launch helper shared by the per-format instantiation files.
#pragma once

#include "scaled_mm_kernel.cuh"
#include "scaled_mm_persistent.cuh"
#include "scaled_mm_pair.cuh"
#include "scaled_mm_streamk.cuh"

namespace lq {

template <int FMT, bool SWAP, int TN, bool FUSE = false, bool GROUPED = false, bool BIAS = false>
cudaError_t launch_tc(const GemmLaunch& l) {
  auto kern = scaled_mm_tc_kernel<FMT, SWAP, TN, FUSE, GROUPED, BIAS>;
  static int configured = 0;   // max dynamic smem set once per instantiation and process
  if (configured < l.smem_bytes) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    configured = 227 * 1024;
  }
  if (l.cluster_z > 8) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = l.grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(l.smem_bytes);
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (l.pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (l.cluster_z > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = static_cast<unsigned>(l.cluster_z);
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, l.tmX, l.tmY, l.p);
}

// The plain GEMM instantiations, with or without the bias epilogue.
template <int FMT, bool BIAS>
cudaError_t launch_dense(const GemmLaunch& l, int swap_ab, int tile_n) {
  if (swap_ab) {
    switch (tile_n) {
      case 16: return launch_tc<FMT, true, 16, false, false, BIAS>(l);
      case 32: return launch_tc<FMT, true, 32, false, false, BIAS>(l);
      case 64: return launch_tc<FMT, true, 64, false, false, BIAS>(l);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (tile_n) {
    case 64: return launch_tc<FMT, false, 64, false, false, BIAS>(l);
    case 128: return launch_tc<FMT, false, 128, false, false, BIAS>(l);
    case 256:   // fp32-scale Block_FP8 promotes in registers: its tiles stop at 128
      if constexpr (FMT != kFmtBlock) return launch_tc<FMT, false, 256, false, false, BIAS>(l);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <int FMT>
cudaError_t launch_format(const GemmLaunch& l, int swap_ab, int tile_n) {
  if (l.grouped) {
    if constexpr (!is_block_fmt(FMT)) {
      if (!swap_ab) return cudaErrorInvalidValue;
      switch (tile_n) {
        case 16: return launch_tc<FMT, true, 16, false, true>(l);
        case 32: return launch_tc<FMT, true, 32, false, true>(l);
        case 64: return launch_tc<FMT, true, 64, false, true>(l);
        default: return cudaErrorInvalidValue;
      }
    }
    return cudaErrorInvalidValue;
  }
  if (l.fuse) {
    if constexpr (!is_block_fmt(FMT)) {
      if (!swap_ab) return cudaErrorInvalidValue;
      switch (tile_n) {
        case 16: return launch_tc<FMT, true, 16, true>(l);
        case 32: return launch_tc<FMT, true, 32, true>(l);
        case 64: return launch_tc<FMT, true, 64, true>(l);
        default: return cudaErrorInvalidValue;
      }
    }
    return cudaErrorInvalidValue;
  }
  if (l.persistent == 3) {
    if (swap_ab) return cudaErrorInvalidValue;
    return l.p.bias ? launch_streamk<FMT, true>(l, tile_n) : launch_streamk<FMT, false>(l, tile_n);
  }
  if (l.persistent == 2) {
    if (swap_ab) return cudaErrorInvalidValue;
    return l.p.bias ? launch_pair<FMT, true>(l, tile_n) : launch_pair<FMT, false>(l, tile_n);
  }
  if (l.persistent) {
    if (swap_ab) return cudaErrorInvalidValue;
    return l.p.bias ? launch_persistent<FMT, true>(l, tile_n) : launch_persistent<FMT, false>(l, tile_n);
  }
  return l.p.bias ? launch_dense<FMT, true>(l, swap_ab, tile_n) : launch_dense<FMT, false>(l, swap_ab, tile_n);
}

template <int FMT>
int pair_capacity(int tile_n, bool bias, int smem_bytes) {
  if constexpr (FMT == kFmtFp8 || FMT == kFmtInt8) {
    switch (tile_n) {
      case 128: return bias ? max_pairs<FMT, 128, true>(smem_bytes) : max_pairs<FMT, 128, false>(smem_bytes);
      case 256: return bias ? max_pairs<FMT, 256, true>(smem_bytes) : max_pairs<FMT, 256, false>(smem_bytes);
      default: return 0;
    }
  }
  if constexpr (FMT == kFmtBlock || FMT == kFmtBlockE8m0) {
    if (tile_n == 128) return bias ? max_pairs<FMT, 128, true>(smem_bytes) : max_pairs<FMT, 128, false>(smem_bytes);
  }
  return 0;
}

}  // namespace lq
