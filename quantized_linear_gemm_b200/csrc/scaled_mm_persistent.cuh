// Persistent scaled_mm for large M (prefill): Standard orientation, split_k 1,
// FP8_Dynamic and W8A8_INT8.
//
// The one-tile-per-CTA kernel (scaled_mm_kernel.cuh) leaves the tensor core
// idle while a CTA fills its ring and while it runs its epilogue: with one
// CTA per SM (a 128 x 256 tile needs ~200 KB of shared memory) nothing else
// runs on the SM meanwhile.  Here one CTA per SM loops over output tiles:
//   - tile t of the launch is (m-block t mod gx, n-block t div gx): the CTAs
//     working at one moment cover a few weight tiles and every m-block, so
//     each weight tile is read once from HBM and reused from L2;
//   - CTA b takes tiles b, b + gridDim.x, ...;
//   - the TMA producer runs through all K blocks of all its tiles without
//     draining the shared-memory ring between tiles;
//   - the accumulator is double-buffered in tensor memory (2 x TN columns):
//     the MMA warp fills buffer j mod 2 with tile j while the epilogue warps
//     scale, round and store tile j - 1 from the other buffer, and release a
//     buffer as soon as its last columns are in registers.
// The arithmetic of each output is the non-persistent kernel's (same MMA
// order, same epilogue expression), so the results are identical bit for bit.
#pragma once

#include "scaled_mm_kernel.cuh"

namespace lq {

constexpr int kPersistentScaleBytes = 2 * 256 * 4;   // b_s of the tile's columns, by tile parity

template <int TN>
__host__ __device__ constexpr int persistent_smem_bytes(int stages) {
  return 1024 + stages * TileShape<TN>::kStageBytes + kCtlBytes + kPersistentScaleBytes;
}

template <int FMT, int TN, bool BIAS>
__global__ void __launch_bounds__(kThreads, 1)
    scaled_mm_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                const GemmParams p) {
  static_assert(FMT == kFmtFp8 || FMT == kFmtInt8, "persistent kernel: FP8_Dynamic / W8A8_INT8");
  using Shape = TileShape<TN>;
  constexpr bool kInt8 = FMT == kFmtInt8;
  constexpr int kTmemCols = tmem_cols_for(2 * TN);
  constexpr int CH = 32;   // TMEM columns per tcgen05.ld

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  const int stages = p.stages;
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + stages * Shape::kStageBytes);
  SmemCtl c;
  c.full = bars;
  c.empty = bars + stages;
  c.tfull = bars + 2 * stages;
  c.tempty = c.tfull + 2;
  c.mma_done = c.tempty + 2;
  c.tmem_slot = reinterpret_cast<uint32_t*>(c.mma_done + 1);
  c.abort_flag = reinterpret_cast<volatile int*>(c.tmem_slot + 1);
  c.last_flag = c.abort_flag + 1;
  float* colsc = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kCtlBytes);   // [2][256]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t gx = (p.M + kTileM - 1) / kTileM;   // m-blocks
  const int64_t gy = (p.N + TN - 1) / TN;           // n-blocks
  const int64_t tiles = gx * gy;
  const int64_t my_tiles =
      tiles > static_cast<int64_t>(blockIdx.x) ? (tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const int T = p.T;
  auto tile_origin = [&](int64_t j, int64_t* m0, int64_t* n0) {
    const int64_t t = blockIdx.x + j * static_cast<int64_t>(gridDim.x);
    *m0 = (t % gx) * kTileM;
    *n0 = (t / gx) * TN;
  };

  if (threadIdx.x == 0) trace_stamp(p, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c.tfull[b], 1);
      mbar_init(&c.tempty[b], kEpiThreads / 32);
    }
    mbar_init(c.mma_done, 1);
    *c.abort_flag = 0;
    *c.last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensor_map(&tmA);
    prefetch_tensor_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(c.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *c.tmem_slot;
  if (threadIdx.x == 0) trace_stamp(p, 1);
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();   // weights: each tile read by the gx CTAs of its n-block
      const uint64_t pol_a = policy_evict_last();    // activations: re-read for every n-block
      int64_t it = 0;                                 // ring position over all tiles
      int64_t issued = 0;
      int pre = 0;
      if (my_tiles > 0) {
        int64_t m0, n0;
        tile_origin(0, &m0, &n0);
        pre = T < stages ? T : stages;
        // the first tile's first stages: weights before the dependency wait
        // when the caller allows it (pdl 2), activations after it
        if (!p.early_weights) grid_dependency_wait();
        for (int i = 0; i < pre; ++i) {
          if (i == p.skip_stage) continue;
          mbar_arrive_expect_tx(&c.full[i], Shape::kStageBytes);
          tma_load_2d(&tmB, &c.full[i], ring + i * Shape::kStageBytes + Shape::kXBytes, i * kTileK,
                      static_cast<int32_t>(n0), pol_w);
        }
        if (p.early_weights) grid_dependency_wait();
        trace_stamp(p, 2);
        for (int i = 0; i < pre; ++i) {
          if (i == p.skip_stage) continue;
          tma_load_2d(&tmA, &c.full[i], ring + i * Shape::kStageBytes, i * kTileK, static_cast<int32_t>(m0), pol_a);
        }
        it = pre;
        issued = pre;
      }
      bool go = true;
      for (int64_t j = 0; j < my_tiles && go; ++j) {
        int64_t m0, n0;
        tile_origin(j, &m0, &n0);
        for (int kb = (j == 0 ? pre : 0); kb < T; ++kb, ++it) {
          const int s = static_cast<int>(it % stages);
          const uint32_t ph = static_cast<uint32_t>(it / stages) & 1u;
          if (!wait_bar(&c.empty[s], ph ^ 1u, p, c, 0)) {
            go = false;
            break;
          }
          if (it == p.skip_stage) continue;
          uint8_t* st = ring + s * Shape::kStageBytes;
          mbar_arrive_expect_tx(&c.full[s], Shape::kStageBytes);
          tma_load_2d(&tmA, &c.full[s], st, kb * kTileK, static_cast<int32_t>(m0), pol_a);
          tma_load_2d(&tmB, &c.full[s], st + Shape::kXBytes, kb * kTileK, static_cast<int32_t>(n0), pol_w);
          issued = it + 1;
        }
      }
      if (*c.abort_flag) {
        // Drain: wait (bounded) for the copies still in flight into shared memory.
        const int64_t first = issued > stages ? issued - stages : 0;
        for (int64_t q = first; q < issued; ++q) {
          if (q == p.skip_stage) continue;   // never armed
          const uint32_t par = static_cast<uint32_t>(q / stages) & 1u;
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&c.full[q % stages], par) && global_timer_ns() - t0 < p.wait_limit_ns) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc<kInt8>(kTileM, TN);
      bool issued_any = false;
      bool go = true;
      int64_t it = 0;
      for (int64_t j = 0; j < my_tiles && go; ++j) {
        const int b = static_cast<int>(j & 1);
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        if (!wait_bar(&c.tempty[b], (use & 1u) ^ 1u, p, c, 1)) break;   // tile j - 2 stored
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * TN);
        for (int kb = 0; kb < T; ++kb, ++it) {
          const int s = static_cast<int>(it % stages);
          const uint32_t ph = static_cast<uint32_t>(it / stages) & 1u;
          if (!wait_bar(&c.full[s], ph, p, c, 2)) {
            go = false;
            break;
          }
          tc_fence_after_sync();
          if (it == 0) trace_stamp(p, 3);
          uint8_t* st = ring + s * Shape::kStageBytes;
          const uint64_t xd = smem_desc_k_sw128(st);
          const uint64_t yd = smem_desc_k_sw128(st + Shape::kXBytes);
#pragma unroll
          for (int kk = 0; kk < kTileK / kMmaK; ++kk) {
            const uint32_t acc = (kb > 0 || kk > 0);
            if (kInt8)
              mma_i8(d_tmem, xd + 2 * kk, yd + 2 * kk, idesc, acc);
            else
              mma_f8f6f4(d_tmem, xd + 2 * kk, yd + 2 * kk, idesc, acc);
          }
          issued_any = true;
          mma_commit(&c.empty[s]);
        }
        if (go) mma_commit(&c.tfull[b]);
      }
      trace_stamp(p, 4);
      if (issued_any) {
        // All MMAs must be complete before TMEM is released at teardown.
        mma_commit(c.mma_done);
        wait_bar(c.mma_done, 0, p, c, 3);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Every epilogue thread runs every tile iteration (also after a timeout,
    // doing nothing), so the named barrier always matches.
    grid_dependency_wait();   // the scales may come from the previous kernel
    const int q = warp & 3;                    // TMEM lane quarter of this warp
    const int r = q * 32 + lane;               // accumulator row (TMEM lane)
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    bool ok = true;
    for (int64_t j = 0; j < my_tiles; ++j) {
      const int b = static_cast<int>(j & 1);
      const uint32_t use = static_cast<uint32_t>(j >> 1);
      int64_t m0, n0;
      tile_origin(j, &m0, &n0);
      // b_s of the tile's columns into this tile parity's buffer (tile j - 2,
      // the last user of that buffer, is finished by every thread: they all
      // passed the barrier of tile j - 1); a_s of this thread's row.
      float* cs = colsc + b * 256;
      for (int col = r; col < TN; col += kEpiThreads) cs[col] = n0 + col < p.N ? __ldg(p.b_s + n0 + col) : 0.f;
      const int64_t m = m0 + r;
      const float as_r = m < p.M ? __ldg(p.a_s + m) : 0.f;
      named_barrier_sync(2, kEpiThreads);
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(&c.tfull[b], use & 1u, p, c, 5) && !*c.abort_flag);
      if (!ok) continue;
      tc_fence_after_sync();
      const uint32_t t_buf = t_row + static_cast<uint32_t>(b * TN);
#pragma unroll
      for (int c0 = 0; c0 < TN; c0 += CH) {
        uint32_t v[CH];
        tmem_ld_32x32b_x32(t_buf + c0, v);
        tmem_ld_wait();
        if (c0 + CH == TN) {
          // the buffer's last columns are in registers: the MMA may refill it
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.tempty[b]);
        }
        if (m < p.M) {
#pragma unroll
          for (int j8 = 0; j8 < CH; j8 += 8) {
            const int64_t n = n0 + c0 + j8;
            if (n < p.N) {   // N % 8 == 0: the 8-wide group is fully inside or outside
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float a = kInt8 ? static_cast<float>(static_cast<int32_t>(v[j8 + e])) : __uint_as_float(v[j8 + e]);
                f[e] = a * as_r * cs[c0 + j8 + e];
              }
              if constexpr (BIAS) {
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] += bias_at(p, n + e);
              }
              const uint4 pk = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                          pack_bf16x2(f[6], f[7]));
              *reinterpret_cast<uint4*>(p.C + m * p.N + n) = pk;
              if (kInt8 && p.acc_out) {
                uint4* ao = reinterpret_cast<uint4*>(p.acc_out + m * p.N + n);
                ao[0] = make_uint4(v[j8 + 0], v[j8 + 1], v[j8 + 2], v[j8 + 3]);
                ao[1] = make_uint4(v[j8 + 4], v[j8 + 5], v[j8 + 6], v[j8 + 7]);
              }
            }
          }
        }
      }
    }
    if (warp == 2 && lane == 0) trace_stamp(p, 6);
  }

  // -------------------------------------------------------------- teardown
  tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) trace_stamp(p, 7);
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int FMT, int TN, bool BIAS>
cudaError_t launch_persistent_tc(const GemmLaunch& l) {
  auto kern = scaled_mm_persistent_kernel<FMT, TN, BIAS>;
  static int configured = 0;   // max dynamic smem set once per instantiation and process
  if (configured < l.smem_bytes) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    configured = 227 * 1024;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = l.grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(l.smem_bytes);
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (l.pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, l.tmX, l.tmY, l.p);
}

template <int FMT, bool BIAS>
cudaError_t launch_persistent(const GemmLaunch& l, int tile_n) {
  if constexpr (FMT == kFmtFp8 || FMT == kFmtInt8) {
    switch (tile_n) {
      case 64: return launch_persistent_tc<FMT, 64, BIAS>(l);
      case 128: return launch_persistent_tc<FMT, 128, BIAS>(l);
      case 256: return launch_persistent_tc<FMT, 256, BIAS>(l);
      default: return cudaErrorInvalidValue;
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace lq
