// Stream-K scaled_mm for large M with few output tiles (Standard
// orientation, FP8_Dynamic / W8A8_INT8).
//
// When the output has fewer tiles than SMs, or a few more (Qwen3-32B down at
// M = 256: 40 tiles of 128 x 256, 200 K blocks each), one tile per CTA
// leaves SMs idle or runs a short second wave, and Split-K only moves the
// problem.  Here the grid's CTAs (at most one per SM) split the whole
// iteration space, tiles x K blocks in tile-major order, into equal
// contiguous ranges.  A CTA walks its range as segments, one per tile it
// touches, each accumulated in one of two tensor-memory buffers:
//   - a segment covering a whole tile is scaled and stored;
//   - a segment that ends before its tile's last K block (the CTA's range
//     ends inside the tile) is written unscaled to the CTA's workspace slot
//     [128 x TN] and published with a flag;
//   - a segment that holds a tile's last K block but not its first is the
//     tile's finisher: it waits for the flags of the CTAs that cover the
//     tile's earlier K blocks (all of lower index), adds their partials in
//     increasing CTA order (that is, increasing K) followed by its own,
//     clears the flags, scales and stores.
// So every output is a fixed-order sum (INT8 partials are int32: exact), and
// a CTA only ever waits for lower-index CTAs, which never wait for it.  The
// waits are bounded; CTAs that cannot finish set the status word.  The flags
// start at zero and are cleared by their one reader, so every launch (and
// every replay of a captured graph) starts from zero.
#pragma once

#include "scaled_mm_persistent.cuh"

namespace lq {

template <int FMT, int TN, bool BIAS>
__global__ void __launch_bounds__(kThreads, 1)
    scaled_mm_streamk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const GemmParams p) {
  static_assert(FMT == kFmtFp8 || FMT == kFmtInt8, "stream-K kernel: FP8_Dynamic / W8A8_INT8");
  using Shape = TileShape<TN>;
  constexpr bool kInt8 = FMT == kFmtInt8;
  constexpr int kTmemCols = tmem_cols_for(2 * TN);
  constexpr int CH = 32;

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
  const int64_t gx = (p.M + kTileM - 1) / kTileM;
  const int64_t gy = (p.N + TN - 1) / TN;
  const int64_t T = p.T;
  const int64_t iters = gx * gy * T;
  const int64_t G = gridDim.x;
  const int64_t cta = blockIdx.x;
  auto range_lo = [&](int64_t k) -> int64_t { return k * iters / G; };
  const int64_t lo = range_lo(cta), hi = range_lo(cta + 1);
  auto tile_origin = [&](int64_t t, int64_t* m0, int64_t* n0) {
    *m0 = (t % gx) * kTileM;
    *n0 = (t / gx) * TN;
  };
  // the CTA whose range holds iteration x
  auto owner_of = [&](int64_t x) -> int64_t {
    int64_t k = x * G / iters;
    while (k > 0 && range_lo(k) > x) --k;
    while (k + 1 < G && range_lo(k + 1) <= x) ++k;
    return k;
  };
  // segments of this CTA's range: (tile, first K block, end K block)
  auto segment = [&](int64_t x, int64_t* t, int64_t* kb0, int64_t* kb1) {
    *t = x / T;
    *kb0 = x - *t * T;
    const int64_t left = hi - x;
    *kb1 = *kb0 + left < T ? *kb0 + left : T;
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
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      grid_dependency_wait();
      trace_stamp(p, 2);
      int64_t issued = 0;
      for (int64_t x = lo, it = 0; x < hi; ++x, ++it) {
        const int64_t t = x / T, kb = x - t * T;
        int64_t m0, n0;
        tile_origin(t, &m0, &n0);
        const int s = static_cast<int>(it % stages);
        const uint32_t ph = static_cast<uint32_t>(it / stages) & 1u;
        if (!wait_bar(&c.empty[s], ph ^ 1u, p, c, 0)) break;
        uint8_t* st = ring + s * Shape::kStageBytes;
        mbar_arrive_expect_tx(&c.full[s], Shape::kStageBytes);
        tma_load_2d(&tmA, &c.full[s], st, static_cast<int32_t>(kb * kTileK), static_cast<int32_t>(m0), pol_a);
        tma_load_2d(&tmB, &c.full[s], st + Shape::kXBytes, static_cast<int32_t>(kb * kTileK), static_cast<int32_t>(n0),
                    pol_w);
        issued = it + 1;
      }
      if (*c.abort_flag) {
        const int64_t first = issued > stages ? issued - stages : 0;
        for (int64_t q = first; q < issued; ++q) {
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
      int64_t j = 0;   // segment index
      for (int64_t x = lo; x < hi && go; ++j) {
        int64_t t, kb0, kb1;
        segment(x, &t, &kb0, &kb1);
        const int b = static_cast<int>(j & 1);
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        if (!wait_bar(&c.tempty[b], (use & 1u) ^ 1u, p, c, 1)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * TN);
        for (int64_t kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = static_cast<int>(it % stages);
          const uint32_t ph = static_cast<uint32_t>(it / stages) & 1u;
          if (!wait_bar(&c.full[s], ph, p, c, 2)) {
            go = false;
            break;
          }
          tc_fence_after_sync();
          uint8_t* st = ring + s * Shape::kStageBytes;
          const uint64_t xd = smem_desc_k_sw128(st);
          const uint64_t yd = smem_desc_k_sw128(st + Shape::kXBytes);
#pragma unroll
          for (int kk = 0; kk < kTileK / kMmaK; ++kk) {
            const uint32_t acc = (kb > kb0 || kk > 0);
            if (kInt8)
              mma_i8(d_tmem, xd + 2 * kk, yd + 2 * kk, idesc, acc);
            else
              mma_f8f6f4(d_tmem, xd + 2 * kk, yd + 2 * kk, idesc, acc);
          }
          issued_any = true;
          mma_commit(&c.empty[s]);
        }
        if (go) mma_commit(&c.tfull[b]);
        x += kb1 - kb0;
      }
      trace_stamp(p, 4);
      if (issued_any) {
        mma_commit(c.mma_done);
        wait_bar(c.mma_done, 0, p, c, 3);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    grid_dependency_wait();
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t* ws_mine = reinterpret_cast<uint32_t*>(p.ws) + cta * (kTileM * TN) + static_cast<int64_t>(r) * TN;
    volatile int* flags = p.counters;
    bool ok = true;
    int64_t j = 0;
    for (int64_t x = lo; x < hi; ++j) {
      int64_t t, kb0, kb1;
      segment(x, &t, &kb0, &kb1);
      x += kb1 - kb0;
      const int b = static_cast<int>(j & 1);
      const uint32_t use = static_cast<uint32_t>(j >> 1);
      int64_t m0, n0;
      tile_origin(t, &m0, &n0);
      const bool publish = kb1 < T;                 // the tile is finished by a later CTA
      const bool finish_others = !publish && kb0 > 0;
      const int64_t c_first = finish_others ? owner_of(t * T) : cta;
      float* cs = colsc + b * 256;
      for (int col = r; col < TN; col += kEpiThreads) cs[col] = n0 + col < p.N ? __ldg(p.b_s + n0 + col) : 0.f;
      const int64_t m = m0 + r;
      const float as_r = m < p.M ? __ldg(p.a_s + m) : 0.f;
      // the finisher first waits (bounded) for every earlier CTA's partial of this tile
      if (finish_others && threadIdx.x == 64 && ok && !*c.abort_flag) {
        for (int64_t k = c_first; k < cta; ++k) {
          const uint64_t t0 = global_timer_ns();
          while (flags[k] == 0) {
            if (global_timer_ns() - t0 > p.wait_limit_ns) {
              *c.abort_flag = 1;
              report_timeout(p, 15);
              break;
            }
          }
          if (*c.abort_flag) break;
        }
        __threadfence();
      }
      named_barrier_sync(2, kEpiThreads);
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(&c.tfull[b], use & 1u, p, c, 5) && !*c.abort_flag);
      if (!ok) {
        named_barrier_sync(2, kEpiThreads);   // matches the publish / clear barrier below
        continue;
      }
      tc_fence_after_sync();
      const uint32_t t_buf = t_row + static_cast<uint32_t>(b * TN);
#pragma unroll
      for (int c0 = 0; c0 < TN; c0 += CH) {
        uint32_t v[CH];
        tmem_ld_32x32b_x32(t_buf + c0, v);
        tmem_ld_wait();
        if (c0 + CH == TN) {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.tempty[b]);
        }
        if (publish) {   // unscaled partial of this segment, row r
#pragma unroll
          for (int j4 = 0; j4 < CH; j4 += 4)
            __stcg(reinterpret_cast<uint4*>(ws_mine + c0 + j4), make_uint4(v[j4], v[j4 + 1], v[j4 + 2], v[j4 + 3]));
          continue;
        }
        // the sum in increasing K order: earlier CTAs' partials, then this one's
        float fs[CH];
        int32_t is[CH];
#pragma unroll
        for (int e = 0; e < CH; ++e) {
          fs[e] = 0.f;
          is[e] = 0;
        }
        if (finish_others) {
          for (int64_t k = c_first; k < cta; ++k) {
            const uint32_t* src = reinterpret_cast<const uint32_t*>(p.ws) + k * (kTileM * TN) + static_cast<int64_t>(r) * TN + c0;
#pragma unroll
            for (int j4 = 0; j4 < CH; j4 += 4) {
              const uint4 w = __ldcg(reinterpret_cast<const uint4*>(src + j4));
              const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                if (kInt8) is[j4 + e] += static_cast<int32_t>(wv[e]);
                else fs[j4 + e] += __uint_as_float(wv[e]);
              }
            }
          }
        }
#pragma unroll
        for (int e = 0; e < CH; ++e) {
          if (kInt8) is[e] += static_cast<int32_t>(v[e]);
          else fs[e] = finish_others ? fs[e] + __uint_as_float(v[e]) : __uint_as_float(v[e]);
        }
        if (m < p.M) {
#pragma unroll
          for (int j8 = 0; j8 < CH; j8 += 8) {
            const int64_t n = n0 + c0 + j8;
            if (n < p.N) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float a = kInt8 ? static_cast<float>(is[j8 + e]) : fs[j8 + e];
                f[e] = a * as_r * cs[c0 + j8 + e];
              }
              if constexpr (BIAS) {
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] += bias_at(p, n + e);
              }
              *reinterpret_cast<uint4*>(p.C + m * p.N + n) =
                  make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                             pack_bf16x2(f[6], f[7]));
              if (kInt8 && p.acc_out) {
                uint4* ao = reinterpret_cast<uint4*>(p.acc_out + m * p.N + n);
                ao[0] = make_uint4(is[j8 + 0], is[j8 + 1], is[j8 + 2], is[j8 + 3]);
                ao[1] = make_uint4(is[j8 + 4], is[j8 + 5], is[j8 + 6], is[j8 + 7]);
              }
            }
          }
        }
      }
      // publish this CTA's partial, or release the partials it has consumed
      __threadfence();
      named_barrier_sync(2, kEpiThreads);
      if (threadIdx.x == 64) {
        if (publish) {
          atomicExch(const_cast<int*>(flags) + cta, 1);
        } else if (finish_others) {
          for (int64_t k = c_first; k < cta; ++k) atomicExch(const_cast<int*>(flags) + k, 0);
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
cudaError_t launch_streamk_tc(const GemmLaunch& l) {
  auto kern = scaled_mm_streamk_kernel<FMT, TN, BIAS>;
  static int configured = 0;
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
cudaError_t launch_streamk(const GemmLaunch& l, int tile_n) {
  if constexpr (FMT == kFmtFp8 || FMT == kFmtInt8) {
    switch (tile_n) {
      case 128: return launch_streamk_tc<FMT, 128, BIAS>(l);
      case 256: return launch_streamk_tc<FMT, 256, BIAS>(l);
      default: return cudaErrorInvalidValue;
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace lq
