// Persistent scaled_mm on CTA pairs (tcgen05 cta_group::2) for large M:
// Standard orientation, FP8_Dynamic, W8A8_INT8, Block_FP8 with fp32 scales
// and Block_FP8 with UE8M0 scales, one split or Split-K with the separate
// fixed-order reduction.
//
// A cluster of two CTAs (two SMs) computes 256 x TN output tiles with one
// MMA of M = 256: each CTA loads its own 128 rows of A and half (TN / 2 rows)
// of B into its shared memory, the pair's first CTA issues the MMAs with
// descriptors of its own tiles (the tensor cores take the other CTA's tiles
// from the same offsets), and each CTA's tensor memory receives its 128 rows
// of the accumulator.  Per SM that is half of B's shared-memory traffic of a
// one-SM 128 x TN tile for the same work, which is what bounds the one-SM
// kernel.  As in the one-SM persistent kernel, the pair loops over tiles,
// its rings run on across tiles and the accumulator is double-buffered
// (2 x TN columns in each CTA), so each tile's epilogue overlaps the next
// tile's MMAs.  With split_k S > 1 the work units are (tile, split) pairs,
// split s covering the K blocks [s T / S, (s + 1) T / S) as in the one-SM
// kernel, and the epilogue writes the raw accumulators to the workspace
// ws[s][M][N] for splitk_reduce_kernel; that fills the SMs when a few
// 256-row tiles have a deep K (M = 256, K = 25600).
//
// Block_FP8 (fp32 block scales, 256 x 128 tiles): every 128-K block's MMA
// goes to one of four 128-column tensor-memory buffers (the MMA may run up
// to four blocks ahead), and each CTA's epilogue warps add their 128 rows of
// it, times a_s[m, kb] * b_s[n / 128, kb], into fp32 registers (fmaf in K
// order, as the one-SM kernel does: the same bits).  Per SM a 128-K block
// then moves 24 KB of operands from L2 instead of the one-SM 128 x 128
// tile's 32 KB, which is what bounds that tile.
//
// Block_FP8 with UE8M0 scales (256 x 128 tiles): the tensor core's block
// scaling (tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale), one
// accumulator per tile as for FP8.  Each CTA's tensor memory holds, at the
// same addresses, the scale factors of its own 128 rows of A and of all 128
// rows of B, in four slots of four K blocks each (row e at lane e mod 32,
// column e / 32, the same in all four lane quarters; block t of a group in
// bits [8t, 8t + 8)).  Four more warps per CTA fill the slots, so that the
// epilogue warps, busy with the previous tile, never hold up the MMA:
//   xfull[g]  first CTA only: slot g written by both CTAs' scale warps;
//   wfull[g]  both CTAs: slot g read by the tensor core (commit multicast).
// Synchronisation:
//   full[s]   first CTA only: both CTAs' TMA loads of slot s count their
//             bytes here (the first CTA announces the pair's total);
//   empty[s]  both CTAs: slot s read by the tensor core (commit multicast);
//   tfull[b]  both CTAs: accumulator buffer b complete (commit multicast;
//             per tile, or per K block for Block_FP8);
//   tempty[b] first CTA only: both CTAs' epilogue warps have read buffer b;
//   mma_done  both CTAs: every MMA of the pair finished (before teardown).
// Every wait is bounded; the CTAs pass two cluster barriers (after set-up,
// before teardown) on every path.  Results equal the one-SM kernels' up to
// the tensor core's order of accumulation within an MMA of twice the rows:
// per output the same MMA sequence over K, so the same bits.
#pragma once

#include "scaled_mm_persistent.cuh"

namespace lq {

constexpr int kPairTileM = 256;

template <int TN>
struct PairShape {
  static constexpr int kABytes = kTileM * kTileK;              // this CTA's 128 rows of A
  static constexpr int kBBytes = (TN / 2) * kTileK;            // this CTA's half of B
  static constexpr int kStageBytes = kABytes + kBBytes;
};

template <int TN>
__host__ __device__ constexpr int pair_smem_bytes(int stages) {
  return 1024 + stages * PairShape<TN>::kStageBytes + kCtlBytes + kPersistentScaleBytes;
}

// Threads of a pair CTA: producer, MMA and four epilogue warps, and for the
// UE8M0 format four scale-factor warps.
__host__ __device__ constexpr int pair_threads(int fmt) { return fmt == kFmtBlockE8m0 ? kThreads + 128 : kThreads; }

constexpr int kPairSfSlots = 4;

template <int FMT, int TN, bool BIAS>
__global__ void __launch_bounds__(pair_threads(FMT), 1)
    scaled_mm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const GemmParams p) {
  static_assert(FMT == kFmtFp8 || FMT == kFmtInt8 || FMT == kFmtBlock || FMT == kFmtBlockE8m0,
                "pair kernel: FP8, INT8, Block_FP8 (fp32 or UE8M0 scales)");
  static_assert(TN == 128 || TN == 256, "pair tiles: 256 x 128 or 256 x 256");
  constexpr bool kPromote = FMT == kFmtBlock;
  constexpr bool kMX = FMT == kFmtBlockE8m0;
  static_assert(!kPromote || TN == 128, "Block_FP8 pairs: 256 x 128 tiles (TN fp32 accumulators per thread)");
  static_assert(!kMX || TN == 128, "UE8M0 pairs: 256 x 128 tiles (two accumulators and the scale factors)");
  using Shape = PairShape<TN>;
  constexpr bool kInt8 = FMT == kFmtInt8;
  constexpr int kNBuf = kPromote ? 4 : 2;     // tensor-memory accumulator buffers
  constexpr int kSfBase = kNBuf * TN;         // UE8M0: scale-factor slots after the accumulators
  constexpr int kSfSlotCols = 8;              // A: 4 columns (128 rows), B: 4 columns (TN = 128 rows)
  constexpr int kTmemCols = kMX ? 512 : kNBuf * TN;
  static_assert(!kMX || kSfBase + kPairSfSlots * kSfSlotCols <= kTmemCols, "tensor memory");
  constexpr int CH = 32;
  constexpr uint16_t kPairMask = 0x3;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  const int stages = p.stages;
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + stages * Shape::kStageBytes);
  SmemCtl c;
  c.full = bars;
  c.empty = bars + stages;
  c.tfull = bars + 2 * stages;
  c.tempty = c.tfull + kNBuf;
  c.mma_done = c.tempty + kNBuf;
  c.xfull = c.mma_done + 1;              // UE8M0 scale-factor slots (unused otherwise)
  c.wfull = c.xfull + kPairSfSlots;
  c.tmem_slot = reinterpret_cast<uint32_t*>(c.wfull + kPairSfSlots);
  c.abort_flag = reinterpret_cast<volatile int*>(c.tmem_slot + 1);
  c.last_flag = c.abort_flag + 1;
  float* colsc = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kCtlBytes);   // [2][256]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();                // 0: issues the MMAs
  const bool leader = rank == 0;
  const int64_t gx = (p.M + kPairTileM - 1) / kPairTileM;   // 256-row blocks
  const int64_t gy = (p.N + TN - 1) / TN;
  const int64_t tiles = gx * gy;
  const int S = p.S;
  const int64_t units = tiles * S;   // unit u: tile u mod tiles, split u / tiles
  const int64_t pair = blockIdx.x >> 1;
  const int64_t npairs = gridDim.x >> 1;
  const int64_t my_tiles = units > pair ? (units - pair + npairs - 1) / npairs : 0;
  const int T = p.T;
  const bool split_mode = S > 1;
  auto tile_origin = [&](int64_t j, int64_t* m0, int64_t* n0) {
    const int64_t t = (pair + j * npairs) % tiles;
    *m0 = (t % gx) * kPairTileM;
    *n0 = (t / gx) * TN;
  };
  auto split_of = [&](int64_t j) { return static_cast<int>((pair + j * npairs) / tiles); };
  auto kb_begin = [&](int s) { return static_cast<int>((static_cast<int64_t>(s) * T) / S); };

  if (threadIdx.x == 0) trace_stamp(p, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int b = 0; b < kNBuf; ++b) {
      mbar_init(&c.tfull[b], 1);
      mbar_init(&c.tempty[b], 2 * kEpiThreads / 32);
    }
    mbar_init(c.mma_done, 1);
    for (int g = 0; g < kPairSfSlots; ++g) {
      mbar_init(&c.xfull[g], 8);   // four scale warps in each CTA
      mbar_init(&c.wfull[g], 1);
    }
    *c.abort_flag = 0;
    *c.last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensor_map(&tmA);
    prefetch_tensor_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(c.tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync_all();   // both CTAs' barriers exist and the pair's tensor memory is allocated
  tc_fence_after_sync();
  const uint32_t tmem_base = *c.tmem_slot;
  if (threadIdx.x == 0) trace_stamp(p, 1);
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      const uint32_t full0 = dsmem_map(smem_addr(c.full), 0);   // the first CTA's full[0]
      int64_t it = 0;
      int64_t issued = 0;
      bool go = true;
      grid_dependency_wait();   // the activations come from the previous kernel
      trace_stamp(p, 2);
      for (int64_t j = 0; j < my_tiles && go; ++j) {
        int64_t m0, n0;
        tile_origin(j, &m0, &n0);
        const int32_t a_row = static_cast<int32_t>(m0 + rank * kTileM);
        const int32_t b_row = static_cast<int32_t>(n0 + rank * (TN / 2));
        const int sp = split_of(j);
        const int kb_hi = kb_begin(sp + 1);
        for (int kb = kb_begin(sp); kb < kb_hi; ++kb, ++it) {
          const int s = static_cast<int>(it % stages);
          const uint32_t ph = static_cast<uint32_t>(it / stages) & 1u;
          if (!wait_bar(&c.empty[s], ph ^ 1u, p, c, 0)) {
            go = false;
            break;
          }
          uint8_t* st = ring + s * Shape::kStageBytes;
          const uint32_t fbar = full0 + static_cast<uint32_t>(s * 8);
          if (leader) mbar_arrive_expect_tx(&c.full[s], 2 * Shape::kStageBytes);   // both CTAs' bytes
          tma_load_2d_pair(&tmA, fbar, st, kb * kTileK, a_row, pol_a);
          tma_load_2d_pair(&tmB, fbar, st + Shape::kABytes, kb * kTileK, b_row, pol_w);
          issued = it + 1;
        }
      }
      if (*c.abort_flag && leader) {
        // Drain: wait (bounded) until the pair's copies still in flight have
        // landed (each slot's barrier counts both CTAs' bytes).
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
    // ------------------------------------------------ MMA issuer (first CTA)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = make_idesc<kInt8>(kPairTileM, TN);
      constexpr uint32_t idesc_mx = make_idesc_mx(kPairTileM, TN);
      bool issued_any = false;
      bool go = true;
      int64_t it = 0;
      if constexpr (kPromote) {
        // one accumulator buffer per 128-K block, buffers in turn across units
        for (int64_t j = 0; j < my_tiles && go; ++j) {
          const int sp = split_of(j);
          const int kb_hi = kb_begin(sp + 1);
          for (int kb = kb_begin(sp); kb < kb_hi; ++kb, ++it) {
            const int b = static_cast<int>(it % kNBuf);
            const uint32_t use = static_cast<uint32_t>(it / kNBuf);
            if (!wait_bar<true>(&c.tempty[b], (use & 1u) ^ 1u, p, c, 1)) {
              go = false;
              break;
            }
            const int s = static_cast<int>(it % stages);
            const uint32_t ph = static_cast<uint32_t>(it / stages) & 1u;
            if (!wait_bar(&c.full[s], ph, p, c, 2)) {
              go = false;
              break;
            }
            tc_fence_after_sync();
            if (it == 0) trace_stamp(p, 3);
            uint8_t* st = ring + s * Shape::kStageBytes;
            const uint64_t ad = smem_desc_k_sw128(st);
            const uint64_t bd = smem_desc_k_sw128(st + Shape::kABytes);
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * TN);
#pragma unroll
            for (int kk = 0; kk < kTileK / kMmaK; ++kk)
              mma_f8f6f4_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, kk > 0 ? 1u : 0u);
            issued_any = true;
            mma_commit_pair_multicast(&c.empty[s], kPairMask);
            mma_commit_pair_multicast(&c.tfull[b], kPairMask);
          }
        }
      }
      // UE8M0: the scale-factor slot of the current group of four K blocks
      // (groups start at each unit's first block), its use count, its address
      int64_t sf_group = -1;
      uint32_t sf_addr = tmem_base + static_cast<uint32_t>(kSfBase);
      int sf_slot = 0;
      for (int64_t j = 0; j < my_tiles && go && !kPromote; ++j) {
        const int b = static_cast<int>(j & 1);
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        // both CTAs' epilogues have read tile j - 2 (arrivals of both CTAs: cluster scope)
        if (!wait_bar<true>(&c.tempty[b], (use & 1u) ^ 1u, p, c, 1)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * TN);
        const int sp = split_of(j);
        const int kb_lo = kb_begin(sp);
        const int kb_hi = kb_begin(sp + 1);
        for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
          if (kMX && ((kb - kb_lo) & 3) == 0) {   // both CTAs' scale factors of blocks kb .. kb+3
            ++sf_group;
            sf_slot = static_cast<int>(sf_group % kPairSfSlots);
            sf_addr = tmem_base + static_cast<uint32_t>(kSfBase + sf_slot * kSfSlotCols);
            const uint32_t sf_ph = static_cast<uint32_t>(sf_group / kPairSfSlots) & 1u;
            if (!wait_bar<true>(&c.xfull[sf_slot], sf_ph, p, c, 13)) {
              go = false;
              break;
            }
          }
          const int s = static_cast<int>(it % stages);
          const uint32_t ph = static_cast<uint32_t>(it / stages) & 1u;
          if (!wait_bar(&c.full[s], ph, p, c, 2)) {
            go = false;
            break;
          }
          tc_fence_after_sync();
          if (it == 0) trace_stamp(p, 3);
          uint8_t* st = ring + s * Shape::kStageBytes;
          const uint64_t ad = smem_desc_k_sw128(st);
          const uint64_t bd = smem_desc_k_sw128(st + Shape::kABytes);
#pragma unroll
          for (int kk = 0; kk < kTileK / kMmaK; ++kk) {
            const uint32_t acc = (kb > kb_lo || kk > 0);
            if constexpr (kMX) {
              const uint32_t t = static_cast<uint32_t>((kb - kb_lo) & 3);   // this block's byte in the slot
              mma_mxf8f6f4_block_scale_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc_with_sf_ids(idesc_mx, t, t),
                                            sf_addr, sf_addr + 4, acc);
            } else if (kInt8) {
              mma_i8_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, acc);
            } else {
              mma_f8f6f4_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, acc);
            }
          }
          issued_any = true;
          mma_commit_pair_multicast(&c.empty[s], kPairMask);
          if (kMX && (((kb - kb_lo) & 3) == 3 || kb + 1 == kb_hi))
            mma_commit_pair_multicast(&c.wfull[sf_slot], kPairMask);   // the slot is read
        }
        // (a unit with no K blocks commits at once; its epilogue stores zeros)
        if (go) mma_commit_pair_multicast(&c.tfull[b], kPairMask);
      }
      trace_stamp(p, 4);
      (void)issued_any;
      // arrives once every MMA issued so far has finished (at once if none was)
      if (my_tiles > 0) mma_commit_pair_multicast(c.mma_done, kPairMask);
    }
  } else if (warp < kThreads / 32) {
    // ------------------------------------------------------------ epilogue
    grid_dependency_wait();   // the scales may come from the previous kernel
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tempty0 = dsmem_map(smem_addr(c.tempty), 0);   // the first CTA's tempty[0]
    bool ok = true;
    if constexpr (kPromote) {
      // Block scale products of this thread's row, a group of kPre K blocks
      // ahead (the loads' latency hides behind a group of promotions).
      constexpr int kPre = 8;
      static_assert(kPre == 8, "two float4 scale loads per group");
      const bool vec_scales = (p.KB & 3) == 0 &&
                              ((reinterpret_cast<uintptr_t>(p.a_s) | reinterpret_cast<uintptr_t>(p.b_s)) & 15u) == 0;
      int64_t g = 0;   // running K block over all units: buffer g mod kNBuf
      for (int64_t j = 0; j < my_tiles; ++j) {
        int64_t m0, n0;
        tile_origin(j, &m0, &n0);
        const int sp = split_of(j);
        const int kb_lo = kb_begin(sp);
        const int nkb = kb_begin(sp + 1) - kb_lo;
        const int64_t m = m0 + rank * kTileM + r;
        const int64_t nb = n0 / 128;
        auto load_scale = [&](int i) -> float {   // 0 past the unit's blocks
          if (i >= nkb) return 0.f;
          const int64_t kb = kb_lo + i;
          const float sb = __ldg(p.b_s + nb * p.KB + kb);
          return (m < p.M ? __ldg(p.a_s + m * p.KB + kb) : 0.f) * sb;
        };
        // The kPre products of blocks i .. i + kPre - 1: where the group lies
        // inside the unit and its first block is 16-byte aligned, a row's
        // scales come as two float4 loads (a quarter of the load requests,
        // each warp instruction touching one cache line per row, on the L1 /
        // shared-memory path the MMA's operands use).  The same products.
        auto load_group = [&](int i, float (&out)[kPre]) {
          const int64_t kb0 = kb_lo + i;
          if (vec_scales && (kb0 & 3) == 0 && i + kPre <= nkb) {
            const float4* bp = reinterpret_cast<const float4*>(p.b_s + nb * p.KB + kb0);
            const float4 b0 = __ldg(bp), b1 = __ldg(bp + 1);
            float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
            if (m < p.M) {
              const float4* ap = reinterpret_cast<const float4*>(p.a_s + m * p.KB + kb0);
              a0 = __ldg(ap);
              a1 = __ldg(ap + 1);
            }
            out[0] = a0.x * b0.x; out[1] = a0.y * b0.y; out[2] = a0.z * b0.z; out[3] = a0.w * b0.w;
            out[4] = a1.x * b1.x; out[5] = a1.y * b1.y; out[6] = a1.z * b1.z; out[7] = a1.w * b1.w;
            return;
          }
#pragma unroll
          for (int e = 0; e < kPre; ++e) out[e] = load_scale(i + e);
        };
        float accr[TN];
#pragma unroll
        for (int e = 0; e < TN; ++e) accr[e] = 0.f;
        float cur[kPre], nxt[kPre];
        load_group(0, cur);
        for (int i0 = 0; i0 < nkb; i0 += kPre) {
          load_group(i0 + kPre, nxt);
#pragma unroll
          for (int e = 0; e < kPre; ++e) {
            if (i0 + e < nkb) {   // the same for every epilogue thread
              const int b = static_cast<int>(g % kNBuf);
              const uint32_t use = static_cast<uint32_t>(g / kNBuf);
              ++g;
              // warp-uniform decision: the tcgen05.ld below is .sync.aligned
              if (ok) ok = __all_sync(0xffffffffu, wait_bar(&c.tfull[b], use & 1u, p, c, 4) && !*c.abort_flag);
              if (ok) {
                tc_fence_after_sync();
                const uint32_t t_buf = t_row + static_cast<uint32_t>(b * TN);
                // two loads in flight per wait (a round trip is most of a load's cost)
#pragma unroll
                for (int c0 = 0; c0 < TN; c0 += 2 * CH) {
                  uint32_t v0[CH], v1[CH];
                  tmem_ld_32x32b_x32(t_buf + c0, v0);
                  tmem_ld_32x32b_x32(t_buf + c0 + CH, v1);
                  tmem_ld_wait();
                  if (c0 + 2 * CH == TN) {
                    // The block's partial is in registers: the pair's MMA may refill
                    // the buffer (before the last multiply-adds: the MMA-epilogue
                    // hand-off per block is what bounds this kernel).  The arrive
                    // publishes no memory writes, so it needs no release fence (one
                    // per block and warp cost hundreds of cycles).
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + static_cast<uint32_t>(b * 8));
                  }
#pragma unroll
                  for (int jj = 0; jj < CH; ++jj) {
                    accr[c0 + jj] = fmaf(__uint_as_float(v0[jj]), cur[e], accr[c0 + jj]);
                    accr[c0 + CH + jj] = fmaf(__uint_as_float(v1[jj]), cur[e], accr[c0 + CH + jj]);
                  }
                }
              }
            }
          }
#pragma unroll
          for (int e = 0; e < kPre; ++e) cur[e] = nxt[e];
        }
        if (!ok || m >= p.M) continue;
#pragma unroll
        for (int j8 = 0; j8 < TN; j8 += 8) {
          const int64_t n = n0 + j8;
          if (n >= p.N) break;
          if (split_mode) {   // the unit's promoted partial; the reduction adds the splits in order
            uint4* wo = reinterpret_cast<uint4*>(static_cast<float*>(p.ws) + (sp * p.M + m) * p.N + n);
            wo[0] = make_uint4(__float_as_uint(accr[j8 + 0]), __float_as_uint(accr[j8 + 1]),
                               __float_as_uint(accr[j8 + 2]), __float_as_uint(accr[j8 + 3]));
            wo[1] = make_uint4(__float_as_uint(accr[j8 + 4]), __float_as_uint(accr[j8 + 5]),
                               __float_as_uint(accr[j8 + 6]), __float_as_uint(accr[j8 + 7]));
          } else {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = accr[j8 + e];
            if constexpr (BIAS) {
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] += bias_at(p, n + e);
            }
            *reinterpret_cast<uint4*>(p.C + m * p.N + n) =
                make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                           pack_bf16x2(f[6], f[7]));
          }
        }
      }
    }
    for (int64_t j = 0; j < my_tiles && !kPromote; ++j) {
      const int b = static_cast<int>(j & 1);
      const uint32_t use = static_cast<uint32_t>(j >> 1);
      int64_t m0, n0;
      tile_origin(j, &m0, &n0);
      const int sp = split_of(j);
      const bool empty_unit = kb_begin(sp + 1) == kb_begin(sp);
      float* cs = colsc + b * 256;
      // (UE8M0: the accumulator carries its scales, and the scale arrays hold bytes)
      if (!split_mode && !kMX)
        for (int col = r; col < TN; col += kEpiThreads) cs[col] = n0 + col < p.N ? __ldg(p.b_s + n0 + col) : 0.f;
      const int64_t m = m0 + rank * kTileM + r;
      const float as_r = (m < p.M && !split_mode && !kMX) ? __ldg(p.a_s + m) : 0.f;
      named_barrier_sync(2, kEpiThreads);
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(&c.tfull[b], use & 1u, p, c, 5) && !*c.abort_flag);
      if (!ok) continue;
      tc_fence_after_sync();
      const uint32_t t_buf = t_row + static_cast<uint32_t>(b * TN);
#pragma unroll
      for (int c0 = 0; c0 < TN; c0 += CH) {
        uint32_t v[CH];
        if (!empty_unit) {
          tmem_ld_32x32b_x32(t_buf + c0, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < CH; ++e) v[e] = 0u;   // a split with no K blocks: zero partial
        }
        if (c0 + CH == TN) {
          // the buffer's last columns are in registers: the pair's MMA may refill it
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty0 + static_cast<uint32_t>(b * 8));
        }
        if (m < p.M) {
#pragma unroll
          for (int j8 = 0; j8 < CH; j8 += 8) {
            const int64_t n = n0 + c0 + j8;
            if (n < p.N && split_mode) {
              // raw accumulators (fp32 or int32 bits); the reduction scales them
              uint4* wo = reinterpret_cast<uint4*>(static_cast<uint32_t*>(p.ws) + (sp * p.M + m) * p.N + n);
              wo[0] = make_uint4(v[j8 + 0], v[j8 + 1], v[j8 + 2], v[j8 + 3]);
              wo[1] = make_uint4(v[j8 + 4], v[j8 + 5], v[j8 + 6], v[j8 + 7]);
            } else if (n < p.N) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float a = kInt8 ? static_cast<float>(static_cast<int32_t>(v[j8 + e])) : __uint_as_float(v[j8 + e]);
                f[e] = kMX ? a : a * as_r * cs[c0 + j8 + e];
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
                ao[0] = make_uint4(v[j8 + 0], v[j8 + 1], v[j8 + 2], v[j8 + 3]);
                ao[1] = make_uint4(v[j8 + 4], v[j8 + 5], v[j8 + 6], v[j8 + 7]);
              }
            }
          }
        }
      }
    }
    if (warp == 2 && lane == 0) trace_stamp(p, 6);
  } else if constexpr (kMX) {
    // --------------------------------------------- UE8M0 scale-factor warps
    // Per group of four K blocks of each unit (the MMA warp's grouping):
    // wait until the slot's previous group has been read (wfull, from the
    // pair's commits), write the UE8M0 bytes of this CTA's 128 A rows and of
    // the tile's 128 B rows to this warp's lane quarter of the slot, and
    // arrive on the first CTA's xfull (release: the tensor-memory stores,
    // complete after tcgen05.wait::st, come before the MMA that reads them).
    grid_dependency_wait();   // the scales may come from the previous kernel
    const int q = warp & 3;   // warps 6..9: lane quarters 2, 3, 0, 1
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t xfull0 = dsmem_map(smem_addr(c.xfull), 0);   // the first CTA's xfull[0]
    const uint8_t* a_b = reinterpret_cast<const uint8_t*>(p.a_s);   // [M, KB]
    const uint8_t* b_b = reinterpret_cast<const uint8_t*>(p.b_s);   // [N / 128, KB]
    const bool words = (p.KB & 3) == 0 && ((reinterpret_cast<uintptr_t>(a_b) | reinterpret_cast<uintptr_t>(b_b)) & 3u) == 0;
    bool ok = true;
    int64_t group = -1;
    for (int64_t j = 0; j < my_tiles && ok; ++j) {
      int64_t m0, n0;
      tile_origin(j, &m0, &n0);
      const int sp = split_of(j);
      const int kb_hi = kb_begin(sp + 1);
      for (int kb0 = kb_begin(sp); kb0 < kb_hi; kb0 += 4) {
        ++group;
        const int slot = static_cast<int>(group % kPairSfSlots);
        if (group >= kPairSfSlots) {
          const uint32_t ph = static_cast<uint32_t>(group / kPairSfSlots - 1) & 1u;
          ok = __all_sync(0xffffffffu, wait_bar(&c.wfull[slot], ph, p, c, 14) && !*c.abort_flag);
          if (!ok) break;
        }
        uint32_t wa[4], wb[4];
        // a row's four bytes as one 32-bit load where the group is whole and aligned
        const bool word = words && (kb0 & 3) == 0 && kb0 + 4 <= kb_hi;
#pragma unroll
        for (int col = 0; col < 4; ++col) {
          const int64_t m = m0 + rank * kTileM + col * 32 + lane;
          const int64_t n = n0 + col * 32 + lane;
          if (word) {
            wa[col] = m < p.M ? __ldg(reinterpret_cast<const uint32_t*>(a_b + m * p.KB + kb0)) : 0x7F7F7F7Fu;
            wb[col] = n < p.N ? __ldg(reinterpret_cast<const uint32_t*>(b_b + (n >> 7) * p.KB + kb0)) : 0x7F7F7F7Fu;
            continue;
          }
          uint32_t xa = 0, xb = 0;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int kb = kb0 + t;   // past the unit's blocks or the matrix: 127 (a factor of one)
            const uint32_t ba = (kb < kb_hi && m < p.M) ? a_b[m * p.KB + kb] : 127u;
            const uint32_t bb = (kb < kb_hi && n < p.N) ? b_b[(n >> 7) * p.KB + kb] : 127u;
            xa |= ba << (8 * t);
            xb |= bb << (8 * t);
          }
          wa[col] = xa;
          wb[col] = xb;
        }
        tc_fence_after_sync();
        const uint32_t col0 = t_row + static_cast<uint32_t>(kSfBase + slot * kSfSlotCols);
        tmem_st_32x32b_x4(col0, wa);
        tmem_st_32x32b_x4(col0 + 4, wb);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(xfull0 + static_cast<uint32_t>(slot * 8));
      }
    }
  }

  // -------------------------------------------------------------- teardown
  // Every MMA of the pair must be finished before either CTA leaves (they
  // read both CTAs' shared memory and write both tensor memories).
  if (warp == 1 && lane == 0 && my_tiles > 0) wait_bar(c.mma_done, 0, p, c, 3);
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync_all();
  if (threadIdx.x == 0) trace_stamp(p, 7);
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int FMT, int TN, bool BIAS>
cudaError_t launch_pair_tc(const GemmLaunch& l) {
  auto kern = scaled_mm_pair_kernel<FMT, TN, BIAS>;
  static int configured = 0;
  if (configured < l.smem_bytes) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    configured = 227 * 1024;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = l.grid;
  cfg.blockDim = dim3(pair_threads(FMT), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(l.smem_bytes);
  cfg.stream = l.stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 2;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (l.pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, l.tmX, l.tmY, l.p);
}

// Largest number of co-resident pairs for (FMT, TN, BIAS) with `smem_bytes`.
template <int FMT, int TN, bool BIAS>
int max_pairs(int smem_bytes) {
  auto kern = scaled_mm_pair_kernel<FMT, TN, BIAS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(pair_threads(FMT), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int FMT, bool BIAS>
cudaError_t launch_pair(const GemmLaunch& l, int tile_n) {
  if constexpr (FMT == kFmtFp8 || FMT == kFmtInt8) {
    switch (tile_n) {
      case 128: return launch_pair_tc<FMT, 128, BIAS>(l);
      case 256: return launch_pair_tc<FMT, 256, BIAS>(l);
      default: return cudaErrorInvalidValue;
    }
  }
  if constexpr (FMT == kFmtBlock || FMT == kFmtBlockE8m0) {
    if (tile_n == 128) return launch_pair_tc<FMT, 128, BIAS>(l);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lq
