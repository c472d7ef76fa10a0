// scaled_mm on sm_100a: a TMA -> shared-memory ring -> tcgen05.mma -> TMEM
// pipeline, one output tile per CTA.
//
// Operation (PyTorch blog "Building a High-Performance and Portable vLLM
// Linear Backend with Helion", "Helion Linear Backend > Scope" for the
// formats and "Kernel Implementation" for the variants):
//
//   C[m, n] = bf16( a_s . b_s . sum_k A[m, k] B[n, k] )          FP8 / INT8
//   C[m, n] = bf16( sum_kb a_s[m, kb] b_s[n/128, kb]
//                          sum_{k in kb} A[m, k] B[n, k] )         Block_FP8
//
// The tensor core computes D[128 x TN] = X[128 x Kt] . Y[TN x Kt]^T from two
// K-major shared-memory tiles:
//   Standard : X = 128 rows of A (tokens), Y = TN rows of B (weights);
//   Swap-AB  : X = 128 rows of B (weights), Y = TN rows of A (tokens), i.e.
//              the blog's (B^T A^T)^T; the epilogue stores D transposed.
// Split-K: blockIdx.z = s owns K tiles [floor(s T / S), floor((s+1) T / S)).
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..5 = epilogue (warp w reads TMEM lanes 32 (w % 4) ..).
// Every wait is bounded; a timeout sets the device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "lq_kernels.h"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace lq {

constexpr int kTileM = 128;      // MMA M (rows of X)
constexpr int kTileK = 128;      // K elements (bytes) per pipeline stage
constexpr int kMmaK = 32;        // K per tcgen05.mma for 8-bit operands
constexpr int kThreads = 192;
constexpr int kScanChunks = 8;   // grouped launch: expert offsets loaded 256 at a time
constexpr int kEpiThreads = 128;
constexpr int kCtlBytes = 64 * 8 + 64;     // mbarriers, TMEM address, flags
constexpr int kScaleBytes = 1024 * 4;      // staged scales: [0,256) per column, [256,384) per row,
                                           // [512,1024) two per-K-block buffers (Block_FP8)

// One ring slot: the X tile, the Y tile and, for the fused quantization, the
// bf16 activation tile (TN x 128, row-major, no swizzle) the codes come from.
template <int TN, bool FUSE = false>
struct TileShape {
  static constexpr int kXBytes = kTileM * kTileK;                 // 16 KB
  static constexpr int kYBytes = TN * kTileK;                     // multiple of 1 KB for TN % 8 == 0
  static constexpr int kStagingBytes = FUSE ? TN * kTileK * 2 : 0;   // multiple of 1 KB as well
  static constexpr int kStageBytes = kXBytes + kYBytes + kStagingBytes;
};

__host__ __device__ constexpr int tmem_cols_for(int cols) {
  return cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : cols <= 256 ? 256 : 512;
}

// Tensor-memory columns of the UE8M0 scale factors of the block-scaled MMA
// (after the accumulator's TN columns).  Up to four slots (as many as ring
// stages, at least two), each the scale factors of four consecutive 128-K
// blocks: one 32-bit column per 32 rows of an operand
// tile, the byte of block t (0..3) of the group in bits [8t, 8t+8), row e of
// the tile at lane e % 32 and column e / 32 of the operand's part of the
// slot, the same in all four lane quarters.  X (128 rows) takes 4 columns, Y
// (TN rows) max(4, TN / 32); slots start on 8-column boundaries.
template <int TN>
struct MxSf {
  static constexpr int kBase = TN < 32 ? 32 : TN;
  static constexpr int kXCols = 4;
  static constexpr int kYCols = TN > 128 ? TN / 32 : 4;
  static constexpr int kSlotCols = (kXCols + kYCols + 7) / 8 * 8;
  static constexpr int kMaxSlots = 4;
  static constexpr int kEnd = kBase + kMaxSlots * kSlotCols;
};

// Scale-factor slots of a launch with `stages` ring slots (their mbarriers
// are the ring's xfull / wfull entries).
__device__ __forceinline__ int mx_slots(int stages) { return stages < 4 ? stages : 4; }

// Tensor-memory columns one CTA of scaled_mm_tc_kernel<FMT, *, TN, ...>
// allocates (the host bounds the CTAs per SM by them).
template <int FMT, int TN>
__host__ __device__ constexpr int tc_tmem_cols() {
  return FMT == kFmtBlockE8m0 ? tmem_cols_for(MxSf<TN>::kEnd) : tmem_cols_for(TN * (FMT == kFmtBlock ? 2 : 1));
}

// Cluster Split-K reduction.  Tiles up to 64 wide push: every CTA sends its
// partial columns, from registers, into slots in the shared memory of the
// CTA that owns those columns (st.async, completion counted in bytes on the
// owner's mbarrier); the slots are a region of their own.  Wider tiles pull:
// each CTA parks its partial in its ring once the ring is free and the
// owners read them remotely between two cluster barriers.
template <int TN>
struct ClusterReduce {
  static constexpr bool kPush = TN <= 64;
  static constexpr int kSlotBytes = TN * 128 * 4;   // S partials of W = TN / S columns
};

// Bytes of the ring region: `stages` slots, and for the pull reduction at
// least the 128 x TN 32-bit partial tile it parks there.
template <int TN, bool FUSE = false>
__host__ __device__ constexpr int ring_bytes(int stages) {
  return (ClusterReduce<TN>::kPush || stages * TileShape<TN, FUSE>::kStageBytes > TN * kTileM * 4)
             ? stages * TileShape<TN, FUSE>::kStageBytes
             : TN * kTileM * 4;
}

// Shared-memory bytes of the kernel for `stages` ring slots; `cluster`: the
// launch uses the cluster Split-K reduction (adds the push slots).
template <int TN, bool FUSE = false>
__host__ __device__ constexpr int gemm_smem_bytes(int stages, bool cluster) {
  return 1024 /* alignment slack */ + ring_bytes<TN, FUSE>(stages) +
         ((cluster && ClusterReduce<TN>::kPush) ? ClusterReduce<TN>::kSlotBytes : 0) + kCtlBytes + kScaleBytes;
}

struct SmemCtl {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* xfull;     // [stages] fused quantization: the bf16 activation tile has landed
  uint64_t* wfull;     // [stages] fused quantization: the weight tile has landed
                       // (full[] then counts the four A-producer warps only)
  uint64_t* tfull;     // [2]
  uint64_t* tempty;    // [2]
  uint64_t* mma_done;  // [1]
  uint64_t* red_bar;   // [1] push reduction: partial columns received
  uint64_t* amax_bar;  // [1] fused quantization: per-token partial amax of every split received
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  volatile int* last_flag;
};

// Bias of output column n (bf16 [N]), added to the scaled accumulator
// before the one rounding to bf16.
__device__ __forceinline__ float bias_at(const GemmParams& p, int64_t n) {
  return __bfloat162float(p.bias[n]);
}

__device__ __forceinline__ void report_timeout(const GemmParams& p, int where) {
  if (p.status) atomicOr(p.status, 1 << where);
}

template <bool kClusterScope = false>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const GemmParams& p, const SmemCtl& c,
                                         int where) {
  auto try_once = [&]() { return kClusterScope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (try_once()) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (try_once()) return true;
    if (*c.abort_flag) return false;
    if (global_timer_ns() - t0 > p.wait_limit_ns) {
      *c.abort_flag = 1;
      report_timeout(p, where);
      return false;
    }
  }
}

// Trace stamp i of this CTA (diagnostics; off when p.trace is null).
//   0 entry, 1 set-up done, 2 producer past the grid dependency wait,
//   3 first stage landed, 4 last MMA issued, 5 accumulator ready in TMEM,
//   6 outputs / partials written, 7 exit, 8 / 9 / 10 cluster reduction:
//   push: past the start barrier / all partials received / reduced tile
//   stored; pull: past the first barrier / tile stored / past the second
__device__ __forceinline__ void trace_stamp(const GemmParams& p, int i) {
  if (p.trace) {
    const uint64_t cta = blockIdx.x + static_cast<uint64_t>(gridDim.x) * (blockIdx.y + static_cast<uint64_t>(gridDim.y) * blockIdx.z);
    p.trace[cta * kTraceSlots + i] = global_timer_ns();
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// The GEMM kernel
// ---------------------------------------------------------------------------
// FUSE (Swap-AB, FP8_Dynamic / W8A8_INT8 only): the activations arrive as
// bf16 (tmY maps them: [M, K] bf16, boxes of TN rows x 128); the TMA stages
// each K tile of them beside the weights, and the epilogue warps, idle during
// the mainloop, quantize it per token into the ring's activation slot (see
// the A-producer below).
// GROUPED (Swap-AB, FP8_Dynamic / W8A8_INT8): the grouped (mixture-of-
// experts) launch below; a compile-time switch so that the other
// instantiations carry none of its code.
// BIAS: the epilogue adds p.bias (also compile-time, for the same reason).
template <int FMT, bool SWAP, int TN, bool FUSE = false, bool GROUPED = false, bool BIAS = false>
__global__ void __launch_bounds__(kThreads, SWAP ? 2 : 1)   // Swap-AB: two CTAs per SM
    scaled_mm_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                        const GemmParams p) {
  static_assert(!FUSE || (SWAP && !is_block_fmt(FMT) && TN <= 64), "fused quantization: Swap-AB FP8/INT8 tiles");
  static_assert(!GROUPED || (SWAP && !is_block_fmt(FMT) && !FUSE && TN <= 64), "grouped launch: Swap-AB FP8/INT8 tiles");
  using Shape = TileShape<TN, FUSE>;
  // bytes the TMA delivers per stage (the fused path writes the activation slot itself)
  constexpr uint32_t kTmaStageBytes = FUSE ? Shape::kXBytes : Shape::kStageBytes;
  constexpr bool kInt8 = FMT == kFmtInt8;
  constexpr bool kBlocked = is_block_fmt(FMT);        // scales per 128-K block: partials carry them
  // UE8M0 Block_FP8: the tensor core applies the power-of-two block scales
  // itself (kind::mxf8f6f4 block scaling, scale factors in tensor memory),
  // so one accumulator runs over the whole K range.  fp32-scale Block_FP8
  // promotes a per-block accumulator into registers instead.
  constexpr bool kMX = FMT == kFmtBlockE8m0;
  constexpr bool kPromote = kBlocked && !kMX;
  constexpr int kAccBufs = kPromote ? 2 : 1;
  constexpr int kTmemCols = tc_tmem_cols<FMT, TN>();
  static_assert(kTmemCols >= TN * kAccBufs, "tensor memory");
  constexpr int CH = TN < 32 ? TN : 32;   // TMEM columns per tcgen05.ld

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  const int stages = p.stages;
  uint8_t* ring = smem;
  const bool cluster_launch = p.S > 1 && p.reduce_mode == 2;
  const bool push_mode = ClusterReduce<TN>::kPush && cluster_launch;
  uint32_t* slots = reinterpret_cast<uint32_t*>(ring + ring_bytes<TN, FUSE>(stages));   // push slots [src][row][col]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + ring_bytes<TN, FUSE>(stages) +
                                               (push_mode ? ClusterReduce<TN>::kSlotBytes : 0));
  SmemCtl c;
  c.full = bars;
  c.empty = bars + stages;
  c.xfull = bars + 2 * stages;
  c.wfull = bars + 3 * stages;
  c.tfull = bars + 4 * stages;
  c.tempty = c.tfull + 2;
  c.mma_done = c.tempty + 2;
  c.red_bar = c.mma_done + 1;
  c.amax_bar = c.red_bar + 1;
  c.tmem_slot = reinterpret_cast<uint32_t*>(c.amax_bar + 1);
  c.abort_flag = reinterpret_cast<volatile int*>(c.tmem_slot + 1);
  c.last_flag = c.abort_flag + 1;
  float* sc = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kCtlBytes);
  float* colsc = sc;          // a_s (Swap-AB) or b_s (Standard) of each tile column
  float* rowsc = sc + 256;    // b_s (Swap-AB) or a_s (Standard) of each accumulator row
  float* blksc = sc + 512;    // Block_FP8: [2][256] per-K-block scale products

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.z;
  const int kb_lo = static_cast<int>((static_cast<int64_t>(split) * p.T) / p.S);
  const int kb_hi = static_cast<int>((static_cast<int64_t>(split + 1) * p.T) / p.S);
  const int nkb = kb_hi - kb_lo;

  if (threadIdx.x == 0) trace_stamp(p, 0);

  // Tile origin, and the bounds / output column offset of the tile's GEMM.
  int64_t x_row0 = static_cast<int64_t>(blockIdx.x) * kTileM;
  int64_t y_row0 = static_cast<int64_t>(blockIdx.y) * TN;
  int64_t m_end = p.M, n_end = p.N, c_off = 0;
  if constexpr (GROUPED) {
    // Grouped (mixture-of-experts) launch, Swap-AB: X = the weights of all
    // experts stacked [E N, K], Y = the tokens sorted by expert [T, K].
    // blockIdx.y enumerates the token tiles of expert 0, then expert 1, ...;
    // warp 0 finds this CTA's expert with a prefix sum of per-expert tile
    // counts.  Expert e's tokens are [H(e-1), H(e)) with H(e) the running
    // max of offsets[1..e+1] clamped to [0, T] (H(-1) = 0): for a valid
    // table (offsets[0] = 0, non-decreasing) that is [offsets[e],
    // offsets[e+1]); for any other no store leaves C.  A CTA past the last
    // tile leaves at once (all CTAs of its cluster share blockIdx.y).
    volatile int* grp = c.last_flag + 1;   // expert (-1: none), tile, first token, end token
    if (warp == 0) {
      // the table may come from the previous kernel on the stream (a router)
      grid_dependency_wait();
      const int E = p.num_experts;
      const int want = static_cast<int>(blockIdx.y);
      const int T = static_cast<int>(p.M);
      int carry = 0, prev_hi = 0, found = -1, f_tile = 0, f_lo = 0, f_hi = 0;
      for (int base0 = 0; base0 < E && found < 0; base0 += 32 * kScanChunks) {
        int his[kScanChunks];   // all loads of this batch in flight at once
#pragma unroll
        for (int k = 0; k < kScanChunks; ++k) {
          const int e = base0 + 32 * k + lane;
          his[k] = e < E ? p.expert_offsets[e + 1] : 0;
        }
#pragma unroll
        for (int k = 0; k < kScanChunks; ++k) {
          const int base = base0 + 32 * k;
          if (base >= E || found >= 0) break;
          const int e = base + lane;
          int hi = e < E ? min(max(his[k], 0), T) : 0;
          hi = max(hi, prev_hi);
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {   // inclusive running max
            const int v = __shfl_up_sync(0xffffffffu, hi, o);
            if (lane >= o) hi = max(hi, v);
          }
          int lo = __shfl_up_sync(0xffffffffu, hi, 1);
          if (lane == 0) lo = prev_hi;
          const int tiles = e < E ? (hi - lo + TN - 1) / TN : 0;
          int incl = tiles;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
          }
          const bool mine = e < E && want >= carry + incl - tiles && want < carry + incl;
          const unsigned who = __ballot_sync(0xffffffffu, mine);
          if (who) {
            const int src = __ffs(who) - 1;
            found = base + src;
            f_tile = __shfl_sync(0xffffffffu, want - (carry + incl - tiles), src);
            f_lo = __shfl_sync(0xffffffffu, lo, src);
            f_hi = __shfl_sync(0xffffffffu, hi, src);
          }
          carry += __shfl_sync(0xffffffffu, incl, 31);
          prev_hi = __shfl_sync(0xffffffffu, hi, 31);
        }
      }
      if (lane == 0) {
        grp[0] = found;
        grp[1] = f_tile;
        grp[2] = f_lo;
        grp[3] = f_hi;
      }
    }
    __syncthreads();
    const int e = grp[0];
    if (e < 0 || x_row0 >= p.N) return;   // before any barrier, TMEM or cluster work
    y_row0 = grp[2] + static_cast<int64_t>(grp[1]) * TN;
    m_end = grp[3];
    c_off = static_cast<int64_t>(e) * p.N;
    x_row0 += c_off;
    n_end = c_off + p.N;
    __syncthreads();   // grp is read by every thread before the control block is initialised
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&c.full[s], FUSE ? kEpiThreads / 32 : 1);   // the TMA, or the four A-producer warps
      mbar_init(&c.empty[s], 1);
      // block-scaled MMA: xfull[slot] = scale-factor slot written (the four
      // epilogue warps), wfull[slot] = slot read by the tensor core (commit)
      mbar_init(&c.xfull[s], (kMX && s < mx_slots(stages)) ? kEpiThreads / 32 : 1);
      mbar_init(&c.wfull[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c.tfull[b], 1);
      mbar_init(&c.tempty[b], kEpiThreads / 32);
    }
    mbar_init(c.mma_done, 1);
    mbar_init(c.red_bar, 1);
    mbar_init(c.amax_bar, 1);
    *c.abort_flag = 0;
    *c.last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensor_map(&tmX);
    prefetch_tensor_map(&tmY);
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
  // Push reduction: announce (cluster-wide, release) that this CTA's barriers
  // exist; the epilogue waits for the whole cluster before pushing.
  if (push_mode) cluster_arrive_release();

  // Let the next kernel on the stream start its own prologue / weight stream.
  grid_launch_dependents();


  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();   // weights: streamed once
      const uint64_t pol_a = policy_evict_last();    // activations: re-read by many CTAs
      const CUtensorMap* tmW = SWAP ? &tmX : &tmY;
      const CUtensorMap* tmA = SWAP ? &tmY : &tmX;
      const int w_row0 = SWAP ? x_row0 : y_row0;
      const int a_row0 = SWAP ? y_row0 : x_row0;
      const int w_off = SWAP ? 0 : Shape::kXBytes;   // byte offset of the weight tile in a stage
      const int a_off = SWAP ? Shape::kXBytes : 0;
      constexpr int kStagingOff = Shape::kXBytes + Shape::kYBytes;   // fused: the bf16 activation tile
      const int pre = nkb < stages ? nkb : stages;
      if (p.early_weights) {
        // The caller guarantees that the weights are not written by a kernel
        // that may still run: start streaming them before waiting for the
        // previous kernel on the stream (programmatic dependent launch).
        for (int i = 0; i < pre; ++i) {
          if (i == p.skip_stage) continue;
          uint8_t* st = ring + i * Shape::kStageBytes;
          uint64_t* wb = FUSE ? &c.wfull[i] : &c.full[i];
          mbar_arrive_expect_tx(wb, kTmaStageBytes);
          tma_load_2d(tmW, wb, st + w_off, (kb_lo + i) * kTileK, w_row0, pol_w);
        }
        grid_dependency_wait();
      } else {
        grid_dependency_wait();
        for (int i = 0; i < pre; ++i) {
          if (i == p.skip_stage) continue;
          uint8_t* st = ring + i * Shape::kStageBytes;
          uint64_t* wb = FUSE ? &c.wfull[i] : &c.full[i];
          mbar_arrive_expect_tx(wb, kTmaStageBytes);
          tma_load_2d(tmW, wb, st + w_off, (kb_lo + i) * kTileK, w_row0, pol_w);
        }
      }
      trace_stamp(p, 2);
      for (int i = 0; i < pre; ++i) {
        if (i == p.skip_stage) continue;
        uint8_t* st = ring + i * Shape::kStageBytes;
        if constexpr (FUSE) {
          mbar_arrive_expect_tx(&c.xfull[i], Shape::kStagingBytes);
          tma_load_2d(tmA, &c.xfull[i], st + kStagingOff, (kb_lo + i) * kTileK, a_row0, pol_a);
        } else {
          tma_load_2d(tmA, &c.full[i], st + a_off, (kb_lo + i) * kTileK, a_row0, pol_a);
        }
      }
      int issued = pre;
      for (int i = pre; i < nkb; ++i) {
        const int s = i % stages;
        const uint32_t ph = static_cast<uint32_t>(i / stages) & 1u;
        if (!wait_bar(&c.empty[s], ph ^ 1u, p, c, 0)) break;
        if (i == p.skip_stage) continue;
        uint8_t* st = ring + s * Shape::kStageBytes;
        uint64_t* wb = FUSE ? &c.wfull[s] : &c.full[s];
        mbar_arrive_expect_tx(wb, kTmaStageBytes);
        tma_load_2d(tmW, wb, st + w_off, (kb_lo + i) * kTileK, w_row0, pol_w);
        if constexpr (FUSE) {
          mbar_arrive_expect_tx(&c.xfull[s], Shape::kStagingBytes);
          tma_load_2d(tmA, &c.xfull[s], st + kStagingOff, (kb_lo + i) * kTileK, a_row0, pol_a);
        } else {
          tma_load_2d(tmA, &c.full[s], st + a_off, (kb_lo + i) * kTileK, a_row0, pol_a);
        }
        issued = i + 1;
      }
      if (*c.abort_flag) {
        // Drain: wait (bounded) for the copies still in flight into shared memory.
        const int first = issued > stages ? issued - stages : 0;
        for (int j = first; j < issued; ++j) {
          if (j == p.skip_stage) continue;   // never armed
          const uint32_t par = static_cast<uint32_t>(j / stages) & 1u;
          uint64_t* bars_tx[2] = {FUSE ? &c.wfull[j % stages] : &c.full[j % stages], &c.xfull[j % stages]};
          for (int b = 0; b < (FUSE ? 2 : 1); ++b) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bars_tx[b], par) && global_timer_ns() - t0 < p.wait_limit_ns) {
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    grid_dependency_wait();
    if (lane == 0) {
      constexpr uint32_t idesc = kMX ? make_idesc_mx(kTileM, TN) : make_idesc<kInt8>(kTileM, TN);
      bool issued_any = false;
      // block-scaled MMA: the scale-factor slot of the current group of four
      // blocks, its phase, and its tensor-memory address (advanced per group)
      const int mx_ns = kMX ? mx_slots(stages) : 1;
      int mx_slot = 0;
      uint32_t mx_phase = 0;
      uint32_t mx_sf = tmem_base + static_cast<uint32_t>(MxSf<TN>::kBase);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages;
        const uint32_t ph = static_cast<uint32_t>(i / stages) & 1u;
        uint32_t d_tmem = tmem_base;
        if (kMX && (i & 3) == 0) {   // the scale factors of blocks i .. i+3 are in tensor memory
          if (i > 0 && ++mx_slot == mx_ns) {
            mx_slot = 0;
            mx_phase ^= 1u;
          }
          mx_sf = tmem_base + static_cast<uint32_t>(MxSf<TN>::kBase + mx_slot * MxSf<TN>::kSlotCols);
          if (!wait_bar(&c.xfull[mx_slot], mx_phase, p, c, 13)) break;
        }
        if (kPromote) {
          const int buf = i & 1;
          const uint32_t use = static_cast<uint32_t>(i >> 1);
          if (!wait_bar(&c.tempty[buf], (use & 1u) ^ 1u, p, c, 1)) break;
          d_tmem += static_cast<uint32_t>(buf * TN);
        }
        if (FUSE && !wait_bar(&c.wfull[s], ph, p, c, 2)) break;
        if (!wait_bar(&c.full[s], ph, p, c, 2)) break;
        tc_fence_after_sync();
        if (i == 0) trace_stamp(p, 3);
        uint8_t* st = ring + s * Shape::kStageBytes;
        const uint64_t xd = smem_desc_k_sw128(st);
        const uint64_t yd = smem_desc_k_sw128(st + Shape::kXBytes);
#pragma unroll
        for (int kk = 0; kk < kTileK / kMmaK; ++kk) {
          // +32 bytes along K inside the 128-byte swizzle row = +2 in the 16-byte address field
          const uint32_t acc = kPromote ? (kk > 0) : (i > 0 || kk > 0);
          if constexpr (kMX) {
            const uint32_t t = static_cast<uint32_t>(i & 3);   // this block's byte in the slot
            mma_mxf8f6f4_block_scale(d_tmem, xd + 2 * kk, yd + 2 * kk, idesc_with_sf_ids(idesc, t, t), mx_sf,
                                     mx_sf + MxSf<TN>::kXCols, acc);
          } else if (kInt8) {
            mma_i8(d_tmem, xd + 2 * kk, yd + 2 * kk, idesc, acc);
          } else {
            mma_f8f6f4(d_tmem, xd + 2 * kk, yd + 2 * kk, idesc, acc);
          }
        }
        issued_any = true;
        mma_commit(&c.empty[s]);
        if (kPromote) mma_commit(&c.tfull[i & 1]);
        if (kMX && ((i & 3) == 3 || i == nkb - 1)) mma_commit(&c.wfull[mx_slot]);   // slot read
      }
      trace_stamp(p, 4);
      if (!kPromote && nkb > 0 && !*c.abort_flag) mma_commit(&c.tfull[0]);
      if (issued_any) {
        // All MMAs must be complete before TMEM is released at teardown.
        mma_commit(c.mma_done);
        wait_bar(c.mma_done, 0, p, c, 3);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    grid_dependency_wait();
    const int q = warp & 3;                    // TMEM lane quarter of this warp
    const int r = q * 32 + lane;               // accumulator row (TMEM lane)
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    // (m, n) of accumulator element (r, j): Standard (x_row0 + r, y_row0 + j),
    // Swap-AB (y_row0 + j, x_row0 + r).
    // bounds of the tile's GEMM: tokens [.., m_end), weight rows [.., n_end)
    const int64_t M = m_end, N = n_end;

    float accr[kPromote ? TN : 1];
#pragma unroll
    for (int j = 0; j < (kPromote ? TN : 1); ++j) accr[j] = 0.f;

    if (!kBlocked) {
      // Scales do not depend on the accumulator: load them while the mainloop
      // runs (these warps are idle until then).  The fused path computes the
      // token scales itself below.
      if (!FUSE) {
        for (int j = r; j < TN; j += kEpiThreads) {
          const int64_t col = y_row0 + j;
          colsc[j] = SWAP ? (col < M ? __ldg(p.a_s + col) : 0.f) : (col < N ? __ldg(p.b_s + col) : 0.f);
        }
      }
      const int64_t row = x_row0 + r;
      rowsc[r] = SWAP ? (row < N ? __ldg(p.b_s + row) : 0.f) : (row < M ? __ldg(p.a_s + row) : 0.f);
      named_barrier_sync(2, kEpiThreads);
    }

    bool cluster_waited = false;
    if constexpr (FUSE) {
      // ------------------------------------------------ A-producer (fused)
      // 1. partial amax of each token over this CTA's K range (read straight
      //    from global memory, eight 16-byte loads in flight per lane; when
      //    the tile has fewer than four tokens, the warps split the range);
      // 2. Split-K cluster: every CTA sends its partials to every CTA
      //    (st.async, counted in bytes on amax_bar) and takes the max, so all
      //    CTAs of a tile derive the same per-token scale;
      // 3. s = max(fp32(amax / Q), 2^-126); q = enc(fp32(x / s)) for each K
      //    tile, read from the bf16 tile the TMA staged in the slot and
      //    written in the 128-byte-swizzled K-major layout that the tensor
      //    core reads, into the slot's activation tile; the four warps'
      //    arrivals complete the stage.
      // Codes and scales equal those of lq_quant_per_token bit for bit.
      constexpr int kChunks = TN * 8 / kEpiThreads;   // 16-byte code chunks per thread per K tile (TN >= 16)
      const int e = warp - 2;                         // epilogue warp 0..3
      const int tid = e * 32 + lane;                  // epilogue thread 0..127
      float* pa = sc + 384;                           // [TN] this CTA's partial amax
      float* slots_amax = sc + 512;                   // [S][TN] partial amax of every split
      float* rcp = sc + 128;                          // [TN] Divisor reciprocal of each token (colsc
                                                      // holds only TN <= 64 entries here)
      const int64_t k_lo = static_cast<int64_t>(kb_lo) * kTileK;
      const int64_t k_hi = min(static_cast<int64_t>(kb_hi) * kTileK, p.K);
      const float qmax = kInt8 ? kInt8Max : kE4m3Max;
      const int mv = (M - y_row0) < TN ? static_cast<int>(M - y_row0) : TN;   // tokens of this tile (>= 1)
      for (int j = tid; j < TN; j += kEpiThreads) pa[j] = 0.f;
      named_barrier_sync(2, kEpiThreads);
      {
        const int64_t nch = (k_hi - k_lo) / 8;   // 16-byte chunks of one token in the K range
        const int parts = mv >= 4 ? 1 : 4 / mv;
        for (int u = e; u < mv * parts; u += 4) {
          const int j = u / parts, part = u - j * parts;
          const int64_t c_lo = nch * part / parts, c_hi = nch * (part + 1) / parts;
          const uint4* xr = reinterpret_cast<const uint4*>(p.x + (y_row0 + j) * p.K + k_lo);
          float a = 0.f;
          for (int64_t v = c_lo + lane; v < c_hi; v += 32 * 8) {
            uint4 buf[8];
#pragma unroll
            for (int w = 0; w < 8; ++w)
              buf[w] = v + 32 * w < c_hi ? __ldg(xr + v + 32 * w) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              float f[8];
              bf16x8_to_f32(buf[w], f);
              a = fmaxf(a, amax8(f));
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
          // a >= 0, so the order of the float bits is the order of the values
          if (lane == 0) atomicMax(reinterpret_cast<int*>(pa) + j, __float_as_int(a));
        }
      }
      named_barrier_sync(2, kEpiThreads);
      if (p.S > 1) {
        cluster_wait_acquire();   // every CTA of the cluster has initialised its barriers
        cluster_waited = true;
        if (tid == 0) mbar_arrive_expect_tx(c.amax_bar, static_cast<uint32_t>(p.S * TN * 4));
        if (tid < p.S) {
          const uint32_t dst = dsmem_map(smem_addr(slots_amax), static_cast<uint32_t>(tid)) +
                               static_cast<uint32_t>(split * TN * 4);
          const uint32_t bar = dsmem_map(smem_addr(c.amax_bar), static_cast<uint32_t>(tid));
#pragma unroll
          for (int j = 0; j < TN; j += 4)
            st_async_v4(dst + j * 4, __float_as_uint(pa[j]), __float_as_uint(pa[j + 1]), __float_as_uint(pa[j + 2]),
                        __float_as_uint(pa[j + 3]), bar);
        }
        wait_bar<true>(c.amax_bar, 0, p, c, 8);
      }
      if (tid < TN) {
        float a = pa[tid];
        if (p.S > 1) {
          a = 0.f;
          for (int s2 = 0; s2 < p.S; ++s2) a = fmaxf(a, slots_amax[s2 * TN + tid]);
        }
        const int64_t m = y_row0 + tid;
        const float sm = scale_from_amax(a, qmax);
        colsc[tid] = sm;
        rcp[tid] = make_divisor(a, sm).y;
        if (p.a_scales_out && blockIdx.x == 0 && split == 0 && m < M) p.a_scales_out[m] = sm;
      }
      named_barrier_sync(2, kEpiThreads);

      // 4. encode the staged tiles stage by stage.  The TMA refills a slot
      //    only after the MMA has released it (empty), so xfull[s] landing
      //    means the activation tile of slot s is free to overwrite as well.
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages;
        const uint32_t ph = static_cast<uint32_t>(i / stages) & 1u;
        if (!wait_bar(&c.xfull[s], ph, p, c, 9)) break;
        uint8_t* slot = ring + s * Shape::kStageBytes + Shape::kXBytes;
        const uint8_t* staged = slot + Shape::kYBytes;
#pragma unroll
        for (int u = 0; u < kChunks; ++u) {
          const int t = tid + u * kEpiThreads;
          const int j = t >> 3, cc = t & 7;
          uint4 qv = make_uint4(0u, 0u, 0u, 0u);   // rows past the last token: any code, their columns are dropped
          if (j < mv) {
            const Divisor d{colsc[j], rcp[j]};
            const uint4* src = reinterpret_cast<const uint4*>(staged + j * (kTileK * 2) + cc * 32);
            float f0[8], f1[8];
            bf16x8_to_f32(src[0], f0);
            bf16x8_to_f32(src[1], f1);
            const uint2 q0 = kInt8 ? encode8_int8(f0, d) : encode8_e4m3(f0, d);
            const uint2 q1 = kInt8 ? encode8_int8(f1, d) : encode8_e4m3(f1, d);
            qv = make_uint4(q0.x, q0.y, q1.x, q1.y);
            const int64_t k0 = static_cast<int64_t>(kb_lo + i) * kTileK + cc * 16;
            if (p.a_codes_out && blockIdx.x == 0 && k0 < p.K)
              *reinterpret_cast<uint4*>(p.a_codes_out + (y_row0 + j) * p.K + k0) = qv;
          }
          // row j of the slot, 16-byte chunk cc placed at cc ^ (j % 8) (128-byte swizzle)
          *reinterpret_cast<uint4*>(slot + j * kTileK + ((cc ^ (j & 7)) << 4)) = qv;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic stores -> tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.full[s]);
      }
    }

    bool ok = true;
    if constexpr (kMX) {
      // ------------------------------------- scale factors (block-scaled MMA)
      // For each group of four K blocks of this CTA's range: gather the UE8M0
      // bytes of the X tile's 128 rows and the Y tile's TN rows, pack four
      // blocks per 32-bit column, write them to the group's slot in tensor
      // memory (each warp its own lane quarter: the layout is the same in all
      // four) and tell the MMA warp.  A slot is rewritten only after the
      // tensor core has read it (wfull, committed by the MMA warp).  The
      // bytes of the next group are loaded while the current one is used.
      using Sf = MxSf<TN>;
      const uint8_t* a_b = reinterpret_cast<const uint8_t*>(p.a_s);   // [M, KB]
      const uint8_t* b_b = reinterpret_cast<const uint8_t*>(p.b_s);   // [N / 128, KB]
      // byte of row e (< 128) of X, or of row e (< TN) of Y, for this CTA's block i
      auto x_byte = [&](int e, int i) -> uint32_t {
        if (i >= nkb) return 127u;
        const int64_t kb = kb_lo + i;
        if (SWAP) {
          const int64_t n = x_row0 + e;
          return n < N ? b_b[(n >> 7) * p.KB + kb] : 127u;
        }
        const int64_t m = x_row0 + e;
        return m < M ? a_b[m * p.KB + kb] : 127u;
      };
      auto y_byte = [&](int e, int i) -> uint32_t {
        if (i >= nkb || e >= TN) return 127u;
        const int64_t kb = kb_lo + i;
        if (SWAP) {
          const int64_t m = y_row0 + e;
          return m < M ? a_b[m * p.KB + kb] : 127u;
        }
        const int64_t n = y_row0 + e;
        return n < N ? b_b[(n >> 7) * p.KB + kb] : 127u;
      };
      // A row's four bytes of a whole, 4-byte aligned group are one 32-bit
      // load (a quarter of the load instructions and cache-line requests
      // of byte loads, which share the L1 / shared-memory path with the MMA's
      // operand reads); otherwise byte by byte.
      const bool words = (p.KB & 3) == 0 && ((reinterpret_cast<uintptr_t>(a_b) | reinterpret_cast<uintptr_t>(b_b)) & 3u) == 0;
      auto a_word = [&](int64_t m, int64_t kb0) -> uint32_t {
        return m < M ? __ldg(reinterpret_cast<const uint32_t*>(a_b + m * p.KB + kb0)) : 0x7F7F7F7Fu;
      };
      auto b_word = [&](int64_t n, int64_t kb0) -> uint32_t {
        return n < N ? __ldg(reinterpret_cast<const uint32_t*>(b_b + (n >> 7) * p.KB + kb0)) : 0x7F7F7F7Fu;
      };
      uint32_t wx[Sf::kXCols], wy[Sf::kYCols];
      auto gather = [&](int g) {
        const int64_t kb0 = kb_lo + 4 * g;
        if (words && (kb0 & 3) == 0 && 4 * g + 4 <= nkb) {
#pragma unroll
          for (int col = 0; col < Sf::kXCols; ++col) {
            const int e = col * 32 + lane;
            wx[col] = SWAP ? b_word(x_row0 + e, kb0) : a_word(x_row0 + e, kb0);
          }
#pragma unroll
          for (int col = 0; col < Sf::kYCols; ++col) {
            const int e = col * 32 + lane;
            wy[col] = e >= TN ? 0x7F7F7F7Fu : (SWAP ? a_word(y_row0 + e, kb0) : b_word(y_row0 + e, kb0));
          }
          return;
        }
#pragma unroll
        for (int col = 0; col < Sf::kXCols; ++col) {
          uint32_t w = 0;
#pragma unroll
          for (int t = 0; t < 4; ++t) w |= x_byte(col * 32 + lane, 4 * g + t) << (8 * t);
          wx[col] = w;
        }
#pragma unroll
        for (int col = 0; col < Sf::kYCols; ++col) {
          uint32_t w = 0;
#pragma unroll
          for (int t = 0; t < 4; ++t) w |= y_byte(col * 32 + lane, 4 * g + t) << (8 * t);
          wy[col] = w;
        }
      };
      const int groups = (nkb + 3) / 4;
      const int ns = mx_slots(stages);
      if (groups > 0) gather(0);
      int slot = 0;
      uint32_t reuse_phase = 0;   // phase of wfull[slot] that frees it for this group
      for (int g = 0; g < groups && ok; ++g) {
        if (g > 0 && ++slot == ns) {
          slot = 0;
          if (g > ns) reuse_phase ^= 1u;
        }
        if (g >= ns) ok = __all_sync(0xffffffffu, wait_bar(&c.wfull[slot], reuse_phase, p, c, 14));
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t col0 = t_row + static_cast<uint32_t>(Sf::kBase + slot * Sf::kSlotCols);
        tmem_st_32x32b_x4(col0, wx);
        if constexpr (Sf::kYCols == 8)
          tmem_st_32x32b_x8(col0 + Sf::kXCols, wy);
        else
          tmem_st_32x32b_x4(col0 + Sf::kXCols, wy);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.xfull[slot]);
        if (g + 1 < groups) gather(g + 1);
      }
      if (ok && nkb > 0) {
        ok = wait_bar(&c.tfull[0], 0, p, c, 5);
        tc_fence_after_sync();
      }
    } else if (kPromote) {
      // Per-128-K-block promotion: acc += D_kb * a_s[m, kb] * b_s[nb, kb].
      // The scale products are loaded kPre blocks at a time, a group ahead:
      // the loads of group g + 1 are issued as group g starts, so their
      // latency (an L2 round trip while the operand stream keeps L2 busy)
      // hides behind kPre blocks of promotion.  (Loaded one block ahead, the
      // register copy that carries the value into the next iteration waited
      // for the load every block.)  Swap-AB stages each block's products in
      // shared memory (double buffer blksc, one named barrier per block).
      // Every thread runs every iteration (also after a timeout), so the
      // named barriers always match.
      constexpr int kPre = SWAP ? 4 : 8;   // Swap-AB: fewer registers (two CTAs per SM at tile_n 64)
      const int nb = SWAP ? x_row0 / 128 : y_row0 / 128;
      const int64_t m_thread = x_row0 + r;   // Standard: this thread's token
      // Block scale i of an operand: fp32, or a UE8M0 byte (2^(b - 127)).
      auto scale_at = [&](const float* base, int64_t i) -> float {
        if constexpr (FMT == kFmtBlockE8m0) {
          const uint32_t b = __ldg(reinterpret_cast<const uint8_t*>(base) + i);
          return __uint_as_float(b == 0u ? 0x00400000u : (b == 255u ? 0x7FC00000u : b << 23));
        } else {
          return __ldg(base + i);
        }
      };
      const bool loader = SWAP ? (r < TN) : true;
      auto load_scale = [&](int i) -> float {   // product of the CTA's i-th block (0 past the range)
        if (!loader || i >= nkb) return 0.f;
        const int kb = kb_lo + i;
        const float sb = scale_at(p.b_s, static_cast<int64_t>(nb) * p.KB + kb);
        if (SWAP) {
          const int64_t m = y_row0 + r;     // column r of the tile (r < TN)
          return (m < M ? scale_at(p.a_s, m * p.KB + kb) : 0.f) * sb;
        }
        return (m_thread < M ? scale_at(p.a_s, m_thread * p.KB + kb) : 0.f) * sb;
      };
      float cur[kPre], nxt[kPre];
#pragma unroll
      for (int j = 0; j < kPre; ++j) cur[j] = load_scale(j);
      if (SWAP) {
        if (loader) blksc[r] = cur[0];
        named_barrier_sync(2, kEpiThreads);
      }
      for (int i0 = 0; i0 < nkb; i0 += kPre) {
#pragma unroll
        for (int j = 0; j < kPre; ++j) nxt[j] = load_scale(i0 + kPre + j);
#pragma unroll
        for (int j = 0; j < kPre; ++j) {
          const int i = i0 + j;
          if (i < nkb) {   // the same for every epilogue thread
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            // warp-uniform decision: the tcgen05.ld below is .sync.aligned
            if (ok) ok = __all_sync(0xffffffffu, wait_bar(&c.tfull[buf], use & 1u, p, c, 4));
            if (ok) {
              tc_fence_after_sync();
              const float* bs = blksc + (i & 1) * 256;
#pragma unroll
              for (int c0 = 0; c0 < TN; c0 += CH) {
                uint32_t v[CH];
                if constexpr (CH == 32)
                  tmem_ld_32x32b_x32(t_row + buf * TN + c0, v);
                else
                  tmem_ld_32x32b_x16(t_row + buf * TN + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < CH; ++jj)
                  accr[c0 + jj] = fmaf(__uint_as_float(v[jj]), SWAP ? bs[c0 + jj] : cur[j], accr[c0 + jj]);
              }
              tc_fence_before_sync();
              __syncwarp();
              if (lane == 0) mbar_arrive(&c.tempty[buf]);
            }
            if (SWAP) {
              if (loader && i + 1 < nkb) blksc[((i + 1) & 1) * 256 + r] = j + 1 < kPre ? cur[j + 1] : nxt[0];
              named_barrier_sync(2, kEpiThreads);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kPre; ++j) cur[j] = nxt[j];
      }
    } else if (nkb > 0) {
      ok = wait_bar(&c.tfull[0], 0, p, c, 5);
      tc_fence_after_sync();
    }
    ok = __all_sync(0xffffffffu, ok && !*c.abort_flag);
    if (warp == 2 && lane == 0) trace_stamp(p, 5);

    const bool cluster_mode = cluster_launch;
    // The ring's last readers were the tensor core (async proxy); order them
    // before the generic-proxy stores of the pulled partial tile.
    if (cluster_mode && !push_mode) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (push_mode) {
      if (!cluster_waited) cluster_wait_acquire();   // every CTA of the cluster has initialised its barriers
      if (warp == 2 && lane == 0) {
        trace_stamp(p, 8);
        mbar_arrive_expect_tx(c.red_bar, static_cast<uint32_t>(ClusterReduce<TN>::kSlotBytes));
      }
    }
    if (ok) {
      float* wsf = reinterpret_cast<float*>(p.ws);
      int32_t* wsi = reinterpret_cast<int32_t*>(p.ws);
      const bool split_mode = p.S > 1 && !cluster_mode;   // partials to the global workspace

#pragma unroll
      for (int c0 = 0; c0 < TN; c0 += CH) {
        uint32_t v[CH];
        if (kPromote) {
#pragma unroll
          for (int j = 0; j < CH; ++j) v[j] = __float_as_uint(accr[c0 + j]);
        } else if (nkb > 0) {
          if constexpr (CH == 32)
            tmem_ld_32x32b_x32(t_row + c0, v);
          else
            tmem_ld_32x32b_x16(t_row + c0, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < CH; ++j) v[j] = 0u;   // empty split: zero partial
        }

        if (push_mode) {
          // columns [o W, (o+1) W) go to CTA o, slot [split][r][0..W)
          const int W = TN / p.S;
          const uint32_t slot_row = static_cast<uint32_t>((split * kTileM + r) * W) * 4u;
          const uint32_t slots_local = smem_addr(slots);
          const uint32_t bar_local = smem_addr(c.red_bar);
          if (W >= 4) {
#pragma unroll
            for (int j = 0; j < CH; j += 4) {
              const int owner = (c0 + j) / W;
              const int jj = (c0 + j) - owner * W;
              st_async_v4(dsmem_map(slots_local, owner) + slot_row + jj * 4u, v[j], v[j + 1], v[j + 2], v[j + 3],
                          dsmem_map(bar_local, owner));
            }
          } else if (W == 2) {
#pragma unroll
            for (int j = 0; j < CH; j += 2) {
              const int owner = (c0 + j) / 2;
              st_async_v2(dsmem_map(slots_local, owner) + slot_row, v[j], v[j + 1], dsmem_map(bar_local, owner));
            }
          } else {
#pragma unroll
            for (int j = 0; j < CH; ++j)
              st_async_b32(dsmem_map(slots_local, c0 + j) + slot_row, v[j], dsmem_map(bar_local, c0 + j));
          }
          continue;
        }
        if (cluster_mode) {
          // partial tile -> own shared memory, [column j][row r] (the ring is free now)
          uint32_t* red = reinterpret_cast<uint32_t*>(ring);
#pragma unroll
          for (int j = 0; j < CH; ++j) red[(c0 + j) * kTileM + r] = v[j];
          continue;
        }

        if (SWAP) {
          const int64_t n = x_row0 + r;
          if (n < N) {
            const float bsn = (!kBlocked && !split_mode) ? rowsc[r] : 1.f;
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              const int64_t m = y_row0 + c0 + j;
              if (m < M) {
                const int64_t idx = m * p.N + (n - c_off);   // c_off: the expert's first weight row (grouped)
                if (split_mode) {
                  const int64_t widx = (static_cast<int64_t>(split) * M + m) * N + n;
                  if (kInt8) wsi[widx] = static_cast<int32_t>(v[j]);
                  else wsf[widx] = __uint_as_float(v[j]);
                } else {
                  float val;
                  if (kBlocked) {
                    val = __uint_as_float(v[j]);
                  } else {
                    const float a = kInt8 ? static_cast<float>(static_cast<int32_t>(v[j])) : __uint_as_float(v[j]);
                    val = a * colsc[c0 + j] * bsn;
                  }
                  if constexpr (BIAS) val += bias_at(p, n - c_off);
                  p.C[idx] = __float2bfloat16_rn(val);
                  if (kInt8 && p.acc_out) p.acc_out[idx] = static_cast<int32_t>(v[j]);
                }
              }
            }
          }
        } else {
          const int64_t m = x_row0 + r;
          if (m < M) {
            const float asm_ = (!kBlocked && !split_mode) ? rowsc[r] : 1.f;
#pragma unroll
            for (int j8 = 0; j8 < CH; j8 += 8) {
              const int64_t n = y_row0 + c0 + j8;
              if (n < N) {   // N % 8 == 0: the 8-wide group is fully inside or outside
                if (split_mode) {
                  const int64_t widx = (static_cast<int64_t>(split) * M + m) * N + n;
                  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint32_t*>(p.ws) + widx);
                  dst[0] = make_uint4(v[j8 + 0], v[j8 + 1], v[j8 + 2], v[j8 + 3]);
                  dst[1] = make_uint4(v[j8 + 4], v[j8 + 5], v[j8 + 6], v[j8 + 7]);
                } else {
                  float f[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    if (kBlocked) {
                      f[e] = __uint_as_float(v[j8 + e]);
                    } else {
                      const float a =
                          kInt8 ? static_cast<float>(static_cast<int32_t>(v[j8 + e])) : __uint_as_float(v[j8 + e]);
                      f[e] = a * asm_ * colsc[c0 + j8 + e];
                    }
                  }
                  if constexpr (BIAS) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] += bias_at(p, n + e);
                  }
                  uint4 pk = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                        pack_bf16x2(f[6], f[7]));
                  *reinterpret_cast<uint4*>(p.C + m * N + n) = pk;
                  if (kInt8 && p.acc_out) {
                    uint4* ao = reinterpret_cast<uint4*>(p.acc_out + m * N + n);
                    ao[0] = make_uint4(v[j8 + 0], v[j8 + 1], v[j8 + 2], v[j8 + 3]);
                    ao[1] = make_uint4(v[j8 + 4], v[j8 + 5], v[j8 + 6], v[j8 + 7]);
                  }
                }
              }
            }
          }
        }
      }

    }

    if (warp == 2 && lane == 0) trace_stamp(p, 6);

    // -------------------------------------------- in-kernel Split-K reduce
    // Every epilogue thread reaches both named barriers, also after a
    // timeout (then this CTA does not count itself and no CTA reduces).
    if (p.S > 1 && p.reduce_mode == 1) {
      float* wsf = reinterpret_cast<float*>(p.ws);
      int32_t* wsi = reinterpret_cast<int32_t*>(p.ws);
      __threadfence();
      named_barrier_sync(1, kEpiThreads);
      const int tile_id = blockIdx.x + blockIdx.y * gridDim.x;
      if (warp == 2 && lane == 0) {
        int last = 0;
        if (!*c.abort_flag) last = atomicAdd(p.counters + tile_id, 1) == p.S - 1;
        *c.last_flag = last;
      }
      named_barrier_sync(1, kEpiThreads);
      if (*c.last_flag) {
        __threadfence();
        if (SWAP) {
          const int64_t n = x_row0 + r;
          if (n < N) {
            const float bsn = kBlocked ? 1.f : rowsc[r];
            for (int j = 0; j < TN; ++j) {
              const int64_t m = y_row0 + j;
              if (m >= M) break;
              float sf = 0.f;
              int32_t si = 0;
              for (int s = 0; s < p.S; ++s) {
                const int64_t widx = (static_cast<int64_t>(s) * M + m) * N + n;
                if (kInt8) si += __ldcg(wsi + widx);
                else sf += __ldcg(wsf + widx);
              }
              float val;
              if (kBlocked) val = sf;
              else val = (kInt8 ? static_cast<float>(si) : sf) * colsc[j] * bsn;
              if constexpr (BIAS) val += bias_at(p, n);
              p.C[m * N + n] = __float2bfloat16_rn(val);
              if (kInt8 && p.acc_out) p.acc_out[m * N + n] = si;
            }
          }
        } else {
          const int64_t m = x_row0 + r;
          if (m < M) {
            const float asm_ = kBlocked ? 1.f : rowsc[r];
            for (int j4 = 0; j4 < TN; j4 += 4) {
              const int64_t n = y_row0 + j4;
              if (n >= N) break;
              float4 sf = make_float4(0.f, 0.f, 0.f, 0.f);
              int4 si = make_int4(0, 0, 0, 0);
              for (int s = 0; s < p.S; ++s) {
                const int64_t widx = (static_cast<int64_t>(s) * M + m) * N + n;
                if (kInt8) {
                  const int4 t = __ldcg(reinterpret_cast<const int4*>(wsi + widx));
                  si.x += t.x; si.y += t.y; si.z += t.z; si.w += t.w;
                } else {
                  const float4 t = __ldcg(reinterpret_cast<const float4*>(wsf + widx));
                  sf.x += t.x; sf.y += t.y; sf.z += t.z; sf.w += t.w;
                }
              }
              float f[4];
              if (kInt8) { f[0] = si.x; f[1] = si.y; f[2] = si.z; f[3] = si.w; }
              else { f[0] = sf.x; f[1] = sf.y; f[2] = sf.z; f[3] = sf.w; }
              if (!kBlocked) {
#pragma unroll
                for (int e = 0; e < 4; ++e) f[e] = f[e] * asm_ * colsc[j4 + e];
              }
              if constexpr (BIAS) {
#pragma unroll
                for (int e = 0; e < 4; ++e) f[e] += bias_at(p, n + e);
              }
              uint2 pk = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
              *reinterpret_cast<uint2*>(p.C + m * N + n) = pk;
              if (kInt8 && p.acc_out) *reinterpret_cast<int4*>(p.acc_out + m * N + n) = si;
            }
          }
        }
        if (warp == 2 && lane == 0) p.counters[tile_id] = 0;   // ready for the next launch / replay
      }
    }

    // --------------------------------------- push-mode cluster reduce (owner)
    if (push_mode) {
      const bool got = __all_sync(0xffffffffu, wait_bar<true>(c.red_bar, 0, p, c, 6));
      if (warp == 2 && lane == 0) trace_stamp(p, 9);
      if (got && !*c.abort_flag) {
        const int S = p.S;
        const int W = TN / S;
        const int j0 = split * W;
        const int64_t M = m_end, N = n_end;
        // partial of split s for column j0 + jj of this thread's row
        auto slot = [&](int s, int jj) -> uint32_t { return slots[(s * kTileM + r) * W + jj]; };
        if (SWAP) {
          const int64_t n = x_row0 + r;
          const float bsn = !kBlocked ? rowsc[r] : 1.f;
          for (int jj = 0; jj < W; ++jj) {
            float sf = 0.f;
            int32_t si = 0;
#pragma unroll
            for (int s = 0; s < 16; ++s)
              if (s < S) {
                const uint32_t u = slot(s, jj);
                if (kInt8) si += static_cast<int32_t>(u);
                else sf += __uint_as_float(u);
              }
            const int64_t m = y_row0 + j0 + jj;
            if (n < N && m < M) {
              float val;
              if (kBlocked) val = sf;
              else val = (kInt8 ? static_cast<float>(si) : sf) * colsc[j0 + jj] * bsn;
              if constexpr (BIAS) val += bias_at(p, n - c_off);
              p.C[m * p.N + (n - c_off)] = __float2bfloat16_rn(val);
              if (kInt8 && p.acc_out) p.acc_out[m * p.N + (n - c_off)] = si;
            }
          }
        } else {
          const int64_t m = x_row0 + r;
          const float asm_ = !kBlocked ? rowsc[r] : 1.f;
          for (int jj = 0; jj < W; jj += 4) {   // W >= 4 for Standard tiles (TN >= 64, S <= 16)
            float f[4];
            int32_t iv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float sf = 0.f;
              int32_t si = 0;
#pragma unroll
              for (int s = 0; s < 16; ++s)
                if (s < S) {
                  const uint32_t u = slot(s, jj + e);
                  if (kInt8) si += static_cast<int32_t>(u);
                  else sf += __uint_as_float(u);
                }
              iv[e] = si;
              f[e] = kInt8 ? static_cast<float>(si) : sf;
            }
            const int64_t n = y_row0 + j0 + jj;
            if (m < M && n < N) {
              if (!kBlocked) {
#pragma unroll
                for (int e = 0; e < 4; ++e) f[e] = f[e] * asm_ * colsc[j0 + jj + e];
              }
              if constexpr (BIAS) {
#pragma unroll
                for (int e = 0; e < 4; ++e) f[e] += bias_at(p, n + e);
              }
              *reinterpret_cast<uint2*>(p.C + m * N + n) =
                  make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
              if (kInt8 && p.acc_out)
                *reinterpret_cast<int4*>(p.acc_out + m * N + n) = make_int4(iv[0], iv[1], iv[2], iv[3]);
            }
          }
        }
      }
      if (warp == 2 && lane == 0) trace_stamp(p, 10);
    }
  }

  // ------------------------------------------------ cluster Split-K reduce
  // The S CTAs of a tile form one cluster (cluster rank == split index).
  // After the first cluster barrier every partial tile sits in its CTA's
  // shared memory; CTA s sums columns [s TN/S, (s+1) TN/S) of all S partials
  // in the fixed order 0..S-1 (the order of the other reduction modes, so the
  // result is the same bit for bit), scales and stores them.  The second
  // barrier keeps every CTA alive until the others have read its partial.
  // All threads of all CTAs execute both barriers on every path.
  if (push_mode && warp < 2) {
    __syncwarp();
    cluster_wait_acquire();   // pairs with the arrive after set-up
  }
  if (cluster_launch && !push_mode) {
    __syncwarp();
    cluster_sync_all();
    if (warp == 2 && lane == 0) trace_stamp(p, 8);
    if (warp >= 2 && !*c.abort_flag) {
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const int S = p.S;
      const int W = TN / S;
      const int j0 = split * W;
      const int64_t M = p.M, N = p.N;
      uint32_t rb[16];
      const uint32_t local = smem_addr(ring);
#pragma unroll
      for (int s = 0; s < 16; ++s) rb[s] = s < S ? dsmem_map(local, static_cast<uint32_t>(s)) : 0u;
      if (SWAP) {
        const int64_t n = x_row0 + r;
        const float bsn = !kBlocked ? rowsc[r] : 1.f;
        for (int j = j0; j < j0 + W; ++j) {
          const uint32_t off = static_cast<uint32_t>((j * kTileM + r) * 4);
          uint32_t u[16];
#pragma unroll
          for (int s = 0; s < 16; ++s)
            if (s < S) u[s] = dsmem_ld_u32(rb[s] + off);
          float sf = 0.f;
          int32_t si = 0;
#pragma unroll
          for (int s = 0; s < 16; ++s)
            if (s < S) {
              if (kInt8) si += static_cast<int32_t>(u[s]);
              else sf += __uint_as_float(u[s]);
            }
          const int64_t m = y_row0 + j;
          if (n < N && m < M) {
            float val;
            if (kBlocked) val = sf;
            else val = (kInt8 ? static_cast<float>(si) : sf) * colsc[j] * bsn;
            if constexpr (BIAS) val += bias_at(p, n);
            p.C[m * N + n] = __float2bfloat16_rn(val);
            if (kInt8 && p.acc_out) p.acc_out[m * N + n] = si;
          }
        }
      } else {
        const int64_t m = x_row0 + r;
        const float asm_ = !kBlocked ? rowsc[r] : 1.f;
        for (int j = j0; j < j0 + W; j += 4) {   // W >= 4 for Standard tiles (TN >= 64, S <= 16)
          uint32_t u[4][16];
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int s = 0; s < 16; ++s)
              if (s < S) u[e][s] = dsmem_ld_u32(rb[s] + static_cast<uint32_t>(((j + e) * kTileM + r) * 4));
          float f[4];
          int32_t iv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float sf = 0.f;
            int32_t si = 0;
#pragma unroll
            for (int s = 0; s < 16; ++s)
              if (s < S) {
                if (kInt8) si += static_cast<int32_t>(u[e][s]);
                else sf += __uint_as_float(u[e][s]);
              }
            iv[e] = si;
            f[e] = kInt8 ? static_cast<float>(si) : sf;
          }
          const int64_t n = y_row0 + j;
          if (m < M && n < N) {
            if (!kBlocked) {
#pragma unroll
              for (int e = 0; e < 4; ++e) f[e] = f[e] * asm_ * colsc[j + e];
            }
            if constexpr (BIAS) {
#pragma unroll
              for (int e = 0; e < 4; ++e) f[e] += bias_at(p, n + e);
            }
            *reinterpret_cast<uint2*>(p.C + m * N + n) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
            if (kInt8 && p.acc_out)
              *reinterpret_cast<int4*>(p.acc_out + m * N + n) = make_int4(iv[0], iv[1], iv[2], iv[3]);
          }
        }
      }
    }
    if (warp == 2 && lane == 0) trace_stamp(p, 9);
    __syncwarp();
    cluster_sync_all();
    if (warp == 2 && lane == 0) trace_stamp(p, 10);
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

// ---------------------------------------------------------------------------
// Separate fixed-order Split-K reduction: C = scale(sum_{s=0..S-1} ws[s]).
// One thread per 4 consecutive outputs (N % 8 == 0).
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const GemmParams p) {
  constexpr bool kInt8 = FMT == kFmtInt8;
  constexpr bool kBlocked = is_block_fmt(FMT);
  grid_launch_dependents();   // before the wait, as the quantization kernels do
  grid_dependency_wait();
  const int64_t MN4 = p.M * p.N / 4;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < MN4;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e0 = t * 4;
    const int64_t m = e0 / p.N;
    const int64_t n = e0 - m * p.N;
    float f[4];
    int4 si = make_int4(0, 0, 0, 0);
    if (kInt8) {
      const int32_t* ws = reinterpret_cast<const int32_t*>(p.ws);
      for (int s = 0; s < p.S; ++s) {
        const int4 v = __ldcg(reinterpret_cast<const int4*>(ws + s * p.M * p.N + e0));
        si.x += v.x; si.y += v.y; si.z += v.z; si.w += v.w;
      }
      f[0] = si.x; f[1] = si.y; f[2] = si.z; f[3] = si.w;
    } else {
      const float* ws = reinterpret_cast<const float*>(p.ws);
      float4 sf = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < p.S; ++s) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(ws + s * p.M * p.N + e0));
        sf.x += v.x; sf.y += v.y; sf.z += v.z; sf.w += v.w;
      }
      f[0] = sf.x; f[1] = sf.y; f[2] = sf.z; f[3] = sf.w;
    }
    if (!kBlocked) {
      const float a = __ldg(p.a_s + m);
#pragma unroll
      for (int e = 0; e < 4; ++e) f[e] = f[e] * a * __ldg(p.b_s + n + e);
    }
    if (p.bias) {   // a separate pass: a runtime test costs nothing here
#pragma unroll
      for (int e = 0; e < 4; ++e) f[e] += bias_at(p, n + e);
    }
    *reinterpret_cast<uint2*>(p.C + e0) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
    if (kInt8 && p.acc_out) *reinterpret_cast<int4*>(p.acc_out + e0) = si;
  }
}

}  // namespace lq
