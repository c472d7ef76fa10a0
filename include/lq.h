/*
 * lq.h - C ABI of liblq, the quantized linear-layer GEMM ("scaled_mm") for
 * NVIDIA B200 (sm_100a).
 *
 * What it computes
 * ----------------
 *   C[m, n] = bf16( sum_k dequant(A_q)[m, k] * dequant(B_q)[k, n] )
 *
 * in the three formats that the PyTorch blog post "Building a
 * High-Performance and Portable vLLM Linear Backend with Helion" defines in
 * its section "Helion Linear Backend > Scope":
 *
 *   LQ_FP8_DYNAMIC : e4m3 codes, one fp32 scale per token (row of A) and one
 *                    per output channel (row n of the stored weight);
 *   LQ_W8A8_INT8   : int8 codes, the same scale granularity, int32 sums;
 *   LQ_BLOCK_FP8   : e4m3 codes, one activation scale per 1x128 K-group and
 *                    one weight scale per 128x128 (n, k) block.
 *   LQ_BLOCK_FP8_UE8M0 : Block_FP8 whose scales are powers of two stored as
 *                    UE8M0 bytes (value 2^(b - 127)), the scale format the
 *                    24-ai.news report (section "実際の制限事項") says DeepGEMM
 *                    needs on B200 and the per-group quantizer lacked.
 *
 * The algorithmic variants Standard, Split-K and Swap-AB of the same page's
 * section "Kernel Implementation" are selected per call by an lq_variant (or
 * by the dispatch table when the caller passes NULL); every variant computes
 * the same C.
 *
 * Conventions shared by all entry points
 * --------------------------------------
 *  - Every pointer argument except file paths and lq_variant* is a DEVICE
 *    pointer of the current CUDA device, owned by the caller.  Arrays are
 *    dense and row-major with the shapes given below.
 *  - A is [M, K], one row per token.  B is stored [N, K] (one row per output
 *    channel, K contiguous), as a linear layer stores its weight: the
 *    logical b[k, n] of the techfeed.io summary's code sample (section
 *    "何が面白いのか"), transposed.  C is [M, N] bf16.
 *  - e4m3 codes are OCP E4M3 "fn" bytes; int8 codes are two's complement.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronise.  They may be captured into a
 *    CUDA graph once the device has been initialised (lq_init_device, or any
 *    earlier non-captured call on that device).
 *  - All arguments are checked before anything is launched; a failed check
 *    launches nothing and returns an error code.  No C++ exception crosses
 *    this interface.
 *  - The library allocates device memory only in lq_init_device,
 *    lq_reserve_workspace and, outside stream capture, when a Split-K call
 *    needs more workspace than it holds.  It never frees device memory that
 *    a call may have used: a workspace that is replaced by a larger one is
 *    kept until the process exits, so a CUDA graph captured earlier stays
 *    valid.
 *  - variant == NULL: the dispatch table's (or the heuristic's) variant,
 *    with pdl lowered from 2 to 1 unless lq_declare_static_weights(1) has
 *    been called, so that a call never reads B before the kernels ahead of
 *    it on the stream have finished (a weight quantized on the same stream
 *    just before is safe).
 */
#ifndef LQ_H_
#define LQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, spelled without the CUDA headers. */
typedef struct CUstream_st *lq_stream_t;

typedef enum {
  LQ_FP8_DYNAMIC = 0,
  LQ_W8A8_INT8 = 1,
  LQ_BLOCK_FP8 = 2,
  LQ_BLOCK_FP8_UE8M0 = 3
} lq_fmt;

typedef enum {
  LQ_OK = 0,
  LQ_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, bad variant field */
  LQ_ERR_ALIGNMENT = 2,         /* a pointer is not aligned as required      */
  LQ_ERR_UNSUPPORTED_SHAPE = 3, /* a size breaks a divisibility/limit rule   */
  LQ_ERR_WORKSPACE = 4,         /* Split-K workspace would have to grow during
                                   stream capture, or allocation failed      */
  LQ_ERR_CUDA = 5,              /* a CUDA runtime/driver call failed          */
  LQ_ERR_DEVICE_TIMEOUT = 6,    /* a kernel gave up on a bounded wait         */
  LQ_ERR_TABLE = 7              /* dispatch table file missing or malformed   */
} lq_status;

/*
 * One point of the variant space (the blog's tunables split_k and swap_ab,
 * plus the tile and pipeline choices of this implementation).
 *
 *  swap_ab : 0 = Standard: tokens on the tensor-core M side (128-row tiles of
 *            A), weights on the N side (tile_n rows of B per tile);
 *            1 = Swap-AB: C^T = B . A^T is computed, 128 weight rows on the M
 *            side and tile_n tokens on the N side; the epilogue transposes
 *            back on store.
 *  split_k : 1..256; a power of two with reduce 2.
 *            Split s owns the 128-wide K tiles
 *            [floor(s*T/S), floor((s+1)*T/S)), T = ceil(K/128); a split may
 *            be empty.  Partials are summed in the fixed order s = 0..S-1,
 *            so results are reproducible bit for bit.
 *  tile_n  : Standard: 64, 128 or 256 (Block_FP8: 64 or 128);
 *            Swap-AB: 16, 32 or 64.
 *  stages  : depth of the shared-memory ring (2..14), 0 = the deepest that
 *            fits.
 *  reduce  : for split_k > 1: 0 = partials to a global workspace and a
 *            separate reduction kernel; 1 = partials to the workspace and the
 *            last CTA to finish a tile reduces it (arrival counter); 2 = the
 *            split_k CTAs of a tile form a thread-block cluster and reduce
 *            through distributed shared memory, each finishing a slice of the
 *            tile (split_k <= 16, no workspace).  All three sum the partials
 *            in the order s = 0..split_k-1 and give identical results.
 *  persistent : 0 = one output tile per CTA; 1 = persistent CTAs (Standard
 *            orientation, split_k 1, FP8_DYNAMIC / W8A8_INT8; tile_n 64, 128
 *            or 256): one CTA per SM loops over the output tiles, its
 *            shared-memory ring runs on across tiles, and the accumulator is
 *            double-buffered in tensor memory so that a tile's epilogue
 *            overlaps the next tile's mainloop; 2 = the same on CTA pairs
 *            (clusters of two, one MMA of 256 rows over both SMs with
 *            tcgen05 cta_group::2; each CTA loads 128 rows of A and half of
 *            the tile's tile_n weight rows): FP8_DYNAMIC / W8A8_INT8 with
 *            tile_n 128 or 256, and BLOCK_FP8 / BLOCK_FP8_UE8M0 with tile_n
 *            128 (fp32 scales: promotion per 128-K block in four
 *            tensor-memory buffers; UE8M0 scales: the tensor core's block
 *            scaling over the pair).  Same results bit for bit as the one-SM
 *            kernels with the same K grouping.  Pairs also take split_k > 1
 *            with reduce 0: the units
 *            (256-row tile, split) are spread over the pairs and the
 *            separate reduction sums the workspace partials, as for the
 *            one-SM tiles; 3 = stream-K (tile_n 128 or 256): one CTA per SM,
 *            each taking an equal contiguous share of all tiles' K blocks;
 *            a tile split between CTAs is finished by the CTA holding its
 *            last K block, which adds the others' partial sums (kept in the
 *            library's workspace: the restrictions of Split-K with reduce
 *            0 / 1 apply) in K order.  Bitwise reproducible, but FP8 results
 *            are not bit-identical to the other schedules (its fp32 partial
 *            sums are grouped differently; INT8 is exact in every schedule).
 *            For shapes with few output tiles.  lq_scaled_mm_noalloc runs it
 *            as 1.
 *  pdl     : 0 = plain launch;
 *            1 = programmatic dependent launch: the kernel's set-up overlaps
 *            the tail of the previous kernel on the stream, and all of its
 *            global-memory accesses wait until that kernel has completed;
 *            2 = as 1, and the first weight tiles (B) are streamed before
 *            that wait.  With 2 the caller guarantees that B and b_scales
 *            are not being written by any kernel that may still be running
 *            when the call is launched (true of model weights, which are
 *            written once before inference).  A NULL variant uses 2 only
 *            after lq_declare_static_weights(1).
 */
typedef struct {
  int32_t swap_ab;
  int32_t split_k;
  int32_t tile_n;
  int32_t stages;
  int32_t reduce;
  int32_t pdl;
  int32_t persistent;
} lq_variant;

/*
 * scaled_mm: C = dequant(A) . dequant(B)^T in bf16 (round to nearest even).
 *
 * Defined by: PyTorch blog "Building a High-Performance and Portable vLLM
 * Linear Backend with Helion", sections "Helion Linear Backend > Scope"
 * (formats, scale granularity) and "Kernel Implementation" (variants).
 *
 *   fmt      : LQ_FP8_DYNAMIC, LQ_W8A8_INT8, LQ_BLOCK_FP8 or
 *              LQ_BLOCK_FP8_UE8M0.
 *   A        : [M, K] codes (uint8 e4m3 or int8), 16-byte aligned.
 *   a_scales : fp32; [M] for FP8_DYNAMIC/W8A8_INT8, [M, K/128] for BLOCK_FP8;
 *              for BLOCK_FP8_UE8M0 [M, K/128] UE8M0 bytes (pass the byte
 *              array's address, any alignment).
 *   B        : [N, K] codes, 16-byte aligned.
 *   b_scales : fp32; [N] for FP8_DYNAMIC/W8A8_INT8, [N/128, K/128] for
 *              BLOCK_FP8; [N/128, K/128] UE8M0 bytes for BLOCK_FP8_UE8M0.
 *   C        : [M, N] bf16 output, 16-byte aligned.
 *   M, N, K  : M >= 0, N >= 0, K >= 0; K % 16 == 0 and N % 8 == 0;
 *              the Block_FP8 formats also need K % 128 == 0, N % 128 == 0;
 *              W8A8_INT8 needs K <= 131071 (so that no int32 sum of int8
 *              products can wrap).  M == 0 or N == 0 is a no-op; K == 0
 *              writes C = 0.
 *   variant  : NULL = the dispatch table's choice for (fmt, M, N, K), which
 *              reads B only after the previous kernels on the stream have
 *              finished unless lq_declare_static_weights(1) was called.
 *   stream   : CUDA stream.
 *
 * Errors: LQ_ERR_INVALID_ARG / LQ_ERR_ALIGNMENT / LQ_ERR_UNSUPPORTED_SHAPE
 * before any launch (an explicit variant is checked first, before the
 * pointers and sizes); LQ_ERR_WORKSPACE when split_k > 1 needs a larger
 * workspace while `stream` is capturing; LQ_ERR_CUDA when a launch fails.
 * A Split-K call with reduce 0 or 1 uses the library's per-device workspace:
 * such calls on different streams of one device must not overlap in time on
 * the GPU (they share the workspace and the arrival counters).  The
 * workspace only grows (a replaced one is kept until exit), so a graph
 * captured before a later call grew it stays valid; capturing such a call
 * needs the workspace reserved first (lq_reserve_workspace with the largest
 * split_k * M * N * 4), since growth is refused during capture.  Calls with
 * split_k == 1 or reduce 2 (the dispatch table's choices) use no workspace
 * and have neither restriction.
 */
lq_status lq_scaled_mm(lq_fmt fmt, const void *A, const float *a_scales,
                       const void *B, const float *b_scales, void *C,
                       int64_t M, int64_t N, int64_t K,
                       const lq_variant *variant, lq_stream_t stream);

/*
 * scaled_mm with a bias: C[m, n] = bf16(acc * a_s * b_s + bias[n]), the
 * scaled accumulator and the bias added in fp32 before the one rounding to
 * bf16.  bias: [N] bf16 (device, 2-byte aligned, not NULL).  Same formats,
 * arguments, variants and errors as lq_scaled_mm; K == 0 is refused with
 * LQ_ERR_UNSUPPORTED_SHAPE.  The blog has no bias (a linear layer of the
 * served models has none); it serves layers that do, and the N-sliced
 * multi-GPU linear, whose shards each add their slice of it.
 */
lq_status lq_scaled_mm_bias(lq_fmt fmt, const void *A, const float *a_scales,
                            const void *B, const float *b_scales, const void *bias,
                            void *C, int64_t M, int64_t N, int64_t K,
                            const lq_variant *variant, lq_stream_t stream);

/*
 * Grouped (mixture-of-experts) scaled_mm: one launch for all experts, each
 * an ordinary FP8_Dynamic / W8A8_INT8 linear layer (a next target named by
 * ai-radar.it, "Helion in vLLM: il tuning dei GEMM diventa ricerca, non
 * artigianato GPU", section "Oltre Hopper: Blackwell, AMD, TPU e il
 * perimetro del fork": many small experts, where Split-K and Swap-AB matter
 * more).
 *
 *   A        : [T, K] token codes, sorted by expert: rows
 *              expert_offsets[e] .. expert_offsets[e+1]-1 go to expert e.
 *   a_scales : [T] per-token scales.
 *   B        : [E, N, K] weight codes (experts stacked), b_scales [E, N].
 *   C        : [T, N] bf16 out; row t = token t times its expert's weights.
 *   expert_offsets : DEVICE int32 [E + 1], offsets[0] = 0, non-decreasing,
 *              offsets[E] = T.  Read by the kernel (no host synchronisation,
 *              so it may come from a router kernel on the same stream).  The
 *              kernel clamps every offset to [0, T] and uses the running max,
 *              so a malformed table gives wrong rows, never a store outside
 *              C.
 *   variant  : NULL = a rule from T, E and N (tuned on the Qwen3-30B-A3B
 *              expert GEMMs: one split, tile_n 16, 2-4 stages); else
 *              Swap-AB only (swap_ab = 1, tile_n 16/32/64), split_k <= 16
 *              with the cluster reduction (reduce is forced to 2).
 * The grid has ceil(T / tile_n) + min(E, T) token tiles per weight tile
 * (a bound on the sum over experts of ceil(count / tile_n)); CTAs past the
 * last tile of the last expert exit at once.  The kernel reads the table
 * after waiting for the previous kernel on the stream.  K % 16 == 0, N % 8 == 0,
 * E * N < 2^31.  Errors as lq_scaled_mm; LQ_ERR_INVALID_ARG for Block_FP8,
 * E = 0 with T > 0, or a Standard variant.
 */
lq_status lq_grouped_scaled_mm(lq_fmt fmt, const void *A, const float *a_scales,
                               const void *B, const float *b_scales, void *C,
                               const int32_t *expert_offsets, int64_t E, int64_t T,
                               int64_t N, int64_t K, const lq_variant *variant,
                               lq_stream_t stream);

/*
 * Test hook for W8A8_INT8: as lq_scaled_mm(LQ_W8A8_INT8, ...) and also
 * writes the exact int32 accumulator sum_k A[m,k]*B[n,k] to acc_out [M, N]
 * (device, 16-byte aligned), so that it can be compared bit for bit with an
 * exact integer reference.  Same arguments and errors as lq_scaled_mm.
 * Source: W8A8_INT8 (int8 operands, int32 accumulation) of the PyTorch blog "Building a High-Performance and Portable vLLM Linear
 * Backend with Helion", section "Helion Linear Backend > Scope";
 * the accumulator output is a test interface of this library.
 */
lq_status lq_scaled_mm_i32acc(const void *A, const float *a_scales,
                              const void *B, const float *b_scales, void *C,
                              int32_t *acc_out, int64_t M, int64_t N, int64_t K,
                              const lq_variant *variant, lq_stream_t stream);

/*
 * Quantize the activations and multiply, in one kernel where possible: the
 * per-token dynamic quantization of lq_quant_per_token fused with
 * lq_scaled_mm (the in-GEMM activation quantization that the report's fused
 * quantization kernels motivate; 24-ai.news report, section "kernels
 * integrated into vLLM", and the blog's aim of fewer kernel calls per
 * forward pass).
 *
 *   fmt      : LQ_FP8_DYNAMIC or LQ_W8A8_INT8.
 *   x        : [M, K] bf16 activations, 16-byte aligned.
 *   B, b_scales, C, M, N, K : as lq_scaled_mm.
 *   a_codes  : [M, K] out, the activation codes (16-byte aligned).
 *   a_scales : [M] out, the per-token scales.
 *   variant  : NULL = the dispatch table's choice for (fmt, M, N, K), with
 *              pdl as for lq_scaled_mm.
 * a_codes, a_scales and C equal, bit for bit, those of lq_quant_per_token
 * followed by lq_scaled_mm with the same variant.  By default the two
 * kernels run (lq_quant_per_token, then lq_scaled_mm).  With a Swap-AB
 * variant (split_k <= 16 and split_k * tile_n <= 512) whose CTAs each see an
 * activation slice (min(M, tile_n) x ceil(K / 128 / split_k) x 128 bf16
 * values) no larger than a limit that is 0 by default (raise it with
 * lq_set_fuse_limit or the environment variable LQ_FUSE_MAX_SLICE_BYTES,
 * read once), one kernel does both: the TMA stages each bf16 activation tile
 * beside the weight tile, the CTA's idle epilogue warps quantize it into the
 * tensor core's operand slot, and the Split-K CTAs form a cluster (reduce is
 * forced to 2) that exchanges the per-token amax; a variant that is not
 * valid with that cluster takes the two-kernel path.  The two-kernel path
 * runs lq_scaled_mm with the caller's variant unchanged.  Errors as
 * lq_scaled_mm, all found before the first launch; LQ_ERR_INVALID_ARG for
 * Block_FP8.
 */
lq_status lq_quant_scaled_mm(lq_fmt fmt, const void *x, const void *B,
                             const float *b_scales, void *C, void *a_codes,
                             float *a_scales, int64_t M, int64_t N, int64_t K,
                             const lq_variant *variant, lq_stream_t stream);

/*
 * Sets, for this process, the largest per-CTA activation slice (bytes) for
 * which lq_quant_scaled_mm uses its one-kernel path; 0 = never fuse, a
 * negative value restores the default (0, or LQ_FUSE_MAX_SLICE_BYTES).
 * Returns the limit in force before the call.  A tuning and test hook: it
 * changes which kernels run, never the results.  No page defines it.
 */
int64_t lq_set_fuse_limit(int64_t max_slice_bytes);

/*
 * Allocation-free scaled_mm, for callers that cannot call cudaMalloc when
 * they run a GEMM: code running while a CUDA graph is captured with the
 * global capture mode (an allocation is an unsafe call there), frameworks
 * whose device memory comes only from their own pool allocator, and
 * latency-critical services that must not allocate or synchronise after
 * start-up.  lq_scaled_mm may allocate its per-device state and Split-K
 * workspace on first use; this entry point never calls cudaMalloc, cudaFree
 * or any allocating routine.  The blog has no counterpart: it is an
 * interface of this library only.
 *
 * Same arguments, layouts and results as lq_scaled_mm.  Differences:
 *  - With split_k > 1 the partial sums go to a fixed 16 MiB array in device
 *    memory that the library reserves when it is loaded (every GPU that
 *    loads the library holds it until the process exits), and are summed by
 *    the separate fixed-order reduction kernel (the variant's reduce field is
 *    ignored).  A call whose split_k * M * N * 4 bytes exceed 16 MiB returns
 *    LQ_ERR_WORKSPACE before launching anything.
 *  - Every call shares that array and it keeps the last call's partials, so
 *    calls that overlap on the GPU (different streams without ordering, or
 *    concurrent graph branches) race and give wrong results.  Calls ordered
 *    on one stream are safe.  Nothing in the array needs to start at zero.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress with that device current); make that first call
 *    before capturing a CUDA graph.
 *  - A kernel that gives up on a bounded wait leaves C undefined; this entry
 *    point has no status word, so lq_device_status does not report it.
 */
lq_status lq_scaled_mm_noalloc(lq_fmt fmt, const void *A, const float *a_scales,
                               const void *B, const float *b_scales, void *C,
                               int64_t M, int64_t N, int64_t K,
                               const lq_variant *variant, lq_stream_t stream);

/*
 * Dynamic per-token activation quantization (the blog's integrated kernel
 * dynamic_per_token_scaled_fp8_quant, as listed in the 24-ai.news report,
 * section "kernels integrated into vLLM"; the int8 form serves W8A8_INT8).
 *
 *   fmt    : LQ_FP8_DYNAMIC (e4m3, Q = 448) or LQ_W8A8_INT8 (int8, Q = 127).
 *   x      : [M, K] bf16, 16-byte aligned.
 *   q      : [M, K] codes out, 8-byte aligned.
 *   scales : [M] fp32 out.  s = max(fp32(amax_row / Q), 2^-126),
 *            q = encode(fp32(x / s)) with x / s correctly rounded,
 *            e4m3 round-to-nearest-even with saturation to +-448, int8
 *            round-half-even clamped to +-127.
 *   K % 16 == 0.  M == 0 is a no-op.
 * The same call quantizes a weight [N, K] per output channel.
 */
lq_status lq_quant_per_token(lq_fmt fmt, const void *x, void *q, float *scales,
                             int64_t M, int64_t K, lq_stream_t stream);

/*
 * 1x128 group quantization of Block_FP8 activations (the blog's
 * per_token_group_fp8_quant): one scale per (row, 128-wide K group).
 *   x [M, K] bf16 (16-byte aligned) -> q [M, K] e4m3, scales [M, K/128] fp32.
 *   K % 128 == 0.  Same rule as lq_quant_per_token with Q = 448.
 */
lq_status lq_quant_per_token_group128(const void *x, void *q, float *scales,
                                      int64_t M, int64_t K, lq_stream_t stream);

/*
 * Producer-side fused quantizers: the kernel that computes a GEMM's input
 * activations quantizes them in the same pass (the blog's integrated kernels
 * rms_norm_dynamic_per_token_quant, rms_norm_per_block_quant,
 * silu_and_mul_dynamic_per_token_quant and silu_and_mul_per_block_quant:
 * 24-ai.news report, section "kernels integrated into vLLM").  The report names
 * them only; the value quantized is the bf16 output of a Qwen3-style layer,
 * with each rounding fixed so that codes and scales are reproducible bit for
 * bit:
 *
 * RMSNorm, with an optional residual added first:
 *   h = bf16(fp32(x + residual)), written back to residual (h = x if NULL);
 *   v = sum_k h^2 / K + eps in fp64; r = fp32(1 / sqrt(v)) (fp64 sqrt and
 *   divide); y = bf16(fp32(bf16(fp32(h * r)) * weight)).
 * SiLU-and-multiply of gate_up = [g | u] ([M, 2I], the fused gate/up output):
 *   y = bf16(fp32(bf16(silu(g)) * u)), silu(g) = g / (1 + exp(-g)) rounded
 *   once from its exact value.
 * Then y is quantized exactly as lq_quant_per_token (per row, FP8 or INT8)
 * or lq_quant_per_token_group128 (per 1 x 128 group, FP8) would.
 *
 *   x, residual, weight, gate_up : bf16, 16-byte aligned; residual may be
 *            NULL and is otherwise read and overwritten in place.
 *   weight : [K] bf16 RMSNorm gain.  eps: finite, >= 0.
 *   q      : [M, K] (or [M, I]) codes out, 8-byte aligned.
 *   scales : [M] (per token) or [M, K/128] (per block) fp32 out.
 *   K (or I): a multiple of 16 (per token) or 128 (per block), at most
 *            32768, else LQ_ERR_UNSUPPORTED_SHAPE (also for K = 0).
 *   M == 0 is a no-op.  One CTA per row; the row stays in registers.
 */
lq_status lq_rms_norm_dynamic_per_token_quant(lq_fmt fmt, const void *x, void *residual,
                                              const void *weight, float eps, void *q,
                                              float *scales, int64_t M, int64_t K,
                                              lq_stream_t stream);
lq_status lq_rms_norm_per_block_quant(const void *x, void *residual, const void *weight,
                                      float eps, void *q, float *scales, int64_t M,
                                      int64_t K, lq_stream_t stream);
lq_status lq_silu_and_mul_dynamic_per_token_quant(lq_fmt fmt, const void *gate_up, void *q,
                                                  float *scales, int64_t M, int64_t I,
                                                  lq_stream_t stream);
lq_status lq_silu_and_mul_per_block_quant(const void *gate_up, void *q, float *scales,
                                          int64_t M, int64_t I, lq_stream_t stream);

/*
 * Block_FP8 quantizers with UE8M0 scales: the scale of a group is the
 * smallest power of two 2^e with amax / 2^e <= 448 (e clamped to
 * [-127, 127]; an all-zero group gets e = -127), written as the byte e + 127;
 * codes are e4m3(x * 2^-e), exact scaling then round to nearest even, so no
 * code saturates.
 *   lq_quant_per_token_group128_ue8m0: x [M, K] bf16 (16-byte aligned) ->
 *     q [M, K] e4m3 (8-byte aligned), scales [M, K/128] bytes; K % 128 == 0.
 *   lq_quant_weight_block128_ue8m0: w [N, K] -> q [N, K], scales
 *     [N/128, K/128] bytes; N % 128 == 0 and K % 128 == 0.
 * Errors as lq_quant_per_token_group128 / lq_quant_weight_block128.
 * Source: 24-ai.news report, section "実際の制限事項" (the UE8M0 scale format
 * needed on B200), read as the OCP microscaling E8M0 scale.
 */
lq_status lq_quant_per_token_group128_ue8m0(const void *x, void *q, uint8_t *scales,
                                           int64_t M, int64_t K, lq_stream_t stream);
lq_status lq_quant_weight_block128_ue8m0(const void *w, void *q, uint8_t *scales,
                                         int64_t N, int64_t K, lq_stream_t stream);

/*
 * 128x128 block quantization of a Block_FP8 weight stored [N, K]: one scale
 * per (n-block, k-block) from the amax over the whole block.
 *   w [N, K] bf16 (16-byte aligned) -> q [N, K] e4m3, scales [N/128, K/128].
 *   N % 128 == 0 and K % 128 == 0.
 * Source: the Block_FP8 weight scales of the PyTorch blog "Building a High-Performance and Portable vLLM Linear
 * Backend with Helion", section "Helion Linear Backend > Scope".
 */
lq_status lq_quant_weight_block128(const void *w, void *q, float *scales,
                                   int64_t N, int64_t K, lq_stream_t stream);

/*
 * The variant that lq_scaled_mm uses for (fmt, M, N, K) when given NULL:
 * the dispatch-table entry for the token bucket of M (the next of
 * 1,2,4,8,16,24,32, then powers of two), else a built-in heuristic.
 * Host-only; writes *out.  Errors: LQ_ERR_INVALID_ARG.
 * Source: the per-shape tuned configurations and the dispatch by token count
 * of the techfeed.io summary of the blog, sections "オートチューニングの仕組み"
 * and "ハイブリッドディスパッチ：Helionの弱点を補う設計" (Fig. 2).
 */
lq_status lq_select_variant(lq_fmt fmt, int64_t M, int64_t N, int64_t K,
                            lq_variant *out);

/*
 * Replace the dispatch table by the entries of a text file (one entry per
 * line: "fmt m_bucket N K swap_ab split_k tile_n stages reduce pdl
 * [persistent]", '#' starts a comment; fmt is fp8_dynamic, w8a8_int8,
 * block_fp8, block_fp8_ue8m0 or 0..3).  path == NULL restores the compiled-in table.  At
 * start-up the environment variable LQ_DISPATCH_TABLE, when set, names a
 * file that replaces the compiled-in table.  On error
 * the current table is kept and LQ_ERR_TABLE is returned.  Safe while other
 * threads call lq_scaled_mm: each call uses the table in force when it looked
 * up its variant.  Source: as lq_select_variant.
 */
lq_status lq_load_dispatch_table(const char *path);

/* Number of entries in the current dispatch table (as lq_select_variant). */
int64_t lq_dispatch_table_size(void);

/*
 * Create the per-device state of `device` (status word, Split-K arrival
 * counters) if it does not exist yet.  Call it before capturing a CUDA graph
 * that contains lq calls.  Errors: LQ_ERR_CUDA.  Library infrastructure: no
 * page defines it (likewise the workspace, status, trace, version and status
 * string entry points below).
 */
lq_status lq_init_device(int device);

/*
 * Make sure the per-device Split-K workspace holds at least `bytes` bytes
 * (a Split-K call needs split_k * M * N * 4).  A smaller workspace that it
 * replaces is kept until exit (graphs captured with it stay valid); growth
 * is at least twofold.  Call it before stream capture.
 */
lq_status lq_reserve_workspace(int device, size_t bytes);

/* Workspace bytes that lq_scaled_mm needs for (fmt, M, N, K, variant):
 * split_k * M * N * 4 for reduce 0 or 1, else 0. */
size_t lq_workspace_bytes(lq_fmt fmt, int64_t M, int64_t N, int64_t K,
                          const lq_variant *variant);

/*
 * Read and clear the device status word of `device`: LQ_OK, or
 * LQ_ERR_DEVICE_TIMEOUT if a kernel since the last read gave up on a
 * bounded wait (its output is then undefined).  Synchronises the device.
 */
lq_status lq_device_status(int device);

/*
 * Declare (static_weights != 0) that the weights B and b_scales of every
 * later call are never written by a kernel that may still be running when a
 * GEMM reading them is launched (model weights, written once before
 * inference).  Then a NULL variant may stream the first weight tiles before
 * waiting for the previous kernel on the stream (the table's pdl 2), which
 * hides their latency behind that kernel's tail.  Without the declaration
 * (the default) a NULL variant waits first (pdl 1), which is safe when a
 * weight is quantized or updated on the same stream just before.  Explicit
 * variants are used as given.  Process-wide; a captured CUDA graph keeps the
 * variants chosen at capture time.  Returns the previous setting (0 or 1).
 * Library infrastructure: no page defines it.
 */
int lq_declare_static_weights(int static_weights);

/*
 * Diagnostics: while `device_buffer` is non-NULL, every scaled_mm kernel
 * launched afterwards writes 12 %globaltimer stamps (ns) per CTA to
 * device_buffer[cta * 12 + i], cta = x + gx * (y + gy * z) over the launch
 * grid: 0 entry, 1 set-up done, 2 producer past the wait for the previous
 * kernel, 3 first operand stage landed, 4 last MMA issued, 5 accumulator
 * ready, 6 outputs or partials written, 7 exit, and for the cluster Split-K
 * reduction 8 past its first barrier, 9 reduced tile stored, 10 past its
 * second barrier (slots a launch does not reach keep their old contents).
 * The buffer must hold 12 uint64 per CTA of every traced launch.  A launch
 * captured into a CUDA graph keeps the pointer that was set at capture
 * time.  NULL turns tracing off.
 */
lq_status lq_set_trace(uint64_t *device_buffer);

/*
 * Test hook for failure detection.  While k_tile >= 0, every scaled_mm
 * kernel launched afterwards leaves the k_tile-th K tile of each CTA
 * unloaded, so the tensor-core warp's bounded wait for it runs out: the
 * kernel sets the device status word, drains its copies, frees its tensor
 * memory and returns (C undefined), and lq_device_status reports
 * LQ_ERR_DEVICE_TIMEOUT.  Nothing faults or hangs.  wait_limit_ns > 0
 * replaces the bound of every wait (default 2 s, or LQ_WAIT_LIMIT_NS) until
 * the hook is called again with 0.  k_tile = -1 turns the hook off.
 * Errors: LQ_ERR_INVALID_ARG for k_tile < -1.
 */
lq_status lq_test_inject_stall(int k_tile, uint64_t wait_limit_ns);

/*
 * Test hook for the SiLU of lq_silu_and_mul_dynamic_per_token_quant and
 * lq_silu_and_mul_per_block_quant: out[i] = bf16(silu(gate[i])), silu(g) =
 * g / (1 + e^-g) rounded once to bf16 from its exact value (24-ai.news
 * report, section "vLLMに統合されたカーネル"), computed by the same device
 * code as those kernels.  gate and out: device bf16 [n], 2-byte aligned,
 * owned by the caller; asynchronous on `stream`.
 * Errors: LQ_ERR_INVALID_ARG (n < 0, NULL pointer with n > 0),
 * LQ_ERR_ALIGNMENT, LQ_ERR_CUDA.
 */
lq_status lq_test_silu_bf16(const void *gate, void *out, int64_t n, lq_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char *lq_status_string(lq_status status);

/* Library version string (static storage). */
const char *lq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LQ_H_ */
