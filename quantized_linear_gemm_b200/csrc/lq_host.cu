// Host side of liblq: argument checks, variant selection (dispatch table +
// heuristic), per-device state (status word, Split-K workspace and arrival
// counters), TMA descriptor encoding and kernel launches.
//
// The variant space is the one of the blog's unified GEMM (PyTorch blog
// "Building a High-Performance and Portable vLLM Linear Backend with Helion",
// "Kernel Implementation": tunables split_k in {1, 2, ..., 256} and swap_ab),
// extended by the tile / pipeline choices of this implementation.  Instead of
// an online autotuner the library reads a static table keyed by
// (format, token bucket, N, K) that an offline on-device sweep writes; the
// token buckets are the decode sizes 1, 2, 4, 8, 16, 24, 32 for which the
// techfeed.io summary of the blog (section on hybrid dispatch, Fig. 2) says
// configs are tuned, followed by powers of two for larger M.
#include <cuda.h>
#include <cuda_runtime.h>

#include <array>
#include <atomic>
#include <cerrno>
#include <cfloat>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <fstream>
#include <memory>
#include <mutex>
#include <sstream>
#include <string>
#include <vector>

#include "../../include/lq.h"
#include "lq_kernels.h"

namespace {

using lq::GemmLaunch;
using lq::GemmParams;

constexpr int kMaxDevices = 64;
constexpr int kMaxSmemPerCta = 227 * 1024;
constexpr size_t kCounterCapacity = size_t(1) << 20;   // Split-K arrival counters per device
constexpr int kMaxStreamKCtas = 1024;                   // stream-K partial-ready flags per device
constexpr int kNumSms = 148;
constexpr int kMaxStages = 14;
// W8A8_INT8 sums products of int8 codes in int32: |a b| <= 128 * 128, so K
// up to 131071 can never wrap the accumulator (131071 * 2^14 < 2^31).
constexpr int64_t kInt8MaxK = 131071;   // the kernel's control block holds 4 x stages + 7 mbarriers (64 at most)
// 0: lq_quant_scaled_mm runs the quantization kernel and the GEMM unless a
// caller raises the limit.  Measured on B200 (Qwen3-8B decode shapes, FP8):
// the one-kernel path saves up to 1.2 us per call at M = 1 on the down
// projection but loses 0.3 - 2 us elsewhere, since its first MMA waits for
// the per-token amax (a pass over the CTA's slice of x plus a cluster
// exchange) that the separate kernel overlaps with the GEMM's weight stream.
constexpr int64_t kFuseMaxSliceBytes = 0;

// ---------------------------------------------------------------- devices
struct DeviceState {
  bool ready = false;
  int* status = nullptr;       // one int, bit i set when wait site i timed out
  int* counters = nullptr;     // kCounterCapacity ints, zero between calls
  int* sk_flags = nullptr;     // kMaxStreamKCtas ints: stream-K partial ready (zero between calls)
  void* ws = nullptr;          // Split-K partials
  size_t ws_bytes = 0;
  std::vector<void*> retired;  // smaller workspaces replaced by ws, kept until exit
};

std::mutex g_dev_mutex;
DeviceState g_dev[kMaxDevices];
std::atomic<uint64_t*> g_trace{nullptr};   // diagnostics: per-CTA stamps of the next launches
std::atomic<int> g_skip_stage{-1};          // test hook: K tile the producer never fills
std::atomic<uint64_t> g_wait_limit_override{0};
// Whether the caller has declared that weight operands are never written
// while a GEMM that reads them may run (lq_declare_static_weights).  Until
// then a variant taken from the dispatch table or the heuristic never
// streams weights before its dependency wait (pdl 2 is lowered to 1).
std::atomic<int> g_static_weights{0};

// The variant for a call that passed none: the table's entry for the token
// bucket, else the heuristic, with pdl 2 allowed only for static weights.
lq_variant default_variant(int fmt, int64_t M, int64_t N, int64_t K);

// Largest per-CTA activation slice (tokens x K range x 2 bytes) for which
// lq_quant_scaled_mm uses the fused kernel; LQ_FUSE_MAX_SLICE_BYTES overrides.
std::atomic<int64_t> g_fuse_limit_override{-1};

int64_t fuse_max_slice_bytes() {
  const int64_t o = g_fuse_limit_override.load();
  if (o >= 0) return o;
  static int64_t v = [] {
    const char* e = std::getenv("LQ_FUSE_MAX_SLICE_BYTES");
    if (e && *e) {
      char* end = nullptr;
      long long x = std::strtoll(e, &end, 10);
      if (end != e && x >= 0) return static_cast<int64_t>(x);
    }
    return static_cast<int64_t>(kFuseMaxSliceBytes);
  }();
  return v;
}

uint64_t wait_limit_ns() {
  const uint64_t o = g_wait_limit_override.load();
  if (o) return o;
  static uint64_t v = [] {
    const char* e = std::getenv("LQ_WAIT_LIMIT_NS");
    if (e && *e) {
      char* end = nullptr;
      unsigned long long x = std::strtoull(e, &end, 10);
      if (end != e && x > 0) return static_cast<uint64_t>(x);
    }
    return static_cast<uint64_t>(2000000000ull);   // 2 s
  }();
  return v;
}

bool stream_capturing(cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) != cudaSuccess) return false;
  return st != cudaStreamCaptureStatusNone;
}

lq_status init_device_locked(int dev) {
  DeviceState& d = g_dev[dev];
  if (d.ready) return LQ_OK;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return LQ_ERR_CUDA;
  if (cudaSetDevice(dev) != cudaSuccess) return LQ_ERR_CUDA;
  lq_status rc = LQ_OK;
  if (cudaMalloc(&d.status, sizeof(int)) != cudaSuccess ||
      cudaMalloc(&d.counters, kCounterCapacity * sizeof(int)) != cudaSuccess ||
      cudaMalloc(&d.sk_flags, kMaxStreamKCtas * sizeof(int)) != cudaSuccess ||
      cudaMemset(d.status, 0, sizeof(int)) != cudaSuccess ||
      cudaMemset(d.counters, 0, kCounterCapacity * sizeof(int)) != cudaSuccess ||
      cudaMemset(d.sk_flags, 0, kMaxStreamKCtas * sizeof(int)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    rc = LQ_ERR_CUDA;
  } else {
    d.ready = true;
  }
  cudaSetDevice(prev);
  return rc;
}

// The state of the current device, created on first use (refused while the
// stream is being captured, since creation allocates and synchronises).
lq_status device_state(cudaStream_t stream, DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mutex);
  if (!g_dev[dev].ready) {
    if (stream_capturing(stream)) return LQ_ERR_WORKSPACE;
    lq_status rc = init_device_locked(dev);
    if (rc != LQ_OK) return rc;
  }
  *out = &g_dev[dev];
  return LQ_OK;
}

// The Split-K workspace only grows.  A replaced buffer is never freed: a CUDA
// graph captured earlier keeps its address, and so may a call that another
// host thread is issuing at the same moment.  It is kept until the process
// exits; growth is at least twofold, so at most about log2(largest / 2 MiB)
// buffers are ever kept.
lq_status ensure_workspace(DeviceState* d, size_t bytes, cudaStream_t stream) {
  if (bytes <= d->ws_bytes) return LQ_OK;
  if (stream_capturing(stream)) return LQ_ERR_WORKSPACE;
  size_t want = bytes > 2 * d->ws_bytes ? bytes : 2 * d->ws_bytes;
  const size_t rounded = (want + (size_t(1) << 21) - 1) & ~((size_t(1) << 21) - 1);
  void* fresh = nullptr;
  if (cudaMalloc(&fresh, rounded) != cudaSuccess) {
    cudaGetLastError();
    return LQ_ERR_WORKSPACE;
  }
  if (d->ws) d->retired.push_back(d->ws);
  d->ws = fresh;
  d->ws_bytes = rounded;
  return LQ_OK;
}

// ---------------------------------------------------------- TMA encoding
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// K-major operand [rows, K] of bytes, tiles of box_rows x 128 bytes with the
// 128-byte swizzle; out-of-range rows / K are zero-filled by the TMA unit.
bool encode_operand(CUtensorMap* map, const void* ptr, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row-major bf16 activations [rows, K], tiles of box_rows x 128 elements
// (256 bytes, no swizzle); out-of-range rows / K are zero-filled.
bool encode_bf16_rows(CUtensorMap* map, const void* ptr, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2u};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// --------------------------------------------------------- dispatch table
struct TableEntry {
  int fmt;
  int64_t m_bucket, N, K;
  lq_variant v;
};

#include "dispatch_table.inc"   // kDefaultTable[], kDefaultTableSize

std::shared_ptr<const std::vector<TableEntry>> default_table() {
  auto t = std::make_shared<std::vector<TableEntry>>();
  for (size_t i = 0; i < kDefaultTableSize; ++i) t->push_back(kDefaultTable[i]);
  return t;
}

bool parse_table_file(const char* path, std::vector<TableEntry>* out, std::string* err);

// The table in force: the file named by LQ_DISPATCH_TABLE when it is set and
// valid, else the compiled-in table.
std::shared_ptr<const std::vector<TableEntry>>& table_slot() {
  static std::shared_ptr<const std::vector<TableEntry>> t = [] {
    const char* env = std::getenv("LQ_DISPATCH_TABLE");
    if (env && *env) {
      auto f = std::make_shared<std::vector<TableEntry>>();
      std::string err;
      if (parse_table_file(env, f.get(), &err)) return std::shared_ptr<const std::vector<TableEntry>>(f);
      std::fprintf(stderr, "lq: LQ_DISPATCH_TABLE=%s not used (%s)\n", env, err.c_str());
    }
    return default_table();
  }();
  return t;
}
std::mutex g_table_mutex;

std::shared_ptr<const std::vector<TableEntry>> current_table() {
  std::lock_guard<std::mutex> lk(g_table_mutex);
  return table_slot();
}

int64_t m_bucket(int64_t M) {
  static const int64_t pts[] = {1, 2, 4, 8, 16, 24, 32};
  for (int64_t p : pts)
    if (M <= p) return p;
  int64_t b = 64;
  while (b < M && b < (int64_t(1) << 40)) b <<= 1;
  return b;
}

// Deepest ring that fits when `ctas_per_sm` CTAs share one SM's shared memory.
int max_stages_fit(int tile_n, int ctas_per_sm, bool cluster_reduce, bool fuse = false) {
  const int share = (228 * 1024) / ctas_per_sm - 1024;
  const int budget = share < kMaxSmemPerCta ? share : kMaxSmemPerCta;
  int best = 2;
  for (int s = 2; s <= kMaxStages; ++s)
    if (lq::gemm_smem_bytes_for(tile_n, s, cluster_reduce, fuse) <= budget) best = s;
  return best;
}

// Deepest ring of the persistent kernels (one CTA per SM): persistent 1
// (one-SM tiles) or 2 (CTA pairs).
int max_persistent_stages(int tile_n, int persistent = 1) {
  int best = 2;
  for (int s = 2; s <= kMaxStages; ++s) {
    const int bytes = persistent == 2 ? lq::pair_smem_bytes_for(tile_n, s) : lq::persistent_smem_bytes_for(tile_n, s);   // 1, 3
    if (bytes > 0 && bytes <= kMaxSmemPerCta) best = s;
  }
  return best;
}

// Streaming multiprocessors of the current device (148 on B200).
int sm_count() {
  static int cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return kNumSms;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = kNumSms;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

// Co-resident CTA pairs of the pair kernel for (fmt, tile_n, bias, smem),
// cached per device (0 if the query fails).
int pair_capacity(int fmt, int tile_n, bool bias, int smem_bytes) {
  static std::mutex mu;
  static std::vector<std::pair<std::array<int, 5>, int>> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const std::array<int, 5> key{dev, fmt, tile_n, bias ? 1 : 0, smem_bytes};
  std::lock_guard<std::mutex> lk(mu);
  for (const auto& e : cache)
    if (e.first == key) return e.second;
  const int n = fmt == lq::kFmtFp8    ? lq::pair_capacity_fp8(tile_n, bias, smem_bytes)
                : fmt == lq::kFmtInt8  ? lq::pair_capacity_int8(tile_n, bias, smem_bytes)
                : fmt == lq::kFmtBlock ? lq::pair_capacity_block(tile_n, bias, smem_bytes)
                                       : lq::pair_capacity_block_e8m0(tile_n, bias, smem_bytes);
  cache.emplace_back(key, n);
  return n;
}

lq_variant heuristic_variant(int fmt, int64_t M, int64_t N, int64_t K) {
  lq_variant v{};
  const int64_t T = (K + 127) / 128;
  v.reduce = 1;
  v.pdl = 1;
  if (M <= 64) {
    v.swap_ab = 1;
    v.tile_n = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    const int64_t tiles = ((N + 127) / 128) * ((M + v.tile_n - 1) / v.tile_n);
    int S = 1;
    while (S < 256 && tiles * S * 2 <= 2 * kNumSms && T / (S * 2) >= 2) S *= 2;
    v.split_k = S;
    v.reduce = S <= 16 ? 2 : 1;
    const int per_split = static_cast<int>((T + S - 1) / S);
    const int cap = max_stages_fit(v.tile_n, 2, S > 1 && v.reduce == 2);
    v.stages = per_split < 2 ? 2 : (per_split > cap ? cap : per_split);
  } else {
    v.swap_ab = 0;
    v.tile_n = fmt == lq::kFmtBlock ? 128 : 256;
    const int64_t tiles = ((M + 127) / 128) * ((N + v.tile_n - 1) / v.tile_n);
    int S = 1;
    while (S < 256 && tiles * S < kNumSms && T / (S * 2) >= 4) S *= 2;
    v.split_k = S;
    v.reduce = S <= 16 ? 2 : 1;
    v.stages = max_stages_fit(v.tile_n, 1, S > 1 && v.reduce == 2);
    // many waves of tiles: persistent CTAs overlap each tile's epilogue with the next mainloop
    if (S == 1 && (fmt == lq::kFmtFp8 || fmt == lq::kFmtInt8) && tiles >= 2 * kNumSms) {
      v.persistent = 1;
      v.stages = max_persistent_stages(v.tile_n);
    }
  }
  return v;
}

bool lookup_table(int fmt, int64_t M, int64_t N, int64_t K, lq_variant* out);

lq_variant default_variant(int fmt, int64_t M, int64_t N, int64_t K) {
  lq_variant v{};
  if (!lookup_table(fmt, M, N, K, &v)) v = heuristic_variant(fmt, M, N, K);
  if (v.pdl == 2 && !g_static_weights.load()) v.pdl = 1;
  return v;
}

bool lookup_table(int fmt, int64_t M, int64_t N, int64_t K, lq_variant* out) {
  auto t = current_table();
  const int64_t mb = m_bucket(M);
  for (const TableEntry& e : *t) {
    if (e.fmt == fmt && e.m_bucket == mb && e.N == N && e.K == K) {
      *out = e.v;
      return true;
    }
  }
  // UE8M0 Block_FP8 without entries of its own: the Block_FP8 entries (every
  // Block_FP8 variant is valid for it)
  if (fmt == lq::kFmtBlockE8m0) return lookup_table(lq::kFmtBlock, M, N, K, out);
  return false;
}

// --------------------------------------------------------------- checks
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

// Dynamic shared memory of a launch whose CTAs each allocate `cols` tensor-
// memory columns, raised where needed so that no more CTAs fit on an SM
// (228 KB of shared memory, 1 KB reserved per CTA) than its 512 columns
// hold.  A CTA's tcgen05.alloc waits until enough columns are free, so two
// CTAs waiting for columns held by each other's cluster peers (Split-K
// clusters, stream-K chains) would never proceed.
int tmem_bounded_smem(int smem_bytes, int cols) {
  if (cols <= 0 || cols >= 512) cols = 512;
  const int fit = 512 / cols;                           // CTAs whose columns fit together
  const int floor_bytes = (228 * 1024) / (fit + 1) - 1024 + 1;   // fit + 1 CTAs exceed the SM
  return smem_bytes < floor_bytes ? floor_bytes : smem_bytes;
}

// Dynamic shared memory of a CTA-pair launch: the pair kernels that take all
// 512 tensor-memory columns (tile_n 256, both Block_FP8 forms) never share an
// SM with another of their CTAs, tile_n 128 pairs at most two.
int pair_launch_smem(int fmt, int tile_n, int stages) {
  return tmem_bounded_smem(lq::pair_smem_bytes_for(tile_n, stages), lq::tmem_cols_per_cta(fmt, tile_n, 2));
}

// Grid of a CTA-pair launch: one pair per (256-row tile, split) unit, at most
// as many pairs as fit on the device at once (each pair loops over units).
dim3 pair_grid(int fmt, int64_t M, int64_t gy, int split_k, int tile_n, bool bias, int smem_bytes) {
  const int64_t units = ((M + 255) / 256) * gy * split_k;
  int cap = pair_capacity(fmt, tile_n, bias, smem_bytes);
  if (cap <= 0) cap = sm_count() / 2;
  const int64_t pairs = units < cap ? units : cap;
  return dim3(static_cast<unsigned>(2 * pairs), 1, 1);
}

lq_status check_variant(int fmt, const lq_variant& v) {
  if (v.swap_ab != 0 && v.swap_ab != 1) return LQ_ERR_INVALID_ARG;
  if (v.split_k < 1 || v.split_k > 256) return LQ_ERR_INVALID_ARG;
  // the cluster reduction gives each CTA tile_n / split_k columns: powers of two; the
  // workspace reductions take any split count
  if (!is_pow2(v.split_k) && v.reduce == 2) return LQ_ERR_INVALID_ARG;
  if (v.reduce < 0 || v.reduce > 2) return LQ_ERR_INVALID_ARG;
  if (v.reduce == 2 && v.split_k > 16) return LQ_ERR_INVALID_ARG;   // a cluster holds at most 16 CTAs
  if (v.pdl < 0 || v.pdl > 2) return LQ_ERR_INVALID_ARG;
  if (v.swap_ab) {
    if (v.tile_n != 16 && v.tile_n != 32 && v.tile_n != 64) return LQ_ERR_INVALID_ARG;
  } else {
    if (v.tile_n != 64 && v.tile_n != 128 && v.tile_n != 256) return LQ_ERR_INVALID_ARG;
    if (fmt == lq::kFmtBlock && v.tile_n == 256) return LQ_ERR_INVALID_ARG;   // promotion in registers
  }
  if (v.stages != 0 && (v.stages < 2 || v.stages > kMaxStages)) return LQ_ERR_INVALID_ARG;
  if (v.persistent < 0 || v.persistent > 3) return LQ_ERR_INVALID_ARG;
  if (v.persistent) {
    // Standard orientation, FP8_Dynamic / W8A8_INT8 (CTA pairs and stream-K: tile_n 128 or 256), and
    // Block_FP8 (fp32 or UE8M0 scales) on CTA pairs with tile_n 128; one split, except CTA pairs, which
    // take Split-K with the separate reduction
    const bool block_pair = (fmt == lq::kFmtBlock || fmt == lq::kFmtBlockE8m0) && v.persistent == 2 && v.tile_n == 128;
    if (v.swap_ab || (fmt != lq::kFmtFp8 && fmt != lq::kFmtInt8 && !block_pair)) return LQ_ERR_INVALID_ARG;
    if (v.split_k != 1 && !(v.persistent == 2 && v.reduce == 0)) return LQ_ERR_INVALID_ARG;
    if (v.persistent >= 2 && v.tile_n == 64) return LQ_ERR_INVALID_ARG;
    const int bytes = v.persistent == 2 ? lq::pair_smem_bytes_for(v.tile_n, v.stages ? v.stages : 2)
                                        : lq::persistent_smem_bytes_for(v.tile_n, v.stages ? v.stages : 2);
    if (bytes > kMaxSmemPerCta) return LQ_ERR_INVALID_ARG;
    return LQ_OK;
  }
  if (v.stages != 0 &&
      lq::gemm_smem_bytes_for(v.tile_n, v.stages, v.split_k > 1 && v.reduce == 2) > kMaxSmemPerCta)
    return LQ_ERR_INVALID_ARG;
  return LQ_OK;
}

lq_status check_gemm_args(int fmt, const void* A, const float* a_s, const void* B, const float* b_s, const void* C,
                          int64_t M, int64_t N, int64_t K) {
  if (fmt < 0 || fmt > 3) return LQ_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return LQ_OK;
  if (!C) return LQ_ERR_INVALID_ARG;
  if (!aligned(C, 16)) return LQ_ERR_ALIGNMENT;
  if (K == 0) return LQ_OK;
  if (!A || !B || !a_s || !b_s) return LQ_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16)) return LQ_ERR_ALIGNMENT;
  if (fmt != lq::kFmtBlockE8m0 && (!aligned(a_s, 4) || !aligned(b_s, 4))) return LQ_ERR_ALIGNMENT;   // e8m0: bytes
  if (K % 16 != 0 || N % 8 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (lq::is_block_fmt(fmt) && (K % 128 != 0 || N % 128 != 0)) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (fmt == lq::kFmtInt8 && K > kInt8MaxK) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1)
    return LQ_ERR_UNSUPPORTED_SHAPE;
  return LQ_OK;
}

lq_status scaled_mm_impl(int fmt, const void* A, const float* a_s, const void* B, const float* b_s, void* C,
                         int32_t* acc_out, int64_t M, int64_t N, int64_t K, const lq_variant* variant,
                         cudaStream_t stream, const void* x_fused = nullptr, void* codes_out = nullptr,
                         float* scales_out = nullptr, const void* bias = nullptr) {
  const bool fused = x_fused != nullptr;
  lq_status rc = LQ_OK;
  if (!fused && variant && fmt >= 0 && fmt <= 3) {   // an explicit variant is checked before the pointers
    rc = check_variant(fmt, *variant);
    if (rc != LQ_OK) return rc;
  }
  rc = fused ? LQ_OK : check_gemm_args(fmt, A, a_s, B, b_s, C, M, N, K);
  if (rc != LQ_OK) return rc;
  if (acc_out && !aligned(acc_out, 16)) return LQ_ERR_ALIGNMENT;
  if (M == 0 || N == 0) return LQ_OK;
  if (K == 0) {
    if (acc_out && cudaMemsetAsync(acc_out, 0, static_cast<size_t>(M * N) * sizeof(int32_t), stream) != cudaSuccess)
      return LQ_ERR_CUDA;
    return lq::launch_fill_zero_bf16(static_cast<__nv_bfloat16*>(C), M * N, stream) == cudaSuccess ? LQ_OK
                                                                                                  : LQ_ERR_CUDA;
  }
  lq_variant v = variant ? *variant : default_variant(fmt, M, N, K);
  rc = check_variant(fmt, v);
  if (rc != LQ_OK) return rc;
  const bool cluster_reduce = v.split_k > 1 && v.reduce == 2;
  if (v.stages == 0)
    v.stages = v.persistent ? max_persistent_stages(v.tile_n, v.persistent)
                            : max_stages_fit(v.tile_n, 1, cluster_reduce, fused);
  if (fused && lq::gemm_smem_bytes_for(v.tile_n, v.stages, cluster_reduce, true) > kMaxSmemPerCta)
    v.stages = max_stages_fit(v.tile_n, 1, cluster_reduce, true);

  const int64_t x_rows = v.swap_ab ? N : M;
  const int64_t y_rows = v.swap_ab ? M : N;
  const int64_t gx = (x_rows + 127) / 128;
  const int64_t gy = (y_rows + v.tile_n - 1) / v.tile_n;
  if (gy > 65535 || gx > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;

  DeviceState* d = nullptr;
  rc = device_state(stream, &d);
  if (rc != LQ_OK) return rc;

  GemmLaunch l;
  std::memset(&l, 0, sizeof(l));
  GemmParams& p = l.p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.T = static_cast<int>((K + 127) / 128);
  p.KB = static_cast<int>(K / 128);
  p.S = v.split_k;
  p.stages = v.stages;
  p.reduce_mode = v.reduce;
  p.early_weights = v.pdl == 2 ? 1 : 0;
  p.a_s = a_s;
  p.b_s = b_s;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.acc_out = acc_out;
  p.status = d->status;
  p.wait_limit_ns = wait_limit_ns();
  p.trace = g_trace.load();
  p.skip_stage = g_skip_stage.load();
  p.x = static_cast<const __nv_bfloat16*>(x_fused);
  p.a_codes_out = static_cast<uint8_t*>(codes_out);
  p.a_scales_out = scales_out;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  if (v.persistent == 3) {   // stream-K: one partial slot [128 x tile_n] per CTA, and the ready flags
    const int64_t iters = ((M + 127) / 128) * gy * p.T;
    const int64_t ctas = iters < sm_count() ? iters : sm_count();
    if (ctas > kMaxStreamKCtas) return LQ_ERR_UNSUPPORTED_SHAPE;
    rc = ensure_workspace(d, static_cast<size_t>(ctas) * 128u * static_cast<size_t>(v.tile_n) * 4u, stream);
    if (rc != LQ_OK) return rc;
    p.ws = d->ws;
    p.counters = d->sk_flags;
  }
  if (v.split_k > 1 && v.reduce != 2) {   // the cluster reduction needs no global workspace
    const size_t need = static_cast<size_t>(v.split_k) * static_cast<size_t>(M) * static_cast<size_t>(N) * 4u;
    rc = ensure_workspace(d, need, stream);
    if (rc != LQ_OK) return rc;
    if (static_cast<size_t>(gx * gy) > kCounterCapacity) return LQ_ERR_UNSUPPORTED_SHAPE;
    p.ws = d->ws;
    p.counters = d->counters;
  }
  const void* x_ptr = v.swap_ab ? B : A;
  const void* y_ptr = v.swap_ab ? A : B;
  if (!encode_operand(&l.tmX, x_ptr, x_rows, K, 128)) return LQ_ERR_CUDA;
  if (v.persistent == 2) {
    // CTA pairs: each CTA loads half of the tile's weight rows
    if (!encode_operand(&l.tmY, y_ptr, y_rows, K, v.tile_n / 2)) return LQ_ERR_CUDA;
  } else if (fused) {
    // the kernel stages the bf16 activations and quantizes them itself
    if (!encode_bf16_rows(&l.tmY, x_fused, M, K, v.tile_n)) return LQ_ERR_CUDA;
  } else if (!encode_operand(&l.tmY, y_ptr, y_rows, K, v.tile_n)) {
    return LQ_ERR_CUDA;
  }
  l.fuse = fused ? 1 : 0;
  l.grid = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), static_cast<unsigned>(v.split_k));
  l.smem_bytes = tmem_bounded_smem(lq::gemm_smem_bytes_for(v.tile_n, v.stages, cluster_reduce, fused),
                                   lq::tmem_cols_per_cta(fmt, v.tile_n, 0));
  if (v.persistent == 1) {   // one CTA per SM (at most one per tile), each looping over tiles
    const int64_t tiles = gx * gy;
    const int64_t ctas = tiles < sm_count() ? tiles : sm_count();
    l.grid = dim3(static_cast<unsigned>(ctas), 1, 1);
    l.smem_bytes = tmem_bounded_smem(lq::persistent_smem_bytes_for(v.tile_n, v.stages),
                                     lq::tmem_cols_per_cta(fmt, v.tile_n, 1));
    l.persistent = 1;
  } else if (v.persistent == 3) {   // stream-K: one CTA per SM splitting tiles x K blocks
    const int64_t iters = ((M + 127) / 128) * gy * p.T;
    const int64_t ctas = iters < sm_count() ? iters : sm_count();
    l.grid = dim3(static_cast<unsigned>(ctas), 1, 1);
    l.smem_bytes = tmem_bounded_smem(lq::persistent_smem_bytes_for(v.tile_n, v.stages),
                                     lq::tmem_cols_per_cta(fmt, v.tile_n, 3));
    l.persistent = 3;
  } else if (v.persistent == 2) {   // clusters of two CTAs, 256-row tiles, each pair looping over units
    l.smem_bytes = pair_launch_smem(fmt, v.tile_n, v.stages);
    l.grid = pair_grid(fmt, M, gy, v.split_k, v.tile_n, bias != nullptr, l.smem_bytes);
    l.persistent = 2;
  }
  l.pdl = v.pdl != 0;
  l.cluster_z = (v.split_k > 1 && v.reduce == 2) ? v.split_k : 1;
  l.stream = stream;

  cudaError_t e;
  switch (fmt) {
    case lq::kFmtFp8: e = lq::launch_scaled_mm_fp8(l, v.swap_ab, v.tile_n); break;
    case lq::kFmtInt8: e = lq::launch_scaled_mm_int8(l, v.swap_ab, v.tile_n); break;
    case lq::kFmtBlockE8m0: e = lq::launch_scaled_mm_block_e8m0(l, v.swap_ab, v.tile_n); break;
    default: e = lq::launch_scaled_mm_block(l, v.swap_ab, v.tile_n); break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return LQ_ERR_CUDA;
  }
  if (v.split_k > 1 && v.reduce == 0) {
    e = lq::launch_splitk_reduce(fmt, p, v.pdl != 0, stream);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return LQ_ERR_CUDA;
    }
  }
  return LQ_OK;
}

bool parse_table_file(const char* path, std::vector<TableEntry>* out, std::string* err) {
  std::ifstream f(path);
  if (!f) {
    *err = "cannot open";
    return false;
  }
  std::string line;
  int lineno = 0;
  while (std::getline(f, line)) {
    ++lineno;
    const size_t hash = line.find('#');
    if (hash != std::string::npos) line.resize(hash);
    std::istringstream is(line);
    std::string fmt_s;
    if (!(is >> fmt_s)) continue;
    TableEntry e{};
    if (fmt_s == "fp8_dynamic" || fmt_s == "0") e.fmt = 0;
    else if (fmt_s == "w8a8_int8" || fmt_s == "1") e.fmt = 1;
    else if (fmt_s == "block_fp8" || fmt_s == "2") e.fmt = 2;
    else if (fmt_s == "block_fp8_ue8m0" || fmt_s == "3") e.fmt = 3;
    else {
      *err = "bad format at line " + std::to_string(lineno);
      return false;
    }
    long long mb, n, k;
    int sw, sk, tn, st, rd, pdl;
    if (!(is >> mb >> n >> k >> sw >> sk >> tn >> st >> rd >> pdl)) {
      *err = "short entry at line " + std::to_string(lineno);
      return false;
    }
    e.m_bucket = mb;
    e.N = n;
    e.K = k;
    int persistent = 0;   // optional 11th column
    if (!(is >> persistent)) persistent = 0;
    e.v = lq_variant{sw, sk, tn, st, rd, pdl, persistent};
    if (check_variant(e.fmt, e.v) != LQ_OK) {
      *err = "invalid variant at line " + std::to_string(lineno);
      return false;
    }
    out->push_back(e);
  }
  return true;
}

}  // namespace

// ======================================================================
extern "C" {

const char* lq_status_string(lq_status s) {
  switch (s) {
    case LQ_OK: return "LQ_OK";
    case LQ_ERR_INVALID_ARG: return "LQ_ERR_INVALID_ARG";
    case LQ_ERR_ALIGNMENT: return "LQ_ERR_ALIGNMENT";
    case LQ_ERR_UNSUPPORTED_SHAPE: return "LQ_ERR_UNSUPPORTED_SHAPE";
    case LQ_ERR_WORKSPACE: return "LQ_ERR_WORKSPACE";
    case LQ_ERR_CUDA: return "LQ_ERR_CUDA";
    case LQ_ERR_DEVICE_TIMEOUT: return "LQ_ERR_DEVICE_TIMEOUT";
    case LQ_ERR_TABLE: return "LQ_ERR_TABLE";
  }
  return "LQ_ERR_UNKNOWN";
}

const char* lq_version(void) { return "lq 0.1.0 (sm_100a)"; }

lq_status lq_test_inject_stall(int k_tile, uint64_t wait_limit_ns) {
  if (k_tile < -1) return LQ_ERR_INVALID_ARG;
  g_skip_stage.store(k_tile);
  g_wait_limit_override.store(wait_limit_ns);
  return LQ_OK;
}

lq_status lq_test_silu_bf16(const void* gate, void* out, int64_t n, lq_stream_t stream) {
  if (n < 0) return LQ_ERR_INVALID_ARG;
  if (n == 0) return LQ_OK;
  if (!gate || !out) return LQ_ERR_INVALID_ARG;
  if (!aligned(gate, 2) || !aligned(out, 2)) return LQ_ERR_ALIGNMENT;
  DeviceState* d = nullptr;
  const lq_status ds = device_state(reinterpret_cast<cudaStream_t>(stream), &d);
  if (ds != LQ_OK) return ds;
  return lq::launch_silu_bf16(gate, out, n, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? LQ_OK
                                                                                                  : LQ_ERR_CUDA;
}

int lq_declare_static_weights(int static_weights) {
  return g_static_weights.exchange(static_weights ? 1 : 0);
}

lq_status lq_set_trace(uint64_t* device_buffer) {
  g_trace.store(device_buffer);
  return LQ_OK;
}

lq_status lq_scaled_mm(lq_fmt fmt, const void* A, const float* a_scales, const void* B, const float* b_scales,
                       void* C, int64_t M, int64_t N, int64_t K, const lq_variant* variant, lq_stream_t stream) {
  return scaled_mm_impl(static_cast<int>(fmt), A, a_scales, B, b_scales, C, nullptr, M, N, K, variant,
                        reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// Variant for a grouped launch when the caller gives none, from an
// on-device sweep of the Qwen3-30B-A3B expert GEMMs (128 experts, top-8,
// 1..64 tokens; tile_n 16/32/64 x split_k 1..16 x 2..6 stages x pdl): one
// split always won (the experts already give enough CTAs), tile_n 16 (32
// only a hair faster at 512 rows), and a shallower ring as the number of
// tiles grows (more CTAs resident per SM).
lq_variant heuristic_grouped(int64_t T, int64_t E, int64_t N, int64_t K) {
  (void)K;
  lq_variant v{};
  v.swap_ab = 1;
  const int64_t per_expert = E > 0 ? (T + E - 1) / E : T;
  v.tile_n = per_expert <= 32 ? 16 : (per_expert <= 64 ? 32 : 64);
  v.split_k = 1;
  v.reduce = 2;
  v.pdl = 1;
  const int64_t tiles = ((N + 127) / 128) * (T < E ? T : E);   // non-empty experts <= min(T, E)
  v.stages = tiles <= 200 ? 4 : (tiles <= 800 ? 3 : 2);
  return v;
}

}  // namespace

lq_status lq_grouped_scaled_mm(lq_fmt fmt_, const void* A, const float* a_scales, const void* B,
                               const float* b_scales, void* C, const int32_t* expert_offsets, int64_t E, int64_t T,
                               int64_t N, int64_t K, const lq_variant* variant, lq_stream_t stream_) {
  const int fmt = static_cast<int>(fmt_);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (fmt != lq::kFmtFp8 && fmt != lq::kFmtInt8) return LQ_ERR_INVALID_ARG;
  if (E < 0 || T < 0 || N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (T == 0 || N == 0) return LQ_OK;
  if (E == 0 || !C) return LQ_ERR_INVALID_ARG;
  if (!aligned(C, 16)) return LQ_ERR_ALIGNMENT;
  if (K == 0)
    return lq::launch_fill_zero_bf16(static_cast<__nv_bfloat16*>(C), T * N, stream) == cudaSuccess ? LQ_OK
                                                                                                   : LQ_ERR_CUDA;
  if (!A || !B || !a_scales || !b_scales || !expert_offsets) return LQ_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(a_scales, 4) || !aligned(b_scales, 4) ||
      !aligned(expert_offsets, 4))
    return LQ_ERR_ALIGNMENT;
  if (K % 16 != 0 || N % 8 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (T > 0x7FFFFFFF || E > 0x7FFFFFFF || E * N > 0x7FFFFFFF || K > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (fmt == lq::kFmtInt8 && K > kInt8MaxK) return LQ_ERR_UNSUPPORTED_SHAPE;
  lq_variant v = variant ? *variant : heuristic_grouped(T, E, N, K);
  if (v.swap_ab != 1) return LQ_ERR_INVALID_ARG;   // tokens on the MMA N side
  if (v.split_k > 16) return LQ_ERR_INVALID_ARG;
  if (v.split_k > 1) v.reduce = 2;   // the Split-K CTAs of a tile reduce in their cluster
  lq_status rc = check_variant(fmt, v);
  if (rc != LQ_OK) return rc;
  const bool cluster_reduce = v.split_k > 1;
  if (v.stages == 0) v.stages = max_stages_fit(v.tile_n, 1, cluster_reduce);
  const int64_t gx = (N + 127) / 128;
  // sum over experts of ceil(count / tile_n) <= T / tile_n + (number of
  // non-empty experts) <= ceil(T / tile_n) + min(E, T)
  const int64_t gy = (T + v.tile_n - 1) / v.tile_n + (E < T ? E : T);
  if (gy > 65535) return LQ_ERR_UNSUPPORTED_SHAPE;

  DeviceState* d = nullptr;
  rc = device_state(stream, &d);
  if (rc != LQ_OK) return rc;
  GemmLaunch l;
  std::memset(&l, 0, sizeof(l));
  GemmParams& p = l.p;
  p.M = T;
  p.N = N;
  p.K = K;
  p.T = static_cast<int>((K + 127) / 128);
  p.KB = static_cast<int>(K / 128);
  p.S = v.split_k;
  p.stages = v.stages;
  p.reduce_mode = 2;
  p.early_weights = v.pdl == 2 ? 1 : 0;
  p.a_s = a_scales;
  p.b_s = b_scales;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.status = d->status;
  p.wait_limit_ns = wait_limit_ns();
  p.trace = g_trace.load();
  p.skip_stage = g_skip_stage.load();
  p.expert_offsets = expert_offsets;
  p.num_experts = static_cast<int>(E);
  if (!encode_operand(&l.tmX, B, E * N, K, 128) || !encode_operand(&l.tmY, A, T, K, v.tile_n)) return LQ_ERR_CUDA;
  l.grid = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), static_cast<unsigned>(v.split_k));
  l.smem_bytes = tmem_bounded_smem(lq::gemm_smem_bytes_for(v.tile_n, v.stages, cluster_reduce),
                                   lq::tmem_cols_per_cta(fmt, v.tile_n, 0));
  l.pdl = v.pdl != 0;
  l.cluster_z = cluster_reduce ? v.split_k : 1;
  l.grouped = 1;
  l.stream = stream;
  const cudaError_t e =
      fmt == lq::kFmtFp8 ? lq::launch_scaled_mm_fp8(l, 1, v.tile_n) : lq::launch_scaled_mm_int8(l, 1, v.tile_n);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return LQ_ERR_CUDA;
  }
  return LQ_OK;
}

lq_status lq_scaled_mm_bias(lq_fmt fmt, const void* A, const float* a_scales, const void* B, const float* b_scales,
                            const void* bias, void* C, int64_t M, int64_t N, int64_t K, const lq_variant* variant,
                            lq_stream_t stream) {
  if (bias && !aligned(bias, 2)) return LQ_ERR_ALIGNMENT;
  if (!bias && M > 0 && N > 0) return LQ_ERR_INVALID_ARG;
  if (K == 0 && M > 0 && N > 0) return LQ_ERR_UNSUPPORTED_SHAPE;   // C would be the bias alone: not a GEMM
  return scaled_mm_impl(static_cast<int>(fmt), A, a_scales, B, b_scales, C, nullptr, M, N, K, variant,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, bias);
}

lq_status lq_scaled_mm_i32acc(const void* A, const float* a_scales, const void* B, const float* b_scales, void* C,
                              int32_t* acc_out, int64_t M, int64_t N, int64_t K, const lq_variant* variant,
                              lq_stream_t stream) {
  if (!acc_out && M > 0 && N > 0) return LQ_ERR_INVALID_ARG;
  return scaled_mm_impl(lq::kFmtInt8, A, a_scales, B, b_scales, C, acc_out, M, N, K, variant,
                        reinterpret_cast<cudaStream_t>(stream));
}

lq_status lq_quant_scaled_mm(lq_fmt fmt_, const void* x, const void* B, const float* b_scales, void* C,
                             void* a_codes, float* a_scales, int64_t M, int64_t N, int64_t K,
                             const lq_variant* variant, lq_stream_t stream_) {
  const int fmt = static_cast<int>(fmt_);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (fmt != lq::kFmtFp8 && fmt != lq::kFmtInt8) return LQ_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return LQ_OK;
  if (!x || !B || !b_scales || !C || !a_codes || !a_scales) return LQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(a_codes, 16) || !aligned(a_scales, 4) ||
      !aligned(b_scales, 4))
    return LQ_ERR_ALIGNMENT;
  if (K % 16 != 0 || N % 8 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;
  if (fmt == lq::kFmtInt8 && K > kInt8MaxK) return LQ_ERR_UNSUPPORTED_SHAPE;
  const lq_variant v = variant ? *variant : default_variant(fmt, M, N, K);
  // Each CTA of the fused kernel reads its tokens' slice of x once more to
  // find the per-token amax before any code exists; that read sits on the
  // critical path, so the kernel is used only while the slice is small.
  const int64_t T = (K + 127) / 128;
  const int64_t slice_bytes = (M < v.tile_n ? M : v.tile_n) * ((T + v.split_k - 1) / v.split_k) * 128 * 2;
  lq_variant vf = v;
  if (vf.split_k > 1) vf.reduce = 2;   // the per-token amax is exchanged inside the Split-K cluster
  const bool fusable = K > 0 && v.swap_ab == 1 && v.split_k <= 16 && v.split_k * v.tile_n <= 512 &&
                       slice_bytes <= fuse_max_slice_bytes() && check_variant(fmt, vf) == LQ_OK;
  if (!fusable) {
    // quantize, then scaled_mm (same codes, scales and result as the fused kernel);
    // the variant is checked before the first launch
    const lq_status vrc = check_variant(fmt, v);
    if (vrc != LQ_OK) return vrc;
    if (lq::launch_quant_per_token(fmt, x, a_codes, a_scales, M, K, stream) != cudaSuccess) {
      cudaGetLastError();
      return LQ_ERR_CUDA;
    }
    return scaled_mm_impl(fmt, a_codes, a_scales, B, b_scales, C, nullptr, M, N, K, &v, stream);
  }
  return scaled_mm_impl(fmt, a_codes, a_scales, B, b_scales, C, nullptr, M, N, K, &vf, stream, x, a_codes,
                        a_scales);
}

int64_t lq_set_fuse_limit(int64_t max_slice_bytes) {
  const int64_t prev = fuse_max_slice_bytes();
  g_fuse_limit_override.store(max_slice_bytes < 0 ? -1 : max_slice_bytes);
  return prev;
}

lq_status lq_quant_per_token(lq_fmt fmt, const void* x, void* q, float* scales, int64_t M, int64_t K,
                             lq_stream_t stream) {
  if (fmt != LQ_FP8_DYNAMIC && fmt != LQ_W8A8_INT8) return LQ_ERR_INVALID_ARG;
  if (M < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (M == 0) return LQ_OK;
  if (!x || !q || !scales) return LQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 8) || !aligned(scales, 4)) return LQ_ERR_ALIGNMENT;
  if (K % 16 != 0 || M > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;
  return lq::launch_quant_per_token(static_cast<int>(fmt), x, q, scales, M, K,
                                    reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_quant_per_token_group128(const void* x, void* q, float* scales, int64_t M, int64_t K,
                                      lq_stream_t stream) {
  if (M < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return LQ_OK;
  if (!x || !q || !scales) return LQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 8) || !aligned(scales, 4)) return LQ_ERR_ALIGNMENT;
  if (K % 128 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if ((M * (K / 128) + 15) / 16 > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;
  return lq::launch_quant_group128(x, q, scales, M, K, false, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

namespace {

lq_status check_producer(int64_t M, int64_t K, int64_t multiple, const void* in, const void* residual,
                         const void* weight, bool need_weight, float eps, const void* q, const float* scales) {
  if (M < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (!in || !q || !scales || (need_weight && !weight)) return LQ_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || eps > FLT_MAX) return LQ_ERR_INVALID_ARG;
  if (!aligned(in, 16) || (residual && !aligned(residual, 16)) || (weight && !aligned(weight, 16)) ||
      !aligned(q, 8) || !aligned(scales, 4))
    return LQ_ERR_ALIGNMENT;
  if (K == 0 || K % multiple != 0 || K > lq::producer_max_row() || M > 0x7FFFFFFF)
    return LQ_ERR_UNSUPPORTED_SHAPE;
  return LQ_OK;
}

}  // namespace

lq_status lq_rms_norm_dynamic_per_token_quant(lq_fmt fmt, const void* x, void* residual, const void* weight,
                                              float eps, void* q, float* scales, int64_t M, int64_t K,
                                              lq_stream_t stream) {
  if (fmt != LQ_FP8_DYNAMIC && fmt != LQ_W8A8_INT8) return LQ_ERR_INVALID_ARG;
  if (M == 0 && K >= 0) return LQ_OK;
  const lq_status rc = check_producer(M, K, 16, x, residual, weight, true, eps, q, scales);
  if (rc != LQ_OK) return rc;
  DeviceState* d = nullptr;
  const lq_status ds = device_state(reinterpret_cast<cudaStream_t>(stream), &d);
  if (ds != LQ_OK) return ds;
  return lq::launch_rms_norm_quant(static_cast<int>(fmt), false, x, residual, weight, eps, q, scales, M, K,
                                   d->status, wait_limit_ns(), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_rms_norm_per_block_quant(const void* x, void* residual, const void* weight, float eps, void* q,
                                      float* scales, int64_t M, int64_t K, lq_stream_t stream) {
  if (M == 0 && K >= 0) return LQ_OK;
  const lq_status rc = check_producer(M, K, 128, x, residual, weight, true, eps, q, scales);
  if (rc != LQ_OK) return rc;
  DeviceState* d = nullptr;
  const lq_status ds = device_state(reinterpret_cast<cudaStream_t>(stream), &d);
  if (ds != LQ_OK) return ds;
  return lq::launch_rms_norm_quant(lq::kFmtFp8, true, x, residual, weight, eps, q, scales, M, K, d->status,
                                   wait_limit_ns(), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_silu_and_mul_dynamic_per_token_quant(lq_fmt fmt, const void* gate_up, void* q, float* scales,
                                                  int64_t M, int64_t I, lq_stream_t stream) {
  if (fmt != LQ_FP8_DYNAMIC && fmt != LQ_W8A8_INT8) return LQ_ERR_INVALID_ARG;
  if (M == 0 && I >= 0) return LQ_OK;
  const lq_status rc = check_producer(M, I, 16, gate_up, nullptr, nullptr, false, 0.f, q, scales);
  if (rc != LQ_OK) return rc;
  DeviceState* d = nullptr;
  const lq_status ds = device_state(reinterpret_cast<cudaStream_t>(stream), &d);
  if (ds != LQ_OK) return ds;
  return lq::launch_silu_mul_quant(static_cast<int>(fmt), false, gate_up, q, scales, M, I, d->status,
                                   wait_limit_ns(), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_silu_and_mul_per_block_quant(const void* gate_up, void* q, float* scales, int64_t M, int64_t I,
                                          lq_stream_t stream) {
  if (M == 0 && I >= 0) return LQ_OK;
  const lq_status rc = check_producer(M, I, 128, gate_up, nullptr, nullptr, false, 0.f, q, scales);
  if (rc != LQ_OK) return rc;
  DeviceState* d = nullptr;
  const lq_status ds = device_state(reinterpret_cast<cudaStream_t>(stream), &d);
  if (ds != LQ_OK) return ds;
  return lq::launch_silu_mul_quant(lq::kFmtFp8, true, gate_up, q, scales, M, I, d->status, wait_limit_ns(),
                                   reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_quant_weight_block128(const void* w, void* q, float* scales, int64_t N, int64_t K,
                                   lq_stream_t stream) {
  if (N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return LQ_OK;
  if (!w || !q || !scales) return LQ_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 8) || !aligned(scales, 4)) return LQ_ERR_ALIGNMENT;
  if (N % 128 != 0 || K % 128 != 0 || N / 128 > 65535 || K / 128 > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;
  return lq::launch_quant_weight_block128(w, q, scales, N, K, false, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_quant_per_token_group128_ue8m0(const void* x, void* q, uint8_t* scales, int64_t M, int64_t K,
                                           lq_stream_t stream) {
  if (M < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return LQ_OK;
  if (!x || !q || !scales) return LQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 8)) return LQ_ERR_ALIGNMENT;
  if (K % 128 != 0) return LQ_ERR_UNSUPPORTED_SHAPE;
  if ((M * (K / 128) + 15) / 16 > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;
  return lq::launch_quant_group128(x, q, scales, M, K, true, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_quant_weight_block128_ue8m0(const void* w, void* q, uint8_t* scales, int64_t N, int64_t K,
                                         lq_stream_t stream) {
  if (N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return LQ_OK;
  if (!w || !q || !scales) return LQ_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 8)) return LQ_ERR_ALIGNMENT;
  if (N % 128 != 0 || K % 128 != 0 || N / 128 > 65535 || K / 128 > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;
  return lq::launch_quant_weight_block128(w, q, scales, N, K, true, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? LQ_OK
             : LQ_ERR_CUDA;
}

lq_status lq_select_variant(lq_fmt fmt, int64_t M, int64_t N, int64_t K, lq_variant* out) {
  if (!out || fmt < 0 || fmt > 3 || M < 0 || N < 0 || K < 0) return LQ_ERR_INVALID_ARG;
  *out = default_variant(static_cast<int>(fmt), M, N, K);
  return LQ_OK;
}

lq_status lq_load_dispatch_table(const char* path) {
  if (!path) {
    std::lock_guard<std::mutex> lk(g_table_mutex);
    table_slot() = default_table();
    return LQ_OK;
  }
  auto t = std::make_shared<std::vector<TableEntry>>();
  std::string err;
  if (!parse_table_file(path, t.get(), &err)) return LQ_ERR_TABLE;
  std::lock_guard<std::mutex> lk(g_table_mutex);
  table_slot() = t;
  return LQ_OK;
}

int64_t lq_dispatch_table_size(void) { return static_cast<int64_t>(current_table()->size()); }

lq_status lq_init_device(int device) {
  if (device < 0 || device >= kMaxDevices) return LQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_dev_mutex);
  return init_device_locked(device);
}

lq_status lq_reserve_workspace(int device, size_t bytes) {
  if (device < 0 || device >= kMaxDevices) return LQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_dev_mutex);
  lq_status rc = init_device_locked(device);
  if (rc != LQ_OK) return rc;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess || cudaSetDevice(device) != cudaSuccess) return LQ_ERR_CUDA;
  rc = ensure_workspace(&g_dev[device], bytes, nullptr);
  cudaSetDevice(prev);
  return rc;
}

size_t lq_workspace_bytes(lq_fmt fmt, int64_t M, int64_t N, int64_t K, const lq_variant* variant) {
  if (M <= 0 || N <= 0 || K <= 0 || fmt < 0 || fmt > 3) return 0;
  const lq_variant v = variant ? *variant : default_variant(static_cast<int>(fmt), M, N, K);
  if (v.persistent == 3 && !v.swap_ab && v.tile_n > 0) {   // stream-K partial slots
    const int64_t iters = ((M + 127) / 128) * ((N + v.tile_n - 1) / v.tile_n) * ((K + 127) / 128);
    const int64_t ctas = iters < sm_count() ? iters : sm_count();
    return static_cast<size_t>(ctas) * 128u * static_cast<size_t>(v.tile_n) * 4u;
  }
  if (v.split_k <= 1 || v.reduce == 2) return 0;
  return static_cast<size_t>(v.split_k) * static_cast<size_t>(M) * static_cast<size_t>(N) * 4u;
}

lq_status lq_device_status(int device) {
  if (device < 0 || device >= kMaxDevices) return LQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_dev_mutex);
  DeviceState& d = g_dev[device];
  if (!d.ready) return LQ_OK;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess || cudaSetDevice(device) != cudaSuccess) return LQ_ERR_CUDA;
  int word = 0;
  lq_status rc = LQ_OK;
  if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpy(&word, d.status, sizeof(int), cudaMemcpyDeviceToHost) !=
                                                    cudaSuccess ||
      cudaMemset(d.status, 0, sizeof(int)) != cudaSuccess) {
    rc = LQ_ERR_CUDA;
  } else if (word != 0) {
    // A CTA that gave up did not count itself: clear the Split-K arrival
    // counters so that later calls start from zero.
    cudaMemset(d.counters, 0, kCounterCapacity * sizeof(int));
    cudaMemset(d.sk_flags, 0, kMaxStreamKCtas * sizeof(int));
    cudaDeviceSynchronize();
    rc = LQ_ERR_DEVICE_TIMEOUT;
  }
  cudaSetDevice(prev);
  return rc;
}

}  // extern "C"

// ======================================================================
// Allocation-free scaled_mm.
//
// Some callers cannot call cudaMalloc when they run a GEMM: code that runs
// while a CUDA graph is being captured with the global capture mode (where
// an allocation is an unsafe call), frameworks whose memory is handed out
// only by their own pool allocator, and latency-critical services that must
// not allocate or synchronise after start-up.  lq_scaled_mm may allocate its
// per-device state and Split-K workspace on first use; the entry point below
// never does.  Its Split-K partials live in a fixed array in device memory
// that the library reserves when it is loaded.
namespace {

// Split-K partial sums of lq_scaled_mm_noalloc: [split_k, M, N] fp32 / int32.
// Every GPU that loads the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};   // device address of g_noalloc_scratch per device

// Device address of the scratch array on the current device.  The first call
// on a device looks it up (cudaGetSymbolAddress, with that device current).
lq_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LQ_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return LQ_OK;
}

}  // namespace

extern "C" lq_status lq_scaled_mm_noalloc(lq_fmt fmt_, const void* A, const float* a_scales, const void* B,
                                          const float* b_scales, void* C, int64_t M, int64_t N, int64_t K,
                                          const lq_variant* variant, lq_stream_t stream_) {
  const int fmt = static_cast<int>(fmt_);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  // Split-K partials always go through the scratch array and the separate
  // fixed-order reduction kernel (no arrival counters, nothing to re-arm);
  // stream-K, whose partials need a workspace, runs as persistent CTAs.
  auto noalloc_form = [](lq_variant v) {
    if (v.split_k > 1) v.reduce = 0;
    if (v.persistent == 3) v.persistent = 1;
    return v;
  };
  lq_status rc = LQ_OK;
  if (variant && fmt >= 0 && fmt <= 3) {   // an explicit variant is checked before the pointers
    rc = check_variant(fmt, noalloc_form(*variant));
    if (rc != LQ_OK) return rc;
  }
  rc = check_gemm_args(fmt, A, a_scales, B, b_scales, C, M, N, K);
  if (rc != LQ_OK) return rc;
  if (M == 0 || N == 0) return LQ_OK;
  if (K == 0)
    return lq::launch_fill_zero_bf16(static_cast<__nv_bfloat16*>(C), M * N, stream) == cudaSuccess ? LQ_OK
                                                                                                  : LQ_ERR_CUDA;
  lq_variant v = noalloc_form(variant ? *variant : default_variant(fmt, M, N, K));
  rc = check_variant(fmt, v);
  if (rc != LQ_OK) return rc;
  const size_t need = v.split_k > 1 ? static_cast<size_t>(v.split_k) * static_cast<size_t>(M) *
                                          static_cast<size_t>(N) * 4u
                                    : 0;
  if (need > kNoAllocScratchBytes) return LQ_ERR_WORKSPACE;
  if (v.stages == 0)
    v.stages = v.persistent ? max_persistent_stages(v.tile_n, v.persistent) : max_stages_fit(v.tile_n, 1, false);

  const int64_t x_rows = v.swap_ab ? N : M;
  const int64_t y_rows = v.swap_ab ? M : N;
  const int64_t gx = (x_rows + 127) / 128;
  const int64_t gy = (y_rows + v.tile_n - 1) / v.tile_n;
  if (gy > 65535 || gx > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED_SHAPE;

  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != LQ_OK) return rc;

  GemmLaunch l;
  std::memset(&l, 0, sizeof(l));
  GemmParams& p = l.p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.T = static_cast<int>((K + 127) / 128);
  p.KB = static_cast<int>(K / 128);
  p.S = v.split_k;
  p.stages = v.stages;
  p.reduce_mode = 0;
  p.early_weights = v.pdl == 2 ? 1 : 0;
  p.a_s = a_scales;
  p.b_s = b_scales;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.ws = v.split_k > 1 ? scratch : nullptr;
  p.counters = nullptr;
  p.acc_out = nullptr;
  p.status = nullptr;   // a timed-out wait leaves C undefined and is not reported here
  p.wait_limit_ns = wait_limit_ns();
  p.trace = nullptr;
  p.skip_stage = -1;
  const void* x_ptr = v.swap_ab ? B : A;
  const void* y_ptr = v.swap_ab ? A : B;
  if (!encode_operand(&l.tmX, x_ptr, x_rows, K, 128) ||
      !encode_operand(&l.tmY, y_ptr, y_rows, K, v.persistent == 2 ? v.tile_n / 2 : v.tile_n))
    return LQ_ERR_CUDA;
  l.grid = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), static_cast<unsigned>(v.split_k));
  l.smem_bytes = tmem_bounded_smem(lq::gemm_smem_bytes_for(v.tile_n, v.stages, false),
                                   lq::tmem_cols_per_cta(fmt, v.tile_n, 0));
  if (v.persistent == 1) {   // split_k 1: no scratch; one CTA per SM looping over tiles
    const int64_t tiles = gx * gy;
    const int64_t ctas = tiles < sm_count() ? tiles : sm_count();
    l.grid = dim3(static_cast<unsigned>(ctas), 1, 1);
    l.smem_bytes = tmem_bounded_smem(lq::persistent_smem_bytes_for(v.tile_n, v.stages),
                                     lq::tmem_cols_per_cta(fmt, v.tile_n, 1));
    l.persistent = 1;
  } else if (v.persistent == 2) {   // clusters of two CTAs, 256-row tiles, each pair looping over units
    l.smem_bytes = pair_launch_smem(fmt, v.tile_n, v.stages);
    l.grid = pair_grid(fmt, M, gy, v.split_k, v.tile_n, false, l.smem_bytes);
    l.persistent = 2;
  }
  l.pdl = v.pdl != 0;
  l.cluster_z = 1;
  l.stream = stream;
  cudaError_t e;
  switch (fmt) {
    case lq::kFmtFp8: e = lq::launch_scaled_mm_fp8(l, v.swap_ab, v.tile_n); break;
    case lq::kFmtInt8: e = lq::launch_scaled_mm_int8(l, v.swap_ab, v.tile_n); break;
    case lq::kFmtBlockE8m0: e = lq::launch_scaled_mm_block_e8m0(l, v.swap_ab, v.tile_n); break;
    default: e = lq::launch_scaled_mm_block(l, v.swap_ab, v.tile_n); break;
  }
  if (e == cudaSuccess && v.split_k > 1) e = lq::launch_splitk_reduce(fmt, p, v.pdl != 0, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return LQ_ERR_CUDA;
  }
  return LQ_OK;
}
