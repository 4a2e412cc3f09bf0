// rlscan_api.cu -- host side of librlscan: argument checks, launch plans,
// look-back workspaces and the extern "C" entry points declared in
// include/rlscan.h.  Every step of the computation runs in the kernels of
// scan_kernel.cuh; this file only validates, plans and launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>
#include <utility>
#include <vector>

#include "../../include/rlscan.h"
#include "estimators.cuh"
#include "retrace.cuh"
#include "scan_core.cuh"
#include "scan_kernel.cuh"
#include "tm_kernel.cuh"

using namespace rlscan;

namespace {

// ---------------------------------------------------------------------------
// options
// ---------------------------------------------------------------------------
std::atomic<int64_t> g_timeout_ns{1000000000LL};
std::atomic<int64_t> g_force_lookback{0};
std::atomic<int64_t> g_force_block{0};
std::atomic<int64_t> g_force_scalar{0};
std::atomic<int64_t> g_check_pointers{1};
std::atomic<int64_t> g_starve{0};
std::atomic<int64_t> g_pdl{1};

// Launch with programmatic stream serialization (when enabled), so the grid
// can be scheduled while the previous kernel on the stream drains; the kernels
// wait for that kernel before touching memory.
template <class Kernel, class... Args>
cudaError_t launch(Kernel kern, uint32_t grid, int block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl.load() != 0 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

constexpr int64_t kMaxStepsPerLaunch = int64_t(1) << 30;
constexpr int64_t kMaxRowSteps = int64_t(1) << 30;
constexpr int64_t kMaxActions = 2048;

// ---------------------------------------------------------------------------
// look-back workspaces, one per (device, stream)
// ---------------------------------------------------------------------------
struct Workspace {
  void *ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_ws_mu;
std::map<std::pair<int, rlscan_stream_t>, Workspace> g_ws;

rlscan_status get_workspace(rlscan_stream_t stream, size_t need, void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RLSCAN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  Workspace &w = g_ws[{dev, stream}];
  if (w.bytes >= need) {
    *out = w.ptr;
    return RLSCAN_OK;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return RLSCAN_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return RLSCAN_ERR_CAPTURE;
  size_t bytes = std::max<size_t>(need, 4096);
  bytes = (bytes + 4095) & ~size_t(4095);
  void *p = nullptr;
  if (w.ptr) {
    // Stream-ordered: earlier launches on this stream finish with the old block first.
    if (cudaFreeAsync(w.ptr, stream) != cudaSuccess) return RLSCAN_ERR_CUDA;
    w.ptr = nullptr;
    w.bytes = 0;
  }
  if (cudaMallocAsync(&p, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    return RLSCAN_ERR_NOMEM;
  }
  if (cudaMemsetAsync(p, 0, bytes, stream) != cudaSuccess) {
    cudaFreeAsync(p, stream);
    return RLSCAN_ERR_CUDA;
  }
  w.ptr = p;
  w.bytes = bytes;
  *out = p;
  return RLSCAN_OK;
}

// ---------------------------------------------------------------------------
// argument checks
// ---------------------------------------------------------------------------
struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

struct Checker {
  rlscan_status st = RLSCAN_OK;
  std::vector<const void *> ptrs;
  std::vector<Range> in, out;

  void fail(rlscan_status s) {
    if (st == RLSCAN_OK) st = s;
  }
  void need(const void *p) {
    if (!p) fail(RLSCAN_ERR_INVALID_ARG);
  }
  void align(const void *p, uintptr_t a) {
    if (p && (reinterpret_cast<uintptr_t>(p) % a) != 0) fail(RLSCAN_ERR_INVALID_ARG);
  }
  void input(const void *p, size_t bytes, uintptr_t a) {
    if (!p) return;
    align(p, a);
    ptrs.push_back(p);
    in.push_back({reinterpret_cast<uintptr_t>(p), reinterpret_cast<uintptr_t>(p) + bytes});
  }
  void output(void *p, size_t bytes, uintptr_t a) {
    if (!p) return;
    align(p, a);
    ptrs.push_back(p);
    out.push_back({reinterpret_cast<uintptr_t>(p), reinterpret_cast<uintptr_t>(p) + bytes});
  }
  void finite(float x) {
    if (!std::isfinite(x)) fail(RLSCAN_ERR_INVALID_ARG);
  }
  void positive(float x) {
    if (!(x > 0.0f) || !std::isfinite(x)) fail(RLSCAN_ERR_INVALID_ARG);
  }
  static bool overlap(const Range &a, const Range &b) { return a.lo < b.hi && b.lo < a.hi; }
  void check_overlaps() {
    for (size_t i = 0; i < out.size(); ++i) {
      for (size_t j = 0; j < in.size(); ++j)
        if (overlap(out[i], in[j])) fail(RLSCAN_ERR_OVERLAP);
      for (size_t j = i + 1; j < out.size(); ++j)
        if (overlap(out[i], out[j])) fail(RLSCAN_ERR_OVERLAP);
    }
  }
  // Every pointer must be readable by the current device.
  void check_device_access(rlscan_stream_t stream) {
    if (st != RLSCAN_OK || g_check_pointers.load() == 0) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
      cudaGetLastError();
      fail(RLSCAN_ERR_CUDA);
      return;
    }
    if (cs != cudaStreamCaptureStatusNone) return;  // checked on the pre-capture call
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      fail(RLSCAN_ERR_CUDA);
      return;
    }
    for (const void *p : ptrs) {
      cudaPointerAttributes at;
      if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        fail(RLSCAN_ERR_INVALID_ARG);
        return;
      }
      bool ok = false;
      switch (at.type) {
        case cudaMemoryTypeDevice: ok = at.device == dev; break;
        case cudaMemoryTypeManaged: ok = true; break;
        case cudaMemoryTypeHost: ok = at.devicePointer == p; break;
        default: ok = false; break;
      }
      if (!ok) {
        fail(RLSCAN_ERR_INVALID_ARG);
        return;
      }
    }
  }
};

bool dims_ok(int64_t N, int64_t T, int64_t A) {
  if (N < 0 || T < 0 || A < 1) return false;
  if (T > 0 && T * A > kMaxRowSteps) return false;
  if (T > 0 && N > (int64_t(1) << 62) / (T * A)) return false;
  return true;
}

bool aligned(const void *p, uintptr_t a) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % a == 0; }

// ---------------------------------------------------------------------------
// launch plans
// ---------------------------------------------------------------------------
struct Plan {
  int block = 256;
  uint32_t L = 2048;        // steps per chunk (look-back plan); rows plan: steps per block
  int64_t rows_per_block = 0;  // rows plan: whole rows per block
  bool lookback = false;
  int64_t rows_per_launch = 0;
  int launches = 0;
  int64_t chunks = 0;       // over all launches
  uint32_t max_chunks = 0;  // in one launch
  size_t ws_bytes = 0;
  // Retrace staging
  uint32_t sub_steps = 0, stages = 0;
  size_t smem = 0;
};

// Thread blocks (chunks) of one launch over `rows` rows.
uint32_t blocks_in_launch(const Plan &pl, int64_t rows, int64_t T) {
  return pl.rows_per_block > 0 ? uint32_t((rows + pl.rows_per_block - 1) / pl.rows_per_block)
                               : uint32_t((rows * T + pl.L - 1) / pl.L);
}

// Threads per block of the scan kernels: multiples of 64 from 128 to 512, so
// that whole rows can fill a block closely.
constexpr int kBlocks[] = {128, 192, 256, 320, 384, 448, 512};
bool valid_block(int64_t b) { return b >= 128 && b <= 512 && b % 64 == 0; }

// Rows plan: the most whole rows of T steps a block of `block` threads, each
// scanning a tile of `tile` steps, can own whatever the alignment of its
// first step (0 if one row does not fit).  k rows span k T steps, whose tiles
// number k T / tile when k T is a multiple of the tile (every block then
// starts aligned) and at most (k T + 2 tile - 2) / tile otherwise.
int64_t rows_per_block(int64_t T, int block, int64_t tile) {
  auto tiles = [T, tile](int64_t k) { return (k * T) % tile == 0 ? k * T / tile : (k * T + 2 * tile - 2) / tile; };
  int64_t k = tile * block / T;
  while (k > 0 && tiles(k) > block) --k;
  return k;
}

using GaeBf16Op = GaeOpT<kTile, __nv_bfloat16>;  // GAE with bf16 I/O

// Steps per thread of each estimator's kernel (Op::K).
int tile_steps(rlscan_estimator est) {
  switch (est) {
    case RLSCAN_EST_GAE: return GaeOp::K;
    case RLSCAN_EST_VTRACE: return VtraceOp::K;
    case RLSCAN_EST_TD_LAMBDA: return TdLambdaOp::K;
    case RLSCAN_EST_DISCOUNTED_RETURN: return DiscountedOp::K;
    case RLSCAN_EST_ELIG_TRACE: return EligOp::K;
    case RLSCAN_EST_EPISODIC_PREFIX_SUM: return PrefixSumOp::K;
    case RLSCAN_EST_AFFINE_SCAN: return AffineOp<false>::K;
    case RLSCAN_EST_AFFINE_SCAN_GRAD: return AffineGradOp<false>::K;
    case RLSCAN_EST_AFFINE_SCAN_BF16: return AffineOp<false, __nv_bfloat16>::K;
    case RLSCAN_EST_GAE_BF16: return GaeBf16Op::K;
    default: return 4;  // Retrace: its own 4-step tiles
  }
}

Plan make_plan(rlscan_estimator est, int64_t N, int64_t T, int64_t A) {
  Plan pl;
  const int64_t fb = g_force_block.load();
  const bool force_lb = g_force_lookback.load() != 0;
  if (est == RLSCAN_EST_RETRACE) {
    // 4-step tiles, 128- or 256-thread blocks.  Rows plan where a row fits
    // (the block the rows fill best, the smaller on a tie); else chunks of
    // 1024 steps with look-back, whose longer chunks halve the chains.
    int64_t best_k = 0;
    int best_b = 128;
    double best_fill = 0.0;
    for (int b : {128, 256}) {
      if ((fb == 128 || fb == 256) && b != fb) continue;
      const int64_t k = rows_per_block(T, b, 4);
      const double fill = double(k * T) / double(4 * b);
      if (k > 0 && fill > best_fill + 1e-9) {
        best_fill = fill;
        best_k = k;
        best_b = b;
      }
    }
    pl.lookback = force_lb || best_k == 0;
    pl.block = (fb == 128 || fb == 256) ? int(fb) : (best_k == 0 ? 256 : best_b);
    if (pl.lookback) {
      pl.L = 4u * uint32_t(pl.block);
    } else {
      pl.rows_per_block = best_k;
      pl.L = uint32_t(best_k * T);
    }
  } else {
    // Rows plan where a row fits a block: the block size whose threads the
    // rows fill best (the smaller one on a tie); else the look-back plan.
    const int K = tile_steps(est);
    int64_t best_k = 0;
    pl.block = 256;
    double best_fill = 0.0;
    for (int b : kBlocks) {
      if (valid_block(fb) && b != fb) continue;
      const int64_t k = rows_per_block(T, b, K);
      const double fill = double(k * T) / double(int64_t(K) * b);
      if (k > 0 && fill > best_fill + 1e-9) {
        best_fill = fill;
        best_k = k;
        pl.block = b;
      }
    }
    if (valid_block(fb)) pl.block = int(fb);
    pl.lookback = force_lb || best_k == 0;
    if (pl.lookback) {
      pl.L = uint32_t(K) * uint32_t(pl.block);
    } else {
      pl.rows_per_block = best_k;
      pl.L = uint32_t(best_k * T);
    }
  }
  pl.rows_per_launch = std::max<int64_t>(1, kMaxStepsPerLaunch / T);
  pl.launches = int((N + pl.rows_per_launch - 1) / pl.rows_per_launch);
  for (int64_t r0 = 0; r0 < N; r0 += pl.rows_per_launch) {
    const uint32_t nch = blocks_in_launch(pl, std::min(pl.rows_per_launch, N - r0), T);
    pl.chunks += nch;
    pl.max_chunks = std::max(pl.max_chunks, nch);
  }
  pl.ws_bytes = sizeof(LookbackHeader) + (pl.lookback ? size_t(pl.max_chunks) * sizeof(LookbackDesc) : 0);
  if (est == RLSCAN_EST_RETRACE) {
    // Sub-tile steps and ring depth: the largest staging within ~56 KB of
    // shared memory per block (four blocks per SM), the size that measured
    // fastest.  The layout is sized for a full chunk of 4 * block steps.
    const uint32_t budget = 56u * 1024u;
    const uint32_t Lmax = 4u * uint32_t(pl.block);
    uint32_t S = uint32_t(pl.block);
    uint32_t NS = 4;
    while (NS > 2 && RetraceOp::smem_bytes(Lmax, S, uint32_t(A), NS) > budget) --NS;
    while (S > 4 && RetraceOp::smem_bytes(Lmax, S, uint32_t(A), NS) > budget) S = std::max(4u, (S / 2) & ~3u);
    pl.sub_steps = S;
    pl.stages = NS;
    pl.smem = RetraceOp::smem_bytes(Lmax, S, uint32_t(A), NS);
  }
  return pl;
}

// (m, l) of FastDiv for divisor d (1 <= d <= 2^30).
void fast_div_params(uint32_t d, uint32_t &m, uint32_t &l) {
  if (d <= 1) {
    m = 0;
    l = 0;
    return;
  }
  l = 0;
  while ((uint64_t(1) << l) < d) ++l;
  m = uint32_t(((uint64_t(1) << (31 + l)) + d - 1) / d);
}

// Blocks of `kern` that fit on the current device at once (occupancy x SMs),
// cached per (device, kernel, dynamic shared size).
int resident_blocks(const void *kern, int block, size_t dyn_smem = 0) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  static std::mutex mu;
  static std::map<std::tuple<int, const void *, size_t>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, kern, dyn_smem);
  const auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, block, dyn_smem) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  const int n = std::max(1, per_sm * sms);
  cache[key] = n;
  return n;
}

// Look-back plan: one block per chunk.  Rows plan: persistent blocks, as
// many as fit at once, each taking every gridDim-th chunk.
template <class Op, int BLOCK, bool LB>
cudaError_t launch_scan(const typename Op::Args &a, ScanGeom g, cudaStream_t s) {
  auto kern = scan_kernel<Op, BLOCK, LB>;
  uint32_t grid = g.nchunks;
  if (!LB) grid = std::min<uint32_t>(grid, uint32_t(resident_blocks(reinterpret_cast<const void *>(kern), BLOCK)));
  const cudaError_t e = launch(kern, grid, BLOCK, 0, s, a, g);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <class Op>
cudaError_t launch_block(const typename Op::Args &a, const ScanGeom &g, int block, bool lb, cudaStream_t s) {
  switch (block) {
#define RLSCAN_BLOCK_CASE(B) \
  case B: return lb ? launch_scan<Op, B, true>(a, g, s) : launch_scan<Op, B, false>(a, g, s);
    RLSCAN_BLOCK_CASE(128)
    RLSCAN_BLOCK_CASE(192)
    RLSCAN_BLOCK_CASE(256)
    RLSCAN_BLOCK_CASE(320)
    RLSCAN_BLOCK_CASE(384)
    RLSCAN_BLOCK_CASE(448)
    RLSCAN_BLOCK_CASE(512)
#undef RLSCAN_BLOCK_CASE
    default: return cudaErrorInvalidValue;
  }
}

template <int BLOCK, bool LB>
cudaError_t launch_retrace(const RetraceOp::Args &a, ScanGeom g, size_t smem, cudaStream_t s) {
  auto kern = retrace_kernel<BLOCK, LB>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = launch(kern, g.nchunks, BLOCK, smem, s, a, g);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_retrace_block(const RetraceOp::Args &a, const ScanGeom &g, int block, bool lb, size_t smem,
                                 cudaStream_t s) {
  switch (block) {
    case 128: return lb ? launch_retrace<128, true>(a, g, smem, s) : launch_retrace<128, false>(a, g, smem, s);
    case 256: return lb ? launch_retrace<256, true>(a, g, smem, s) : launch_retrace<256, false>(a, g, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

// Runs every row slice of a call.  `make_args(row0)` returns the estimator's
// arguments with every pointer advanced to row `row0`; `slice_vec(row0)`
// tells whether that slice's pointers allow vectorised access.
template <class Op, class MakeArgs, class SliceVec>
rlscan_status run(const Plan &pl, int64_t N, int64_t T, rlscan_stream_t stream, MakeArgs make_args,
                  SliceVec slice_vec) {
  void *ws = nullptr;
  rlscan_status st = get_workspace(stream, pl.ws_bytes, &ws);
  if (st != RLSCAN_OK) return st;
  for (int64_t r0 = 0; r0 < N; r0 += pl.rows_per_launch) {
    const int64_t rows = std::min(pl.rows_per_launch, N - r0);
    ScanGeom g{};
    g.total = uint32_t(rows * T);
    g.T = uint32_t(T);
    g.nchunks = blocks_in_launch(pl, rows, T);
    g.span = pl.L;
    g.rows_per_chunk = uint32_t(pl.rows_per_block);
    g.cpr = (pl.lookback && T % int64_t(pl.L) == 0) ? uint32_t(T / int64_t(pl.L)) : 0u;
    const bool vec = g_force_scalar.load() == 0 && slice_vec(r0);
    g.vec = vec ? 1u : 0u;
    fast_div_params(uint32_t(T), g.div_m, g.div_l);
    g.lb.hdr = static_cast<LookbackHeader *>(ws);
    g.lb.desc = reinterpret_cast<LookbackDesc *>(static_cast<LookbackHeader *>(ws) + 1);
    g.lb.timeout_ns = uint64_t(std::max<int64_t>(1000, g_timeout_ns.load()));
    g.lb.starve = g_starve.load() != 0 ? 1u : 0u;
    const typename Op::Args a = make_args(r0);
    cudaError_t e;
    if constexpr (std::is_same<Op, RetraceOp>::value)
      e = launch_retrace_block(a, g, pl.block, pl.lookback, pl.smem, stream);
    else
      e = launch_block<Op>(a, g, pl.block, pl.lookback, stream);
    if (e != cudaSuccess) return RLSCAN_ERR_LAUNCH;
  }
  return RLSCAN_OK;
}

template <class T>
T *adv(T *p, int64_t elems) {
  return p ? p + elems : nullptr;
}

// ---------------------------------------------------------------------------
// time-major [T, N] plans (tm_kernel.cuh)
// ---------------------------------------------------------------------------
constexpr int64_t kMaxTmEnvs = int64_t(1) << 26;  // keeps K N inside 32-bit offsets

// Every time-major kernel scans 8 steps per thread (16 kept too many
// registers live across the look-back).
using TmGaeOp = GaeOpT<8>;
using TmVtraceOp = VtraceOpT<8>;
using TmTdLambdaOp = TdLambdaOpT<8>;
using TmDiscountedOp = DiscountedOpT<8>;
using TmEligOp = EligOpT<8>;
using TmPrefixSumOp = PrefixSumOpT<8>;
template <bool BWD>
using TmAffineOp = AffineOp<BWD, float, 8>;
constexpr int kTmTile = 8;

struct TmPlan {
  uint32_t wt_log2 = 0, nct = 0, nbc = 0, nchunks = 0, dpitch = 0;
  size_t ws_bytes = 0;
};

// Time slices per block: the fewest (a power of two, at most 8) whose K-step
// tiles cover T, so short windows put more environments in a block.  With
// forced look-back, the most slices whose span stays below T (when T > K).
bool make_tm_plan(int K, int64_t N, int64_t T, TmPlan &pl) {
  if (N > kMaxTmEnvs || T > kMaxRowSteps) return false;
  uint32_t wl = 0;
  if (g_force_lookback.load() != 0) {
    while (wl < 3 && (int64_t(K) << (wl + 1)) < T) ++wl;
  } else {
    while (wl < 3 && (int64_t(K) << wl) < T) ++wl;
  }
  const int64_t span = int64_t(K) << wl, cols = int64_t(256) >> wl;
  const int64_t nct = (T + span - 1) / span, nbc = (N + cols - 1) / cols;
  if (nct * nbc >= (int64_t(1) << 31)) return false;
  pl.wt_log2 = wl;
  pl.nct = uint32_t(nct);
  pl.nbc = uint32_t(nbc);
  pl.nchunks = uint32_t(nct * nbc);
  pl.dpitch = uint32_t(nbc * cols);
  pl.ws_bytes = sizeof(LookbackHeader) + (nct > 1 ? size_t(nct) * size_t(pl.dpitch) * sizeof(LookbackDesc) : 0);
  return true;
}

// One launch over the whole [T, N] problem: a block per chunk.
template <class Op>
rlscan_status run_tm(const TmPlan &pl, int64_t N, int64_t T, const typename Op::Args &a, rlscan_stream_t stream) {
  void *ws = nullptr;
  rlscan_status st = get_workspace(stream, pl.ws_bytes, &ws);
  if (st != RLSCAN_OK) return st;
  TmGeom g{};
  g.N = uint32_t(N);
  g.T = uint32_t(T);
  g.wt_log2 = pl.wt_log2;
  g.nct = pl.nct;
  g.nbc = pl.nbc;
  g.nchunks = pl.nchunks;
  g.dpitch = pl.dpitch;
  g.lb.hdr = static_cast<LookbackHeader *>(ws);
  g.lb.desc = reinterpret_cast<LookbackDesc *>(static_cast<LookbackHeader *>(ws) + 1);
  g.lb.timeout_ns = uint64_t(std::max<int64_t>(1000, g_timeout_ns.load()));
  g.lb.starve = g_starve.load() != 0 ? 1u : 0u;
  cudaError_t e = launch(tm_scan_kernel<Op>, pl.nchunks, kTmBlock, 0, stream, a, g);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? RLSCAN_OK : RLSCAN_ERR_LAUNCH;
}

}  // namespace

// ===========================================================================
// extern "C" entry points
// ===========================================================================
extern "C" {

rlscan_status rlscan_gae(const float *rewards, const float *values, const float *bootstrap,
                         const uint8_t *terminated, const uint8_t *truncated,
                         const float *trunc_value, float *advantages, float *returns, int64_t N,
                         int64_t T, float gamma, float lambda, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(values), c.need(bootstrap), c.need(advantages);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda);
  c.input(rewards, nt * 4, 4), c.input(values, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(advantages, nt * 4, 4), c.output(returns, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_GAE, N, T, 1);
  const float *tv = truncated ? trunc_value : nullptr;
  return run<GaeOp>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return GaeOp::Args{adv(rewards, o), adv(values, o), adv(bootstrap, r0), adv(tv, o),
                           adv(terminated, o), adv(truncated, o), adv(advantages, o), adv(returns, o),
                           gamma, gamma * lambda};
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(rewards, o), 32) && aligned(adv(values, o), 32) &&
               aligned(adv(advantages, o), 32) && aligned(adv(returns, o), 32) &&
               aligned(adv(terminated, o), 8) && aligned(adv(truncated, o), 8);
      });
}

rlscan_status rlscan_gae_bf16(const uint16_t *rewards, const uint16_t *values, const uint16_t *bootstrap,
                              const uint8_t *terminated, const uint8_t *truncated, const uint16_t *trunc_value,
                              uint16_t *advantages, uint16_t *returns, int64_t N, int64_t T, float gamma,
                              float lambda, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(values), c.need(bootstrap), c.need(advantages);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda);
  c.input(rewards, nt * 2, 2), c.input(values, nt * 2, 2), c.input(bootstrap, size_t(N) * 2, 2);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 2, 2);
  c.output(advantages, nt * 2, 2), c.output(returns, nt * 2, 2);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  using B16 = __nv_bfloat16;
  using Op = GaeBf16Op;
  const Plan pl = make_plan(RLSCAN_EST_GAE_BF16, N, T, 1);
  auto b16 = [](const uint16_t *p) { return reinterpret_cast<const B16 *>(p); };
  B16 *advb = reinterpret_cast<B16 *>(advantages), *retb = reinterpret_cast<B16 *>(returns);
  const B16 *tv = truncated ? b16(trunc_value) : nullptr;
  return run<Op>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return Op::Args{adv(b16(rewards), o), adv(b16(values), o), adv(b16(bootstrap), r0), adv(tv, o),
                        adv(terminated, o),   adv(truncated, o),   adv(advb, o),             adv(retb, o),
                        gamma,                gamma * lambda};
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(rewards, o), 16) && aligned(adv(values, o), 16) && aligned(adv(advantages, o), 16) &&
               aligned(adv(returns, o), 16) && aligned(adv(terminated, o), 8) && aligned(adv(truncated, o), 8);
      });
}

rlscan_status rlscan_vtrace(const float *log_rhos, const float *rewards, const float *values,
                            const float *bootstrap, const uint8_t *terminated,
                            const uint8_t *truncated, const float *trunc_value, float *vs,
                            float *pg_advantages, int64_t N, int64_t T, float gamma, float lambda,
                            float rho_bar, float c_bar, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(log_rhos), c.need(rewards), c.need(values), c.need(bootstrap), c.need(vs);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda), c.positive(rho_bar), c.positive(c_bar);
  c.input(log_rhos, nt * 4, 4), c.input(rewards, nt * 4, 4), c.input(values, nt * 4, 4);
  c.input(bootstrap, size_t(N) * 4, 4), c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(vs, nt * 4, 4), c.output(pg_advantages, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_VTRACE, N, T, 1);
  const float *tv = truncated ? trunc_value : nullptr;
  return run<VtraceOp>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return VtraceOp::Args{adv(log_rhos, o), adv(rewards, o), adv(values, o), adv(bootstrap, r0),
                              adv(tv, o), adv(terminated, o), adv(truncated, o), adv(vs, o),
                              adv(pg_advantages, o), gamma, lambda, rho_bar, c_bar};
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(log_rhos, o), 32) && aligned(adv(rewards, o), 32) &&
               aligned(adv(values, o), 32) && aligned(adv(vs, o), 32) &&
               aligned(adv(pg_advantages, o), 32) && aligned(adv(terminated, o), 8) &&
               aligned(adv(truncated, o), 8);
      });
}

rlscan_status rlscan_retrace(const float *q, const float *pi, const float *mu_a,
                             const int32_t *actions, const float *rewards, const float *bootstrap,
                             const uint8_t *terminated, const uint8_t *truncated,
                             const float *trunc_value, float *q_ret, int64_t N, int64_t T,
                             int64_t A, float gamma, float lambda, rlscan_stream_t stream) {
  if (A < 1 || A > kMaxActions || !dims_ok(N, T, A)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(q), c.need(pi), c.need(mu_a), c.need(actions), c.need(rewards), c.need(bootstrap);
  c.need(q_ret);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda);
  c.input(q, nt * size_t(A) * 4, 4), c.input(pi, nt * size_t(A) * 4, 4), c.input(mu_a, nt * 4, 4);
  c.input(actions, nt * 4, 4), c.input(rewards, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(q_ret, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_RETRACE, N, T, A);
  const float *tv = truncated ? trunc_value : nullptr;
  return run<RetraceOp>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        const int64_t oa = o * A;
        RetraceOp::Args a{};
        a.q = adv(q, oa), a.pi = adv(pi, oa), a.mu = adv(mu_a, o), a.r = adv(rewards, o);
        a.boot = adv(bootstrap, r0), a.tv = adv(tv, o), a.act = adv(actions, o);
        a.term = adv(terminated, o), a.trunc = adv(truncated, o), a.out = adv(q_ret, o);
        a.A = uint32_t(A), a.sub_steps = pl.sub_steps, a.stages = pl.stages;
        a.tma = (g_force_scalar.load() == 0 && aligned(a.q, 16) && aligned(a.pi, 16)) ? 1u : 0u;
        a.gamma = gamma, a.lambda = lambda;
        return a;
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(rewards, o), 16) && aligned(adv(q_ret, o), 16) &&
               aligned(adv(terminated, o), 4) && aligned(adv(truncated, o), 4);
      });
}

rlscan_status rlscan_td_lambda(const float *rewards, const float *values, const float *bootstrap,
                               const uint8_t *terminated, const uint8_t *truncated,
                               const float *trunc_value, float *returns, int64_t N, int64_t T,
                               float gamma, float lambda, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(values), c.need(bootstrap), c.need(returns);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda);
  c.input(rewards, nt * 4, 4), c.input(values, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(returns, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_TD_LAMBDA, N, T, 1);
  const float *tv = truncated ? trunc_value : nullptr;
  return run<TdLambdaOp>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return TdLambdaOp::Args{adv(rewards, o), adv(values, o), adv(bootstrap, r0), adv(tv, o),
                                adv(terminated, o), adv(truncated, o), adv(returns, o), gamma,
                                gamma * lambda, gamma * (1.0f - lambda)};
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(rewards, o), 32) && aligned(adv(values, o), 32) &&
               aligned(adv(returns, o), 32) && aligned(adv(terminated, o), 8) &&
               aligned(adv(truncated, o), 8);
      });
}

rlscan_status rlscan_discounted_return(const float *rewards, const float *bootstrap,
                                       const uint8_t *terminated, const uint8_t *truncated,
                                       const float *trunc_value, float *returns, int64_t N,
                                       int64_t T, float gamma, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(returns);
  if (truncated) c.need(trunc_value);
  c.finite(gamma);
  c.input(rewards, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(returns, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_DISCOUNTED_RETURN, N, T, 1);
  const float *tv = truncated ? trunc_value : nullptr;
  return run<DiscountedOp>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return DiscountedOp::Args{adv(rewards, o), adv(bootstrap, r0), adv(tv, o), adv(terminated, o),
                                  adv(truncated, o), adv(returns, o), gamma};
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(rewards, o), 32) && aligned(adv(returns, o), 32) &&
               aligned(adv(terminated, o), 8) && aligned(adv(truncated, o), 8);
      });
}

rlscan_status rlscan_elig_trace(const float *inputs, const float *init_trace,
                                const uint8_t *terminated, const uint8_t *truncated,
                                float *traces, int64_t N, int64_t T, float gamma, float lambda,
                                rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(inputs), c.need(traces);
  c.finite(gamma), c.finite(lambda);
  c.input(inputs, nt * 4, 4), c.input(init_trace, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  c.output(traces, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_ELIG_TRACE, N, T, 1);
  return run<EligOp>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return EligOp::Args{adv(inputs, o), adv(init_trace, r0), adv(terminated, o), adv(truncated, o),
                            adv(traces, o), gamma * lambda};
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(inputs, o), 32) && aligned(adv(traces, o), 32) &&
               aligned(adv(terminated, o), 8) && aligned(adv(truncated, o), 8);
      });
}

rlscan_status rlscan_episodic_prefix_sum(const int32_t *x, const uint8_t *terminated,
                                         const uint8_t *truncated, int32_t *out, int64_t N,
                                         int64_t T, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(x), c.need(out);
  c.input(x, nt * 4, 4), c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  c.output(out, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_EPISODIC_PREFIX_SUM, N, T, 1);
  return run<PrefixSumOp>(
      pl, N, T, stream,
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return PrefixSumOp::Args{adv(x, o), adv(terminated, o), adv(truncated, o), adv(out, o)};
      },
      [&](int64_t r0) {
        const int64_t o = r0 * T;
        return aligned(adv(x, o), 32) && aligned(adv(out, o), 32) && aligned(adv(terminated, o), 8) &&
               aligned(adv(truncated, o), 8);
      });
}

rlscan_status rlscan_affine_scan(const float *a, const float *b, const uint8_t *reset, const float *init,
                                 float *x, int64_t N, int64_t T, int32_t reverse, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1) || (reverse != 0 && reverse != 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(a), c.need(b), c.need(x);
  c.input(a, nt * 4, 4), c.input(b, nt * 4, 4), c.input(reset, nt, 1), c.input(init, size_t(N) * 4, 4);
  c.output(x, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_AFFINE_SCAN, N, T, 1);
  auto vec = [&](int64_t r0) {
    const int64_t o = r0 * T;
    return aligned(adv(a, o), 32) && aligned(adv(b, o), 32) && aligned(adv(x, o), 32) && aligned(adv(reset, o), 8);
  };
  auto go = [&](auto op) {
    using Op = decltype(op);
    return run<Op>(
        pl, N, T, stream,
        [&](int64_t r0) {
          const int64_t o = r0 * T;
          return typename Op::Args{adv(a, o), adv(b, o), adv(init, r0), adv(reset, o), nullptr, adv(x, o)};
        },
        vec);
  };
  return reverse ? go(AffineOp<true>{}) : go(AffineOp<false>{});
}

rlscan_status rlscan_affine_scan_bf16(const uint16_t *a, const uint16_t *b, const uint8_t *reset,
                                      const uint16_t *init, uint16_t *x, int64_t N, int64_t T, int32_t reverse,
                                      rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1) || (reverse != 0 && reverse != 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(a), c.need(b), c.need(x);
  c.input(a, nt * 2, 2), c.input(b, nt * 2, 2), c.input(reset, nt, 1), c.input(init, size_t(N) * 2, 2);
  c.output(x, nt * 2, 2);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_AFFINE_SCAN_BF16, N, T, 1);
  using B16 = __nv_bfloat16;
  const B16 *ab = reinterpret_cast<const B16 *>(a), *bb = reinterpret_cast<const B16 *>(b);
  const B16 *ib = reinterpret_cast<const B16 *>(init);
  B16 *xb = reinterpret_cast<B16 *>(x);
  auto vec = [&](int64_t r0) {
    const int64_t o = r0 * T;
    return aligned(adv(ab, o), 16) && aligned(adv(bb, o), 16) && aligned(adv(xb, o), 16) && aligned(adv(reset, o), 8);
  };
  auto go = [&](auto op) {
    using Op = decltype(op);
    return run<Op>(
        pl, N, T, stream,
        [&](int64_t r0) {
          const int64_t o = r0 * T;
          return typename Op::Args{adv(ab, o), adv(bb, o), adv(ib, r0), adv(reset, o), nullptr, adv(xb, o)};
        },
        vec);
  };
  return reverse ? go(AffineOp<true, B16>{}) : go(AffineOp<false, B16>{});
}

rlscan_status rlscan_affine_scan_grad(const float *a, const float *x, const float *dy, const uint8_t *reset,
                                      const float *init, float *da, float *db, float *dinit, int64_t N,
                                      int64_t T, int32_t reverse, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1) || (reverse != 0 && reverse != 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(a), c.need(x), c.need(dy), c.need(db);
  c.input(a, nt * 4, 4), c.input(x, nt * 4, 4), c.input(dy, nt * 4, 4), c.input(reset, nt, 1);
  c.input(init, size_t(N) * 4, 4);
  c.output(db, nt * 4, 4), c.output(da, nt * 4, 4), c.output(dinit, size_t(N) * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const Plan pl = make_plan(RLSCAN_EST_AFFINE_SCAN_GRAD, N, T, 1);
  auto vec = [&](int64_t r0) {
    const int64_t o = r0 * T;
    return aligned(adv(a, o), 32) && aligned(adv(x, o), 32) && aligned(adv(dy, o), 32) &&
           aligned(adv(db, o), 32) && aligned(adv(da, o), 32) && aligned(adv(reset, o), 8);
  };
  auto go = [&](auto op) {
    using Op = decltype(op);
    return run<Op>(
        pl, N, T, stream,
        [&](int64_t r0) {
          const int64_t o = r0 * T;
          return typename Op::Args{adv(a, o),     adv(x, o),  adv(dy, o),    adv(init, r0), adv(reset, o),
                                   nullptr,        adv(da, o), adv(db, o),    adv(dinit, r0), uint32_t(T)};
        },
        vec);
  };
  return reverse ? go(AffineGradOp<true>{}) : go(AffineGradOp<false>{});
}

// ---------------------------------------------------------------------------
// time-major entry points: every per-step array is [T, N] (element (t, n) at
// t * N + n); per-environment arrays stay [N].  Same checks and results as
// the row-major calls.
// ---------------------------------------------------------------------------
rlscan_status rlscan_gae_tm(const float *rewards, const float *values, const float *bootstrap,
                            const uint8_t *terminated, const uint8_t *truncated, const float *trunc_value,
                            float *advantages, float *returns, int64_t N, int64_t T, float gamma, float lambda,
                            rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(values), c.need(bootstrap), c.need(advantages);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda);
  c.input(rewards, nt * 4, 4), c.input(values, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(advantages, nt * 4, 4), c.output(returns, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const TmGaeOp::Args a{rewards, values, bootstrap, truncated ? trunc_value : nullptr, terminated, truncated,
                      advantages, returns, gamma, gamma * lambda};
  return run_tm<TmGaeOp>(pl, N, T, a, stream);
}

rlscan_status rlscan_vtrace_tm(const float *log_rhos, const float *rewards, const float *values,
                               const float *bootstrap, const uint8_t *terminated, const uint8_t *truncated,
                               const float *trunc_value, float *vs, float *pg_advantages, int64_t N, int64_t T,
                               float gamma, float lambda, float rho_bar, float c_bar, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(log_rhos), c.need(rewards), c.need(values), c.need(bootstrap), c.need(vs);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda), c.positive(rho_bar), c.positive(c_bar);
  c.input(log_rhos, nt * 4, 4), c.input(rewards, nt * 4, 4), c.input(values, nt * 4, 4);
  c.input(bootstrap, size_t(N) * 4, 4), c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(vs, nt * 4, 4), c.output(pg_advantages, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const TmVtraceOp::Args a{log_rhos, rewards, values, bootstrap, truncated ? trunc_value : nullptr, terminated,
                         truncated, vs, pg_advantages, gamma, lambda, rho_bar, c_bar};
  return run_tm<TmVtraceOp>(pl, N, T, a, stream);
}

rlscan_status rlscan_td_lambda_tm(const float *rewards, const float *values, const float *bootstrap,
                                  const uint8_t *terminated, const uint8_t *truncated, const float *trunc_value,
                                  float *returns, int64_t N, int64_t T, float gamma, float lambda,
                                  rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(values), c.need(bootstrap), c.need(returns);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda);
  c.input(rewards, nt * 4, 4), c.input(values, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(returns, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const TmTdLambdaOp::Args a{rewards,  values,  bootstrap, truncated ? trunc_value : nullptr,
                           terminated, truncated, returns, gamma, gamma * lambda, gamma * (1.0f - lambda)};
  return run_tm<TmTdLambdaOp>(pl, N, T, a, stream);
}

rlscan_status rlscan_discounted_return_tm(const float *rewards, const float *bootstrap, const uint8_t *terminated,
                                          const uint8_t *truncated, const float *trunc_value, float *returns,
                                          int64_t N, int64_t T, float gamma, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(returns);
  if (truncated) c.need(trunc_value);
  c.finite(gamma);
  c.input(rewards, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(returns, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const TmDiscountedOp::Args a{rewards, bootstrap, truncated ? trunc_value : nullptr, terminated, truncated, returns,
                             gamma};
  return run_tm<TmDiscountedOp>(pl, N, T, a, stream);
}

rlscan_status rlscan_elig_trace_tm(const float *inputs, const float *init_trace, const uint8_t *terminated,
                                   const uint8_t *truncated, float *traces, int64_t N, int64_t T, float gamma,
                                   float lambda, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(inputs), c.need(traces);
  c.finite(gamma), c.finite(lambda);
  c.input(inputs, nt * 4, 4), c.input(init_trace, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  c.output(traces, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const TmEligOp::Args a{inputs, init_trace, terminated, truncated, traces, gamma * lambda};
  return run_tm<TmEligOp>(pl, N, T, a, stream);
}

rlscan_status rlscan_episodic_prefix_sum_tm(const int32_t *x, const uint8_t *terminated, const uint8_t *truncated,
                                            int32_t *out, int64_t N, int64_t T, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(x), c.need(out);
  c.input(x, nt * 4, 4), c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  c.output(out, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  const TmPrefixSumOp::Args a{x, terminated, truncated, out};
  return run_tm<TmPrefixSumOp>(pl, N, T, a, stream);
}

rlscan_status rlscan_affine_scan_tm(const float *a, const float *b, const uint8_t *reset, const float *init,
                                    float *x, int64_t N, int64_t T, int32_t reverse, rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1) || (reverse != 0 && reverse != 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(a), c.need(b), c.need(x);
  c.input(a, nt * 4, 4), c.input(b, nt * 4, 4), c.input(reset, nt, 1), c.input(init, size_t(N) * 4, 4);
  c.output(x, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;
  if (reverse) return run_tm<TmAffineOp<true>>(pl, N, T, TmAffineOp<true>::Args{a, b, init, reset, nullptr, x}, stream);
  return run_tm<TmAffineOp<false>>(pl, N, T, TmAffineOp<false>::Args{a, b, init, reset, nullptr, x}, stream);
}

rlscan_status rlscan_query_plan_tm(rlscan_estimator est, int64_t N, int64_t T, rlscan_plan_info *info) {
  if (!info || !dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  switch (est) {
    case RLSCAN_EST_GAE: case RLSCAN_EST_VTRACE: case RLSCAN_EST_TD_LAMBDA: case RLSCAN_EST_DISCOUNTED_RETURN:
    case RLSCAN_EST_ELIG_TRACE: case RLSCAN_EST_EPISODIC_PREFIX_SUM: case RLSCAN_EST_AFFINE_SCAN: break;
    default: return RLSCAN_ERR_INVALID_ARG;
  }
  std::memset(info, 0, sizeof(*info));
  if (N == 0 || T == 0) return RLSCAN_OK;
  TmPlan pl;
  if (!make_tm_plan(kTmTile, N, T, pl)) return RLSCAN_ERR_INVALID_ARG;
  info->block_threads = kTmBlock;
  info->chunk_steps = int32_t((int64_t(kTmTile) << pl.wt_log2) * (int64_t(256) >> pl.wt_log2));
  info->lookback = pl.nct > 1 ? 1 : 0;
  info->launches = 1;
  info->chunks = pl.nchunks;
  info->workspace_bytes = int64_t(pl.ws_bytes);
  return RLSCAN_OK;
}

rlscan_status rlscan_sync_status(rlscan_stream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return RLSCAN_ERR_CUDA;
  }
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_rlscan_device_status, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return RLSCAN_ERR_CUDA;
  }
  if (v != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_rlscan_device_status, &zero, sizeof(zero)) != cudaSuccess) {
      cudaGetLastError();
      return RLSCAN_ERR_CUDA;
    }
  }
  switch (v) {
    case kDevStatusOk: return RLSCAN_OK;
    case kDevStatusInvalidArg: return RLSCAN_ERR_INVALID_ARG;
    case kDevStatusTimeout: return RLSCAN_ERR_TIMEOUT;
    default: return RLSCAN_ERR_CUDA;
  }
}

const char *rlscan_status_string(rlscan_status s) {
  switch (s) {
    case RLSCAN_OK: return "RLSCAN_OK";
    case RLSCAN_ERR_INVALID_ARG: return "RLSCAN_ERR_INVALID_ARG";
    case RLSCAN_ERR_OVERLAP: return "RLSCAN_ERR_OVERLAP";
    case RLSCAN_ERR_LAUNCH: return "RLSCAN_ERR_LAUNCH";
    case RLSCAN_ERR_TIMEOUT: return "RLSCAN_ERR_TIMEOUT";
    case RLSCAN_ERR_NOMEM: return "RLSCAN_ERR_NOMEM";
    case RLSCAN_ERR_CUDA: return "RLSCAN_ERR_CUDA";
    case RLSCAN_ERR_CAPTURE: return "RLSCAN_ERR_CAPTURE";
    case RLSCAN_ERR_TOO_LARGE: return "RLSCAN_ERR_TOO_LARGE";
  }
  return "RLSCAN_ERR_UNKNOWN";
}

void rlscan_release_workspaces(void) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  int cur = 0;
  const bool have_dev = cudaGetDevice(&cur) == cudaSuccess;
  for (auto &kv : g_ws) {
    if (kv.second.ptr) {
      cudaSetDevice(kv.first.first);
      cudaFree(kv.second.ptr);
    }
  }
  g_ws.clear();
  if (have_dev) cudaSetDevice(cur);
  cudaGetLastError();
}

rlscan_status rlscan_reserve_workspace(int64_t bytes, rlscan_stream_t stream) {
  if (bytes < 0) return RLSCAN_ERR_INVALID_ARG;
  void *ws = nullptr;
  return get_workspace(stream, std::max<size_t>(size_t(bytes), sizeof(LookbackHeader)), &ws);
}

int rlscan_abi_version(void) { return RLSCAN_ABI_VERSION; }

rlscan_status rlscan_query_plan(rlscan_estimator est, int64_t N, int64_t T, int64_t A,
                                rlscan_plan_info *info) {
  if (!info || int(est) < 0 || int(est) > int(RLSCAN_EST_GAE_BF16)) return RLSCAN_ERR_INVALID_ARG;
  if (est != RLSCAN_EST_RETRACE) A = 1;
  if (A < 1 || A > kMaxActions || !dims_ok(N, T, A)) return RLSCAN_ERR_INVALID_ARG;
  std::memset(info, 0, sizeof(*info));
  if (N == 0 || T == 0) return RLSCAN_OK;
  const Plan pl = make_plan(est, N, T, A);
  info->block_threads = pl.block;
  info->chunk_steps = int32_t(pl.L);
  info->lookback = pl.lookback ? 1 : 0;
  info->launches = pl.launches;
  info->chunks = pl.chunks;
  info->workspace_bytes = int64_t(pl.ws_bytes);
  return RLSCAN_OK;
}

rlscan_status rlscan_set_option(rlscan_option opt, int64_t v) {
  switch (opt) {
    case RLSCAN_OPT_LOOKBACK_TIMEOUT_NS:
      if (v < 1000) return RLSCAN_ERR_INVALID_ARG;
      g_timeout_ns = v;
      return RLSCAN_OK;
    case RLSCAN_OPT_FORCE_LOOKBACK: g_force_lookback = v ? 1 : 0; return RLSCAN_OK;
    case RLSCAN_OPT_FORCE_BLOCK:
      if (v != 0 && !valid_block(v)) return RLSCAN_ERR_INVALID_ARG;
      g_force_block = v;
      return RLSCAN_OK;
    case RLSCAN_OPT_FORCE_SCALAR: g_force_scalar = v ? 1 : 0; return RLSCAN_OK;
    case RLSCAN_OPT_CHECK_POINTERS: g_check_pointers = v ? 1 : 0; return RLSCAN_OK;
    case RLSCAN_OPT_TEST_STARVE_LOOKBACK: g_starve = v ? 1 : 0; return RLSCAN_OK;
    case RLSCAN_OPT_PDL: g_pdl = v ? 1 : 0; return RLSCAN_OK;
  }
  return RLSCAN_ERR_INVALID_ARG;
}

int64_t rlscan_get_option(rlscan_option opt) {
  switch (opt) {
    case RLSCAN_OPT_LOOKBACK_TIMEOUT_NS: return g_timeout_ns.load();
    case RLSCAN_OPT_FORCE_LOOKBACK: return g_force_lookback.load();
    case RLSCAN_OPT_FORCE_BLOCK: return g_force_block.load();
    case RLSCAN_OPT_FORCE_SCALAR: return g_force_scalar.load();
    case RLSCAN_OPT_CHECK_POINTERS: return g_check_pointers.load();
    case RLSCAN_OPT_TEST_STARVE_LOOKBACK: return g_starve.load();
    case RLSCAN_OPT_PDL: return g_pdl.load();
  }
  return -1;
}

}  // extern "C"

// ===========================================================================
// rlscan_gae_noalloc: GAE whose look-back scratch is a fixed device array
// ===========================================================================
// For callers that must not allocate device memory (graph capture, foreign
// allocators, latency-critical loops): the carry hand-off between thread
// blocks uses this file-scope array instead of a per-stream workspace.  Host
// code cannot use the array's name as a device address; its address is
// resolved once per device with cudaGetSymbolAddress.
namespace {

constexpr int64_t kNoAllocMaxSteps = int64_t(1) << 27;
// Header plus one descriptor per chunk of the smallest chunk size (1024 steps).
constexpr size_t kNoAllocScratchBytes =
    sizeof(LookbackHeader) + sizeof(LookbackDesc) * size_t(kNoAllocMaxSteps / 1024);
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device, with that device current).
rlscan_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    cudaGetLastError();
    return RLSCAN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return RLSCAN_ERR_CUDA;
    }
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return RLSCAN_OK;
}

}  // namespace

extern "C" rlscan_status rlscan_gae_noalloc(const float *rewards, const float *values, const float *bootstrap,
                                            const uint8_t *terminated, const uint8_t *truncated,
                                            const float *trunc_value, float *advantages, float *returns,
                                            int64_t N, int64_t T, float gamma, float lambda,
                                            rlscan_stream_t stream) {
  if (!dims_ok(N, T, 1)) return RLSCAN_ERR_INVALID_ARG;
  if (N == 0 || T == 0) return RLSCAN_OK;
  if (N * T > kNoAllocMaxSteps) return RLSCAN_ERR_TOO_LARGE;
  const size_t nt = size_t(N) * size_t(T);
  Checker c;
  c.need(rewards), c.need(values), c.need(bootstrap), c.need(advantages);
  if (truncated) c.need(trunc_value);
  c.finite(gamma), c.finite(lambda);
  c.input(rewards, nt * 4, 4), c.input(values, nt * 4, 4), c.input(bootstrap, size_t(N) * 4, 4);
  c.input(terminated, nt, 1), c.input(truncated, nt, 1);
  if (truncated) c.input(trunc_value, nt * 4, 4);
  c.output(advantages, nt * 4, 4), c.output(returns, nt * 4, 4);
  c.check_overlaps();
  c.check_device_access(stream);
  if (c.st != RLSCAN_OK) return c.st;

  const Plan pl = make_plan(RLSCAN_EST_GAE, N, T, 1);  // N * T <= 2^27: a single launch
  ScanGeom g{};
  g.total = uint32_t(nt);
  g.T = uint32_t(T);
  g.nchunks = blocks_in_launch(pl, N, T);
  g.span = pl.L;
  g.rows_per_chunk = uint32_t(pl.rows_per_block);
  g.cpr = (pl.lookback && T % int64_t(pl.L) == 0) ? uint32_t(T / int64_t(pl.L)) : 0u;
  g.vec = (g_force_scalar.load() == 0 && aligned(rewards, 32) && aligned(values, 32) && aligned(advantages, 32) &&
           aligned(returns, 32) && aligned(terminated, 8) && aligned(truncated, 8))
              ? 1u
              : 0u;
  fast_div_params(uint32_t(T), g.div_m, g.div_l);
  g.lb.timeout_ns = uint64_t(std::max<int64_t>(1000, g_timeout_ns.load()));
  g.lb.starve = 0u;
  if (pl.lookback) {
    void *scratch = nullptr;
    const rlscan_status st = noalloc_scratch(&scratch);
    if (st != RLSCAN_OK) return st;
    // Start from a clean header and clean descriptors for this call's chunks.
    const size_t used = sizeof(LookbackHeader) + size_t(g.nchunks) * sizeof(LookbackDesc);
    if (cudaMemsetAsync(scratch, 0, used, stream) != cudaSuccess) {
      cudaGetLastError();
      return RLSCAN_ERR_CUDA;
    }
    g.lb.hdr = static_cast<LookbackHeader *>(scratch);
    g.lb.desc = reinterpret_cast<LookbackDesc *>(static_cast<LookbackHeader *>(scratch) + 1);
  }
  const float *tv = truncated ? trunc_value : nullptr;
  const GaeOp::Args a{rewards, values, bootstrap, tv, terminated, truncated, advantages, returns, gamma,
                      gamma * lambda};
  const cudaError_t e = launch_block<GaeOp>(a, g, pl.block, pl.lookback, stream);
  return e == cudaSuccess ? RLSCAN_OK : RLSCAN_ERR_LAUNCH;
}
