// tm_kernel.cuh -- the fused scan over time-major [T, N] arrays.
//
// The same method as scan_kernel.cuh ("rl-triton: High-Performance Triton GPU
// Kernels for Reinforcement Learning Credit Assignment", gist.science
// technical summary, Methodologie 1-2: coefficients built on chip, one
// associative scan, one HBM read and write per element) for rollout buffers
// stored time-major, the memory-layout option of the same project's API page
// (Hugging Face model card, "Key Features": contiguous vs strided layout):
// element (t, n) at t * N + n, each time step one contiguous run of the N
// environments.
//
// Work decomposition (ours).  The 32 lanes of a warp own 32 neighbouring
// environments, so every warp access is one contiguous run of 32 elements; a
// thread owns K (= Op::K) consecutive steps of its environment, K scalar
// accesses N elements apart.  The 8 warps of a block are WT time slices times
// 8 / WT column groups (WT = 1, 2, 4 or 8, the smallest that covers T, at
// most 8), so a block's chunk is WT K steps of 256 / WT environments.  Inside
// the chunk the slices' aggregates combine through shared memory; along T,
// chunks hand carries on with a decoupled look-back per environment: the
// chunk's composite is published per environment, and all warps of the block
// fetch the descriptors of the chunks before it at once, a window of several
// chunks per memory round trip.  Chunks take tickets in dependency order, the
// column blocks of one time chunk after another, so a block only ever waits
// on blocks that drew earlier tickets.
//
// Each estimator's coefficients are exactly the row-major kernel's
// (estimators.cuh, Op::coef); only its loads and stores are restated here
// (TmIO<Op>), for a column of steps instead of a contiguous tile.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "estimators.cuh"
#include "scan_core.cuh"

namespace rlscan {

constexpr int kTmBlock = 256;  // threads per block: 8 warps

struct TmGeom {
  uint32_t N;        // environments: the row pitch of every [T, N] array
  uint32_t T;        // steps
  uint32_t wt_log2;  // time slices per block: 1 << wt_log2
  uint32_t nct;      // chunks along T, each (1 << wt_log2) K steps
  uint32_t nbc;      // column blocks, each 256 >> wt_log2 environments
  uint32_t nchunks;  // nct * nbc
  uint32_t dpitch;   // descriptors per chunk row: nbc * (256 >> wt_log2)
  LookbackCtl lb;    // look-back only (nct > 1)
};

// K steps of one environment: t0 .. t0 + K - 1.
struct ColTile {
  uint64_t off;    // element offset of the first step: t0 * N + n
  uint32_t N;      // elements between consecutive steps
  uint32_t n, t0;  // environment, first step
  uint32_t valid;  // bit k: step t0 + k exists (t < T) in an existing environment
  uint32_t edge;   // bit k: step t0 + k is the dependency edge (backward T - 1, forward 0)
  bool next;       // step t0 + K exists (halo of backward estimators)
  bool prev;       // step t0 - 1 exists (halo of forward estimators)
};

// ---------------------------------------------------------------------------
// column loads / stores: one scalar access per step, 32 lanes contiguous
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ld_na(const float *p) {
  float v;
  asm("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_na(const int32_t *p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_na(const uint8_t *p) {
  uint16_t v;
  asm("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// Full tiles (every step valid, the common case) take the unpredicated path.
template <int K>
__device__ __forceinline__ bool col_full(const ColTile &c) {
  return c.valid == (K == 32 ? 0xffffffffu : (1u << K) - 1u);
}
template <int K>
__device__ __forceinline__ void ld_col(const float *p, const ColTile &c, float (&v)[K]) {
  const float *q = p + c.off;
  if (col_full<K>(c)) {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = ld_na(q + uint32_t(k) * c.N);
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = ((c.valid >> k) & 1u) ? ld_na(q + uint32_t(k) * c.N) : 0.0f;
  }
}
template <int K>
__device__ __forceinline__ void ld_col(const int32_t *p, const ColTile &c, uint32_t (&v)[K]) {
  const int32_t *q = p + c.off;
  if (col_full<K>(c)) {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = ld_na(q + uint32_t(k) * c.N);
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = ((c.valid >> k) & 1u) ? ld_na(q + uint32_t(k) * c.N) : 0u;
  }
}
template <int K>
__device__ __forceinline__ uint32_t ld_col_flags(const uint8_t *p, const ColTile &c) {
  if (p == nullptr) return 0u;
  const uint8_t *q = p + c.off;
  uint32_t m = 0;
  if (col_full<K>(c)) {
#pragma unroll
    for (int k = 0; k < K; ++k) m |= (ld_na(q + uint32_t(k) * c.N) != 0u ? 1u : 0u) << k;
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if (((c.valid >> k) & 1u) && ld_na(q + uint32_t(k) * c.N) != 0u) m |= 1u << k;
  }
  return m;
}
template <int K>
__device__ __forceinline__ void st_col(float *p, const ColTile &c, const float (&v)[K]) {
  float *q = p + c.off;
  if (col_full<K>(c)) {
#pragma unroll
    for (int k = 0; k < K; ++k) __stcs(q + uint32_t(k) * c.N, v[k]);
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((c.valid >> k) & 1u) __stcs(q + uint32_t(k) * c.N, v[k]);
  }
}
template <int K>
__device__ __forceinline__ void st_col(int32_t *p, const ColTile &c, const uint32_t (&v)[K]) {
  int32_t *q = p + c.off;
  if (col_full<K>(c)) {
#pragma unroll
    for (int k = 0; k < K; ++k) __stcs(q + uint32_t(k) * c.N, int(v[k]));
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((c.valid >> k) & 1u) __stcs(q + uint32_t(k) * c.N, int(v[k]));
  }
}

// Done flag (terminated or truncated) of the step before the tile.
__device__ __forceinline__ uint32_t col_prev_done(const uint8_t *term, const uint8_t *trunc, const ColTile &c) {
  if (!c.prev) return 0u;
  const uint64_t i = c.off - c.N;
  return ((term && ld_na(term + i) != 0u) || (trunc && ld_na(trunc + i) != 0u)) ? 1u : 0u;
}

// Successor values of the tile's boundary steps (backward estimators), 0
// elsewhere: 0 after termination, trunc_value after truncation, the
// environment's bootstrap at the window end (`boot` NULL: 0); termination
// wins over truncation, and both over the window end.
template <int K>
__device__ __forceinline__ void col_successors(const float *tv, const float *boot, const ColTile &c, Flags f,
                                               float (&bv)[K]) {
  const uint32_t tr = f.trunc & ~f.term & c.valid;
  const uint32_t ed = c.edge & ~f.term & ~f.trunc;
#pragma unroll
  for (int k = 0; k < K; ++k) bv[k] = 0.0f;
  if (__any_sync(0xffffffffu, tr != 0u)) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((tr >> k) & 1u) bv[k] = ld_na(tv + c.off + uint32_t(k) * c.N);
  }
  if (ed != 0u) {
    const float b = boot ? ld_na(boot + c.n) : 0.0f;
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((ed >> k) & 1u) bv[k] = b;
  }
}

// ---------------------------------------------------------------------------
// Per-estimator loads and stores of a column tile.  Each fills the Raw state
// its Op::coef reads (the same fields the row-major loads fill) and writes the
// same outputs as its Op::emit.
//   load(args, tile, flags, raw)   every load whose address follows from the
//                                  tile position, halo step included
//   fetch_boundary(args, tile, raw) the loads that depend on the flags
//   nbr(raw)                       the neighbour value Op::coef takes
//   emit(args, tile, raw, c, x, xdep)
// ---------------------------------------------------------------------------
template <class Op>
struct TmIO;

template <int K>
struct TmIO<GaeOpT<K>> {
  using Op = GaeOpT<K>;
  static constexpr int kRegs = 64;  // registers per thread, chosen by measurement
  static __device__ __forceinline__ void load(const typename Op::Args &p, const ColTile &c, Flags f,
                                              typename Op::Raw &w) {
    ld_col(p.r, c, w.r);
    ld_col(p.v, c, w.v);
    w.f = f;
    w.halo = c.next ? ld_na(p.v + c.off + uint32_t(K) * c.N) : 0.0f;
    w.ev = 0.0f;
  }
  static __device__ __forceinline__ void fetch_boundary(const typename Op::Args &p, const ColTile &c,
                                                        typename Op::Raw &w) {
    col_successors(p.tv, p.boot, c, w.f, w.bv);
  }
  static __device__ __forceinline__ float nbr(const typename Op::Raw &w) { return w.halo; }
  static __device__ __forceinline__ void emit(const typename Op::Args &p, const ColTile &c, const typename Op::Raw &w,
                                              const Aff<float> (&)[K], const float (&x)[K], const float (&)[K]) {
    st_col(p.adv, c, x);
    if (p.ret) {
      float ret[K];
#pragma unroll
      for (int k = 0; k < K; ++k) ret[k] = x[k] + w.v[k];
      st_col(p.ret, c, ret);
    }
  }
};

template <int K>
struct TmIO<TdLambdaOpT<K>> {
  using Op = TdLambdaOpT<K>;
  static constexpr int kRegs = 64;  // registers per thread, chosen by measurement
  static __device__ __forceinline__ void load(const typename Op::Args &p, const ColTile &c, Flags f,
                                              typename Op::Raw &w) {
    ld_col(p.r, c, w.r);
    ld_col(p.v, c, w.v);
    w.f = f;
    w.halo = c.next ? ld_na(p.v + c.off + uint32_t(K) * c.N) : 0.0f;
    w.ev = 0.0f;
  }
  static __device__ __forceinline__ void fetch_boundary(const typename Op::Args &p, const ColTile &c,
                                                        typename Op::Raw &w) {
    col_successors(p.tv, p.boot, c, w.f, w.bv);
  }
  static __device__ __forceinline__ float nbr(const typename Op::Raw &w) { return w.halo; }
  static __device__ __forceinline__ void emit(const typename Op::Args &p, const ColTile &c, const typename Op::Raw &,
                                              const Aff<float> (&)[K], const float (&x)[K], const float (&)[K]) {
    st_col(p.out, c, x);
  }
};

template <int K>
struct TmIO<DiscountedOpT<K>> {
  using Op = DiscountedOpT<K>;
  static constexpr int kRegs = 48;  // registers per thread, chosen by measurement
  static __device__ __forceinline__ void load(const typename Op::Args &p, const ColTile &c, Flags f,
                                              typename Op::Raw &w) {
    ld_col(p.r, c, w.r);
    w.f = f;
    w.ev = 0.0f;
  }
  static __device__ __forceinline__ void fetch_boundary(const typename Op::Args &p, const ColTile &c,
                                                        typename Op::Raw &w) {
    col_successors(p.tv, p.boot, c, w.f, w.bv);
  }
  static __device__ __forceinline__ float nbr(const typename Op::Raw &) { return 0.0f; }
  static __device__ __forceinline__ void emit(const typename Op::Args &p, const ColTile &c, const typename Op::Raw &,
                                              const Aff<float> (&)[K], const float (&x)[K], const float (&)[K]) {
    st_col(p.out, c, x);
  }
};

template <int K>
struct TmIO<VtraceOpT<K>> {
  using Op = VtraceOpT<K>;
  static constexpr int kRegs = 64;  // registers per thread, chosen by measurement
  static __device__ __forceinline__ void load(const typename Op::Args &p, const ColTile &c, Flags f,
                                              typename Op::Raw &w) {
    ld_col(p.lr, c, w.lr);
    ld_col(p.r, c, w.r);
    ld_col(p.v, c, w.v);
    w.f = f;
    w.halo = c.next ? ld_na(p.v + c.off + uint32_t(K) * c.N) : 0.0f;
    w.ev = 0.0f;
  }
  static __device__ __forceinline__ void fetch_boundary(const typename Op::Args &p, const ColTile &c,
                                                        typename Op::Raw &w) {
    col_successors(p.tv, p.boot, c, w.f, w.bv);
  }
  static __device__ __forceinline__ float nbr(const typename Op::Raw &w) { return w.halo; }
  // Op::coef leaves gamma rho cont in w.lr: pg = b + gamma rho cont x_{t+1}.
  static __device__ __forceinline__ void emit(const typename Op::Args &p, const ColTile &c, const typename Op::Raw &w,
                                              const Aff<float> (&cf)[K], const float (&x)[K], const float (&xn)[K]) {
    float o[K];
#pragma unroll
    for (int k = 0; k < K; ++k) o[k] = x[k] + w.v[k];
    st_col(p.vs, c, o);
    if (p.pg) {
#pragma unroll
      for (int k = 0; k < K; ++k) o[k] = fmaf(w.lr[k], xn[k], cf[k].b);
      st_col(p.pg, c, o);
    }
  }
};

template <int K>
struct TmIO<EligOpT<K>> {
  using Op = EligOpT<K>;
  static constexpr int kRegs = 48;  // registers per thread, chosen by measurement
  static __device__ __forceinline__ void load(const typename Op::Args &p, const ColTile &c, Flags f,
                                              typename Op::Raw &w) {
    ld_col(p.g, c, w.g);
    w.done = f.term | f.trunc;
    w.halo = col_prev_done(p.term, p.trunc, c);
    w.ev = (c.edge && p.init) ? ld_na(p.init + c.n) : 0.0f;
  }
  static __device__ __forceinline__ void fetch_boundary(const typename Op::Args &, const ColTile &,
                                                        typename Op::Raw &) {}
  static __device__ __forceinline__ uint32_t nbr(const typename Op::Raw &w) { return w.halo; }
  static __device__ __forceinline__ void emit(const typename Op::Args &p, const ColTile &c, const typename Op::Raw &,
                                              const Aff<float> (&)[K], const float (&x)[K], const float (&)[K]) {
    st_col(p.out, c, x);
  }
};

template <int K>
struct TmIO<PrefixSumOpT<K>> {
  using Op = PrefixSumOpT<K>;
  static constexpr int kRegs = 48;  // registers per thread, chosen by measurement
  static __device__ __forceinline__ void load(const typename Op::Args &p, const ColTile &c, Flags f,
                                              typename Op::Raw &w) {
    ld_col(p.x, c, w.x);
    w.done = f.term | f.trunc;
    w.halo = col_prev_done(p.term, p.trunc, c);
  }
  static __device__ __forceinline__ void fetch_boundary(const typename Op::Args &, const ColTile &,
                                                        typename Op::Raw &) {}
  static __device__ __forceinline__ uint32_t nbr(const typename Op::Raw &w) { return w.halo; }
  static __device__ __forceinline__ void emit(const typename Op::Args &p, const ColTile &c, const typename Op::Raw &,
                                              const Aff<uint32_t> (&)[K], const uint32_t (&x)[K],
                                              const uint32_t (&)[K]) {
    st_col(p.out, c, x);
  }
};

template <bool BWD, int K>
struct TmIO<AffineOp<BWD, float, K>> {
  using Op = AffineOp<BWD, float, K>;
  static constexpr int kRegs = 48;  // registers per thread, chosen by measurement
  static __device__ __forceinline__ void load(const typename Op::Args &p, const ColTile &c, Flags f,
                                              typename Op::Raw &w) {
    ld_col(p.a, c, w.a);
    ld_col(p.b, c, w.b);
    w.f = f;
    w.ev = (c.edge && p.init) ? ld_na(p.init + c.n) : 0.0f;
  }
  static __device__ __forceinline__ void fetch_boundary(const typename Op::Args &, const ColTile &,
                                                        typename Op::Raw &) {}
  static __device__ __forceinline__ float nbr(const typename Op::Raw &) { return 0.0f; }
  static __device__ __forceinline__ void emit(const typename Op::Args &p, const ColTile &c, const typename Op::Raw &,
                                              const Aff<float> (&)[K], const float (&x)[K], const float (&)[K]) {
    st_col(p.out, c, x);
  }
};

// ---------------------------------------------------------------------------
// Look-back along T, one environment per lane, the whole block fetching.
// Descriptor (chunk j, environment n) sits at j * dpitch + n, so a warp's 32
// descriptors of one chunk are contiguous; the protocol is scan_core.cuh's
// (self-validating 64-bit words tagged with the launch's epoch, no fences).
// In each round every warp of a column group fetches kTmWin descriptors per
// lane, so the group's WT warps see WT kTmWin chunks in one memory round
// trip; each thread polls its own until ready (bounded by timeout_ns of
// global time and an iteration cap), combines them in dependency order up to
// the first final one (an inclusive value, an aggregate that cuts, or the
// array end) and posts that one entry to shared memory.  After a barrier the
// group's publishing warp walks the WT entries in dependency order; columns
// still open fetch the next window.
// ---------------------------------------------------------------------------
constexpr int kTmWin = 2;  // descriptors per thread per round
enum : uint32_t { kWinAggregate = 0, kWinFinal = 1 };

template <typename V>
struct TmWindow {
  uint32_t state[kTmBlock / 32][32];  // per fetching thread: its kTmWin descriptors combined
  V a[kTmBlock / 32][32], b[kTmBlock / 32][32];
  V cin[kTmBlock / 32][32];           // [column group][lane]: carry entering the chunk
  uint32_t open[kTmBlock / 32][32];   // [column group][lane]: walk not finished
};

// Decodes a descriptor's two words: false if not ready yet, else the entry
// (state, a, b): an aggregate, or a final value in b.
template <typename V>
__device__ __forceinline__ bool decode_desc(unsigned long long w0, unsigned long long w1, uint32_t tag,
                                            uint32_t &st, V &a, V &b) {
  const uint32_t f0 = uint32_t(w0 >> 32);
  if (f0 == (tag | kDescInclusive)) {
    st = kWinFinal;
    b = from_bits<V>(uint32_t(w0));
    return true;
  }
  if (f0 == (tag | kDescAggregate) && uint32_t(w1 >> 32) == (tag | kDescAggregate)) {
    a = from_bits<V>(uint32_t(w0));
    b = from_bits<V>(uint32_t(w1));
    st = cuts(Aff<V>{a, b}) ? kWinFinal : kWinAggregate;  // an aggregate that cuts carries its own value
    return true;
  }
  return false;
}

// Polls a descriptor whose first read was not ready until it is, bounded by
// limit_ns of global time from t0 and an iteration cap; on expiry it records
// the timeout status and returns a final 0, so the walk ends with the partial
// carry.
template <typename V>
__device__ __forceinline__ void wait_desc(const LookbackDesc *d, uint32_t tag, uint32_t t0, uint32_t limit_ns,
                                          uint32_t &st, V &a, V &b) {
  const uint32_t max_polls = 64u + limit_ns / 32u;
  uint32_t sleep_ns = 16u;
  for (uint32_t polls = 0;; ++polls) {
    __nanosleep(sleep_ns);
    sleep_ns = min(sleep_ns * 2u, 256u);
    unsigned long long w0, w1;
    ld_relaxed_desc(d, w0, w1);
    if (decode_desc<V>(w0, w1, tag, st, a, b)) return;
    if (polls > max_polls || uint32_t(global_timer_ns()) - t0 > limit_ns) {
      record_status(kDevStatusTimeout);
      st = kWinFinal;
      b = V(0);
      return;
    }
  }
}

// Blocks per SM that the estimator's register budget (TmIO<Op>::kRegs)
// leaves, over the four 16K-register partitions.  A thread's K steps stay
// live (coefficients and the values its outputs need) across the slice
// combine and the look-back: 64 registers for the estimators with two or
// three per-step inputs, 48 (more blocks resident; a few spilled bytes for
// the eligibility trace and the prefix sum) for the lighter ones, where it
// measured faster.
template <class IO>
constexpr int tm_min_blocks() {
  constexpr int warps = kTmBlock / 32;
  int b = 2048 / kTmBlock;
  while (b > 1 && ((b * warps + 3) / 4) * 32 * IO::kRegs > 16384) --b;
  return b;
}

template <class Op>
__global__ void __launch_bounds__(kTmBlock, tm_min_blocks<TmIO<Op>>())
    tm_scan_kernel(const typename Op::Args p, const TmGeom g) {
  using V = typename Op::V;
  using IO = TmIO<Op>;
  constexpr bool BWD = Op::kBackward;
  constexpr int K = Op::K;
  constexpr uint32_t kFull = K == 32 ? 0xffffffffu : (1u << K) - 1u;

  __shared__ Aff<V> s_agg[kTmBlock / 32][32];    // [warp][lane]: each thread's K-step composite
  __shared__ uint32_t s_ticket, s_epoch;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t wt = 1u << g.wt_log2;
  const uint32_t slice = uint32_t(warp) & (wt - 1u), group = uint32_t(warp) >> g.wt_log2;
  const bool lb = g.nct > 1u;
  // With programmatic dependent launch this grid may start while the previous
  // kernel on the stream finishes; wait for it before touching memory.
  grid_dependency_wait();

  uint32_t chunk = blockIdx.x, ticket = 0, epoch = 0;
  if (lb) {
    if (tid == 0 && !draw_ticket(g.lb.hdr, g.nchunks, s_ticket, s_epoch)) record_status(kDevStatusTimeout);
    __syncthreads();
    ticket = s_ticket;
    epoch = s_epoch;
    if (ticket >= g.nchunks) return;  // counter left inconsistent by an aborted launch
    chunk = ticket;
  }
  // Tickets run over column blocks fastest, time chunks in dependency order.
  const uint32_t jd = chunk / g.nbc, cb = chunk - jd * g.nbc;
  const uint32_t j = BWD ? g.nct - 1u - jd : jd;

  ColTile c;
  c.N = g.N;
  c.n = cb * (256u >> g.wt_log2) + (group << 5) + uint32_t(lane);
  c.t0 = ((j << g.wt_log2) + slice) * uint32_t(K);
  const bool col_ok = c.n < g.N;
  uint32_t v = 0u;
  if (col_ok && c.t0 < g.T) v = g.T - c.t0 >= uint32_t(K) ? kFull : (1u << (g.T - c.t0)) - 1u;
  c.valid = v;
  c.edge = 0u;
  if (v != 0u) {
    if (BWD) {
      const uint32_t rend = g.T - 1u - c.t0;
      c.edge = rend < uint32_t(K) ? (1u << rend) : 0u;
    } else {
      c.edge = c.t0 == 0u ? 1u : 0u;
    }
  }
  c.next = col_ok && c.t0 + uint32_t(K) < g.T;
  c.prev = v != 0u && c.t0 > 0u;
  c.off = uint64_t(c.t0) * g.N + c.n;

  // a1: the tile's loads, halo included.
  typename Op::Raw w;
  const Flags f{ld_col_flags<K>(p.term, c), ld_col_flags<K>(p.trunc, c)};
  IO::load(p, c, f, w);
  grid_dependents_launch();
  IO::fetch_boundary(p, c, w);

  // a2: coefficients, by the row-major builder (one window edge per column).
  Tile tl{};
  tl.valid = c.valid;
  tl.edge = c.edge;
  tl.nvalid = K;
  tl.few_rows = true;
  Aff<V> cf[K];
  Op::coef(p, tl, FastDiv{0u, 0u}, w, IO::nbr(w), cf);
  if (c.valid != kFull) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if (!((c.valid >> k) & 1u)) cf[k] = aff_identity<V>();
  }

  // a4: the thread's composite in dependency order.
  Aff<V> agg;
  if (BWD) {
    agg = cf[K - 1];
#pragma unroll
    for (int k = K - 2; k >= 0; --k) agg = compose(cf[k], agg);
  } else {
    agg = cf[0];
#pragma unroll
    for (int k = 1; k < K; ++k) agg = compose(cf[k], agg);
  }
  s_agg[warp][lane] = agg;
  __syncthreads();

  // a6: composite of the slices this one depends on (later slices backward,
  // earlier forward), in dependency order.
  const uint32_t w0 = group << g.wt_log2;
  Aff<V> pre = aff_identity<V>();
  if (BWD) {
    for (uint32_t u = slice + 1u; u < wt; ++u) pre = compose(pre, s_agg[w0 + u][lane]);
  } else {
    for (uint32_t u = slice; u-- > 0u;) pre = compose(pre, s_agg[w0 + u][lane]);
  }

  V cin = V(0);
  if (lb) {
    // a7: the slice farthest from the chunk's dependency edge holds the
    // chunk's composite once its own is added, and publishes it.
    __shared__ TmWindow<V> s_win;
    const uint32_t tag = epoch << 2;
    const bool silent = g.lb.starve && ticket == 0;
    const bool owner = slice == (BWD ? 0u : wt - 1u);
    const Aff<V> tot = compose(agg, pre);
    LookbackDesc *mine = g.lb.desc + size_t(j) * g.dpitch + c.n;
    if (owner && col_ok && !silent) {
      if (cuts(tot)) {
        st_relaxed_u64(&mine->w[0], desc_word(tag | kDescInclusive, to_bits(tot.b)));
      } else {
        st_relaxed_u64(&mine->w[1], desc_word(tag | kDescAggregate, to_bits(tot.b)));
        st_relaxed_u64(&mine->w[0], desc_word(tag | kDescAggregate, to_bits(tot.a)));
      }
    }
    const uint32_t limit_ns = uint32_t(min(g.lb.timeout_ns, uint64_t(1) << 31));
    const uint32_t per_round = wt * uint32_t(kTmWin);
    Aff<V> acc = aff_identity<V>();  // publishing warp: composite walked so far
    bool open = col_ok && !(BWD ? (j == g.nct - 1u) : (j == 0u));
    const bool walked = open;  // the column needs a carry (else it enters 0)
    for (uint32_t base = 1u;; base += per_round) {
      // Fetch this round's window, chunk distances base + slice kTmWin + d:
      // every load goes out before any is waited on.
      if (open) {
        const uint32_t t0 = uint32_t(global_timer_ns());
        unsigned long long w0[kTmWin], w1[kTmWin];
#pragma unroll
        for (int d = 0; d < kTmWin; ++d) {
          const uint32_t dist = base + slice * uint32_t(kTmWin) + uint32_t(d);
          w0[d] = w1[d] = 0ull;
          if (BWD ? (dist < g.nct - j) : (dist <= j))
            ld_relaxed_desc(g.lb.desc + size_t(BWD ? j + dist : j - dist) * g.dpitch + c.n, w0[d], w1[d]);
        }
        uint32_t est = kWinAggregate;
        Aff<V> e = aff_identity<V>();
#pragma unroll
        for (int d = 0; d < kTmWin; ++d) {
          if (est == kWinAggregate) {
            const uint32_t dist = base + slice * uint32_t(kTmWin) + uint32_t(d);
            uint32_t st = kWinFinal;  // past the array end: nothing enters
            V ea = V(1), eb = V(0);
            if (BWD ? (dist < g.nct - j) : (dist <= j)) {
              if (!decode_desc<V>(w0[d], w1[d], tag, st, ea, eb))
                wait_desc<V>(g.lb.desc + size_t(BWD ? j + dist : j - dist) * g.dpitch + c.n, tag, t0, limit_ns,
                             st, ea, eb);
            }
            if (st == kWinFinal) {
              e = Aff<V>{V(0), apply(e, eb)};
              est = kWinFinal;
            } else {
              e = compose(e, Aff<V>{ea, eb});
            }
          }
        }
        s_win.state[warp][lane] = est;
        s_win.a[warp][lane] = e.a;
        s_win.b[warp][lane] = e.b;
      }
      __syncthreads();
      // The publishing warp walks the group's window in dependency order.
      if (owner && open) {
        for (uint32_t u = 0; u < wt; ++u) {
          const Aff<V> e{s_win.a[w0 + u][lane], s_win.b[w0 + u][lane]};
          if (s_win.state[w0 + u][lane] == kWinFinal) {
            cin = apply(acc, e.b);
            open = false;
            break;
          }
          acc = compose(acc, e);
        }
        s_win.cin[group][lane] = cin;
        s_win.open[group][lane] = open ? 1u : 0u;
      }
      if (!__syncthreads_or(owner && open)) break;
      if (!owner && open) open = s_win.open[group][lane] != 0u;
    }
    if (!owner && walked) cin = s_win.cin[group][lane];
    if (owner && col_ok && !silent && !cuts(tot))
      st_relaxed_u64(&mine->w[0], desc_word(tag | kDescInclusive, to_bits(apply(tot, cin))));
  }

  // a8: re-sweep from the carry entering the tile, then the outputs.
  V x = apply(pre, cin);
  V xs[K], xd[K];
  if (BWD) {
#pragma unroll
    for (int k = K - 1; k >= 0; --k) {
      xd[k] = x;
      x = apply(cf[k], x);
      xs[k] = x;
    }
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      xd[k] = x;
      x = apply(cf[k], x);
      xs[k] = x;
    }
  }
  IO::emit(p, c, w, cf, xs, xd);
}

}  // namespace rlscan
