// scan_core.cuh -- the affine-composition scan shared by every estimator.
//
// "rl-triton: High-Performance Triton GPU Kernels for Reinforcement Learning
// Credit Assignment" (gist.science technical summary), Methodologie 1: the
// estimators are instances of x_t = b_t + a_t * x_{t+1} (backward) or its
// forward-time mirror x_t = b_t + a_t * x_{t-1}, solved as an associative scan
// of the affine maps f_t(x) = b_t + a_t x under composition.  The page's
// combine (alpha_B, beta_B) (+) (alpha_A, beta_A) = (alpha_B + beta_B alpha_A,
// beta_A beta_B) is compose(outer = B, inner = A) below with alpha = b and
// beta = a.  It is associative (not commutative) with identity (a, b) = (1, 0).
//
// Hierarchy used by the kernels (B200-first, not the pages' Triton design):
//   thread  : 4 contiguous steps composed sequentially in registers
//   warp    : 5-round Kogge-Stone shuffle scan of the thread aggregates
//   block   : warp aggregates through shared memory, scanned by warp 0
//   grid    : decoupled look-back over per-block descriptors in global memory
//             (only where a row is longer than one block's chunk).
// Row boundaries need no special casing in the scan: the coefficient builders
// set a = 0 on the step that ends a row (backward) or starts one (forward),
// which cuts every composite that crosses it.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace rlscan {

// Unsigned division by a launch-wide constant d (1 <= d <= 2^30) for
// numerators below 2^31: q = umulhi(n, m) >> (l - 1) with l = ceil(log2 d) and
// m = ceil(2^(31+l) / d) (the round-up method of Granlund & Montgomery); the
// host computes (m, l).  d = 1 is flagged by l = 0.
struct FastDiv {
  uint32_t m, l;
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    return l == 0u ? n : (__umulhi(n, m) >> (l - 1u));
  }
};

// The affine map x -> b + a * x.
template <typename V>
struct Aff {
  V a, b;
};

template <typename V>
__device__ __forceinline__ Aff<V> aff_identity() {
  return Aff<V>{V(1), V(0)};
}

// outer o inner: apply `inner` first, then `outer`.
__device__ __forceinline__ Aff<float> compose(Aff<float> o, Aff<float> i) {
  return Aff<float>{o.a * i.a, fmaf(o.a, i.b, o.b)};
}
// Integer variant for the episodic prefix sum: a is 0 or 1, b wraps mod 2^32.
__device__ __forceinline__ Aff<uint32_t> compose(Aff<uint32_t> o, Aff<uint32_t> i) {
  return Aff<uint32_t>{o.a & i.a, o.b + o.a * i.b};
}

__device__ __forceinline__ float apply(Aff<float> f, float x) { return fmaf(f.a, x, f.b); }
__device__ __forceinline__ uint32_t apply(Aff<uint32_t> f, uint32_t x) { return f.b + f.a * x; }

__device__ __forceinline__ bool cuts(Aff<float> f) { return f.a == 0.0f; }
__device__ __forceinline__ bool cuts(Aff<uint32_t> f) { return f.a == 0u; }

// Lane l receives the inclusive composite, in dependency order, of the lanes
// it depends on: BACKWARD lanes l..31 (agg_l o agg_{l+1} o ... o agg_31),
// forward lanes l..0 (agg_l o agg_{l-1} o ... o agg_0).
template <bool BACKWARD, typename V>
__device__ __forceinline__ Aff<V> warp_inclusive_scan(Aff<V> s, int lane) {
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    V oa, ob;
    if (BACKWARD) {
      oa = __shfl_down_sync(0xffffffffu, s.a, d);
      ob = __shfl_down_sync(0xffffffffu, s.b, d);
      if (lane + d < 32) s = compose(s, Aff<V>{oa, ob});
    } else {
      oa = __shfl_up_sync(0xffffffffu, s.a, d);
      ob = __shfl_up_sync(0xffffffffu, s.b, d);
      if (lane >= d) s = compose(s, Aff<V>{oa, ob});
    }
  }
  return s;
}

// The neighbour's inclusive composite in dependency order (what lane l needs
// applied to the carry that enters the warp); identity at the warp edge.
template <bool BACKWARD, typename V>
__device__ __forceinline__ Aff<V> warp_exclusive_from_inclusive(Aff<V> inc, int lane, int last) {
  V a = BACKWARD ? __shfl_down_sync(0xffffffffu, inc.a, 1) : __shfl_up_sync(0xffffffffu, inc.a, 1);
  V b = BACKWARD ? __shfl_down_sync(0xffffffffu, inc.b, 1) : __shfl_up_sync(0xffffffffu, inc.b, 1);
  bool edge = BACKWARD ? (lane >= last) : (lane == 0);
  return edge ? aff_identity<V>() : Aff<V>{a, b};
}

// ---------------------------------------------------------------------------
// Device status word (one per device, shared by all streams).  The first
// recorded error wins; the host reads and clears it in rlscan_sync_status().
// ---------------------------------------------------------------------------
enum : uint32_t { kDevStatusOk = 0, kDevStatusInvalidArg = 1, kDevStatusTimeout = 4 };

// Defined here: the library is built as a single translation unit.
__device__ uint32_t g_rlscan_device_status = 0;

__device__ __forceinline__ void record_status(uint32_t code) {
  atomicCAS(&g_rlscan_device_status, 0u, code);
}

// ---------------------------------------------------------------------------
// Decoupled look-back workspace.
// ---------------------------------------------------------------------------
// Per launch: a ticket counter hands out chunk indices in dependency order (so
// every chunk a block waits on belongs to a block that is already running),
// a done counter lets the last block reset both counters and advance the
// epoch, and every descriptor's flag carries the epoch of the launch that
// wrote it, so descriptors left over from earlier launches are never read as
// current and the workspace never needs clearing between launches.
struct LookbackHeader {
  uint32_t ticket;
  uint32_t done;
  uint32_t epoch;
  uint32_t pad;
};

// flag = (epoch << 2) | state.  State 1: the chunk's aggregate (a, b) is
// published.  State 2: its outgoing value x is published -- the scan value at
// the step its dependent neighbour reads as carry (backward: the chunk's
// first step; forward: its last step).
struct LookbackDesc {
  uint32_t flag;
  uint32_t a;
  uint32_t b;
  uint32_t x;
};

enum : uint32_t { kDescAggregate = 1, kDescInclusive = 2 };

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t *p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t to_bits(float v) { return __float_as_uint(v); }
__device__ __forceinline__ uint32_t to_bits(uint32_t v) { return v; }
template <typename V>
__device__ __forceinline__ V from_bits(uint32_t u);
template <>
__device__ __forceinline__ float from_bits<float>(uint32_t u) {
  return __uint_as_float(u);
}
template <>
__device__ __forceinline__ uint32_t from_bits<uint32_t>(uint32_t u) {
  return u;
}

struct LookbackCtl {
  LookbackHeader *hdr;
  LookbackDesc *desc;
  uint64_t timeout_ns;
  uint32_t starve;  // test only: the block holding ticket 0 never publishes
};

// Run by one thread per block.  Publishes the chunk's aggregate (or its final
// value at once if the aggregate already cuts the dependency), finds the
// carry entering the chunk's dependency edge by walking successors (backward)
// or predecessors (forward), then publishes the chunk's final value.
//
// `edge_closed`: the chunk's dependency edge is a row boundary, so its
// elements need no carry.  Every wait is bounded by `timeout_ns` of global
// time (and an iteration cap as a second bound); on expiry the block records
// RLSCAN timeout status, uses the partial carry, and still publishes so no
// other block waits on it.
template <bool BACKWARD, typename V>
__device__ V decoupled_lookback(const LookbackCtl &ctl, uint32_t chunk, uint32_t nchunks,
                                uint32_t epoch, uint32_t ticket, Aff<V> agg, bool edge_closed) {
  const uint32_t tag = epoch << 2;
  const bool silent = ctl.starve && ticket == 0;
  LookbackDesc *mine = ctl.desc + chunk;
  const bool self_cut = cuts(agg);
  if (!silent) {
    if (self_cut) {
      st_relaxed_u32(&mine->x, to_bits(agg.b));
      st_release_u32(&mine->flag, tag | kDescInclusive);
    } else {
      st_relaxed_u32(&mine->a, to_bits(agg.a));
      st_relaxed_u32(&mine->b, to_bits(agg.b));
      st_release_u32(&mine->flag, tag | kDescAggregate);
    }
  }
  V carry = V(0);
  if (!edge_closed) {
    Aff<V> acc = aff_identity<V>();
    int64_t j = BACKWARD ? int64_t(chunk) + 1 : int64_t(chunk) - 1;
    bool resolved = false;
    const uint64_t t0 = global_timer_ns();
    const uint64_t max_iters = 64 + ctl.timeout_ns / 64;
    while (!resolved && j >= 0 && j < int64_t(nchunks)) {
      const LookbackDesc *d = ctl.desc + j;
      uint32_t f = 0;
      uint32_t sleep_ns = 32;
      uint64_t iters = 0;
      bool timed_out = false;
      for (;;) {
        f = ld_acquire_u32(&d->flag);
        if ((f & ~3u) == tag && (f & 3u) != 0u) break;
        if (++iters > max_iters || global_timer_ns() - t0 > ctl.timeout_ns) {
          timed_out = true;
          break;
        }
        __nanosleep(sleep_ns);
        if (sleep_ns < 1024) sleep_ns <<= 1;
      }
      if (timed_out) {
        record_status(kDevStatusTimeout);
        carry = acc.b;
        resolved = true;
        break;
      }
      if ((f & 3u) == kDescInclusive) {
        carry = apply(acc, from_bits<V>(ld_relaxed_u32(&d->x)));
        resolved = true;
      } else {
        Aff<V> pa{from_bits<V>(ld_relaxed_u32(&d->a)), from_bits<V>(ld_relaxed_u32(&d->b))};
        acc = compose(acc, pa);
        if (cuts(acc)) {
          carry = acc.b;
          resolved = true;
        }
        j += BACKWARD ? 1 : -1;
      }
    }
    if (!resolved) carry = acc.b;  // ran past the array end: nothing enters
  }
  if (!silent && !self_cut) {
    st_relaxed_u32(&mine->x, to_bits(apply(agg, carry)));
    st_release_u32(&mine->flag, tag | kDescInclusive);
  }
  return carry;
}

}  // namespace rlscan
