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

// Programmatic dependent launch (sm_90+): both are no-ops when the grid was
// launched without the programmatic-serialization attribute.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

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
// forward lanes l..0 (agg_l o agg_{l-1} o ... o agg_0).  With WIDTH < 32 only
// lanes 0..WIDTH-1 are scanned (log2 WIDTH rounds).
template <bool BACKWARD, typename V, int WIDTH = 32>
__device__ __forceinline__ Aff<V> warp_inclusive_scan(Aff<V> s, int lane) {
#pragma unroll
  for (int d = 1; d < WIDTH; d <<= 1) {
    V oa, ob;
    if (BACKWARD) {
      oa = __shfl_down_sync(0xffffffffu, s.a, d);
      ob = __shfl_down_sync(0xffffffffu, s.b, d);
      if (lane + d < WIDTH) s = compose(s, Aff<V>{oa, ob});
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
// Per launch: one 64-bit counter, (epoch << 32) | next ticket, hands out
// chunk indices in dependency order (so every chunk a block waits on belongs
// to a block that is already running) together with the launch's epoch, in
// a single atomic.  The block that draws the launch's last ticket moves the
// counter on to (epoch + 1, 0); no other block touches it afterwards, and
// stream order keeps the next launch from drawing before this one has ended.
// Every descriptor's flag carries the epoch of the launch that wrote it, so
// descriptors left over from earlier launches are never read as current and
// the workspace never needs clearing between launches.  A launch that ends
// early (a dead context) leaves the counter inconsistent; the next launch
// reports it as a timeout, and releasing the workspaces clears it.
struct LookbackHeader {
  unsigned long long counter;
  unsigned long long pad;
};

// Draws this block's ticket and the launch's epoch.  False if the counter was
// left inconsistent (ticket out of range).
__device__ __forceinline__ bool draw_ticket(LookbackHeader *h, uint32_t nchunks, uint32_t &ticket,
                                            uint32_t &epoch) {
  const unsigned long long old = atomicAdd(&h->counter, 1ull);
  ticket = uint32_t(old);
  epoch = uint32_t(old >> 32);
  if (ticket == nchunks - 1u) atomicAdd(&h->counter, (1ull << 32) - nchunks);
  return ticket < nchunks;
}

// A chunk's descriptor is two 64-bit words, each (flag << 32) | value with
// flag = (epoch << 2) | state, written and read as single-copy-atomic 64-bit
// accesses.  Every word validates itself, so no fence orders one word against
// another:
//   word 0 = (A, a): the chunk's aggregate's a;  word 1 = (A, b): its b;
//   word 0 = (P, x): its outgoing value x, the scan value at the step its
//            dependent neighbour reads as carry (backward: the chunk's first
//            step; forward: its last step).  Replaces (A, a) when known.
// A reader that sees (P, x) in word 0 is done; one that sees (A, a) needs
// (A, b) in word 1 too, and otherwise polls again.
struct LookbackDesc {
  unsigned long long w[2];
};

enum : uint32_t { kDescAggregate = 1, kDescInclusive = 2 };

__device__ __forceinline__ unsigned long long desc_word(uint32_t flag, uint32_t value) {
  return (static_cast<unsigned long long>(flag) << 32) | value;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Both words of a descriptor in one access; each 64-bit element is
// single-copy atomic on its own, which is all the protocol needs.
__device__ __forceinline__ void ld_relaxed_desc(const LookbackDesc *p, unsigned long long &w0,
                                                unsigned long long &w1) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
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

// Run by all 32 lanes of one warp per block.  Lane 0 publishes the chunk's
// aggregate (or its final value at once if the aggregate already cuts the
// dependency).  The warp then finds the carry entering the chunk's
// dependency edge by polling the descriptors of the next 32 chunks in
// dependency order at once (successors backward, predecessors forward): the
// nearest one that is final -- published value, an aggregate that cuts, or
// the end of the array -- ends the walk as soon as it and every descriptor
// before it are ready, and the aggregates before it are composed with one
// warp scan.  One window normally suffices; otherwise the window slides by
// 32.  Lane 0 finally publishes the chunk's value.
//
// `edge_closed`: the chunk's dependency edge is a row boundary, so its
// elements need no carry.  Every wait is bounded by `timeout_ns` of global
// time (and an iteration cap as a second bound); on expiry the block records
// the timeout status, uses the partial carry, and still publishes so no other
// block waits on it.
template <bool BACKWARD, typename V>
__device__ V decoupled_lookback(const LookbackCtl &ctl, uint32_t chunk, uint32_t nchunks, uint32_t epoch,
                                uint32_t ticket, Aff<V> agg, bool edge_closed, int lane) {
  const uint32_t tag = epoch << 2;
  const bool silent = ctl.starve && ticket == 0;
  LookbackDesc *mine = ctl.desc + chunk;
  const bool self_cut = cuts(agg);
  if (lane == 0 && !silent) {
    if (self_cut) {
      st_relaxed_u64(&mine->w[0], desc_word(tag | kDescInclusive, to_bits(agg.b)));
    } else {
      st_relaxed_u64(&mine->w[1], desc_word(tag | kDescAggregate, to_bits(agg.b)));
      st_relaxed_u64(&mine->w[0], desc_word(tag | kDescAggregate, to_bits(agg.a)));
    }
  }
  V carry = V(0);
  if (!edge_closed) {
    Aff<V> acc = aff_identity<V>();
    // 32-bit bookkeeping keeps the walk light in registers: chunk indices fit
    // (nchunks < 2^31), and the timer's low word measures waits up to 2^31 ns.
    int32_t base = BACKWARD ? int32_t(chunk) + 1 : int32_t(chunk) - 1;
    const uint32_t t0 = uint32_t(global_timer_ns());
    const uint32_t limit_ns = uint32_t(min(ctl.timeout_ns, uint64_t(1) << 31));
    const uint32_t max_polls = 64u + limit_ns / 32u;
    uint32_t polls = 0;
    for (;;) {
      // Lane i looks at the i-th predecessor of the window.  Each lane polls
      // its descriptor only until it is ready; the window is usable as soon
      // as every lane up to the nearest final one is ready, so a far lane
      // never holds up the walk.  Past the array end nothing enters.
      const int32_t j = base + (BACKWARD ? lane : -lane);
      const bool in_range = j >= 0 && uint32_t(j) < nchunks;
      const LookbackDesc *d = ctl.desc + (in_range ? j : 0);
      bool ready = !in_range, final_here = !in_range;
      Aff<V> e = aff_identity<V>();
      V xval = V(0);
      uint32_t sleep_ns = 0;
      bool timed_out = false;
      uint32_t fmask, lead;
      for (;;) {
        if (!ready) {
          unsigned long long w0, w1;
          ld_relaxed_desc(d, w0, w1);
          const uint32_t f0 = uint32_t(w0 >> 32);
          if (f0 == (tag | kDescInclusive)) {
            ready = final_here = true;
            xval = from_bits<V>(uint32_t(w0));
          } else if (f0 == (tag | kDescAggregate) && uint32_t(w1 >> 32) == (tag | kDescAggregate)) {
            ready = true;
            e = Aff<V>{from_bits<V>(uint32_t(w0)), from_bits<V>(uint32_t(w1))};
            if (cuts(e)) {  // an aggregate that cuts carries its own value
              final_here = true;
              xval = e.b;
            }
          }
        }
        const uint32_t rmask = __ballot_sync(0xffffffffu, ready);
        fmask = __ballot_sync(0xffffffffu, final_here);
        lead = rmask == 0xffffffffu ? 32u : uint32_t(__ffs(~rmask) - 1);  // ready lanes 0..lead-1
        const uint32_t first = fmask ? uint32_t(__ffs(fmask) - 1) : 32u;
        if (first < lead || lead == 32u) break;
        // lanes may read the timer a tick apart: decide for the whole warp
        const bool expired = ++polls > max_polls || uint32_t(global_timer_ns()) - t0 > limit_ns;
        if (__any_sync(0xffffffffu, expired)) {
          timed_out = true;
          break;
        }
        if (sleep_ns) __nanosleep(sleep_ns);
        sleep_ns = sleep_ns ? min(sleep_ns * 2u, 256u) : 16u;
      }
      if (timed_out) {
        if (lane == 0) record_status(kDevStatusTimeout);
        carry = acc.b;
        break;
      }
      const int first = fmask ? __ffs(fmask) - 1 : 32;
      // lanes 0..first-1 in dependency order, the nearest outermost
      const Aff<V> win = warp_inclusive_scan<true>(lane < first ? e : aff_identity<V>(), lane);
      const V wa = __shfl_sync(0xffffffffu, win.a, 0);
      const V wb = __shfl_sync(0xffffffffu, win.b, 0);
      acc = compose(acc, Aff<V>{wa, wb});
      if (first < 32) {
        carry = apply(acc, __shfl_sync(0xffffffffu, xval, first));
        break;
      }
      base += BACKWARD ? 32 : -32;
    }
  }
  if (lane == 0 && !silent && !self_cut) st_relaxed_u64(&mine->w[0], desc_word(tag | kDescInclusive, to_bits(apply(agg, carry))));
  return carry;
}

}  // namespace rlscan
