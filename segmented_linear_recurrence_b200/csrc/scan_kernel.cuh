// scan_kernel.cuh -- the fused load -> coefficients -> scan -> outputs kernel.
//
// "rl-triton: High-Performance Triton GPU Kernels for Reinforcement Learning
// Credit Assignment" (gist.science technical summary), Methodologie 2: one
// kernel per estimator loads the raw rollout inputs once, builds (a_t, b_t)
// on chip, runs the associative scan on chip and writes each output once, so
// a call moves each element through HBM exactly once.
//
// Work decomposition (ours, B200-first).  Thread j of a block owns the K
// (= Op::K, 8 or 16) consecutive steps starting at base + K j, base a
// multiple of K (one 256-bit load per 8 steps of an fp32 array).  Two plans:
//   LB == false (rows fit a block): block b owns rows [b k, (b + 1) k), i.e.
//     the steps [b span, (b + 1) span) with span = k T.  Its tiles start at
//     that range's first step rounded down to a multiple of K, so the first
//     and last tile may hold steps of the neighbouring blocks: those are
//     loaded (in bounds, harmless) but neither scanned nor stored.  Every
//     block's range starts and ends on row edges, so no block needs a carry
//     from another.  The host picks k (and the block size) to fill the
//     block's threads.
//   LB == true (rows longer than a block): the launch's steps are one flat
//     sequence cut into chunks of L = K * BLOCK steps; chunks take tickets
//     in dependency order and hand carries over with a decoupled look-back
//     (scan_core.cuh).  Because the coefficient builders put a = 0 on each
//     row's dependency edge, chunks may straddle rows freely: the flat scan
//     never leaks a value across a row.
//
// Memory-level parallelism comes from occupancy: blocks are small in
// registers, so several per SM have their loads in flight while others scan,
// and the hardware block scheduler keeps refilling SMs.  Every load whose
// address follows from the tile's position (per-step arrays, the halo step,
// the bootstrap of a row end) is issued up front; only trunc_value at
// truncated steps depends on loaded data.
#pragma once

#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "estimators.cuh"
#include "scan_core.cuh"

namespace rlscan {

struct ScanGeom {
  uint32_t total;         // steps in this launch (rows * T)
  uint32_t T;             // steps per row
  uint32_t nchunks;       // chunks (blocks) in this launch
  uint32_t span;          // rows plan: steps per chunk (k T)
  uint32_t rows_per_chunk;  // rows plan: k
  uint32_t vec;           // 1: arrays aligned for 256-bit (flags: 64-bit) accesses
  uint32_t div_m, div_l;  // FastDiv by T
  uint32_t cpr;           // look-back plan: chunks per row when rows are whole chunks, else 0
  LookbackCtl lb;         // ticket / done / epoch counters and descriptors (look-back only)
};

// Look-back plan: the chunk a ticket stands for.  Tickets go out in
// dependency order, so a block only waits on chunks whose tickets were drawn
// earlier.  When rows are whole chunks (cpr > 0) the tickets interleave the
// rows -- the first chunk in dependency order of every row, then the second
// of every row, ... -- so a chunk's predecessor drew its ticket a whole
// launch's rows earlier and has normally published by the time it is needed;
// a row's first chunk needs no carry.  Otherwise the flat order: chunks
// straddle rows and the predecessor is the previous ticket.
__device__ __forceinline__ uint32_t chunk_of_ticket(const ScanGeom &g, uint32_t ticket, bool backward) {
  if (g.cpr == 0u) return backward ? g.nchunks - 1u - ticket : ticket;
  const uint32_t rows = g.nchunks / g.cpr;
  const uint32_t s = ticket / rows, r = ticket - s * rows;
  return r * g.cpr + (backward ? g.cpr - 1u - s : s);
}

// Steps, row position and row edges of the K-step tile at step i0 (a multiple of K)
// of a block that owns the steps [lo, hi), i0 + 8 > lo.
template <bool BWD, int K>
__device__ __forceinline__ Tile make_tile(const ScanGeom &g, const FastDiv &fd, uint32_t i0, uint32_t lo,
                                          uint32_t hi) {
  Tile t;
  t.i0 = i0;
  t.nvalid = i0 < g.total ? int(min(uint32_t(K), g.total - i0)) : 0;
  uint32_t v = i0 < hi ? (1u << min(uint32_t(K), hi - i0)) - 1u : 0u;
  if (i0 < lo) v &= ~((1u << (lo - i0)) - 1u);
  t.valid = v;
  t.fast = g.vec != 0u && t.nvalid == K;
  t.full = t.fast && v == (K == 32 ? 0xffffffffu : (1u << K) - 1u);
  t.few_rows = g.T >= uint32_t(K);
  t.n0 = 0;
  t.t0 = 0;
  t.edge = 0;
  if (v == 0u) return t;
  t.n0 = fd.div(t.i0);
  t.t0 = t.i0 - t.n0 * g.T;
  uint32_t e = 0;
  if (t.few_rows) {
    if (BWD) {
      const uint32_t rend = g.T - 1u - t.t0;
      e = rend < uint32_t(K) ? (1u << rend) : 0u;
    } else {
      const uint32_t s = t.t0 == 0u ? 0u : g.T - t.t0;
      e = s < uint32_t(K) ? (1u << s) : 0u;
    }
  } else {
    uint32_t tt = t.t0;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if (BWD ? (tt == g.T - 1u) : (tt == 0u)) e |= 1u << k;
      if (++tt == g.T) tt = 0;
    }
  }
  t.edge = e & t.valid;
  return t;
}

// Word-wise copy of a register-resident value to / from column `lane` of a
// [words][32] shared array (conflict-free).  Warp 0 parks its coefficients
// there while it runs the look-back, so the look-back's registers do not add
// to the tile's.
template <class T>
__device__ __forceinline__ void park(uint32_t (*s)[32], int lane, const T &v) {
  static_assert(sizeof(T) % 4 == 0, "parked values are whole words");
#pragma unroll
  for (int i = 0; i < int(sizeof(T) / 4); ++i) {
    uint32_t u;
    memcpy(&u, reinterpret_cast<const char *>(&v) + 4 * i, 4);
    s[i][lane] = u;
  }
}
template <class T>
__device__ __forceinline__ void unpark(const uint32_t (*s)[32], int lane, T &v) {
#pragma unroll
  for (int i = 0; i < int(sizeof(T) / 4); ++i) {
    const uint32_t u = s[i][lane];
    memcpy(reinterpret_cast<char *>(&v) + 4 * i, &u, 4);
  }
}

// Blocks per SM the register budget must allow: each estimator states the
// registers per thread its tile needs (Op::kRegs, and Op::kRegsLookback for
// the look-back kernel, whose walk runs in warp 0 only and may spill there).
// More resident blocks keep more loads in flight.  The register file is four
// 16K-register partitions, one per warp scheduler, so the count is the most
// blocks whose warps, spread over the four, each get `regs` (rounded up to
// the allocation unit of 8).
template <class Op, int BLOCK, bool LB>
constexpr int min_blocks_per_sm() {
  constexpr int regs = ((LB ? Op::kRegsLookback : Op::kRegs) + 7) / 8 * 8;
  constexpr int warps = BLOCK / 32;
  int b = 2048 / BLOCK;
  while (b > 1 && ((b * warps + 3) / 4) * 32 * regs > 16384) --b;
  return b;
}

// Flag bytes of one tile, prefetched into shared memory for the block's next
// chunk: each thread copies its own tile's 8 terminated and 8 truncated bytes
// with cp.async and reads them back itself (no barrier needed).
// 16-byte aligned: the 8-byte cp.async copies need an 8-byte aligned
// destination, whatever the shared-memory layout around the slots.
template <int K>
struct __align__(16) FlagSlot {
  uint32_t term[K / 4], trunc[K / 4];
};
static_assert(alignof(FlagSlot<8>) >= 8 && sizeof(FlagSlot<8>) == 16, "cp.async destinations must stay aligned");
static_assert(alignof(FlagSlot<16>) >= 8 && sizeof(FlagSlot<16>) == 32, "cp.async destinations must stay aligned");

// Flag masks from a prefetched slot (bit k: step k).
template <int K>
__device__ __forceinline__ uint32_t slot_mask(const uint32_t (&w)[K / 4]) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < K / 4; ++j) m |= nonzero_bytes4(w[j]) << (4 * j);
  return m;
}

__device__ __forceinline__ void cp_async8(void *dst_smem, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))),
               "l"(src)
               : "memory");
}

// Shared state of one block, reused chunk after chunk.
template <class Op, int BLOCK, bool LB>
struct ScanSmem {
  using V = typename Op::V;
  static constexpr int W = BLOCK / 32;
  static constexpr int kParked = LB ? int(sizeof(Aff<V>) * Op::K / 4) : 1;
  Aff<V> wagg[W];
  Aff<V> wagg2[2][W];  // rows plan: double-buffered by chunk
  V wcarry[W];
  uint32_t ticket, epoch;
  uint32_t park[kParked][32];
};

// One chunk: the block's steps [lo, hi), tiles from `base`.  `f` holds the
// thread's flag masks.  Look-back plan: `chunk` is the ticketed chunk.
// a8: re-sweep the thread's steps from the carry x entering its tile and
// write the outputs.
template <class Op>
__device__ __forceinline__ void resweep_and_emit(const typename Op::Args &p, const Tile &tl,
                                                 const typename Op::Raw &w,
                                                 const Aff<typename Op::V> (&c)[Op::K], typename Op::V x) {
  using V = typename Op::V;
  constexpr int K = Op::K;
  V xs[K], xd[K];
  if (Op::kBackward) {
#pragma unroll
    for (int k = K - 1; k >= 0; --k) {
      xd[k] = x;
      x = apply(c[k], x);
      xs[k] = x;
    }
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      xd[k] = x;
      x = apply(c[k], x);
      xs[k] = x;
    }
  }
  Op::emit(p, tl, w, c, xs, xd);
}

// Rows plan: the loads that depend on the flags go out right behind the
// tile's other loads (the flags are normally in hand already, prefetched).
// Look-back plan: they follow once the tile's own loads have arrived, which
// keeps their registers out of the load phase.
template <class Op, int BLOCK, bool LB>
__device__ __forceinline__ void scan_chunk(const typename Op::Args &p, const ScanGeom &g, const FastDiv &fd,
                                           ScanSmem<Op, BLOCK, LB> &sm, uint32_t chunk, const Tile &tl, Flags f,
                                           int tid, int sm_buf) {
  constexpr bool early = !LB;
  using V = typename Op::V;
  using Raw = typename Op::Raw;
  constexpr bool BWD = Op::kBackward;
  constexpr int W = BLOCK / 32;
  constexpr int K = Op::K;
  constexpr uint32_t L = uint32_t(K) * BLOCK;
  const int lane = tid & 31, warp = tid >> 5;

  // a1: every load of the tile goes out together.
  Raw w;
  Op::load(p, tl, fd, lane, g.total, f, w);
  if constexpr (early) Op::fetch_boundary(p, tl, fd, w);
  // Every block has issued its loads: the next kernel may start launching.
  grid_dependents_launch();

  // Neighbouring step across the lane edge (t+1 backward, t-1 forward).
  auto mine = Op::nbr_of(w);
  auto from = BWD ? __shfl_down_sync(0xffffffffu, mine, 1) : __shfl_up_sync(0xffffffffu, mine, 1);
  if (BWD ? lane == 31 : lane == 0) from = Op::halo_of(w);
  if constexpr (!early) Op::fetch_boundary(p, tl, fd, w);

  // a2: coefficients in registers.
  Aff<V> c[K];
  Op::coef(p, tl, fd, w, from, c);
  if (tl.valid != (K == 32 ? 0xffffffffu : (1u << K) - 1u)) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if (!((tl.valid >> k) & 1u)) c[k] = aff_identity<V>();
  }

  // a4: sequential composite of the thread's K steps, in dependency order.
  Aff<V> agg;
  if (BWD) {
    agg = c[K - 1];
#pragma unroll
    for (int k = K - 2; k >= 0; --k) agg = compose(c[k], agg);
  } else {
    agg = c[0];
#pragma unroll
    for (int k = 1; k < K; ++k) agg = compose(c[k], agg);
  }

  // a5: warp scan.
  const Aff<V> inc = warp_inclusive_scan<BWD>(agg, lane);
  const Aff<V> exc = warp_exclusive_from_inclusive<BWD>(inc, lane, 31);
  if (BWD ? lane == 0 : lane == 31) {
    if constexpr (LB)
      sm.wagg[warp] = inc;
    else
      sm.wagg2[sm_buf][warp] = inc;
  }
  __syncthreads();

  if constexpr (!LB) {
    // Rows plan: the chunk needs no carry from outside, so every warp scans
    // the W warp aggregates itself (one barrier per chunk): the carry entering
    // warp w is the composite of the warps after it (backward) / before it
    // (forward), applied to 0.  Aggregates alternate between two buffers so
    // the next chunk's writes never meet this chunk's reads.
    constexpr int kWidth = W <= 4 ? 4 : (W <= 8 ? 8 : (W <= 16 ? 16 : 32));
    const Aff<V> wv = lane < W ? sm.wagg2[sm_buf][lane] : aff_identity<V>();
    const Aff<V> winc = warp_inclusive_scan<BWD, V, kWidth>(wv, lane);
    const int src = BWD ? warp + 1 : warp - 1;
    const V nb = __shfl_sync(0xffffffffu, winc.b, src < 0 ? 0 : (src >= W ? W - 1 : src));
    const V carry_w = (src < 0 || src >= W) ? V(0) : nb;
    resweep_and_emit<Op>(p, tl, w, c, apply(exc, carry_w));
    return;
  }

  // a6 (+ a7): warp 0 scans the warp aggregates; with look-back it also
  // obtains the carry entering the chunk.
  if (warp == 0) {
    const Aff<V> wv = lane < W ? sm.wagg[lane] : aff_identity<V>();
    const Aff<V> winc = warp_inclusive_scan<BWD>(wv, lane);
    const Aff<V> wexc = warp_exclusive_from_inclusive<BWD>(winc, lane, W - 1);
    V carry = V(0);
    if constexpr (LB) {
      const V ca = __shfl_sync(0xffffffffu, winc.a, BWD ? 0 : W - 1);
      const V cb = __shfl_sync(0xffffffffu, winc.b, BWD ? 0 : W - 1);
      park(sm.park, lane, c);
      // Re-read from shared memory rather than kept live through the loads.
      const uint32_t tk = *reinterpret_cast<volatile uint32_t *>(&sm.ticket);
      const uint32_t ep = *reinterpret_cast<volatile uint32_t *>(&sm.epoch);
      const bool edge_closed = BWD ? (min((chunk + 1u) * L, g.total) % g.T) == 0u : ((chunk * L) % g.T) == 0u;
      carry = decoupled_lookback<BWD, V>(g.lb, chunk, g.nchunks, ep, tk, Aff<V>{ca, cb}, edge_closed, lane);
      unpark(sm.park, lane, c);
    }
    if (lane < W) sm.wcarry[lane] = apply(wexc, carry);
  }
  __syncthreads();

  resweep_and_emit<Op>(p, tl, w, c, apply(exc, sm.wcarry[warp]));
}

template <class Op, int BLOCK, bool LB>
__global__ void __launch_bounds__(BLOCK, (min_blocks_per_sm<Op, BLOCK, LB>()))
    scan_kernel(const typename Op::Args p, const ScanGeom g) {
  constexpr bool BWD = Op::kBackward;
  constexpr int K = Op::K;
  constexpr uint32_t L = uint32_t(K) * BLOCK;
  static_assert(BLOCK % 32 == 0 && BLOCK / 32 <= 32, "block must be whole warps, at most 32");

  __shared__ ScanSmem<Op, BLOCK, LB> sm;
  const int tid = threadIdx.x;
  const FastDiv fd{g.div_m, g.div_l};
  // With programmatic dependent launch this grid may start while the previous
  // kernel on the stream finishes; wait for it before touching memory.
  grid_dependency_wait();

  if constexpr (LB) {
    // Chunk selection: tickets go out in dependency order (chunk_of_ticket),
    // so whatever a block waits for is owned by a block that has already
    // started.
    if (tid == 0 && !draw_ticket(g.lb.hdr, g.nchunks, sm.ticket, sm.epoch)) record_status(kDevStatusTimeout);
    __syncthreads();
    const uint32_t ticket = sm.ticket;
    if (ticket >= g.nchunks) return;  // counter left inconsistent by an aborted launch
    const uint32_t chunk = chunk_of_ticket(g, ticket, BWD);
    const uint32_t lo = chunk * L, hi = min(lo + L, g.total);
    const Tile tl = make_tile<BWD, K>(g, fd, lo + uint32_t(K) * uint32_t(tid), lo, hi);
    const Flags f{ld_flags<K>(p.term, tl), ld_flags<K>(p.trunc, tl)};
    scan_chunk<Op, BLOCK, LB>(p, g, fd, sm, chunk, tl, f, tid, 0);
  } else {
    // Rows plan, persistent: the block takes chunks blockIdx.x, + gridDim.x,
    // ...  While it scans one chunk, its threads prefetch the next chunk's
    // flag bytes, so the trunc_value loads that depend on them go out with
    // the chunk's other loads instead of a memory round trip later.
    __shared__ FlagSlot<K> slots[2][BLOCK];
    auto tile_of = [&](uint32_t chunk) {
      const uint32_t lo = chunk * g.span, hi = min(lo + g.span, g.total);
      return make_tile<BWD, K>(g, fd, (lo & ~uint32_t(K - 1)) + uint32_t(K) * uint32_t(tid), lo, hi);
    };
    // Prefetch needs the 8-byte copies in bounds and aligned: full tiles of
    // vectorised launches only; any other tile loads its flags directly.
    // Only the next tile's first step is computed ahead; its full geometry
    // is built after the current chunk, to keep the loop light in registers.
    auto prefetch = [&](uint32_t chunk, FlagSlot<K> &slot) {
      const uint32_t i0 = ((chunk * g.span) & ~uint32_t(K - 1)) + uint32_t(K) * uint32_t(tid);
      if (g.vec == 0u || i0 + uint32_t(K) > g.total) return false;
#pragma unroll
      for (int j = 0; j < K / 8; ++j) {
        if (p.term) cp_async8(slot.term + 2 * j, p.term + i0 + 8 * j);
        if (p.trunc) cp_async8(slot.trunc + 2 * j, p.trunc + i0 + 8 * j);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      return true;
    };
    // When every chunk starts on a K-step boundary (k T a multiple of K), a
    // thread's tile has the same offset, time and row edges in every full
    // chunk: only its first step and row move.  Holding that tile across the
    // loop costs registers, so estimators on a 32-register budget (where it
    // measured slower) rebuild the tile per chunk instead.
    constexpr bool kKeepTile = Op::kRegs >= 40;
    const bool aligned = kKeepTile && (g.span % uint32_t(K)) == 0u && g.span <= g.total;
    Tile inv = make_tile<BWD, K>(g, fd, uint32_t(K) * uint32_t(tid), 0u, g.span);
    if (inv.valid == 0u) {  // thread beyond the chunk's steps: loads nothing
      inv.nvalid = 0;
      inv.fast = inv.full = false;
    }
    bool have = false;  // slots[buf][tid] holds this chunk's flags
    int buf = 0;
    for (uint32_t chunk = blockIdx.x; chunk < g.nchunks; chunk += gridDim.x) {
      const uint32_t lo = chunk * g.span;
      Tile tl;
      if (aligned && lo + g.span <= g.total) {
        tl = inv;
        tl.i0 = lo + uint32_t(K) * uint32_t(tid);
        tl.n0 = inv.n0 + chunk * g.rows_per_chunk;
      } else {
        tl = tile_of(chunk);
      }
      Flags f;
      if (have) {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        const FlagSlot<K> &s = slots[buf][tid];
        f.term = p.term ? slot_mask<K>(s.term) : 0u;
        f.trunc = p.trunc ? slot_mask<K>(s.trunc) : 0u;
      } else {
        f = Flags{ld_flags<K>(p.term, tl), ld_flags<K>(p.trunc, tl)};
      }
      const uint32_t next = chunk + gridDim.x;
      have = next < g.nchunks && prefetch(next, slots[buf ^ 1][tid]);
      scan_chunk<Op, BLOCK, LB>(p, g, fd, sm, chunk, tl, f, tid, buf);
      buf ^= 1;
    }
  }
}

}  // namespace rlscan
