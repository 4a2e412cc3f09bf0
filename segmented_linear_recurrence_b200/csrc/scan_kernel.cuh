// scan_kernel.cuh -- the fused load -> coefficients -> scan -> outputs kernel.
//
// "rl-triton: High-Performance Triton GPU Kernels for Reinforcement Learning
// Credit Assignment" (gist.science technical summary), Methodologie 2: one
// kernel per estimator loads the raw rollout inputs once, builds (a_t, b_t)
// on chip, runs the associative scan on chip and writes each output once, so
// a call moves each element through HBM exactly once.
//
// Work decomposition (ours, B200-first).  A launch sees its [rows, T] slice as
// one flat sequence of `total` steps cut into chunks of L = 8 * BLOCK steps,
// one chunk per thread block; thread j of a block owns the 8 consecutive steps
// starting at chunk * L + 8j (one 256-bit load per fp32 array).  Because the
// coefficient builders put a = 0 on each row's dependency edge, chunks may
// straddle rows freely: the flat scan never leaks a value across a row.
//
// Memory-level parallelism comes from occupancy: blocks are small in
// registers, so several per SM have their loads in flight while others scan,
// and the hardware block scheduler keeps refilling SMs.  Every load whose
// address follows from the chunk's position (per-step arrays, the halo step,
// the bootstrap of a row end) is issued up front; only trunc_value at
// truncated steps depends on loaded data.
//   LB == false : the host only picks this when L is a multiple of T, so every
//                 chunk ends (backward) / starts (forward) on a row edge and
//                 needs no carry from another chunk.
//   LB == true  : chunks take tickets in dependency order and hand carries
//                 over with a decoupled look-back (scan_core.cuh).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "estimators.cuh"
#include "scan_core.cuh"

namespace rlscan {

struct ScanGeom {
  uint32_t total;         // steps in this launch (rows * T)
  uint32_t T;             // steps per row
  uint32_t nchunks;       // chunks (blocks) in this launch
  uint32_t vec;           // 1: arrays aligned for 256-bit (flags: 64-bit) accesses
  uint32_t div_m, div_l;  // FastDiv by T
  uint32_t fetch_wrap;    // the ticket counter wraps to 0 after this value
  LookbackCtl lb;         // ticket / done / epoch counters and descriptors (look-back only)
};

// Steps, row position and row edges of one thread's tile.
template <bool BWD>
__device__ __forceinline__ Tile make_tile(const ScanGeom &g, const FastDiv &fd, uint32_t chunk, uint32_t L,
                                          int tid) {
  Tile t;
  t.i0 = chunk * L + uint32_t(kTile) * uint32_t(tid);
  t.nvalid = t.i0 < g.total ? int(min(uint32_t(kTile), g.total - t.i0)) : 0;
  t.valid = (1u << t.nvalid) - 1u;
  t.fast = g.vec != 0u && t.nvalid == kTile;
  t.few_rows = g.T >= uint32_t(kTile);
  t.n0 = 0;
  t.t0 = 0;
  t.edge = 0;
  if (t.nvalid == 0) return t;
  t.n0 = fd.div(t.i0);
  t.t0 = t.i0 - t.n0 * g.T;
  uint32_t e = 0;
  if (t.few_rows) {
    if (BWD) {
      const uint32_t rend = g.T - 1u - t.t0;
      e = rend < uint32_t(kTile) ? (1u << rend) : 0u;
    } else {
      const uint32_t s = t.t0 == 0u ? 0u : g.T - t.t0;
      e = s < uint32_t(kTile) ? (1u << s) : 0u;
    }
  } else {
    uint32_t tt = t.t0;
#pragma unroll
    for (int k = 0; k < kTile; ++k) {
      if (BWD ? (tt == g.T - 1u) : (tt == 0u)) e |= 1u << k;
      if (++tt == g.T) tt = 0;
    }
  }
  t.edge = e & t.valid;
  return t;
}

template <class Op, int BLOCK, bool LB>
__global__ void __launch_bounds__(BLOCK, 1024 / BLOCK) scan_kernel(const typename Op::Args p, const ScanGeom g) {
  using V = typename Op::V;
  using Raw = typename Op::Raw;
  constexpr bool BWD = Op::kBackward;
  constexpr int W = BLOCK / 32;
  constexpr uint32_t L = uint32_t(kTile) * BLOCK;
  static_assert(BLOCK % 32 == 0 && W <= 32, "block must be whole warps, at most 32");

  __shared__ Aff<V> s_wagg[W];
  __shared__ V s_wcarry[W];
  __shared__ uint32_t s_ticket, s_epoch;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const FastDiv fd{g.div_m, g.div_l};

  // Chunk selection.  With look-back, tickets go out in dependency order
  // (backward: the highest chunk first), so whatever a block waits for is
  // owned by a block that has already started.  atomicInc wraps the counter
  // back to 0 after the launch's last ticket.
  uint32_t chunk = blockIdx.x, ticket = 0, epoch = 0;
  if constexpr (LB) {
    if (tid == 0) {
      s_ticket = atomicInc(&g.lb.hdr->ticket, g.fetch_wrap);
      s_epoch = *reinterpret_cast<volatile uint32_t *>(&g.lb.hdr->epoch);
    }
    __syncthreads();
    ticket = s_ticket;
    epoch = s_epoch;
    if (ticket >= g.nchunks) {  // counter left inconsistent by an aborted launch
      if (tid == 0) record_status(kDevStatusTimeout);
      return;
    }
    chunk = BWD ? g.nchunks - 1u - ticket : ticket;
  }

  // a1: every position-determined load of the tile goes out together.
  const Tile tl = make_tile<BWD>(g, fd, chunk, L, tid);
  Raw w;
  Op::load(p, tl, fd, lane, g.total, w);

  // Neighbouring step across the lane edge (t+1 backward, t-1 forward).
  auto mine = Op::nbr_of(w);
  auto from = BWD ? __shfl_down_sync(0xffffffffu, mine, 1) : __shfl_up_sync(0xffffffffu, mine, 1);
  if (BWD ? lane == 31 : lane == 0) from = Op::halo_of(w);

  // a2: coefficients in registers.
  Aff<V> c[kTile];
  Op::coef(p, tl, fd, w, from, c);
#pragma unroll
  for (int k = 0; k < kTile; ++k)
    if (!((tl.valid >> k) & 1u)) c[k] = aff_identity<V>();

  // a4: sequential composite of the thread's 8 steps, in dependency order.
  Aff<V> agg;
  if (BWD) {
    agg = c[kTile - 1];
#pragma unroll
    for (int k = kTile - 2; k >= 0; --k) agg = compose(c[k], agg);
  } else {
    agg = c[0];
#pragma unroll
    for (int k = 1; k < kTile; ++k) agg = compose(c[k], agg);
  }

  // a5: warp scan.
  const Aff<V> inc = warp_inclusive_scan<BWD>(agg, lane);
  const Aff<V> exc = warp_exclusive_from_inclusive<BWD>(inc, lane, 31);
  if (BWD ? lane == 0 : lane == 31) s_wagg[warp] = inc;
  __syncthreads();

  // a6 (+ a7): warp 0 scans the warp aggregates; with look-back its lane 0
  // also obtains the carry entering the chunk.
  if (warp == 0) {
    const Aff<V> wv = lane < W ? s_wagg[lane] : aff_identity<V>();
    const Aff<V> winc = warp_inclusive_scan<BWD>(wv, lane);
    const Aff<V> wexc = warp_exclusive_from_inclusive<BWD>(winc, lane, W - 1);
    V carry = V(0);
    if constexpr (LB) {
      const V ca = __shfl_sync(0xffffffffu, winc.a, BWD ? 0 : W - 1);
      const V cb = __shfl_sync(0xffffffffu, winc.b, BWD ? 0 : W - 1);
      if (lane == 0) {
        const uint32_t cbase = chunk * L;
        const bool edge_closed = BWD ? (min(cbase + L, g.total) % g.T) == 0u : (cbase % g.T) == 0u;
        carry = decoupled_lookback<BWD, V>(g.lb, chunk, g.nchunks, epoch, ticket, Aff<V>{ca, cb}, edge_closed);
      }
      carry = __shfl_sync(0xffffffffu, carry, 0);
    }
    if (lane < W) s_wcarry[lane] = apply(wexc, carry);
  }
  __syncthreads();

  // a8: re-sweep the thread's steps from the carry and write the outputs.
  V x = apply(exc, s_wcarry[warp]);
  V xs[kTile], xd[kTile];
  if (BWD) {
#pragma unroll
    for (int k = kTile - 1; k >= 0; --k) {
      xd[k] = x;
      x = apply(c[k], x);
      xs[k] = x;
    }
  } else {
#pragma unroll
    for (int k = 0; k < kTile; ++k) {
      xd[k] = x;
      x = apply(c[k], x);
      xs[k] = x;
    }
  }
  Op::emit(p, tl, w, c, xs, xd);

  if constexpr (LB) {
    // The last block of the launch advances the epoch (its done counter wraps
    // to 0 by itself); every block has read the epoch and finished its
    // look-back before it counts itself done.
    if (tid == 0) {
      __threadfence();
      if (atomicInc(&g.lb.hdr->done, g.nchunks - 1u) == g.nchunks - 1u) atomicAdd(&g.lb.hdr->epoch, 1u);
    }
  }
}

}  // namespace rlscan
