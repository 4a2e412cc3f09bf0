// scan_kernel.cuh -- the fused load -> coefficients -> scan -> outputs kernel.
//
// "rl-triton: High-Performance Triton GPU Kernels for Reinforcement Learning
// Credit Assignment" (gist.science technical summary), Methodologie 2: one
// kernel per estimator loads the raw rollout inputs once, builds (a_t, b_t)
// on chip, runs the associative scan on chip and writes each output once, so
// a call moves each element through HBM exactly once.
//
// Work decomposition (ours).  A launch sees its [rows, T] slice as one flat
// sequence of `total` steps; block c owns the chunk [c*L, (c+1)*L) with
// L = 4 * BLOCK steps, thread j of it the 4 consecutive steps starting at
// c*L + 4j (one 128-bit load per array when aligned).  Because the
// coefficient builders put a = 0 on each row's dependency edge, chunks may
// straddle rows freely: the flat scan never leaks a value across a row.
//   LB == false : the host only picks this when L is a multiple of T, so every
//                 chunk ends (backward) / starts (forward) on a row edge and
//                 needs no carry from another block.
//   LB == true  : chunks take tickets in dependency order and hand carries
//                 over with a decoupled look-back (scan_core.cuh).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "estimators.cuh"
#include "scan_core.cuh"

namespace rlscan {

struct ScanGeom {
  uint32_t total;    // steps in this launch (rows * T)
  uint32_t T;        // steps per row
  uint32_t nchunks;  // blocks in this launch
  uint32_t vec;      // 1: every array is aligned for 128-bit (flags: 32-bit) accesses
  LookbackCtl lb;    // used only when LB
};

template <class Op, int BLOCK, bool LB>
__global__ void __launch_bounds__(BLOCK) scan_kernel(const typename Op::Args p, const ScanGeom g) {
  using V = typename Op::V;
  using Item = typename Op::Item;
  using Nbr = typename Op::Nbr;
  using Aux = typename Op::Aux;
  constexpr bool BWD = Op::kBackward;
  constexpr int W = BLOCK / 32;
  constexpr uint32_t L = 4u * BLOCK;
  static_assert(BLOCK % 32 == 0 && W <= 32, "block must be whole warps, at most 32");

  __shared__ Aff<V> s_wagg[W];
  __shared__ V s_wcarry[W];
  __shared__ uint32_t s_ticket, s_epoch;
  extern __shared__ __align__(16) unsigned char dyn_smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // Chunk selection.  With look-back, tickets go out in dependency order
  // (backward: the highest chunk first), so whatever a block waits for is
  // owned by a block that has already started.  atomicInc wraps the counter
  // back to 0 after the launch's last ticket.
  uint32_t chunk = blockIdx.x, ticket = 0, epoch = 0;
  if constexpr (LB) {
    if (tid == 0) {
      s_ticket = atomicInc(&g.lb.hdr->ticket, g.nchunks - 1u);
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
  const uint32_t cbase = chunk * L;

  if constexpr (Op::kPrologue) Op::prologue(p, cbase, L, g.total, dyn_smem, tid, BLOCK, g.lb.timeout_ns);

  // a1: load this thread's 4 steps.
  const uint32_t i0 = cbase + 4u * uint32_t(tid);
  const int nvalid = i0 < g.total ? int(min(4u, g.total - i0)) : 0;
  uint32_t n = 0, t = 0;
  if (nvalid) {
    n = i0 / g.T;
    t = i0 - n * g.T;
  }
  Item it[4];
  Op::load(p, i0, nvalid, g.vec != 0u, it);

  // Neighbouring step (t+1 backward, t-1 forward): inside the thread, from the
  // adjacent lane by shuffle, or one halo load at the warp edge.
  Nbr nb[4];
  if constexpr (Op::kNeedsNbr) {
    if constexpr (Op::kPrologue) {
#pragma unroll
      for (int k = 0; k < 4; ++k) nb[k] = Op::nbr_smem(dyn_smem, L, 4u * uint32_t(tid) + k + 1u);
    } else {
      Nbr mine = BWD ? Op::nbr_of(it[0]) : Op::nbr_of(it[3]);
      Nbr from = BWD ? __shfl_down_sync(0xffffffffu, mine, 1) : __shfl_up_sync(0xffffffffu, mine, 1);
      if (BWD) {
        if (lane == 31 && nvalid == 4 && i0 + 4u < g.total) from = Op::nbr_load(p, i0 + 4u);
        nb[3] = from;
#pragma unroll
        for (int k = 0; k < 3; ++k) nb[k] = Op::nbr_of(it[k + 1]);
      } else {
        if (lane == 0 && nvalid > 0 && i0 > 0u) from = Op::nbr_load(p, i0 - 1u);
        nb[0] = from;
#pragma unroll
        for (int k = 1; k < 4; ++k) nb[k] = Op::nbr_of(it[k - 1]);
      }
    }
  }

  // a2: coefficients in registers.
  Aff<V> c[4];
  Aux aux[4] = {};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k < nvalid) {
      const bool row_edge = BWD ? (t == g.T - 1u) : (t == 0u);
      c[k] = Op::coef(p, it[k], nb[k], row_edge, n, i0 + k, aux[k]);
    } else {
      c[k] = aff_identity<V>();
    }
    if (++t == g.T) {
      t = 0;
      ++n;
    }
  }

  // a4: sequential composite of the thread's 4 steps, in dependency order.
  Aff<V> agg;
  if (BWD) {
    agg = compose(c[2], c[3]);
    agg = compose(c[1], agg);
    agg = compose(c[0], agg);
  } else {
    agg = compose(c[1], c[0]);
    agg = compose(c[2], agg);
    agg = compose(c[3], agg);
  }

  // a5: warp scan.
  const Aff<V> inc = warp_inclusive_scan<BWD>(agg, lane);
  const Aff<V> exc = warp_exclusive_from_inclusive<BWD>(inc, lane, 31);
  if (BWD ? lane == 0 : lane == 31) s_wagg[warp] = inc;
  __syncthreads();

  // a6 (+ a7): warp 0 scans the warp aggregates; with look-back, its lane 0
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
        bool edge_closed;
        if (BWD)
          edge_closed = (min(cbase + L, g.total) % g.T) == 0u;
        else
          edge_closed = (cbase % g.T) == 0u;
        carry = decoupled_lookback<BWD, V>(g.lb, chunk, g.nchunks, epoch, ticket, Aff<V>{ca, cb},
                                           edge_closed);
      }
      carry = __shfl_sync(0xffffffffu, carry, 0);
    }
    if (lane < W) s_wcarry[lane] = apply(wexc, carry);
  }
  __syncthreads();

  // a8: re-sweep the thread's steps from the carry and write the outputs.
  V x = apply(exc, s_wcarry[warp]);
  V xs[4], xd[4];
  if (BWD) {
#pragma unroll
    for (int k = 3; k >= 0; --k) {
      xd[k] = x;
      x = apply(c[k], x);
      xs[k] = x;
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      xd[k] = x;
      x = apply(c[k], x);
      xs[k] = x;
    }
  }
  Op::emit(p, i0, nvalid, g.vec != 0u, it, xs, xd, aux);

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
