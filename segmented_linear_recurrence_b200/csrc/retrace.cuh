// retrace.cuh -- Retrace(lambda) coefficient builder with an on-chip reduction
// of E_pi Q over the action dimension.
//
// "rl-triton: High-Performance Triton GPU Kernels for Reinforcement Learning
// Credit Assignment" (gist.science technical summary), Resultaten: Retrace is
// the estimator with the heaviest per-step work (it loads the action
// probabilities) and, in the pages' row-per-program design, runs short of
// registers beyond T = 2048.  Here the per-step action rows never sit in
// registers: each block stages its chunk's q and pi rows in shared memory
// with TMA bulk copies (cp.async.bulk, completion on an mbarrier, no
// multicast), a ring of `stages` sub-tiles deep, and reduces each step's row
// to three scalars -- E_t = sum_a pi[t,a] q[t,a], q_t = q[t, a_t] and
// c_t = lambda min(1, pi[t, a_t] / mu_t) -- kept in shared memory for the scan
// (Munos et al. 2016).  Step t's coefficients read those of step t+1 only:
//   a_t = gamma c_{t+1} cont_t,
//   b_t = r_t + gamma cont_t (E_{t+1} - c_{t+1} q_{t+1}) + gamma (1 - cont_t) nv_t.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "async_copy.cuh"
#include "estimators.cuh"
#include "scan_core.cuh"
#include "scan_kernel.cuh"

namespace rlscan {

// 4 consecutive steps per thread (128-bit accesses when aligned).
__device__ __forceinline__ void load4(const float *__restrict__ p, uint32_t i0, int nvalid, bool vec,
                                      float (&v)[4]) {
  if (vec && nvalid == 4) {
    float4 t = __ldcs(reinterpret_cast<const float4 *>(p + i0));
    v[0] = t.x;
    v[1] = t.y;
    v[2] = t.z;
    v[3] = t.w;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = k < nvalid ? p[i0 + k] : 0.0f;
  }
}

// Four flag bytes packed little-endian into one word (byte k = step i0+k).
__device__ __forceinline__ uint32_t load4_flags(const uint8_t *__restrict__ p, uint32_t i0, int nvalid,
                                                bool vec) {
  if (p == nullptr) return 0u;
  if (vec && nvalid == 4) return __ldcs(reinterpret_cast<const unsigned int *>(p + i0));
  uint32_t w = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k < nvalid) w |= uint32_t(p[i0 + k]) << (8 * k);
  return w;
}

// Stores the steps whose bit is set in `valid` (bit k: step i0 + k).
__device__ __forceinline__ void store4(float *__restrict__ p, uint32_t i0, uint32_t valid, bool vec,
                                       const float (&v)[4]) {
  if (vec && valid == 0xfu) {
    __stcs(reinterpret_cast<float4 *>(p + i0), make_float4(v[0], v[1], v[2], v[3]));
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if ((valid >> k) & 1u) p[i0 + k] = v[k];
  }
}

// Flag bits of step k: bit 0 terminated, bit 1 truncated.
__device__ __forceinline__ uint32_t step_flags(uint32_t term4, uint32_t trunc4, int k) {
  return (((term4 >> (8 * k)) & 0xffu) ? 1u : 0u) | (((trunc4 >> (8 * k)) & 0xffu) ? 2u : 0u);
}

// Successor value of a backward step (boundary semantics).
__device__ __forceinline__ float successor_value(uint32_t fl, bool row_end, float next,
                                                 const float *__restrict__ tv,
                                                 const float *__restrict__ boot, uint32_t n,
                                                 uint32_t i, bool &cont) {
  cont = false;
  if (fl & 1u) return 0.0f;
  if (fl & 2u) return __ldg(tv + i);
  if (row_end) return boot ? __ldg(boot + n) : 0.0f;
  cont = true;
  return next;
}

struct RetraceOp {
  using V = float;
  static constexpr bool kBackward = true, kNeedsNbr = true, kPrologue = true;
  struct Args {
    const float *q, *pi, *mu, *r, *boot, *tv;
    const int32_t *act;
    const uint8_t *term, *trunc;
    float *out;
    uint32_t A;
    uint32_t sub_steps;  // steps per staged sub-tile (multiple of 4, <= block size)
    uint32_t stages;     // ring depth
    uint32_t tma;        // 1: q / pi are 16-byte aligned at this launch's base
    float gamma, lambda;
  };
  struct Item {
    float r;
    uint32_t fl;
  };
  struct Nbr {
    float e, qa, c;
  };

  // Dynamic shared memory layout for a chunk of L steps:
  //   float E[L + 1], Qa[L + 1], C[L + 1]   (index L: first step after the chunk)
  //   stages x { float q[S * A], pi[S * A] }
  //   stages x uint64_t mbarrier
  static __host__ __device__ inline uint32_t scalars_bytes(uint32_t L) {
    return ((3u * (L + 1u) * 4u) + 15u) & ~15u;
  }
  static __host__ __device__ inline uint32_t smem_bytes(uint32_t L, uint32_t S, uint32_t A,
                                                        uint32_t stages) {
    return scalars_bytes(L) + stages * 2u * S * A * 4u + stages * 8u;
  }

  static __device__ __forceinline__ void load(const Args &p, uint32_t i0, int nv, bool vec,
                                              Item (&it)[4]) {
    float r[4];
    load4(p.r, i0, nv, vec, r);
    uint32_t te = load4_flags(p.term, i0, nv, vec), tr = load4_flags(p.trunc, i0, nv, vec);
#pragma unroll
    for (int k = 0; k < 4; ++k) it[k] = Item{r[k], step_flags(te, tr, k)};
  }

  static __device__ __forceinline__ Nbr nbr_smem(const unsigned char *smem, uint32_t L,
                                                 uint32_t local) {
    const float *sE = reinterpret_cast<const float *>(smem);
    return Nbr{sE[local], sE[(L + 1) + local], sE[2 * (L + 1) + local]};
  }

  // `cont`, `nv`: from successor_value() (loaded ahead of the staging).
  static __device__ __forceinline__ Aff<float> coef(const Args &p, const Item &it, const Nbr &nx, bool cont,
                                                    float nv) {
    if (cont) return Aff<float>{p.gamma * nx.c, fmaf(p.gamma, fmaf(-nx.c, nx.qa, nx.e), it.r)};
    return Aff<float>{0.0f, fmaf(p.gamma, nv, it.r)};
  }

  static __device__ __forceinline__ void emit(const Args &p, uint32_t i0, uint32_t valid, bool vec,
                                              const float (&x)[4]) {
    store4(p.out, i0, valid, vec, x);
  }

  // E, q_a and c of one step from its staged rows (act, mu: the step's
  // action and behaviour probability, loaded ahead).
  static __device__ __forceinline__ void reduce_step(const Args &p, const float *qrow,
                                                     const float *prow, int32_t act, float mu, float &e,
                                                     float &qa, float &c) {
    const uint32_t A = p.A;
    float acc = 0.0f;
    if ((A & 1u) == 0u) {
      const float2 *q2 = reinterpret_cast<const float2 *>(qrow);
      const float2 *p2 = reinterpret_cast<const float2 *>(prow);
      for (uint32_t a = 0; a < A / 2u; ++a) {
        float2 qq = q2[a], pp = p2[a];
        acc = fmaf(pp.x, qq.x, acc);
        acc = fmaf(pp.y, qq.y, acc);
      }
    } else {
      for (uint32_t a = 0; a < A; ++a) acc = fmaf(prow[a], qrow[a], acc);
    }
    float qv = 0.0f, pv = 0.0f;
    if (act >= 0 && uint32_t(act) < A) {
      qv = qrow[act];
      pv = prow[act];
    } else {
      record_status(kDevStatusInvalidArg);
    }
    e = acc;
    qa = qv;
    c = p.lambda * fminf(1.0f, pv / mu);
  }

  // Fill E / Qa / C for the staged steps [cbase, cbase + Lc) (Lc <= L, cbase
  // a multiple of 4) and, if `with_next`, for the first step after them.
  // Ends with a block barrier.  `before_wait()` runs once every copy and load
  // of the prologue is in flight, before its first wait.
  template <class Hook>
  static __device__ void prologue(const Args &p, uint32_t cbase, uint32_t Lc, uint32_t L, bool with_next,
                                  unsigned char *smem, int tid, int nthreads, uint64_t timeout_ns,
                                  Hook before_wait) {
    float *sE = reinterpret_cast<float *>(smem);
    float *sQ = sE + (L + 1);
    float *sC = sQ + (L + 1);
    const uint32_t A = p.A, S = p.sub_steps, NS = p.stages;
    float *ring = reinterpret_cast<float *>(smem + scalars_bytes(L));
    const uint32_t stage_floats = 2u * S * A;
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + NS * stage_floats);
    const uint32_t nsub = (Lc + S - 1u) / S;
    const bool use_tma = p.tma != 0u;
    auto full = [&](uint32_t j) { return (j + 1u) * S <= Lc; };

    // Action and behaviour probability of the steps this thread reduces in
    // the first kAhead sub-tiles: loaded before any wait, so their latency
    // hides behind the staging copies.
    constexpr uint32_t kAhead = 4;
    int32_t act_ahead[kAhead];
    float mu_ahead[kAhead];
#pragma unroll
    for (uint32_t j = 0; j < kAhead; ++j) {
      const uint32_t local = j * S + uint32_t(tid);
      const bool mine = j < nsub && uint32_t(tid) < S && local < Lc;
      act_ahead[j] = mine ? __ldg(p.act + cbase + local) : 0;
      mu_ahead[j] = mine ? __ldg(p.mu + cbase + local) : 1.0f;
    }

    if (use_tma) {
      if (tid == 0) {
        for (uint32_t s = 0; s < NS; ++s) mbar_init(&bars[s], 1u);
        fence_mbar_init();
      }
      __syncthreads();
      if (tid == 0) {
        for (uint32_t j = 0; j < min(NS, nsub); ++j) {
          if (!full(j)) break;
          float *dq = ring + (j % NS) * stage_floats;
          const uint32_t bytes = S * A * 4u;
          const size_t off = size_t(cbase + j * S) * A;
          mbar_arrive_expect_tx(&bars[j % NS], 2u * bytes);
          bulk_copy_g2s(dq, p.q + off, bytes, &bars[j % NS]);
          bulk_copy_g2s(dq + S * A, p.pi + off, bytes, &bars[j % NS]);
        }
      }
    }

    // The step after the chunk (its E, q_a, c feed the chunk's last step):
    // one warp reduces it straight from global memory.
    if (tid < 32 && with_next) {
      const uint32_t step = cbase + Lc;
      const size_t off = size_t(step) * A;
      float part = 0.0f;
      for (uint32_t a = tid; a < A; a += 32u) part = fmaf(__ldg(p.pi + off + a), __ldg(p.q + off + a), part);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (tid == 0) {
        const int32_t act = __ldg(p.act + step);
        const float mu = __ldg(p.mu + step);
        float qv = 0.0f, pv = 0.0f;
        if (act >= 0 && uint32_t(act) < A) {
          qv = __ldg(p.q + off + act);
          pv = __ldg(p.pi + off + act);
        } else {
          record_status(kDevStatusInvalidArg);
        }
        sE[Lc] = part;
        sQ[Lc] = qv;
        sC[Lc] = p.lambda * fminf(1.0f, pv / mu);
      }
    }

    before_wait();
    for (uint32_t j = 0; j < nsub; ++j) {
      const uint32_t stage = j % NS;
      float *sq = ring + stage * stage_floats;
      float *sp = sq + S * A;
      const uint32_t nst = min(S, Lc - j * S);
      if (use_tma && full(j)) {
        mbar_wait_bounded(&bars[stage], (j / NS) & 1u, timeout_ns);
      } else {
        const size_t off = size_t(cbase + j * S) * A;
        for (uint32_t e = tid; e < nst * A; e += nthreads) {
          sq[e] = __ldg(p.q + off + e);
          sp[e] = __ldg(p.pi + off + e);
        }
        __syncthreads();
      }
      if (uint32_t(tid) < nst) {
        const uint32_t local = j * S + tid;
        int32_t act;
        float mu;
        if (j < kAhead) {
          // select from the registers without dynamic indexing
          act = act_ahead[0];
          mu = mu_ahead[0];
#pragma unroll
          for (uint32_t jj = 1; jj < kAhead; ++jj)
            if (j == jj) {
              act = act_ahead[jj];
              mu = mu_ahead[jj];
            }
        } else {
          act = __ldg(p.act + cbase + local);
          mu = __ldg(p.mu + cbase + local);
        }
        float e, qa, c;
        reduce_step(p, sq + tid * A, sp + tid * A, act, mu, e, qa, c);
        sE[local] = e;
        sQ[local] = qa;
        sC[local] = c;
      }
      __syncthreads();
      if (use_tma && tid == 0 && j + NS < nsub && full(j + NS)) {
        fence_proxy_async_smem();
        const uint32_t jn = j + NS;
        const uint32_t bytes = S * A * 4u;
        const size_t off = size_t(cbase + jn * S) * A;
        mbar_arrive_expect_tx(&bars[stage], 2u * bytes);
        bulk_copy_g2s(sq, p.q + off, bytes, &bars[stage]);
        bulk_copy_g2s(sp, p.pi + off, bytes, &bars[stage]);
      }
    }
  }
};

// One block per chunk: the prologue fills E, q_a, c for the chunk's steps
// (and, with look-back, the step after them) in shared memory, then each
// thread scans 4 consecutive steps; warps and blocks combine as in
// scan_kernel.cuh.  Two plans, as there:
//   LB == false: block b owns the whole rows of the steps [b span, (b + 1)
//     span); its tiles (and the staging) start at that range's first step
//     rounded down to a multiple of 4, and steps outside the range are
//     neither scanned nor stored.
//   LB == true: chunks of L = 4 * BLOCK steps of the flat sequence, taken in
//     dependency order by ticket, chained by the decoupled look-back.
template <int BLOCK, bool LB>
__global__ void __launch_bounds__(BLOCK) retrace_kernel(const RetraceOp::Args p, const ScanGeom g) {
  using Op = RetraceOp;
  using V = float;
  using Item = Op::Item;
  using Nbr = Op::Nbr;
  constexpr int W = BLOCK / 32;
  constexpr uint32_t L = 4u * BLOCK;
  __shared__ Aff<V> s_wagg[W];
  __shared__ V s_wcarry[W];
  __shared__ uint32_t s_ticket, s_epoch;
  extern __shared__ __align__(16) unsigned char dyn_smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const FastDiv fd{g.div_m, g.div_l};
  grid_dependency_wait();
  uint32_t chunk = blockIdx.x, ticket = 0, epoch = 0;
  if constexpr (LB) {
    if (tid == 0 && !draw_ticket(g.lb.hdr, g.nchunks, s_ticket, s_epoch)) record_status(kDevStatusTimeout);
    __syncthreads();
    ticket = s_ticket;
    epoch = s_epoch;
    if (ticket >= g.nchunks) return;  // counter left inconsistent by an aborted launch
    chunk = chunk_of_ticket(g, ticket, true);
  }
  uint32_t lo, hi, base;
  if constexpr (LB) {
    lo = chunk * L;
    hi = min(lo + L, g.total);
    base = lo;
  } else {
    lo = chunk * g.span;
    hi = min(lo + g.span, g.total);
    base = lo & ~3u;
  }

  // The thread's own steps first: their loads are in flight while the
  // prologue stages and reduces the chunk's action rows.
  const uint32_t i0 = base + 4u * uint32_t(tid);
  const int nvalid = i0 < g.total ? int(min(4u, g.total - i0)) : 0;
  uint32_t valid = i0 < hi ? (1u << min(4u, hi - i0)) - 1u : 0u;
  if (i0 < lo) valid &= ~((1u << (lo - i0)) - 1u);
  uint32_t n = 0, t = 0;
  if (valid) {
    n = fd.div(i0);
    t = i0 - n * g.T;
  }
  Item it[4];
  Op::load(p, i0, nvalid, g.vec != 0u, it);
  // Successor values of the thread's boundary steps (trunc_value, bootstrap):
  // fetched while the staging copies are in flight.
  bool cont[4];
  float nvb[4];
  Op::prologue(p, base, hi - base, L, LB && hi < g.total, dyn_smem, tid, BLOCK, g.lb.timeout_ns, [&] {
    uint32_t tt = t, nn = n;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      nvb[k] = 0.0f;
      cont[k] = false;
      if ((valid >> k) & 1u)
        nvb[k] = successor_value(it[k].fl, tt == g.T - 1u, 0.0f, p.tv, p.boot, nn, i0 + k, cont[k]);
      if (++tt == g.T) {
        tt = 0;
        ++nn;
      }
    }
  });
  grid_dependents_launch();
  Nbr nb[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) nb[k] = Op::nbr_smem(dyn_smem, L, 4u * uint32_t(tid) + k + 1u);

  Aff<V> c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) c[k] = ((valid >> k) & 1u) ? Op::coef(p, it[k], nb[k], cont[k], nvb[k]) : aff_identity<V>();
  Aff<V> agg = compose(c[2], c[3]);
  agg = compose(c[1], agg);
  agg = compose(c[0], agg);

  const Aff<V> inc = warp_inclusive_scan<true>(agg, lane);
  const Aff<V> exc = warp_exclusive_from_inclusive<true>(inc, lane, 31);
  if (lane == 0) s_wagg[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const Aff<V> wv = lane < W ? s_wagg[lane] : aff_identity<V>();
    const Aff<V> winc = warp_inclusive_scan<true>(wv, lane);
    const Aff<V> wexc = warp_exclusive_from_inclusive<true>(winc, lane, W - 1);
    V carry = 0.0f;
    if constexpr (LB) {
      const V ca = __shfl_sync(0xffffffffu, winc.a, 0);
      const V cb = __shfl_sync(0xffffffffu, winc.b, 0);
      const bool edge_closed = (hi % g.T) == 0u;
      carry = decoupled_lookback<true, V>(g.lb, chunk, g.nchunks, epoch, ticket, Aff<V>{ca, cb}, edge_closed,
                                          lane);
    }
    if (lane < W) s_wcarry[lane] = apply(wexc, carry);
  }
  __syncthreads();

  V x = apply(exc, s_wcarry[warp]);
  V xs[4];
#pragma unroll
  for (int k = 3; k >= 0; --k) {
    x = apply(c[k], x);
    xs[k] = x;
  }
  Op::emit(p, i0, valid, g.vec != 0u, xs);
}

}  // namespace rlscan
