// estimators.cuh -- per-estimator coefficient builders for the fused scan.
//
// "rl-triton: High-Performance Triton GPU Kernels for Reinforcement Learning
// Credit Assignment" (gist.science technical summary), Methodologie 2, "On-Chip
// Constructie": each kernel loads the raw rollout inputs and builds the
// recurrence coefficients in registers; they are never written to HBM.  Each
// struct below is one estimator: which arrays it streams, how a step's
// (a_t, b_t) follow from them and from the neighbouring step, and which
// outputs derive from the solved x_t.  The formulas are the estimators'
// original papers' (named per struct); the boundary rules are Methodologie 3
// of the same page: termination -> successor value 0, truncation ->
// trunc_value, window end -> bootstrap, counted once in the local term.
//
// A thread owns a tile of K consecutive steps (K = 8, or 16 where measured
// faster): one 256-bit load per 8 steps of an fp32 array, one 64-bit load per
// 8 flag bytes.  Interface used by scan_kernel.cuh
// (all members static __device__):
//   V, kBackward, Args, Raw
//   load(args, tile, fd, lane, total, flags, raw)   given the tile's
//        terminated / truncated masks, issues every load whose address
//        follows from the tile's position: the per-step arrays, the halo step
//        across the lane edge (lane 31 backward / lane 0 forward) and the
//        per-row value (bootstrap / initial trace) of the tile's row edge
//   fetch_boundary(args, tile, raw)      issues the loads that depend on the
//        flags (trunc_value at truncated steps, backward estimators)
//   nbr_of(raw) / halo_of(raw)           the step a neighbouring lane needs
//   coef(args, tile, fd, raw, nbr, c)    fills the 8 coefficients; may keep
//        per-step state in `raw` for emit()
//   emit(args, tile, raw, c, x, xdep)    writes the outputs
// x[k] is the solved value at step k, xdep[k] the one it was derived from
// (x_{t+1} backward, x_{t-1} forward).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "scan_core.cuh"

namespace rlscan {

constexpr int kTile = 8;  // default steps per thread; an estimator may use 16 (Op::K)

// Geometry of one thread's tile of K consecutive steps (K = 8 or 16).
struct Tile {
  uint32_t i0;     // first step (flat, launch-local; a multiple of K)
  int nvalid;      // steps of the tile inside the launch (0..K): these may be loaded
  uint32_t valid;  // bit k: step k belongs to this block (scanned and stored)
  uint32_t n0, t0; // row and time of step i0
  uint32_t edge;   // bit k: step k is on its row's dependency edge
                   //   (backward: t = T-1, forward: t = 0)
  bool fast;       // 256-bit (flags: 64-bit) loads allowed
  bool full;       // ... and all K steps are the block's: 256-bit stores
  bool few_rows;   // T >= K: at most one row edge in the tile
};

// ---------------------------------------------------------------------------
// loads / stores of a tile: 8 steps per 256-bit access (flags: 64-bit)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ld8_raw(const float *a, float *v) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
               : "l"(a));
}
__device__ __forceinline__ void ld8_raw(const int32_t *a, uint32_t *v) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "l"(a));
}
template <int K>
__device__ __forceinline__ void ld_tile(const float *p, const Tile &tl, float (&v)[K]) {
  if (tl.fast) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) ld8_raw(p + tl.i0 + 8 * j, &v[8 * j]);
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = k < tl.nvalid ? __ldg(p + tl.i0 + k) : 0.0f;
  }
}
template <int K>
__device__ __forceinline__ void ld_tile(const int32_t *p, const Tile &tl, uint32_t (&v)[K]) {
  if (tl.fast) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) ld8_raw(p + tl.i0 + 8 * j, &v[8 * j]);
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = k < tl.nvalid ? uint32_t(__ldg(p + tl.i0 + k)) : 0u;
  }
}

// Bit j set iff byte j of the word is nonzero.  Per byte x, (x & 0x7f) + 0x7f
// carries into bit 7 iff x & 0x7f != 0 and never out of the byte; or-ing x
// adds x's own bit 7.  The multiply then moves bits 7, 15, 23, 31 to 28..31
// (shifts of 21, 14, 7, 0; no two partial products share a bit).
__device__ __forceinline__ uint32_t nonzero_bytes4(uint32_t w) {
  const uint32_t hi = (((w & 0x7f7f7f7fu) + 0x7f7f7f7fu) | w) & 0x80808080u;
  return (hi * 0x00204081u) >> 28;
}
template <int K>
__device__ __forceinline__ uint32_t ld_flags(const uint8_t *p, const Tile &tl) {
  if (p == nullptr) return 0u;
  uint32_t m = 0;
  if (tl.fast) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) {
      uint32_t lo, hi;
      asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                   : "=r"(lo), "=r"(hi)
                   : "l"(p + tl.i0 + 8 * j));
      m |= (nonzero_bytes4(lo) | (nonzero_bytes4(hi) << 4)) << (8 * j);
    }
    return m;
  }
#pragma unroll
  for (int k = 0; k < K; ++k)
    if (k < tl.nvalid && __ldg(p + tl.i0 + k) != 0) m |= 1u << k;
  return m;
}

__device__ __forceinline__ void st8_raw(float *a, const float *v) {
  asm volatile("st.global.cs.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(a), "f"(v[0]), "f"(v[1]), "f"(v[2]),
               "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}
__device__ __forceinline__ void st8_raw(int32_t *a, const uint32_t *v) {
  asm volatile("st.global.cs.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(a), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
template <int K>
__device__ __forceinline__ void st_tile(float *p, const Tile &tl, const float (&v)[K]) {
  if (tl.full) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) st8_raw(p + tl.i0 + 8 * j, &v[8 * j]);
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((tl.valid >> k) & 1u) p[tl.i0 + k] = v[k];
  }
}
template <int K>
__device__ __forceinline__ void st_tile(int32_t *p, const Tile &tl, const uint32_t (&v)[K]) {
  if (tl.full) {
#pragma unroll
    for (int j = 0; j < K / 8; ++j) st8_raw(p + tl.i0 + 8 * j, &v[8 * j]);
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((tl.valid >> k) & 1u) p[tl.i0 + k] = int32_t(v[k]);
  }
}

// bf16 storage (bf16 I/O): 8 steps are 16 bytes, one 128-bit access; values
// widen to fp32 exactly (the bf16 bits are the top half of the fp32 bits) and
// narrow with round-to-nearest-even.
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
template <int K>
__device__ __forceinline__ void ld_tile(const __nv_bfloat16 *p, const Tile &tl, float (&v)[K]) {
  if (tl.fast) {
#pragma unroll
    for (int q = 0; q < K / 8; ++q) {
      uint32_t u[4];
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
                   : "l"(p + tl.i0 + 8 * q));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * q + 2 * j] = bf16_lo(u[j]);
        v[8 * q + 2 * j + 1] = bf16_hi(u[j]);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = k < tl.nvalid ? __bfloat162float(__ldg(p + tl.i0 + k)) : 0.0f;
  }
}
template <int K>
__device__ __forceinline__ void st_tile(__nv_bfloat16 *p, const Tile &tl, const float (&v)[K]) {
  if (tl.full) {
#pragma unroll
    for (int q = 0; q < K / 8; ++q) {
      uint32_t u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * q + 2 * j], v[8 * q + 2 * j + 1]);
        u[j] = *reinterpret_cast<const uint32_t *>(&h);
      }
      asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p + tl.i0 + 8 * q), "r"(u[0]), "r"(u[1]),
                   "r"(u[2]), "r"(u[3])
                   : "memory");
    }
  } else {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((tl.valid >> k) & 1u) p[tl.i0 + k] = __float2bfloat16_rn(v[k]);
  }
}
__device__ __forceinline__ float ld1(const float *p) { return __ldg(p); }
__device__ __forceinline__ float ld1(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }

// Per-row value (bootstrap / initial trace) of the tile's row edge, issued
// with the tile's other loads: its address follows from the tile position.
// Tiles of rows shorter than K steps (several edges) load theirs in coef().
template <class E>
__device__ __forceinline__ float edge_value(const E *src, const Tile &tl, const FastDiv &fd) {
  if (src == nullptr || !tl.few_rows || tl.edge == 0u) return 0.0f;
  const uint32_t k = __ffs(tl.edge) - 1u;
  return ld1(src + tl.n0 + fd.div(tl.t0 + k));
}

// Terminated / truncated masks of a tile (bit k: step k).
struct Flags {
  uint32_t term, trunc;
};

// Successor values of the tile's boundary steps (backward estimators), 0 at
// every other step: 0 after termination, trunc_value after truncation, the
// row's bootstrap at a row end (`boot` may be NULL: 0); termination wins over
// truncation, and both over the row end.  trunc_value is the only load whose
// address depends on loaded data; warps without a truncated step skip it.
template <int K, class E = float>
__device__ __forceinline__ void boundary_successors(const E *tv, const E *boot, float ev, const Tile &tl,
                                                    Flags f, const FastDiv &fd, float (&bv)[K]) {
  const uint32_t tr = f.trunc & ~f.term & tl.valid;
  const uint32_t ed = tl.edge & ~f.term & ~f.trunc;
#pragma unroll
  for (int k = 0; k < K; ++k) bv[k] = 0.0f;
  if (__any_sync(0xffffffffu, tr != 0u)) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((tr >> k) & 1u) bv[k] = ld1(tv + tl.i0 + k);
  }
  if (ed != 0u) {  // at most one row end per tile when T >= 8
#pragma unroll
    for (int k = 0; k < K; ++k)
      if ((ed >> k) & 1u) bv[k] = tl.few_rows ? ev : (boot ? ld1(boot + tl.n0 + fd.div(tl.t0 + k)) : 0.0f);
  }
}

// ---------------------------------------------------------------------------
// GAE (Schulman et al. 2016): x = advantage, a = gamma lambda cont,
// b = r + gamma nv - v.  Outputs advantages = x, returns = x + v.  E is the
// storage type of every real array: float, or __nv_bfloat16 (bf16 I/O, fp32
// arithmetic, outputs rounded to nearest even).
// ---------------------------------------------------------------------------
template <int K_ = kTile, class E = float>
struct GaeOpT {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 48, kRegsLookback = 48;  // registers per thread, chosen by measurement
  using V = float;
  static constexpr bool kBackward = true;
  struct Args {
    const E *r, *v, *boot, *tv;
    const uint8_t *term, *trunc;
    E *adv, *ret;
    float gamma, gl;
  };
  struct Raw {
    float r[K], v[K], bv[K];  // bv: successor values at boundary steps
    Flags f;
    float halo;  // v of the step after the tile (lane 31 only)
    float ev;    // bootstrap of the tile's row end
  };
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &fd, int lane,
                                              uint32_t total, Flags f, Raw &w) {
    ld_tile(p.r, tl, w.r);
    ld_tile(p.v, tl, w.v);
    w.f = f;
    w.halo = (lane == 31 && tl.nvalid == K && tl.i0 + uint32_t(K) < total) ? ld1(p.v + tl.i0 + uint32_t(K)) : 0.0f;
    w.ev = edge_value(p.boot, tl, fd);
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w) {
    boundary_successors<K, E>(p.tv, p.boot, w.ev, tl, w.f, fd, w.bv);
  }
  static __device__ __forceinline__ float nbr_of(const Raw &w) { return w.v[0]; }
  static __device__ __forceinline__ float halo_of(const Raw &w) { return w.halo; }
  static __device__ __forceinline__ void coef(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w,
                                              float next7, Aff<float> (&c)[K]) {
    const uint32_t special = w.f.term | w.f.trunc | tl.edge;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const bool sp = (special >> k) & 1u;
      const float next = k < K - 1 ? w.v[k < K - 1 ? k + 1 : K - 1] : next7;
      const float nv = sp ? w.bv[k] : next;
      c[k] = Aff<float>{sp ? 0.0f : p.gl, fmaf(p.gamma, nv, w.r[k]) - w.v[k]};
    }
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &w, const Aff<float> (&)[K],
                                              const float (&x)[K], const float (&)[K]) {
    st_tile(p.adv, tl, x);
    if (p.ret) {
      float ret[K];
#pragma unroll
      for (int k = 0; k < K; ++k) ret[k] = x[k] + w.v[k];
      st_tile(p.ret, tl, ret);
    }
  }
};
using GaeOp = GaeOpT<>;

// ---------------------------------------------------------------------------
// TD(lambda) returns: a = gamma lambda cont, b = r + gamma (1 - lambda) v_{t+1}
// inside an episode, b = r + gamma nv at a boundary.  Output x.
// ---------------------------------------------------------------------------
template <int K_ = kTile>
struct TdLambdaOpT {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 48, kRegsLookback = 48;  // registers per thread, chosen by measurement
  using V = float;
  static constexpr bool kBackward = true;
  struct Args {
    const float *r, *v, *boot, *tv;
    const uint8_t *term, *trunc;
    float *out;
    float gamma, gl, g1l;  // gamma, gamma*lambda, gamma*(1-lambda)
  };
  struct Raw {
    float r[K], v[K], bv[K];
    Flags f;
    float halo, ev;
  };
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &fd, int lane,
                                              uint32_t total, Flags f, Raw &w) {
    ld_tile(p.r, tl, w.r);
    ld_tile(p.v, tl, w.v);
    w.f = f;
    w.halo = (lane == 31 && tl.nvalid == K && tl.i0 + uint32_t(K) < total) ? __ldg(p.v + tl.i0 + uint32_t(K)) : 0.0f;
    w.ev = edge_value(p.boot, tl, fd);
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w) {
    boundary_successors(p.tv, p.boot, w.ev, tl, w.f, fd, w.bv);
  }
  static __device__ __forceinline__ float nbr_of(const Raw &w) { return w.v[0]; }
  static __device__ __forceinline__ float halo_of(const Raw &w) { return w.halo; }
  static __device__ __forceinline__ void coef(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w,
                                              float next7, Aff<float> (&c)[K]) {
    const uint32_t special = w.f.term | w.f.trunc | tl.edge;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const bool sp = (special >> k) & 1u;
      const float next = k < K - 1 ? w.v[k < K - 1 ? k + 1 : K - 1] : next7;
      c[k] = sp ? Aff<float>{0.0f, fmaf(p.gamma, w.bv[k], w.r[k])} : Aff<float>{p.gl, fmaf(p.g1l, next, w.r[k])};
    }
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &, const Aff<float> (&)[K],
                                              const float (&x)[K], const float (&)[K]) {
    st_tile(p.out, tl, x);
  }
};
using TdLambdaOp = TdLambdaOpT<>;

// ---------------------------------------------------------------------------
// Discounted return: a = gamma cont, b = r (+ gamma nv at a boundary).
// bootstrap may be NULL (zero at the window end).  Output x.
// ---------------------------------------------------------------------------
template <int K_ = kTile>
struct DiscountedOpT {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 32, kRegsLookback = 40;  // registers per thread, chosen by measurement
  using V = float;
  static constexpr bool kBackward = true;
  struct Args {
    const float *r, *boot, *tv;
    const uint8_t *term, *trunc;
    float *out;
    float gamma;
  };
  struct Raw {
    float r[K], bv[K];
    Flags f;
    float ev;
  };
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &fd, int, uint32_t,
                                              Flags f, Raw &w) {
    ld_tile(p.r, tl, w.r);
    w.f = f;
    w.ev = edge_value(p.boot, tl, fd);
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w) {
    boundary_successors(p.tv, p.boot, w.ev, tl, w.f, fd, w.bv);
  }
  static __device__ __forceinline__ float nbr_of(const Raw &) { return 0.0f; }
  static __device__ __forceinline__ float halo_of(const Raw &) { return 0.0f; }
  static __device__ __forceinline__ void coef(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w, float,
                                              Aff<float> (&c)[K]) {
    const uint32_t special = w.f.term | w.f.trunc | tl.edge;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const bool sp = (special >> k) & 1u;
      c[k] = Aff<float>{sp ? 0.0f : p.gamma, fmaf(p.gamma, w.bv[k], w.r[k])};
    }
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &, const Aff<float> (&)[K],
                                              const float (&x)[K], const float (&)[K]) {
    st_tile(p.out, tl, x);
  }
};
using DiscountedOp = DiscountedOpT<>;

// ---------------------------------------------------------------------------
// V-trace (Espeholt et al. 2018) with lambda-scaled traces, on d = vs - v:
// rho = min(rho_bar, e^lr), c = lambda min(c_bar, e^lr),
// a = gamma c cont, b = rho (r + gamma nv - v).  Outputs vs = x + v and
// pg_adv = b + gamma rho cont x_{t+1}: rho (r + gamma vs_{t+1} - v) inside an
// episode (vs_{t+1} = v_{t+1} + x_{t+1}), rho (r + gamma nv - v) at a boundary.
// ---------------------------------------------------------------------------
template <int K_ = kTile>
struct VtraceOpT {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 56, kRegsLookback = 48;  // registers per thread, chosen by measurement
  using V = float;
  static constexpr bool kBackward = true;
  struct Args {
    const float *lr, *r, *v, *boot, *tv;
    const uint8_t *term, *trunc;
    float *vs, *pg;
    float gamma, lambda, rho_bar, c_bar;
  };
  struct Raw {
    float lr[K], r[K], v[K], bv[K];  // coef() keeps gamma * rho * cont in lr for emit()
    Flags f;
    float halo, ev;
  };
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &fd, int lane,
                                              uint32_t total, Flags f, Raw &w) {
    ld_tile(p.lr, tl, w.lr);
    ld_tile(p.r, tl, w.r);
    ld_tile(p.v, tl, w.v);
    w.f = f;
    w.halo = (lane == 31 && tl.nvalid == K && tl.i0 + uint32_t(K) < total) ? __ldg(p.v + tl.i0 + uint32_t(K)) : 0.0f;
    w.ev = edge_value(p.boot, tl, fd);
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w) {
    boundary_successors(p.tv, p.boot, w.ev, tl, w.f, fd, w.bv);
  }
  static __device__ __forceinline__ float nbr_of(const Raw &w) { return w.v[0]; }
  static __device__ __forceinline__ float halo_of(const Raw &w) { return w.halo; }
  static __device__ __forceinline__ void coef(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w,
                                              float next7, Aff<float> (&c)[K]) {
    const uint32_t special = w.f.term | w.f.trunc | tl.edge;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const bool sp = (special >> k) & 1u;
      const float next = k < K - 1 ? w.v[k < K - 1 ? k + 1 : K - 1] : next7;
      const float nv = sp ? w.bv[k] : next;
      const float ratio = __expf(w.lr[k]);
      const float rho = fminf(p.rho_bar, ratio);
      const float cc = p.lambda * fminf(p.c_bar, ratio);
      c[k] = Aff<float>{sp ? 0.0f : p.gamma * cc, rho * (fmaf(p.gamma, nv, w.r[k]) - w.v[k])};
      w.lr[k] = sp ? 0.0f : p.gamma * rho;
    }
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &w, const Aff<float> (&c)[K],
                                              const float (&x)[K], const float (&xn)[K]) {
    float o[K];
#pragma unroll
    for (int k = 0; k < K; ++k) o[k] = x[k] + w.v[k];
    st_tile(p.vs, tl, o);
    if (p.pg) {
#pragma unroll
      for (int k = 0; k < K; ++k) o[k] = fmaf(w.lr[k], xn[k], c[k].b);
      st_tile(p.pg, tl, o);
    }
  }
};
using VtraceOp = VtraceOpT<>;

// ---------------------------------------------------------------------------
// Accumulating eligibility trace, forward: a = gamma lambda (1 - done_{t-1}),
// b = g; the first step of a row folds in the carried-in trace:
// b = g + gamma lambda init[n], a = 0.  Output x.
// ---------------------------------------------------------------------------
template <int K_ = kTile>
struct EligOpT {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 56, kRegsLookback = 56;  // registers per thread, chosen by measurement
  using V = float;
  static constexpr bool kBackward = false;
  struct Args {
    const float *g, *init;
    const uint8_t *term, *trunc;
    float *out;
    float gl;
  };
  struct Raw {
    float g[K];
    uint32_t done;  // bit k: step k terminated or truncated
    uint32_t halo;  // done flag of the step before the tile (lane 0 only)
    float ev;       // initial trace of the tile's row start
  };
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &fd, int lane, uint32_t,
                                              Flags f, Raw &w) {
    ld_tile(p.g, tl, w.g);
    w.done = f.term | f.trunc;
    w.halo = 0u;
    if (lane == 0 && tl.i0 > 0u && tl.nvalid > 0)
      w.halo = ((p.term && __ldg(p.term + tl.i0 - 1u)) || (p.trunc && __ldg(p.trunc + tl.i0 - 1u))) ? 1u : 0u;
    w.ev = edge_value(p.init, tl, fd);
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &, const Tile &, const FastDiv &, Raw &) {}
  static __device__ __forceinline__ uint32_t nbr_of(const Raw &w) { return (w.done >> (K - 1)) & 1u; }
  static __device__ __forceinline__ uint32_t halo_of(const Raw &w) { return w.halo; }
  static __device__ __forceinline__ void coef(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w,
                                              uint32_t prev7, Aff<float> (&c)[K]) {
    const uint32_t cut = (((w.done << 1) | prev7) | tl.edge) & ((1u << K) - 1u);  // bit k: a_k = 0
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float b = w.g[k];
      if (((tl.edge >> k) & 1u) && p.init)
        b = fmaf(p.gl, tl.few_rows ? w.ev : __ldg(p.init + tl.n0 + fd.div(tl.t0 + k)), b);
      c[k] = Aff<float>{((cut >> k) & 1u) ? 0.0f : p.gl, b};
    }
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &, const Aff<float> (&)[K],
                                              const float (&x)[K], const float (&)[K]) {
    st_tile(p.out, tl, x);
  }
};
using EligOp = EligOpT<16>;  // 16 steps per thread: measured faster

// ---------------------------------------------------------------------------
// Episodic inclusive prefix sum, forward, exact in uint32 (two's complement):
// a = 0 at a row start or after a done step, else 1; b = x.
// ---------------------------------------------------------------------------
template <int K_ = kTile>
struct PrefixSumOpT {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 56, kRegsLookback = 56;  // registers per thread, chosen by measurement
  using V = uint32_t;
  static constexpr bool kBackward = false;
  struct Args {
    const int32_t *x;
    const uint8_t *term, *trunc;
    int32_t *out;
  };
  struct Raw {
    uint32_t x[K];
    uint32_t done;
    uint32_t halo;
  };
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &, int lane, uint32_t,
                                              Flags f, Raw &w) {
    ld_tile(p.x, tl, w.x);
    w.done = f.term | f.trunc;
    w.halo = 0u;
    if (lane == 0 && tl.i0 > 0u && tl.nvalid > 0)
      w.halo = ((p.term && __ldg(p.term + tl.i0 - 1u)) || (p.trunc && __ldg(p.trunc + tl.i0 - 1u))) ? 1u : 0u;
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &, const Tile &, const FastDiv &, Raw &) {}
  static __device__ __forceinline__ uint32_t nbr_of(const Raw &w) { return (w.done >> (K - 1)) & 1u; }
  static __device__ __forceinline__ uint32_t halo_of(const Raw &w) { return w.halo; }
  static __device__ __forceinline__ void coef(const Args &, const Tile &tl, const FastDiv &, Raw &w, uint32_t prev7,
                                              Aff<uint32_t> (&c)[K]) {
    const uint32_t cut = (((w.done << 1) | prev7) | tl.edge) & ((1u << K) - 1u);
#pragma unroll
    for (int k = 0; k < K; ++k) c[k] = Aff<uint32_t>{((cut >> k) & 1u) ^ 1u, w.x[k]};
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &, const Aff<uint32_t> (&)[K],
                                              const uint32_t (&x)[K], const uint32_t (&)[K]) {
    st_tile(p.out, tl, x);
  }
};
using PrefixSumOp = PrefixSumOpT<16>;  // 16 steps per thread: measured faster

// ---------------------------------------------------------------------------
// Generic affine scan: the pages' unified recurrence with its coefficients
// given (gist.science technical summary, Methodologie 1).  In scan order
// (forward, or backward when BWD) x_t = b_t + a_t x_prev; reset[t] cuts the
// dependency (a = 0, x = b); the row's first step in scan order -- its
// dependency edge -- takes the per-row initial carry in its local term:
// b + a init (init NULL: 0).  The reset flags travel in the flag slot of
// `term`; `trunc` is NULL.
// ---------------------------------------------------------------------------
template <bool BWD, class E = float, int K_ = kTile>
struct AffineOp {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 40, kRegsLookback = 40;  // registers per thread, chosen by measurement
  using V = float;
  static constexpr bool kBackward = BWD;
  struct Args {
    const E *a, *b, *init;        // E: float, or __nv_bfloat16 for bf16 I/O (fp32 arithmetic)
    const uint8_t *term, *trunc;  // term: reset flags (nullable); trunc: NULL
    E *out;
  };
  struct Raw {
    float a[K], b[K];
    Flags f;
    float ev;  // init of the tile's row edge
  };
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &fd, int, uint32_t,
                                              Flags f, Raw &w) {
    ld_tile(p.a, tl, w.a);
    ld_tile(p.b, tl, w.b);
    w.f = f;
    w.ev = edge_value(p.init, tl, fd);
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &, const Tile &, const FastDiv &, Raw &) {}
  static __device__ __forceinline__ float nbr_of(const Raw &) { return 0.0f; }
  static __device__ __forceinline__ float halo_of(const Raw &) { return 0.0f; }
  static __device__ __forceinline__ void coef(const Args &p, const Tile &tl, const FastDiv &fd, Raw &w, float,
                                              Aff<float> (&c)[K]) {
    const uint32_t cut = w.f.term | tl.edge;
    const uint32_t init_at = tl.edge & ~w.f.term;  // edge steps that take the initial carry
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float b = w.b[k];
      if (((init_at >> k) & 1u) && p.init)
        b = fmaf(w.a[k], tl.few_rows ? w.ev : ld1(p.init + tl.n0 + fd.div(tl.t0 + k)), b);
      c[k] = Aff<float>{((cut >> k) & 1u) ? 0.0f : w.a[k], b};
    }
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &, const Aff<float> (&)[K],
                                              const float (&x)[K], const float (&)[K]) {
    st_tile(p.out, tl, x);
  }
};

// ---------------------------------------------------------------------------
// Adjoint of the generic affine scan (its gradient), for upstream gradients
// dy and the forward output x of a scan in direction R (R: backward in t).
// The chain rule through the recurrence is itself an affine scan, run in the
// opposite direction:  g_t = dy_t + a'_t g_nxt,  a'_t = a_nxt unless the
// following step in the forward order (nxt) resets or does not exist; then
// db = g, da_t = g_t x_prv (0 where reset; x_prv = init[n] at the forward
// scan's first step), dinit[n] = a g at that first step (0 if it resets).
// ---------------------------------------------------------------------------
template <bool R, int K_ = kTile>
struct AffineGradOp {
  static constexpr int K = K_;  // steps per thread
  static constexpr int kRegs = 56, kRegsLookback = 56;  // registers per thread: no spills
  using V = float;
  static constexpr bool kBackward = !R;  // the adjoint runs against the forward scan
  struct Args {
    const float *a, *x, *dy, *init;
    const uint8_t *term, *trunc;  // term: reset flags (nullable); trunc: NULL
    float *da, *db, *dinit;       // da, dinit nullable
    uint32_t T;
  };
  struct Raw {
    float a[K], x[K], dy[K];
    Flags f;
    float ahalo;  // effective a (0 where reset) of the dependency neighbour past the tile
    float xhalo;  // x of the neighbour past the tile on the other side
    float iv;     // init of the row whose forward first step is in the tile (T >= 8)
    uint32_t lane;
  };
  // Steps of the tile that are the forward scan's first step of their row.
  static __device__ __forceinline__ uint32_t first_steps(const Tile &tl, uint32_t T) {
    uint32_t e = 0;
    if (tl.few_rows) {
      if (R) {
        const uint32_t rend = T - 1u - tl.t0;
        e = rend < uint32_t(K) ? (1u << rend) : 0u;
      } else {
        const uint32_t s = tl.t0 == 0u ? 0u : T - tl.t0;
        e = s < uint32_t(K) ? (1u << s) : 0u;
      }
    } else {
      uint32_t tt = tl.t0;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if (R ? (tt == T - 1u) : (tt == 0u)) e |= 1u << k;
        if (++tt == T) tt = 0;
      }
    }
    return e & tl.valid;
  }
  static __device__ __forceinline__ void load(const Args &p, const Tile &tl, const FastDiv &fd, int lane,
                                              uint32_t total, Flags f, Raw &w) {
    ld_tile(p.a, tl, w.a);
    ld_tile(p.x, tl, w.x);
    ld_tile(p.dy, tl, w.dy);
    w.f = f;
    w.lane = uint32_t(lane);
    // dependency neighbour past the tile: t+1 (adjoint backward) / t-1 (forward)
    w.ahalo = 0.0f;
    if (!R && lane == 31 && tl.nvalid == K && tl.i0 + uint32_t(K) < total)
      w.ahalo = (p.term && __ldg(p.term + tl.i0 + uint32_t(K))) ? 0.0f : __ldg(p.a + tl.i0 + uint32_t(K));
    if (R && lane == 0 && tl.i0 > 0u && tl.nvalid > 0)
      w.ahalo = (p.term && __ldg(p.term + tl.i0 - 1u)) ? 0.0f : __ldg(p.a + tl.i0 - 1u);
    // the other neighbour, for x_prv: t-1 (R false) / t+1 (R true)
    w.xhalo = 0.0f;
    if (!R && lane == 0 && tl.i0 > 0u && tl.nvalid > 0) w.xhalo = __ldg(p.x + tl.i0 - 1u);
    if (R && lane == 31 && tl.nvalid == K && tl.i0 + uint32_t(K) < total) w.xhalo = __ldg(p.x + tl.i0 + uint32_t(K));
    w.iv = 0.0f;
    const uint32_t fs = first_steps(tl, p.T);
    if (p.init && tl.few_rows && fs) w.iv = __ldg(p.init + tl.n0 + fd.div(tl.t0 + uint32_t(__ffs(fs) - 1)));
  }
  static __device__ __forceinline__ void fetch_boundary(const Args &, const Tile &, const FastDiv &, Raw &) {}
  // a' of the tile's first step in dependency order comes from the neighbour
  static __device__ __forceinline__ float nbr_of(const Raw &w) {
    return R ? (((w.f.term >> (K - 1)) & 1u) ? 0.0f : w.a[K - 1]) : ((w.f.term & 1u) ? 0.0f : w.a[0]);
  }
  static __device__ __forceinline__ float halo_of(const Raw &w) { return w.ahalo; }
  static __device__ __forceinline__ void coef(const Args &, const Tile &tl, const FastDiv &, Raw &w, float nb,
                                              Aff<float> (&c)[K]) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float an;  // effective a of the following step in forward order
      if (R)
        an = k > 0 ? (((w.f.term >> (k - 1)) & 1u) ? 0.0f : w.a[k > 0 ? k - 1 : 0]) : nb;
      else
        an = k < K - 1 ? (((w.f.term >> (k + 1)) & 1u) ? 0.0f : w.a[k < K - 1 ? k + 1 : K - 1]) : nb;
      c[k] = Aff<float>{((tl.edge >> k) & 1u) ? 0.0f : an, w.dy[k]};
    }
  }
  static __device__ __forceinline__ void emit(const Args &p, const Tile &tl, const Raw &w, const Aff<float> (&)[K],
                                              const float (&g)[K], const float (&)[K]) {
    st_tile(p.db, tl, g);
    if (!p.da && !p.dinit) return;
    // x_prv of each step: the other neighbour, by shuffle across the lane edge
    const float mine = R ? w.x[0] : w.x[K - 1];
    float other = R ? __shfl_down_sync(0xffffffffu, mine, 1) : __shfl_up_sync(0xffffffffu, mine, 1);
    if (R ? w.lane == 31u : w.lane == 0u) other = w.xhalo;
    const uint32_t fs = first_steps(tl, p.T);
    float da[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float xp = R ? (k < K - 1 ? w.x[k < K - 1 ? k + 1 : K - 1] : other) : (k > 0 ? w.x[k > 0 ? k - 1 : 0] : other);
      if ((fs >> k) & 1u)
        xp = !p.init ? 0.0f : (tl.few_rows ? w.iv : __ldg(p.init + tl.n0 + (tl.t0 + k) / p.T));
      da[k] = ((w.f.term >> k) & 1u) ? 0.0f : g[k] * xp;
      if (p.dinit && ((fs >> k) & 1u))
        p.dinit[tl.n0 + (tl.t0 + k) / p.T] = ((w.f.term >> k) & 1u) ? 0.0f : w.a[k] * g[k];
    }
    if (p.da) st_tile(p.da, tl, da);
  }
};

}  // namespace rlscan
