// estimators.cuh -- per-estimator coefficient builders for the fused scan.
//
// "rl-triton: High-Performance Triton GPU Kernels for Reinforcement Learning
// Credit Assignment" (gist.science technical summary), Methodologie 2, "On-Chip
// Constructie": each kernel loads the raw rollout inputs and builds the
// recurrence coefficients in registers; they are never written to HBM.  Each
// struct below is one estimator: which arrays it streams, how a step's
// (a_t, b_t) follow from them and from the neighbouring step, and which
// outputs it derives from the solved x_t.  The formulas are the estimators'
// original papers' (listed per struct); the boundary rules are Methodologie 3
// of the same page: termination -> successor value 0, truncation ->
// trunc_value, window end -> bootstrap, counted once in the local term.
//
// Interface used by scan_kernel.cuh (all members static __device__):
//   V                value type of the scan (float, or uint32_t for integers)
//   kBackward        true: x_t = b_t + a_t x_{t+1};  false: x_t = b_t + a_t x_{t-1}
//   kNeedsNbr        whether coef() reads the neighbouring step (t+1 / t-1)
//   kPrologue        whether per-step inputs are first reduced into shared memory
//   Args, Item, Nbr, Aux
//   load(args, i0, nvalid, vec, item[4])      4 consecutive steps starting at i0
//   nbr_of(item) / nbr_load(args, i)          what a step gives its neighbour
//   coef(args, item, nbr, row_edge, n, i, aux) -> Aff<V>
//   emit(args, i0, nvalid, vec, item, x, x_dep, aux)
//     x[k] is the solved value at step i0+k and x_dep[k] the value it was
//     derived from (x_{t+1} backward, x_{t-1} forward).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "scan_core.cuh"

namespace rlscan {

// ---------------------------------------------------------------------------
// Streaming load / store of 4 consecutive steps.  `vec` means the array is
// 16-byte aligned (4-byte for flags) at every thread's first step, so a single
// 128-bit (32-bit) access moves all four; otherwise elements are moved one by
// one.  Steps past the end (k >= nvalid) are neither read nor written.
// ---------------------------------------------------------------------------
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

__device__ __forceinline__ void load4(const int32_t *__restrict__ p, uint32_t i0, int nvalid,
                                      bool vec, uint32_t (&v)[4]) {
  if (vec && nvalid == 4) {
    int4 t = __ldcs(reinterpret_cast<const int4 *>(p + i0));
    v[0] = uint32_t(t.x);
    v[1] = uint32_t(t.y);
    v[2] = uint32_t(t.z);
    v[3] = uint32_t(t.w);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = k < nvalid ? uint32_t(p[i0 + k]) : 0u;
  }
}

// Four flag bytes packed little-endian into one word (byte k = step i0+k).
__device__ __forceinline__ uint32_t load4_flags(const uint8_t *__restrict__ p, uint32_t i0,
                                                int nvalid, bool vec) {
  if (p == nullptr) return 0u;
  if (vec && nvalid == 4) return __ldcs(reinterpret_cast<const unsigned int *>(p + i0));
  uint32_t w = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k < nvalid) w |= uint32_t(p[i0 + k]) << (8 * k);
  return w;
}

__device__ __forceinline__ void store4(float *__restrict__ p, uint32_t i0, int nvalid, bool vec,
                                       const float (&v)[4]) {
  if (vec && nvalid == 4) {
    __stcs(reinterpret_cast<float4 *>(p + i0), make_float4(v[0], v[1], v[2], v[3]));
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < nvalid) p[i0 + k] = v[k];
  }
}

__device__ __forceinline__ void store4(int32_t *__restrict__ p, uint32_t i0, int nvalid, bool vec,
                                       const uint32_t (&v)[4]) {
  if (vec && nvalid == 4) {
    __stcs(reinterpret_cast<int4 *>(p + i0),
           make_int4(int(v[0]), int(v[1]), int(v[2]), int(v[3])));
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < nvalid) p[i0 + k] = int32_t(v[k]);
  }
}

// Flag bits of step k: bit 0 terminated, bit 1 truncated.
__device__ __forceinline__ uint32_t step_flags(uint32_t term4, uint32_t trunc4, int k) {
  return (((term4 >> (8 * k)) & 0xffu) ? 1u : 0u) | (((trunc4 >> (8 * k)) & 0xffu) ? 2u : 0u);
}

// Successor value of a backward step (boundary semantics).  `next` is the
// value of step t+1, used only when the step continues inside the window.
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

struct NoNbr {};
struct NoAux {};

// ---------------------------------------------------------------------------
// GAE (Schulman et al. 2016): x = advantage, a = gamma lambda cont,
// b = r + gamma nv - v.  Outputs advantages = x, returns = x + v.
// ---------------------------------------------------------------------------
struct GaeOp {
  using V = float;
  static constexpr bool kBackward = true, kNeedsNbr = true, kPrologue = false;
  struct Args {
    const float *r, *v, *boot, *tv;
    const uint8_t *term, *trunc;
    float *adv, *ret;
    float gamma, gl;
  };
  struct Item {
    float r, v;
    uint32_t fl;
  };
  using Nbr = float;
  using Aux = NoAux;
  static __device__ __forceinline__ void load(const Args &p, uint32_t i0, int nv, bool vec,
                                              Item (&it)[4]) {
    float r[4], v[4];
    load4(p.r, i0, nv, vec, r);
    load4(p.v, i0, nv, vec, v);
    uint32_t te = load4_flags(p.term, i0, nv, vec), tr = load4_flags(p.trunc, i0, nv, vec);
#pragma unroll
    for (int k = 0; k < 4; ++k) it[k] = Item{r[k], v[k], step_flags(te, tr, k)};
  }
  static __device__ __forceinline__ Nbr nbr_of(const Item &it) { return it.v; }
  static __device__ __forceinline__ Nbr nbr_load(const Args &p, uint32_t i) { return __ldg(p.v + i); }
  static __device__ __forceinline__ Aff<float> coef(const Args &p, const Item &it, Nbr next,
                                                    bool row_end, uint32_t n, uint32_t i, Aux &) {
    bool cont;
    float nv = successor_value(it.fl, row_end, next, p.tv, p.boot, n, i, cont);
    return Aff<float>{cont ? p.gl : 0.0f, fmaf(p.gamma, nv, it.r) - it.v};
  }
  static __device__ __forceinline__ void emit(const Args &p, uint32_t i0, int nv, bool vec,
                                              const Item (&it)[4], const float (&x)[4],
                                              const float (&)[4], const Aux (&)[4]) {
    store4(p.adv, i0, nv, vec, x);
    if (p.ret) {
      float ret[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) ret[k] = x[k] + it[k].v;
      store4(p.ret, i0, nv, vec, ret);
    }
  }
};

// ---------------------------------------------------------------------------
// TD(lambda) returns: a = gamma lambda cont, b = r + gamma (1 - lambda) v_{t+1}
// inside an episode, b = r + gamma nv at a boundary.  Output x.
// ---------------------------------------------------------------------------
struct TdLambdaOp {
  using V = float;
  static constexpr bool kBackward = true, kNeedsNbr = true, kPrologue = false;
  struct Args {
    const float *r, *v, *boot, *tv;
    const uint8_t *term, *trunc;
    float *out;
    float gamma, gl, g1l;  // gamma, gamma*lambda, gamma*(1-lambda)
  };
  struct Item {
    float r;
    uint32_t fl;
    float v;
  };
  using Nbr = float;
  using Aux = NoAux;
  static __device__ __forceinline__ void load(const Args &p, uint32_t i0, int nv, bool vec,
                                              Item (&it)[4]) {
    float r[4], v[4];
    load4(p.r, i0, nv, vec, r);
    load4(p.v, i0, nv, vec, v);
    uint32_t te = load4_flags(p.term, i0, nv, vec), tr = load4_flags(p.trunc, i0, nv, vec);
#pragma unroll
    for (int k = 0; k < 4; ++k) it[k] = Item{r[k], step_flags(te, tr, k), v[k]};
  }
  static __device__ __forceinline__ Nbr nbr_of(const Item &it) { return it.v; }
  static __device__ __forceinline__ Nbr nbr_load(const Args &p, uint32_t i) { return __ldg(p.v + i); }
  static __device__ __forceinline__ Aff<float> coef(const Args &p, const Item &it, Nbr next,
                                                    bool row_end, uint32_t n, uint32_t i, Aux &) {
    bool cont;
    float nv = successor_value(it.fl, row_end, next, p.tv, p.boot, n, i, cont);
    return cont ? Aff<float>{p.gl, fmaf(p.g1l, nv, it.r)} : Aff<float>{0.0f, fmaf(p.gamma, nv, it.r)};
  }
  static __device__ __forceinline__ void emit(const Args &p, uint32_t i0, int nv, bool vec,
                                              const Item (&)[4], const float (&x)[4],
                                              const float (&)[4], const Aux (&)[4]) {
    store4(p.out, i0, nv, vec, x);
  }
};

// ---------------------------------------------------------------------------
// Discounted return: a = gamma cont, b = r (+ gamma nv at a boundary).
// bootstrap may be NULL (zero at the window end).  Output x.
// ---------------------------------------------------------------------------
struct DiscountedOp {
  using V = float;
  static constexpr bool kBackward = true, kNeedsNbr = false, kPrologue = false;
  struct Args {
    const float *r, *boot, *tv;
    const uint8_t *term, *trunc;
    float *out;
    float gamma;
  };
  struct Item {
    float r;
    uint32_t fl;
  };
  using Nbr = NoNbr;
  using Aux = NoAux;
  static __device__ __forceinline__ void load(const Args &p, uint32_t i0, int nv, bool vec,
                                              Item (&it)[4]) {
    float r[4];
    load4(p.r, i0, nv, vec, r);
    uint32_t te = load4_flags(p.term, i0, nv, vec), tr = load4_flags(p.trunc, i0, nv, vec);
#pragma unroll
    for (int k = 0; k < 4; ++k) it[k] = Item{r[k], step_flags(te, tr, k)};
  }
  static __device__ __forceinline__ Nbr nbr_of(const Item &) { return NoNbr{}; }
  static __device__ __forceinline__ Nbr nbr_load(const Args &, uint32_t) { return NoNbr{}; }
  static __device__ __forceinline__ Aff<float> coef(const Args &p, const Item &it, Nbr,
                                                    bool row_end, uint32_t n, uint32_t i, Aux &) {
    bool cont;
    float nv = successor_value(it.fl, row_end, 0.0f, p.tv, p.boot, n, i, cont);
    return cont ? Aff<float>{p.gamma, it.r} : Aff<float>{0.0f, fmaf(p.gamma, nv, it.r)};
  }
  static __device__ __forceinline__ void emit(const Args &p, uint32_t i0, int nv, bool vec,
                                              const Item (&)[4], const float (&x)[4],
                                              const float (&)[4], const Aux (&)[4]) {
    store4(p.out, i0, nv, vec, x);
  }
};

// ---------------------------------------------------------------------------
// V-trace (Espeholt et al. 2018) with lambda-scaled traces, on d = vs - v:
// rho = min(rho_bar, e^lr), c = lambda min(c_bar, e^lr),
// a = gamma c cont, b = rho (r + gamma nv - v).  Outputs vs = x + v and
// pg_adv = rho (r + gamma (nv + [cont] x_{t+1}) - v), since vs_{t+1} =
// v_{t+1} + d_{t+1} inside an episode and nv at a boundary.
// ---------------------------------------------------------------------------
struct VtraceOp {
  using V = float;
  static constexpr bool kBackward = true, kNeedsNbr = true, kPrologue = false;
  struct Args {
    const float *lr, *r, *v, *boot, *tv;
    const uint8_t *term, *trunc;
    float *vs, *pg;
    float gamma, lambda, rho_bar, c_bar;
  };
  struct Item {
    float lr, r, v;
    uint32_t fl;
  };
  using Nbr = float;
  struct Aux {
    float rho, nv, contf;
  };
  static __device__ __forceinline__ void load(const Args &p, uint32_t i0, int nv, bool vec,
                                              Item (&it)[4]) {
    float lr[4], r[4], v[4];
    load4(p.lr, i0, nv, vec, lr);
    load4(p.r, i0, nv, vec, r);
    load4(p.v, i0, nv, vec, v);
    uint32_t te = load4_flags(p.term, i0, nv, vec), tr = load4_flags(p.trunc, i0, nv, vec);
#pragma unroll
    for (int k = 0; k < 4; ++k) it[k] = Item{lr[k], r[k], v[k], step_flags(te, tr, k)};
  }
  static __device__ __forceinline__ Nbr nbr_of(const Item &it) { return it.v; }
  static __device__ __forceinline__ Nbr nbr_load(const Args &p, uint32_t i) { return __ldg(p.v + i); }
  static __device__ __forceinline__ Aff<float> coef(const Args &p, const Item &it, Nbr next,
                                                    bool row_end, uint32_t n, uint32_t i,
                                                    Aux &aux) {
    bool cont;
    float nv = successor_value(it.fl, row_end, next, p.tv, p.boot, n, i, cont);
    float ratio = expf(it.lr);
    float rho = fminf(p.rho_bar, ratio);
    float c = p.lambda * fminf(p.c_bar, ratio);
    aux = Aux{rho, nv, cont ? 1.0f : 0.0f};
    return Aff<float>{cont ? p.gamma * c : 0.0f, rho * (fmaf(p.gamma, nv, it.r) - it.v)};
  }
  static __device__ __forceinline__ void emit(const Args &p, uint32_t i0, int nv, bool vec,
                                              const Item (&it)[4], const float (&x)[4],
                                              const float (&xn)[4], const Aux (&aux)[4]) {
    float vs[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) vs[k] = x[k] + it[k].v;
    store4(p.vs, i0, nv, vec, vs);
    if (p.pg) {
      float pg[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        pg[k] = aux[k].rho * (fmaf(p.gamma, fmaf(aux[k].contf, xn[k], aux[k].nv), it[k].r) - it[k].v);
      store4(p.pg, i0, nv, vec, pg);
    }
  }
};

// ---------------------------------------------------------------------------
// Accumulating eligibility trace, forward: a = gamma lambda (1 - done_{t-1}),
// b = g; the first step of a row folds in the carried-in trace:
// b = g + gamma lambda init[n], a = 0.  Output x.
// ---------------------------------------------------------------------------
struct EligOp {
  using V = float;
  static constexpr bool kBackward = false, kNeedsNbr = true, kPrologue = false;
  struct Args {
    const float *g, *init;
    const uint8_t *term, *trunc;
    float *out;
    float gl;
  };
  struct Item {
    float g;
    uint32_t fl;
  };
  using Nbr = uint32_t;  // previous step done (0/1)
  using Aux = NoAux;
  static __device__ __forceinline__ void load(const Args &p, uint32_t i0, int nv, bool vec,
                                              Item (&it)[4]) {
    float g[4];
    load4(p.g, i0, nv, vec, g);
    uint32_t te = load4_flags(p.term, i0, nv, vec), tr = load4_flags(p.trunc, i0, nv, vec);
#pragma unroll
    for (int k = 0; k < 4; ++k) it[k] = Item{g[k], step_flags(te, tr, k)};
  }
  static __device__ __forceinline__ Nbr nbr_of(const Item &it) { return it.fl ? 1u : 0u; }
  static __device__ __forceinline__ Nbr nbr_load(const Args &p, uint32_t i) {
    return ((p.term != nullptr && p.term[i] != 0) || (p.trunc != nullptr && p.trunc[i] != 0)) ? 1u : 0u;
  }
  static __device__ __forceinline__ Aff<float> coef(const Args &p, const Item &it, Nbr prev_done,
                                                    bool row_start, uint32_t n, uint32_t, Aux &) {
    if (row_start) return Aff<float>{0.0f, p.init ? fmaf(p.gl, __ldg(p.init + n), it.g) : it.g};
    return Aff<float>{prev_done ? 0.0f : p.gl, it.g};
  }
  static __device__ __forceinline__ void emit(const Args &p, uint32_t i0, int nv, bool vec,
                                              const Item (&)[4], const float (&x)[4],
                                              const float (&)[4], const Aux (&)[4]) {
    store4(p.out, i0, nv, vec, x);
  }
};

// ---------------------------------------------------------------------------
// Episodic inclusive prefix sum, forward, exact in uint32 (two's complement):
// a = 0 at a row start or after a done step, else 1; b = x.
// ---------------------------------------------------------------------------
struct PrefixSumOp {
  using V = uint32_t;
  static constexpr bool kBackward = false, kNeedsNbr = true, kPrologue = false;
  struct Args {
    const int32_t *x;
    const uint8_t *term, *trunc;
    int32_t *out;
  };
  struct Item {
    uint32_t x;
    uint32_t fl;
  };
  using Nbr = uint32_t;
  using Aux = NoAux;
  static __device__ __forceinline__ void load(const Args &p, uint32_t i0, int nv, bool vec,
                                              Item (&it)[4]) {
    uint32_t x[4];
    load4(p.x, i0, nv, vec, x);
    uint32_t te = load4_flags(p.term, i0, nv, vec), tr = load4_flags(p.trunc, i0, nv, vec);
#pragma unroll
    for (int k = 0; k < 4; ++k) it[k] = Item{x[k], step_flags(te, tr, k)};
  }
  static __device__ __forceinline__ Nbr nbr_of(const Item &it) { return it.fl ? 1u : 0u; }
  static __device__ __forceinline__ Nbr nbr_load(const Args &p, uint32_t i) {
    return ((p.term != nullptr && p.term[i] != 0) || (p.trunc != nullptr && p.trunc[i] != 0)) ? 1u : 0u;
  }
  static __device__ __forceinline__ Aff<uint32_t> coef(const Args &, const Item &it, Nbr prev_done,
                                                       bool row_start, uint32_t, uint32_t, Aux &) {
    return Aff<uint32_t>{(row_start || prev_done) ? 0u : 1u, it.x};
  }
  static __device__ __forceinline__ void emit(const Args &p, uint32_t i0, int nv, bool vec,
                                              const Item (&)[4], const uint32_t (&x)[4],
                                              const uint32_t (&)[4], const Aux (&)[4]) {
    store4(p.out, i0, nv, vec, x);
  }
};

}  // namespace rlscan
