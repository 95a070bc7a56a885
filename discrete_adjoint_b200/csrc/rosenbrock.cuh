// rosenbrock.cuh -- pieces shared by the fused replay + reverse sweep kernels
// of the Rosenbrock methods (grad_ros2.cu, grad_ros3.cu, grad_kin8.cu): the
// kernels' arguments, the right-hand sides' vector-Jacobian products, and the
// loss terms and their gradients at the save points.
#pragma once

#include "steps.cuh"

namespace gs {

template <typename T>
struct RosArgs {
  int64_t n;
  const T* p;
  const T* u0;
  const T* h;
  const int32_t* order;
  const int32_t* nsteps;
  const int32_t* save_idx;
  const int32_t* status;
  int32_t nsave;
  int32_t smax;
  int32_t loss_kind;
  const T* target;
  const T* weight;
  T* loss;
  T* dp;
  T* du0;
  T* ck;
  const T* theta;  // [nsave][n] by slot: dense save points (d = 3 systems), or null
};

// ubar += J(u)^T w,  pbar += f_p(u)^T w.
template <typename T, int SYS>
__device__ __forceinline__ void vjp3(const T u[3], const T p[3], const T w[3], T ub[3], T pb[3]) {
  if (SYS == GS_LORENZ) {
    T m = p[0] * w[0];
    ub[0] += fmaT(p[1] - u[2], w[1], fmaT(u[1], w[2], -m));
    ub[1] += fmaT(u[0], w[2], m - w[1]);
    ub[2] -= fmaT(u[0], w[1], p[2] * w[2]);
    pb[0] = fmaT(u[1] - u[0], w[0], pb[0]);
    pb[1] = fmaT(u[0], w[1], pb[1]);
    pb[2] = fmaT(-u[2], w[2], pb[2]);
  } else {
    // f = (k3 y2 y3 - k1 y1, k1 y1 - k3 y2 y3 - k2 y2^2, k2 y2^2)
    T d21 = w[1] - w[0], d12 = w[0] - w[1], d32 = w[2] - w[1];
    ub[0] = fmaT(p[0], d21, ub[0]);
    ub[1] += fmaT(p[2] * u[2], d12, cst<T>(2.0) * (p[1] * u[1]) * d32);
    ub[2] = fmaT(p[2] * u[1], d12, ub[2]);
    pb[0] = fmaT(u[0], d21, pb[0]);
    pb[1] = fmaT(u[1] * u[1], d32, pb[1]);
    pb[2] = fmaT(u[1] * u[2], d12, pb[2]);
  }
}

// Loss terms of one save point (D components at o + c n of target / weight).
template <typename T, int D = 3>
__device__ __forceinline__ void loss_terms(int kind, const T* target, const T* weight, int64_t o, int64_t n,
                                            const T* u, T& L) {
#pragma unroll
  for (int c = 0; c < D; ++c) {
    if (kind == GS_LOSS_SUMSQ) {
      T dl = target ? u[c] - target[o + c * n] : u[c];
      L = fmaT(dl, dl, L);
    } else {
      L = fmaT(weight[o + c * n], u[c], L);
    }
  }
}

template <typename T, int D = 3>
__device__ __forceinline__ void loss_grad(int kind, const T* target, const T* weight, int64_t o, int64_t n,
                                           const T* u, T* lam) {
#pragma unroll
  for (int c = 0; c < D; ++c) {
    if (kind == GS_LOSS_SUMSQ)
      lam[c] = fmaT(cst<T>(2.0), target ? u[c] - target[o + c * n] : u[c], lam[c]);
    else
      lam[c] += weight[o + c * n];
  }
}

// Save points of step st (save_idx = st + 1), forward: their loss terms.  A
// landing record has at most one, at the step's end u_{st+1}; a dense one
// (theta) any number, each read off the cubic Hermite interpolant of the step
// on u_st, u_{st+1} and their slopes (the floating-point contract's order, as
// in the recorder's dense solve).
template <typename T, int SYS>
__device__ __forceinline__ void save_points_fwd(const RosArgs<T>& a, int64_t i, int64_t j, int st, const T p[3],
                                                const T us[3], const T un[3], T h, int& kk, int& next, T& L) {
  const int64_t n = a.n;
  bool slopes = false;
  T fs[3], fn[3];
  while (st + 1 == next) {
    T ut[3] = {un[0], un[1], un[2]};
    if (a.theta) {
      const T th = a.theta[(int64_t)kk * n + j];
      if (th != cst<T>(1.0)) {
        if (!slopes) {
          rhs3<T, SYS>(us, p, fs);
          rhs3<T, SYS>(un, p, fn);
          slopes = true;
        }
        const HermiteW<T> w = hermite_w(th);
#pragma unroll
        for (int c = 0; c < 3; ++c) ut[c] = hermite_c(w, us[c], un[c], fs[c], fn[c], h);
      }
    }
    loss_terms(a.loss_kind, a.target, a.weight, (int64_t)kk * 3 * n + i, n, ut, L);
    ++kk;
    next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    if (!a.theta) break;
  }
}

// Save points of step st, reverse, before the transposed step of st: with g
// the loss gradient at the saved state, a landing save point adds g to
// lam = dL/du_{st+1}; an interior one (theta < 1) adds
// H01 g + J(u_{st+1})^T (h H11 g) to lam and f_p(u_{st+1})^T (h H11 g) to pb,
// and leaves for u_st (after the transposed step, save_points_rev_finish)
// pg = H00 g and pn = h H10 g.
template <typename T, int SYS>
__device__ __forceinline__ bool save_points_rev(const RosArgs<T>& a, int64_t i, int64_t j, int st, const T p[3],
                                                const T us[3], const T un[3], T h, int& kk, int& next, T lam[3],
                                                T pb[3], T pg[3], T pn[3]) {
  const int64_t n = a.n;
  bool interior = false, slopes = false;
  T fs[3], fn[3];
  while (st + 1 == next) {
    T ut[3] = {un[0], un[1], un[2]};
    T th = cst<T>(1.0);
    HermiteW<T> w;
    if (a.theta) {
      th = a.theta[(int64_t)kk * n + j];
      if (th != cst<T>(1.0)) {
        if (!slopes) {
          rhs3<T, SYS>(us, p, fs);
          rhs3<T, SYS>(un, p, fn);
          slopes = true;
        }
        w = hermite_w(th);
#pragma unroll
        for (int c = 0; c < 3; ++c) ut[c] = hermite_c(w, us[c], un[c], fs[c], fn[c], h);
      }
    }
    if (th == cst<T>(1.0)) {
      loss_grad(a.loss_kind, a.target, a.weight, (int64_t)kk * 3 * n + i, n, ut, lam);
    } else {
      T g[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
      loss_grad(a.loss_kind, a.target, a.weight, (int64_t)kk * 3 * n + i, n, ut, g);
      T wn[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) wn[c] = (h * w.h11) * g[c];
      vjp3<T, SYS>(un, p, wn, lam, pb);
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        lam[c] = fmaT(w.h01, g[c], lam[c]);
        pg[c] = fmaT(w.h00, g[c], pg[c]);
        pn[c] = fmaT(h * w.h10, g[c], pn[c]);
      }
      interior = true;
    }
    --kk;
    next = kk >= 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
    if (!a.theta) break;
  }
  return interior;
}

// After the transposed step of st (lam = dL/du_st): the interior save points'
// share of u_st, H00 g + J(u_st)^T (h H10 g), and of p, f_p(u_st)^T (h H10 g).
template <typename T, int SYS>
__device__ __forceinline__ void save_points_rev_finish(const T p[3], const T us[3], const T pg[3], const T pn[3],
                                                       T lam[3], T pb[3]) {
  vjp3<T, SYS>(us, p, pn, lam, pb);
#pragma unroll
  for (int c = 0; c < 3; ++c) lam[c] += pg[c];
}

// Launch shape of the d = 3 Rosenbrock gradient kernels: the pipelined
// reverse step keeps two recomputed steps live (~150 fp64 registers), and the
// resident threads per SM must cover an ensemble of 65,536 in one wave
// (>= 443 per SM): 64-thread blocks, 7 per SM, at most 144 registers.
#ifndef GS_ROS_BS
#define GS_ROS_BS 128
#endif
#ifndef GS_ROS_MINB
#define GS_ROS_MINB 4
#endif
// 1: the reverse step of s overlaps the recompute of s - 1 (software pipeline)
#ifndef GS_ROS_PIPE
#define GS_ROS_PIPE 0
#endif

// Per-thread copy ring in dynamic shared memory: ROWS values per step for
// DEPTH steps (a power of two).  Value r of step s of a thread lives at
// base[((s % DEPTH) * ROWS + r) * blockDim.x], so consecutive threads touch
// consecutive words.  A thread copies its own values with cp.async, one
// commit group per step, and waits on its own groups only (no barrier).
template <typename T, int ROWS, int DEPTH>
struct ThreadRing {
  static_assert((DEPTH & (DEPTH - 1)) == 0 && DEPTH >= 2, "ring depth: a power of two, at least 2");
  static constexpr int kElems = ROWS * DEPTH;  // per thread
  T* base;
  int stride;
  __device__ __forceinline__ ThreadRing(void* smem) : base(reinterpret_cast<T*>(smem) + threadIdx.x),
                                                      stride((int)blockDim.x) {}
  __device__ __forceinline__ T* at(int s, int r) const { return base + ((s & (DEPTH - 1)) * ROWS + r) * stride; }
};

template <typename T>
RosArgs<T> ros_args(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                    void* ws) {
  RosArgs<T> a;
  a.n = P->n;
  a.p = (const T*)P->p;
  a.u0 = (const T*)P->u0;
  a.h = (const T*)M->h;
  a.order = M->order;
  a.nsteps = M->nsteps;
  a.save_idx = M->save_idx;
  a.status = M->status;
  a.nsave = P->nsave;
  a.smax = M->smax;
  a.loss_kind = Ls->kind;
  a.target = (const T*)Ls->target;
  a.weight = (const T*)Ls->weight;
  a.loss = (T*)loss;
  a.dp = (T*)dp;
  a.du0 = (T*)du0;
  a.ck = (T*)ws;
  a.theta = P->system != GS_KIN8 ? (const T*)M->save_theta : nullptr;
  return a;
}

}  // namespace gs
