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
  return a;
}

}  // namespace gs
