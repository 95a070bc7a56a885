// grad_ros2.cu -- fused fixed-step replay + reverse sweep for the Rosenbrock
// method ROS2 (d = 3: Robertson, Lorenz), one thread per trajectory slot.
//
// GRADSOLVE (arXiv 2609.02876) supports explicit and Rosenbrock integrators
// (abstract); the second-order Rosenbrock method is its stiff default (evolve.pub
// review "Summary").  ROS2 (Verwer, Spee, Blom & Hundsdorfer 1999):
//   M = I - gamma h J(u),  M k1 = f(u),  v = u + h k1,
//   M k2 = f(v) - 2 k1,    u_{s+1} = u + h (3/2 k1 + 1/2 k2).
// The forward replay follows the floating-point contract (LU with partial
// pivoting in registers, fixed operation order), so it is bitwise equal to any
// replay that keeps it.
//
// Reverse sweep of one step, lambda = dL/du_{s+1}:
//   kbar1 = 3/2 h lambda,  kbar2 = 1/2 h lambda,  ubar = lambda
//   rbar  = M^{-T} kbar2;  kbar1 -= 2 rbar
//   ubar += J(v)^T rbar;   pbar += f_p(v)^T rbar;  kbar1 += h J(v)^T rbar
//   qbar  = M^{-T} kbar1
//   ubar += J(u)^T qbar;   pbar += f_p(u)^T qbar
//   Jbar  = gamma h (rbar k2^T + qbar k1^T)          (from M = I - gamma h J)
//   ubar += d<Jbar, J(u,p)>/du;  pbar += d<Jbar, J(u,p)>/dp
// The last line carries the second derivatives of f that a Rosenbrock adjoint
// needs; they are hand-registered per system below.  M^T solves reuse the LU
// factors of the recomputed forward step.
#include "rosenbrock.cuh"

namespace gs {

// ubar += d<Jbar, J(u,p)>/du,  pbar += d<Jbar, J(u,p)>/dp, with
// Jbar_ab = g (rb_a k2_b + qb_a k1_b).
template <typename T, int SYS>
__device__ __forceinline__ void jac_adjoint3(const T u[3], const T p[3], T g, const T rb[3], const T qb[3],
                                             const T k1[3], const T k2[3], T ub[3], T pb[3]) {
  auto Jb = [&](int a, int b) { return g * fmaT(rb[a], k2[b], qb[a] * k1[b]); };
  if (SYS == GS_LORENZ) {
    // J = [[-s, s, 0], [r - u3, -1, -u1], [u2, u1, -b]]
    ub[0] += Jb(2, 1) - Jb(1, 2);
    ub[1] += Jb(2, 0);
    ub[2] -= Jb(1, 0);
    pb[0] += Jb(0, 1) - Jb(0, 0);
    pb[1] += Jb(1, 0);
    pb[2] -= Jb(2, 2);
  } else {
    // J = [[-k1, k3 y3, k3 y2], [k1, -k3 y3 - 2 k2 y2, -k3 y2], [0, 2 k2 y2, 0]]
    const T dr12 = rb[0] - rb[1], dq12 = qb[0] - qb[1];
    const T dr32 = rb[2] - rb[1], dq32 = qb[2] - qb[1];
    const T A = g * fmaT(dr12, k2[1], dq12 * k1[1]);     // Jb12 - Jb22
    const T B = g * fmaT(dr12, k2[2], dq12 * k1[2]);     // Jb13 - Jb23
    const T C = g * fmaT(dr32, k2[1], dq32 * k1[1]);     // Jb32 - Jb22
    const T D = -(g * fmaT(dr12, k2[0], dq12 * k1[0]));  // Jb21 - Jb11
    ub[1] += fmaT(p[2], B, cst<T>(2.0) * p[1] * C);
    ub[2] = fmaT(p[2], A, ub[2]);
    pb[0] += D;
    pb[1] = fmaT(cst<T>(2.0) * u[1], C, pb[1]);
    pb[2] += fmaT(u[2], A, u[1] * B);
  }
}

template <typename T, int SYS>
__global__ void __launch_bounds__(128) k_grad_ros2(RosArgs<T> a) {
  const int64_t n = a.n;
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t i = a.order[j];
  if (i < 0 || i >= n) return;  // not a permutation entry: nothing to write
  const int S = a.nsteps[j];
  const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
  if (a.status[j] != GS_TRAJ_OK || S < 0 || S > a.smax) {
    a.loss[i] = nan;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      a.dp[c * n + i] = nan;
      a.du0[c * n + i] = nan;
    }
    return;
  }
  T p[3], u[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    p[c] = a.p[c * n + i];
    u[c] = a.u0[c * n + i];
  }
  const T* __restrict__ hp = a.h + j;
  T* __restrict__ cp = a.ck + j;
  const int64_t n3 = 3 * n;
  T L = cst<T>(0.0);
  int kk = 0;
  int next = a.save_idx[j];
  bool ok = true;
  for (int st = 0; st < S; ++st) {
    const T h = hp[(int64_t)st * n];
    cp[0] = u[0];
    cp[n] = u[1];
    cp[2 * n] = u[2];
    cp += n3;
    T LU[9], R[3], k1[3], v[3], k2[3], un[3];
    int P[3];
    ok = ros2_fwd<T, SYS>(u, p, h, LU, P, R, k1, v, k2, un) && ok;
#pragma unroll
    for (int c = 0; c < 3; ++c) u[c] = un[c];
    if (st + 1 == next) {
      loss_terms(a.loss_kind, a.target, a.weight, (int64_t)kk * n3 + i, n, u, L);
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
  }
  T lam[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  T pb[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  kk = a.nsave - 1;
  next = a.save_idx[(int64_t)kk * n + j];
  T unx[3] = {u[0], u[1], u[2]};
  for (int st = S - 1; st >= 0; --st) {
    if (st + 1 == next) {
      loss_grad(a.loss_kind, a.target, a.weight, (int64_t)kk * n3 + i, n, unx, lam);
      --kk;
      next = kk >= 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
    cp -= n3;
    T us[3] = {cp[0], cp[n], cp[2 * n]};
    const T h = hp[(int64_t)st * n];
    T LU[9], R[3], k1[3], v[3], k2[3], un[3];
    int P[3];
    ros2_fwd<T, SYS>(us, p, h, LU, P, R, k1, v, k2, un);
    const T gh = cst<T>(ROS2_GAMMA) * h;
    T ub[3] = {lam[0], lam[1], lam[2]};
    T kb1[3], rb[3], qb[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) kb1[c] = (cst<T>(1.5) * h) * lam[c];
    lu3_solve_T(LU, P, R, (cst<T>(0.5) * h) * lam[0], (cst<T>(0.5) * h) * lam[1], (cst<T>(0.5) * h) * lam[2], rb[0],
                rb[1], rb[2]);
    T vb[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
    vjp3<T, SYS>(v, p, rb, vb, pb);
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      ub[c] += vb[c];
      kb1[c] = fmaT(h, vb[c], fmaT(cst<T>(-2.0), rb[c], kb1[c]));
    }
    lu3_solve_T(LU, P, R, kb1[0], kb1[1], kb1[2], qb[0], qb[1], qb[2]);
    vjp3<T, SYS>(us, p, qb, ub, pb);
    jac_adjoint3<T, SYS>(us, p, gh, rb, qb, k1, k2, ub, pb);
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      lam[c] = ub[c];
      unx[c] = us[c];
    }
  }
  if (!ok) {
    L = nan;
#pragma unroll
    for (int c = 0; c < 3; ++c) lam[c] = pb[c] = nan;
  }
  a.loss[i] = L;
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    a.dp[c * n + i] = pb[c];
    a.du0[c * n + i] = lam[c];
  }
}

template <typename T>
gs_status launch_grad_ros2(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                           void* ws, cudaStream_t st) {
  const RosArgs<T> a = ros_args<T>(P, M, Ls, loss, dp, du0, ws);
  const int bs = 128;
  const unsigned grid = (unsigned)((P->n + bs - 1) / bs);
  if (P->system == GS_ROBERTSON)
    k_grad_ros2<T, GS_ROBERTSON><<<grid, bs, 0, st>>>(a);
  else
    k_grad_ros2<T, GS_LORENZ><<<grid, bs, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_ros2<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                            void*, cudaStream_t);
template gs_status launch_grad_ros2<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                           void*, cudaStream_t);

}  // namespace gs
