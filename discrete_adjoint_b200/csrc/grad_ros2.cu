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

// Copy rings: the forward streams h, the reverse (u_s, h_s), kRosRing steps
// ahead (DRAM latency is most of a step at the few warps per SM that these
// ensembles fill).
constexpr int kRosRing = 8;

// One recomputed forward step, as its transposed step needs it.
template <typename T>
struct Ros2Step {
  T us[3], h, LU[9], R[3], k1[3], v[3], k2[3];
  int P[3];
};

template <typename T, int SYS>
__device__ __forceinline__ void ros2_recompute(Ros2Step<T>& q, const T p[3]) {
  T un[3];
  ros2_fwd<T, SYS>(q.us, p, q.h, q.LU, q.P, q.R, q.k1, q.v, q.k2, un);
}

// The transposed step of q: lam <- dL/du_s from lam = dL/du_{s+1}; pb += dL/dp.
template <typename T, int SYS>
__device__ __forceinline__ void ros2_transpose(const Ros2Step<T>& q, const T p[3], T lam[3], T pb[3]) {
  const T h = q.h;
  const T gh = cst<T>(ROS2_GAMMA) * h;
  T ub[3] = {lam[0], lam[1], lam[2]};
  T kb1[3], rb[3], qb[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) kb1[c] = (cst<T>(1.5) * h) * lam[c];
  lu3_solve_T(q.LU, q.P, q.R, (cst<T>(0.5) * h) * lam[0], (cst<T>(0.5) * h) * lam[1], (cst<T>(0.5) * h) * lam[2],
              rb[0], rb[1], rb[2]);
  T vb[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  vjp3<T, SYS>(q.v, p, rb, vb, pb);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    ub[c] += vb[c];
    kb1[c] = fmaT(h, vb[c], fmaT(cst<T>(-2.0), rb[c], kb1[c]));
  }
  lu3_solve_T(q.LU, q.P, q.R, kb1[0], kb1[1], kb1[2], qb[0], qb[1], qb[2]);
  vjp3<T, SYS>(q.us, p, qb, ub, pb);
  jac_adjoint3<T, SYS>(q.us, p, gh, rb, qb, q.k1, q.k2, ub, pb);
#pragma unroll
  for (int c = 0; c < 3; ++c) lam[c] = ub[c];
}

// Reverse loop, software-pipelined: iteration st recomputes step st - 1 from
// its checkpoint while it runs the transposed step of st (recomputed by the
// iteration before).  The recompute does not depend on lambda, so the two are
// independent chains in one instruction stream.
template <typename T, int SYS>
__global__ void __launch_bounds__(GS_ROS_BS, GS_ROS_MINB) k_grad_ros2(RosArgs<T> a) {
  extern __shared__ __align__(16) unsigned char ring_raw[];
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
  // ---------------------------------------------------------------- forward
  const ThreadRing<T, 1, kRosRing> rf(ring_raw);
  auto issue_f = [&](int sf) {
    if (sf < S) cp_async_el(rf.at(sf, 0), hp + (int64_t)sf * n);
    cp_async_commit();
  };
#pragma unroll
  for (int sf = 0; sf < kRosRing; ++sf) issue_f(sf);
  for (int st = 0; st < S; ++st) {
    cp_async_wait<kRosRing - 1>();  // the group of step st
    const T h = *rf.at(st, 0);
    cp[0] = u[0];
    cp[n] = u[1];
    cp[2 * n] = u[2];
    cp += n3;
    T LU[9], R[3], k1[3], v[3], k2[3], un[3];
    int P[3];
    ok = ros2_fwd<T, SYS>(u, p, h, LU, P, R, k1, v, k2, un) && ok;
    save_points_fwd<T, SYS>(a, i, j, st, p, u, un, h, kk, next, L);
#pragma unroll
    for (int c = 0; c < 3; ++c) u[c] = un[c];
    issue_f(st + kRosRing);  // into the slot step st has left
  }
  cp_async_wait<0>();  // the reverse reuses the ring
  // ---------------------------------------------------------------- reverse
  const ThreadRing<T, 4, kRosRing> rr(ring_raw);
  auto issue_r = [&](int sr) {
    if (sr >= 0 && sr < S) {
      const T* c = a.ck + (int64_t)sr * n3 + j;
      cp_async_el(rr.at(sr, 0), c);
      cp_async_el(rr.at(sr, 1), c + n);
      cp_async_el(rr.at(sr, 2), c + 2 * n);
      cp_async_el(rr.at(sr, 3), hp + (int64_t)sr * n);
    }
    cp_async_commit();
  };
  auto take_r = [&](int sr, Ros2Step<T>& q) {
    q.us[0] = *rr.at(sr, 0);
    q.us[1] = *rr.at(sr, 1);
    q.us[2] = *rr.at(sr, 2);
    q.h = *rr.at(sr, 3);
  };
  T lam[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  T pb[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  kk = a.nsave - 1;
  next = S > 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
  T unx[3] = {u[0], u[1], u[2]};  // u_{st+1}
#pragma unroll
  for (int i2 = 0; i2 < kRosRing; ++i2) issue_r(S - 1 - i2);
  Ros2Step<T> cur;
  if (S > 0) {
    cp_async_wait<kRosRing - 1>();
    take_r(S - 1, cur);
    ros2_recompute<T, SYS>(cur, p);
  }
  for (int st = S - 1; st >= 0; --st) {
    T pg[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)}, pn[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
    const bool interior = save_points_rev<T, SYS>(a, i, j, st, p, cur.us, unx, cur.h, kk, next, lam, pb, pg, pn);
    // step st - 1 (step 0 again on the last iteration, whose result is unused:
    // its ring slot still holds step 0, since no later copy targets it)
    Ros2Step<T> nxt;
    if constexpr (GS_ROS_PIPE != 0) {
      cp_async_wait<kRosRing - 2>();
      take_r(st > 0 ? st - 1 : 0, nxt);
      ros2_recompute<T, SYS>(nxt, p);
      ros2_transpose<T, SYS>(cur, p, lam, pb);
    } else {  // one step at a time: transpose st, then load and recompute st - 1
      ros2_transpose<T, SYS>(cur, p, lam, pb);
      cp_async_wait<kRosRing - 2>();
      take_r(st > 0 ? st - 1 : 0, nxt);
      ros2_recompute<T, SYS>(nxt, p);
    }
    if (interior) save_points_rev_finish<T, SYS>(p, cur.us, pg, pn, lam, pb);
#pragma unroll
    for (int c = 0; c < 3; ++c) unx[c] = cur.us[c];
    cur = nxt;
    issue_r(st - kRosRing);  // into the slot step st has left
  }
  cp_async_wait<0>();
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
  const int bs = GS_ROS_BS;
  const unsigned grid = (unsigned)((P->n + bs - 1) / bs);
  const size_t smem = (size_t)ThreadRing<T, 4, kRosRing>::kElems * bs * sizeof(T);
  auto kern = P->system == GS_ROBERTSON ? k_grad_ros2<T, GS_ROBERTSON> : k_grad_ros2<T, GS_LORENZ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return GS_ECUDA;
  kern<<<grid, bs, smem, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_ros2<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                            void*, cudaStream_t);
template gs_status launch_grad_ros2<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                           void*, cudaStream_t);

}  // namespace gs
