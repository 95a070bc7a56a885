// grad_ros3.cu -- fused fixed-step replay + reverse sweep for the third-order
// Rosenbrock method ROS3 (d = 3: Robertson, Lorenz), one thread per slot.
//
// GRADSOLVE (arXiv 2609.02876) supports explicit and Rosenbrock integrators
// (abstract) and names higher-order integrators among its next steps
// ("Future directions").  ROS3 (Sandu, Verwer, Blom, Spee, Carmichael & Potra
// 1997) in the stage form of steps.cuh, k_i = K_i / h of the paper's
// transformed form:
//   M = I/gamma - h J(u);  M k1 = f(u);  v = u + h k1;
//   M k2 = f(v) + c21 k1;  M k3 = f(v) + c31 k1 + c32 k2;
//   u_{s+1} = u + h (k1 + m2 k2 + m3 k3).
// The forward replay follows the floating-point contract, so it is bitwise
// equal to any replay that keeps it (the recorder's included).
//
// Reverse sweep of one step, lambda = dL/du_{s+1} (r_i: the right-hand side
// solved for k_i; rbar_i = dL/dr_i):
//   ubar = lambda;  kbar1 = h lambda,  kbar2 = m2 h lambda,  kbar3 = m3 h lambda
//   rbar3 = M^{-T} kbar3;  fbar = rbar3;  kbar1 += c31 rbar3;  kbar2 += c32 rbar3
//   rbar2 = M^{-T} kbar2;  fbar += rbar2; kbar1 += c21 rbar2
//   ubar += J(v)^T fbar;   pbar += f_p(v)^T fbar;   kbar1 += h J(v)^T fbar
//   rbar1 = M^{-T} kbar1
//   ubar += J(u)^T rbar1;  pbar += f_p(u)^T rbar1
//   Jbar  = h (rbar1 k1^T + rbar2 k2^T + rbar3 k3^T)      (from M = I/gamma - h J)
//   ubar += d<Jbar, J(u,p)>/du;  pbar += d<Jbar, J(u,p)>/dp
// M^T solves reuse the LU factors of the recomputed forward step; the last
// line carries the second derivatives of f, hand-registered per system.
#include "rosenbrock.cuh"

namespace gs {

// ubar += d<Jbar, J(u,p)>/du,  pbar += d<Jbar, J(u,p)>/dp for
// Jbar_ab = h sum_i rbar_i[a] k_i[b].
template <typename T, int SYS>
__device__ __forceinline__ void jac_adjoint3_ros3(const T u[3], const T p[3], T h, const T r1[3], const T r2[3],
                                                  const T r3[3], const T k1[3], const T k2[3], const T k3[3], T ub[3],
                                                  T pb[3]) {
  // sum_i w_i[a] k_i[b] for a weight vector per stage given by its components
  auto outer = [&](T w1, T w2, T w3, int b) { return h * fmaT(w3, k3[b], fmaT(w2, k2[b], w1 * k1[b])); };
  if (SYS == GS_LORENZ) {
    // J = [[-s, s, 0], [r - u3, -1, -u1], [u2, u1, -b]]
    auto Jb = [&](int a, int b) { return outer(r1[a], r2[a], r3[a], b); };
    ub[0] += Jb(2, 1) - Jb(1, 2);
    ub[1] += Jb(2, 0);
    ub[2] -= Jb(1, 0);
    pb[0] += Jb(0, 1) - Jb(0, 0);
    pb[1] += Jb(1, 0);
    pb[2] -= Jb(2, 2);
  } else {
    // J = [[-k1, k3 y3, k3 y2], [k1, -k3 y3 - 2 k2 y2, -k3 y2], [0, 2 k2 y2, 0]]; with
    // row differences of Jbar: A = Jb12 - Jb22, B = Jb13 - Jb23, C = Jb32 - Jb22,
    // D = Jb21 - Jb11 (1-based)
    const T d12_1 = r1[0] - r1[1], d12_2 = r2[0] - r2[1], d12_3 = r3[0] - r3[1];
    const T d32_1 = r1[2] - r1[1], d32_2 = r2[2] - r2[1], d32_3 = r3[2] - r3[1];
    const T A = outer(d12_1, d12_2, d12_3, 1);
    const T B = outer(d12_1, d12_2, d12_3, 2);
    const T C = outer(d32_1, d32_2, d32_3, 1);
    const T D = -outer(d12_1, d12_2, d12_3, 0);
    ub[1] += fmaT(p[2], B, cst<T>(2.0) * p[1] * C);
    ub[2] = fmaT(p[2], A, ub[2]);
    pb[0] += D;
    pb[1] = fmaT(cst<T>(2.0) * u[1], C, pb[1]);
    pb[2] += fmaT(u[2], A, u[1] * B);
  }
}

// Copy rings: the forward streams h, the reverse (u_s, h_s), kRos3Ring steps
// ahead (DRAM latency is most of a step at the few warps per SM that these
// ensembles fill).
constexpr int kRos3Ring = 8;

// One recomputed forward step, as its transposed step needs it.
template <typename T>
struct Ros3Step {
  T us[3], h, LU[9], R[3], k1[3], v[3], k2[3], k3[3];
  int P[3];
};

template <typename T, int SYS>
__device__ __forceinline__ void ros3_recompute(Ros3Step<T>& q, const T p[3]) {
  T un[3];
  ros3_fwd<T, SYS>(q.us, p, q.h, q.LU, q.P, q.R, q.k1, q.v, q.k2, q.k3, un);
}

// The transposed step of q: lam <- dL/du_s from lam = dL/du_{s+1}; pb += dL/dp.
template <typename T, int SYS>
__device__ __forceinline__ void ros3_transpose(const Ros3Step<T>& q, const T p[3], T lam[3], T pb[3]) {
  const T h = q.h;
  T ub[3] = {lam[0], lam[1], lam[2]};
  T kb1[3], kb2[3], r1[3], r2[3], r3[3], fb[3];
  const T hm2 = cst<T>(ROS3_M2) * h, hm3 = cst<T>(ROS3_M3) * h;
  lu3_solve_T(q.LU, q.P, q.R, hm3 * lam[0], hm3 * lam[1], hm3 * lam[2], r3[0], r3[1], r3[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    kb1[c] = fmaT(cst<T>(ROS3_C31), r3[c], h * lam[c]);
    kb2[c] = fmaT(cst<T>(ROS3_C32), r3[c], hm2 * lam[c]);
  }
  lu3_solve_T(q.LU, q.P, q.R, kb2[0], kb2[1], kb2[2], r2[0], r2[1], r2[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    fb[c] = r3[c] + r2[c];
    kb1[c] = fmaT(cst<T>(ROS3_C21), r2[c], kb1[c]);
  }
  T vb[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  vjp3<T, SYS>(q.v, p, fb, vb, pb);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    ub[c] += vb[c];
    kb1[c] = fmaT(h, vb[c], kb1[c]);
  }
  lu3_solve_T(q.LU, q.P, q.R, kb1[0], kb1[1], kb1[2], r1[0], r1[1], r1[2]);
  vjp3<T, SYS>(q.us, p, r1, ub, pb);
  jac_adjoint3_ros3<T, SYS>(q.us, p, h, r1, r2, r3, q.k1, q.k2, q.k3, ub, pb);
#pragma unroll
  for (int c = 0; c < 3; ++c) lam[c] = ub[c];
}

// Reverse loop, software-pipelined: iteration st recomputes step st - 1 from
// its checkpoint while it runs the transposed step of st (recomputed by the
// iteration before).  The recompute does not depend on lambda, so the two are
// independent chains in one instruction stream.
template <typename T, int SYS>
__global__ void __launch_bounds__(GS_ROS_BS, GS_ROS_MINB) k_grad_ros3(RosArgs<T> a) {
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
  const ThreadRing<T, 1, kRos3Ring> rf(ring_raw);
  auto issue_f = [&](int sf) {
    if (sf < S) cp_async_el(rf.at(sf, 0), hp + (int64_t)sf * n);
    cp_async_commit();
  };
#pragma unroll
  for (int sf = 0; sf < kRos3Ring; ++sf) issue_f(sf);
  for (int st = 0; st < S; ++st) {
    cp_async_wait<kRos3Ring - 1>();  // the group of step st
    const T h = *rf.at(st, 0);
    cp[0] = u[0];
    cp[n] = u[1];
    cp[2 * n] = u[2];
    cp += n3;
    T LU[9], R[3], k1[3], v[3], k2[3], k3[3], un[3];
    int P[3];
    ok = ros3_fwd<T, SYS>(u, p, h, LU, P, R, k1, v, k2, k3, un) && ok;
    save_points_fwd<T, SYS>(a, i, j, st, p, u, un, h, kk, next, L);
#pragma unroll
    for (int c = 0; c < 3; ++c) u[c] = un[c];
    issue_f(st + kRos3Ring);  // into the slot step st has left
  }
  cp_async_wait<0>();  // the reverse reuses the ring
  // ---------------------------------------------------------------- reverse
  const ThreadRing<T, 4, kRos3Ring> rr(ring_raw);
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
  auto take_r = [&](int sr, Ros3Step<T>& q) {
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
  for (int i2 = 0; i2 < kRos3Ring; ++i2) issue_r(S - 1 - i2);
  Ros3Step<T> cur;
  if (S > 0) {
    cp_async_wait<kRos3Ring - 1>();
    take_r(S - 1, cur);
    ros3_recompute<T, SYS>(cur, p);
  }
  for (int st = S - 1; st >= 0; --st) {
    T pg[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)}, pn[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
    const bool interior = save_points_rev<T, SYS>(a, i, j, st, p, cur.us, unx, cur.h, kk, next, lam, pb, pg, pn);
    // step st - 1 (step 0 again on the last iteration, whose result is unused:
    // its ring slot still holds step 0, since no later copy targets it)
    Ros3Step<T> nxt;
    if constexpr (GS_ROS_PIPE != 0) {
      cp_async_wait<kRos3Ring - 2>();
      take_r(st > 0 ? st - 1 : 0, nxt);
      ros3_recompute<T, SYS>(nxt, p);
      ros3_transpose<T, SYS>(cur, p, lam, pb);
    } else {  // one step at a time: transpose st, then load and recompute st - 1
      ros3_transpose<T, SYS>(cur, p, lam, pb);
      cp_async_wait<kRos3Ring - 2>();
      take_r(st > 0 ? st - 1 : 0, nxt);
      ros3_recompute<T, SYS>(nxt, p);
    }
    if (interior) save_points_rev_finish<T, SYS>(p, cur.us, pg, pn, lam, pb);
#pragma unroll
    for (int c = 0; c < 3; ++c) unx[c] = cur.us[c];
    cur = nxt;
    issue_r(st - kRos3Ring);  // into the slot step st has left
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
gs_status launch_grad_ros3(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                           void* ws, cudaStream_t st) {
  const RosArgs<T> a = ros_args<T>(P, M, Ls, loss, dp, du0, ws);
  const int bs = GS_ROS_BS;
  const unsigned grid = (unsigned)((P->n + bs - 1) / bs);
  const size_t smem = (size_t)ThreadRing<T, 4, kRos3Ring>::kElems * bs * sizeof(T);
  auto kern = P->system == GS_ROBERTSON ? k_grad_ros3<T, GS_ROBERTSON> : k_grad_ros3<T, GS_LORENZ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return GS_ECUDA;
  kern<<<grid, bs, smem, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_ros3<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                            void*, cudaStream_t);
template gs_status launch_grad_ros3<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                           void*, cudaStream_t);

}  // namespace gs
