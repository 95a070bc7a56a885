// grad_kin8.cu -- fused fixed-step replay + reverse sweep of the Rosenbrock
// methods ROS2 and ROS3 on the d = 8 system kin8 (kin8.cuh), one thread per
// trajectory slot, the 8 x 8 LU of each step in registers.
//
// The method is that of grad_ros2.cu / grad_ros3.cu (GRADSOLVE, arXiv
// 2609.02876: the recorded mesh replayed with the steps held as data, the
// exact discrete adjoint by a reverse sweep over stage-wise vector-Jacobian
// products); the stage equations are the same at any d.  Per step, with
// lambda = dL/du_{s+1} and the step recomputed from its checkpoint u_s:
//   ROS2 (M = I - gamma h J):
//     rbar = M^{-T} (h/2 lambda);  kbar1 = 3/2 h lambda - 2 rbar + h J(v)^T rbar
//     qbar = M^{-T} kbar1;  ubar = lambda + J(v)^T rbar + J(u)^T qbar
//     pbar += f_p(v)^T rbar + f_p(u)^T qbar;
//     Jbar = gamma h (rbar k2^T + qbar k1^T)
//   ROS3 (M = I/gamma - h J):
//     rbar3 = M^{-T} (m3 h lambda);  rbar2 = M^{-T} (m2 h lambda + c32 rbar3)
//     fbar = rbar3 + rbar2;  kbar1 = h lambda + c31 rbar3 + c21 rbar2 + h J(v)^T fbar
//     rbar1 = M^{-T} kbar1;  ubar = lambda + J(v)^T fbar + J(u)^T rbar1
//     pbar += f_p(v)^T fbar + f_p(u)^T rbar1;
//     Jbar = h (rbar1 k1^T + rbar2 k2^T + rbar3 k3^T)
//   and ubar += d<Jbar, J(u,p)>/du, pbar += d<Jbar, J(u,p)>/dp (Kin8JacAdj).
#include "kin8.cuh"
#include "rosenbrock.cuh"

namespace gs {

// Threads per block: at 255 registers a thread, 64 gives the same occupancy as
// 128 (8 warps per SM) and twice the blocks to spread a small ensemble over
// the SMs.
constexpr int kKin8Block = 64;

template <typename T, int METHOD>
__global__ void __launch_bounds__(kKin8Block) k_grad_kin8(RosArgs<T> a) {
  constexpr int D = 8;
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
    for (int c = 0; c < D; ++c) {
      a.dp[c * n + i] = nan;
      a.du0[c * n + i] = nan;
    }
    return;
  }
  T p[D], u[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    p[c] = a.p[c * n + i];
    u[c] = a.u0[c * n + i];
  }
  const T* __restrict__ hp = a.h + j;
  T* __restrict__ cp = a.ck + j;
  const int64_t nD = D * n;
  T L = cst<T>(0.0);
  int kk = 0;
  int next = a.save_idx[j];
  bool ok = true;
  // ---------------------------------------------------------------- forward
  for (int st = 0; st < S; ++st) {
    const T h = hp[(int64_t)st * n];
#pragma unroll
    for (int c = 0; c < D; ++c) cp[c * n] = u[c];
    cp += nD;
    T LU[D * D], R[D], k1[D], v[D], k2[D], un[D];
    int P[D];
    if constexpr (METHOD == GS_ROS3) {
      T k3[D];
      ok = kin8_ros3_fwd<T>(u, p, h, LU, P, R, k1, v, k2, k3, un) && ok;
    } else {
      ok = kin8_ros2_fwd<T>(u, p, h, LU, P, R, k1, v, k2, un) && ok;
    }
#pragma unroll
    for (int c = 0; c < D; ++c) u[c] = un[c];
    if (st + 1 == next) {
      loss_terms<T, D>(a.loss_kind, a.target, a.weight, (int64_t)kk * nD + i, n, u, L);
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
  }
  // ---------------------------------------------------------------- reverse
  T lam[D], pb[D], unx[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    lam[c] = cst<T>(0.0);
    pb[c] = cst<T>(0.0);
    unx[c] = u[c];  // u_{st+1}
  }
  kk = a.nsave - 1;
  next = a.save_idx[(int64_t)kk * n + j];
  for (int st = S - 1; st >= 0; --st) {
    if (st + 1 == next) {
      loss_grad<T, D>(a.loss_kind, a.target, a.weight, (int64_t)kk * nD + i, n, unx, lam);
      --kk;
      next = kk >= 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
    cp -= nD;
    T us[D];
#pragma unroll
    for (int c = 0; c < D; ++c) us[c] = cp[c * n];
    const T h = hp[(int64_t)st * n];
    T LU[D * D], R[D], kv[3][D], v[D], un[D], ub[D], vb[D], kb1[D], w[3][D], t[D];
    int P[D];
    if constexpr (METHOD == GS_ROS3)
      kin8_ros3_fwd<T>(us, p, h, LU, P, R, kv[0], v, kv[1], kv[2], un);
    else
      kin8_ros2_fwd<T>(us, p, h, LU, P, R, kv[0], v, kv[1], un);
    auto lu = [&](int e) -> T { return LU[e]; };
    auto rc = [&](int q) -> T { return R[q]; };
#pragma unroll
    for (int c = 0; c < D; ++c) {
      ub[c] = lam[c];
      vb[c] = cst<T>(0.0);
    }
    Kin8JacAdj<T> ja;
    if constexpr (METHOD == GS_ROS3) {
      // w[0..2] = rbar1..3 (each pairs with k1..k3)
      const T hm2 = cst<T>(ROS3_M2) * h, hm3 = cst<T>(ROS3_M3) * h;
#pragma unroll
      for (int c = 0; c < D; ++c) t[c] = hm3 * lam[c];
      lu_d_solve_T<T, D>(lu, rc, P, t, w[2]);
#pragma unroll
      for (int c = 0; c < D; ++c) {
        kb1[c] = fmaT(cst<T>(ROS3_C31), w[2][c], h * lam[c]);
        t[c] = fmaT(cst<T>(ROS3_C32), w[2][c], hm2 * lam[c]);
      }
      lu_d_solve_T<T, D>(lu, rc, P, t, w[1]);
#pragma unroll
      for (int c = 0; c < D; ++c) {
        t[c] = w[2][c] + w[1][c];  // fbar
        kb1[c] = fmaT(cst<T>(ROS3_C21), w[1][c], kb1[c]);
      }
      kin8_vjp<T>(v, p, t, vb, pb);
#pragma unroll
      for (int c = 0; c < D; ++c) {
        ub[c] += vb[c];
        kb1[c] = fmaT(h, vb[c], kb1[c]);
      }
      lu_d_solve_T<T, D>(lu, rc, P, kb1, w[0]);
      kin8_vjp<T>(us, p, w[0], ub, pb);
#pragma unroll
      for (int q = 0; q < 3; ++q) ja.add(w[q], kv[q]);
      ja.finish(us, p, h, ub, pb);
    } else {
      // w[0] = qbar (pairs with k1), w[1] = rbar (pairs with k2)
#pragma unroll
      for (int c = 0; c < D; ++c) {
        kb1[c] = (cst<T>(1.5) * h) * lam[c];
        t[c] = (cst<T>(0.5) * h) * lam[c];
      }
      lu_d_solve_T<T, D>(lu, rc, P, t, w[1]);
      kin8_vjp<T>(v, p, w[1], vb, pb);
#pragma unroll
      for (int c = 0; c < D; ++c) {
        ub[c] += vb[c];
        kb1[c] = fmaT(h, vb[c], fmaT(cst<T>(-2.0), w[1][c], kb1[c]));
      }
      lu_d_solve_T<T, D>(lu, rc, P, kb1, w[0]);
      kin8_vjp<T>(us, p, w[0], ub, pb);
#pragma unroll
      for (int q = 0; q < 2; ++q) ja.add(w[q], kv[q]);
      ja.finish(us, p, cst<T>(ROS2_GAMMA) * h, ub, pb);
    }
#pragma unroll
    for (int c = 0; c < D; ++c) {
      lam[c] = ub[c];
      unx[c] = us[c];
    }
  }
  if (!ok) {
    L = nan;
#pragma unroll
    for (int c = 0; c < D; ++c) lam[c] = pb[c] = nan;
  }
  a.loss[i] = L;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    a.dp[c * n + i] = pb[c];
    a.du0[c * n + i] = lam[c];
  }
}

template <typename T>
gs_status launch_grad_kin8(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                           void* ws, cudaStream_t st) {
  const RosArgs<T> a = ros_args<T>(P, M, Ls, loss, dp, du0, ws);
  const int bs = kKin8Block;
  const unsigned grid = (unsigned)((P->n + bs - 1) / bs);
  if (P->method == GS_ROS3)
    k_grad_kin8<T, GS_ROS3><<<grid, bs, 0, st>>>(a);
  else
    k_grad_kin8<T, GS_ROS2><<<grid, bs, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_kin8<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                            void*, cudaStream_t);
template gs_status launch_grad_kin8<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                           void*, cudaStream_t);

}  // namespace gs
