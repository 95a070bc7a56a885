// sens_ros.cu -- forward sensitivities of the fixed-step Rosenbrock replays
// (ROS2, ROS3) on the d = 3 systems (Robertson, Lorenz): the tangent of the
// replay along each input direction (the three parameters, the three initial
// states), integrated alongside the state.
//
// The derivative is the one the adjoint returns: the exact derivative of the
// fixed-step replay of the recorded steps, the mesh held as data (GRADSOLVE,
// evolve.pub review, "Strengths: precisely scoped exactness claim"), here by
// forward mode, which also yields d u(t_k) / d (p, u0) at every save point.
//
// Tangent of one step along (v = du, w = dp).  Every stage solves
// M k_i = r_i with one M (J = J(u) at the step's start), so
//   dk_i = M^{-1} (dr_i - dM k_i),   dM = -c dJ,   dJ = J'(u)[v] + J_p(u)[w],
// with c = gamma h (ROS2: M = I - gamma h J) or c = h (ROS3: M = I/gamma - h J);
// the right-hand sides' tangents follow the stage formulas of steps.cuh:
//   ROS2: dr_1 = df(u), dr_2 = df(u + h k1) - 2 dk1,
//         du' = v + h (3/2 dk1 + 1/2 dk2)
//   ROS3: dr_1 = df(u), dr_2 = df(v_s) + c21 dk1, dr_3 = df(v_s) + c31 dk1 + c32 dk2,
//         du' = v + h (dk1 + m2 dk2 + m3 dk3),   v_s = u + h k1
// where df(x) = J(x) dx + f_p(x) w.  The state is the replay's own arithmetic
// (ros2_fwd / ros3_fwd), so the loss is bitwise that of gs_solve / gs_grad,
// and the tangent solves reuse its LU factors.
//
// Dense save points (theta in (0, 1) inside a step): the state there is the
// cubic Hermite interpolant of the step on u_s, u_{s+1} and f at both ends,
// theta and h data; its tangent is the same combination of the end tangents
// and of df = J(u) du + f_p(u) w at both ends, evaluated on the steps that
// hold such a save point.
//
// Execution: one thread per (slot, ND directions), the state's step (its
// Jacobian, LU and stages) taken once per thread and shared by its ND
// tangent steps.  The default carries all six directions in one thread
// (ND = 6, 251 registers, no spill): on the 65,536-trajectory Robertson
// ensemble it measured 5.7 ms against 7.5 ms for one direction per thread
// (ROS3; ROS2 59 against 87 ms, dense records 1.4-1.6x), the outputs bit for
// bit the same -- six threads per slot gave the latency-bound stiff replay
// more warps, but each replayed the state again.  With ND < 6 the directions
// of a slot run in 6 / ND blocks of one range of 128 slots (block b: slots
// 128 (b / G) .., direction set b % G), which read the same mesh lines
// through L2.  No workspace.
#include "steps.cuh"

namespace gs {

template <typename T>
struct RosSensArgs {
  int64_t n;
  const T* p;   // [3][n] by trajectory
  const T* u0;  // [3][n] by trajectory
  const T* h;   // [smax][n] by slot
  const int32_t* order;
  const int32_t* nsteps;
  const int32_t* save_idx;  // [nsave][n] by slot
  const int32_t* status;
  int32_t nsave, smax, loss_kind;
  const T* target;  // [nsave][3][n] by trajectory, may be null
  const T* weight;  // [nsave][3][n] by trajectory
  T* loss;          // [n]
  T* dp;            // [3][n]
  T* du0;           // [3][n]
  T* sens;          // [nsave][3][6][n], may be null
  const T* theta;   // [nsave][n] by slot: dense save points, or null
};

// df = J(x) dx + f_p(x) w.
template <typename T, int SYS>
__device__ __forceinline__ void jvp3(const T x[3], const T p[3], const T dx[3], const T w[3], T df[3]) {
  if (SYS == GS_LORENZ) {
    df[0] = fmaT(p[0], dx[1] - dx[0], w[0] * (x[1] - x[0]));
    df[1] = fmaT(p[1] - x[2], dx[0], fmaT(x[0], w[1] - dx[2], -dx[1]));
    df[2] = fmaT(x[1], dx[0], fmaT(x[0], dx[1], -fmaT(p[2], dx[2], w[2] * x[2])));
  } else {
    // f = (k3 y2 y3 - k1 y1, -(f_1 + f_3), k2 y2^2)
    const T d0 = fmaT(w[2], x[1] * x[2], p[2] * fmaT(dx[1], x[2], x[1] * dx[2])) - fmaT(w[0], x[0], p[0] * dx[0]);
    const T d2 = fmaT(w[1], x[1] * x[1], cst<T>(2.0) * (p[1] * x[1]) * dx[1]);
    df[0] = d0;
    df[1] = -(d0 + d2);
    df[2] = d2;
  }
}

// out = dJ k with dJ = J'(u)[v] + J_p(u)[w].
template <typename T, int SYS>
__device__ __forceinline__ void djk3(const T u[3], const T p[3], const T v[3], const T w[3], const T k[3],
                                     T out[3]) {
  if (SYS == GS_LORENZ) {
    // J = [[-s, s, 0], [r - u3, -1, -u1], [u2, u1, -b]]
    out[0] = w[0] * (k[1] - k[0]);
    out[1] = fmaT(w[1] - v[2], k[0], -(v[0] * k[2]));
    out[2] = fmaT(v[1], k[0], fmaT(v[0], k[1], -(w[2] * k[2])));
  } else {
    // J = [[-k1, k3 y3, k3 y2], [k1, -k3 y3 - 2 k2 y2, -k3 y2], [0, 2 k2 y2, 0]]
    const T A = fmaT(w[2], u[2], p[2] * v[2]);
    const T B = fmaT(w[2], u[1], p[2] * v[1]);
    const T C = cst<T>(2.0) * fmaT(w[1], u[1], p[1] * v[1]);
    out[0] = fmaT(A, k[1], fmaT(B, k[2], -(w[0] * k[0])));
    out[1] = fmaT(w[0], k[0], -fmaT(A + C, k[1], B * k[2]));
    out[2] = C * k[1];
  }
}

#ifndef GS_SENS_ROS_NDIR
#define GS_SENS_ROS_NDIR 6
#endif
#ifndef GS_SENS_ROS_MINB
#define GS_SENS_ROS_MINB 1
#endif

template <typename T, int SYS, int METHOD, bool DENSE, int ND>
__global__ void __launch_bounds__(128, GS_SENS_ROS_MINB) k_sens_ros(RosSensArgs<T> a) {
  constexpr int G = 6 / ND;  // threads per slot
  const int64_t n = a.n;
  const int64_t j = (int64_t)(blockIdx.x / G) * blockDim.x + threadIdx.x;
  const int dir0 = (int)(blockIdx.x % G) * ND;  // this thread's directions: dir0 .. dir0 + ND - 1
  if (j >= n) return;
  const int64_t i = a.order[j];
  if (i < 0 || i >= n) return;
  const int S = a.nsteps[j];
  const int64_t n3 = 3 * n;
  const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
  auto fail = [&]() {
    if (dir0 == 0) a.loss[i] = nan;
#pragma unroll
    for (int q = 0; q < ND; ++q) {
      const int dq = dir0 + q;
      (dq < 3 ? a.dp : a.du0)[(dq % 3) * n + i] = nan;
      if (a.sens)
        for (int k = 0; k < a.nsave; ++k)
#pragma unroll
          for (int c = 0; c < 3; ++c) a.sens[(((int64_t)k * 3 + c) * 6 + dq) * n + i] = nan;
    }
  };
  if (a.status[j] != GS_TRAJ_OK || S < 0 || S > a.smax) {
    fail();
    return;
  }
  T p[3], u[3], v[ND][3], w[ND][3];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    p[c] = a.p[c * n + i];
    u[c] = a.u0[c * n + i];
#pragma unroll
    for (int q = 0; q < ND; ++q) {
      w[q][c] = dir0 + q == c ? cst<T>(1.0) : cst<T>(0.0);
      v[q][c] = dir0 + q == 3 + c ? cst<T>(1.0) : cst<T>(0.0);
    }
  }
  T L = cst<T>(0.0), dL[ND];
#pragma unroll
  for (int q = 0; q < ND; ++q) dL[q] = cst<T>(0.0);
  int kk = 0, next = S > 0 ? a.save_idx[j] : -1;
  bool ok = true;
  const T* hq = a.h + j;
  for (int st = 0; st < S; ++st) {
    const T h = hq[(int64_t)st * n];
    if (st + 8 < S) prefetch_l2(hq + (int64_t)(st + 8) * n);
    T LU[9], R[3], k1[3], vs[3], k2[3], k3[3], un[3], dun[ND][3];
    int P[3];
    if (METHOD == GS_ROS3)
      ok = ros3_fwd<T, SYS>(u, p, h, LU, P, R, k1, vs, k2, k3, un) && ok;
    else
      ok = ros2_fwd<T, SYS>(u, p, h, LU, P, R, k1, vs, k2, un) && ok;
    // the tangent step of each direction on the step's factors
#pragma unroll
    for (int q = 0; q < ND; ++q) {
      T r[3], t[3], df[3], dk1[3], dk2[3], dU[3];
      if (METHOD == GS_ROS3) {
        jvp3<T, SYS>(u, p, v[q], w[q], df);
        djk3<T, SYS>(u, p, v[q], w[q], k1, t);
#pragma unroll
        for (int c = 0; c < 3; ++c) r[c] = fmaT(h, t[c], df[c]);
        lu3_solve(LU, P, R, r[0], r[1], r[2], dk1[0], dk1[1], dk1[2]);
#pragma unroll
        for (int c = 0; c < 3; ++c) dU[c] = fmaT(h, dk1[c], v[q][c]);
        jvp3<T, SYS>(vs, p, dU, w[q], df);
        djk3<T, SYS>(u, p, v[q], w[q], k2, t);
#pragma unroll
        for (int c = 0; c < 3; ++c) r[c] = fmaT(h, t[c], fmaT(cst<T>(ROS3_C21), dk1[c], df[c]));
        lu3_solve(LU, P, R, r[0], r[1], r[2], dk2[0], dk2[1], dk2[2]);
        T dk3[3];
        djk3<T, SYS>(u, p, v[q], w[q], k3, t);
#pragma unroll
        for (int c = 0; c < 3; ++c)
          r[c] = fmaT(h, t[c], fmaT(cst<T>(ROS3_C32), dk2[c], fmaT(cst<T>(ROS3_C31), dk1[c], df[c])));
        lu3_solve(LU, P, R, r[0], r[1], r[2], dk3[0], dk3[1], dk3[2]);
#pragma unroll
        for (int c = 0; c < 3; ++c)
          dun[q][c] = fmaT(h, fmaT(cst<T>(ROS3_M3), dk3[c], fmaT(cst<T>(ROS3_M2), dk2[c], dk1[c])), v[q][c]);
      } else {
        const T gh = cst<T>(ROS2_GAMMA) * h;
        jvp3<T, SYS>(u, p, v[q], w[q], df);
        djk3<T, SYS>(u, p, v[q], w[q], k1, t);
#pragma unroll
        for (int c = 0; c < 3; ++c) r[c] = fmaT(gh, t[c], df[c]);
        lu3_solve(LU, P, R, r[0], r[1], r[2], dk1[0], dk1[1], dk1[2]);
#pragma unroll
        for (int c = 0; c < 3; ++c) dU[c] = fmaT(h, dk1[c], v[q][c]);
        jvp3<T, SYS>(vs, p, dU, w[q], df);
        djk3<T, SYS>(u, p, v[q], w[q], k2, t);
#pragma unroll
        for (int c = 0; c < 3; ++c) r[c] = fmaT(gh, t[c], fmaT(cst<T>(-2.0), dk1[c], df[c]));
        lu3_solve(LU, P, R, r[0], r[1], r[2], dk2[0], dk2[1], dk2[2]);
#pragma unroll
        for (int c = 0; c < 3; ++c) dun[q][c] = fmaT(h, fmaT(cst<T>(0.5), dk2[c], cst<T>(1.5) * dk1[c]), v[q][c]);
      }
    }
    // save points of this step (a landing record: at most one, at its end)
    bool slopes = false;
    T fs[3], fn[3];
    while (st + 1 == next) {
      T ut[3] = {un[0], un[1], un[2]};
      HermiteW<T> hw;
      bool interp = false;
      if (DENSE) {
        const T th = a.theta[(int64_t)kk * n + j];
        if (th != cst<T>(1.0)) {
          if (!slopes) {
            rhs3<T, SYS>(u, p, fs);
            rhs3<T, SYS>(un, p, fn);
            slopes = true;
          }
          hw = hermite_w(th);
          interp = true;
#pragma unroll
          for (int c = 0; c < 3; ++c) ut[c] = hermite_c(hw, u[c], un[c], fs[c], fn[c], h);
        }
      }
      const int64_t o = (int64_t)kk * n3 + i;
      T e[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        if (a.loss_kind == GS_LOSS_SUMSQ) {
          e[c] = a.target ? ut[c] - a.target[o + c * n] : ut[c];
          L = fmaT(e[c], e[c], L);
        } else {
          e[c] = a.weight[o + c * n];
          L = fmaT(e[c], ut[c], L);
        }
      }
#pragma unroll
      for (int q = 0; q < ND; ++q) {
        T vt[3] = {dun[q][0], dun[q][1], dun[q][2]};
        if (DENSE && interp) {
          T dfs[3], dfn[3];
          jvp3<T, SYS>(u, p, v[q], w[q], dfs);
          jvp3<T, SYS>(un, p, dun[q], w[q], dfn);
#pragma unroll
          for (int c = 0; c < 3; ++c) vt[c] = hermite_c(hw, v[q][c], dun[q][c], dfs[c], dfn[c], h);
        }
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          if (a.loss_kind == GS_LOSS_SUMSQ)
            dL[q] = fmaT(cst<T>(2.0) * e[c], vt[c], dL[q]);
          else
            dL[q] = fmaT(e[c], vt[c], dL[q]);
          if (a.sens) a.sens[(((int64_t)kk * 3 + c) * 6 + dir0 + q) * n + i] = vt[c];
        }
      }
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
      if (!DENSE) break;
    }
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      u[c] = un[c];
#pragma unroll
      for (int q = 0; q < ND; ++q) v[q][c] = dun[q][c];
    }
  }
  if (!ok) {
    fail();
    return;
  }
  if (dir0 == 0) a.loss[i] = L;
#pragma unroll
  for (int q = 0; q < ND; ++q) {
    const int dq = dir0 + q;
    (dq < 3 ? a.dp : a.du0)[(dq % 3) * n + i] = dL[q];
  }
}

template <typename T>
gs_status launch_sens_ros(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                          void* sens, cudaStream_t st) {
  RosSensArgs<T> a;
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
  a.sens = (T*)sens;
  a.theta = (const T*)M->save_theta;
  constexpr int ND = GS_SENS_ROS_NDIR;
  static_assert(6 % ND == 0, "directions per thread must divide 6");
  const unsigned grid = (unsigned)((P->n + 127) / 128 * (6 / ND));
  const bool rob = P->system == GS_ROBERTSON, ros3 = P->method == GS_ROS3, dense = a.theta != nullptr;
  auto kern = rob ? (ros3 ? (dense ? k_sens_ros<T, GS_ROBERTSON, GS_ROS3, true, ND>
                                   : k_sens_ros<T, GS_ROBERTSON, GS_ROS3, false, ND>)
                          : (dense ? k_sens_ros<T, GS_ROBERTSON, GS_ROS2, true, ND>
                                   : k_sens_ros<T, GS_ROBERTSON, GS_ROS2, false, ND>))
                  : (ros3 ? (dense ? k_sens_ros<T, GS_LORENZ, GS_ROS3, true, ND> : k_sens_ros<T, GS_LORENZ, GS_ROS3, false, ND>)
                          : (dense ? k_sens_ros<T, GS_LORENZ, GS_ROS2, true, ND> : k_sens_ros<T, GS_LORENZ, GS_ROS2, false, ND>));
  kern<<<grid, 128, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_sens_ros<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                           void*, cudaStream_t);
template gs_status launch_sens_ros<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                          void*, cudaStream_t);

}  // namespace gs
