// sens_kin8.cu -- forward sensitivities of the fixed-step Rosenbrock replays
// (ROS2, ROS3) on the d = 8 system kin8: the tangent of the replay along each
// of the 16 input directions (the eight rate constants, the eight initial
// states), integrated alongside the state.
//
// The derivative is the one the adjoint returns: the exact derivative of the
// fixed-step replay of the recorded steps, the mesh held as data (GRADSOLVE,
// evolve.pub review, "Strengths: precisely scoped exactness claim"), here by
// forward mode, which also yields d u(t_k) / d (p, u0) at every save point.
//
// Tangent of one step along (v = du, w = dp), as for the d = 3 systems
// (sens_ros.cu): every stage solves M k_i = r_i with one M built from
// J = J(u) at the step's start, so dk_i = M^{-1} (dr_i + c dJ k_i), c = gamma h
// (ROS2) or h (ROS3), dJ = J'(u)[v] + J_p(u)[w]; dr_i follows the stage
// formulas with df(x)[dx] = J(x) dx + f_p(x) w.  kin8 is f = N r(u, p) with
// mass-action rates r_j = p_j m_j(u) (m_j a monomial of degree one or two),
// so both products go through the rates:
//   df = N dr,   dr_j = w_j m_j(x) + p_j Dm_j(x)[dx]
//   dJ k = N d(Dr[k]),  Dr_j[k] = p_j Dm_j(u)[k],
//   d(Dr_j[k]) = w_j Dm_j(u)[k] + p_j D^2 m_j(u)[k, v]
// (the second derivative is nonzero only for the two bilinear rates r3, r7).
// The state is the replay's own arithmetic, so the loss is bitwise that of
// gs_solve / gs_grad, and the tangent solves reuse its LU factors.
//
// Execution: one thread per (slot, direction); block b takes slots
// 64 (b / 16) .. and direction b % 16, so the sixteen blocks of a slot range
// read the same mesh lines through L2.  No workspace.
#include "kin8.cuh"

namespace gs {

template <typename T>
struct Kin8SensArgs {
  int64_t n;
  const T* p;   // [8][n] by trajectory
  const T* u0;  // [8][n] by trajectory
  const T* h;   // [smax][n] by slot
  const int32_t* order;
  const int32_t* nsteps;
  const int32_t* save_idx;  // [nsave][n] by slot
  const int32_t* status;
  int32_t nsave, smax, loss_kind;
  const T* target;  // [nsave][8][n] by trajectory, may be null
  const T* weight;  // [nsave][8][n] by trajectory
  T* loss;          // [n]
  T* dp;            // [8][n]
  T* du0;           // [8][n]
  T* sens;          // [nsave][8][16][n], may be null
};

constexpr int kSensKin8Block = 64;

// df = N dr with dr_j = w_j m_j(x) + p_j Dm_j(x)[dx].
template <typename T>
__device__ __forceinline__ void kin8_jvp(const T x[8], const T p[8], const T dx[8], const T w[8], T df[8]) {
  T dr[8];
  dr[0] = fmaT(w[0], x[0], p[0] * dx[0]);
  dr[1] = fmaT(w[1], x[1], p[1] * dx[1]);
  dr[2] = fmaT(w[2], x[1] * x[2], p[2] * fmaT(dx[1], x[2], x[1] * dx[2]));
  dr[3] = fmaT(w[3], x[3], p[3] * dx[3]);
  dr[4] = fmaT(w[4], x[4], p[4] * dx[4]);
  dr[5] = fmaT(w[5], x[5], p[5] * dx[5]);
  dr[6] = fmaT(w[6], x[5] * x[6], p[6] * fmaT(dx[5], x[6], x[5] * dx[6]));
  dr[7] = fmaT(w[7], x[7], p[7] * dx[7]);
  // the stoichiometry of kin8_f
  df[0] = (dr[1] - dr[0]) + dr[7];
  df[1] = (dr[0] - dr[1]) - dr[2];
  df[2] = dr[3] - dr[2];
  df[3] = dr[2] - dr[3];
  df[4] = (dr[3] - dr[4]) + dr[5];
  df[5] = (dr[4] - dr[5]) - dr[6];
  df[6] = dr[7] - dr[6];
  df[7] = dr[6] - dr[7];
}

// out = dJ k = N d(Dr[k]) with d(Dr_j[k]) = w_j Dm_j(u)[k] + p_j D^2 m_j(u)[k, v].
template <typename T>
__device__ __forceinline__ void kin8_djk(const T u[8], const T p[8], const T v[8], const T w[8], const T k[8],
                                         T out[8]) {
  T e[8];
  e[0] = w[0] * k[0];
  e[1] = w[1] * k[1];
  e[2] = fmaT(w[2], fmaT(k[1], u[2], u[1] * k[2]), p[2] * fmaT(k[1], v[2], v[1] * k[2]));
  e[3] = w[3] * k[3];
  e[4] = w[4] * k[4];
  e[5] = w[5] * k[5];
  e[6] = fmaT(w[6], fmaT(k[5], u[6], u[5] * k[6]), p[6] * fmaT(k[5], v[6], v[5] * k[6]));
  e[7] = w[7] * k[7];
  out[0] = (e[1] - e[0]) + e[7];
  out[1] = (e[0] - e[1]) - e[2];
  out[2] = e[3] - e[2];
  out[3] = e[2] - e[3];
  out[4] = (e[3] - e[4]) + e[5];
  out[5] = (e[4] - e[5]) - e[6];
  out[6] = e[7] - e[6];
  out[7] = e[6] - e[7];
}

template <typename T, int METHOD>
__global__ void __launch_bounds__(kSensKin8Block) k_sens_kin8(Kin8SensArgs<T> a) {
  constexpr int D = 8;
  const int64_t n = a.n;
  const int64_t j = (int64_t)(blockIdx.x / 16) * blockDim.x + threadIdx.x;
  const int dq = (int)(blockIdx.x % 16);  // this thread's direction
  if (j >= n) return;
  const int64_t i = a.order[j];
  if (i < 0 || i >= n) return;
  const int S = a.nsteps[j];
  const int64_t nD = D * n;
  const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
  auto fail = [&]() {
    if (dq == 0) a.loss[i] = nan;
    (dq < D ? a.dp : a.du0)[(dq % D) * n + i] = nan;
    if (a.sens)
      for (int k = 0; k < a.nsave; ++k)
        for (int c = 0; c < D; ++c) a.sens[(((int64_t)k * D + c) * 16 + dq) * n + i] = nan;
  };
  if (a.status[j] != GS_TRAJ_OK || S < 0 || S > a.smax) {
    fail();
    return;
  }
  T p[D], u[D], v[D], w[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    p[c] = a.p[c * n + i];
    u[c] = a.u0[c * n + i];
    w[c] = dq == c ? cst<T>(1.0) : cst<T>(0.0);
    v[c] = dq == D + c ? cst<T>(1.0) : cst<T>(0.0);
  }
  T L = cst<T>(0.0), dL = cst<T>(0.0);
  int kk = 0, next = S > 0 ? a.save_idx[j] : -1;
  bool ok = true;
  const T* hq = a.h + j;
  for (int st = 0; st < S; ++st) {
    const T h = hq[(int64_t)st * n];
    if (st + 8 < S) prefetch_l2(hq + (int64_t)(st + 8) * n);
    T LU[D * D], R[D], k1[D], vs[D], k2[D], un[D], dun[D];
    int P[D];
    T r[D], t[D], df[D], dk1[D], dk2[D], dU[D];
    // the contract's forward step and the pieces the tangent reuses
    T k3[D];
    if constexpr (METHOD == GS_ROS3)
      ok = kin8_ros3_fwd<T>(u, p, h, LU, P, R, k1, vs, k2, k3, un) && ok;
    else
      ok = kin8_ros2_fwd<T>(u, p, h, LU, P, R, k1, vs, k2, un) && ok;
    const T c = METHOD == GS_ROS3 ? h : cst<T>(ROS2_GAMMA) * h;  // M = I/gamma - h J, or I - gamma h J
    kin8_jvp<T>(u, p, v, w, df);
    kin8_djk<T>(u, p, v, w, k1, t);
#pragma unroll
    for (int q = 0; q < D; ++q) r[q] = fmaT(c, t[q], df[q]);
    lu_d_solve<T, D>(LU, P, R, r, dk1);
#pragma unroll
    for (int q = 0; q < D; ++q) dU[q] = fmaT(h, dk1[q], v[q]);
    kin8_jvp<T>(vs, p, dU, w, df);
    kin8_djk<T>(u, p, v, w, k2, t);
    if constexpr (METHOD == GS_ROS3) {
#pragma unroll
      for (int q = 0; q < D; ++q) r[q] = fmaT(c, t[q], fmaT(cst<T>(ROS3_C21), dk1[q], df[q]));
      lu_d_solve<T, D>(LU, P, R, r, dk2);
      T dk3[D];
      kin8_djk<T>(u, p, v, w, k3, t);
#pragma unroll
      for (int q = 0; q < D; ++q)
        r[q] = fmaT(c, t[q], fmaT(cst<T>(ROS3_C32), dk2[q], fmaT(cst<T>(ROS3_C31), dk1[q], df[q])));
      lu_d_solve<T, D>(LU, P, R, r, dk3);
#pragma unroll
      for (int q = 0; q < D; ++q)
        dun[q] = fmaT(h, fmaT(cst<T>(ROS3_M3), dk3[q], fmaT(cst<T>(ROS3_M2), dk2[q], dk1[q])), v[q]);
    } else {
#pragma unroll
      for (int q = 0; q < D; ++q) r[q] = fmaT(c, t[q], fmaT(cst<T>(-2.0), dk1[q], df[q]));
      lu_d_solve<T, D>(LU, P, R, r, dk2);
#pragma unroll
      for (int q = 0; q < D; ++q) dun[q] = fmaT(h, fmaT(cst<T>(0.5), dk2[q], cst<T>(1.5) * dk1[q]), v[q]);
    }
#pragma unroll
    for (int q = 0; q < D; ++q) {
      u[q] = un[q];
      v[q] = dun[q];
    }
    if (st + 1 == next) {  // a landing record: at most one save point per step
      const int64_t o = (int64_t)kk * nD + i;
#pragma unroll
      for (int q = 0; q < D; ++q) {
        if (a.loss_kind == GS_LOSS_SUMSQ) {
          const T e = a.target ? u[q] - a.target[o + q * n] : u[q];
          L = fmaT(e, e, L);
          dL = fmaT(cst<T>(2.0) * e, v[q], dL);
        } else {
          const T wq = a.weight[o + q * n];
          L = fmaT(wq, u[q], L);
          dL = fmaT(wq, v[q], dL);
        }
        if (a.sens) a.sens[(((int64_t)kk * D + q) * 16 + dq) * n + i] = v[q];
      }
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
  }
  if (!ok) {
    fail();
    return;
  }
  if (dq == 0) a.loss[i] = L;
  (dq < D ? a.dp : a.du0)[(dq % D) * n + i] = dL;
}

template <typename T>
gs_status launch_sens_kin8(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp,
                           void* du0, void* sens, cudaStream_t st) {
  Kin8SensArgs<T> a;
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
  const int bs = kSensKin8Block;
  const unsigned grid = (unsigned)((P->n + bs - 1) / bs * 16);
  if (P->method == GS_ROS3)
    k_sens_kin8<T, GS_ROS3><<<grid, bs, 0, st>>>(a);
  else
    k_sens_kin8<T, GS_ROS2><<<grid, bs, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_sens_kin8<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                            void*, cudaStream_t);
template gs_status launch_sens_kin8<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*,
                                           void*, cudaStream_t);

}  // namespace gs
