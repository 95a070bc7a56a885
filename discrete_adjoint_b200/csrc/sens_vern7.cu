// sens_vern7.cu -- forward sensitivities of the fixed-step replay with
// Verner's 7(6) pair on the Lorenz system: the tangent of the replay along
// each input direction (sigma, rho, beta, x0, y0, z0), integrated alongside
// the state.
//
// The derivative is the one the adjoint returns: the exact derivative of the
// fixed-step replay of the recorded steps, the mesh held as data (GRADSOLVE,
// evolve.pub review, "Strengths: precisely scoped exactness claim").  The
// forward sensitivities integrated beside the state in the same kernel, with
// Verner 7 or Tsit5, are the route of the gist.science summary of arXiv
// 2609.28458 ("Methodology", "Forward Sensitivities"; "Results").
//
// Tangent of one step along a direction (v = du, w = dp):
//   dk_j = J(U_j) dU_j + f_p(U_j) w,   dU_j = v + h sum_{m<j} a_jm dk_m,
//   v' = v + h sum_j b_j dk_j,
// over the pair's nonzero coefficients; k_1 = f(u) at every step (not FSAL).
// The state is the replay's own arithmetic (the order of vern7_step3), so the
// loss is bitwise that of the replay and of gs_grad.
//
// Execution: one thread per (slot, NDIR directions); the 6 / NDIR threads of
// a slot each replay the state.  Every stage state needs all earlier slopes,
// so a step holds 9 slopes x 3 components of the state and of each tangent.
// Measured on the 2^20 Lorenz ensemble (fp64, 234 steps per trajectory): one
// direction per thread 38.8 ms per pass, two 31.7, three 27.3 (238
// registers, no spill), six 31.0 (spilling 0.9 KB).
#include "steps.cuh"
#include "vec.cuh"

namespace gs {

#ifndef GS_SENS_V7_NDIR
#define GS_SENS_V7_NDIR 3
#endif

template <typename T>
struct SensV7Args {
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
};

// J(u) v + f_p(u) w for f = (s (y - x), x (r - z) - y, x y - b z).
template <typename T, typename V>
__device__ __forceinline__ void lorenz_jvp3(const T u[3], T s, T r, T b, const V dv[3], const V& ws, const V& wr,
                                            const V& wb, V g[3]) {
  g[0] = fmaT(s, dv[1] - dv[0], ws * (u[1] - u[0]));
  g[1] = fmaT(r - u[2], dv[0], fmaT(u[0], wr - dv[2], -dv[1]));
  g[2] = fmaT(u[1], dv[0], fmaT(u[0], dv[1], -fmaT(b, dv[2], wb * u[2])));
}

template <typename T, int NDIR>
__global__ void __launch_bounds__(128) k_sens_vern7_lorenz(SensV7Args<T> a) {
  using V = vec<T, NDIR>;
  const int64_t n = a.n;
  constexpr int G = 6 / NDIR;
  const int64_t j = (int64_t)(blockIdx.x / G) * blockDim.x + threadIdx.x;
  const int dir0 = (int)(blockIdx.x % G) * NDIR;  // this thread's directions: dir0 .. dir0 + NDIR - 1
  if (j >= n) return;
  const int64_t i = a.order[j];
  if (i < 0 || i >= n) return;
  const int S = a.nsteps[j];
  const int64_t n3 = 3 * n;
  if (a.status[j] != GS_TRAJ_OK || S < 0 || S > a.smax) {
    const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
    if (dir0 == 0) a.loss[i] = nan;
#pragma unroll
    for (int q = 0; q < NDIR; ++q) {
      const int dq = dir0 + q;
      (dq < 3 ? a.dp : a.du0)[(dq % 3) * n + i] = nan;
      if (a.sens)
        for (int k = 0; k < a.nsave; ++k)
#pragma unroll
          for (int c = 0; c < 3; ++c) a.sens[(((int64_t)k * 3 + c) * 6 + dq) * n + i] = nan;
    }
    return;
  }
  const T pr[3] = {a.p[i], a.p[n + i], a.p[2 * n + i]};
  const T s = pr[0], r = pr[1], b = pr[2];
  T u[3] = {a.u0[i], a.u0[n + i], a.u0[2 * n + i]};
  V ws, wr, wb, v[3];
#pragma unroll
  for (int q = 0; q < NDIR; ++q) {
    const int dq = dir0 + q;
    ws.e[q] = dq == 0 ? cst<T>(1.0) : cst<T>(0.0);
    wr.e[q] = dq == 1 ? cst<T>(1.0) : cst<T>(0.0);
    wb.e[q] = dq == 2 ? cst<T>(1.0) : cst<T>(0.0);
    v[0].e[q] = dq == 3 ? cst<T>(1.0) : cst<T>(0.0);
    v[1].e[q] = dq == 4 ? cst<T>(1.0) : cst<T>(0.0);
    v[2].e[q] = dq == 5 ? cst<T>(1.0) : cst<T>(0.0);
  }
  T L = cst<T>(0.0);
  V dL = vsplat<T, NDIR>(cst<T>(0.0));
  int kk = 0, next = S > 0 ? a.save_idx[j] : -1;
  const T* hq = a.h + j;
  T hn = S > 0 ? hq[0] : cst<T>(0.0);
  for (int st = 0; st < S; ++st) {
    const T h = hn;
    hq += n;
    if (st + 1 < S) hn = *hq;
    if (st + 8 < S) prefetch_l2(hq + 7 * n);
    T k[9][3];
    V dk[9][3];
    rhs3<T, kSysLorenz>(u, pr, k[0]);
    lorenz_jvp3(u, s, r, b, v, ws, wr, wb, dk[0]);
#pragma unroll
    for (int jj = 2; jj <= 9; ++jj) {
      T U[3];
      V dU[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        T acc = cst<T>(v7_a(jj, 1)) * k[0][c];
        V dacc = cst<T>(v7_a(jj, 1)) * dk[0][c];
#pragma unroll
        for (int m = 2; m < jj; ++m)
          if (v7_a(jj, m) != 0.0) {
            acc = fmaT(cst<T>(v7_a(jj, m)), k[m - 1][c], acc);
            dacc = fmaT(cst<T>(v7_a(jj, m)), dk[m - 1][c], dacc);
          }
        U[c] = fmaT(h, acc, u[c]);
        dU[c] = fmaT(h, dacc, v[c]);
      }
      rhs3<T, kSysLorenz>(U, pr, k[jj - 1]);
      lorenz_jvp3(U, s, r, b, dU, ws, wr, wb, dk[jj - 1]);
    }
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      T acc = cst<T>(v7_b(1)) * k[0][c];
      V dacc = cst<T>(v7_b(1)) * dk[0][c];
#pragma unroll
      for (int m = 2; m <= 9; ++m)
        if (v7_b(m) != 0.0) {
          acc = fmaT(cst<T>(v7_b(m)), k[m - 1][c], acc);
          dacc = fmaT(cst<T>(v7_b(m)), dk[m - 1][c], dacc);
        }
      u[c] = fmaT(h, acc, u[c]);
      v[c] = fmaT(h, dacc, v[c]);
    }
    // a landing record has at most one save point per step
    if (st + 1 == next) {
      const int64_t o = (int64_t)kk * n3 + i;
      if (a.loss_kind == GS_LOSS_SUMSQ) {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const T e = a.target ? u[c] - a.target[o + c * n] : u[c];
          L = fmaT(e, e, L);
          dL = fmaT(cst<T>(2.0) * e, v[c], dL);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const T w = a.weight[o + c * n];
          L = fmaT(w, u[c], L);
          dL = fmaT(w, v[c], dL);
        }
      }
      if (a.sens) {
#pragma unroll
        for (int q = 0; q < NDIR; ++q) {
          T* o6 = a.sens + ((int64_t)kk * 18 + dir0 + q) * n + i;
          o6[0] = v[0].e[q];
          o6[6 * n] = v[1].e[q];
          o6[12 * n] = v[2].e[q];
        }
      }
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
  }
  if (dir0 == 0) a.loss[i] = L;
#pragma unroll
  for (int q = 0; q < NDIR; ++q) {
    const int dq = dir0 + q;
    (dq < 3 ? a.dp : a.du0)[(dq % 3) * n + i] = dL.e[q];
  }
}

template <typename T>
gs_status launch_sens_vern7_lorenz(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp,
                                   void* du0, void* sens, cudaStream_t st) {
  SensV7Args<T> a;
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
  constexpr int ND = GS_SENS_V7_NDIR;
  static_assert(6 % ND == 0, "directions per thread must divide 6");
  const int64_t grid = (P->n + 127) / 128 * (6 / ND);
  k_sens_vern7_lorenz<T, ND><<<(unsigned)grid, 128, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_sens_vern7_lorenz<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                    void*, void*, cudaStream_t);
template gs_status launch_sens_vern7_lorenz<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                   void*, void*, cudaStream_t);

}  // namespace gs
