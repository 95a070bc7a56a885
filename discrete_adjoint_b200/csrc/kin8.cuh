// kin8.cuh -- the d = 8 Rosenbrock path: the kin8 system, a D x D LU with
// partial pivoting held in registers, and the ROS2 / ROS3 forward steps at
// d = 8 in the floating-point contract's operation order (so the recorder, the
// replay and the gradient kernels agree bit for bit with any implementation
// that keeps it).
//
// kin8 is an 8-species stiff mass-action network defined by this library (not
// a published test problem; it exercises the Rosenbrock path at d = 8, the
// size of HIRES).  Species A1..A8 = u[0..7], rate constants p[0..7]:
//   r1 = k1 u1      A1 -> A2          r5 = k5 u5      A5 -> A6
//   r2 = k2 u2      A2 -> A1          r6 = k6 u6      A6 -> A5
//   r3 = k3 u2 u3   A2 + A3 -> A4     r7 = k7 u6 u7   A6 + A7 -> A8
//   r4 = k4 u4      A4 -> A3 + A5     r8 = k8 u8      A8 -> A7 + A1
// f = N r(u) with the stoichiometric matrix N of these reactions;
// u1+u2+u4+u5+u6+u8, u3+u4 and u7+u8 are conserved.
#pragma once

#include "steps.cuh"

namespace gs {

constexpr int kSysKin8 = GS_KIN8;

template <typename T>
__device__ __forceinline__ void kin8_f(const T u[8], const T p[8], T f[8]) {
  const T r1 = p[0] * u[0];
  const T r2 = p[1] * u[1];
  const T r3 = p[2] * (u[1] * u[2]);
  const T r4 = p[3] * u[3];
  const T r5 = p[4] * u[4];
  const T r6 = p[5] * u[5];
  const T r7 = p[6] * (u[5] * u[6]);
  const T r8 = p[7] * u[7];
  f[0] = (r2 - r1) + r8;
  f[1] = (r1 - r2) - r3;
  f[2] = r4 - r3;
  f[3] = r3 - r4;
  f[4] = (r4 - r5) + r6;
  f[5] = (r5 - r6) - r7;
  f[6] = r8 - r7;
  f[7] = r7 - r8;
}

// State dimension of each system (all have as many parameters as states), and
// f(u) of any system but the d = 64 one: the dispatch of the recorder and the
// replay.
template <int SYS> struct SysDim { static constexpr int D = 3; };
template <> struct SysDim<GS_KIN8> { static constexpr int D = 8; };

template <typename T, int SYS>
__device__ __forceinline__ void rhs_s(const T* u, const T* p, T* f) {
  if constexpr (SYS == GS_KIN8)
    kin8_f(u, p, f);
  else
    rhs3<T, SYS>(u, p, f);
}

// Jacobian df/du, row-major 8 x 8.
template <typename T>
__device__ __forceinline__ void kin8_J(const T u[8], const T p[8], T J[64]) {
#pragma unroll
  for (int q = 0; q < 64; ++q) J[q] = cst<T>(0.0);
  const T a = p[2] * u[2];  // k3 u3
  const T b = p[2] * u[1];  // k3 u2
  const T c = p[6] * u[6];  // k7 u7
  const T e = p[6] * u[5];  // k7 u6
  J[0 * 8 + 0] = -p[0];
  J[0 * 8 + 1] = p[1];
  J[0 * 8 + 7] = p[7];
  J[1 * 8 + 0] = p[0];
  J[1 * 8 + 1] = -(p[1] + a);
  J[1 * 8 + 2] = -b;
  J[2 * 8 + 1] = -a;
  J[2 * 8 + 2] = -b;
  J[2 * 8 + 3] = p[3];
  J[3 * 8 + 1] = a;
  J[3 * 8 + 2] = b;
  J[3 * 8 + 3] = -p[3];
  J[4 * 8 + 3] = p[3];
  J[4 * 8 + 4] = -p[4];
  J[4 * 8 + 5] = p[5];
  J[5 * 8 + 4] = p[4];
  J[5 * 8 + 5] = -(p[5] + c);
  J[5 * 8 + 6] = -e;
  J[6 * 8 + 5] = -c;
  J[6 * 8 + 6] = -e;
  J[6 * 8 + 7] = p[7];
  J[7 * 8 + 5] = c;
  J[7 * 8 + 6] = e;
  J[7 * 8 + 7] = -p[7];
}

// Per-reaction weights of a vector w: g_r = N[:, r] . w (the change of w . u
// per unit of reaction r).
template <typename T>
__device__ __forceinline__ void kin8_gw(const T w[8], T g[8]) {
  g[0] = w[1] - w[0];
  g[1] = w[0] - w[1];
  g[2] = w[3] - (w[1] + w[2]);
  g[3] = (w[2] + w[4]) - w[3];
  g[4] = w[5] - w[4];
  g[5] = w[4] - w[5];
  g[6] = w[7] - (w[5] + w[6]);
  g[7] = (w[0] + w[6]) - w[7];
}

// ubar += J(u)^T w,  pbar += f_p(u)^T w  (f = N r: J^T w = (dr/du)^T g,
// f_p^T w = (dr/dk)^T g with g = N^T w).
template <typename T>
__device__ __forceinline__ void kin8_vjp(const T u[8], const T p[8], const T w[8], T ub[8], T pb[8]) {
  T g[8];
  kin8_gw(w, g);
  ub[0] = fmaT(p[0], g[0], ub[0]);
  ub[1] = fmaT(p[1], g[1], fmaT(p[2] * u[2], g[2], ub[1]));
  ub[2] = fmaT(p[2] * u[1], g[2], ub[2]);
  ub[3] = fmaT(p[3], g[3], ub[3]);
  ub[4] = fmaT(p[4], g[4], ub[4]);
  ub[5] = fmaT(p[5], g[5], fmaT(p[6] * u[6], g[6], ub[5]));
  ub[6] = fmaT(p[6] * u[5], g[6], ub[6]);
  ub[7] = fmaT(p[7], g[7], ub[7]);
  pb[0] = fmaT(u[0], g[0], pb[0]);
  pb[1] = fmaT(u[1], g[1], pb[1]);
  pb[2] = fmaT(u[1] * u[2], g[2], pb[2]);
  pb[3] = fmaT(u[3], g[3], pb[3]);
  pb[4] = fmaT(u[4], g[4], pb[4]);
  pb[5] = fmaT(u[5], g[5], pb[5]);
  pb[6] = fmaT(u[5] * u[6], g[6], pb[6]);
  pb[7] = fmaT(u[7], g[7], pb[7]);
}

// ubar += d<Jbar, J(u,p)>/du,  pbar += d<Jbar, J(u,p)>/dp for
// Jbar = s sum_i w_i k_i^T.  With J = N dr/du, <Jbar, J> = sum_r G_r . grad_u r_r,
// G_r = Jbar^T N[:, r] = s sum_i g_r(w_i) k_i; only the components of G_r that
// meet a nonzero rate derivative are kept.  add() takes one stage pair
// (w_i, k_i); finish() applies the sums.  The linear rates contribute only to
// pbar; the two bilinear ones (r3, r7) to both.
template <typename T>
struct Kin8JacAdj {
  T G0, G1, G2a, G2b, G3, G4, G5, G6a, G6b, G7;
  __device__ __forceinline__ Kin8JacAdj() {
    G0 = G1 = G2a = G2b = G3 = G4 = G5 = G6a = G6b = G7 = cst<T>(0.0);
  }
  __device__ __forceinline__ void add(const T w[8], const T k[8]) {
    T g[8];
    kin8_gw(w, g);
    G0 = fmaT(g[0], k[0], G0);    // reaction 1 on u1
    G1 = fmaT(g[1], k[1], G1);    // reaction 2 on u2
    G2a = fmaT(g[2], k[1], G2a);  // reaction 3 on u2
    G2b = fmaT(g[2], k[2], G2b);  // reaction 3 on u3
    G3 = fmaT(g[3], k[3], G3);    // reaction 4 on u4
    G4 = fmaT(g[4], k[4], G4);    // reaction 5 on u5
    G5 = fmaT(g[5], k[5], G5);    // reaction 6 on u6
    G6a = fmaT(g[6], k[5], G6a);  // reaction 7 on u6
    G6b = fmaT(g[6], k[6], G6b);  // reaction 7 on u7
    G7 = fmaT(g[7], k[7], G7);    // reaction 8 on u8
  }
  // r3 = k3 u2 u3: <.> += k3 (u3 G2a + u2 G2b); r7 = k7 u6 u7 likewise
  __device__ __forceinline__ void finish(const T u[8], const T p[8], T s, T ub[8], T pb[8]) const {
    const T s3 = s * p[2], s7 = s * p[6];
    ub[1] = fmaT(s3, G2b, ub[1]);
    ub[2] = fmaT(s3, G2a, ub[2]);
    ub[5] = fmaT(s7, G6b, ub[5]);
    ub[6] = fmaT(s7, G6a, ub[6]);
    pb[0] = fmaT(s, G0, pb[0]);
    pb[1] = fmaT(s, G1, pb[1]);
    pb[2] = fmaT(s, fmaT(u[2], G2a, u[1] * G2b), pb[2]);
    pb[3] = fmaT(s, G3, pb[3]);
    pb[4] = fmaT(s, G4, pb[4]);
    pb[5] = fmaT(s, G5, pb[5]);
    pb[6] = fmaT(s, fmaT(u[6], G6a, u[5] * G6b), pb[6]);
    pb[7] = fmaT(s, G7, pb[7]);
  }
};

// ---------------------------------------------------------------------------
// Compile-time loops.  sfor<B, E>(f) calls f(Ix<B>{}) .. f(Ix<E-1>{}); the body
// reads its index as a constant (GS_IX(i)).  The triangular loop nests of an 8 x 8
// LU written with #pragma unroll are not fully unrolled by the compiler, which
// then keeps the matrix in local memory; with constant indices it stays in
// registers.
// ---------------------------------------------------------------------------
template <int I>
struct Ix {
  static constexpr int v = I;
};
template <int B, int E, typename F>
__device__ __forceinline__ void sfor(F&& f) {
  if constexpr (B < E) {
    f(Ix<B>{});
    sfor<B + 1, E>(f);
  }
}
#define GS_IX(x) decltype(x)::v

// ---------------------------------------------------------------------------
// D x D LU with partial pivoting (largest |entry|, ties to the lowest row),
// right-looking, whole rows swap (multipliers included); R receives the
// reciprocals of the pivots.  The row exchange is a select per entry, so M and
// P stay in registers.  Returns false on a zero or non-finite pivot.
// ---------------------------------------------------------------------------
template <typename T, int D>
__device__ __forceinline__ bool lu_d(T M[D * D], int P[D], T R[D]) {
  sfor<0, D>([&](auto q_) { P[GS_IX(q_)] = GS_IX(q_); });
  bool ok = true;
  sfor<0, D>([&](auto k_) {
    constexpr int k = GS_IX(k_);
    int piv = k;
    T best = fabs(M[k * D + k]);
    sfor<k + 1, D>([&](auto i_) {
      constexpr int i = GS_IX(i_);
      const T a = fabs(M[i * D + k]);
      const bool gt = a > best;
      best = gt ? a : best;
      piv = gt ? i : piv;
    });
    sfor<k + 1, D>([&](auto i_) {
      constexpr int i = GS_IX(i_);
      const bool sw = piv == i;
      sfor<0, D>([&](auto j_) {
        constexpr int j = GS_IX(j_);
        const T x = M[k * D + j], y = M[i * D + j];
        M[k * D + j] = sw ? y : x;
        M[i * D + j] = sw ? x : y;
      });
      const int pk = P[k], pi = P[i];
      P[k] = sw ? pi : pk;
      P[i] = sw ? pk : pi;
    });
    const T pv = M[k * D + k];
    ok = ok && (pv != cst<T>(0.0)) && isfinite(pv);
    R[k] = cst<T>(1.0) / pv;
    sfor<k + 1, D>([&](auto i_) {
      constexpr int i = GS_IX(i_);
      const T l = M[i * D + k] * R[k];
      M[i * D + k] = l;
      sfor<k + 1, D>([&](auto j_) {
        constexpr int j = GS_IX(j_);
        M[i * D + j] = fmaT(-l, M[k * D + j], M[i * D + j]);
      });
    });
  });
  return ok;
}

// Solve M x = b with the factors of lu_d (P M = L U): x = P b, forward
// substitution with L (unit diagonal), back substitution with U (times the
// pivot reciprocals), in the contract's order.
template <typename T, int D>
__device__ __forceinline__ void lu_d_solve(const T LU[D * D], const int P[D], const T R[D], const T b[D], T x[D]) {
  sfor<0, D>([&](auto i_) {
    constexpr int i = GS_IX(i_);
    T v = b[0];
    sfor<1, D>([&](auto q_) { v = P[i] == GS_IX(q_) ? b[GS_IX(q_)] : v; });
    x[i] = v;
  });
  sfor<1, D>([&](auto i_) {
    constexpr int i = GS_IX(i_);
    sfor<0, i>([&](auto j_) { x[i] = fmaT(-LU[i * D + GS_IX(j_)], x[GS_IX(j_)], x[i]); });
  });
  sfor<0, D>([&](auto r_) {
    constexpr int i = D - 1 - GS_IX(r_);
    sfor<i + 1, D>([&](auto j_) { x[i] = fmaT(-LU[i * D + GS_IX(j_)], x[GS_IX(j_)], x[i]); });
    x[i] = x[i] * R[i];
  });
}

// Solve M^T x = b with the factors of lu_d (M^T = U^T L^T P): U^T y = b
// (forward), L^T z = y (backward, unit diagonal), x[P[i]] = z[i].  Reverse
// sweep only (not part of the bitwise contract).  lu(e) / rc(i) read the
// caller's factors at compile-time indices.
template <typename T, int D, typename LUA, typename RA>
__device__ __forceinline__ void lu_d_solve_T(LUA lu, RA rc, const int P[D], const T b[D], T x[D]) {
  T y[D];
  sfor<0, D>([&](auto i_) {
    constexpr int i = GS_IX(i_);
    T acc = b[i];
    sfor<0, i>([&](auto j_) { acc = fmaT(-lu(GS_IX(j_) * D + i), y[GS_IX(j_)], acc); });
    y[i] = acc * rc(i);
  });
  sfor<1, D>([&](auto r_) {
    constexpr int i = D - 1 - GS_IX(r_);
    sfor<i + 1, D>([&](auto j_) { y[i] = fmaT(-lu(GS_IX(j_) * D + i), y[GS_IX(j_)], y[i]); });
  });
  sfor<0, D>([&](auto q_) {
    constexpr int q = GS_IX(q_);
    T v = y[0];
    sfor<1, D>([&](auto i_) { v = P[GS_IX(i_)] == q ? y[GS_IX(i_)] : v; });
    x[q] = v;
  });
}

// ---------------------------------------------------------------------------
// ROS2 / ROS3 forward steps at d = 8 (the stage equations of the d = 3 forms
// in steps.cuh).  Each returns the pieces its reverse sweep needs.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ bool kin8_ros2_fwd(const T u[8], const T p[8], T h, T LU[64], int P[8], T R[8], T k1[8],
                                              T v[8], T k2[8], T un[8]) {
  kin8_J(u, p, LU);
  const T gh = cst<T>(ROS2_GAMMA) * h;
#pragma unroll
  for (int q = 0; q < 64; ++q) LU[q] = fmaT(-gh, LU[q], cst<T>((q % 9) == 0 ? 1.0 : 0.0));
  const bool ok = lu_d<T, 8>(LU, P, R);
  T f[8];
  kin8_f(u, p, f);
  lu_d_solve<T, 8>(LU, P, R, f, k1);
#pragma unroll
  for (int c = 0; c < 8; ++c) v[c] = fmaT(h, k1[c], u[c]);
  kin8_f(v, p, f);
#pragma unroll
  for (int c = 0; c < 8; ++c) f[c] = fmaT(cst<T>(-2.0), k1[c], f[c]);
  lu_d_solve<T, 8>(LU, P, R, f, k2);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    T acc = cst<T>(1.5) * k1[c];
    acc = fmaT(cst<T>(0.5), k2[c], acc);
    un[c] = fmaT(h, acc, u[c]);
  }
  return ok;
}

template <typename T>
__device__ __forceinline__ bool kin8_ros3_fwd(const T u[8], const T p[8], T h, T LU[64], int P[8], T R[8], T k1[8],
                                              T v[8], T k2[8], T k3[8], T un[8]) {
  kin8_J(u, p, LU);
#pragma unroll
  for (int q = 0; q < 64; ++q) LU[q] = fmaT(-h, LU[q], cst<T>((q % 9) == 0 ? ROS3_INV_GAMMA : 0.0));
  const bool ok = lu_d<T, 8>(LU, P, R);
  T f[8], r[8];
  kin8_f(u, p, f);
  lu_d_solve<T, 8>(LU, P, R, f, k1);
#pragma unroll
  for (int c = 0; c < 8; ++c) v[c] = fmaT(h, k1[c], u[c]);
  kin8_f(v, p, f);
#pragma unroll
  for (int c = 0; c < 8; ++c) r[c] = fmaT(cst<T>(ROS3_C21), k1[c], f[c]);
  lu_d_solve<T, 8>(LU, P, R, r, k2);
#pragma unroll
  for (int c = 0; c < 8; ++c) r[c] = fmaT(cst<T>(ROS3_C32), k2[c], fmaT(cst<T>(ROS3_C31), k1[c], f[c]));
  lu_d_solve<T, 8>(LU, P, R, r, k3);
#pragma unroll
  for (int c = 0; c < 8; ++c) un[c] = fmaT(h, fmaT(cst<T>(ROS3_M3), k3[c], fmaT(cst<T>(ROS3_M2), k2[c], k1[c])), u[c]);
  return ok;
}

// Steps with the embedded error estimate (the recorder's).
template <typename T>
__device__ __forceinline__ bool kin8_ros2_err_step(const T u[8], const T p[8], T h, T un[8], T e[8]) {
  T LU[64], R[8], k1[8], v[8], k2[8];
  int P[8];
  const bool ok = kin8_ros2_fwd(u, p, h, LU, P, R, k1, v, k2, un);
#pragma unroll
  for (int c = 0; c < 8; ++c) e[c] = (h * cst<T>(0.5)) * (k1[c] + k2[c]);
  return ok;
}

template <typename T>
__device__ __forceinline__ bool kin8_ros3_err_step(const T u[8], const T p[8], T h, T un[8], T e[8]) {
  T LU[64], R[8], k1[8], v[8], k2[8], k3[8];
  int P[8];
  const bool ok = kin8_ros3_fwd(u, p, h, LU, P, R, k1, v, k2, k3, un);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    e[c] = h * fmaT(cst<T>(ROS3_E3), k3[c], fmaT(cst<T>(ROS3_E2), k2[c], cst<T>(ROS3_E1) * k1[c]));
  return ok;
}

}  // namespace gs
