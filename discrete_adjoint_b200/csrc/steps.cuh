// steps.cuh -- the d = 3 step formulas of the forward replay (Tsit5, ROS2
// and ROS3 on Lorenz and Robertson), written in the floating-point contract's
// operation order.  Shared by the recorder, the Rosenbrock gradient kernels
// and the forward-only solve (kin8.cuh adds the d = 8 system on top).
#pragma once

#include "common.cuh"

namespace gs {

constexpr int kSysLorenz = GS_LORENZ;
constexpr int kSysRobertson = GS_ROBERTSON;

// std::max / std::min semantics (the CPU reference's), NaN included.
template <typename T> __device__ __forceinline__ T smax_(T a, T b) { return (a < b) ? b : a; }
template <typename T> __device__ __forceinline__ T smin_(T a, T b) { return (b < a) ? b : a; }

template <typename T, int SYS>
__device__ __forceinline__ void rhs3(const T u[3], const T p[3], T f[3]) {
  if (SYS == kSysLorenz)
    lorenz_f(u[0], u[1], u[2], p[0], p[1], p[2], f[0], f[1], f[2]);
  else
    robertson_f(u[0], u[1], u[2], p[0], p[1], p[2], f[0], f[1], f[2]);
}

template <typename T, int SYS>
__device__ __forceinline__ void jac3(const T u[3], const T p[3], T J[9]) {
  if (SYS == kSysLorenz) {
    J[0] = -p[0];
    J[1] = p[0];
    J[2] = cst<T>(0.0);
    J[3] = p[1] - u[2];
    J[4] = cst<T>(-1.0);
    J[5] = -u[0];
    J[6] = u[1];
    J[7] = u[0];
    J[8] = -p[2];
  } else {
    robertson_J(u[0], u[1], u[2], p[0], p[1], p[2], J);
  }
}

// Logarithm and exponential for the step-size controller (its powers are
// x^y = exp(y ln x)).  Library pow may differ from other implementations by an
// ulp, and the embedded error estimate (a sum with heavy
// cancellation) turns such an ulp into ~1e-10 relative step-size differences
// within a few steps, which chaos then amplifies.  This one uses only IEEE
// +, -, *, /, fma and the exact frexp / ldexp / rint, in a fixed order, so its
// bits are reproducible on any IEEE machine that keeps the order:
//   ln x : x = m 2^e, m in [sqrt(1/2), sqrt(2)); ln m = 2 atanh(s),
//          s = (m-1)/(m+1), series s (1 + z/3 + ... + z^12/25), z = s^2,
//          the polynomial by Estrin's scheme;
//   exp w: Cody & Waite reduction w = k ln2 + r (ln2 = 21-bit head + tail),
//          Taylor polynomial of e^r to degree 14 by Estrin's scheme, times 2^k.
// Accuracy: ~1 ulp for the controller's arguments (errors 1e-4..1e3, |y| <= 1).
__device__ __forceinline__ double frexpT(double x, int* e) { return frexp(x, e); }
__device__ __forceinline__ float frexpT(float x, int* e) { return frexpf(x, e); }
__device__ __forceinline__ double ldexpT(double x, int e) { return ldexp(x, e); }
__device__ __forceinline__ float ldexpT(float x, int e) { return ldexpf(x, e); }
__device__ __forceinline__ double rintT(double x) { return rint(x); }
__device__ __forceinline__ float rintT(float x) { return rintf(x); }

template <typename T>
__device__ T ctrl_ln(T x) {  // x > 0 finite
  int e = 0;
  T m = frexpT(x, &e);
  if (m < cst<T>(0.7071067811865476)) {
    m = m + m;
    e = e - 1;
  }
  const T s = (m - cst<T>(1.0)) / (m + cst<T>(1.0));
  const T z = s * s;
  // sum_{k=0..12} z^k / (2k+1), Estrin's scheme: pairs in z, then z^2, z^4,
  // z^8 (four dependent levels)
#define GS_LNC(k) cst<T>(1.0 / double(2 * (k) + 1))
  const T z2 = z * z, z4 = z2 * z2, z8 = z4 * z4;
  const T q0 = fmaT(GS_LNC(1), z, GS_LNC(0)), q1 = fmaT(GS_LNC(3), z, GS_LNC(2)), q2 = fmaT(GS_LNC(5), z, GS_LNC(4));
  const T q3 = fmaT(GS_LNC(7), z, GS_LNC(6)), q4 = fmaT(GS_LNC(9), z, GS_LNC(8)), q5 = fmaT(GS_LNC(11), z, GS_LNC(10));
  const T r0 = fmaT(q1, z2, q0), r1 = fmaT(q3, z2, q2), r2 = fmaT(q5, z2, q4);
  const T s0 = fmaT(r1, z4, r0), s1 = fmaT(GS_LNC(12), z4, r2);
  const T poly = fmaT(s1, z8, s0);
#undef GS_LNC
  const T lnm = (s + s) * poly;
  const T ef = (T)e;
  return fmaT(ef, cst<T>(0.6931467056274414), fmaT(ef, cst<T>(4.7493250390316726e-07), lnm));
}

template <typename T>
__device__ T ctrl_exp(T w) {
  if (isnan(w)) return w;
  const T kf = rintT(w * cst<T>(1.4426950408889634));
  if (kf > cst<T>(2000.0)) return cst<T>(1.0) / cst<T>(0.0);
  if (kf < cst<T>(-2000.0)) return cst<T>(0.0);
  T r = fmaT(-kf, cst<T>(0.6931467056274414), w);
  r = fmaT(-kf, cst<T>(4.7493250390316726e-07), r);
  // Horner over 1/j!, j = 14 .. 0 (j! exact in double for j <= 14)
  constexpr double inv_fact[15] = {1.0,
                                   1.0,
                                   1.0 / 2.0,
                                   1.0 / 6.0,
                                   1.0 / 24.0,
                                   1.0 / 120.0,
                                   1.0 / 720.0,
                                   1.0 / 5040.0,
                                   1.0 / 40320.0,
                                   1.0 / 362880.0,
                                   1.0 / 3628800.0,
                                   1.0 / 39916800.0,
                                   1.0 / 479001600.0,
                                   1.0 / 6227020800.0,
                                   1.0 / 87178291200.0};
  // Estrin's scheme: pairs in r, then r^2, r^4, r^8 (four dependent levels)
  const T r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
  T q[7];
#pragma unroll
  for (int i = 0; i < 7; ++i) q[i] = fmaT(cst<T>(inv_fact[2 * i + 1]), r, cst<T>(inv_fact[2 * i]));
  const T t0 = fmaT(q[1], r2, q[0]), t1 = fmaT(q[3], r2, q[2]), t2 = fmaT(q[5], r2, q[4]);
  const T t3 = fmaT(cst<T>(inv_fact[14]), r2, q[6]);
  const T u0 = fmaT(t1, r4, t0), u1 = fmaT(t3, r4, t2);
  const T p = fmaT(u1, r8, u0);
  return ldexpT(p, (int)kf);
}

template <typename T>
__device__ T ctrl_pow(T x, T y) {
  if (isnan(x) || isnan(y)) return x + y;
  if (x == cst<T>(0.0)) return y > cst<T>(0.0) ? cst<T>(0.0) : (y < cst<T>(0.0) ? cst<T>(1.0) / x : cst<T>(1.0));
  if (isinf(x)) return y > cst<T>(0.0) ? x : (y < cst<T>(0.0) ? cst<T>(0.0) : cst<T>(1.0));
  return ctrl_exp<T>(y * ctrl_ln<T>(x));
}

// Dense output of the Rosenbrock methods inside one step [t_s, t_s + h] at
// theta in (0, 1]: the cubic Hermite interpolant on the end states and slopes,
//   u = H00 u_s + H01 u_{s+1} + h (H10 f(u_s) + H11 f(u_{s+1})),
// weights and combination in the floating-point contract's order (the same
// operations as the CPU reference, so the values agree bit for bit).
template <typename T>
struct HermiteW {
  T h00, h01, h10, h11;
};

template <typename T>
__device__ __forceinline__ HermiteW<T> hermite_w(T th) {
  const T t2 = th * th, om = cst<T>(1.0) - th;
  HermiteW<T> w;
  w.h01 = t2 * fmaT(cst<T>(-2.0), th, cst<T>(3.0));
  w.h00 = cst<T>(1.0) - w.h01;
  w.h10 = (th * om) * om;
  w.h11 = -(t2 * om);
  return w;
}

template <typename T>
__device__ __forceinline__ T hermite_c(const HermiteW<T>& w, T us, T un, T fs, T fn, T h) {
  return fmaT(w.h00, us, fmaT(w.h01, un, h * fmaT(w.h10, fs, w.h11 * fn)));
}

// Tsit5's dense output: Tsitouras' continuous extension of the pair.  The
// state at t_s + theta h is u_s + h sum_i b_i(theta) k_i over the seven
// stages (k_7 = f(u_{s+1})), b_i(theta) = sum_m ts_r(i, m-1) theta^m, fourth
// order for every theta, b(1) = b, and C1 across step ends.  Weights in the
// contract's order:
//   P_i = fma(fma(r_i4, theta, r_i3), theta, r_i2),
//   b_1 = fma(theta^2, P_1, theta),  b_i = theta^2 P_i (i >= 2).
__host__ __device__ constexpr double ts_r(int i, int m) {
  constexpr double v[7][4] = {{1.0, -2.763706197274826, 2.9132554618219126, -1.0530884977290216},
                              {0.0, 0.13169999999999998, -0.2234, 0.1017},
                              {0.0, 3.9302962368947516, -5.941033872131505, 2.490627285651253},
                              {0.0, -12.411077166933676, 30.33818863028232, -16.548102889244902},
                              {0.0, 37.50931341651104, -88.1789048947664, 47.37952196281928},
                              {0.0, -27.896526289197286, 65.09189467479366, -34.87065786149660},
                              {0.0, 1.5, -4.0, 2.5}};
  return v[i][m];
}

template <typename T>
__device__ __forceinline__ void tsit5_dense_w(T th, T bw[7]) {
  const T t2 = th * th;
#pragma unroll
  for (int i = 0; i < 7; ++i) {
    const T P = fmaT(fmaT(cst<T>(ts_r(i, 3)), th, cst<T>(ts_r(i, 2))), th, cst<T>(ts_r(i, 1)));
    bw[i] = i == 0 ? fmaT(t2, P, th) : t2 * P;
  }
}

// u(theta) = fma(h, b_1 k_1 + ... + b_7 k_7, u_s), the sum an fma chain in
// increasing i, for one component.
template <typename T>
__device__ __forceinline__ T tsit5_dense_c(const T bw[7], T us, T k1, T k2, T k3, T k4, T k5, T k6, T k7, T h) {
  T acc = bw[0] * k1;
  acc = fmaT(bw[1], k2, acc);
  acc = fmaT(bw[2], k3, acc);
  acc = fmaT(bw[3], k4, acc);
  acc = fmaT(bw[4], k5, acc);
  acc = fmaT(bw[5], k6, acc);
  acc = fmaT(bw[6], k7, acc);
  return fmaT(h, acc, us);
}

// The dense output of one Tsit5 step of size h from u (k1 = f(u)) at theta:
// the stages recomputed in the step's own order (bitwise those of the step).
// Not inlined: it runs only at a dense save point, and inlined into a
// recorder loop its stages would raise the register pressure of every
// attempt.  Arguments and result travel by value.
template <typename T>
struct Tri {
  T v[3];
};

template <typename T, int SYS>
__device__ __noinline__ Tri<T> tsit5_dense3_call(Tri<T> uu, Tri<T> pp, T h, Tri<T> kk1, T th) {
  const T* u = uu.v;
  const T* p = pp.v;
  const T* k1 = kk1.v;
  Tri<T> out;
  T k2[3], k3[3], k4[3], k5[3], k6[3], k7[3], U[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) U[c] = fmaT(h, tsc<T, kTsA21>() * k1[c], u[c]);
  rhs3<T, SYS>(U, p, k2);
#pragma unroll
  for (int c = 0; c < 3; ++c) U[c] = fmaT(h, fmaT(tsc<T, kTsA32>(), k2[c], tsc<T, kTsA31>() * k1[c]), u[c]);
  rhs3<T, SYS>(U, p, k3);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsA41>() * k1[c];
    acc = fmaT(tsc<T, kTsA42>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsA43>(), k3[c], acc);
    U[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(U, p, k4);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsA51>() * k1[c];
    acc = fmaT(tsc<T, kTsA52>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsA53>(), k3[c], acc);
    acc = fmaT(tsc<T, kTsA54>(), k4[c], acc);
    U[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(U, p, k5);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsA61>() * k1[c];
    acc = fmaT(tsc<T, kTsA62>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsA63>(), k3[c], acc);
    acc = fmaT(tsc<T, kTsA64>(), k4[c], acc);
    acc = fmaT(tsc<T, kTsA65>(), k5[c], acc);
    U[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(U, p, k6);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsB1>() * k1[c];
    acc = fmaT(tsc<T, kTsB2>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsB3>(), k3[c], acc);
    acc = fmaT(tsc<T, kTsB4>(), k4[c], acc);
    acc = fmaT(tsc<T, kTsB5>(), k5[c], acc);
    acc = fmaT(tsc<T, kTsB6>(), k6[c], acc);
    U[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(U, p, k7);
  T bw[7];
  tsit5_dense_w(th, bw);
#pragma unroll
  for (int c = 0; c < 3; ++c) out.v[c] = tsit5_dense_c(bw, u[c], k1[c], k2[c], k3[c], k4[c], k5[c], k6[c], k7[c], h);
  return out;
}

template <typename T, int SYS>
__device__ __forceinline__ void tsit5_dense3(const T u[3], const T p[3], T h, const T k1[3], T th, T out[3]) {
  const Tri<T> r = tsit5_dense3_call<T, SYS>(Tri<T>{{u[0], u[1], u[2]}}, Tri<T>{{p[0], p[1], p[2]}}, h,
                                             Tri<T>{{k1[0], k1[1], k1[2]}}, th);
#pragma unroll
  for (int c = 0; c < 3; ++c) out[c] = r.v[c];
}

// RMS of x / sc over D components (the error norm), in the contract's order.
template <typename T, int D>
__device__ __forceinline__ T rms_d(const T* x, const T* sc) {
  T s = cst<T>(0.0);
#pragma unroll
  for (int c = 0; c < D; ++c) {
    T q = x[c] / sc[c];
    s = fmaT(q, q, s);
  }
  return sqrt(s / cst<T>((double)D));
}

// One Tsit5 step with error estimate; k1 = f(u) on entry, k7 = f(u_new) out.
template <typename T, int SYS>
__device__ __forceinline__ void tsit5_err_step(const T u[3], const T p[3], T h, const T k1[3], T un[3], T k7[3],
                                               T e[3]) {
  T k2[3], k3[3], k4[3], k5[3], k6[3], U[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) U[c] = fmaT(h, tsc<T, kTsA21>() * k1[c], u[c]);
  rhs3<T, SYS>(U, p, k2);
#pragma unroll
  for (int c = 0; c < 3; ++c) U[c] = fmaT(h, fmaT(tsc<T, kTsA32>(), k2[c], tsc<T, kTsA31>() * k1[c]), u[c]);
  rhs3<T, SYS>(U, p, k3);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsA41>() * k1[c];
    acc = fmaT(tsc<T, kTsA42>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsA43>(), k3[c], acc);
    U[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(U, p, k4);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsA51>() * k1[c];
    acc = fmaT(tsc<T, kTsA52>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsA53>(), k3[c], acc);
    acc = fmaT(tsc<T, kTsA54>(), k4[c], acc);
    U[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(U, p, k5);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsA61>() * k1[c];
    acc = fmaT(tsc<T, kTsA62>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsA63>(), k3[c], acc);
    acc = fmaT(tsc<T, kTsA64>(), k4[c], acc);
    acc = fmaT(tsc<T, kTsA65>(), k5[c], acc);
    U[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(U, p, k6);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsB1>() * k1[c];
    acc = fmaT(tsc<T, kTsB2>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsB3>(), k3[c], acc);
    acc = fmaT(tsc<T, kTsB4>(), k4[c], acc);
    acc = fmaT(tsc<T, kTsB5>(), k5[c], acc);
    acc = fmaT(tsc<T, kTsB6>(), k6[c], acc);
    un[c] = fmaT(h, acc, u[c]);
  }
  rhs3<T, SYS>(un, p, k7);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = tsc<T, kTsE1>() * k1[c];
    acc = fmaT(tsc<T, kTsE2>(), k2[c], acc);
    acc = fmaT(tsc<T, kTsE3>(), k3[c], acc);
    acc = fmaT(tsc<T, kTsE4>(), k4[c], acc);
    acc = fmaT(tsc<T, kTsE5>(), k5[c], acc);
    acc = fmaT(tsc<T, kTsE6>(), k6[c], acc);
    acc = fmaT(tsc<T, kTsE7>(), k7[c], acc);
    e[c] = h * acc;
  }
}

// One step of Verner's 7(6) pair (k1 = f(u) on entry): stage j's state is
// acc = a_j1 k1, then acc = fma(a_jm, k_m, acc) over the nonzero a_jm in
// increasing m, U_j = fma(h, acc, u); u_new the same over the nonzero b_m.
// With E != nullptr, stage 10 and the embedded error estimate
// e = h (E_1 k_1 + ... over the nonzero E_m), E = b - bhat.  The operation
// order is the floating-point contract of the method.
template <typename T, int SYS>
__device__ __forceinline__ void vern7_step3(const T u[3], const T p[3], T h, const T k1[3], T un[3], T* e) {
  T k[10][3], U[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) k[0][c] = k1[c];
#pragma unroll
  for (int j = 2; j <= 10; ++j) {
    if (j == 10 && e == nullptr) break;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      T acc = cst<T>(v7_a(j, 1)) * k[0][c];
#pragma unroll
      for (int m = 2; m < j; ++m)
        if (v7_a(j, m) != 0.0) acc = fmaT(cst<T>(v7_a(j, m)), k[m - 1][c], acc);
      U[c] = fmaT(h, acc, u[c]);
    }
    rhs3<T, SYS>(U, p, k[j - 1]);
  }
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = cst<T>(v7_b(1)) * k[0][c];
#pragma unroll
    for (int m = 2; m <= 9; ++m)
      if (v7_b(m) != 0.0) acc = fmaT(cst<T>(v7_b(m)), k[m - 1][c], acc);
    un[c] = fmaT(h, acc, u[c]);
  }
  if (e == nullptr) return;
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = cst<T>(v7_e(1)) * k[0][c];
#pragma unroll
    for (int m = 2; m <= 10; ++m)
      if (v7_e(m) != 0.0) acc = fmaT(cst<T>(v7_e(m)), k[m - 1][c], acc);
    e[c] = h * acc;
  }
}

// One ROS2 step with error estimate.  Returns false on a singular matrix.
template <typename T, int SYS>
__device__ __forceinline__ bool ros2_err_step(const T u[3], const T p[3], T h, T un[3], T e[3]) {
  T J[9], M[9], R[3];
  int P[3];
  jac3<T, SYS>(u, p, J);
  const T gh = cst<T>(ROS2_GAMMA) * h;
#pragma unroll
  for (int q = 0; q < 9; ++q) M[q] = fmaT(-gh, J[q], cst<T>((q % 4) == 0 ? 1.0 : 0.0));
  if (!lu3(M, P, R)) return false;
  T f0[3], k1[3], v[3], f1[3], k2[3];
  rhs3<T, SYS>(u, p, f0);
  lu3_solve(M, P, R, f0[0], f0[1], f0[2], k1[0], k1[1], k1[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) v[c] = fmaT(h, k1[c], u[c]);
  rhs3<T, SYS>(v, p, f1);
  T r0 = fmaT(cst<T>(-2.0), k1[0], f1[0]);
  T r1 = fmaT(cst<T>(-2.0), k1[1], f1[1]);
  T r2 = fmaT(cst<T>(-2.0), k1[2], f1[2]);
  lu3_solve(M, P, R, r0, r1, r2, k2[0], k2[1], k2[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = cst<T>(1.5) * k1[c];
    acc = fmaT(cst<T>(0.5), k2[c], acc);
    un[c] = fmaT(h, acc, u[c]);
    e[c] = (h * cst<T>(0.5)) * (k1[c] + k2[c]);
  }
  return true;
}

// Bitwise forward step; also returns the pieces the reverse sweep needs.
template <typename T, int SYS>
__device__ __forceinline__ bool ros2_fwd(const T u[3], const T p[3], T h, T LU[9], int P[3], T R[3], T k1[3],
                                         T v[3], T k2[3], T un[3]) {
  T J[9];
  jac3<T, SYS>(u, p, J);
  const T gh = cst<T>(ROS2_GAMMA) * h;
#pragma unroll
  for (int q = 0; q < 9; ++q) LU[q] = fmaT(-gh, J[q], cst<T>((q % 4) == 0 ? 1.0 : 0.0));
  bool ok = lu3(LU, P, R);
  T f0[3], f1[3];
  rhs3<T, SYS>(u, p, f0);
  lu3_solve(LU, P, R, f0[0], f0[1], f0[2], k1[0], k1[1], k1[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) v[c] = fmaT(h, k1[c], u[c]);
  rhs3<T, SYS>(v, p, f1);
  T r0 = fmaT(cst<T>(-2.0), k1[0], f1[0]);
  T r1 = fmaT(cst<T>(-2.0), k1[1], f1[1]);
  T r2 = fmaT(cst<T>(-2.0), k1[2], f1[2]);
  lu3_solve(LU, P, R, r0, r1, r2, k2[0], k2[1], k2[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T acc = cst<T>(1.5) * k1[c];
    acc = fmaT(cst<T>(0.5), k2[c], acc);
    un[c] = fmaT(h, acc, u[c]);
  }
  return ok;
}

// ROS3 (Sandu et al. 1997) in the transformed stage form with k_i = K_i / h:
//   M = I/gamma - h J(u);  M k1 = f(u);  v = u + h k1;
//   M k2 = f(v) + c21 k1;  M k3 = f(v) + c31 k1 + c32 k2;
//   u_new = u + h (k1 + m2 k2 + m3 k3);  e = h (e1 k1 + e2 k2 + e3 k3).
// The operation order below is the floating-point contract of the method.
template <typename T, int SYS>
__device__ __forceinline__ bool ros3_fwd(const T u[3], const T p[3], T h, T LU[9], int P[3], T R[3], T k1[3],
                                         T v[3], T k2[3], T k3[3], T un[3]) {
  T J[9];
  jac3<T, SYS>(u, p, J);
#pragma unroll
  for (int q = 0; q < 9; ++q) LU[q] = fmaT(-h, J[q], cst<T>((q % 4) == 0 ? ROS3_INV_GAMMA : 0.0));
  bool ok = lu3(LU, P, R);
  T f0[3], f1[3];
  rhs3<T, SYS>(u, p, f0);
  lu3_solve(LU, P, R, f0[0], f0[1], f0[2], k1[0], k1[1], k1[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) v[c] = fmaT(h, k1[c], u[c]);
  rhs3<T, SYS>(v, p, f1);
  lu3_solve(LU, P, R, fmaT(cst<T>(ROS3_C21), k1[0], f1[0]), fmaT(cst<T>(ROS3_C21), k1[1], f1[1]),
            fmaT(cst<T>(ROS3_C21), k1[2], f1[2]), k2[0], k2[1], k2[2]);
  T r[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) r[c] = fmaT(cst<T>(ROS3_C32), k2[c], fmaT(cst<T>(ROS3_C31), k1[c], f1[c]));
  lu3_solve(LU, P, R, r[0], r[1], r[2], k3[0], k3[1], k3[2]);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const T acc = fmaT(cst<T>(ROS3_M3), k3[c], fmaT(cst<T>(ROS3_M2), k2[c], k1[c]));
    un[c] = fmaT(h, acc, u[c]);
  }
  return ok;
}

// One ROS3 step with error estimate.  Returns false on a singular matrix.
template <typename T, int SYS>
__device__ __forceinline__ bool ros3_err_step(const T u[3], const T p[3], T h, T un[3], T e[3]) {
  T LU[9], R[3], k1[3], v[3], k2[3], k3[3];
  int P[3];
  if (!ros3_fwd<T, SYS>(u, p, h, LU, P, R, k1, v, k2, k3, un)) return false;
#pragma unroll
  for (int c = 0; c < 3; ++c)
    e[c] = h * fmaT(cst<T>(ROS3_E3), k3[c], fmaT(cst<T>(ROS3_E2), k2[c], cst<T>(ROS3_E1) * k1[c]));
  return true;
}

}  // namespace gs
