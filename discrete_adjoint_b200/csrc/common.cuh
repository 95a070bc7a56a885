// common.cuh -- device-side building blocks shared by the kernels of
// libgradsolve: method constants, registered right-hand sides, the step
// formulas of the forward replay, and the host-side launch bookkeeping.
//
// Floating-point contract.  The forward arithmetic of every step (stage
// sums, right-hand sides, Rosenbrock LU and solves, error norm, loss) follows
// one fixed operation order with explicit fused multiply-adds; this library
// is compiled with -fmad=false so that no other multiply-add is fused.  A
// replay is then bitwise reproducible by any IEEE implementation that keeps
// the same order, which is what lets a chaotic 10-time-unit Lorenz replay be
// checked to 1e-12.  The reverse sweep uses fused multiply-adds freely.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gradsolve.h"

namespace gs {

// ---------------------------------------------------------------------------
// Tsitouras (2011) 5(4) pair.  TS_Ajm: stage j's weight on slope m; row 7 is
// the propagating weight vector b (FSAL).  TS_Ej = b_j - bhat_j, the weights of
// the embedded error estimate.
// ---------------------------------------------------------------------------
#define TS_A21 0.161
#define TS_A31 (-0.008480655492356989)
#define TS_A32 0.335480655492357
#define TS_A41 2.897153057105493
#define TS_A42 (-6.359448489975075)
#define TS_A43 4.3622954328695815
#define TS_A51 5.325864828439257
#define TS_A52 (-11.748883564062828)
#define TS_A53 7.4955393428898365
#define TS_A54 (-0.09249506636175525)
#define TS_A61 5.86145544294642
#define TS_A62 (-12.92096931784711)
#define TS_A63 8.159367898576159
#define TS_A64 (-0.071584973281401)
#define TS_A65 (-0.028269050394068383)
#define TS_B1 0.09646076681806523
#define TS_B2 0.01
#define TS_B3 0.4798896504144996
#define TS_B4 1.379008574103742
#define TS_B5 (-3.290069515436081)
#define TS_B6 2.324710524099774
#define TS_E1 (-0.00178001105222577714)
#define TS_E2 (-0.0008164344596567469)
#define TS_E3 0.007880878010261995
#define TS_E4 (-0.1447110071732629)
#define TS_E5 0.5823571654525552
#define TS_E6 (-0.45808210592918697)
#define TS_E7 (1.0 / 66.0)

// ROS2 (Verwer, Spee, Blom & Hundsdorfer 1999): gamma = 1 + 1/sqrt(2).
#define ROS2_GAMMA 1.7071067811865475

// ROS3 (Sandu, Verwer, Blom, Spee, Carmichael & Potra 1997): three stages,
// order 3, L-stable, embedded order 2.  Coefficients of the transformed stage
// form (a21 = a31 = 1, a32 = 0, m1 = 1) rounded to double; gamma is the root
// in (1/6, 1/2) of x^3 - 3x^2 + 3/2 x - 1/6, ROS3_INV_GAMMA its reciprocal
// rounded once.
#define ROS3_INV_GAMMA 2.294280360279042
#define ROS3_C21 (-1.0156171083877703)
#define ROS3_C31 4.07599564525377
#define ROS3_C32 9.20767942983308
#define ROS3_M2 6.1697947043828245
#define ROS3_M3 (-0.42772256543218573)
#define ROS3_E1 0.5
#define ROS3_E2 (-2.907955871680547)
#define ROS3_E3 0.2235406989781157

// Error order q of the step-size controller for each method: the local error
// estimate of Tsit5 is O(h^5), of ROS2 O(h^2), of ROS3 O(h^3), of Verner's
// 7(6) pair O(h^7).
__host__ __device__ constexpr double method_order(int method) {
  return method == GS_TSIT5 ? 5.0 : (method == GS_ROS3 ? 3.0 : (method == GS_VERN7 ? 7.0 : 2.0));
}

// ---------------------------------------------------------------------------
// Verner's 7(6) pair: v7_a(j, m) is stage j's weight on slope m (1-based,
// m < j <= 10, zero where the pair has none), v7_b(m) the seventh-order
// weights, v7_e(m) = b_m - bhat_m the weights of the embedded error estimate
// (one double subtraction of the two stored weights).
// ---------------------------------------------------------------------------
__host__ __device__ constexpr double v7_a(int j, int m) {
  constexpr double a[10][9] = {
      {0, 0, 0, 0, 0, 0, 0, 0, 0},
      {0.005, 0, 0, 0, 0, 0, 0, 0, 0},
      {-1.07679012345679, 1.185679012345679, 0, 0, 0, 0, 0, 0, 0},
      {0.04083333333333333, 0, 0.1225, 0, 0, 0, 0, 0, 0},
      {0.6389139236255726, 0, -2.455672638223657, 2.272258714598084, 0, 0, 0, 0, 0},
      {-2.6615773750187572, 0, 10.804513886456137, -8.3539146573962, 0.820487594956657, 0, 0, 0, 0},
      {6.067741434696772, 0, -24.711273635911088, 20.427517930788895, -1.9061579788166472, 1.006172249242068, 0,
       0, 0},
      {12.054670076253203, 0, -49.75478495046899, 41.142888638604674, -4.461760149974004, 2.042334822239175,
       -0.09834843665406107, 0, 0},
      {10.138146522881808, 0, -42.6411360317175, 35.76384003992257, -4.3480228403929075, 2.0098622683770357,
       0.3487490460338272, -0.27143900510483127, 0},
      {-45.030072034298676, 0, 187.3272437654589, -154.02882369350186, 18.56465306347536, -7.141809679295079,
       1.3088085781613787, 0, 0}};
  return a[j - 1][m - 1];
}
__host__ __device__ constexpr double v7_b(int m) {
  constexpr double b[10] = {0.04715561848627222, 0, 0, 0.25750564298434153, 0.26216653977412624,
                            0.15216092656738558, 0.4939969170032485, -0.29430311714032503, 0.08131747232495111, 0};
  return b[m - 1];
}
__host__ __device__ constexpr double v7_bhat(int m) {
  constexpr double b[10] = {0.044608606606341174, 0, 0, 0.26716403785713727, 0.22010183001772932,
                            0.2188431703143157, 0.22898717054112028, 0, 0, 0.02029518466335628};
  return b[m - 1];
}
__host__ __device__ constexpr double v7_e(int m) { return v7_b(m) - v7_bhat(m); }

template <typename T>
__device__ __forceinline__ T cst(double x) {
  return static_cast<T>(x);
}

// The same Tsit5 coefficients by index.  A double literal inside a loop is
// rebuilt from two 32-bit halves at every use (two issue slots, ~55 uses per
// replay step); read from this constant-bank table it enters its DFMA as an
// operand and holds no register.  float coefficients stay immediates.  The
// values are the #defines above, so results are bitwise unchanged.
enum TsIdx : int {
  kTsA21, kTsA31, kTsA32, kTsA41, kTsA42, kTsA43, kTsA51, kTsA52, kTsA53, kTsA54,
  kTsA61, kTsA62, kTsA63, kTsA64, kTsA65, kTsB1, kTsB2, kTsB3, kTsB4, kTsB5, kTsB6,
  kTsE1, kTsE2, kTsE3, kTsE4, kTsE5, kTsE6, kTsE7, kTsCount
};
#define GS_TS_LIST                                                                                      \
  TS_A21, TS_A31, TS_A32, TS_A41, TS_A42, TS_A43, TS_A51, TS_A52, TS_A53, TS_A54, TS_A61, TS_A62, TS_A63, \
      TS_A64, TS_A65, TS_B1, TS_B2, TS_B3, TS_B4, TS_B5, TS_B6, TS_E1, TS_E2, TS_E3, TS_E4, TS_E5, TS_E6, TS_E7
static __constant__ double kTsTab[kTsCount] = {GS_TS_LIST};
__host__ __device__ constexpr double ts_lit(int i) {
  constexpr double v[kTsCount] = {GS_TS_LIST};
  return v[i];
}
#undef GS_TS_LIST
template <typename T, int I>
__device__ __forceinline__ T tsc() {
  static_assert(I >= 0 && I < kTsCount, "Tsit5 coefficient index");
  if constexpr (sizeof(T) == 8) return kTsTab[I];
  else return static_cast<T>(ts_lit(I));
}

__device__ __forceinline__ double fmaT(double a, double b, double c) { return fma(a, b, c); }
__device__ __forceinline__ float fmaT(float a, float b, float c) { return fmaf(a, b, c); }

template <typename T> struct Eps;
template <> struct Eps<double> { static constexpr double v = 2.220446049250313e-16; };
template <> struct Eps<float> { static constexpr float v = 1.1920928955078125e-07f; };

// ---------------------------------------------------------------------------
// Lorenz: u' = (s (u2 - u1), u1 (r - u3) - u2, u1 u2 - b u3),
// p = (sigma, rho, beta) -- the listing on the DiffEqGPU "ad" page.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void lorenz_f(T x, T y, T z, T s, T r, T b, T& fx, T& fy, T& fz) {
  fx = s * (y - x);
  fy = fmaT(x, r - z, -y);
  fz = fmaT(x, y, -(b * z));
}

// ---------------------------------------------------------------------------
// Robertson kinetics, mass action for A->B (k1), 2B->B+C (k2), B+C->A+C (k3).
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void robertson_f(T y1, T y2, T y3, T k1, T k2, T k3, T& f1, T& f2, T& f3) {
  T r1 = k1 * y1;
  T r2 = k2 * (y2 * y2);
  T r3 = k3 * (y2 * y3);
  f1 = r3 - r1;
  f2 = (r1 - r3) - r2;
  f3 = r2;
}

// Robertson Jacobian, row-major 3x3.
template <typename T>
__device__ __forceinline__ void robertson_J(T y1, T y2, T y3, T k1, T k2, T k3, T J[9]) {
  (void)y1;
  T a = k3 * y3;
  T b = k3 * y2;
  T c = cst<T>(2.0) * (k2 * y2);
  J[0] = -k1;
  J[1] = a;
  J[2] = b;
  J[3] = k1;
  J[4] = -(a + c);
  J[5] = -b;
  J[6] = cst<T>(0.0);
  J[7] = c;
  J[8] = cst<T>(0.0);
}

// 3x3 LU with partial pivoting (largest |entry|, ties to the lowest row),
// right-looking; whole rows swap.  Fully unrolled so M and P stay in registers.
// R receives the reciprocals of the pivots (one division each); multipliers
// and back substitution multiply by them.  Returns false on a zero or
// non-finite pivot.
template <typename T>
__device__ __forceinline__ bool lu3(T M[9], int P[3], T R[3]) {
  P[0] = 0;
  P[1] = 1;
  P[2] = 2;
  bool ok = true;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    int piv = k;
#pragma unroll
    for (int i = k + 1; i < 3; ++i)
      if (fabs(M[i * 3 + k]) > fabs(M[piv * 3 + k])) piv = i;
#pragma unroll
    for (int i = k + 1; i < 3; ++i) {
      if (piv == i) {
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          T t = M[k * 3 + j];
          M[k * 3 + j] = M[i * 3 + j];
          M[i * 3 + j] = t;
        }
        int tp = P[k];
        P[k] = P[i];
        P[i] = tp;
      }
    }
    T pv = M[k * 3 + k];
    ok = ok && (pv != cst<T>(0.0)) && isfinite(pv);
    R[k] = cst<T>(1.0) / pv;
#pragma unroll
    for (int i = k + 1; i < 3; ++i) {
      T l = M[i * 3 + k] * R[k];
      M[i * 3 + k] = l;
#pragma unroll
      for (int j = k + 1; j < 3; ++j) M[i * 3 + j] = fmaT(-l, M[k * 3 + j], M[i * 3 + j]);
    }
  }
  return ok;
}

template <typename T>
__device__ __forceinline__ T pick3(int i, T a, T b, T c) {
  return i == 0 ? a : (i == 1 ? b : c);
}

// Solve (P M) x = P b with the factors of lu3: x = M^{-1} b.
template <typename T>
__device__ __forceinline__ void lu3_solve(const T LU[9], const int P[3], const T R[3], T b0, T b1, T b2, T& x0,
                                          T& x1, T& x2) {
  x0 = pick3(P[0], b0, b1, b2);
  x1 = pick3(P[1], b0, b1, b2);
  x2 = pick3(P[2], b0, b1, b2);
  x1 = fmaT(-LU[3], x0, x1);
  x2 = fmaT(-LU[6], x0, x2);
  x2 = fmaT(-LU[7], x1, x2);
  x2 = x2 * R[2];
  x1 = fmaT(-LU[5], x2, x1);
  x1 = x1 * R[1];
  x0 = fmaT(-LU[1], x1, x0);
  x0 = fmaT(-LU[2], x2, x0);
  x0 = x0 * R[0];
}

// Solve M^T x = b with the factors of lu3 (P M = L U, so M^T = U^T L^T P):
// U^T y = b (forward), L^T z = y (backward, unit diagonal), x[P[i]] = z[i].
// Used by the reverse sweep only (not part of the bitwise contract).
template <typename T>
__device__ __forceinline__ void lu3_solve_T(const T LU[9], const int P[3], const T R[3], T b0, T b1, T b2, T& x0,
                                            T& x1, T& x2) {
  T y0 = b0 * R[0];
  T y1 = fmaT(-LU[1], y0, b1) * R[1];
  T y2 = fmaT(-LU[5], y1, fmaT(-LU[2], y0, b2)) * R[2];
  T z2 = y2;
  T z1 = fmaT(-LU[7], z2, y1);
  T z0 = fmaT(-LU[6], z2, fmaT(-LU[3], z1, y0));
  // scatter through the permutation
  x0 = P[0] == 0 ? z0 : (P[1] == 0 ? z1 : z2);
  x1 = P[0] == 1 ? z0 : (P[1] == 1 ? z1 : z2);
  x2 = P[0] == 2 ? z0 : (P[1] == 2 ? z1 : z2);
}

// Bring the line holding *p into L2 ahead of its use (no register, no wait).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// One element global -> shared by the issuing thread, asynchronously
// (cp.async, cached in L1 and L2).  A thread's copies are grouped by
// cp_async_commit; cp_async_wait<N> returns once at most N of its groups are
// still in flight.  The wait is on the thread's own copies only.
template <typename T>
__device__ __forceinline__ void cp_async_el(T* dst, const T* src) {
  static_assert(sizeof(T) == 4 || sizeof(T) == 8, "cp.async element size");
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  if constexpr (sizeof(T) == 8)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// Host-side helpers.
// ---------------------------------------------------------------------------
void count_launch(int k = 1);

inline bool launch_ok() { return cudaGetLastError() == cudaSuccess; }

}  // namespace gs
