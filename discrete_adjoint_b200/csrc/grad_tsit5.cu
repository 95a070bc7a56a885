// grad_tsit5.cu -- fused fixed-step replay + reverse sweep (the discrete
// adjoint) for Tsit5 on the Lorenz system, one thread per trajectory slot.
//
// GRADSOLVE (arXiv 2609.02876), evolve.pub review "Summary" and "Strengths:
// precisely scoped exactness claim": the gradient is the exact derivative of
// the fixed-step replay of the recorded steps, the mesh held as data.
//
// Forward half: for s < S_j replay step s with h[s][j] (the forward arithmetic
// follows the floating-point contract, so it is bitwise equal to any replay
// that keeps the same operation order), store the state u_s to the checkpoint
// workspace ck[s][c][j], and add the loss terms at the save points.
//
// Reverse half: for s = S_j-1 .. 0, reload u_s, recompute the stage states
// U_1..U_6 of step s, and apply the transposed step.  With
//   u_{s+1} = u_s + h sum_j b_j k_j,  k_j = f(U_j),  U_j = u_s + h sum_{m<j} a_jm k_m
// and lambda = dL/du_{s+1}:
//   nu_j  = h (b_j lambda + sum_{m>j} a_mj mu_m)     (= dL/dk_j)
//   mu_j  = J(U_j)^T nu_j                              (= dL/dU_j)
//   pbar += f_p(U_j)^T nu_j
//   lambda <- lambda + sum_j mu_j                      (= dL/du_s)
// for j = 6 .. 1 (b_7 = 0, so the FSAL stage drops out).  Loss gradients enter
// lambda at the save points.  Output: dL/dp = pbar, dL/du0 = lambda.
//
// Memory layout: h [smax][n] and ck [smax][3][n] are step-major over slots, so
// at a given step the 32 threads of a warp touch 32 consecutive elements
// (256 B in fp64) of every array; gs_record orders slots by step count, so the
// threads of a warp also run chains of (nearly) equal length.
#include "common.cuh"

namespace gs {

template <typename T>
struct TsitLorenzArgs {
  int64_t n;
  const T* p;   // [3][n] by trajectory
  const T* u0;  // [3][n] by trajectory
  const T* h;   // [smax][n] by slot
  const int32_t* order;
  const int32_t* nsteps;
  const int32_t* save_idx;  // [nsave][n] by slot
  const int32_t* status;
  int32_t nsave;
  int32_t smax;
  int32_t loss_kind;
  const T* target;  // [nsave][3][n] by trajectory, may be null
  const T* weight;  // [nsave][3][n] by trajectory
  T* loss;          // [n] by trajectory
  T* dp;            // [3][n]
  T* du0;           // [3][n]
  T* ck;            // workspace [smax][3][n] by slot
};

// dL/dU = J(U)^T nu and pbar += f_p(U)^T nu for Lorenz.
template <typename T>
__device__ __forceinline__ void lorenz_vjp(T ux, T uy, T uz, T s, T r, T b, T nx, T ny, T nz, T& mx, T& my,
                                           T& mz, T& ps, T& pr, T& pb) {
  T m = s * nx;
  mx = fmaT(r - uz, ny, fmaT(uy, nz, -m));
  my = fmaT(ux, nz, m - ny);
  mz = -fmaT(ux, ny, b * nz);
  ps = fmaT(uy - ux, nx, ps);
  pr = fmaT(ux, ny, pr);
  pb = fmaT(-uz, nz, pb);
}

// Stage state U = fma(h, acc, u) for the three components.
#define GS_STAGE(UX, UY, UZ, AX, AY, AZ) \
  UX = fmaT(h, AX, x);                   \
  UY = fmaT(h, AY, y);                   \
  UZ = fmaT(h, AZ, z);

template <typename T>
__global__ void __launch_bounds__(128, 4) k_grad_tsit5_lorenz(TsitLorenzArgs<T> a) {
  const int64_t n = a.n;
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t i = a.order[j];
  if (i < 0 || i >= n) return;  // not a permutation entry: nothing to write
  const int S = a.nsteps[j];
  if (a.status[j] != GS_TRAJ_OK || S < 0 || S > a.smax) {
    const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
    a.loss[i] = nan;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      a.dp[c * n + i] = nan;
      a.du0[c * n + i] = nan;
    }
    return;
  }
  const T s = a.p[i], r = a.p[n + i], b = a.p[2 * n + i];
  T x = a.u0[i], y = a.u0[n + i], z = a.u0[2 * n + i];
  const T* __restrict__ hp = a.h + j;
  T* __restrict__ cp = a.ck + j;
  const int64_t n3 = 3 * n;

  // ---------------------------------------------------------------- forward
  T L = cst<T>(0.0);
  int kk = 0;
  int next = a.save_idx[j];
  T k1x, k1y, k1z;
  lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);
  T hn = S > 0 ? hp[0] : cst<T>(0.0);
  for (int st = 0; st < S; ++st) {
    const T h = hn;
    if (st + 1 < S) hn = hp[(int64_t)(st + 1) * n];
    cp[0] = x;
    cp[n] = y;
    cp[2 * n] = z;
    cp += n3;
    T ax, ay, az, Ux, Uy, Uz;
    // stage 2
    ax = cst<T>(TS_A21) * k1x;
    ay = cst<T>(TS_A21) * k1y;
    az = cst<T>(TS_A21) * k1z;
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    T k2x, k2y, k2z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k2x, k2y, k2z);
    // stage 3
    ax = cst<T>(TS_A31) * k1x;
    ay = cst<T>(TS_A31) * k1y;
    az = cst<T>(TS_A31) * k1z;
    ax = fmaT(cst<T>(TS_A32), k2x, ax);
    ay = fmaT(cst<T>(TS_A32), k2y, ay);
    az = fmaT(cst<T>(TS_A32), k2z, az);
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    T k3x, k3y, k3z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k3x, k3y, k3z);
    // stage 4
    ax = cst<T>(TS_A41) * k1x;
    ay = cst<T>(TS_A41) * k1y;
    az = cst<T>(TS_A41) * k1z;
    ax = fmaT(cst<T>(TS_A42), k2x, ax);
    ay = fmaT(cst<T>(TS_A42), k2y, ay);
    az = fmaT(cst<T>(TS_A42), k2z, az);
    ax = fmaT(cst<T>(TS_A43), k3x, ax);
    ay = fmaT(cst<T>(TS_A43), k3y, ay);
    az = fmaT(cst<T>(TS_A43), k3z, az);
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    T k4x, k4y, k4z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k4x, k4y, k4z);
    // stage 5
    ax = cst<T>(TS_A51) * k1x;
    ay = cst<T>(TS_A51) * k1y;
    az = cst<T>(TS_A51) * k1z;
    ax = fmaT(cst<T>(TS_A52), k2x, ax);
    ay = fmaT(cst<T>(TS_A52), k2y, ay);
    az = fmaT(cst<T>(TS_A52), k2z, az);
    ax = fmaT(cst<T>(TS_A53), k3x, ax);
    ay = fmaT(cst<T>(TS_A53), k3y, ay);
    az = fmaT(cst<T>(TS_A53), k3z, az);
    ax = fmaT(cst<T>(TS_A54), k4x, ax);
    ay = fmaT(cst<T>(TS_A54), k4y, ay);
    az = fmaT(cst<T>(TS_A54), k4z, az);
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    T k5x, k5y, k5z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k5x, k5y, k5z);
    // stage 6
    ax = cst<T>(TS_A61) * k1x;
    ay = cst<T>(TS_A61) * k1y;
    az = cst<T>(TS_A61) * k1z;
    ax = fmaT(cst<T>(TS_A62), k2x, ax);
    ay = fmaT(cst<T>(TS_A62), k2y, ay);
    az = fmaT(cst<T>(TS_A62), k2z, az);
    ax = fmaT(cst<T>(TS_A63), k3x, ax);
    ay = fmaT(cst<T>(TS_A63), k3y, ay);
    az = fmaT(cst<T>(TS_A63), k3z, az);
    ax = fmaT(cst<T>(TS_A64), k4x, ax);
    ay = fmaT(cst<T>(TS_A64), k4y, ay);
    az = fmaT(cst<T>(TS_A64), k4z, az);
    ax = fmaT(cst<T>(TS_A65), k5x, ax);
    ay = fmaT(cst<T>(TS_A65), k5y, ay);
    az = fmaT(cst<T>(TS_A65), k5z, az);
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    T k6x, k6y, k6z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k6x, k6y, k6z);
    // stage 7 = u_{s+1}
    ax = cst<T>(TS_B1) * k1x;
    ay = cst<T>(TS_B1) * k1y;
    az = cst<T>(TS_B1) * k1z;
    ax = fmaT(cst<T>(TS_B2), k2x, ax);
    ay = fmaT(cst<T>(TS_B2), k2y, ay);
    az = fmaT(cst<T>(TS_B2), k2z, az);
    ax = fmaT(cst<T>(TS_B3), k3x, ax);
    ay = fmaT(cst<T>(TS_B3), k3y, ay);
    az = fmaT(cst<T>(TS_B3), k3z, az);
    ax = fmaT(cst<T>(TS_B4), k4x, ax);
    ay = fmaT(cst<T>(TS_B4), k4y, ay);
    az = fmaT(cst<T>(TS_B4), k4z, az);
    ax = fmaT(cst<T>(TS_B5), k5x, ax);
    ay = fmaT(cst<T>(TS_B5), k5y, ay);
    az = fmaT(cst<T>(TS_B5), k5z, az);
    ax = fmaT(cst<T>(TS_B6), k6x, ax);
    ay = fmaT(cst<T>(TS_B6), k6y, ay);
    az = fmaT(cst<T>(TS_B6), k6z, az);
    x = fmaT(h, ax, x);
    y = fmaT(h, ay, y);
    z = fmaT(h, az, z);
    lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);  // FSAL: next step's first slope
    if (st + 1 == next) {
      const int64_t o = (int64_t)kk * n3 + i;
      if (a.loss_kind == GS_LOSS_SUMSQ) {
        T dx = a.target ? x - a.target[o] : x;
        T dy = a.target ? y - a.target[o + n] : y;
        T dz = a.target ? z - a.target[o + 2 * n] : z;
        L = fmaT(dx, dx, L);
        L = fmaT(dy, dy, L);
        L = fmaT(dz, dz, L);
      } else {
        L = fmaT(a.weight[o], x, L);
        L = fmaT(a.weight[o + n], y, L);
        L = fmaT(a.weight[o + 2 * n], z, L);
      }
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
  }

  // ---------------------------------------------------------------- reverse
  T lx = cst<T>(0.0), ly = cst<T>(0.0), lz = cst<T>(0.0);
  T ps = cst<T>(0.0), pr = cst<T>(0.0), pb = cst<T>(0.0);
  kk = a.nsave - 1;
  next = a.save_idx[(int64_t)kk * n + j];
  // u_{s+1} for the save-point test of step s; prefetched u_s and h_s
  T nx = x, ny = y, nz = z;
  T cx = cst<T>(0.0), cy = cst<T>(0.0), cz = cst<T>(0.0), hc = cst<T>(0.0);
  if (S > 0) {
    cp -= n3;
    cx = cp[0];
    cy = cp[n];
    cz = cp[2 * n];
    hc = hp[(int64_t)(S - 1) * n];
  }
  for (int st = S - 1; st >= 0; --st) {
    if (st + 1 == next) {
      const int64_t o = (int64_t)kk * n3 + i;
      if (a.loss_kind == GS_LOSS_SUMSQ) {
        T dx = a.target ? nx - a.target[o] : nx;
        T dy = a.target ? ny - a.target[o + n] : ny;
        T dz = a.target ? nz - a.target[o + 2 * n] : nz;
        lx = fmaT(cst<T>(2.0), dx, lx);
        ly = fmaT(cst<T>(2.0), dy, ly);
        lz = fmaT(cst<T>(2.0), dz, lz);
      } else {
        lx += a.weight[o];
        ly += a.weight[o + n];
        lz += a.weight[o + 2 * n];
      }
      --kk;
      next = kk >= 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
    x = cx;
    y = cy;
    z = cz;
    const T h = hc;
    if (st > 0) {
      cp -= n3;
      cx = cp[0];
      cy = cp[n];
      cz = cp[2 * n];
      hc = hp[(int64_t)(st - 1) * n];
    }
    // recompute the stage states of step st (same arithmetic as the forward)
    T ax, ay, az;
    T f1x, f1y, f1z;
    lorenz_f(x, y, z, s, r, b, f1x, f1y, f1z);
    T U2x, U2y, U2z, U3x, U3y, U3z, U4x, U4y, U4z, U5x, U5y, U5z, U6x, U6y, U6z;
    ax = cst<T>(TS_A21) * f1x;
    ay = cst<T>(TS_A21) * f1y;
    az = cst<T>(TS_A21) * f1z;
    GS_STAGE(U2x, U2y, U2z, ax, ay, az)
    T f2x, f2y, f2z;
    lorenz_f(U2x, U2y, U2z, s, r, b, f2x, f2y, f2z);
    ax = cst<T>(TS_A31) * f1x;
    ay = cst<T>(TS_A31) * f1y;
    az = cst<T>(TS_A31) * f1z;
    ax = fmaT(cst<T>(TS_A32), f2x, ax);
    ay = fmaT(cst<T>(TS_A32), f2y, ay);
    az = fmaT(cst<T>(TS_A32), f2z, az);
    GS_STAGE(U3x, U3y, U3z, ax, ay, az)
    T f3x, f3y, f3z;
    lorenz_f(U3x, U3y, U3z, s, r, b, f3x, f3y, f3z);
    ax = cst<T>(TS_A41) * f1x;
    ay = cst<T>(TS_A41) * f1y;
    az = cst<T>(TS_A41) * f1z;
    ax = fmaT(cst<T>(TS_A42), f2x, ax);
    ay = fmaT(cst<T>(TS_A42), f2y, ay);
    az = fmaT(cst<T>(TS_A42), f2z, az);
    ax = fmaT(cst<T>(TS_A43), f3x, ax);
    ay = fmaT(cst<T>(TS_A43), f3y, ay);
    az = fmaT(cst<T>(TS_A43), f3z, az);
    GS_STAGE(U4x, U4y, U4z, ax, ay, az)
    T f4x, f4y, f4z;
    lorenz_f(U4x, U4y, U4z, s, r, b, f4x, f4y, f4z);
    ax = cst<T>(TS_A51) * f1x;
    ay = cst<T>(TS_A51) * f1y;
    az = cst<T>(TS_A51) * f1z;
    ax = fmaT(cst<T>(TS_A52), f2x, ax);
    ay = fmaT(cst<T>(TS_A52), f2y, ay);
    az = fmaT(cst<T>(TS_A52), f2z, az);
    ax = fmaT(cst<T>(TS_A53), f3x, ax);
    ay = fmaT(cst<T>(TS_A53), f3y, ay);
    az = fmaT(cst<T>(TS_A53), f3z, az);
    ax = fmaT(cst<T>(TS_A54), f4x, ax);
    ay = fmaT(cst<T>(TS_A54), f4y, ay);
    az = fmaT(cst<T>(TS_A54), f4z, az);
    GS_STAGE(U5x, U5y, U5z, ax, ay, az)
    T f5x, f5y, f5z;
    lorenz_f(U5x, U5y, U5z, s, r, b, f5x, f5y, f5z);
    ax = cst<T>(TS_A61) * f1x;
    ay = cst<T>(TS_A61) * f1y;
    az = cst<T>(TS_A61) * f1z;
    ax = fmaT(cst<T>(TS_A62), f2x, ax);
    ay = fmaT(cst<T>(TS_A62), f2y, ay);
    az = fmaT(cst<T>(TS_A62), f2z, az);
    ax = fmaT(cst<T>(TS_A63), f3x, ax);
    ay = fmaT(cst<T>(TS_A63), f3y, ay);
    az = fmaT(cst<T>(TS_A63), f3z, az);
    ax = fmaT(cst<T>(TS_A64), f4x, ax);
    ay = fmaT(cst<T>(TS_A64), f4y, ay);
    az = fmaT(cst<T>(TS_A64), f4z, az);
    ax = fmaT(cst<T>(TS_A65), f5x, ax);
    ay = fmaT(cst<T>(TS_A65), f5y, ay);
    az = fmaT(cst<T>(TS_A65), f5z, az);
    GS_STAGE(U6x, U6y, U6z, ax, ay, az)

    // transposed step, stages 6 .. 1
    T m6x, m6y, m6z, m5x, m5y, m5z, m4x, m4y, m4z, m3x, m3y, m3z, m2x, m2y, m2z, m1x, m1y, m1z;
    T vx, vy, vz;
    vx = h * (cst<T>(TS_B6) * lx);
    vy = h * (cst<T>(TS_B6) * ly);
    vz = h * (cst<T>(TS_B6) * lz);
    lorenz_vjp(U6x, U6y, U6z, s, r, b, vx, vy, vz, m6x, m6y, m6z, ps, pr, pb);

    vx = h * fmaT(cst<T>(TS_A65), m6x, cst<T>(TS_B5) * lx);
    vy = h * fmaT(cst<T>(TS_A65), m6y, cst<T>(TS_B5) * ly);
    vz = h * fmaT(cst<T>(TS_A65), m6z, cst<T>(TS_B5) * lz);
    lorenz_vjp(U5x, U5y, U5z, s, r, b, vx, vy, vz, m5x, m5y, m5z, ps, pr, pb);

    vx = h * fmaT(cst<T>(TS_A54), m5x, fmaT(cst<T>(TS_A64), m6x, cst<T>(TS_B4) * lx));
    vy = h * fmaT(cst<T>(TS_A54), m5y, fmaT(cst<T>(TS_A64), m6y, cst<T>(TS_B4) * ly));
    vz = h * fmaT(cst<T>(TS_A54), m5z, fmaT(cst<T>(TS_A64), m6z, cst<T>(TS_B4) * lz));
    lorenz_vjp(U4x, U4y, U4z, s, r, b, vx, vy, vz, m4x, m4y, m4z, ps, pr, pb);

    vx = h * fmaT(cst<T>(TS_A43), m4x, fmaT(cst<T>(TS_A53), m5x, fmaT(cst<T>(TS_A63), m6x, cst<T>(TS_B3) * lx)));
    vy = h * fmaT(cst<T>(TS_A43), m4y, fmaT(cst<T>(TS_A53), m5y, fmaT(cst<T>(TS_A63), m6y, cst<T>(TS_B3) * ly)));
    vz = h * fmaT(cst<T>(TS_A43), m4z, fmaT(cst<T>(TS_A53), m5z, fmaT(cst<T>(TS_A63), m6z, cst<T>(TS_B3) * lz)));
    lorenz_vjp(U3x, U3y, U3z, s, r, b, vx, vy, vz, m3x, m3y, m3z, ps, pr, pb);

    vx = h * fmaT(cst<T>(TS_A32), m3x,
                  fmaT(cst<T>(TS_A42), m4x, fmaT(cst<T>(TS_A52), m5x, fmaT(cst<T>(TS_A62), m6x, cst<T>(TS_B2) * lx))));
    vy = h * fmaT(cst<T>(TS_A32), m3y,
                  fmaT(cst<T>(TS_A42), m4y, fmaT(cst<T>(TS_A52), m5y, fmaT(cst<T>(TS_A62), m6y, cst<T>(TS_B2) * ly))));
    vz = h * fmaT(cst<T>(TS_A32), m3z,
                  fmaT(cst<T>(TS_A42), m4z, fmaT(cst<T>(TS_A52), m5z, fmaT(cst<T>(TS_A62), m6z, cst<T>(TS_B2) * lz))));
    lorenz_vjp(U2x, U2y, U2z, s, r, b, vx, vy, vz, m2x, m2y, m2z, ps, pr, pb);

    vx = h * fmaT(cst<T>(TS_A21), m2x,
                  fmaT(cst<T>(TS_A31), m3x,
                       fmaT(cst<T>(TS_A41), m4x, fmaT(cst<T>(TS_A51), m5x, fmaT(cst<T>(TS_A61), m6x, cst<T>(TS_B1) * lx)))));
    vy = h * fmaT(cst<T>(TS_A21), m2y,
                  fmaT(cst<T>(TS_A31), m3y,
                       fmaT(cst<T>(TS_A41), m4y, fmaT(cst<T>(TS_A51), m5y, fmaT(cst<T>(TS_A61), m6y, cst<T>(TS_B1) * ly)))));
    vz = h * fmaT(cst<T>(TS_A21), m2z,
                  fmaT(cst<T>(TS_A31), m3z,
                       fmaT(cst<T>(TS_A41), m4z, fmaT(cst<T>(TS_A51), m5z, fmaT(cst<T>(TS_A61), m6z, cst<T>(TS_B1) * lz)))));
    lorenz_vjp(x, y, z, s, r, b, vx, vy, vz, m1x, m1y, m1z, ps, pr, pb);

    lx += ((m1x + m2x) + (m3x + m4x)) + (m5x + m6x);
    ly += ((m1y + m2y) + (m3y + m4y)) + (m5y + m6y);
    lz += ((m1z + m2z) + (m3z + m4z)) + (m5z + m6z);
    nx = x;
    ny = y;
    nz = z;
  }
  // save points at step 0 cannot exist (save times lie in (t0, t1])
  a.loss[i] = L;
  a.dp[i] = ps;
  a.dp[n + i] = pr;
  a.dp[2 * n + i] = pb;
  a.du0[i] = lx;
  a.du0[n + i] = ly;
  a.du0[2 * n + i] = lz;
}

#undef GS_STAGE

template <typename T>
gs_status launch_grad_tsit5_lorenz(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp,
                                   void* du0, void* ws, cudaStream_t st) {
  TsitLorenzArgs<T> a;
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
  a.ck = (T*)ws;
  const int bs = 128;
  const int64_t grid = (P->n + bs - 1) / bs;
  k_grad_tsit5_lorenz<T><<<(unsigned)grid, bs, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_tsit5_lorenz<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                    void*, void*, cudaStream_t);
template gs_status launch_grad_tsit5_lorenz<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                   void*, void*, cudaStream_t);

}  // namespace gs
