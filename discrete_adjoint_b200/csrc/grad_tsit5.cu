// grad_tsit5.cu -- fused fixed-step replay + reverse sweep (the discrete
// adjoint) for Tsit5 on the Lorenz system.
//
// GRADSOLVE (arXiv 2609.02876), evolve.pub review "Summary" and "Strengths:
// precisely scoped exactness claim": the gradient is the exact derivative of
// the fixed-step replay of the recorded steps, the mesh held as data.
//
// Forward half: for s < S replay step s with h[s] (the forward arithmetic
// follows the floating-point contract, so it is bitwise equal to any replay
// that keeps the same operation order), store the state u_s to the checkpoint
// workspace ck[s][c][slot], and add the loss terms at the save points.
//
// Reverse half: for s = S-1 .. 0, reload u_s, recompute the stage states
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
// Execution: the kernel is bound by the FP64 pipe, and one Lorenz trajectory
// offers only three independent chains (x, y, z) per instruction stream, which
// leaves the pipe idle a quarter of the time at the occupancy its registers
// allow.  Each thread therefore carries K adjacent slots (vec<T, K>), giving 3K
// independent chains.  gs_record orders slots by decreasing step count, so the
// K chains of a thread (and the 32K of a warp) have nearly equal length; the
// shorter ones run the remaining iterations as steps of size 0, which are
// exact identities in both halves (u + 0 * acc = u; nu = 0 * (...) = 0), so the
// results are bitwise those of one slot per thread.
//
// Memory layout: h [smax][n] and ck [smax][3][n] are step-major over slots, so
// at a given step a warp touches 32K consecutive elements of every array.
// With one slot per thread, h and the checkpoints stream into per-thread
// shared-memory rings (cp.async, kRingF / kRingR steps ahead) and are read
// from there one step ahead; with K > 1 they are loaded one step ahead into
// registers and prefetched several steps ahead into L2.
#include "steps.cuh"
#include "vec.cuh"

namespace gs {

#ifndef GS_GRAD_K
#define GS_GRAD_K 1
#endif
#ifndef GS_GRAD_BS
#define GS_GRAD_BS 128
#endif
#ifndef GS_GRAD_MINB
#define GS_GRAD_MINB (GS_GRAD_K == 1 ? 4 : 2)
#endif
#ifndef GS_PF_F
#define GS_PF_F 8
#endif
#ifndef GS_PF_R
#define GS_PF_R 4
#endif
#ifndef GS_GRAD_ASYNC
#define GS_GRAD_ASYNC 1
#endif
// Copy rings (one trajectory per thread): the forward streams h kRingF steps
// ahead, the reverse streams (u_s, h_s) kRingR steps ahead, each thread into
// its own shared-memory slots with cp.async, so that no register waits on DRAM.
#ifndef GS_RING_F
#define GS_RING_F 8
#endif
#ifndef GS_RING_R
#define GS_RING_R 8
#endif
constexpr int kRingF = GS_RING_F;
constexpr int kRingR = GS_RING_R;
static_assert((kRingF & (kRingF - 1)) == 0 && kRingF >= 2 && (kRingR & (kRingR - 1)) == 0 && kRingR >= 2,
              "ring depths: powers of two, at least 2");
// L2 prefetch distances in steps (a warp's forward step takes ~0.5 us and its
// reverse step ~1 us, against a DRAM latency of ~1 us under load).
constexpr int kPrefetchF = GS_PF_F;
constexpr int kPrefetchR = GS_PF_R;

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
  const T* theta;   // [nsave][n] by slot: dense save points, or null
};

// dL/dU = J(U)^T nu and pbar += f_p(U)^T nu for Lorenz.
template <typename V>
__device__ __forceinline__ void lorenz_vjp(const V& ux, const V& uy, const V& uz, const V& s, const V& r, const V& b,
                                           const V& nx, const V& ny, const V& nz, V& mx, V& my, V& mz, V& ps, V& pr,
                                           V& pb) {
  V m = s * nx;
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

// acc = a1 k1 (+ a2 k2 ...) for the three components, in the contract's order.
#define GS_ACC1(A1, K1)    \
  ax = tsc<T, A1>() * K1##x; \
  ay = tsc<T, A1>() * K1##y; \
  az = tsc<T, A1>() * K1##z;
#define GS_ACCN(AN, KN)             \
  ax = fmaT(tsc<T, AN>(), KN##x, ax); \
  ay = fmaT(tsc<T, AN>(), KN##y, ay); \
  az = fmaT(tsc<T, AN>(), KN##z, az);

template <typename T, int K, bool DENSE>
__global__ void __launch_bounds__(GS_GRAD_BS, GS_GRAD_MINB) k_grad_tsit5_lorenz(TsitLorenzArgs<T> a) {
  using V = vec<T, K>;
  const int64_t n = a.n;
  const int64_t n3 = 3 * n;
  const int64_t j0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * K;
  if (j0 >= n) return;
  const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));

  // per-slot set-up; inactive slots (past n, failed, malformed) run no steps
  int64_t i[K];
  int S[K];
  int Smax = 0;
  V s, r, b, x, y, z;
#pragma unroll
  for (int q = 0; q < K; ++q) {
    const int64_t j = j0 + q;
    i[q] = -1;
    S[q] = 0;
    s.e[q] = r.e[q] = b.e[q] = x.e[q] = y.e[q] = z.e[q] = cst<T>(0.0);
    if (j < n) {
      const int64_t ii = a.order[j];
      if (ii >= 0 && ii < n) {
        const int sq = a.nsteps[j];
        if (a.status[j] != GS_TRAJ_OK || sq < 0 || sq > a.smax) {
          a.loss[ii] = nan;
#pragma unroll
          for (int c = 0; c < 3; ++c) {
            a.dp[c * n + ii] = nan;
            a.du0[c * n + ii] = nan;
          }
        } else {
          i[q] = ii;
          S[q] = sq;
          Smax = sq > Smax ? sq : Smax;
          s.e[q] = a.p[ii];
          r.e[q] = a.p[n + ii];
          b.e[q] = a.p[2 * n + ii];
          x.e[q] = a.u0[ii];
          y.e[q] = a.u0[n + ii];
          z.e[q] = a.u0[2 * n + ii];
        }
      }
    }
  }
  const T* __restrict__ hp = a.h + j0;
  T* __restrict__ cp = a.ck + j0;
  constexpr bool kAsync = GS_GRAD_ASYNC != 0 && K == 1;
  __shared__ T ring[kAsync ? 4 * kRingR * GS_GRAD_BS : 1];
  T* const rg = ring + threadIdx.x;  // this thread's element of slot row w: rg[w * GS_GRAD_BS]

  // ---------------------------------------------------------------- forward
  V L = vsplat<T, K>(cst<T>(0.0));
  int kk[K], next[K];
#pragma unroll
  for (int q = 0; q < K; ++q) {
    kk[q] = 0;
    next[q] = S[q] > 0 ? a.save_idx[j0 + q] : -1;
  }
  V k1x, k1y, k1z;
  lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);
  V hn;
  if constexpr (kAsync) {  // h of step s in slot s % kRingF
#pragma unroll
    for (int s = 0; s < kRingF; ++s) {
      if (s < S[0]) cp_async_el(rg + s * GS_GRAD_BS, hp + (int64_t)s * n);
      cp_async_commit();
    }
    cp_async_wait<kRingF - 1>();
    hn.e[0] = 0 < S[0] ? rg[0] : cst<T>(0.0);
  } else {
#pragma unroll
    for (int q = 0; q < K; ++q) hn.e[q] = 0 < S[q] ? hp[q] : cst<T>(0.0);
  }
  const T* hq = hp + n;                        // h of step st + 1
  const T* hf = hp + (int64_t)kPrefetchF * n;  // h of step st + kPrefetchF
  for (int st = 0; st < Smax; ++st) {
    const V h = hn;
    if constexpr (kAsync) {
      cp_async_wait<kRingF - 2>();  // the group of step st + 1
      hn.e[0] = st + 1 < S[0] ? rg[((st + 1) & (kRingF - 1)) * GS_GRAD_BS] : cst<T>(0.0);
    } else {
      if (st + kPrefetchF < Smax) prefetch_l2(hf);
      hf += n;
    }
#pragma unroll
    for (int q = 0; q < K; ++q) {
      if constexpr (!kAsync) hn.e[q] = st + 1 < S[q] ? hq[q] : cst<T>(0.0);
      if (st < S[q]) {
        cp[q] = x.e[q];
        cp[n + q] = y.e[q];
        cp[2 * n + q] = z.e[q];
      }
    }
    hq += n;
    cp += n3;
    V ax, ay, az, Ux, Uy, Uz;
    GS_ACC1(kTsA21, k1)
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    V k2x, k2y, k2z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k2x, k2y, k2z);
    GS_ACC1(kTsA31, k1)
    GS_ACCN(kTsA32, k2)
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    V k3x, k3y, k3z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k3x, k3y, k3z);
    GS_ACC1(kTsA41, k1)
    GS_ACCN(kTsA42, k2)
    GS_ACCN(kTsA43, k3)
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    V k4x, k4y, k4z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k4x, k4y, k4z);
    GS_ACC1(kTsA51, k1)
    GS_ACCN(kTsA52, k2)
    GS_ACCN(kTsA53, k3)
    GS_ACCN(kTsA54, k4)
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    V k5x, k5y, k5z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k5x, k5y, k5z);
    GS_ACC1(kTsA61, k1)
    GS_ACCN(kTsA62, k2)
    GS_ACCN(kTsA63, k3)
    GS_ACCN(kTsA64, k4)
    GS_ACCN(kTsA65, k5)
    GS_STAGE(Ux, Uy, Uz, ax, ay, az)
    V k6x, k6y, k6z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k6x, k6y, k6z);
    // stage 7 = u_{s+1}
    GS_ACC1(kTsB1, k1)
    GS_ACCN(kTsB2, k2)
    GS_ACCN(kTsB3, k3)
    GS_ACCN(kTsB4, k4)
    GS_ACCN(kTsB5, k5)
    GS_ACCN(kTsB6, k6)
    V xs, ys, zs, fsx, fsy, fsz;  // dense save points: u_s and f(u_s)
    if (DENSE) {
      xs = x;
      ys = y;
      zs = z;
      fsx = k1x;
      fsy = k1y;
      fsz = k1z;
    }
    x = fmaT(h, ax, x);
    y = fmaT(h, ay, y);
    z = fmaT(h, az, z);
    lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);  // FSAL: next step's first slope
#pragma unroll
    for (int q = 0; q < K; ++q) {
      // a landing record has at most one save point per step; a dense one any number
      while (st + 1 == next[q]) {
        const int64_t o = (int64_t)kk[q] * n3 + i[q];
        T ux = x.e[q], uy = y.e[q], uz = z.e[q];
        if (DENSE) {
          const T th = a.theta[(int64_t)kk[q] * n + j0 + q];
          if (th != cst<T>(1.0)) {
            const HermiteW<T> w = hermite_w(th);
            ux = hermite_c(w, xs.e[q], ux, fsx.e[q], k1x.e[q], h.e[q]);
            uy = hermite_c(w, ys.e[q], uy, fsy.e[q], k1y.e[q], h.e[q]);
            uz = hermite_c(w, zs.e[q], uz, fsz.e[q], k1z.e[q], h.e[q]);
          }
        }
        T Lq = L.e[q];
        if (a.loss_kind == GS_LOSS_SUMSQ) {
          const T dx = a.target ? ux - a.target[o] : ux;
          const T dy = a.target ? uy - a.target[o + n] : uy;
          const T dz = a.target ? uz - a.target[o + 2 * n] : uz;
          Lq = fmaT(dx, dx, Lq);
          Lq = fmaT(dy, dy, Lq);
          Lq = fmaT(dz, dz, Lq);
        } else {
          Lq = fmaT(a.weight[o], ux, Lq);
          Lq = fmaT(a.weight[o + n], uy, Lq);
          Lq = fmaT(a.weight[o + 2 * n], uz, Lq);
        }
        L.e[q] = Lq;
        ++kk[q];
        next[q] = kk[q] < a.nsave ? a.save_idx[(int64_t)kk[q] * n + j0 + q] : -1;
        if (!DENSE) break;
      }
    }
    if constexpr (kAsync) {  // step st + kRingF into the slot that step st has left
      const int sn = st + kRingF;
      if (sn < S[0]) cp_async_el(rg + (sn & (kRingF - 1)) * GS_GRAD_BS, hp + (int64_t)sn * n);
      cp_async_commit();
    }
  }
  if constexpr (kAsync) cp_async_wait<0>();  // the reverse reuses the slots
#pragma unroll
  for (int q = 0; q < K; ++q)
    if (i[q] >= 0) a.loss[i[q]] = L.e[q];

  // ---------------------------------------------------------------- reverse
  // At the top of iteration st, (x, y, z) holds u_{st+1} (the final state
  // first, then the state loaded by the previous iteration), which is what the
  // save-point test needs; (cx, cy, cz, hc) are the prefetched u_st and h_st.
  V lx = vsplat<T, K>(cst<T>(0.0)), ly = lx, lz = lx;
  V ps = lx, pr = lx, pb = lx;
#pragma unroll
  for (int q = 0; q < K; ++q) {
    kk[q] = a.nsave - 1;
    next[q] = S[q] > 0 ? a.save_idx[(int64_t)kk[q] * n + j0 + q] : -1;
  }
  V cx = x, cy = y, cz = z, hc = vsplat<T, K>(cst<T>(0.0));
  const T* hq2 = hp + (int64_t)(Smax - 1) * n;  // h of the step being loaded
  // reverse ring: (u_s, h_s) of step s in slot s % kRingR, components in rows
  // 4 (s % kRingR) + c; the copies of one step form one group
  auto issue_r = [&](int sr) {
    if (sr >= 0 && sr < S[0]) {
      T* d = rg + (sr & (kRingR - 1)) * 4 * GS_GRAD_BS;
      const T* c = a.ck + (int64_t)sr * n3 + j0;
      cp_async_el(d, c);
      cp_async_el(d + GS_GRAD_BS, c + n);
      cp_async_el(d + 2 * GS_GRAD_BS, c + 2 * n);
      cp_async_el(d + 3 * GS_GRAD_BS, hp + (int64_t)sr * n);
    }
    cp_async_commit();
  };
  auto take_r = [&](int sr) {  // step sr's values, its group complete
    const T* d = rg + (sr & (kRingR - 1)) * 4 * GS_GRAD_BS;
    cx.e[0] = d[0];
    cy.e[0] = d[GS_GRAD_BS];
    cz.e[0] = d[2 * GS_GRAD_BS];
    hc.e[0] = d[3 * GS_GRAD_BS];
  };
  if constexpr (kAsync) {
#pragma unroll
    for (int i2 = 0; i2 < kRingR; ++i2) issue_r(Smax - 1 - i2);
    cp_async_wait<kRingR - 1>();
    if (Smax > 0 && Smax - 1 < S[0]) take_r(Smax - 1);
  } else if (Smax > 0) {
    cp -= n3;
#pragma unroll
    for (int q = 0; q < K; ++q) {
      if (Smax - 1 < S[q]) {
        cx.e[q] = cp[q];
        cy.e[q] = cp[n + q];
        cz.e[q] = cp[2 * n + q];
        hc.e[q] = hq2[q];
      }
    }
  }
  for (int st = Smax - 1; st >= 0; --st) {
    if (!kAsync && st >= kPrefetchR) {
      const T* c = cp - (int64_t)kPrefetchR * n3;
      prefetch_l2(c);
      prefetch_l2(c + n);
      prefetch_l2(c + 2 * n);
      prefetch_l2(hq2 - (int64_t)kPrefetchR * n);
    }
    // dense save points inside step st: the interpolant's cotangent g reaches
    // u_{st+1} now (H01 g + J(u_{st+1})^T (h H11 g)) and u_st after the
    // transposed step (H00 g + J(u_st)^T (h H10 g)), with the matching
    // parameter terms f_p^T (.)
    V pgx, pgy, pgz, pnx, pny, pnz;
    if (DENSE) {
      pgx = vsplat<T, K>(cst<T>(0.0));
      pgy = pgx, pgz = pgx, pnx = pgx, pny = pgx, pnz = pgx;
    }
#pragma unroll
    for (int q = 0; q < K; ++q) {
      while (st + 1 == next[q]) {
        const int64_t o = (int64_t)kk[q] * n3 + i[q];
        T th = cst<T>(1.0);
        HermiteW<T> w;
        T ux = x.e[q], uy = y.e[q], uz = z.e[q], fsx, fsy, fsz, fnx, fny, fnz;
        if (DENSE) {
          th = a.theta[(int64_t)kk[q] * n + j0 + q];
          if (th != cst<T>(1.0)) {
            w = hermite_w(th);
            lorenz_f(cx.e[q], cy.e[q], cz.e[q], s.e[q], r.e[q], b.e[q], fsx, fsy, fsz);
            lorenz_f(ux, uy, uz, s.e[q], r.e[q], b.e[q], fnx, fny, fnz);
            const T hh = hc.e[q];
            ux = hermite_c(w, cx.e[q], x.e[q], fsx, fnx, hh);
            uy = hermite_c(w, cy.e[q], y.e[q], fsy, fny, hh);
            uz = hermite_c(w, cz.e[q], z.e[q], fsz, fnz, hh);
          }
        }
        T gx, gy, gz;  // d loss_k / d u(t_k)
        if (a.loss_kind == GS_LOSS_SUMSQ) {
          gx = cst<T>(2.0) * (a.target ? ux - a.target[o] : ux);
          gy = cst<T>(2.0) * (a.target ? uy - a.target[o + n] : uy);
          gz = cst<T>(2.0) * (a.target ? uz - a.target[o + 2 * n] : uz);
        } else {
          gx = a.weight[o];
          gy = a.weight[o + n];
          gz = a.weight[o + 2 * n];
        }
        if (!DENSE || th == cst<T>(1.0)) {
          lx.e[q] += gx;
          ly.e[q] += gy;
          lz.e[q] += gz;
        } else {
          const T hh = hc.e[q];
          T mx, my, mz;
          lorenz_vjp(x.e[q], y.e[q], z.e[q], s.e[q], r.e[q], b.e[q], (hh * w.h11) * gx, (hh * w.h11) * gy,
                     (hh * w.h11) * gz, mx, my, mz, ps.e[q], pr.e[q], pb.e[q]);
          lx.e[q] = fmaT(w.h01, gx, lx.e[q] + mx);
          ly.e[q] = fmaT(w.h01, gy, ly.e[q] + my);
          lz.e[q] = fmaT(w.h01, gz, lz.e[q] + mz);
          pgx.e[q] = fmaT(w.h00, gx, pgx.e[q]);
          pgy.e[q] = fmaT(w.h00, gy, pgy.e[q]);
          pgz.e[q] = fmaT(w.h00, gz, pgz.e[q]);
          pnx.e[q] = fmaT(hh * w.h10, gx, pnx.e[q]);
          pny.e[q] = fmaT(hh * w.h10, gy, pny.e[q]);
          pnz.e[q] = fmaT(hh * w.h10, gz, pnz.e[q]);
        }
        --kk[q];
        next[q] = kk[q] >= 0 ? a.save_idx[(int64_t)kk[q] * n + j0 + q] : -1;
        if (!DENSE) break;
      }
    }
    x = cx;
    y = cy;
    z = cz;
    const V h = hc;
    if (kAsync && st > 0) {
      cp_async_wait<kRingR - 2>();  // the group of step st - 1
      if (st - 1 < S[0])
        take_r(st - 1);
      else
        hc.e[0] = cst<T>(0.0);
    } else if (st > 0) {
      cp -= n3;
      hq2 -= n;
#pragma unroll
      for (int q = 0; q < K; ++q) {
        if (st - 1 < S[q]) {
          cx.e[q] = cp[q];
          cy.e[q] = cp[n + q];
          cz.e[q] = cp[2 * n + q];
          hc.e[q] = hq2[q];
        } else {
          hc.e[q] = cst<T>(0.0);  // a slot past its last step: an identity step
        }
      }
    }
    // recompute the stage states of step st (same arithmetic as the forward)
    V ax, ay, az;
    V f1x, f1y, f1z;
    lorenz_f(x, y, z, s, r, b, f1x, f1y, f1z);
    V U2x, U2y, U2z, U3x, U3y, U3z, U4x, U4y, U4z, U5x, U5y, U5z, U6x, U6y, U6z;
    GS_ACC1(kTsA21, f1)
    GS_STAGE(U2x, U2y, U2z, ax, ay, az)
    V f2x, f2y, f2z;
    lorenz_f(U2x, U2y, U2z, s, r, b, f2x, f2y, f2z);
    GS_ACC1(kTsA31, f1)
    GS_ACCN(kTsA32, f2)
    GS_STAGE(U3x, U3y, U3z, ax, ay, az)
    V f3x, f3y, f3z;
    lorenz_f(U3x, U3y, U3z, s, r, b, f3x, f3y, f3z);
    GS_ACC1(kTsA41, f1)
    GS_ACCN(kTsA42, f2)
    GS_ACCN(kTsA43, f3)
    GS_STAGE(U4x, U4y, U4z, ax, ay, az)
    V f4x, f4y, f4z;
    lorenz_f(U4x, U4y, U4z, s, r, b, f4x, f4y, f4z);
    GS_ACC1(kTsA51, f1)
    GS_ACCN(kTsA52, f2)
    GS_ACCN(kTsA53, f3)
    GS_ACCN(kTsA54, f4)
    GS_STAGE(U5x, U5y, U5z, ax, ay, az)
    V f5x, f5y, f5z;
    lorenz_f(U5x, U5y, U5z, s, r, b, f5x, f5y, f5z);
    GS_ACC1(kTsA61, f1)
    GS_ACCN(kTsA62, f2)
    GS_ACCN(kTsA63, f3)
    GS_ACCN(kTsA64, f4)
    GS_ACCN(kTsA65, f5)
    GS_STAGE(U6x, U6y, U6z, ax, ay, az)

    // transposed step, stages 6 .. 1
#define GS_C(N) tsc<T, kTs##N>()
    V m6x, m6y, m6z, m5x, m5y, m5z, m4x, m4y, m4z, m3x, m3y, m3z, m2x, m2y, m2z, m1x, m1y, m1z;
    V vx, vy, vz;
    vx = h * (GS_C(B6) * lx);
    vy = h * (GS_C(B6) * ly);
    vz = h * (GS_C(B6) * lz);
    lorenz_vjp(U6x, U6y, U6z, s, r, b, vx, vy, vz, m6x, m6y, m6z, ps, pr, pb);

    vx = h * fmaT(GS_C(A65), m6x, GS_C(B5) * lx);
    vy = h * fmaT(GS_C(A65), m6y, GS_C(B5) * ly);
    vz = h * fmaT(GS_C(A65), m6z, GS_C(B5) * lz);
    lorenz_vjp(U5x, U5y, U5z, s, r, b, vx, vy, vz, m5x, m5y, m5z, ps, pr, pb);

    vx = h * fmaT(GS_C(A54), m5x, fmaT(GS_C(A64), m6x, GS_C(B4) * lx));
    vy = h * fmaT(GS_C(A54), m5y, fmaT(GS_C(A64), m6y, GS_C(B4) * ly));
    vz = h * fmaT(GS_C(A54), m5z, fmaT(GS_C(A64), m6z, GS_C(B4) * lz));
    lorenz_vjp(U4x, U4y, U4z, s, r, b, vx, vy, vz, m4x, m4y, m4z, ps, pr, pb);

    vx = h * fmaT(GS_C(A43), m4x, fmaT(GS_C(A53), m5x, fmaT(GS_C(A63), m6x, GS_C(B3) * lx)));
    vy = h * fmaT(GS_C(A43), m4y, fmaT(GS_C(A53), m5y, fmaT(GS_C(A63), m6y, GS_C(B3) * ly)));
    vz = h * fmaT(GS_C(A43), m4z, fmaT(GS_C(A53), m5z, fmaT(GS_C(A63), m6z, GS_C(B3) * lz)));
    lorenz_vjp(U3x, U3y, U3z, s, r, b, vx, vy, vz, m3x, m3y, m3z, ps, pr, pb);

    vx = h * fmaT(GS_C(A32), m3x, fmaT(GS_C(A42), m4x, fmaT(GS_C(A52), m5x, fmaT(GS_C(A62), m6x, GS_C(B2) * lx))));
    vy = h * fmaT(GS_C(A32), m3y, fmaT(GS_C(A42), m4y, fmaT(GS_C(A52), m5y, fmaT(GS_C(A62), m6y, GS_C(B2) * ly))));
    vz = h * fmaT(GS_C(A32), m3z, fmaT(GS_C(A42), m4z, fmaT(GS_C(A52), m5z, fmaT(GS_C(A62), m6z, GS_C(B2) * lz))));
    lorenz_vjp(U2x, U2y, U2z, s, r, b, vx, vy, vz, m2x, m2y, m2z, ps, pr, pb);

    vx = h * fmaT(GS_C(A21), m2x,
                  fmaT(GS_C(A31), m3x,
                       fmaT(GS_C(A41), m4x, fmaT(GS_C(A51), m5x, fmaT(GS_C(A61), m6x, GS_C(B1) * lx)))));
    vy = h * fmaT(GS_C(A21), m2y,
                  fmaT(GS_C(A31), m3y,
                       fmaT(GS_C(A41), m4y, fmaT(GS_C(A51), m5y, fmaT(GS_C(A61), m6y, GS_C(B1) * ly)))));
    vz = h * fmaT(GS_C(A21), m2z,
                  fmaT(GS_C(A31), m3z,
                       fmaT(GS_C(A41), m4z, fmaT(GS_C(A51), m5z, fmaT(GS_C(A61), m6z, GS_C(B1) * lz)))));
    lorenz_vjp(x, y, z, s, r, b, vx, vy, vz, m1x, m1y, m1z, ps, pr, pb);

    lx += ((m1x + m2x) + (m3x + m4x)) + (m5x + m6x);
    ly += ((m1y + m2y) + (m3y + m4y)) + (m5y + m6y);
    lz += ((m1z + m2z) + (m3z + m4z)) + (m5z + m6z);
    if (DENSE) {  // the interpolants' share of u_st
      V qx, qy, qz;
      lorenz_vjp(x, y, z, s, r, b, pnx, pny, pnz, qx, qy, qz, ps, pr, pb);
      lx += pgx + qx;
      ly += pgy + qy;
      lz += pgz + qz;
    }
    if constexpr (kAsync) issue_r(st - kRingR);  // into the slot that step st has left
  }
  if constexpr (kAsync) cp_async_wait<0>();
  // save points at step 0 cannot exist (save times lie in (t0, t1])
#pragma unroll
  for (int q = 0; q < K; ++q) {
    if (i[q] < 0) continue;
    a.dp[i[q]] = ps.e[q];
    a.dp[n + i[q]] = pr.e[q];
    a.dp[2 * n + i[q]] = pb.e[q];
    a.du0[i[q]] = lx.e[q];
    a.du0[n + i[q]] = ly.e[q];
    a.du0[2 * n + i[q]] = lz.e[q];
  }
}

#undef GS_STAGE
#undef GS_ACC1
#undef GS_ACCN
#undef GS_C

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
  a.theta = (const T*)M->save_theta;
  constexpr int K = GS_GRAD_K;
  const int bs = GS_GRAD_BS;
  const int64_t threads = (P->n + K - 1) / K;
  const int64_t grid = (threads + bs - 1) / bs;
  if (a.theta)
    k_grad_tsit5_lorenz<T, K, true><<<(unsigned)grid, bs, 0, st>>>(a);
  else
    k_grad_tsit5_lorenz<T, K, false><<<(unsigned)grid, bs, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_tsit5_lorenz<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                    void*, void*, cudaStream_t);
template gs_status launch_grad_tsit5_lorenz<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                   void*, void*, cudaStream_t);

}  // namespace gs
