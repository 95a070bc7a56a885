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
// offers only three independent chains (x, y, z) per instruction stream.  Each
// thread may carry K adjacent slots (vec<T, K>), giving 3K independent chains.
// gs_record orders slots by decreasing step count, so the K chains of a thread
// (and the 32K of a warp) have nearly equal length; the shorter ones run the
// remaining iterations as steps of size 0, which are exact identities in both
// halves (u + 0 * acc = u; nu = 0 * (...) = 0), so the results are bitwise
// those of one slot per thread.
//
// Store or recompute: the reverse step needs the stage states U_2..U_6 of its
// step.  It recomputes U_2..U_5 from the checkpointed u_s; with KEEP6 the
// forward also keeps U_6 (the costliest to rebuild: a five-term combination
// and the right-hand side at U_5, ~22 FP64 instructions per step) beside u_s,
// for 48 more bytes per step (fp64) of HBM traffic.  The kept U_6 is the value
// the forward computed, so a recompute would give the same bits.
//
// Memory layout: h [smax][n] and the checkpoints ck [smax][R][n] (R = 3 rows
// u_s, or 6 with U_6) are step-major over slots, so at a given step a warp
// touches 32K consecutive elements of every array.  They stream into
// per-thread shared-memory rings with cp.async, kRingF (forward: h) and kRingR
// (reverse: checkpoint rows and h) steps ahead, and are read from there one
// step ahead, so no register waits on DRAM and no barrier is involved: each
// thread waits only on its own copies.
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
// keep U_6 in the checkpoint workspace (1) or recompute it (0), per dtype
#ifndef GS_GRAD_KEEP6_F64
#define GS_GRAD_KEEP6_F64 0
#endif
#ifndef GS_GRAD_KEEP6_F32
#define GS_GRAD_KEEP6_F32 0
#endif
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

template <typename T>
__host__ __device__ constexpr bool keep6() {
  return sizeof(T) == 8 ? GS_GRAD_KEEP6_F64 != 0 : GS_GRAD_KEEP6_F32 != 0;
}
// checkpoint rows per step and slot
template <typename T>
__host__ __device__ constexpr int ck_rows() {
  return keep6<T>() ? 6 : 3;
}
// shared-memory ring elements per thread: the larger of the two rings
template <typename T, int K>
__host__ __device__ constexpr int ring_elems() {
  return (kRingF * K > kRingR * (ck_rows<T>() + 1) * K) ? kRingF * K : kRingR * (ck_rows<T>() + 1) * K;
}

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
  T* ck;            // workspace [smax][ck_rows][n] by slot
  T* gsave;         // workspace tail [nsave][3][n] by slot: landing save points' loss gradients
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

// Tsit5's dense output inside one step of the Lorenz replay (a dense save
// point at theta in (0, 1) of a step of size h from u_s to u_{s+1}).
// Value: the stage states are recomputed from u_s as the forward forms them
// (U[0] = u_s, U[j-1] = U_j for j = 2..6), and
//   u(theta) = u_s + h sum_i b_i(theta) k_i,  k_7 = f(u_{s+1}).
// Adjoint, for a cotangent g of u(theta) (theta and h are data): the slope at
// the step's end gives nu_7 = h b_7 g and A = J(u_{s+1})^T nu_7 at u_{s+1};
// the stage chain
//   nu_j = h (b_j g + sum_{m=j+1..6} a_mj mu_m),  mu_j = J(U_j)^T nu_j,  j = 6..1,
// gives B = g + sum_j mu_j at u_s; pbar gains P = sum_{j=1..7} f_p(U_j)^T nu_j.
__host__ __device__ constexpr int ts_a_idx(int j, int m) { return (j - 2) * (j - 1) / 2 + (m - 1); }
template <typename T>
__device__ __forceinline__ T ts_a(int j, int m) {
  return cst<T>(ts_lit(ts_a_idx(j, m)));
}

template <typename T>
__device__ __forceinline__ void dense_point_lorenz(const T us[3], const T un[3], T s, T r, T b, T h, T th, T ut[3],
                                                   T U[6][3], T bw[7]) {
  T k[7][3];
#pragma unroll
  for (int c = 0; c < 3; ++c) U[0][c] = us[c];
  lorenz_f(us[0], us[1], us[2], s, r, b, k[0][0], k[0][1], k[0][2]);
#pragma unroll
  for (int j = 2; j <= 6; ++j) {
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      T acc = ts_a<T>(j, 1) * k[0][c];
#pragma unroll
      for (int m = 2; m < j; ++m) acc = fmaT(ts_a<T>(j, m), k[m - 1][c], acc);
      U[j - 1][c] = fmaT(h, acc, us[c]);
    }
    lorenz_f(U[j - 1][0], U[j - 1][1], U[j - 1][2], s, r, b, k[j - 1][0], k[j - 1][1], k[j - 1][2]);
  }
  lorenz_f(un[0], un[1], un[2], s, r, b, k[6][0], k[6][1], k[6][2]);
  tsit5_dense_w(th, bw);
#pragma unroll
  for (int c = 0; c < 3; ++c)
    ut[c] = tsit5_dense_c(bw, us[c], k[0][c], k[1][c], k[2][c], k[3][c], k[4][c], k[5][c], k[6][c], h);
}

template <typename T>
__device__ __forceinline__ void dense_point_lorenz_vjp(const T U[6][3], const T un[3], T s, T r, T b, T h,
                                                       const T bw[7], const T g[3], T A[3], T B[3], T P[3]) {
  P[0] = P[1] = P[2] = cst<T>(0.0);
  lorenz_vjp(un[0], un[1], un[2], s, r, b, (h * bw[6]) * g[0], (h * bw[6]) * g[1], (h * bw[6]) * g[2], A[0], A[1],
             A[2], P[0], P[1], P[2]);
  T mu[6][3];
#pragma unroll
  for (int j = 6; j >= 1; --j) {
    T nu[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      T acc = bw[j - 1] * g[c];
#pragma unroll
      for (int m = 6; m > j; --m) acc = fmaT(ts_a<T>(m, j), mu[m - 1][c], acc);
      nu[c] = h * acc;
    }
    lorenz_vjp(U[j - 1][0], U[j - 1][1], U[j - 1][2], s, r, b, nu[0], nu[1], nu[2], mu[j - 1][0], mu[j - 1][1],
               mu[j - 1][2], P[0], P[1], P[2]);
  }
#pragma unroll
  for (int c = 0; c < 3; ++c)
    B[c] = g[c] + (((mu[0][c] + mu[1][c]) + (mu[2][c] + mu[3][c])) + (mu[4][c] + mu[5][c]));
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
  constexpr bool kKeep6 = keep6<T>();
  constexpr int kCk = ck_rows<T>();   // checkpoint rows per step
  constexpr int kRowsR = kCk + 1;     // reverse ring rows per step: checkpoint + h
  constexpr int BS = GS_GRAD_BS;
  const int64_t n = a.n;
  const int64_t nck = kCk * n;        // checkpoint elements per step
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
  // Per-thread copy rings.  Element (row w, slot q) of a thread lives at
  // rg[(w * K + q) * BS]: consecutive threads touch consecutive words.
  // Forward: row w = s % kRingF holds h of step s.  Reverse: rows
  // kRowsR (s % kRingR) + c hold checkpoint row c (c < kCk) and h (c = kCk) of
  // step s.  One commit group per step; a thread waits on its own groups only.
  extern __shared__ __align__(16) unsigned char ring_raw[];  // ring_elems<T, K>() * BS elements
  T* const rg = reinterpret_cast<T*>(ring_raw) + threadIdx.x;

  // ---------------------------------------------------------------- forward
  auto issue_f = [&](int sf) {  // h of step sf into its ring row
#pragma unroll
    for (int q = 0; q < K; ++q)
      if (sf < S[q]) cp_async_el(rg + ((sf & (kRingF - 1)) * K + q) * BS, hp + (int64_t)sf * n + q);
    cp_async_commit();
  };
  auto take_f = [&](int sf, V& hv) {  // its group complete; 0 past a slot's last step
#pragma unroll
    for (int q = 0; q < K; ++q) hv.e[q] = sf < S[q] ? rg[((sf & (kRingF - 1)) * K + q) * BS] : cst<T>(0.0);
  };
  // A save point's step count, and its loss vector (the target for SUMSQ,
  // zero without one; the weights for LINEAR).
  auto sp_idx = [&](int q, int k) -> int {
    return (k >= 0 && k < a.nsave && S[q] > 0) ? a.save_idx[(int64_t)k * n + j0 + q] : -1;
  };
  const T* const lvec = a.loss_kind == GS_LOSS_SUMSQ ? a.target : a.weight;
  auto sp_vec = [&](int q, int k, T& v0, T& v1, T& v2) {
    v0 = v1 = v2 = cst<T>(0.0);
    if (lvec && k >= 0 && k < a.nsave && i[q] >= 0) {
      const int64_t o = (int64_t)k * 3 * n + i[q];
      v0 = lvec[o];
      v1 = lvec[o + n];
      v2 = lvec[o + 2 * n];
    }
  };
  V L = vsplat<T, K>(cst<T>(0.0));
  V k1x, k1y, k1z;
  lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);
  V hn;
#pragma unroll
  for (int sf = 0; sf < kRingF; ++sf) issue_f(sf);
  cp_async_wait<kRingF - 1>();
  take_f(0, hn);
  for (int st = 0; st < Smax; ++st) {
    const V h = hn;
    cp_async_wait<kRingF - 2>();  // the group of step st + 1
    take_f(st + 1, hn);
#pragma unroll
    for (int q = 0; q < K; ++q) {
      if (st < S[q]) {
        cp[q] = x.e[q];
        cp[n + q] = y.e[q];
        cp[2 * n + q] = z.e[q];
      }
    }
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
    if constexpr (kKeep6) {  // U_6 beside u_s
#pragma unroll
      for (int q = 0; q < K; ++q) {
        if (st < S[q]) {
          cp[3 * n + q] = Ux.e[q];
          cp[4 * n + q] = Uy.e[q];
          cp[5 * n + q] = Uz.e[q];
        }
      }
    }
    cp += nck;
    V k6x, k6y, k6z;
    lorenz_f(Ux, Uy, Uz, s, r, b, k6x, k6y, k6z);
    // stage 7 = u_{s+1}
    GS_ACC1(kTsB1, k1)
    GS_ACCN(kTsB2, k2)
    GS_ACCN(kTsB3, k3)
    GS_ACCN(kTsB4, k4)
    GS_ACCN(kTsB5, k5)
    GS_ACCN(kTsB6, k6)
    x = fmaT(h, ax, x);
    y = fmaT(h, ay, y);
    z = fmaT(h, az, z);
    lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);  // FSAL: next step's first slope
    issue_f(st + kRingF);  // into the row that step st has left
  }
  cp_async_wait<0>();  // the reverse reuses the rows
  // Save points: u(t_k) is read off the checkpoints -- the state after step
  // save_idx[k] (the checkpoint of that step, or the final state) for a
  // landing record, Tsit5's continuous extension over the stages of step
  // save_idx[k] - 1 at theta_k (recomputed from its checkpoint) for a dense
  // one -- so every lane
  // sums its loss here at once, in the contract's order (save points, then
  // components), instead of one lane at a time inside the step loop; the
  // values are bitwise those of the step loop.  The loss gradient at each
  // save point (2 (u - target) or the weights) goes to the workspace for the
  // reverse half; for a dense save point its share of the adjoint at the
  // step's two ends, which needs forward values only, is formed here too,
  // so the reverse half just adds it.  Save points are taken while their step counts stay in
  // [1, S] and increase (landing) or do not decrease (dense); nvalid[q] counts
  // them (all of them for a well-formed mesh).
  int nvalid[K];
  {
    int prev[K];
    bool alive[K];
#pragma unroll
    for (int q = 0; q < K; ++q) {
      nvalid[q] = 0;
      prev[q] = DENSE ? 1 : 0;
      alive[q] = S[q] > 0;
    }
    for (int k = 0; k < a.nsave; ++k) {
#pragma unroll
      for (int q = 0; q < K; ++q) {
        if (!alive[q]) continue;
        const int sk = a.save_idx[(int64_t)k * n + j0 + q];
        if (!((DENSE ? sk >= prev[q] : sk > prev[q]) && sk <= S[q])) {
          alive[q] = false;
          continue;
        }
        prev[q] = sk;
        T ux = x.e[q], uy = y.e[q], uz = z.e[q];  // the state after step sk (final: registers)
        if (sk < S[q]) {
          const T* c = a.ck + (int64_t)sk * nck + j0 + q;
          ux = c[0];
          uy = c[n];
          uz = c[2 * n];
        }
        // dense save point inside step sk - 1: Tsit5's continuous extension
        // over that step's stages, recomputed from its checkpoint
        bool inside = false;
        T hs = cst<T>(0.0);
        const T un[3] = {ux, uy, uz};
        T Us[6][3], bw[7];
        if (DENSE) {
          const T th = a.theta[(int64_t)k * n + j0 + q];
          if (th != cst<T>(1.0)) {
            inside = true;
            const T* c = a.ck + (int64_t)(sk - 1) * nck + j0 + q;
            const T us[3] = {c[0], c[n], c[2 * n]};
            hs = hp[(int64_t)(sk - 1) * n + q];
            T ut[3];
            dense_point_lorenz(us, un, s.e[q], r.e[q], b.e[q], hs, th, ut, Us, bw);
            ux = ut[0];
            uy = ut[1];
            uz = ut[2];
          }
        }
        T v0, v1, v2, g0, g1, g2;
        sp_vec(q, k, v0, v1, v2);
        T Lq = L.e[q];
        if (a.loss_kind == GS_LOSS_SUMSQ) {  // u - 0 = u bitwise when there is no target
          const T dx = ux - v0;
          const T dy = uy - v1;
          const T dz = uz - v2;
          Lq = fmaT(dx, dx, Lq);
          Lq = fmaT(dy, dy, Lq);
          Lq = fmaT(dz, dz, Lq);
          g0 = cst<T>(2.0) * dx;
          g1 = cst<T>(2.0) * dy;
          g2 = cst<T>(2.0) * dz;
        } else {
          Lq = fmaT(v0, ux, Lq);
          Lq = fmaT(v1, uy, Lq);
          Lq = fmaT(v2, uz, Lq);
          g0 = v0;
          g1 = v1;
          g2 = v2;
        }
        L.e[q] = Lq;
        if (!DENSE) {
          T* G = a.gsave + (int64_t)k * 3 * n + j0 + q;
          G[0] = g0;
          G[n] = g1;
          G[2 * n] = g2;
        } else {
          // The dense output's cotangent g, split between the step's ends
          // (it depends on forward values only, so it is formed here): A
          // joins lambda at u_sk, B at u_sk-1 and P joins pbar
          // (dense_point_lorenz_vjp); a save point at a step end has A = g,
          // B = P = 0.
          T A[3] = {g0, g1, g2}, B[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)}, Pp[3] = {B[0], B[1], B[2]};
          if (inside) {
            const T g[3] = {g0, g1, g2};
            dense_point_lorenz_vjp(Us, un, s.e[q], r.e[q], b.e[q], hs, bw, g, A, B, Pp);
          }
          T* G = a.gsave + (int64_t)k * 9 * n + j0 + q;
          G[0] = A[0];
          G[n] = A[1];
          G[2 * n] = A[2];
          G[3 * n] = B[0];
          G[4 * n] = B[1];
          G[5 * n] = B[2];
          G[6 * n] = Pp[0];
          G[7 * n] = Pp[1];
          G[8 * n] = Pp[2];
        }
        nvalid[q] = k + 1;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < K; ++q)
    if (i[q] >= 0) a.loss[i[q]] = L.e[q];

  // ---------------------------------------------------------------- reverse
  // At the top of iteration st, (x, y, z) holds u_{st+1} (the final state
  // first, then the state loaded by the previous iteration), which is what the
  // save-point test needs; (cx, cy, cz, hc) and, with KEEP6, (gx6, gy6, gz6)
  // are u_st, h_st and U_6 of step st, taken from the ring at the end of the
  // previous iteration.
  V lx = vsplat<T, K>(cst<T>(0.0)), ly = lx, lz = lx;
  V ps = lx, pr = lx, pb = lx;
  // Save points in reverse, read one save point ahead: next[q] is the step
  // count at which slot q's current save point kk[q] falls, (tv0, tv1,
  // tv2)[q] its loss gradient (from the workspace) and next2[q] the step count
  // of the save point before it.  Each load is issued a whole save interval
  // before its value is used, so the divergent save-point branch never waits
  // on DRAM.
  int kk[K], next[K], next2[K];
  T tv0[K], tv1[K], tv2[K];
  auto sp_g = [&](int q, int k, T& v0, T& v1, T& v2) {
    v0 = v1 = v2 = cst<T>(0.0);
    if (k >= 0 && k < nvalid[q]) {
      const T* G = a.gsave + (int64_t)k * 3 * n + j0 + q;
      v0 = G[0];
      v1 = G[n];
      v2 = G[2 * n];
    }
  };
#pragma unroll
  for (int q = 0; q < K; ++q) {
    kk[q] = nvalid[q] - 1;
    next[q] = sp_idx(q, kk[q]);
    next2[q] = sp_idx(q, kk[q] - 1);
    if (!DENSE) sp_g(q, kk[q], tv0[q], tv1[q], tv2[q]);
  }
  V cx = x, cy = y, cz = z, hc = vsplat<T, K>(cst<T>(0.0));
  V gx6 = x, gy6 = y, gz6 = z;
  auto issue_r = [&](int sr) {  // step sr's checkpoint rows and h
#pragma unroll
    for (int q = 0; q < K; ++q) {
      if (sr >= 0 && sr < S[q]) {
        T* d = rg + ((sr & (kRingR - 1)) * kRowsR * K + q) * BS;
        const T* c = a.ck + (int64_t)sr * nck + j0 + q;
#pragma unroll
        for (int w = 0; w < kCk; ++w) cp_async_el(d + w * K * BS, c + w * n);
        cp_async_el(d + kCk * K * BS, hp + (int64_t)sr * n + q);
      }
    }
    cp_async_commit();
  };
  // step sr's values, its group complete; a slot past its last step runs an
  // identity step (h = 0) at its final state
  auto take_r = [&](int sr) {
#pragma unroll
    for (int q = 0; q < K; ++q) {
      const T* d = rg + ((sr & (kRingR - 1)) * kRowsR * K + q) * BS;
      if (sr < S[q]) {
        cx.e[q] = d[0];
        cy.e[q] = d[K * BS];
        cz.e[q] = d[2 * K * BS];
        if constexpr (kKeep6) {
          gx6.e[q] = d[3 * K * BS];
          gy6.e[q] = d[4 * K * BS];
          gz6.e[q] = d[5 * K * BS];
        }
        hc.e[q] = d[kCk * K * BS];
      } else {
        hc.e[q] = cst<T>(0.0);
      }
    }
  };
#pragma unroll
  for (int i2 = 0; i2 < kRingR; ++i2) issue_r(Smax - 1 - i2);
  cp_async_wait<kRingR - 1>();
  if (Smax > 0) take_r(Smax - 1);
  for (int st = Smax - 1; st >= 0; --st) {
    // save points reached at u_{st+1}: landing ones add their loss gradient to
    // lambda; dense ones add A now, B once step st is transposed (pgx..z) and
    // P to pbar (the increments formed after the forward half)
    V pgx, pgy, pgz;
    if (DENSE) {
      pgx = vsplat<T, K>(cst<T>(0.0));
      pgy = pgx, pgz = pgx;
    }
#pragma unroll
    for (int q = 0; q < K; ++q) {
      while (st + 1 == next[q]) {
        if (!DENSE) {
          lx.e[q] += tv0[q];  // d loss_k / d u(t_k), from the forward half
          ly.e[q] += tv1[q];
          lz.e[q] += tv2[q];
        } else {
          const T* G = a.gsave + (int64_t)kk[q] * 9 * n + j0 + q;
          if (kk[q] >= 0 && kk[q] < nvalid[q]) {
            lx.e[q] += G[0];
            ly.e[q] += G[n];
            lz.e[q] += G[2 * n];
            pgx.e[q] += G[3 * n];
            pgy.e[q] += G[4 * n];
            pgz.e[q] += G[5 * n];
            ps.e[q] += G[6 * n];
            pr.e[q] += G[7 * n];
            pb.e[q] += G[8 * n];
          }
        }
        --kk[q];
        next[q] = next2[q];
        next2[q] = sp_idx(q, kk[q] - 1);
        if (!DENSE) sp_g(q, kk[q], tv0[q], tv1[q], tv2[q]);
        if (!DENSE) break;
      }
    }
    x = cx;
    y = cy;
    z = cz;
    const V h = hc;
    V U6x, U6y, U6z;
    if constexpr (kKeep6) {
      U6x = gx6;
      U6y = gy6;
      U6z = gz6;
    }
    // recompute the stage states of step st (same arithmetic as the forward)
    V ax, ay, az;
    V f1x, f1y, f1z;
    lorenz_f(x, y, z, s, r, b, f1x, f1y, f1z);
    V U2x, U2y, U2z, U3x, U3y, U3z, U4x, U4y, U4z, U5x, U5y, U5z;
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
    if constexpr (!kKeep6) {
      V f5x, f5y, f5z;
      lorenz_f(U5x, U5y, U5z, s, r, b, f5x, f5y, f5z);
      GS_ACC1(kTsA61, f1)
      GS_ACCN(kTsA62, f2)
      GS_ACCN(kTsA63, f3)
      GS_ACCN(kTsA64, f4)
      GS_ACCN(kTsA65, f5)
      GS_STAGE(U6x, U6y, U6z, ax, ay, az)
    }

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
      lx += pgx;
      ly += pgy;
      lz += pgz;
    }
    // step st - 1's ring entries into registers only now, after the
    // transposed step: they are not live across it (3 fewer registers at its
    // peak, ~1 % faster than taking them at the top of the iteration), and
    // their copies have had the whole iteration to land
    if (st > 0) {
      cp_async_wait<kRingR - 2>();  // the group of step st - 1
      take_r(st - 1);
    }
    issue_r(st - kRingR);  // into the rows that step st has left
  }
  cp_async_wait<0>();
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

// Gradient workspace: checkpoint rows per step and slot (3, or 6 when U_6 is
// kept), then per save point the loss gradients of a landing record
// ([nsave][3][n]) or the increments A, B, P of a dense one ([nsave][9][n]).
size_t grad_tsit5_lorenz_ws_bytes(int32_t dtype, int64_t n, int32_t smax, int32_t nsave, bool dense) {
  const size_t rows = dtype == GS_F64 ? ck_rows<double>() : ck_rows<float>();
  const size_t tsize = dtype == GS_F64 ? 8 : 4;
  return ((size_t)smax * rows + (size_t)nsave * (dense ? 9 : 3)) * (size_t)n * tsize;
}

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
  a.gsave = (T*)ws + (size_t)M->smax * ck_rows<T>() * (size_t)P->n;
  a.theta = (const T*)M->save_theta;
  constexpr int K = GS_GRAD_K;
  const int bs = GS_GRAD_BS;
  const int64_t threads = (P->n + K - 1) / K;
  const int64_t grid = (threads + bs - 1) / bs;
  const size_t smem = (size_t)ring_elems<T, K>() * bs * sizeof(T);
  auto kern = a.theta ? k_grad_tsit5_lorenz<T, K, true> : k_grad_tsit5_lorenz<T, K, false>;
  // the rings may exceed the 48 KB a launch gets without asking
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return GS_ECUDA;
  kern<<<(unsigned)grid, bs, smem, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_tsit5_lorenz<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                    void*, void*, cudaStream_t);
template gs_status launch_grad_tsit5_lorenz<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                   void*, void*, cudaStream_t);

}  // namespace gs
