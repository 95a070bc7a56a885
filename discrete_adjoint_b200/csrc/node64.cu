// node64.cu -- the d = 64 shared-weight system  du/dt = tanh(W u + b_i) - u
// (one W for the whole ensemble, a bias b_i per trajectory): adaptive Tsit5
// recorder, forward-only solve, and the fused replay + reverse sweep with the
// weight gradient summed over the ensemble.
//
// GRADSOLVE (arXiv 2609.02876) differentiates registered right-hand sides up to
// state dimension 64 (evolve.pub review, "Summary"); this is the neural
// right-hand side of its neural-ODE study, with gradients dL/db_i, dL/du0_i and
// dL/dW = sum_i dL_i/dW.
//
// Layout: a CTA of 256 threads carries 32 trajectories (slots).  Every
// per-trajectory vector of the CTA is a 64 x 32 tile [component][slot]; thread
// (ty, tx) = (tid / 16, tid % 16) owns rows 4ty..4ty+3 of slots 2tx, 2tx+1 of
// every tile, in registers, so all element-wise stage arithmetic is local.
// The stage products are matrix products over the CTA's 32 trajectories, with
// operands staged in shared memory:
//   Z = W U      (z_r = b_r + sum_k W_rk U_k, accumulated in k = 0..63 order:
//                 the floating-point contract's order for this right-hand side)
//   M = W^T G    (mu = W^T g - nu, the vector-Jacobian product)
//   dW += G U^T  (over the 32 slots; per-CTA partials, summed afterwards in
//                 a fixed order so the weight gradient is deterministic)
// The per-trajectory parts of the recorder (error norm as the contract's
// sequential sum over components, the PI controller) run one thread per slot.
#include <atomic>

#include "steps.cuh"

namespace gs {

namespace n64 {

constexpr int D = 64;
constexpr int TB = 32;     // trajectories (slots) per CTA
constexpr int NT = 256;    // threads per CTA
constexpr int LDT = D + 4;  // row stride of the [slot][component] tiles

// Per-thread block of a 64 x 32 tile: 4 rows x 2 slots.
template <typename T>
struct Blk {
  T v[4][2];
};

template <typename T>
__device__ __forceinline__ Blk<T> bzero() {
  Blk<T> r;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 2; ++c) r.v[a][c] = cst<T>(0.0);
  return r;
}

template <typename T>
struct Smem {
  T W[D][D];    // W[r][k]
  T Wt[D][D];   // Wt[k][r] = W[r][k]
  T B[D][TB];   // operand [component][slot]
  T G[D][TB];   // second operand [component][slot]
  T Gt[TB][LDT];  // [slot][component]
  T Ut[TB][LDT];  // [slot][component]
  T red[D][TB];   // per-slot reductions (scaled errors, norms)
  T hs[TB];       // per-slot step of the current attempt
  int flag[TB];   // per-slot accept / state flags
  int sv[TB];     // per-slot save point reached by the accepted step, or -1
  int any;
};

// Z_block = W * B (contract order: start at bias, fma over k = 0..63).
template <typename T>
__device__ __forceinline__ Blk<T> matmul_WB(const Smem<T>& s, const Blk<T>& bias, int ty, int tx) {
  Blk<T> z = bias;
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    T w[4], u[2];
#pragma unroll
    for (int a = 0; a < 4; ++a) w[a] = s.Wt[k][4 * ty + a];
    u[0] = s.B[k][2 * tx];
    u[1] = s.B[k][2 * tx + 1];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 2; ++c) z.v[a][c] = fmaT(w[a], u[c], z.v[a][c]);
  }
  return z;
}

// M_block = W^T * G.
template <typename T>
__device__ __forceinline__ Blk<T> matmul_WtG(const Smem<T>& s, int ty, int tx) {
  Blk<T> m = bzero<T>();
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    T w[4], g[2];
#pragma unroll
    for (int a = 0; a < 4; ++a) w[a] = s.W[k][4 * ty + a];
    g[0] = s.G[k][2 * tx];
    g[1] = s.G[k][2 * tx + 1];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 2; ++c) m.v[a][c] = fmaT(w[a], g[c], m.v[a][c]);
  }
  return m;
}

template <typename T>
__device__ __forceinline__ void store_B(Smem<T>& s, const Blk<T>& x, int ty, int tx) {
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    s.B[4 * ty + a][2 * tx] = x.v[a][0];
    s.B[4 * ty + a][2 * tx + 1] = x.v[a][1];
  }
}

// y = tanh(z), k = y - U  (the right-hand side on a stage state)
template <typename T>
__device__ __forceinline__ void rhs_tail(const Blk<T>& z, const Blk<T>& U, Blk<T>& y, Blk<T>& k) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      y.v[a][c] = tanh(z.v[a][c]);
      k.v[a][c] = y.v[a][c] - U.v[a][c];
    }
}

// f(U) for the CTA: stage U through shared memory, multiply, apply tanh.
template <typename T>
__device__ __forceinline__ void eval_f(Smem<T>& s, const Blk<T>& U, const Blk<T>& bias, Blk<T>& y, Blk<T>& k, int ty,
                                       int tx) {
  __syncthreads();  // previous readers of B are done
  store_B(s, U, ty, tx);
  __syncthreads();
  Blk<T> z = matmul_WB(s, bias, ty, tx);
  rhs_tail(z, U, y, k);
}

// U = fma(h, sum_m a_m k_m, u) with the contract's order (first term a plain
// product, then fmas in increasing m).
template <typename T, int NS>
__device__ __forceinline__ Blk<T> stage(const T (&coef)[NS], const Blk<T>* const (&ks)[NS], const Blk<T>& u,
                                        const T (&h)[2]) {
  Blk<T> U;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      T acc = coef[0] * ks[0]->v[a][c];
#pragma unroll
      for (int m = 1; m < NS; ++m) acc = fmaT(coef[m], ks[m]->v[a][c], acc);
      U.v[a][c] = fmaT(h[c], acc, u.v[a][c]);
    }
  return U;
}

// Tsit5 stages 2..7 from u and k1; returns u_new (stage 7) and k2..k7.
template <typename T>
__device__ __forceinline__ void tsit5_stages(Smem<T>& s, const Blk<T>& u, const Blk<T>& bias, const T (&h)[2],
                                             const Blk<T>& k1, Blk<T>& k2, Blk<T>& k3, Blk<T>& k4, Blk<T>& k5,
                                             Blk<T>& k6, Blk<T>& k7, Blk<T>& un, int ty, int tx) {
  Blk<T> y, U;
  {
    const T c[1] = {cst<T>(TS_A21)};
    const Blk<T>* const ks[1] = {&k1};
    U = stage<T, 1>(c, ks, u, h);
    eval_f(s, U, bias, y, k2, ty, tx);
  }
  {
    const T c[2] = {cst<T>(TS_A31), cst<T>(TS_A32)};
    const Blk<T>* const ks[2] = {&k1, &k2};
    U = stage<T, 2>(c, ks, u, h);
    eval_f(s, U, bias, y, k3, ty, tx);
  }
  {
    const T c[3] = {cst<T>(TS_A41), cst<T>(TS_A42), cst<T>(TS_A43)};
    const Blk<T>* const ks[3] = {&k1, &k2, &k3};
    U = stage<T, 3>(c, ks, u, h);
    eval_f(s, U, bias, y, k4, ty, tx);
  }
  {
    const T c[4] = {cst<T>(TS_A51), cst<T>(TS_A52), cst<T>(TS_A53), cst<T>(TS_A54)};
    const Blk<T>* const ks[4] = {&k1, &k2, &k3, &k4};
    U = stage<T, 4>(c, ks, u, h);
    eval_f(s, U, bias, y, k5, ty, tx);
  }
  {
    const T c[5] = {cst<T>(TS_A61), cst<T>(TS_A62), cst<T>(TS_A63), cst<T>(TS_A64), cst<T>(TS_A65)};
    const Blk<T>* const ks[5] = {&k1, &k2, &k3, &k4, &k5};
    U = stage<T, 5>(c, ks, u, h);
    eval_f(s, U, bias, y, k6, ty, tx);
  }
  {
    const T c[6] = {cst<T>(TS_B1), cst<T>(TS_B2), cst<T>(TS_B3), cst<T>(TS_B4), cst<T>(TS_B5), cst<T>(TS_B6)};
    const Blk<T>* const ks[6] = {&k1, &k2, &k3, &k4, &k5, &k6};
    un = stage<T, 6>(c, ks, u, h);
    eval_f(s, un, bias, y, k7, ty, tx);
  }
}

template <typename T>
__device__ __forceinline__ void load_W(Smem<T>& s, const T* W, int tid) {
  for (int q = tid; q < D * D; q += NT) {
    const int r = q / D, k = q % D;
    const T w = W[q];
    s.W[r][k] = w;
    s.Wt[k][r] = w;
  }
}

// Sequential per-slot sum over components of red[c][slot] (contract order):
// slot t's thread returns sqrt(sum / 64) -- the RMS norm of the scaled values.
template <typename T>
__device__ __forceinline__ T slot_rms(const Smem<T>& s, int t) {
  T acc = cst<T>(0.0);
  for (int c = 0; c < D; ++c) acc = fmaT(s.red[c][t], s.red[c][t], acc);
  return sqrt(acc / cst<T>(64.0));
}

// ---------------------------------------------------------------------------
// Recorder: one CTA per 32 trajectories, in trajectory order (slot = index).
// ---------------------------------------------------------------------------
template <typename T>
struct RecArgs64 {
  int64_t n;
  const T* p;   // b [64][n]
  const T* u0;  // [64][n]
  const T* W;   // [64][64]
  T t0, t1, rtol, atol, h0;
  int32_t nsave, smax;
  T tsave[GS_MAX_SAVE];
  bool store;
  T* h;               // [n][smax] (trajectory-major workspace copy)
  int32_t* save_idx;  // [nsave][n]
  int32_t* nsteps;
  int32_t* status;
  int32_t* nreject;
  T* u_save;  // adaptive forward-only solve: [nsave][64][n] by trajectory, else null
};

// Per-trajectory state of the d = 64 recorders: time, proposal, the
// controller's ln(errprev), counts, next save point, status.
template <typename T>
struct Ctl64 {
  T tcur, hprop, lnprev;
  int nst, nrej, kk, status;
  bool prev_rej, done;
};

// The outcome of trajectory it's attempt with scaled error err and step hcur
// (clipped onto tstop, or ending at tn): accepted -> the step is stored (a
// trajectory-major workspace copy), t advances, the save point reached is
// returned in hit, and the PI factor 0.9 err^(-0.7/q) errprev^(0.4/q)
// (clipped to [0.2, 10], at most 1 right after a rejection) scales the
// proposal; rejected -> the proposal shrinks by max(0.2, 0.9 err^(-1/q)).
// Exceeding smax accepted or rejected attempts ends the trajectory with
// MAXSTEPS.  Returns 1 when the step is accepted.
template <typename T>
__device__ __forceinline__ int ctl_decide(Ctl64<T>& rec, const RecArgs64<T>& a, int64_t it, T err, T hcur,
                                          bool clipped, T tstop, T tn, T ln_floor, int& hit) {
  const int64_t n = a.n;
  const T qord = cst<T>(5.0);
  int accept = 0;
  hit = -1;
  if (err <= cst<T>(1.0)) {
    if (rec.nst >= a.smax) {
      rec.status = GS_TRAJ_MAXSTEPS;
      rec.done = true;
    } else {
      accept = 1;
      if (a.store) a.h[it * a.smax + rec.nst] = hcur;  // trajectory-major workspace copy
      ++rec.nst;
      rec.tcur = clipped ? tstop : tn;
      while (rec.kk < a.nsave && rec.tcur == a.tsave[rec.kk]) {  // save times increase: one hit at most
        if (a.store) a.save_idx[(int64_t)rec.kk * n + it] = rec.nst;
        hit = rec.kk;
        ++rec.kk;
      }
      T fac, lnerr = ln_floor;
      if (err == cst<T>(0.0)) {
        fac = cst<T>(10.0);
      } else {
        lnerr = ctrl_ln<T>(err);
        fac = cst<T>(0.9) * ctrl_exp<T>(fmaT(-(cst<T>(0.7) / qord), lnerr, (cst<T>(0.4) / qord) * rec.lnprev));
        fac = smin_(cst<T>(10.0), smax_(cst<T>(0.2), fac));
      }
      if (rec.prev_rej) fac = smin_(fac, cst<T>(1.0));
      rec.lnprev = err < cst<T>(1e-4) ? ln_floor : lnerr;
      rec.prev_rej = false;
      rec.hprop = fac * rec.hprop;
      if (rec.tcur >= a.t1) rec.done = true;
    }
  } else {
    ++rec.nrej;
    if (rec.nrej > a.smax) {
      rec.status = GS_TRAJ_MAXSTEPS;
      rec.done = true;
    } else {
      const T fac = !isfinite(err) ? cst<T>(0.2)
                                   : smax_(cst<T>(0.2), cst<T>(0.9) * ctrl_exp<T>(-(cst<T>(1.0) / qord) *
                                                                                    ctrl_ln<T>(err)));
      rec.hprop = fac * rec.hprop;
      rec.prev_rej = true;
    }
  }
  return accept;
}

template <typename T>
__global__ void __launch_bounds__(NT, 1) k_record_node64(RecArgs64<T> a) {
  extern __shared__ unsigned char smem_raw[];
  Smem<T>& s = *reinterpret_cast<Smem<T>*>(smem_raw);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t n = a.n;
  const int64_t base = (int64_t)blockIdx.x * TB;
  load_W(s, a.W, tid);
  Blk<T> u, bias;
  bool col_ok[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int64_t i = base + 2 * tx + c;
    col_ok[c] = i < n;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = 4 * ty + q;
      u.v[q][c] = col_ok[c] ? a.u0[(int64_t)r * n + i] : cst<T>(0.0);
      bias.v[q][c] = col_ok[c] ? a.p[(int64_t)r * n + i] : cst<T>(0.0);
    }
  }
  // per-slot controller state, held by thread t < 32 for slot t
  const int t = tid;
  const bool ctl = t < TB;
  const int64_t it = base + t;
  const bool live = ctl && it < n;
  const T eps = Eps<T>::v;
  const T qord = cst<T>(5.0);
  Ctl64<T> rec{a.t0, cst<T>(0.0), cst<T>(0.0), 0, 0, 0, live ? GS_TRAJ_OK : GS_TRAJ_MAXSTEPS, false, !live};
  const T ln_floor = ctrl_ln<T>(cst<T>(1e-4));

  // k1 = f(u0) and the starting step (Hairer, Norsett & Wanner I, II.4)
  Blk<T> y, k1;
  eval_f(s, u, bias, y, k1, ty, tx);
  // finiteness of u0 and f(u0): per-slot flag via shared memory
  if (ctl) s.flag[t] = 1;
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < 2; ++c)
      if (!isfinite(u.v[q][c]) || !isfinite(k1.v[q][c])) s.flag[2 * tx + c] = 0;
  // d0 = rms(u0 / sc), sc = fma(rtol, |u0|, atol)
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < 2; ++c) s.red[4 * ty + q][2 * tx + c] = u.v[q][c] / fmaT(a.rtol, fabs(u.v[q][c]), a.atol);
  __syncthreads();
  T d0 = ctl ? slot_rms(s, t) : cst<T>(0.0);
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < 2; ++c) s.red[4 * ty + q][2 * tx + c] = k1.v[q][c] / fmaT(a.rtol, fabs(u.v[q][c]), a.atol);
  __syncthreads();
  T d1 = ctl ? slot_rms(s, t) : cst<T>(0.0);
  T h0 = (d0 < cst<T>(1e-5) || d1 < cst<T>(1e-5)) ? cst<T>(1e-6) : cst<T>(0.01) * (d0 / d1);
  h0 = smin_(h0, a.t1 - a.t0);
  if (ctl) s.hs[t] = h0;
  __syncthreads();
  Blk<T> u1, k1b;
  {
    const T hh[2] = {s.hs[2 * tx], s.hs[2 * tx + 1]};
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int c = 0; c < 2; ++c) u1.v[q][c] = fmaT(hh[c], k1.v[q][c], u.v[q][c]);
  }
  eval_f(s, u1, bias, y, k1b, ty, tx);
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < 2; ++c)
      s.red[4 * ty + q][2 * tx + c] = (k1b.v[q][c] - k1.v[q][c]) / fmaT(a.rtol, fabs(u.v[q][c]), a.atol);
  __syncthreads();
  if (ctl) {
    const T d2 = slot_rms(s, t) / h0;
    const T dm = smax_(d1, d2);
    const T h1 = dm <= cst<T>(1e-15) ? smax_(cst<T>(1e-6), h0 * cst<T>(1e-3))
                                     : ctrl_pow<T>(cst<T>(0.01) / dm, cst<T>(1.0) / qord);
    rec.hprop = a.h0 > cst<T>(0.0) ? a.h0 : smin_(smin_(cst<T>(100.0) * h0, h1), a.t1 - a.t0);
    if (live && (s.flag[t] == 0 || !(rec.hprop > cst<T>(0.0)) || !isfinite(rec.hprop))) {
      rec.status = GS_TRAJ_NONFINITE;
      rec.done = true;
    }
  }

  Blk<T> k2, k3, k4, k5, k6, k7, un;
  for (int iter = 0;; ++iter) {
    // --- per-slot: choose the attempt
    bool clipped = false;
    T tstop = a.t1, tn = rec.tcur;
    if (ctl) {
      if (!rec.done && rec.hprop < cst<T>(16.0) * eps * fabs(rec.tcur)) {
        rec.status = GS_TRAJ_DTMIN;
        rec.done = true;
      }
      T hh = cst<T>(0.0);
      if (!rec.done) {
        tstop = rec.kk < a.nsave ? a.tsave[rec.kk] : a.t1;
        tn = rec.tcur + rec.hprop;
        clipped = tn >= tstop - cst<T>(4.0) * eps * fabs(tstop);
        hh = clipped ? tstop - rec.tcur : rec.hprop;
      }
      s.hs[t] = hh;
      s.flag[t] = rec.done ? 0 : 1;
    }
    __syncthreads();
    if (ctl) {
      // any slot still running?
      if (t == 0) {
        int any = 0;
        for (int q = 0; q < TB; ++q) any |= s.flag[q];
        s.any = any;
      }
    }
    __syncthreads();
    if (!s.any) break;
    const T hh[2] = {s.hs[2 * tx], s.hs[2 * tx + 1]};
    tsit5_stages(s, u, bias, hh, k1, k2, k3, k4, k5, k6, k7, un, ty, tx);
    // scaled error e / sc into red
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        T acc = cst<T>(TS_E1) * k1.v[q][c];
        acc = fmaT(cst<T>(TS_E2), k2.v[q][c], acc);
        acc = fmaT(cst<T>(TS_E3), k3.v[q][c], acc);
        acc = fmaT(cst<T>(TS_E4), k4.v[q][c], acc);
        acc = fmaT(cst<T>(TS_E5), k5.v[q][c], acc);
        acc = fmaT(cst<T>(TS_E6), k6.v[q][c], acc);
        acc = fmaT(cst<T>(TS_E7), k7.v[q][c], acc);
        const T e = hh[c] * acc;
        const T sc = fmaT(a.rtol, smax_(fabs(u.v[q][c]), fabs(un.v[q][c])), a.atol);
        s.red[4 * ty + q][2 * tx + c] = e / sc;
      }
    __syncthreads();
    // --- per-slot: accept / reject, controller
    if (ctl) {
      int accept = 0, hit = -1;
      if (!rec.done)
        accept = ctl_decide(rec, a, it, slot_rms(s, t), s.hs[t], clipped, tstop, tn, ln_floor, hit);
      s.flag[t] = accept;
      s.sv[t] = hit;
    }
    __syncthreads();
    // --- every thread: take the accepted steps
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      if (s.flag[2 * tx + c]) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          u.v[q][c] = un.v[q][c];
          k1.v[q][c] = k7.v[q][c];
        }
        const int k = s.sv[2 * tx + c];
        if (a.u_save && k >= 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q) a.u_save[((int64_t)k * D + 4 * ty + q) * n + base + 2 * tx + c] = u.v[q][c];
        }
      }
    }
  }
  if (live && a.u_save && rec.status != GS_TRAJ_OK) {
    // a failed trajectory has no solution: NaN at every save point
    const T nan = cst<T>(__int_as_float(0x7fc00000));
    for (int k = 0; k < a.nsave; ++k)
      for (int r = 0; r < D; ++r) a.u_save[((int64_t)k * D + r) * n + it] = nan;
  }
  if (live) {
    if (a.store)
      for (int k = rec.kk; k < a.nsave; ++k) a.save_idx[(int64_t)k * n + it] = 0;
    if (a.nsteps) a.nsteps[it] = rec.nst;
    if (a.status) a.status[it] = rec.status;
    if (a.nreject) a.nreject[it] = rec.nrej;
  }
}

// ---------------------------------------------------------------------------
// Forward replay (solve) and fused replay + reverse sweep (grad), on slots.
// ---------------------------------------------------------------------------
template <typename T>
struct GradArgs64 {
  int64_t n;
  const T* p;
  const T* u0;
  const T* W;
  const T* h;
  const int32_t* order;
  const int32_t* nsteps;
  const int32_t* save_idx;
  const int32_t* status;
  int32_t nsave, smax;
  int32_t loss_kind;
  const T* target;
  const T* weight;
  T* loss;
  T* dp;
  T* du0;
  T* ck;       // workspace [smax][64][n] by slot
  T* dW_part;  // workspace [parts][64][64]: one per CTA
  T* kst;      // tensor-core gradient: stage slopes k_1..k_6 [smax][6][64][n] by slot
  T* u_save;   // solve: [nsave][64][n] by trajectory
};

// Loss of the save point each flagged slot has reached: the terms of the
// thread's rows go to red (and G for a linear loss), then the slot's thread
// sums them in the contract's order (components 0..63, fma chain).
template <typename T, typename SM>
__device__ __forceinline__ void save_point_loss(SM& s, const GradArgs64<T>& a, const Blk<T>& u,
                                                const int64_t (&o)[2], const bool (&hit)[2], T& Lslot, int ty,
                                                int tx, int tid) {
  __syncthreads();
  if (tid < TB) s.flag[tid] = 0;
  __syncthreads();
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    if (!hit[c]) continue;
    if (ty == 0) s.flag[2 * tx + c] = 1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = 4 * ty + q;
      const int64_t oo = o[c] + (int64_t)r * a.n;
      if (a.loss_kind == GS_LOSS_SUMSQ) {
        s.red[r][2 * tx + c] = a.target ? u.v[q][c] - a.target[oo] : u.v[q][c];
      } else {
        s.red[r][2 * tx + c] = a.weight[oo];
        s.G[r][2 * tx + c] = u.v[q][c];
      }
    }
  }
  __syncthreads();
  if (tid < TB && s.flag[tid]) {
    T L = Lslot;
    for (int r = 0; r < D; ++r)
      L = a.loss_kind == GS_LOSS_SUMSQ ? fmaT(s.red[r][tid], s.red[r][tid], L) : fmaT(s.red[r][tid], s.G[r][tid], L);
    Lslot = L;
  }
}

template <typename T, bool GRAD>
__global__ void __launch_bounds__(NT, 1) k_replay_node64(GradArgs64<T> a) {
  extern __shared__ unsigned char smem_raw[];
  Smem<T>& s = *reinterpret_cast<Smem<T>*>(smem_raw);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t n = a.n;
  const int64_t base = (int64_t)blockIdx.x * TB;
  const int64_t n64 = (int64_t)D * n;
  const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
  load_W(s, a.W, tid);

  // slots of this thread's two columns
  int64_t traj[2];
  int S[2];
  bool act[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int64_t j = base + 2 * tx + c;
    traj[c] = -1;
    S[c] = 0;
    act[c] = false;
    if (j < n) {
      const int64_t i = a.order[j];
      if (i >= 0 && i < n) {
        traj[c] = i;
        const int sq = a.nsteps[j];
        if (a.status[j] == GS_TRAJ_OK && sq >= 0 && sq <= a.smax) {
          S[c] = sq;
          act[c] = true;
        }
      }
    }
  }
  // CTA-wide chain length
  if (tid < TB) s.flag[tid] = 0;
  __syncthreads();
  if (ty == 0) {
    s.flag[2 * tx] = S[0];
    s.flag[2 * tx + 1] = S[1];
  }
  __syncthreads();
  int Smax = 0;
  for (int q = 0; q < TB; ++q) Smax = s.flag[q] > Smax ? s.flag[q] : Smax;
  // the thread that owns slot tid (tid < 32) keeps that slot's loss
  T Lslot = cst<T>(0.0);

  Blk<T> u, bias;
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = 4 * ty + q;
      u.v[q][c] = act[c] ? a.u0[(int64_t)r * n + traj[c]] : cst<T>(0.0);
      bias.v[q][c] = act[c] ? a.p[(int64_t)r * n + traj[c]] : cst<T>(0.0);
    }
  int kk[2] = {0, 0}, next[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) next[c] = act[c] && S[c] > 0 ? a.save_idx[base + 2 * tx + c] : -1;

  // ---------------------------------------------------------------- forward
  {
    Blk<T> y, k1, k2, k3, k4, k5, k6, k7, un;
    eval_f(s, u, bias, y, k1, ty, tx);
    for (int st = 0; st < Smax; ++st) {
      T hh[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        hh[c] = st < S[c] ? a.h[(int64_t)st * n + base + 2 * tx + c] : cst<T>(0.0);
        if (GRAD && st < S[c]) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            a.ck[(int64_t)st * n64 + (int64_t)(4 * ty + q) * n + base + 2 * tx + c] = u.v[q][c];
        }
      }
      tsit5_stages(s, u, bias, hh, k1, k2, k3, k4, k5, k6, k7, un, ty, tx);
      u = un;
      k1 = k7;
      bool hit[2];
      int64_t o[2];
      int anyhit = 0;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        hit[c] = st + 1 == next[c];
        o[c] = hit[c] ? (int64_t)kk[c] * n64 + traj[c] : 0;
        anyhit |= hit[c];
        if (hit[c]) {
          if (!GRAD) {
#pragma unroll
            for (int q = 0; q < 4; ++q) a.u_save[o[c] + (int64_t)(4 * ty + q) * n] = u.v[q][c];
          }
          ++kk[c];
          next[c] = kk[c] < a.nsave ? a.save_idx[(int64_t)kk[c] * n + base + 2 * tx + c] : -1;
        }
      }
      if (GRAD && __syncthreads_or(anyhit)) save_point_loss(s, a, u, o, hit, Lslot, ty, tx, tid);
    }
  }
  if (!GRAD) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
      if (!act[c] && traj[c] >= 0)
        for (int k = 0; k < a.nsave; ++k)
#pragma unroll
          for (int q = 0; q < 4; ++q) a.u_save[(int64_t)k * n64 + (int64_t)(4 * ty + q) * n + traj[c]] = nan;
    return;
  }
  // loss per slot (thread tid < 32 owns slot tid)
  if (tid < TB) {
    const int64_t j = base + tid;
    if (j < n) {
      const int64_t i = a.order[j];
      if (i >= 0 && i < n) {
        const bool ok = a.status[j] == GS_TRAJ_OK && a.nsteps[j] >= 0 && a.nsteps[j] <= a.smax;
        a.loss[i] = ok ? Lslot : nan;
      }
    }
  }

  // ---------------------------------------------------------------- reverse
  // u holds u_{st+1} at the top of iteration st.
  Blk<T> lam = bzero<T>(), bbar = bzero<T>();
  T dWacc[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int w = 0; w < 4; ++w) dWacc[q][w] = cst<T>(0.0);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    kk[c] = a.nsave - 1;
    next[c] = act[c] && S[c] > 0 ? a.save_idx[(int64_t)kk[c] * n + base + 2 * tx + c] : -1;
  }
  for (int st = Smax - 1; st >= 0; --st) {
    T hh[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      if (st + 1 == next[c]) {
        const int64_t o = (int64_t)kk[c] * n64 + traj[c];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int64_t oo = o + (int64_t)(4 * ty + q) * n;
          if (a.loss_kind == GS_LOSS_SUMSQ)
            lam.v[q][c] = fmaT(cst<T>(2.0), a.target ? u.v[q][c] - a.target[oo] : u.v[q][c], lam.v[q][c]);
          else
            lam.v[q][c] += a.weight[oo];
        }
        --kk[c];
        next[c] = kk[c] >= 0 ? a.save_idx[(int64_t)kk[c] * n + base + 2 * tx + c] : -1;
      }
      const bool run = st < S[c];
      hh[c] = run ? a.h[(int64_t)st * n + base + 2 * tx + c] : cst<T>(0.0);
      if (run) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          u.v[q][c] = a.ck[(int64_t)st * n64 + (int64_t)(4 * ty + q) * n + base + 2 * tx + c];
      }
    }
    // recompute stage states U_j and tanh values y_j (k_j = y_j - U_j)
    Blk<T> U1 = u, U2, U3, U4, U5, U6, y1, y2, y3, y4, y5, y6, kd;
    eval_f(s, U1, bias, y1, kd, ty, tx);
    Blk<T> k1 = kd;
    {
      const T c[1] = {cst<T>(TS_A21)};
      const Blk<T>* const ks[1] = {&k1};
      U2 = stage<T, 1>(c, ks, U1, hh);
    }
    eval_f(s, U2, bias, y2, kd, ty, tx);
    Blk<T> k2 = kd;
    {
      const T c[2] = {cst<T>(TS_A31), cst<T>(TS_A32)};
      const Blk<T>* const ks[2] = {&k1, &k2};
      U3 = stage<T, 2>(c, ks, U1, hh);
    }
    eval_f(s, U3, bias, y3, kd, ty, tx);
    Blk<T> k3 = kd;
    {
      const T c[3] = {cst<T>(TS_A41), cst<T>(TS_A42), cst<T>(TS_A43)};
      const Blk<T>* const ks[3] = {&k1, &k2, &k3};
      U4 = stage<T, 3>(c, ks, U1, hh);
    }
    eval_f(s, U4, bias, y4, kd, ty, tx);
    Blk<T> k4 = kd;
    {
      const T c[4] = {cst<T>(TS_A51), cst<T>(TS_A52), cst<T>(TS_A53), cst<T>(TS_A54)};
      const Blk<T>* const ks[4] = {&k1, &k2, &k3, &k4};
      U5 = stage<T, 4>(c, ks, U1, hh);
    }
    eval_f(s, U5, bias, y5, kd, ty, tx);
    Blk<T> k5 = kd;
    {
      const T c[5] = {cst<T>(TS_A61), cst<T>(TS_A62), cst<T>(TS_A63), cst<T>(TS_A64), cst<T>(TS_A65)};
      const Blk<T>* const ks[5] = {&k1, &k2, &k3, &k4, &k5};
      U6 = stage<T, 5>(c, ks, U1, hh);
    }
    eval_f(s, U6, bias, y6, kd, ty, tx);

    // transposed step, stages 6 .. 1:
    //   nu_j = h (b_j lambda + sum_{m>j} a_mj mu_m), g_j = nu_j (1 - y_j^2),
    //   mu_j = W^T g_j - nu_j, bbar += g_j, dW += g_j U_j^T
    Blk<T> mu[6];
    const Blk<T>* Ys[6] = {&y1, &y2, &y3, &y4, &y5, &y6};
    const Blk<T>* Us[6] = {&U1, &U2, &U3, &U4, &U5, &U6};
    const double bw[6] = {TS_B1, TS_B2, TS_B3, TS_B4, TS_B5, TS_B6};
    const double aw[6][6] = {{0, 0, 0, 0, 0, 0},
                             {TS_A21, 0, 0, 0, 0, 0},
                             {TS_A31, TS_A32, 0, 0, 0, 0},
                             {TS_A41, TS_A42, TS_A43, 0, 0, 0},
                             {TS_A51, TS_A52, TS_A53, TS_A54, 0, 0},
                             {TS_A61, TS_A62, TS_A63, TS_A64, TS_A65, 0}};
#pragma unroll
    for (int jj = 5; jj >= 0; --jj) {
      Blk<T> nu, g;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          T acc = cst<T>(bw[jj]) * lam.v[q][c];
#pragma unroll
          for (int m = 5; m > jj; --m) acc = fmaT(cst<T>(aw[m][jj]), mu[m].v[q][c], acc);
          nu.v[q][c] = hh[c] * acc;
          const T yv = Ys[jj]->v[q][c];
          g.v[q][c] = nu.v[q][c] * fmaT(-yv, yv, cst<T>(1.0));
          bbar.v[q][c] += g.v[q][c];
        }
      __syncthreads();  // previous readers of G / Gt / Ut are done
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int r = 4 * ty + q, t = 2 * tx + c;
          s.G[r][t] = g.v[q][c];
          s.Gt[t][r] = g.v[q][c];
          s.Ut[t][r] = Us[jj]->v[q][c];
        }
      __syncthreads();
      Blk<T> m = matmul_WtG(s, ty, tx);
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < 2; ++c) mu[jj].v[q][c] = m.v[q][c] - nu.v[q][c];
      // dW block (rows 4ty.., columns 4tx..) over the CTA's slots
#pragma unroll 4
      for (int t = 0; t < TB; ++t) {
        T gr[4], uc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          gr[q] = s.Gt[t][4 * ty + q];
          uc[q] = s.Ut[t][4 * tx + q];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int w = 0; w < 4; ++w) dWacc[q][w] = fmaT(gr[q], uc[w], dWacc[q][w]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int c = 0; c < 2; ++c)
        lam.v[q][c] += ((mu[0].v[q][c] + mu[1].v[q][c]) + (mu[2].v[q][c] + mu[3].v[q][c])) +
                       (mu[4].v[q][c] + mu[5].v[q][c]);
  }
  // outputs: dL/db (bias), dL/du0, and this CTA's weight-gradient partial
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    if (!act[c]) {
      if (traj[c] >= 0)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          a.dp[(int64_t)(4 * ty + q) * n + traj[c]] = nan;
          a.du0[(int64_t)(4 * ty + q) * n + traj[c]] = nan;
        }
      continue;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      a.dp[(int64_t)(4 * ty + q) * n + traj[c]] = bbar.v[q][c];
      a.du0[(int64_t)(4 * ty + q) * n + traj[c]] = lam.v[q][c];
    }
  }
  T* part = a.dW_part + (int64_t)blockIdx.x * D * D;
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int w = 0; w < 4; ++w) part[(4 * ty + q) * D + 4 * tx + w] = dWacc[q][w];
}

// dW = sum over CTAs of the partials, in CTA order (deterministic).
template <typename T>
__global__ void k_reduce_dW(const T* part, int nblk, T* dW) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= D * D) return;
  T acc = cst<T>(0.0);
  for (int b = 0; b < nblk; ++b) acc += part[(int64_t)b * D * D + e];
  dW[e] = acc;
}

// ---------------------------------------------------------------------------
// tcgen05 building blocks for the d = 64 products (sm_100a): TF32 rounding and
// the 3xTF32 split (x = hi + lo, both rounded to TF32; A B ~ hi lo + lo hi +
// hi hi keeps fp32 accuracy: measured 5.6e-7 relative against a float64
// product), byte offsets of K-major no-swizzle operand tiles (8-row x 16-byte
// core matrices, row groups 128 B apart, 4-column K chunks one chunk stride
// apart), shared-memory and instruction descriptors, the MMA issue and TMEM
// loads.  TF32 operands cannot be MN-major here, so an operand needed with
// either dimension as K is written twice.  An M = 128 accumulator holds row
// m in TMEM lane m; an M = 64 one holds row m in lane (m / 16) * 32 + m % 16.
// ---------------------------------------------------------------------------
namespace tc {

constexpr int kSpin = 1 << 22;  // mbarrier polls before a CTA gives up

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// byte offset of element (row r, column k) in a tile of R rows
__device__ __forceinline__ uint32_t off(int r, int k, int R) {
  return (uint32_t)(((k >> 2) * (R >> 3) + (r >> 3)) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

__device__ __forceinline__ void put(float* hi, float* lo, uint32_t o, float x) {
  const float h = tf32_rna(x);
  *(float*)((char*)hi + o) = h;
  *(float*)((char*)lo + o) = tf32_rna(x - h);
}

// shared-memory matrix descriptor: start, leading (K chunk) and stride (row
// group) byte offsets, descriptor version 1, no swizzle
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46);
}

// instruction descriptor: fp32 accumulate, tf32 A and B, both K-major
__host__ __device__ constexpr uint32_t idesc(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
      :
      : "r"(d), "l"(a), "l"(b), "r"(id), "r"(acc));
}

// 3xTF32 product over nk K-steps of 8: D (+)= A B^T with A, B K-major tiles of
// chunk strides ca, cb (bytes); acc0 = 0 overwrites D with the first MMA.
__device__ __forceinline__ void mma3(uint32_t d, uint32_t ahi, uint32_t alo, uint32_t ca, uint32_t bhi, uint32_t blo,
                                     uint32_t cb, int nk, uint32_t id, uint32_t acc0) {
  for (int st = 0; st < nk; ++st) {
    const uint32_t oa = 2 * st * ca, ob = 2 * st * cb;
    mma(d, sdesc(ahi + oa, ca, 128), sdesc(blo + ob, cb, 128), id, st > 0 ? 1u : acc0);
    mma(d, sdesc(alo + oa, ca, 128), sdesc(bhi + ob, cb, 128), id, 1u);
    mma(d, sdesc(ahi + oa, ca, 128), sdesc(bhi + ob, cb, 128), id, 1u);
  }
}

__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int c = 0; c < 32; ++c) v[c] = __uint_as_float(r[c]);
}

}  // namespace tc

__device__ __forceinline__ void ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int c = 0; c < 16; ++c) v[c] = __uint_as_float(r[c]);
}

// ---------------------------------------------------------------------------
// Tensor-core replay with 128 trajectories per CTA (k_node64_t128).
//
// One TMEM lane per trajectory: the products are M = 128 MMAs whose
// accumulator row t is trajectory t's vector, so every element-wise step runs
// on the thread that owns the lane, without shuffles or shared-memory round
// trips.  A CTA has NT threads; trajectory t = 32 (w mod 4) + lane is owned by
// warps w, w + 4, ..., which hold its components in groups of HC (warp w + 4g:
// [g HC, (g + 1) HC)).
//   Z   = U W^T      M = 128 (t) x N = 64 (r) x K = 64 (k): A = U (rows t,
//                    K = component), B = W (rows r, K = k)
//   VJP = G W        M = 128 (t) x N = 64 (c) x K = 64 (r): A = G, B = W^T
//   dW += G^T U      M = 64 (c) x N = 64 (e) x K = 128 (t), in two halves of
//                    64 trajectories: A = G^T, B = U^T (rows component,
//                    K = trajectory)
// each as 3xTF32 (hi lo + lo hi + hi hi, hi = tf32(x), lo = tf32(x - hi)).
// TMEM (512 columns): [0, 64) the M = 128 accumulator (Z, then W^T g);
// [64 + 64 (j - 1), 64 + 64 j) stage slot j = 1..6, holding k_j during the
// forward step and the stage recompute and mu_j once the transposed sweep has
// passed stage j; [448, 512) the dW accumulator (M = 64: row c in lane
// 32 (c / 16) + c mod 16).  The slots hold each trajectory's stage slopes, so
// a stage sum reads them back lane by lane.  The arithmetic of the stage
// sums, the transposed step and the outputs is that of k_replay_node64; the
// products round differently (3xTF32 against an fp32 fma chain).
// ---------------------------------------------------------------------------
namespace t128 {

// Threads per CTA: 128 trajectories x NG component groups.  Trajectory t is
// held by warps (t / 32) + 4 g, g = 0..NG-1, each with HC = 64 / NG of its
// components, so every warp reads and writes only its own TMEM lane quarter.
#ifndef GS_N64_NT
#define GS_N64_NT 512
#endif
constexpr int TT = 128;                              // trajectories per CTA
constexpr int NT = GS_N64_NT;                        // threads per CTA
constexpr int NG = NT / TT;                          // component groups per trajectory
constexpr int HC = D / NG;                           // components per thread
constexpr int NQ = HC / 16;                          // 16-column passes per thread
static_assert(NT % TT == 0 && (NG == 2 || NG == 4), "128 trajectories x 2 or 4 component groups");
constexpr uint32_t kChunkT = (TT / 8) * 128;         // K-chunk stride, trajectory-row tile (B)
constexpr uint32_t kChunkW = (D / 8) * 128;          // K-chunk stride, 64-row weight tiles (B)
constexpr uint32_t kChunkC = (D / 8) * 128 + 16;     // K-chunk stride, component-row tiles, padded (B)
constexpr int kTileC = (TT / 2 / 4) * kChunkC / 4;   // floats per component-row tile (64 trajectories)
constexpr uint32_t kColAcc = 0, kColSlot = 64, kColDW = 448;
// Tsit5 weights in float for the transposed sweep (row m: a_{m+1, j+1}; b_j)
__constant__ float kA[6][6] = {{0.f, 0.f, 0.f, 0.f, 0.f, 0.f},
                               {(float)TS_A21, 0.f, 0.f, 0.f, 0.f, 0.f},
                               {(float)TS_A31, (float)TS_A32, 0.f, 0.f, 0.f, 0.f},
                               {(float)TS_A41, (float)TS_A42, (float)TS_A43, 0.f, 0.f, 0.f},
                               {(float)TS_A51, (float)TS_A52, (float)TS_A53, (float)TS_A54, 0.f, 0.f},
                               {(float)TS_A61, (float)TS_A62, (float)TS_A63, (float)TS_A64, (float)TS_A65, 0.f}};
__constant__ float kB[6] = {(float)TS_B1, (float)TS_B2, (float)TS_B3, (float)TS_B4, (float)TS_B5, (float)TS_B6};

struct Smem {
  float Whi[D * D], Wlo[D * D];      // W: rows r, K = k
  float WThi[D * D], WTlo[D * D];    // W^T: rows c, K = r (element (c, r) = W[r][c])
  float Thi[TT * D], Tlo[TT * D];    // A operand of Z and the VJP: rows t, K = component
  float GChi[kTileC], GClo[kTileC];  // G^T of one half: rows c, K = trajectory
  float UEhi[kTileC], UElo[kTileC];  // U^T of one half: rows e, K = trajectory
  float lpart[NG - 1][TT];           // loss partials of component groups 1..NG-1
  unsigned long long bar;            // MMA completion
  uint32_t tmem;                     // TMEM base (512 columns)
  int failed;                        // an MMA wait ran out
  int smax;                          // CTA-wide chain length
};

// byte offset of (row c, trajectory t) in a component-row tile
__device__ __forceinline__ uint32_t offC(int c, int t) {
  return (uint32_t)(t >> 2) * kChunkC + (uint32_t)((c >> 3) * 128 + (c & 7) * 16 + (t & 3) * 4);
}

// Operands written by the CTA's threads become visible to its MMAs; earlier
// TMEM reads are ordered before the MMAs that follow the barrier.
__device__ __forceinline__ void publish() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
}

template <typename SM>
__device__ __forceinline__ void commit(SM& s) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   tc::smem_u32(&s.bar))
               : "memory");
}

// Wait for the next completion of the CTA's mbarrier (bounded; a timeout
// marks the CTA failed, after which no MMA is issued and no wait spins).
template <typename SM>
__device__ __forceinline__ void wait(SM& s, uint32_t& phase) {
  if (!s.failed) {
    uint32_t done = 0;
    for (int it = 0; it < tc::kSpin && !done; ++it)
      asm volatile(
          "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
          "selp.b32 %0, 1, 0, P1;\n\t}\n"
          : "=r"(done)
          : "r"(tc::smem_u32(&s.bar)), "r"(phase)
          : "memory");
    if (!done) s.failed = 1;
  }
  phase ^= 1u;
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Z for the CTA: ACC = T W^T (Z[t][r] = sum_k U[t][k] W[r][k]).
template <typename SM>
__device__ __forceinline__ void product(SM& s, int tid, uint32_t& phase) {
  publish();
  if (tid == 0 && !s.failed) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    tc::mma3(s.tmem + kColAcc, tc::smem_u32(s.Thi), tc::smem_u32(s.Tlo), kChunkT, tc::smem_u32(s.Whi),
             tc::smem_u32(s.Wlo), kChunkW, D / 8, tc::idesc(TT, D), 0u);
    commit(s);
  }
  wait(s, phase);
}

// this thread's HC columns of a TMEM row
template <int N>
__device__ __forceinline__ void load_hc(uint32_t taddr, float (&v)[N]) {
  if constexpr (N == 32) {
    tc::ld32(taddr, v);
  } else {
#pragma unroll
    for (int q = 0; q < N / 16; ++q) {
      float w[16];
      ld16(taddr + 16 * q, w);
#pragma unroll
      for (int c = 0; c < 16; ++c) v[16 * q + c] = w[c];
    }
  }
}

__device__ __forceinline__ void st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      :
      : "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 16 components [k0, k0 + 16) of a trajectory-row operand (hi / lo).
template <typename SM>
__device__ __forceinline__ void put_rows16(SM& s, int t, int k0, const float (&x)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float4 h, l;
    h.x = tc::tf32_rna(x[4 * q]);
    h.y = tc::tf32_rna(x[4 * q + 1]);
    h.z = tc::tf32_rna(x[4 * q + 2]);
    h.w = tc::tf32_rna(x[4 * q + 3]);
    l.x = tc::tf32_rna(x[4 * q] - h.x);
    l.y = tc::tf32_rna(x[4 * q + 1] - h.y);
    l.z = tc::tf32_rna(x[4 * q + 2] - h.z);
    l.w = tc::tf32_rna(x[4 * q + 3] - h.w);
    const uint32_t o = tc::off(t, k0 + 4 * q, TT);
    *(float4*)((char*)s.Thi + o) = h;
    *(float4*)((char*)s.Tlo + o) = l;
  }
}

// Stage J's state U = fma(h, sum_{m<J} a_Jm k_m, u) (the contract's order;
// J = 1: U = u, J = 7: u_{s+1}) into the A operand and, to wait out the
// product, into slot `dst`; k_1 is read from slot s1, k_2..k_6 from slots
// 2..6; 16 columns per pass (a pass reads only its own columns, so dst may
// be s1).  For J = 7, un receives u_{s+1} (un may be u).
template <int J, typename SM>
__device__ __forceinline__ void stage_in(SM& s, uint32_t tl, int t, int c0, float h, const float (&u)[HC],
                                         float (&un)[HC], int s1, int dst) {
  constexpr double A[8][7] = {{0, 0, 0, 0, 0, 0, 0},
                              {0, 0, 0, 0, 0, 0, 0},
                              {TS_A21, 0, 0, 0, 0, 0, 0},
                              {TS_A31, TS_A32, 0, 0, 0, 0, 0},
                              {TS_A41, TS_A42, TS_A43, 0, 0, 0, 0},
                              {TS_A51, TS_A52, TS_A53, TS_A54, 0, 0, 0},
                              {TS_A61, TS_A62, TS_A63, TS_A64, TS_A65, 0, 0},
                              {TS_B1, TS_B2, TS_B3, TS_B4, TS_B5, TS_B6, 0}};
#pragma unroll
  for (int qh = 0; qh < NQ; ++qh) {
    float U[16], v[16];
    if (J == 1) {
#pragma unroll
      for (int c = 0; c < 16; ++c) U[c] = u[16 * qh + c];
    } else {
      ld16(tl + kColSlot + 64 * (s1 - 1) + 16 * qh, v);
#pragma unroll
      for (int c = 0; c < 16; ++c) U[c] = cst<float>(A[J][0]) * v[c];
#pragma unroll
      for (int m = 2; m < J; ++m) {
        ld16(tl + kColSlot + 64 * (m - 1) + 16 * qh, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) U[c] = fmaT(cst<float>(A[J][m - 1]), v[c], U[c]);
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) U[c] = fmaT(h, U[c], u[16 * qh + c]);
    }
    put_rows16(s, t, c0 + 16 * qh, U);
    st16(tl + kColSlot + 64 * (dst - 1) + 16 * qh, U);
    if (J == 7) {
#pragma unroll
      for (int c = 0; c < 16; ++c) un[16 * qh + c] = U[c];
    }
  }
}

// After the product: k = tanh(Z + b) - U, U from the slot, k into the slot.
// gk (may be null): this thread's 32 components of k, component stride n.
__device__ __forceinline__ void stage_out(uint32_t tl, const float (&bias)[HC], int slot, float* gk = nullptr,
                                          int64_t n = 0) {
#pragma unroll
  for (int qh = 0; qh < NQ; ++qh) {
    float z[16], U[16];
    ld16(tl + kColAcc + 16 * qh, z);
    ld16(tl + kColSlot + 64 * (slot - 1) + 16 * qh, U);
#pragma unroll
    for (int c = 0; c < 16; ++c) z[c] = tanh(bias[16 * qh + c] + z[c]) - U[c];
    st16(tl + kColSlot + 64 * (slot - 1) + 16 * qh, z);
    if (gk) {
#pragma unroll
      for (int c = 0; c < 16; ++c) gk[(int64_t)(16 * qh + c) * n] = z[c];
    }
  }
}

// One stage of the replay: k_1 in slot 1, k_7 into slot 1 (FSAL), u <- u_{s+1};
// gk (may be null) receives k_J.
template <int J>
__device__ __forceinline__ void fwd_stage(Smem& s, int tid, int t, int c0, uint32_t& phase, uint32_t tl, float h,
                                          float (&u)[HC], const float (&bias)[HC], float* gk = nullptr,
                                          int64_t n = 0) {
  constexpr int slot = J <= 6 ? J : 1;
  stage_in<J>(s, tl, t, c0, h, u, u, 1, slot);
  product(s, tid, phase);
  stage_out(tl, bias, slot, gk, n);
}

// 16 components of trajectory tk (0..63 within its half) into G^T and U^T.
__device__ __forceinline__ void put_cols16(Smem& s, int tk, int c0, const float (&g)[16], const float (&U)[16]) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t o = offC(c0 + c, tk);
    tc::put(s.GChi, s.GClo, o, g[c]);
    tc::put(s.UEhi, s.UElo, o, U[c]);
  }
}

// nu_j on 16 columns: h (b_j lambda + sum_{m>j} a_mj mu_m), mu_m from slots m > j.
__device__ __forceinline__ void sweep_nu(uint32_t tl, int jj, int qh, float h, const float (&lam)[HC],
                                         float (&nu)[16]) {
  float v[16];
  const float bj = kB[jj];
#pragma unroll
  for (int c = 0; c < 16; ++c) nu[c] = bj * lam[16 * qh + c];
#pragma unroll 1
  for (int m = 5; m > jj; --m) {
    ld16(tl + kColSlot + 64 * m + 16 * qh, v);
    const float am = kA[m][jj];
#pragma unroll
    for (int c = 0; c < 16; ++c) nu[c] = fmaT(am, v[c], nu[c]);
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) nu[c] = h * nu[c];
}

// U_j on 16 columns: fma(h, sum_{m<j} a_jm k_m, u) from slots m < j (u for j = 1).
__device__ __forceinline__ void sweep_U(uint32_t tl, int jj, int qh, float h, const float (&u)[HC], float (&U)[16]) {
  if (jj == 0) {
#pragma unroll
    for (int c = 0; c < 16; ++c) U[c] = u[16 * qh + c];
    return;
  }
  float v[16];
  ld16(tl + kColSlot + 16 * qh, v);
  const float a0 = kA[jj][0];
#pragma unroll
  for (int c = 0; c < 16; ++c) U[c] = a0 * v[c];
#pragma unroll 1
  for (int m = 1; m < jj; ++m) {
    ld16(tl + kColSlot + 64 * m + 16 * qh, v);
    const float am = kA[jj][m];
#pragma unroll
    for (int c = 0; c < 16; ++c) U[c] = fmaT(am, v[c], U[c]);
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) U[c] = fmaT(h, U[c], u[16 * qh + c]);
}

template <bool GRAD>
__global__ void __launch_bounds__(NT, 1) k_node64_t128(GradArgs64<float> a) {
  using T = float;
  extern __shared__ __align__(1024) unsigned char smem_raw_t128[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw_t128);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = 32 * (warp & 3) + lane, hf = warp >> 2, c0 = HC * hf;
  const int64_t n = a.n;
  const int64_t base = (int64_t)blockIdx.x * TT;
  const int64_t n64 = (int64_t)D * n;
  const T nan = cst<T>(__int_as_float(0x7fc00000));
  for (int e = tid; e < D * D; e += NT) {
    const int r = e / D, c = e % D;
    const T w = a.W[e];  // W[r][c]
    tc::put(s.Whi, s.Wlo, tc::off(r, c, D), w);
    tc::put(s.WThi, s.WTlo, tc::off(c, r, D), w);
  }
  if (tid == 0) {
    s.failed = 0;
    s.smax = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc::smem_u32(&s.bar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(tc::smem_u32(&s.tmem)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  uint32_t phase = 0;
  const uint32_t tl = s.tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)c0;  // lane t, this group

  // this thread's slot
  const int64_t j = base + t;
  int64_t traj = -1;
  int S = 0;
  bool act = false;
  if (j < n) {
    const int64_t i = a.order[j];
    if (i >= 0 && i < n) {
      traj = i;
      const int sq = a.nsteps[j];
      if (a.status[j] == GS_TRAJ_OK && sq >= 0 && sq <= a.smax) {
        S = sq;
        act = true;
      }
    }
  }
  atomicMax(&s.smax, S);
  __syncthreads();
  const int Smax = s.smax;

  T u[HC], bias[HC];
#pragma unroll
  for (int c = 0; c < HC; ++c) {
    u[c] = act ? a.u0[(int64_t)(c0 + c) * n + traj] : cst<T>(0.0);
    bias[c] = act ? a.p[(int64_t)(c0 + c) * n + traj] : cst<T>(0.0);
  }
  T Lh = cst<T>(0.0);  // loss terms of this thread's components
  int kk = 0, next = act && S > 0 ? a.save_idx[j] : -1;

  // ---------------------------------------------------------------- forward
  // the stage slopes of step st go to kst[st][j - 1][c][slot] for the reverse sweep
  const int64_t kstep = (int64_t)6 * n64;
  T* const kj = GRAD ? a.kst + (int64_t)c0 * n + j : nullptr;
  auto kdst = [&](int st, int jslot) -> T* {
    return (GRAD && st < S) ? kj + (int64_t)st * kstep + (int64_t)(jslot - 1) * n64 : nullptr;
  };
  fwd_stage<1>(s, tid, t, c0, phase, tl, cst<T>(0.0), u, bias, kdst(0, 1), n);  // k1 = f(u0)
  for (int st = 0; st < Smax; ++st) {
    const T h = st < S ? a.h[(int64_t)st * n + j] : cst<T>(0.0);
    if (GRAD && st < S) {
#pragma unroll
      for (int c = 0; c < HC; ++c) a.ck[(int64_t)st * n64 + (int64_t)(c0 + c) * n + j] = u[c];
    }
    fwd_stage<2>(s, tid, t, c0, phase, tl, h, u, bias, kdst(st, 2), n);
    fwd_stage<3>(s, tid, t, c0, phase, tl, h, u, bias, kdst(st, 3), n);
    fwd_stage<4>(s, tid, t, c0, phase, tl, h, u, bias, kdst(st, 4), n);
    fwd_stage<5>(s, tid, t, c0, phase, tl, h, u, bias, kdst(st, 5), n);
    fwd_stage<6>(s, tid, t, c0, phase, tl, h, u, bias, kdst(st, 6), n);
    // u <- u_{st+1}; k7 -> slot 1 (FSAL) and, as the next step's k_1, to kst
    fwd_stage<7>(s, tid, t, c0, phase, tl, h, u, bias, kdst(st + 1, 1), n);
    if (st + 1 == next) {
      const int64_t o = (int64_t)kk * n64 + traj;
#pragma unroll
      for (int c = 0; c < HC; ++c) {
        const int64_t oo = o + (int64_t)(c0 + c) * n;
        if (!GRAD) {
          a.u_save[oo] = u[c];
        } else if (a.loss_kind == GS_LOSS_SUMSQ) {
          const T d = a.target ? u[c] - a.target[oo] : u[c];
          Lh = fmaT(d, d, Lh);
        } else {
          Lh = fmaT(a.weight[oo], u[c], Lh);
        }
      }
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
  }
  const bool bad0 = s.failed != 0;
  if (!GRAD) {
    if ((!act || bad0) && traj >= 0)
      for (int k = 0; k < a.nsave; ++k)
#pragma unroll
        for (int c = 0; c < HC; ++c) a.u_save[(int64_t)k * n64 + (int64_t)(c0 + c) * n + traj] = nan;
  } else {
    if (hf > 0) s.lpart[hf - 1][t] = Lh;
    __syncthreads();
    if (hf == 0 && traj >= 0) {
      T L = Lh;
#pragma unroll
      for (int g = 0; g < NG - 1; ++g) L += s.lpart[g][t];
      a.loss[traj] = (act && !bad0) ? L : nan;
    }

    // -------------------------------------------------------------- reverse
    // u holds u_{st+1} at the top of iteration st
    T lam[HC], bbar[HC];
#pragma unroll
    for (int c = 0; c < HC; ++c) lam[c] = bbar[c] = cst<T>(0.0);
    uint32_t dw_acc = 0;  // 1 once the dW accumulator holds a product
    kk = a.nsave - 1;
    next = act && S > 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
    for (int st = Smax - 1; st >= 0; --st) {
      if (st + 1 == next) {
        const int64_t o = (int64_t)kk * n64 + traj;
#pragma unroll
        for (int c = 0; c < HC; ++c) {
          const int64_t oo = o + (int64_t)(c0 + c) * n;
          if (a.loss_kind == GS_LOSS_SUMSQ)
            lam[c] = fmaT(cst<T>(2.0), a.target ? u[c] - a.target[oo] : u[c], lam[c]);
          else
            lam[c] += a.weight[oo];
        }
        --kk;
        next = kk >= 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
      }
      const bool run = st < S;
      const T h = run ? a.h[(int64_t)st * n + j] : cst<T>(0.0);
      if (run) {
#pragma unroll
        for (int c = 0; c < HC; ++c) u[c] = a.ck[(int64_t)st * n64 + (int64_t)(c0 + c) * n + j];
      }
      // the stage slopes k_1..k_6 of step st from the forward pass into the
      // slots (zero for a slot past its last step, whose step is 0)
#pragma unroll
      for (int jj = 0; jj < 6; ++jj) {
        const T* src = kj + (int64_t)st * kstep + (int64_t)jj * n64;
#pragma unroll
        for (int qh = 0; qh < NQ; ++qh) {
          T v[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] = run ? src[(int64_t)(16 * qh + c) * n] : cst<T>(0.0);
          st16(tl + kColSlot + 64 * jj + 16 * qh, v);
        }
      }
      // Step st - 1's rows into L2 while step st is transposed: its h, its
      // 64 checkpoint rows and its 6 x 64 slope rows, the CTA's 128
      // trajectories each (512 B, four 128-byte lines).  Every warp of the CTA
      // reaches these loads at the same time, so nothing else would hide
      // their DRAM latency.  Only lines of trajectories below n are touched.
      if (st > 0) {
        const int64_t sp = st - 1;
        for (int row = tid; row < 1 + 64 + 6 * 64; row += NT) {
          const T* r0 = row == 0 ? a.h + sp * n
                                 : (row <= 64 ? a.ck + sp * n64 + (int64_t)(row - 1) * n
                                              : a.kst + sp * kstep + (int64_t)(row - 65) * n);
#pragma unroll
          for (int l = 0; l < TT / 32; ++l)
            if (base + 32 * l < n) asm volatile("prefetch.L2 [%0];" ::"l"(r0 + base + 32 * l));
        }
      }

      // transposed step, stages 6 .. 1:
      //   nu_j = h (b_j lambda + sum_{m>j} a_mj mu_m), g_j = nu_j (1 - y_j^2),
      //   y_j = k_j + U_j, mu_j = W^T g_j - nu_j, bbar += g_j, dW += g_j U_j^T.
      // Element-wise work runs in two passes of 16 columns; slot j takes g_j
      // once k_j is spent, and mu_j after the VJP (nu_j and U_j are recomputed
      // from the slots where they are needed again, which keeps them out of
      // registers across the waits).
#pragma unroll 1
      for (int jj = 5; jj >= 0; --jj) {
#pragma unroll
        for (int qh = 0; qh < NQ; ++qh) {
          T nu[16], Uq[16], v[16];
          sweep_nu(tl, jj, qh, h, lam, nu);
          sweep_U(tl, jj, qh, h, u, Uq);
          ld16(tl + kColSlot + 64 * jj + 16 * qh, v);  // k_j
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const T y = v[c] + Uq[c];
            v[c] = nu[c] * fmaT(-y, y, cst<T>(1.0));  // g_j
            bbar[16 * qh + c] += v[c];
          }
          st16(tl + kColSlot + 64 * jj + 16 * qh, v);
          put_rows16(s, t, c0 + 16 * qh, v);
          if (t < TT / 2) put_cols16(s, t, c0 + 16 * qh, v, Uq);
        }
        publish();
        if (tid == 0 && !s.failed) {
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          tc::mma3(s.tmem + kColAcc, tc::smem_u32(s.Thi), tc::smem_u32(s.Tlo), kChunkT, tc::smem_u32(s.WThi),
                   tc::smem_u32(s.WTlo), kChunkW, D / 8, tc::idesc(TT, D), 0u);
          tc::mma3(s.tmem + kColDW, tc::smem_u32(s.GChi), tc::smem_u32(s.GClo), kChunkC, tc::smem_u32(s.UEhi),
                   tc::smem_u32(s.UElo), kChunkC, TT / 2 / 8, tc::idesc(D, D), dw_acc);
          commit(s);
        }
        dw_acc = 1u;
        wait(s, phase);
        // mu_j = W^T g_j - nu_j into slot j (the VJP completed at this wait)
        auto mu_into_slot = [&]() {
#pragma unroll
          for (int qh = 0; qh < NQ; ++qh) {
            T nu[16], v[16];
            sweep_nu(tl, jj, qh, h, lam, nu);
            ld16(tl + kColAcc + 16 * qh, v);
#pragma unroll
            for (int c = 0; c < 16; ++c) v[c] = v[c] - nu[c];
            st16(tl + kColSlot + 64 * jj + 16 * qh, v);
          }
        };
        // The upper trajectory half writes its dW operands (its g_j from slot
        // j, U_j again) while the lower half forms its mu_j; the upper half's
        // mu_j follows while the upper dW products run.  Each thread touches
        // only its own TMEM lane, so slot j holds g_j for the one half and
        // mu_j for the other at the same time.
        if (t >= TT / 2) {
#pragma unroll
          for (int qh = 0; qh < NQ; ++qh) {
            T g[16], Uq[16];
            ld16(tl + kColSlot + 64 * jj + 16 * qh, g);
            sweep_U(tl, jj, qh, h, u, Uq);
            put_cols16(s, t - TT / 2, c0 + 16 * qh, g, Uq);
          }
        } else {
          mu_into_slot();
        }
        publish();
        if (tid == 0 && !s.failed) {
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          tc::mma3(s.tmem + kColDW, tc::smem_u32(s.GChi), tc::smem_u32(s.GClo), kChunkC, tc::smem_u32(s.UEhi),
                   tc::smem_u32(s.UElo), kChunkC, TT / 2 / 8, tc::idesc(D, D), 1u);
          commit(s);
        }
        if (t >= TT / 2) mu_into_slot();
        wait(s, phase);  // the upper-half dW products have read G^T / U^T
      }
      // lambda += ((mu_1 + mu_2) + (mu_3 + mu_4)) + (mu_5 + mu_6)
#pragma unroll
      for (int qh = 0; qh < NQ; ++qh) {
        T m1[16], m3[16], v[16];
        ld16(tl + kColSlot + 16 * qh, m1);
        ld16(tl + kColSlot + 64 + 16 * qh, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) m1[c] = m1[c] + v[c];
        ld16(tl + kColSlot + 128 + 16 * qh, m3);
        ld16(tl + kColSlot + 192 + 16 * qh, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) m3[c] = m3[c] + v[c];
        ld16(tl + kColSlot + 256 + 16 * qh, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) m1[c] = m1[c] + m3[c], m3[c] = v[c];
        ld16(tl + kColSlot + 320 + 16 * qh, v);
#pragma unroll
        for (int c = 0; c < 16; ++c) lam[16 * qh + c] += m1[c] + (m3[c] + v[c]);
      }
    }
    const bool bad = s.failed != 0;
    if (traj >= 0) {
#pragma unroll
      for (int c = 0; c < HC; ++c) {
        a.dp[(int64_t)(c0 + c) * n + traj] = act && !bad ? bbar[c] : nan;
        a.du0[(int64_t)(c0 + c) * n + traj] = act && !bad ? lam[c] : nan;
      }
    }
    // the CTA's weight-gradient partial: warp w reads rows 16 (w mod 4) .. + 15,
    // columns [32 (w / 4), + 32)
    T* part = a.dW_part + (int64_t)blockIdx.x * D * D;
    T v[HC];
#pragma unroll
    for (int c = 0; c < HC; ++c) v[c] = cst<T>(0.0);
    if (dw_acc && !bad) load_hc(s.tmem + ((uint32_t)(32 * (warp & 3)) << 16) + kColDW + (uint32_t)c0, v);
    if (lane < 16) {
      const int row = 16 * (warp & 3) + lane;
#pragma unroll
      for (int c = 0; c < HC; ++c) part[row * D + c0 + c] = bad ? nan : v[c];
    }
  }
  // no MMA in flight and every TMEM access done before the columns are freed
  if (s.failed && tid == 0) {
    uint32_t done = 0;
    for (int it = 0; it < tc::kSpin && !done; ++it)
      asm volatile(
          "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
          "selp.b32 %0, 1, 0, P1;\n\t}\n"
          : "=r"(done)
          : "r"(tc::smem_u32(&s.bar)), "r"(phase ^ 1u)
          : "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(s.tmem));
  }
}

// ---------------------------------------------------------------------------
// Tensor-core recorder (k_record_node64_t128): the adaptive Tsit5 iteration of
// k_record_node64 in the layout of k_node64_t128 -- 128 trajectories per CTA
// (in trajectory order), one TMEM lane each, the stage products Z = U W^T as
// M = 128 3xTF32 MMAs -- so that the recorded states are bit for bit those of
// the tensor-core replay.  TMEM: the accumulator and seven stage slots (k_1 in
// slot 1, k_j in slot j, k_7 in slot 7; an accepted step copies k_7 into slot
// 1, FSAL).  Each trajectory's controller (starting step, error norm, PI
// control, save points, statuses) runs on its group-0 thread with the
// arithmetic of k_record_node64; the RMS norms keep the contract's sequential
// sum over components 0..63 (the other groups' scaled values pass through
// shared memory).
// ---------------------------------------------------------------------------
struct RecSmem {
  float Whi[D * D], Wlo[D * D];    // W: rows r, K = k
  float Thi[TT * D], Tlo[TT * D];  // stage operand: rows t, K = component
  float red[D - HC][TT];           // scaled values of components HC..63, for the norms
  float hs[TT];                    // the attempt's step per trajectory
  int flag[TT];                    // per trajectory: finite start / accepted
  int sv[TT];                      // save point the accepted step reached, or -1
  unsigned long long bar;          // MMA completion
  uint32_t tmem;                   // TMEM base (512 columns)
  int failed;                      // an MMA wait ran out
};

// RMS of a trajectory's 64 scaled values in the contract's order: acc holds
// the squares of components 0..HC-1 (summed in order by the caller), red the
// values of components HC..63.
__device__ __forceinline__ float rms_finish(const RecSmem& s, int t, float acc) {
  for (int c = 0; c < D - HC; ++c) acc = fmaT(s.red[c][t], s.red[c][t], acc);
  return sqrt(acc / cst<float>(64.0));
}

// Scaled values x_c / sc_c of this thread's components into the norm: group
// 0 accumulates squares in order, the other groups store their values.
__device__ __forceinline__ void norm_part(RecSmem& s, int t, int hf, int c, float r, float& acc) {
  if (hf == 0)
    acc = fmaT(r, r, acc);
  else
    s.red[(hf - 1) * HC + c][t] = r;
}

// One stage of the recorder: state of stage J into the A operand and slot J,
// the product, k_J = tanh(Z + b) - U into slot J (J = 7: un <- u_{s+1}).
template <int J>
__device__ __forceinline__ void rec_stage(RecSmem& s, int tid, int t, int c0, uint32_t& phase, uint32_t tl, float h,
                                          const float (&u)[HC], float (&un)[HC], const float (&bias)[HC]) {
  stage_in<J>(s, tl, t, c0, h, u, un, 1, J);
  product(s, tid, phase);
  stage_out(tl, bias, J);
}

__global__ void __launch_bounds__(NT, 1) k_record_node64_t128(RecArgs64<float> a) {
  using T = float;
  extern __shared__ __align__(1024) unsigned char smem_raw_rec128[];
  RecSmem& s = *reinterpret_cast<RecSmem*>(smem_raw_rec128);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = 32 * (warp & 3) + lane, hf = warp >> 2, c0 = HC * hf;
  const bool ctl = hf == 0;  // the trajectory's controller thread
  const int64_t n = a.n;
  const int64_t it = (int64_t)blockIdx.x * TT + t;
  const bool live = it < n;
  for (int e = tid; e < D * D; e += NT) {
    const int r = e / D, c = e % D;
    tc::put(s.Whi, s.Wlo, tc::off(r, c, D), a.W[e]);
  }
  if (tid == 0) {
    s.failed = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc::smem_u32(&s.bar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(tc::smem_u32(&s.tmem)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  uint32_t phase = 0;
  const uint32_t tl = s.tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)c0;
  const uint32_t slot1 = tl + kColSlot, slot2 = tl + kColSlot + 64, slot7 = tl + kColSlot + 6 * 64;

  T u[HC], bias[HC], un[HC];
#pragma unroll
  for (int c = 0; c < HC; ++c) {
    u[c] = live ? a.u0[(int64_t)(c0 + c) * n + it] : cst<T>(0.0);
    bias[c] = live ? a.p[(int64_t)(c0 + c) * n + it] : cst<T>(0.0);
  }
  const T eps = Eps<T>::v;
  const T qord = cst<T>(5.0);
  Ctl64<T> rec{a.t0, cst<T>(0.0), cst<T>(0.0), 0, 0, 0, live ? GS_TRAJ_OK : GS_TRAJ_MAXSTEPS, false, !live};
  const T ln_floor = ctrl_ln<T>(cst<T>(1e-4));

  // k1 = f(u0) and the starting step (Hairer, Norsett & Wanner I, II.4)
  rec_stage<1>(s, tid, t, c0, phase, tl, cst<T>(0.0), u, un, bias);
  if (ctl) s.flag[t] = 1;
  __syncthreads();
  T acc0 = cst<T>(0.0), acc1 = cst<T>(0.0);
#pragma unroll
  for (int qh = 0; qh < NQ; ++qh) {
    T k[16];
    ld16(slot1 + 16 * qh, k);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int cc = 16 * qh + c;
      if (!isfinite(u[cc]) || !isfinite(k[c])) s.flag[t] = 0;
      norm_part(s, t, hf, cc, u[cc] / fmaT(a.rtol, fabs(u[cc]), a.atol), acc0);
    }
  }
  __syncthreads();
  const T d0 = ctl ? rms_finish(s, t, acc0) : cst<T>(0.0);
  __syncthreads();
#pragma unroll
  for (int qh = 0; qh < NQ; ++qh) {
    T k[16];
    ld16(slot1 + 16 * qh, k);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int cc = 16 * qh + c;
      norm_part(s, t, hf, cc, k[c] / fmaT(a.rtol, fabs(u[cc]), a.atol), acc1);
    }
  }
  __syncthreads();
  T d1 = cst<T>(0.0), h0 = cst<T>(0.0);
  if (ctl) {
    d1 = rms_finish(s, t, acc1);
    h0 = (d0 < cst<T>(1e-5) || d1 < cst<T>(1e-5)) ? cst<T>(1e-6) : cst<T>(0.01) * (d0 / d1);
    h0 = smin_(h0, a.t1 - a.t0);
    s.hs[t] = h0;
  }
  __syncthreads();
  h0 = s.hs[t];
  // f(u0 + h0 f(u0)) into slot 2
#pragma unroll
  for (int qh = 0; qh < NQ; ++qh) {
    T k[16], U[16];
    ld16(slot1 + 16 * qh, k);
#pragma unroll
    for (int c = 0; c < 16; ++c) U[c] = fmaT(h0, k[c], u[16 * qh + c]);
    put_rows16(s, t, c0 + 16 * qh, U);
    st16(slot2 + 16 * qh, U);
  }
  product(s, tid, phase);
  stage_out(tl, bias, 2);
  T acc2 = cst<T>(0.0);
#pragma unroll
  for (int qh = 0; qh < NQ; ++qh) {
    T k[16], kb[16];
    ld16(slot1 + 16 * qh, k);
    ld16(slot2 + 16 * qh, kb);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int cc = 16 * qh + c;
      norm_part(s, t, hf, cc, (kb[c] - k[c]) / fmaT(a.rtol, fabs(u[cc]), a.atol), acc2);
    }
  }
  __syncthreads();
  if (ctl) {
    const T d2 = rms_finish(s, t, acc2) / h0;
    const T dm = smax_(d1, d2);
    const T h1 = dm <= cst<T>(1e-15) ? smax_(cst<T>(1e-6), h0 * cst<T>(1e-3))
                                     : ctrl_pow<T>(cst<T>(0.01) / dm, cst<T>(1.0) / qord);
    rec.hprop = a.h0 > cst<T>(0.0) ? a.h0 : smin_(smin_(cst<T>(100.0) * h0, h1), a.t1 - a.t0);
    if (live && (s.flag[t] == 0 || !(rec.hprop > cst<T>(0.0)) || !isfinite(rec.hprop))) {
      rec.status = GS_TRAJ_NONFINITE;
      rec.done = true;
    }
  }

  for (;;) {
    // --- controller: choose the attempt
    bool clipped = false;
    T tstop = a.t1, tn = rec.tcur;
    if (ctl) {
      if (!rec.done && rec.hprop < cst<T>(16.0) * eps * fabs(rec.tcur)) {
        rec.status = GS_TRAJ_DTMIN;
        rec.done = true;
      }
      T hh = cst<T>(0.0);
      if (!rec.done) {
        tstop = rec.kk < a.nsave ? a.tsave[rec.kk] : a.t1;
        tn = rec.tcur + rec.hprop;
        clipped = tn >= tstop - cst<T>(4.0) * eps * fabs(tstop);
        hh = clipped ? tstop - rec.tcur : rec.hprop;
      }
      s.hs[t] = hh;
    }
    if (!__syncthreads_or(ctl && !rec.done)) break;
    const T hh = s.hs[t];
    rec_stage<2>(s, tid, t, c0, phase, tl, hh, u, un, bias);
    rec_stage<3>(s, tid, t, c0, phase, tl, hh, u, un, bias);
    rec_stage<4>(s, tid, t, c0, phase, tl, hh, u, un, bias);
    rec_stage<5>(s, tid, t, c0, phase, tl, hh, u, un, bias);
    rec_stage<6>(s, tid, t, c0, phase, tl, hh, u, un, bias);
    rec_stage<7>(s, tid, t, c0, phase, tl, hh, u, un, bias);  // un = u_{s+1}, k7 in slot 7
    // scaled error e / sc, e = h sum_j E_j k_j (the contract's order)
    T acc = cst<T>(0.0);
    {
      constexpr double E[7] = {TS_E1, TS_E2, TS_E3, TS_E4, TS_E5, TS_E6, TS_E7};
#pragma unroll
      for (int qh = 0; qh < NQ; ++qh) {
        T e[16], k[16];
        ld16(slot1 + 16 * qh, k);
#pragma unroll
        for (int c = 0; c < 16; ++c) e[c] = cst<T>(E[0]) * k[c];
#pragma unroll
        for (int m = 1; m < 7; ++m) {
          ld16(tl + kColSlot + 64 * m + 16 * qh, k);
#pragma unroll
          for (int c = 0; c < 16; ++c) e[c] = fmaT(cst<T>(E[m]), k[c], e[c]);
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int cc = 16 * qh + c;
          const T sc = fmaT(a.rtol, smax_(fabs(u[cc]), fabs(un[cc])), a.atol);
          norm_part(s, t, hf, cc, (hh * e[c]) / sc, acc);
        }
      }
    }
    __syncthreads();
    // --- controller: accept / reject
    if (ctl) {
      int accept = 0, hit = -1;
      if (!rec.done)
        accept = ctl_decide(rec, a, it, rms_finish(s, t, acc), s.hs[t], clipped, tstop, tn, ln_floor, hit);
      s.flag[t] = accept;
      s.sv[t] = hit;
    }
    __syncthreads();
    // --- the accepted steps: u <- u_{s+1}, k1 <- k7 (every thread rewrites
    // slot 1 with its own choice: the TMEM address is the warp's)
    const bool acc_t = s.flag[t] != 0;
#pragma unroll
    for (int qh = 0; qh < NQ; ++qh) {
      T k1[16], k7[16];
      ld16(slot1 + 16 * qh, k1);
      ld16(slot7 + 16 * qh, k7);
#pragma unroll
      for (int c = 0; c < 16; ++c) k1[c] = acc_t ? k7[c] : k1[c];
      st16(slot1 + 16 * qh, k1);
    }
    if (acc_t) {
#pragma unroll
      for (int c = 0; c < HC; ++c) u[c] = un[c];
      const int k = s.sv[t];
      if (a.u_save && k >= 0) {
#pragma unroll
        for (int c = 0; c < HC; ++c) a.u_save[((int64_t)k * D + c0 + c) * n + it] = u[c];
      }
    }
  }
  // outcome: statuses and counts from the controller threads; a failed
  // trajectory of the solve has NaN at every save point
  if (ctl && s.failed && live) rec.status = GS_TRAJ_NONFINITE;
  if (ctl) s.flag[t] = rec.status;
  __syncthreads();
  if (live && a.u_save && s.flag[t] != GS_TRAJ_OK) {
    const T nan = cst<T>(__int_as_float(0x7fc00000));
    for (int k = 0; k < a.nsave; ++k)
#pragma unroll
      for (int c = 0; c < HC; ++c) a.u_save[((int64_t)k * D + c0 + c) * n + it] = nan;
  }
  if (ctl && live) {
    if (a.store)
      for (int k = rec.kk; k < a.nsave; ++k) a.save_idx[(int64_t)k * n + it] = 0;
    if (a.nsteps) a.nsteps[it] = rec.nst;
    if (a.status) a.status[it] = rec.status;
    if (a.nreject) a.nreject[it] = rec.nrej;
  }
  // no MMA in flight and every TMEM access rec.done before the columns are freed
  if (s.failed && tid == 0) {
    uint32_t done_w = 0;
    for (int itw = 0; itw < tc::kSpin && !done_w; ++itw)
      asm volatile(
          "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
          "selp.b32 %0, 1, 0, P1;\n\t}\n"
          : "=r"(done_w)
          : "r"(tc::smem_u32(&s.bar)), "r"(phase ^ 1u)
          : "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(s.tmem));
  }
}

}  // namespace t128

}  // namespace n64

// Which products the d = 64 recorder, replay and gradient use (process-wide,
// set by gs_set_option): the tcgen05 3xTF32 products with 128 trajectories
// per CTA (default) or the SIMT FP32 products.
static std::atomic<int> g_node64_tensor{1};
void node64_set_tensor(int on) { g_node64_tensor.store(on ? 1 : 0, std::memory_order_relaxed); }

// Gradient workspace: the checkpoints [smax][64][n], one weight-gradient
// partial per CTA (fewer CTAs with tensor cores) and, with the tensor-core
// products, the stage slopes [smax][6][64][n] that the reverse sweep reads
// instead of recomputing them.  The size follows the product option in force.
static size_t align256(size_t b) { return (b + 255) / 256 * 256; }
size_t node64_grad_ws_bytes(int64_t n, int32_t smax, size_t tsize) {
  const int64_t nblk = (n + n64::TB - 1) / n64::TB;
  const size_t ck = align256((size_t)smax * 64 * n * tsize);
  const size_t dw = align256((size_t)nblk * 64 * 64 * tsize);
  const size_t kst = g_node64_tensor.load(std::memory_order_relaxed) != 0 ? (size_t)smax * 6 * 64 * n * tsize : 0;
  return ck + dw + kst;
}

template <typename T>
static n64::GradArgs64<T> grad64_args(const gs_problem* P, const gs_mesh* M) {
  n64::GradArgs64<T> a{};
  a.n = P->n;
  a.p = (const T*)P->p;
  a.u0 = (const T*)P->u0;
  a.W = (const T*)P->shared;
  a.h = (const T*)M->h;
  a.order = M->order;
  a.nsteps = M->nsteps;
  a.save_idx = M->save_idx;
  a.status = M->status;
  a.nsave = P->nsave;
  a.smax = M->smax;
  return a;
}

gs_status node64_grad(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                      void* dshared, void* ws, cudaStream_t st) {
  using T = float;
  n64::GradArgs64<T> a = grad64_args<T>(P, M);
  a.loss_kind = Ls->kind;
  a.target = (const T*)Ls->target;
  a.weight = (const T*)Ls->weight;
  a.loss = (T*)loss;
  a.dp = (T*)dp;
  a.du0 = (T*)du0;
  a.ck = (T*)ws;
  const int nblk = (int)((P->n + n64::TB - 1) / n64::TB);
  const size_t ck_bytes = align256((size_t)M->smax * 64 * P->n * sizeof(T));
  a.dW_part = (T*)((char*)ws + ck_bytes);
  a.kst = (T*)((char*)ws + ck_bytes + align256((size_t)nblk * 64 * 64 * sizeof(T)));
  const bool tensor = g_node64_tensor.load(std::memory_order_relaxed) != 0;
  const int nblk128 = (int)((P->n + n64::t128::TT - 1) / n64::t128::TT);
  if (tensor) {
    const size_t smem = sizeof(n64::t128::Smem);
    if (cudaFuncSetAttribute(n64::t128::k_node64_t128<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return GS_ECUDA;
    n64::t128::k_node64_t128<true><<<nblk128, n64::t128::NT, smem, st>>>(a);
  } else {
    const size_t smem = sizeof(n64::Smem<T>);
    if (cudaFuncSetAttribute(n64::k_replay_node64<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return GS_ECUDA;
    n64::k_replay_node64<T, true><<<nblk, n64::NT, smem, st>>>(a);
  }
  count_launch();
  if (!launch_ok()) return GS_ECUDA;
  if (dshared) {
    n64::k_reduce_dW<T><<<(64 * 64 + 255) / 256, 256, 0, st>>>(a.dW_part, tensor ? nblk128 : nblk,
                                                                (T*)dshared);
    count_launch();
  }
  return launch_ok() ? GS_OK : GS_ECUDA;
}

gs_status node64_solve(const gs_problem* P, const gs_mesh* M, void* u_save, cudaStream_t st) {
  using T = float;
  n64::GradArgs64<T> a = grad64_args<T>(P, M);
  a.u_save = (T*)u_save;
  const int nblk = (int)((P->n + n64::TB - 1) / n64::TB);
  if (g_node64_tensor.load(std::memory_order_relaxed) != 0) {
    const size_t smem = sizeof(n64::t128::Smem);
    if (cudaFuncSetAttribute(n64::t128::k_node64_t128<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return GS_ECUDA;
    n64::t128::k_node64_t128<false><<<(unsigned)((P->n + n64::t128::TT - 1) / n64::t128::TT), n64::t128::NT,
                                       smem, st>>>(a);
  } else {
    const size_t smem = sizeof(n64::Smem<T>);
    if (cudaFuncSetAttribute(n64::k_replay_node64<T, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return GS_ECUDA;
    n64::k_replay_node64<T, false><<<nblk, n64::NT, smem, st>>>(a);
  }
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

// Adaptive record (store = true: into h / save_idx, trajectory order), the
// sizing pass (store = false), or with u_save set the adaptive forward-only
// solve (the state at each save time).
gs_status node64_record_pass(const gs_problem* P, const gs_tol* tol, int32_t smax, bool store, float* h,
                             int32_t* save_idx, int32_t* nsteps, int32_t* status, int32_t* nreject, cudaStream_t st,
                             float* u_save) {
  using T = float;
  n64::RecArgs64<T> a{};
  a.n = P->n;
  a.p = (const T*)P->p;
  a.u0 = (const T*)P->u0;
  a.W = (const T*)P->shared;
  a.t0 = (T)P->t0;
  a.t1 = (T)P->t1;
  a.rtol = (T)tol->rtol;
  a.atol = (T)tol->atol;
  a.h0 = (T)tol->h0;
  a.nsave = P->nsave;
  a.smax = smax;
  for (int k = 0; k < P->nsave; ++k) a.tsave[k] = (T)P->tsave[k];
  a.store = store;
  a.h = h;
  a.save_idx = save_idx;
  a.nsteps = nsteps;
  a.status = status;
  a.nreject = nreject;
  a.u_save = u_save;
  if (g_node64_tensor.load(std::memory_order_relaxed) != 0) {
    // the recorder of the tensor-core replay (the same stage arithmetic)
    const size_t smem = sizeof(n64::t128::RecSmem);
    if (cudaFuncSetAttribute(n64::t128::k_record_node64_t128, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return GS_ECUDA;
    n64::t128::k_record_node64_t128<<<(unsigned)((P->n + n64::t128::TT - 1) / n64::t128::TT), n64::t128::NT, smem,
                                       st>>>(a);
  } else {
    const int nblk = (int)((P->n + n64::TB - 1) / n64::TB);
    const size_t smem = sizeof(n64::Smem<T>);
    if (cudaFuncSetAttribute(n64::k_record_node64<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return GS_ECUDA;
    n64::k_record_node64<T><<<nblk, n64::NT, smem, st>>>(a);
  }
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

}  // namespace gs
