// record.cu -- adaptive recorder (Tsit5 / ROS2 / ROS3 on the d = 3 systems,
// ROS2 / ROS3 on the d = 8 one), the sizing pass and the ordering of mesh
// slots by step count.
//
// GRADSOLVE (arXiv 2609.02876), gptget summary "Methodology" and evolve.pub
// review "Summary": one adaptive solve per trajectory records the accepted
// step sizes into a zero-padded fixed-length mesh.  The pages print no
// controller; the one used here (also written out in the header of the CPU
// reference used by the tests):
//   err = sqrt(mean_c (e_c / (atol + rtol max(|u_c|, |u'_c|)))^2), accept iff
//   err <= 1; PI control with error order q (Tsit5 5, ROS2 2):
//   accept: fac = 0.9 err^(-0.7/q) errprev^(0.4/q) in [0.2, 10] (10 if
//   err == 0), <= 1 right after a rejection, errprev = max(err, 1e-4);
//   reject: fac = max(0.2, 0.9 err^(-1/q)) (0.2 for NaN or inf); the proposal is
//   multiplied by fac either way.  A step whose end would reach the next stop
//   (save time or t1, within 4 eps) is shortened to land on it exactly.
//   Starting step: Hairer, Norsett & Wanner I, II.4.
// Lanes take trajectories in turn from their warp's share (k_record3); every
// loop is bounded by the step capacity.
//
// Order of a record: gs_record runs the adaptive solve once, in trajectory
// order, into workspace copies of the mesh arrays (h trajectory-major, so each
// thread writes its own row front to back and L2 merges the partial sectors);
// a stable counting sort by decreasing step count gives the slot order; a
// gather copies every array into slot order (tiles of 32 slots x 32 steps
// turned in shared memory, so reads and writes are both coalesced) and
// zero-fills the h rows past each slot's last step.  The gradient kernels then find chains of
// nearly equal length in every warp.
#include "kin8.cuh"

namespace gs {

template <typename T>
struct RecArgs {
  int64_t n;
  const T* p;   // [d][n] by trajectory
  const T* u0;  // [d][n] by trajectory
  T t0, t1, rtol, atol, h0;
  int32_t nsave;
  int32_t smax;
  T tsave[GS_MAX_SAVE];
  int64_t chunk;         // trajectories per warp (set by the launcher)
  int32_t dense;         // 1: steps stop only at t1, save times located by theta (Tsit5)
  T* theta;              // mesh mode, dense: [nsave][n] by trajectory
  T* h;                  // mesh mode: step s of trajectory i at h[i * hcol + s * hstep]
  int64_t hcol, hstep;
  int32_t* save_idx;     // mesh mode: [nsave][n] by trajectory
  int32_t* nsteps;       // [n] (may be null in solve mode)
  int32_t* status;       // [n] (may be null in count and solve modes)
  int32_t* nreject;      // [n] (may be null)
  T* u_save;             // solve mode: [nsave][d][n] by trajectory
};

// What a recorder pass writes besides the counts: nothing (the sizing pass),
// the mesh, or the state at each save time (the adaptive forward-only solve).
enum RecMode { kRecCount = 0, kRecMesh = 1, kRecSolve = 2 };

template <typename T, int SYS, int METHOD>
__device__ T initial_step_d(const T* u0, const T* p, T t0, T t1, T rtol, T atol) {
  constexpr int D = SysDim<SYS>::D;
  const T q = cst<T>(method_order(METHOD));
  T sc[D], f0[D], u1[D], f1[D], df[D];
#pragma unroll
  for (int c = 0; c < D; ++c) sc[c] = fmaT(rtol, fabs(u0[c]), atol);
  rhs_s<T, SYS>(u0, p, f0);
  T d0 = rms_d<T, D>(u0, sc);
  T d1 = rms_d<T, D>(f0, sc);
  T h0 = (d0 < cst<T>(1e-5) || d1 < cst<T>(1e-5)) ? cst<T>(1e-6) : cst<T>(0.01) * (d0 / d1);
  h0 = smin_(h0, t1 - t0);
#pragma unroll
  for (int c = 0; c < D; ++c) u1[c] = fmaT(h0, f0[c], u0[c]);
  rhs_s<T, SYS>(u1, p, f1);
#pragma unroll
  for (int c = 0; c < D; ++c) df[c] = f1[c] - f0[c];
  T d2 = rms_d<T, D>(df, sc) / h0;
  T dm = smax_(d1, d2);
  T h1 = dm <= cst<T>(1e-15) ? smax_(cst<T>(1e-6), h0 * cst<T>(1e-3)) : ctrl_pow<T>(cst<T>(0.01) / dm, cst<T>(1.0) / q);
  return smin_(smin_(cst<T>(100.0) * h0, h1), t1 - t0);
}

// One recorder trajectory held by a lane (D components).
template <typename T, int D>
struct Traj {
  int64_t i;  // trajectory index (inputs)
  int64_t o;  // where its outputs go: the trajectory index, or its slot (in-place re-record)
  T u[D], p[D], k1[D];
  T t, hprop, lnprev;
  int nst, nrej, status, kk;
  bool prev_rej;
};

// Load trajectory i and choose its first step; false if it cannot start.
template <typename T, int SYS, int METHOD>
__device__ __forceinline__ bool traj_start(const RecArgs<T>& a, int64_t i, Traj<T, SysDim<SYS>::D>& r) {
  constexpr int D = SysDim<SYS>::D;
  const int64_t n = a.n;
  r.i = i;
  r.o = i;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    r.u[c] = a.u0[c * n + i];
    r.p[c] = a.p[c * n + i];
  }
  r.nst = 0;
  r.nrej = 0;
  r.kk = 0;
  r.status = GS_TRAJ_OK;
  r.prev_rej = false;
  r.t = a.t0;
  r.lnprev = cst<T>(0.0);  // the controller carries ln(errprev); errprev starts at 1
  rhs_s<T, SYS>(r.u, r.p, r.k1);
  bool finite = true;
#pragma unroll
  for (int c = 0; c < D; ++c) finite = finite && isfinite(r.k1[c]) && isfinite(r.u[c]);
  r.hprop = cst<T>(0.0);
  if (finite) {
    r.hprop = a.h0 > cst<T>(0.0) ? a.h0 : initial_step_d<T, SYS, METHOD>(r.u, r.p, a.t0, a.t1, a.rtol, a.atol);
    if (!(r.hprop > cst<T>(0.0)) || !isfinite(r.hprop)) finite = false;
  }
  if (!finite) r.status = GS_TRAJ_NONFINITE;
  return finite;
}

// One attempted step of a running trajectory; true when it has ended (reached
// t1 or failed).
template <typename T, int SYS, int METHOD, int MODE>
__device__ __forceinline__ bool traj_attempt(const RecArgs<T>& a, Traj<T, SysDim<SYS>::D>& r, T ln_floor) {
  constexpr int D = SysDim<SYS>::D;
  const int64_t n = a.n;
  const T eps = Eps<T>::v;
  const T q = cst<T>(method_order(METHOD));
  const T tstop = (r.kk < a.nsave && !a.dense) ? a.tsave[r.kk] : a.t1;
  if (r.hprop < cst<T>(16.0) * eps * fabs(r.t)) {
    r.status = GS_TRAJ_DTMIN;
    return true;
  }
  const T tn = r.t + r.hprop;
  const bool clipped = tn >= tstop - cst<T>(4.0) * eps * fabs(tstop);
  const T h = clipped ? tstop - r.t : r.hprop;
  T un[D], k7[D], e[D];
  if constexpr (METHOD == GS_TSIT5) {
    static_assert(D == 3, "Tsit5 recorder: d = 3 systems");
    tsit5_err_step<T, SYS>(r.u, r.p, h, r.k1, un, k7, e);
  } else if constexpr (METHOD == GS_VERN7) {
    static_assert(D == 3, "Verner 7 recorder: d = 3 systems");
    vern7_step3<T, SYS>(r.u, r.p, h, r.k1, un, e);
  } else {
    bool ok;
    if constexpr (SYS == GS_KIN8)
      ok = METHOD == GS_ROS3 ? kin8_ros3_err_step<T>(r.u, r.p, h, un, e) : kin8_ros2_err_step<T>(r.u, r.p, h, un, e);
    else
      ok = METHOD == GS_ROS3 ? ros3_err_step<T, SYS>(r.u, r.p, h, un, e) : ros2_err_step<T, SYS>(r.u, r.p, h, un, e);
    if (!ok) {
      r.status = GS_TRAJ_SINGULAR;
      return true;
    }
  }
  T sc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) sc[c] = fmaT(a.rtol, smax_(fabs(r.u[c]), fabs(un[c])), a.atol);
  const T err = rms_d<T, D>(e, sc);
  const bool accept = err <= cst<T>(1.0);
  // The controller's power function, once for either outcome (each outcome's
  // own formula, so a lane's arithmetic is that of a branch per outcome, but a
  // warp whose lanes disagree evaluates ln and exp once, not twice):
  //   accept: 0.9 exp(-(0.7/q) ln err + (0.4/q) ln errprev)
  //   reject: 0.9 exp(-(1/q) ln err)
  const bool finite_pos = err > cst<T>(0.0) && isfinite(err);
  const T lnerr = ctrl_ln<T>(finite_pos ? err : cst<T>(1.0));
  const T w = accept ? fmaT(-(cst<T>(0.7) / q), lnerr, (cst<T>(0.4) / q) * r.lnprev) : -(cst<T>(1.0) / q) * lnerr;
  const T pw = cst<T>(0.9) * ctrl_exp<T>(w);
  if (accept) {
    if (r.nst >= a.smax) {
      r.status = GS_TRAJ_MAXSTEPS;
      return true;
    }
    if (MODE == kRecMesh) a.h[r.o * a.hcol + (int64_t)r.nst * a.hstep] = h;
    ++r.nst;
    const T tprev = r.t;
    r.t = clipped ? tstop : tn;
    if (D == 3 && a.dense) {
      // every save time this step passed: its position inside the step, and
      // (solve) the state there -- for Tsit5 its continuous extension over
      // the step's stages (recomputed from u and k1 in a call that is not
      // inlined, so that its registers stay out of every attempt's), for the
      // Rosenbrock methods the Hermite interpolant from u, f(u), u_new,
      // f(u_new)
      while (r.kk < a.nsave && a.tsave[r.kk] <= r.t) {
        const T th = (a.tsave[r.kk] - tprev) / h;
        if (MODE == kRecMesh) {
          a.save_idx[(int64_t)r.kk * n + r.o] = r.nst;
          a.theta[(int64_t)r.kk * n + r.o] = th;
        }
        if constexpr (MODE == kRecSolve) {
          T ut[D];
#pragma unroll
          for (int c = 0; c < D; ++c) ut[c] = un[c];
          if (th != cst<T>(1.0)) {
            if constexpr (METHOD == GS_TSIT5) {
              tsit5_dense3<T, SYS>(r.u, r.p, h, r.k1, th, ut);
            } else {
              const HermiteW<T> w = hermite_w(th);
              T fs[D], fn[D];
              rhs_s<T, SYS>(r.u, r.p, fs);
              rhs_s<T, SYS>(un, r.p, fn);
#pragma unroll
              for (int c = 0; c < D; ++c) ut[c] = hermite_c(w, r.u[c], un[c], fs[c], fn[c], h);
            }
          }
#pragma unroll
          for (int c = 0; c < D; ++c) a.u_save[((int64_t)r.kk * D + c) * n + r.i] = ut[c];
        }
        ++r.kk;
      }
    }
#pragma unroll
    for (int c = 0; c < D; ++c) {
      r.u[c] = un[c];
      if (METHOD == GS_TSIT5) r.k1[c] = k7[c];
    }
    if constexpr (METHOD == GS_VERN7) rhs_s<T, SYS>(r.u, r.p, r.k1);  // not FSAL: the next step's first slope
    while (!a.dense && r.kk < a.nsave && r.t == a.tsave[r.kk]) {
      if (MODE == kRecMesh) a.save_idx[(int64_t)r.kk * n + r.o] = r.nst;
      if (MODE == kRecSolve) {
#pragma unroll
        for (int c = 0; c < D; ++c) a.u_save[((int64_t)r.kk * D + c) * n + r.i] = r.u[c];
      }
      ++r.kk;
    }
    // fac in [0.2, 10], 10 if err == 0, at most 1 right after a rejection
    T fac = err == cst<T>(0.0) ? cst<T>(10.0) : smin_(cst<T>(10.0), smax_(cst<T>(0.2), pw));
    if (r.prev_rej) fac = smin_(fac, cst<T>(1.0));
    r.lnprev = err < cst<T>(1e-4) ? ln_floor : lnerr;
    r.prev_rej = false;
    r.hprop = fac * r.hprop;
    return r.t >= a.t1;
  }
  ++r.nrej;
  if (r.nrej > a.smax) {
    r.status = GS_TRAJ_MAXSTEPS;
    return true;
  }
  // fac >= 0.2, 0.2 for NaN or inf
  const T fac = finite_pos ? smax_(cst<T>(0.2), pw) : cst<T>(0.2);
  r.hprop = fac * r.hprop;
  r.prev_rej = true;
  return false;
}

// Outputs of an ended trajectory.
template <typename T, int MODE, int D>
__device__ __forceinline__ void traj_finish(const RecArgs<T>& a, const Traj<T, D>& r) {
  const int64_t n = a.n;
  if (MODE == kRecMesh) {
    // unreached save points (a failed trajectory); the h tail stays unwritten
    for (int k = r.kk; k < a.nsave; ++k) {
      a.save_idx[(int64_t)k * n + r.o] = 0;
      if (a.dense) a.theta[(int64_t)k * n + r.o] = cst<T>(1.0);
    }
  }
  if (MODE == kRecSolve && r.status != GS_TRAJ_OK) {
    // a failed trajectory has no solution: NaN at every save point
    const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
    for (int k = 0; k < a.nsave; ++k)
#pragma unroll
      for (int c = 0; c < D; ++c) a.u_save[((int64_t)k * D + c) * n + r.i] = nan;
  }
  if (a.nsteps) a.nsteps[r.o] = r.nst;
  if (a.status) a.status[r.o] = r.status;
  if (a.nreject) a.nreject[r.o] = r.nrej;
}

// 6 resident blocks of 128 per SM (85 registers a thread): measured faster on
// B200 than the unconstrained 90-92 registers at 5 blocks, and than 7 or 8
// blocks (more spilling).  The d = 8 system (an 8 x 8 LU per step) takes the
// registers it needs.
#ifndef GS_REC_MINB
#define GS_REC_MINB 6
#endif
template <int SYS> constexpr int rec_minb() { return SYS == GS_KIN8 ? 1 : GS_REC_MINB; }

// Each warp owns the trajectories [w * chunk, (w + 1) * chunk) and its lanes
// take them in turn: a lane whose trajectory has ended takes the next one of
// the chunk (handed out with a ballot), so lanes do not idle while the
// longest trajectory of the warp finishes.  The launch gives one resident
// wave of warps, each with an equal share.  A trajectory's arithmetic does
// not depend on which lane runs it or when.  The loop ends: every pass either
// hands out chunk entries or advances some trajectory's accepted or rejected
// step count, and both are capped by smax.
template <typename T, int SYS, int METHOD, int MODE>
__global__ void __launch_bounds__(128, rec_minb<SYS>()) k_record3(RecArgs<T> a) {
  const unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t c0 = w * a.chunk;
  const int64_t c1 = c0 + a.chunk < a.n ? c0 + a.chunk : a.n;
  if (c0 >= c1) return;  // whole warp
  int64_t next = c0;
  const T ln_floor = ctrl_ln<T>(cst<T>(1e-4));  // errprev is floored at 1e-4
  Traj<T, SysDim<SYS>::D> r;
  bool run = false;
  for (;;) {
    const unsigned need = __ballot_sync(kFull, !run);
    if (need) {
      const int64_t cand = next + __popc(need & lt);
      if (!run && cand < c1) {
        run = traj_start<T, SYS, METHOD>(a, cand, r);
        if (!run) traj_finish<T, MODE>(a, r);
      }
      next += __popc(need);
    }
    if (!__any_sync(kFull, run) && next >= c1) break;
    if (run && traj_attempt<T, SYS, METHOD, MODE>(a, r, ln_floor)) {
      traj_finish<T, MODE>(a, r);
      run = false;
    }
  }
}

// In-place re-record: the slots keep the order an earlier record gave them
// (slot j runs trajectory order[j]) and every output goes straight to its
// slot (h step-major at s * n + j).  Slots are handed out in groups of 32, one
// group per warp at a time from a global counter, in slot order: an earlier
// record sorted them by decreasing step count, so the 32 lanes of a group run
// chains of about equal length side by side, and the longest groups go first.
// A lane whose chain ends waits for its group (the chains differ only by
// their rejections when the ensemble is unchanged).  Rows from the new count
// up to the slot's previous count are zeroed, so the mesh stays zero padded.
// An order entry outside [0, n) leaves its slot with GS_TRAJ_BADORDER, no
// steps, and its rows zeroed up to the previous count.  The loop ends: every
// pass takes a group from a counter that only grows, and a group's inner loop
// advances some chain's accepted or rejected count, both capped by smax.
// MODE kRecSolve runs the adaptive forward-only solve in the same grouped
// order with its outputs by trajectory (an entry outside [0, n) is skipped).
template <typename T, int SYS, int METHOD, int MODE>
__global__ void __launch_bounds__(128, rec_minb<SYS>()) k_record3_inplace(RecArgs<T> a, const int32_t* order,
                                                                         unsigned long long* next_group) {
  static_assert(MODE == kRecMesh || MODE == kRecSolve, "grouped passes: mesh or solve");
  const unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int64_t n = a.n;
  const unsigned long long ngroups = (unsigned long long)((n + 31) / 32);
  const T ln_floor = ctrl_ln<T>(cst<T>(1e-4));
  Traj<T, SysDim<SYS>::D> r;
  for (;;) {
    unsigned long long g = 0;
    if (lane == 0) g = atomicAdd(next_group, 1ull);
    g = __shfl_sync(kFull, g, 0);
    if (g >= ngroups) break;  // whole warp
    const int64_t j = (int64_t)g * 32 + lane;
    bool run = false;
    int old = 0;
    if (j < n) {
      if (MODE == kRecMesh) {
        old = a.nsteps[j];
        old = old < 0 ? 0 : (old > a.smax ? a.smax : old);
      }
      const int32_t i = order[j];
      if (i >= 0 && i < n) {
        run = traj_start<T, SYS, METHOD>(a, i, r);
        if (MODE == kRecMesh) r.o = j;
        if (!run) traj_finish<T, MODE>(a, r);
      } else if (MODE == kRecMesh) {
        r.o = j;
        r.nst = r.nrej = r.kk = 0;
        r.status = GS_TRAJ_BADORDER;
        traj_finish<T, kRecMesh>(a, r);
      }
    }
    while (__any_sync(kFull, run)) {
      if (run && traj_attempt<T, SYS, METHOD, MODE>(a, r, ln_floor)) {
        traj_finish<T, MODE>(a, r);
        run = false;
      }
    }
    if (MODE == kRecMesh && j < n)
      for (int s = r.nst < 0 ? 0 : r.nst; s < old; ++s) a.h[j * a.hcol + (int64_t)s * a.hstep] = cst<T>(0.0);
  }
}

// ---------------------------------------------------------------------------
// Slot order: stable counting sort of trajectories by decreasing step count.
// Keys are bucketed into nb bins; chunk c of kChunk trajectories contributes
// hist[b][c].  An exclusive scan over (bin, chunk) gives every chunk's first
// position per bin, and one warp per chunk scatters its trajectories in index
// order (warp match + prefix popcount), so the result is deterministic.
// ---------------------------------------------------------------------------
constexpr int kChunk = 2048;

__device__ __forceinline__ int sort_bin(int cnt, int smax) {
  // descending count: bin 0 holds the longest chains
  int c = cnt < 0 ? 0 : (cnt > smax ? smax : cnt);
  return smax - c;
}

__global__ void k_hist(const int32_t* cnt, int64_t n, int smax, int nchunk, int32_t* hist) {
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int b = sort_bin(cnt[i], smax);
  atomicAdd(&hist[(int64_t)b * nchunk + (i / kChunk)], 1);
}

// Exclusive scan of hist (len entries) by one block of 1024 threads.
__global__ void k_scan(int32_t* hist, int64_t len) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  const int64_t per = (len + 1023) / 1024;
  const int64_t a0 = tid * per, a1 = a0 + per < len ? a0 + per : len;
  int64_t s = 0;
  for (int64_t q = a0; q < a1; ++q) s += hist[q];
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    int64_t v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int64_t run = part[tid] - s;
  for (int64_t q = a0; q < a1; ++q) {
    int64_t v = hist[q];
    hist[q] = (int32_t)run;
    run += v;
  }
}

__global__ void k_scatter(const int32_t* cnt, int64_t n, int smax, int nchunk, int32_t* hist, int32_t* order) {
  const int c = blockIdx.x;
  const int lane = threadIdx.x;
  const int64_t base = (int64_t)c * kChunk;
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kChunk; r += 32) {
    const int64_t i = base + r + lane;
    const bool act = i < n;
    const unsigned mask = __ballot_sync(0xffffffffu, act);
    if (!mask) break;
    const int b = act ? sort_bin(cnt[i], smax) : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, b);
    int32_t pos = 0;
    if (act) pos = hist[(int64_t)b * nchunk + c] + __popc(peers & lt);
    __syncwarp();
    if (act) {
      order[pos] = (int32_t)i;
      if ((peers & lt) == 0) hist[(int64_t)b * nchunk + c] += __popc(peers);
    }
    __syncwarp();
  }
}

template <typename T>
static RecArgs<T> rec_args(const gs_problem* P, const gs_tol* tol, int32_t smax) {
  RecArgs<T> a{};
  a.n = P->n;
  a.p = (const T*)P->p;
  a.u0 = (const T*)P->u0;
  a.t0 = (T)P->t0;
  a.t1 = (T)P->t1;
  a.rtol = (T)tol->rtol;
  a.atol = (T)tol->atol;
  a.h0 = (T)tol->h0;
  a.nsave = P->nsave;
  a.smax = smax;
  a.dense = tol->dense;
  for (int k = 0; k < P->nsave; ++k) a.tsave[k] = (T)P->tsave[k];
  return a;
}

#ifndef GS_REC_WAVES
#define GS_REC_WAVES 1
#endif

template <typename T, int SYS, int METHOD, int MODE>
static gs_status launch_rec(RecArgs<T> a, cudaStream_t st) {
  // one resident wave of warps, each with an equal share of the trajectories
  const int bs = 128;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_record3<T, SYS, METHOD, MODE>, bs, 0) != cudaSuccess)
    return GS_ECUDA;
  const int64_t warps = (int64_t)(per_sm > 0 ? per_sm : 1) * sms * (bs / 32) * GS_REC_WAVES;
  a.chunk = (a.n + warps - 1) / warps;
  if (a.chunk < 32) a.chunk = 32;
  const int64_t nwarps = (a.n + a.chunk - 1) / a.chunk;
  const int64_t grid = (nwarps * 32 + bs - 1) / bs;
  k_record3<T, SYS, METHOD, MODE><<<(unsigned)grid, bs, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template <typename T, int SYS, int METHOD, int MODE>
static gs_status launch_rec_inplace(RecArgs<T> a, const int32_t* order, unsigned long long* ctr, cudaStream_t st) {
  // one resident wave; the warps take groups of 32 slots until none is left
  const int bs = 128;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_record3_inplace<T, SYS, METHOD, MODE>, bs, 0) !=
          cudaSuccess)
    return GS_ECUDA;
  const int64_t groups = (a.n + 31) / 32;
  int64_t grid = (int64_t)(per_sm > 0 ? per_sm : 1) * sms;
  if (grid * (bs / 32) > groups) grid = (groups + bs / 32 - 1) / (bs / 32);
  if (cudaMemsetAsync(ctr, 0, sizeof(unsigned long long), st) != cudaSuccess) return GS_ECUDA;
  k_record3_inplace<T, SYS, METHOD, MODE><<<(unsigned)grid, bs, 0, st>>>(a, order, ctr);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template <typename T, int MODE>
static gs_status dispatch_rec_inplace(int sys, int method, const RecArgs<T>& a, const int32_t* order,
                                      unsigned long long* ctr, cudaStream_t st) {
  if (sys == GS_LORENZ && method == GS_TSIT5)
    return launch_rec_inplace<T, kSysLorenz, GS_TSIT5, MODE>(a, order, ctr, st);
  if (sys == GS_LORENZ && method == GS_ROS2) return launch_rec_inplace<T, kSysLorenz, GS_ROS2, MODE>(a, order, ctr, st);
  if (sys == GS_ROBERTSON && method == GS_TSIT5)
    return launch_rec_inplace<T, kSysRobertson, GS_TSIT5, MODE>(a, order, ctr, st);
  if (sys == GS_ROBERTSON && method == GS_ROS2)
    return launch_rec_inplace<T, kSysRobertson, GS_ROS2, MODE>(a, order, ctr, st);
  if (sys == GS_LORENZ && method == GS_ROS3) return launch_rec_inplace<T, kSysLorenz, GS_ROS3, MODE>(a, order, ctr, st);
  if (sys == GS_ROBERTSON && method == GS_ROS3)
    return launch_rec_inplace<T, kSysRobertson, GS_ROS3, MODE>(a, order, ctr, st);
  if (sys == GS_KIN8 && method == GS_ROS2) return launch_rec_inplace<T, kSysKin8, GS_ROS2, MODE>(a, order, ctr, st);
  if (sys == GS_KIN8 && method == GS_ROS3) return launch_rec_inplace<T, kSysKin8, GS_ROS3, MODE>(a, order, ctr, st);
  if (sys == GS_LORENZ && method == GS_VERN7)
    return launch_rec_inplace<T, kSysLorenz, GS_VERN7, MODE>(a, order, ctr, st);
  if (sys == GS_ROBERTSON && method == GS_VERN7)
    return launch_rec_inplace<T, kSysRobertson, GS_VERN7, MODE>(a, order, ctr, st);
  return GS_EUNSUPPORTED;
}

template <typename T, int MODE>
static gs_status dispatch_rec(int sys, int method, const RecArgs<T>& a, cudaStream_t st) {
  if (sys == GS_LORENZ && method == GS_TSIT5) return launch_rec<T, kSysLorenz, GS_TSIT5, MODE>(a, st);
  if (sys == GS_LORENZ && method == GS_ROS2) return launch_rec<T, kSysLorenz, GS_ROS2, MODE>(a, st);
  if (sys == GS_ROBERTSON && method == GS_TSIT5) return launch_rec<T, kSysRobertson, GS_TSIT5, MODE>(a, st);
  if (sys == GS_ROBERTSON && method == GS_ROS2) return launch_rec<T, kSysRobertson, GS_ROS2, MODE>(a, st);
  if (sys == GS_LORENZ && method == GS_ROS3) return launch_rec<T, kSysLorenz, GS_ROS3, MODE>(a, st);
  if (sys == GS_ROBERTSON && method == GS_ROS3) return launch_rec<T, kSysRobertson, GS_ROS3, MODE>(a, st);
  if (sys == GS_KIN8 && method == GS_ROS2) return launch_rec<T, kSysKin8, GS_ROS2, MODE>(a, st);
  if (sys == GS_KIN8 && method == GS_ROS3) return launch_rec<T, kSysKin8, GS_ROS3, MODE>(a, st);
  if (sys == GS_LORENZ && method == GS_VERN7) return launch_rec<T, kSysLorenz, GS_VERN7, MODE>(a, st);
  if (sys == GS_ROBERTSON && method == GS_VERN7) return launch_rec<T, kSysRobertson, GS_VERN7, MODE>(a, st);
  return GS_EUNSUPPORTED;
}

gs_status count3(const gs_problem* P, const gs_tol* tol, int32_t smax, int32_t* nsteps, int32_t* status,
                 cudaStream_t st) {
  if (P->dtype == GS_F64) {
    RecArgs<double> a = rec_args<double>(P, tol, smax);
    a.nsteps = nsteps;
    a.status = status;
    return dispatch_rec<double, kRecCount>(P->system, P->method, a, st);
  }
  RecArgs<float> a = rec_args<float>(P, tol, smax);
  a.nsteps = nsteps;
  a.status = status;
  return dispatch_rec<float, kRecCount>(P->system, P->method, a, st);
}

// Adaptive forward-only solve: one recorder pass in trajectory order writing
// the state at every save time (no mesh, no workspace).
gs_status solve_adaptive3(const gs_problem* P, const gs_tol* tol, int32_t smax, void* u_save, int32_t* nsteps,
                          int32_t* status, cudaStream_t st) {
  if (P->dtype == GS_F64) {
    RecArgs<double> a = rec_args<double>(P, tol, smax);
    a.nsteps = nsteps;
    a.status = status;
    a.u_save = (double*)u_save;
    return dispatch_rec<double, kRecSolve>(P->system, P->method, a, st);
  }
  RecArgs<float> a = rec_args<float>(P, tol, smax);
  a.nsteps = nsteps;
  a.status = status;
  a.u_save = (float*)u_save;
  return dispatch_rec<float, kRecSolve>(P->system, P->method, a, st);
}

// The adaptive forward-only solve in a given trajectory order (groups of 32
// consecutive entries side by side, outputs by trajectory); ws holds the
// group counter.
gs_status solve_adaptive3_ordered(const gs_problem* P, const gs_tol* tol, int32_t smax, const int32_t* order,
                                  void* u_save, int32_t* nsteps, int32_t* status, void* ws, cudaStream_t st) {
  if (P->dtype == GS_F64) {
    RecArgs<double> a = rec_args<double>(P, tol, smax);
    a.nsteps = nsteps;
    a.status = status;
    a.u_save = (double*)u_save;
    return dispatch_rec_inplace<double, kRecSolve>(P->system, P->method, a, order, (unsigned long long*)ws, st);
  }
  RecArgs<float> a = rec_args<float>(P, tol, smax);
  a.nsteps = nsteps;
  a.status = status;
  a.u_save = (float*)u_save;
  return dispatch_rec_inplace<float, kRecSolve>(P->system, P->method, a, order, (unsigned long long*)ws, st);
}

static size_t al256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace of gs_record: trajectory-order copies of nsteps, status, nreject,
// save_idx, h and (dense records) the save-point positions, then the sort
// histogram.
size_t record_ws_bytes(int64_t n, int32_t smax, int32_t nsave, size_t tsize) {
  const int64_t nchunk = (n + kChunk - 1) / kChunk;
  return 3 * al256((size_t)n * 4) + al256((size_t)nsave * n * 4) + al256((size_t)smax * n * tsize) +
         al256((size_t)nsave * n * tsize) + (size_t)(smax + 1) * (size_t)nchunk * 4;
}

// Gather into slot order.  A block owns 32 slots and walks their steps in
// tiles of 32: each warp reads whole 32-step pieces of the trajectory-major
// rows (256 contiguous bytes per row in fp64), the tile turns in shared
// memory, and each warp writes 32 consecutive slots of one step.  Steps past
// a slot's count are written as zeros (the mesh is zero padded); rows of
// inactive slots (past n) are neither read nor written.
constexpr int kGatherWarps = 8;

template <typename T>
__global__ void __launch_bounds__(32 * kGatherWarps) k_gather_mesh(
    int64_t n, int smax, int nsave, const int32_t* __restrict__ order, const T* __restrict__ h_tmp,
    const int32_t* __restrict__ si_tmp, const int32_t* __restrict__ ns_tmp, const int32_t* __restrict__ st_tmp,
    const int32_t* __restrict__ nr_tmp, const T* __restrict__ th_tmp, T* h, int32_t* save_idx, int32_t* nsteps,
    int32_t* status, int32_t* nreject, T* theta) {
  __shared__ T tile[32][33];
  __shared__ int64_t row[32];
  __shared__ int cnt[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t j0 = (int64_t)blockIdx.x * 32;
  if (warp == 0) {
    const int64_t j = j0 + lane;
    int S = 0;
    int64_t i = -1;
    if (j < n) {
      i = order[j];
      S = ns_tmp[i];
      nsteps[j] = S;
      status[j] = st_tmp[i];
      nreject[j] = nr_tmp[i];
      for (int k = 0; k < nsave; ++k) save_idx[(int64_t)k * n + j] = si_tmp[(int64_t)k * n + i];
      if (theta)
        for (int k = 0; k < nsave; ++k) theta[(int64_t)k * n + j] = th_tmp[(int64_t)k * n + i];
    }
    row[lane] = i;
    cnt[lane] = S < 0 ? 0 : (S > smax ? smax : S);
  }
  __syncthreads();
  for (int s0 = 0; s0 < smax; s0 += 32) {
    // read: warp w takes slots w, w + 8, ...; lane = step within the tile
    for (int r = warp; r < 32; r += kGatherWarps) {
      const int s = s0 + lane;
      T v = cst<T>(0.0);
      if (row[r] >= 0 && s < cnt[r]) v = h_tmp[row[r] * smax + s];
      tile[r][lane] = v;
    }
    __syncthreads();
    // write: warp w takes steps w, w + 8, ...; lane = slot
    const int64_t j = j0 + lane;
    for (int c = warp; c < 32; c += kGatherWarps) {
      const int s = s0 + c;
      if (s < smax && j < n) h[(int64_t)s * n + j] = tile[lane][c];
    }
    __syncthreads();
  }
}

gs_status order_slots(const int32_t* cnt, int64_t n, int32_t smax, int32_t* hist, int32_t* order, cudaStream_t st) {
  const int nchunk = (int)((n + kChunk - 1) / kChunk);
  const int64_t len = (int64_t)(smax + 1) * nchunk;
  if (cudaMemsetAsync(hist, 0, (size_t)len * 4, st) != cudaSuccess) return GS_ECUDA;
  k_hist<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(cnt, n, smax, nchunk, hist);
  k_scan<<<1, 1024, 0, st>>>(hist, len);
  k_scatter<<<nchunk, 32, 0, st>>>(cnt, n, smax, nchunk, hist, order);
  count_launch(3);
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template <typename T>
static gs_status record3_t(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws, cudaStream_t st) {
  const int64_t n = P->n;
  char* w = (char*)ws;
  int32_t* ns_tmp = (int32_t*)w;
  w += al256((size_t)n * 4);
  int32_t* st_tmp = (int32_t*)w;
  w += al256((size_t)n * 4);
  int32_t* nr_tmp = (int32_t*)w;
  w += al256((size_t)n * 4);
  int32_t* si_tmp = (int32_t*)w;
  w += al256((size_t)P->nsave * n * 4);
  T* h_tmp = (T*)w;
  w += al256((size_t)M->smax * n * sizeof(T));
  T* th_tmp = (T*)w;
  w += al256((size_t)P->nsave * n * sizeof(T));
  int32_t* hist = (int32_t*)w;
  RecArgs<T> a = rec_args<T>(P, tol, M->smax);
  a.theta = th_tmp;
  a.h = h_tmp;
  a.hcol = M->smax;  // trajectory-major workspace copy: each thread writes its own row
  a.hstep = 1;
  a.save_idx = si_tmp;
  a.nsteps = ns_tmp;
  a.status = st_tmp;
  a.nreject = nr_tmp;
  gs_status rc = dispatch_rec<T, kRecMesh>(P->system, P->method, a, st);
  if (rc != GS_OK) return rc;
  rc = order_slots(ns_tmp, n, M->smax, hist, M->order, st);
  if (rc != GS_OK) return rc;
  k_gather_mesh<T><<<(unsigned)((n + 31) / 32), 32 * kGatherWarps, 0, st>>>(
      n, M->smax, P->nsave, M->order, h_tmp, si_tmp, ns_tmp, st_tmp, nr_tmp, th_tmp, (T*)M->h, M->save_idx,
      M->nsteps, M->status, M->nreject, tol->dense ? (T*)M->save_theta : nullptr);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

gs_status record3(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws, cudaStream_t st) {
  return P->dtype == GS_F64 ? record3_t<double>(P, tol, M, ws, st) : record3_t<float>(P, tol, M, ws, st);
}

// In-place re-record into the caller's mesh, in its slot order (no workspace
// copy, no sort, no gather); ws holds the group counter.
template <typename T>
static gs_status record3_inplace_t(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws,
                                   cudaStream_t st) {
  RecArgs<T> a = rec_args<T>(P, tol, M->smax);
  a.theta = tol->dense ? (T*)M->save_theta : nullptr;
  a.h = (T*)M->h;
  a.hcol = 1;  // step-major: step s of slot j at s * n + j
  a.hstep = P->n;
  a.save_idx = M->save_idx;
  a.nsteps = M->nsteps;
  a.status = M->status;
  a.nreject = M->nreject;
  return dispatch_rec_inplace<T, kRecMesh>(P->system, P->method, a, M->order, (unsigned long long*)ws, st);
}

gs_status record3_inplace(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws, cudaStream_t st) {
  return P->dtype == GS_F64 ? record3_inplace_t<double>(P, tol, M, ws, st)
                            : record3_inplace_t<float>(P, tol, M, ws, st);
}

gs_status node64_record_pass(const gs_problem*, const gs_tol*, int32_t, bool, float*, int32_t*, int32_t*, int32_t*,
                             int32_t*, cudaStream_t, float*);

// The d = 64 record: the same trajectory-order pass / sort / gather sequence,
// with the CTA-per-32-trajectories recorder of node64.cu.
gs_status record_node64(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws, cudaStream_t st) {
  using T = float;
  const int64_t n = P->n;
  char* w = (char*)ws;
  int32_t* ns_tmp = (int32_t*)w;
  w += al256((size_t)n * 4);
  int32_t* st_tmp = (int32_t*)w;
  w += al256((size_t)n * 4);
  int32_t* nr_tmp = (int32_t*)w;
  w += al256((size_t)n * 4);
  int32_t* si_tmp = (int32_t*)w;
  w += al256((size_t)P->nsave * n * 4);
  T* h_tmp = (T*)w;
  w += al256((size_t)M->smax * n * sizeof(T));
  int32_t* hist = (int32_t*)w;
  gs_status rc = node64_record_pass(P, tol, M->smax, true, h_tmp, si_tmp, ns_tmp, st_tmp, nr_tmp, st, nullptr);
  if (rc != GS_OK) return rc;
  rc = order_slots(ns_tmp, n, M->smax, hist, M->order, st);
  if (rc != GS_OK) return rc;
  k_gather_mesh<T><<<(unsigned)((n + 31) / 32), 32 * kGatherWarps, 0, st>>>(n, M->smax, P->nsave, M->order, h_tmp, si_tmp, ns_tmp,
                                                                 st_tmp, nr_tmp, nullptr, (T*)M->h, M->save_idx,
                                                                 M->nsteps, M->status, M->nreject, nullptr);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

}  // namespace gs
