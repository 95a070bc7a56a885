// record.cu -- adaptive recorder (Tsit5 / ROS2, d = 3 systems), the sizing
// pass and the ordering of mesh slots by step count.
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
// One thread per trajectory; every loop is bounded by the step capacity.
//
// Order of a record: gs_record runs the adaptive solve once, in trajectory
// order, into workspace copies of the mesh arrays (h trajectory-major, so each
// thread writes its own row front to back and L2 merges the partial sectors);
// a stable counting sort by decreasing step count gives the slot order; a
// gather copies every array into slot order (each thread reads one source row
// in order, writes coalesced) and zero-fills the h rows past each slot's last
// step.  The gradient kernels then find chains of
// nearly equal length in every warp.
#include "steps.cuh"

namespace gs {

template <typename T>
struct RecArgs {
  int64_t n;
  const T* p;   // [3][n] by trajectory
  const T* u0;  // [3][n] by trajectory
  T t0, t1, rtol, atol, h0;
  int32_t nsave;
  int32_t smax;
  T tsave[GS_MAX_SAVE];
  const int32_t* order;  // slot -> trajectory (null: identity)
  T* h;                  // step sizes (null: count only); step s of slot j at
  int64_t hcol, hstep;   // h[j * hcol + s * hstep]
  int32_t* save_idx;     // [nsave][n] by slot
  int32_t* nsteps;       // [n]
  int32_t* status;       // [n] (may be null in count mode)
  int32_t* nreject;      // [n] (may be null)
};

template <typename T, int SYS, int METHOD>
__device__ T initial_step3(const T u0[3], const T p[3], T t0, T t1, T rtol, T atol) {
  const T q = METHOD == GS_TSIT5 ? cst<T>(5.0) : cst<T>(2.0);
  T sc[3], f0[3], u1[3], f1[3], df[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) sc[c] = fmaT(rtol, fabs(u0[c]), atol);
  rhs3<T, SYS>(u0, p, f0);
  T d0 = rms3(u0, sc);
  T d1 = rms3(f0, sc);
  T h0 = (d0 < cst<T>(1e-5) || d1 < cst<T>(1e-5)) ? cst<T>(1e-6) : cst<T>(0.01) * (d0 / d1);
  h0 = smin_(h0, t1 - t0);
#pragma unroll
  for (int c = 0; c < 3; ++c) u1[c] = fmaT(h0, f0[c], u0[c]);
  rhs3<T, SYS>(u1, p, f1);
#pragma unroll
  for (int c = 0; c < 3; ++c) df[c] = f1[c] - f0[c];
  T d2 = rms3(df, sc) / h0;
  T dm = smax_(d1, d2);
  T h1 = dm <= cst<T>(1e-15) ? smax_(cst<T>(1e-6), h0 * cst<T>(1e-3)) : ctrl_pow<T>(cst<T>(0.01) / dm, cst<T>(1.0) / q);
  return smin_(smin_(cst<T>(100.0) * h0, h1), t1 - t0);
}

template <typename T, int SYS, int METHOD, bool STORE>
__global__ void __launch_bounds__(128) k_record3(RecArgs<T> a) {
  const int64_t n = a.n;
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t i = a.order ? (int64_t)a.order[j] : j;
  const T eps = Eps<T>::v;
  const T q = METHOD == GS_TSIT5 ? cst<T>(5.0) : cst<T>(2.0);
  T u[3], p[3], k1[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    u[c] = a.u0[c * n + i];
    p[c] = a.p[c * n + i];
  }
  int nst = 0, nrej = 0, status = GS_TRAJ_OK;
  rhs3<T, SYS>(u, p, k1);
  bool finite = true;
#pragma unroll
  for (int c = 0; c < 3; ++c) finite = finite && isfinite(k1[c]) && isfinite(u[c]);
  T hprop = cst<T>(0.0);
  if (finite) {
    hprop = a.h0 > cst<T>(0.0) ? a.h0 : initial_step3<T, SYS, METHOD>(u, p, a.t0, a.t1, a.rtol, a.atol);
    if (!(hprop > cst<T>(0.0)) || !isfinite(hprop)) finite = false;
  }
  if (!finite) status = GS_TRAJ_NONFINITE;
  // the controller carries ln(errprev); errprev starts at 1 and is floored at 1e-4
  T t = a.t0, lnprev = cst<T>(0.0);
  const T ln_floor = ctrl_ln<T>(cst<T>(1e-4));
  bool prev_rej = false;
  int kk = 0;
  T* hout = STORE ? a.h + j * a.hcol : nullptr;
  while (status == GS_TRAJ_OK) {
    const T tstop = kk < a.nsave ? a.tsave[kk] : a.t1;
    if (hprop < cst<T>(16.0) * eps * fabs(t)) {
      status = GS_TRAJ_DTMIN;
      break;
    }
    const T tn = t + hprop;
    const bool clipped = tn >= tstop - cst<T>(4.0) * eps * fabs(tstop);
    const T h = clipped ? tstop - t : hprop;
    T un[3], k7[3], e[3];
    if (METHOD == GS_TSIT5) {
      tsit5_err_step<T, SYS>(u, p, h, k1, un, k7, e);
    } else {
      if (!ros2_err_step<T, SYS>(u, p, h, un, e)) {
        status = GS_TRAJ_SINGULAR;
        break;
      }
    }
    T sc[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) sc[c] = fmaT(a.rtol, smax_(fabs(u[c]), fabs(un[c])), a.atol);
    const T err = rms3(e, sc);
    if (err <= cst<T>(1.0)) {
      if (nst >= a.smax) {
        status = GS_TRAJ_MAXSTEPS;
        break;
      }
      if (STORE) hout[(int64_t)nst * a.hstep] = h;
      ++nst;
      t = clipped ? tstop : tn;
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        u[c] = un[c];
        if (METHOD == GS_TSIT5) k1[c] = k7[c];
      }
      while (kk < a.nsave && t == a.tsave[kk]) {
        if (STORE) a.save_idx[(int64_t)kk * n + j] = nst;
        ++kk;
      }
      // fac = 0.9 err^(-0.7/q) errprev^(0.4/q), as 0.9 exp(-(0.7/q) ln err + (0.4/q) ln errprev)
      T fac, lnerr = ln_floor;
      if (err == cst<T>(0.0)) {
        fac = cst<T>(10.0);
      } else {
        lnerr = ctrl_ln<T>(err);
        fac = cst<T>(0.9) * ctrl_exp<T>(fmaT(-(cst<T>(0.7) / q), lnerr, (cst<T>(0.4) / q) * lnprev));
        fac = smin_(cst<T>(10.0), smax_(cst<T>(0.2), fac));
      }
      if (prev_rej) fac = smin_(fac, cst<T>(1.0));
      lnprev = err < cst<T>(1e-4) ? ln_floor : lnerr;
      prev_rej = false;
      hprop = fac * hprop;
      if (t >= a.t1) break;
    } else {
      ++nrej;
      if (nrej > a.smax) {
        status = GS_TRAJ_MAXSTEPS;
        break;
      }
      const T fac = !isfinite(err) ? cst<T>(0.2)
                                   : smax_(cst<T>(0.2), cst<T>(0.9) * ctrl_exp<T>(-(cst<T>(1.0) / q) * ctrl_ln<T>(err)));
      hprop = fac * hprop;
      prev_rej = true;
    }
  }
  if (STORE) {
    // unreached save points (a failed trajectory); the h tail stays unwritten
    for (int k = kk; k < a.nsave; ++k) a.save_idx[(int64_t)k * n + j] = 0;
  }
  a.nsteps[j] = nst;
  if (a.status) a.status[j] = status;
  if (a.nreject) a.nreject[j] = nrej;
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
  for (int k = 0; k < P->nsave; ++k) a.tsave[k] = (T)P->tsave[k];
  return a;
}

template <typename T, int SYS, int METHOD, bool STORE>
static gs_status launch_rec(const RecArgs<T>& a, cudaStream_t st) {
  const int bs = 128;
  const int64_t grid = (a.n + bs - 1) / bs;
  k_record3<T, SYS, METHOD, STORE><<<(unsigned)grid, bs, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template <typename T, bool STORE>
static gs_status dispatch_rec(int sys, int method, const RecArgs<T>& a, cudaStream_t st) {
  if (sys == GS_LORENZ && method == GS_TSIT5) return launch_rec<T, kSysLorenz, GS_TSIT5, STORE>(a, st);
  if (sys == GS_LORENZ && method == GS_ROS2) return launch_rec<T, kSysLorenz, GS_ROS2, STORE>(a, st);
  if (sys == GS_ROBERTSON && method == GS_TSIT5) return launch_rec<T, kSysRobertson, GS_TSIT5, STORE>(a, st);
  if (sys == GS_ROBERTSON && method == GS_ROS2) return launch_rec<T, kSysRobertson, GS_ROS2, STORE>(a, st);
  return GS_EUNSUPPORTED;
}

gs_status count3(const gs_problem* P, const gs_tol* tol, int32_t smax, int32_t* nsteps, int32_t* status,
                 cudaStream_t st) {
  if (P->dtype == GS_F64) {
    RecArgs<double> a = rec_args<double>(P, tol, smax);
    a.nsteps = nsteps;
    a.status = status;
    return dispatch_rec<double, false>(P->system, P->method, a, st);
  }
  RecArgs<float> a = rec_args<float>(P, tol, smax);
  a.nsteps = nsteps;
  a.status = status;
  return dispatch_rec<float, false>(P->system, P->method, a, st);
}

static size_t al256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace of gs_record: trajectory-order copies of nsteps, status, nreject,
// save_idx and h, then the sort histogram.
size_t record_ws_bytes(int64_t n, int32_t smax, int32_t nsave, size_t tsize) {
  const int64_t nchunk = (n + kChunk - 1) / kChunk;
  return 3 * al256((size_t)n * 4) + al256((size_t)nsave * n * 4) + al256((size_t)smax * n * tsize) +
         (size_t)(smax + 1) * (size_t)nchunk * 4;
}

template <typename T>
__global__ void k_gather_mesh(int64_t n, int smax, int nsave, const int32_t* __restrict__ order,
                              const T* __restrict__ h_tmp, const int32_t* __restrict__ si_tmp,
                              const int32_t* __restrict__ ns_tmp, const int32_t* __restrict__ st_tmp,
                              const int32_t* __restrict__ nr_tmp, T* h, int32_t* save_idx, int32_t* nsteps,
                              int32_t* status, int32_t* nreject) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t i = order[j];
  const int S = ns_tmp[i];
  nsteps[j] = S;
  status[j] = st_tmp[i];
  nreject[j] = nr_tmp[i];
  for (int k = 0; k < nsave; ++k) save_idx[(int64_t)k * n + j] = si_tmp[(int64_t)k * n + i];
  const T* src = h_tmp + i * smax;  // trajectory-major: a thread reads one row in order
  for (int s = 0; s < smax; ++s) h[(int64_t)s * n + j] = s < S ? src[s] : cst<T>(0.0);
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
  int32_t* hist = (int32_t*)w;
  RecArgs<T> a = rec_args<T>(P, tol, M->smax);
  a.order = nullptr;  // trajectory order
  a.h = h_tmp;
  a.hcol = M->smax;  // trajectory-major workspace copy: each thread writes its own row
  a.hstep = 1;
  a.save_idx = si_tmp;
  a.nsteps = ns_tmp;
  a.status = st_tmp;
  a.nreject = nr_tmp;
  gs_status rc = dispatch_rec<T, true>(P->system, P->method, a, st);
  if (rc != GS_OK) return rc;
  rc = order_slots(ns_tmp, n, M->smax, hist, M->order, st);
  if (rc != GS_OK) return rc;
  k_gather_mesh<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(n, M->smax, P->nsave, M->order, h_tmp, si_tmp, ns_tmp,
                                                                 st_tmp, nr_tmp, (T*)M->h, M->save_idx, M->nsteps,
                                                                 M->status, M->nreject);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

gs_status record3(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws, cudaStream_t st) {
  return P->dtype == GS_F64 ? record3_t<double>(P, tol, M, ws, st) : record3_t<float>(P, tol, M, ws, st);
}

gs_status node64_record_pass(const gs_problem*, const gs_tol*, int32_t, bool, float*, int32_t*, int32_t*, int32_t*,
                             int32_t*, cudaStream_t);

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
  gs_status rc = node64_record_pass(P, tol, M->smax, true, h_tmp, si_tmp, ns_tmp, st_tmp, nr_tmp, st);
  if (rc != GS_OK) return rc;
  rc = order_slots(ns_tmp, n, M->smax, hist, M->order, st);
  if (rc != GS_OK) return rc;
  k_gather_mesh<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(n, M->smax, P->nsave, M->order, h_tmp, si_tmp, ns_tmp,
                                                                 st_tmp, nr_tmp, (T*)M->h, M->save_idx, M->nsteps,
                                                                 M->status, M->nreject);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

}  // namespace gs
