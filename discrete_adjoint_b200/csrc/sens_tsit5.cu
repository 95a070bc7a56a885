// sens_tsit5.cu -- forward sensitivities of the fixed-step Tsit5 replay on the
// Lorenz system: the tangent of the replay along each input direction
// (sigma, rho, beta, x0, y0, z0), integrated alongside the state.
//
// The derivative is the one the adjoint returns: the exact derivative of the
// fixed-step replay of the recorded steps, the mesh held as data (GRADSOLVE,
// evolve.pub review, "Strengths: precisely scoped exactness claim").  Forward
// mode gives, besides the loss gradient, the whole sensitivity matrix
// d u(t_k) / d (p, u0) at every save point; it is the few-parameter route the
// gptget summary contrasts with the adjoint.
//
// Tangent of one Tsit5 step along a direction (v = du, w = dp):
//   dk_j = J(U_j) dU_j + f_p(U_j) w,   dU_j = v + h sum_{m<j} a_jm dk_m,
//   v' = v + h sum_j b_j dk_j,
// with dk_1 carried over from the previous step (FSAL, as k_1).
//
// Dense save points (a dense record: theta in (0, 1) inside a step): the
// state there is Tsit5's continuous extension over the step's stages,
//   u(theta) = u_s + h sum_i b_i(theta) k_i   (k_7 = f(u_{s+1})),
// theta and h data, so its tangent is v_s + h sum_i b_i(theta) dk_i.  The
// branch recomputes the step's stages and their tangents from (u_s, v_s),
// which the dense instance keeps; k_7 and dk_7 are the FSAL slope and its
// tangent the step has just formed.
//
// Execution: one thread per (slot, NDIR directions).  The six directions of a
// slot run in 6 / NDIR threads, each of which replays the state itself (192
// flop a step against 252 per direction).  The default carries all six in one
// thread (NDIR = 6: the state replays once; 7 slopes x 3 components x 6
// tangents take the fp64 instance to 255 registers with a small spill), which
// measured 1.66x faster than one direction per thread (2^20 Lorenz
// trajectories: 25.6 ms against 42.4 ms; 3 directions: 28.9 ms) and 1.45-1.8x
// for the dense and fp32 instances.  With NDIR < 6, consecutive blocks take
// the direction sets of one range of 128 slots (block b: slots 128 (b / G) ..,
// direction set b % G, G = 6 / NDIR), so the threads of a warp share one
// direction set and read consecutive elements of the step-major mesh, and the
// G blocks of a range share those lines through L2.  No workspace: nothing is
// stored but the save-point sensitivities.
#include "steps.cuh"
#include "vec.cuh"

namespace gs {

#ifndef GS_SENS_NDIR
#define GS_SENS_NDIR 6
#endif
// Directions per thread on dense meshes, and whether their save-point branch
// is a call (1) or inlined (0).  At a dense save point the branch recomputes
// the step's stages and their tangents; with six directions per thread that
// spills heavily.  Measured on the 2^20 Lorenz dense mesh (fp64): six
// directions, call 88 ms / inlined 68 ms; three, call 58.5 / inlined 40.3;
// two, inlined 39.0; one, inlined 57.8 (landing meshes, six: 25.5 ms).
#ifndef GS_SENS_NDIR_DENSE
#define GS_SENS_NDIR_DENSE 2
#endif
#ifndef GS_SENS_DENSE_NOINLINE
#define GS_SENS_DENSE_NOINLINE 0
#endif
#if GS_SENS_DENSE_NOINLINE
#define GS_SENS_DENSE_FN __noinline__
#else
#define GS_SENS_DENSE_FN __forceinline__
#endif
template <int NDIR>
constexpr int sens_minb() {
  return NDIR == 6 ? 1 : (NDIR == 1 ? 4 : 2);
}

template <typename T>
struct SensArgs {
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
  const T* theta;   // [nsave][n] by slot: dense save points, or null
};

// J(u) v + f_p(u) w for f = (s (y - x), x (r - z) - y, x y - b z).
template <typename T, typename V>
__device__ __forceinline__ void lorenz_jvp(T x, T y, T z, T s, T r, T b, const V& vx, const V& vy, const V& vz,
                                           const V& ws, const V& wr, const V& wb, V& gx, V& gy, V& gz) {
  gx = fmaT(s, vy - vx, ws * (y - x));
  gy = fmaT(r - z, vx, fmaT(x, wr - vz, -vy));
  gz = fmaT(y, vx, fmaT(x, vy, -fmaT(b, vz, wb * z)));
}

// stage accumulators in the contract's order (state) and the same order for
// the tangents
#define GS_S_ACC1(A, K)          \
  ax = tsc<T, A>() * K##x;         \
  ay = tsc<T, A>() * K##y;         \
  az = tsc<T, A>() * K##z;         \
  dax = tsc<T, A>() * d##K##x;     \
  day = tsc<T, A>() * d##K##y;     \
  daz = tsc<T, A>() * d##K##z;
#define GS_S_ACCN(A, K)                 \
  ax = fmaT(tsc<T, A>(), K##x, ax);       \
  ay = fmaT(tsc<T, A>(), K##y, ay);       \
  az = fmaT(tsc<T, A>(), K##z, az);       \
  dax = fmaT(tsc<T, A>(), d##K##x, dax);  \
  day = fmaT(tsc<T, A>(), d##K##y, day);  \
  daz = fmaT(tsc<T, A>(), d##K##z, daz);
#define GS_S_STAGE(KN)                                                \
  Ux = fmaT(h, ax, x);                                                \
  Uy = fmaT(h, ay, y);                                                \
  Uz = fmaT(h, az, z);                                                \
  dUx = fmaT(h, dax, vx);                                             \
  dUy = fmaT(h, day, vy);                                             \
  dUz = fmaT(h, daz, vz);                                             \
  lorenz_f(Ux, Uy, Uz, s, r, b, KN##x, KN##y, KN##z);                 \
  lorenz_jvp(Ux, Uy, Uz, s, r, b, dUx, dUy, dUz, ws, wr, wb, d##KN##x, d##KN##y, d##KN##z);

// A dense save point inside a step: Tsit5's continuous extension and its
// tangent, from the step's stages and their tangents recomputed from
// (u_s, v_s) with the step's own arithmetic; k_7 and dk_7 are the FSAL slope
// and its tangent that the step has formed.
template <typename T, int NDIR>
struct DenseTanIn {
  T x, y, z, k1x, k1y, k1z, k7x, k7y, k7z, s, r, b, h, th;
  vec<T, NDIR> vx, vy, vz, dk1x, dk1y, dk1z, dk7x, dk7y, dk7z, ws, wr, wb;
};
template <typename T, int NDIR>
struct DenseTanOut {
  T ux, uy, uz;
  vec<T, NDIR> tx, ty, tz;
};

template <typename T, int NDIR>
__device__ GS_SENS_DENSE_FN DenseTanOut<T, NDIR> tsit5_dense_tangent(const DenseTanIn<T, NDIR> in) {
  using V = vec<T, NDIR>;
  const T x = in.x, y = in.y, z = in.z, k1x = in.k1x, k1y = in.k1y, k1z = in.k1z, s = in.s, r = in.r, b = in.b,
          h = in.h;
  const V vx = in.vx, vy = in.vy, vz = in.vz, dk1x = in.dk1x, dk1y = in.dk1y, dk1z = in.dk1z, ws = in.ws,
          wr = in.wr, wb = in.wb;
  T ax, ay, az, Ux, Uy, Uz;
  V dax, day, daz, dUx, dUy, dUz;
  T k2x, k2y, k2z, k3x, k3y, k3z, k4x, k4y, k4z, k5x, k5y, k5z, k6x, k6y, k6z;
  V dk2x, dk2y, dk2z, dk3x, dk3y, dk3z, dk4x, dk4y, dk4z, dk5x, dk5y, dk5z, dk6x, dk6y, dk6z;
  GS_S_ACC1(kTsA21, k1)
  GS_S_STAGE(k2)
  GS_S_ACC1(kTsA31, k1)
  GS_S_ACCN(kTsA32, k2)
  GS_S_STAGE(k3)
  GS_S_ACC1(kTsA41, k1)
  GS_S_ACCN(kTsA42, k2)
  GS_S_ACCN(kTsA43, k3)
  GS_S_STAGE(k4)
  GS_S_ACC1(kTsA51, k1)
  GS_S_ACCN(kTsA52, k2)
  GS_S_ACCN(kTsA53, k3)
  GS_S_ACCN(kTsA54, k4)
  GS_S_STAGE(k5)
  GS_S_ACC1(kTsA61, k1)
  GS_S_ACCN(kTsA62, k2)
  GS_S_ACCN(kTsA63, k3)
  GS_S_ACCN(kTsA64, k4)
  GS_S_ACCN(kTsA65, k5)
  GS_S_STAGE(k6)
  T bw[7];
  tsit5_dense_w(in.th, bw);
  DenseTanOut<T, NDIR> o;
  o.ux = tsit5_dense_c(bw, x, k1x, k2x, k3x, k4x, k5x, k6x, in.k7x, h);
  o.uy = tsit5_dense_c(bw, y, k1y, k2y, k3y, k4y, k5y, k6y, in.k7y, h);
  o.uz = tsit5_dense_c(bw, z, k1z, k2z, k3z, k4z, k5z, k6z, in.k7z, h);
#pragma unroll
  for (int q = 0; q < NDIR; ++q) {
    o.tx.e[q] = tsit5_dense_c(bw, vx.e[q], dk1x.e[q], dk2x.e[q], dk3x.e[q], dk4x.e[q], dk5x.e[q], dk6x.e[q],
                              in.dk7x.e[q], h);
    o.ty.e[q] = tsit5_dense_c(bw, vy.e[q], dk1y.e[q], dk2y.e[q], dk3y.e[q], dk4y.e[q], dk5y.e[q], dk6y.e[q],
                              in.dk7y.e[q], h);
    o.tz.e[q] = tsit5_dense_c(bw, vz.e[q], dk1z.e[q], dk2z.e[q], dk3z.e[q], dk4z.e[q], dk5z.e[q], dk6z.e[q],
                              in.dk7z.e[q], h);
  }
  return o;
}

template <typename T, int NDIR, bool DENSE>
__global__ void __launch_bounds__(128, sens_minb<NDIR>()) k_sens_tsit5_lorenz(SensArgs<T> a) {
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
  const T s = a.p[i], r = a.p[n + i], b = a.p[2 * n + i];
  T x = a.u0[i], y = a.u0[n + i], z = a.u0[2 * n + i];
  V ws, wr, wb, vx, vy, vz;
#pragma unroll
  for (int q = 0; q < NDIR; ++q) {
    const int dq = dir0 + q;
    ws.e[q] = dq == 0 ? cst<T>(1.0) : cst<T>(0.0);
    wr.e[q] = dq == 1 ? cst<T>(1.0) : cst<T>(0.0);
    wb.e[q] = dq == 2 ? cst<T>(1.0) : cst<T>(0.0);
    vx.e[q] = dq == 3 ? cst<T>(1.0) : cst<T>(0.0);
    vy.e[q] = dq == 4 ? cst<T>(1.0) : cst<T>(0.0);
    vz.e[q] = dq == 5 ? cst<T>(1.0) : cst<T>(0.0);
  }
  T L = cst<T>(0.0);
  V dL = vsplat<T, NDIR>(cst<T>(0.0));
  int kk = 0, next = S > 0 ? a.save_idx[j] : -1;
  T k1x, k1y, k1z;
  V dk1x, dk1y, dk1z;
  lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);
  lorenz_jvp(x, y, z, s, r, b, vx, vy, vz, ws, wr, wb, dk1x, dk1y, dk1z);
  const T* hq = a.h + j;
  T hn = S > 0 ? hq[0] : cst<T>(0.0);
  for (int st = 0; st < S; ++st) {
    const T h = hn;
    hq += n;
    if (st + 1 < S) hn = *hq;
    if (st + 8 < S) prefetch_l2(hq + 7 * n);
    T ax, ay, az, Ux, Uy, Uz;
    V dax, day, daz, dUx, dUy, dUz;
    T k2x, k2y, k2z, k3x, k3y, k3z, k4x, k4y, k4z, k5x, k5y, k5z, k6x, k6y, k6z;
    V dk2x, dk2y, dk2z, dk3x, dk3y, dk3z, dk4x, dk4y, dk4z, dk5x, dk5y, dk5z, dk6x, dk6y, dk6z;
    GS_S_ACC1(kTsA21, k1)
    GS_S_STAGE(k2)
    GS_S_ACC1(kTsA31, k1)
    GS_S_ACCN(kTsA32, k2)
    GS_S_STAGE(k3)
    GS_S_ACC1(kTsA41, k1)
    GS_S_ACCN(kTsA42, k2)
    GS_S_ACCN(kTsA43, k3)
    GS_S_STAGE(k4)
    GS_S_ACC1(kTsA51, k1)
    GS_S_ACCN(kTsA52, k2)
    GS_S_ACCN(kTsA53, k3)
    GS_S_ACCN(kTsA54, k4)
    GS_S_STAGE(k5)
    GS_S_ACC1(kTsA61, k1)
    GS_S_ACCN(kTsA62, k2)
    GS_S_ACCN(kTsA63, k3)
    GS_S_ACCN(kTsA64, k4)
    GS_S_ACCN(kTsA65, k5)
    GS_S_STAGE(k6)
    // dense save points: u_s, f(u_s) and their tangents
    T xs, ys, zs, fsx, fsy, fsz;
    V vsx, vsy, vsz, dfsx, dfsy, dfsz;
    if (DENSE) {
      xs = x, ys = y, zs = z, fsx = k1x, fsy = k1y, fsz = k1z;
      vsx = vx, vsy = vy, vsz = vz, dfsx = dk1x, dfsy = dk1y, dfsz = dk1z;
    }
    // u_{s+1} and its tangent
    GS_S_ACC1(kTsB1, k1)
    GS_S_ACCN(kTsB2, k2)
    GS_S_ACCN(kTsB3, k3)
    GS_S_ACCN(kTsB4, k4)
    GS_S_ACCN(kTsB5, k5)
    GS_S_ACCN(kTsB6, k6)
    x = fmaT(h, ax, x);
    y = fmaT(h, ay, y);
    z = fmaT(h, az, z);
    vx = fmaT(h, dax, vx);
    vy = fmaT(h, day, vy);
    vz = fmaT(h, daz, vz);
    lorenz_f(x, y, z, s, r, b, k1x, k1y, k1z);  // FSAL
    lorenz_jvp(x, y, z, s, r, b, vx, vy, vz, ws, wr, wb, dk1x, dk1y, dk1z);
    // a landing record has at most one save point per step; a dense one any number
    while (st + 1 == next) {
      T ux = x, uy = y, uz = z;
      V tx = vx, ty = vy, tz = vz;
      if (DENSE) {
        const T th = a.theta[(int64_t)kk * n + j];
        if (th != cst<T>(1.0)) {
          DenseTanIn<T, NDIR> in;
          in.x = xs, in.y = ys, in.z = zs, in.k1x = fsx, in.k1y = fsy, in.k1z = fsz;
          in.k7x = k1x, in.k7y = k1y, in.k7z = k1z;  // f(u_{s+1}), the FSAL slope just formed
          in.s = s, in.r = r, in.b = b, in.h = h, in.th = th;
          in.vx = vsx, in.vy = vsy, in.vz = vsz, in.dk1x = dfsx, in.dk1y = dfsy, in.dk1z = dfsz;
          in.dk7x = dk1x, in.dk7y = dk1y, in.dk7z = dk1z;
          in.ws = ws, in.wr = wr, in.wb = wb;
          const DenseTanOut<T, NDIR> dt = tsit5_dense_tangent<T, NDIR>(in);
          ux = dt.ux, uy = dt.uy, uz = dt.uz;
          tx = dt.tx, ty = dt.ty, tz = dt.tz;
        }
      }
      const int64_t o = (int64_t)kk * n3 + i;
      if (a.loss_kind == GS_LOSS_SUMSQ) {
        const T ex = a.target ? ux - a.target[o] : ux;
        const T ey = a.target ? uy - a.target[o + n] : uy;
        const T ez = a.target ? uz - a.target[o + 2 * n] : uz;
        L = fmaT(ex, ex, L);
        L = fmaT(ey, ey, L);
        L = fmaT(ez, ez, L);
        dL = fmaT(cst<T>(2.0) * ex, tx, dL);
        dL = fmaT(cst<T>(2.0) * ey, ty, dL);
        dL = fmaT(cst<T>(2.0) * ez, tz, dL);
      } else {
        const T w0 = a.weight[o], w1 = a.weight[o + n], w2 = a.weight[o + 2 * n];
        L = fmaT(w0, ux, L);
        L = fmaT(w1, uy, L);
        L = fmaT(w2, uz, L);
        dL = fmaT(w0, tx, dL);
        dL = fmaT(w1, ty, dL);
        dL = fmaT(w2, tz, dL);
      }
      if (a.sens) {
#pragma unroll
        for (int q = 0; q < NDIR; ++q) {
          T* o6 = a.sens + ((int64_t)kk * 18 + dir0 + q) * n + i;
          o6[0] = tx.e[q];
          o6[6 * n] = ty.e[q];
          o6[12 * n] = tz.e[q];
        }
      }
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
      if (!DENSE) break;
    }
  }
  if (dir0 == 0) a.loss[i] = L;
#pragma unroll
  for (int q = 0; q < NDIR; ++q) {
    const int dq = dir0 + q;
    (dq < 3 ? a.dp : a.du0)[(dq % 3) * n + i] = dL.e[q];
  }
}

#undef GS_S_ACC1
#undef GS_S_ACCN
#undef GS_S_STAGE

template <typename T>
gs_status launch_sens_tsit5_lorenz(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp,
                                   void* du0, void* sens, cudaStream_t st) {
  SensArgs<T> a;
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
  a.theta = (const T*)M->save_theta;
  constexpr int ND = GS_SENS_NDIR, NDD = GS_SENS_NDIR_DENSE;
  static_assert(6 % ND == 0 && 6 % NDD == 0, "directions per thread must divide 6");
  const int64_t blocks = (P->n + 127) / 128;
  if (a.theta)
    k_sens_tsit5_lorenz<T, NDD, true><<<(unsigned)(blocks * (6 / NDD)), 128, 0, st>>>(a);
  else
    k_sens_tsit5_lorenz<T, ND, false><<<(unsigned)(blocks * (6 / ND)), 128, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_sens_tsit5_lorenz<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                    void*, void*, cudaStream_t);
template gs_status launch_sens_tsit5_lorenz<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                   void*, void*, cudaStream_t);

}  // namespace gs
