// grad_vern7.cu -- fused fixed-step replay + reverse sweep (the discrete
// adjoint) for Verner's 7(6) pair on the Lorenz system.
//
// GRADSOLVE (arXiv 2609.02876), evolve.pub review "Summary" and "Strengths:
// precisely scoped exactness claim": the gradient is the exact derivative of
// the fixed-step replay of the recorded steps, the mesh held as data.  The
// gist.science summary of arXiv 2609.28458 ("Results", "Source of Speed-up")
// names Verner 7 beside Tsit5 as the explicit methods compared.
//
// Forward half: for s < S replay step s with h[s] in the method's
// floating-point contract (vern7_step3: nine stages, no error estimate) and
// store u_s to the checkpoint workspace ck[s][c][slot].  The loss is then
// summed from the checkpoints, every lane at once, in the contract's order,
// and each save point's loss gradient goes to a workspace tail.
//
// Reverse half: for s = S-1 .. 0, reload u_s, recompute the stage states
// U_2..U_9 of step s (the same arithmetic as the forward), and apply the
// transposed step.  With u_{s+1} = u_s + h sum_j b_j k_j, k_j = f(U_j),
// U_j = u_s + h sum_{m<j} a_jm k_m and lambda = dL/du_{s+1}:
//   nu_j  = h (b_j lambda + sum_{m>j} a_mj mu_m)     (= dL/dk_j)
//   mu_j  = J(U_j)^T nu_j                              (= dL/dU_j)
//   pbar += f_p(U_j)^T nu_j
//   lambda <- lambda + sum_j mu_j                      (= dL/du_s)
// for j = 9 .. 1, over the pair's nonzero coefficients (stage 10 belongs to
// the error estimate only).  The mu_m are kept until the nu_j that need them
// are formed: as U_j is consumed mu_j takes its place, so U and mu together
// hold 27 values through the transposed step.
//
// Execution: one thread per slot (blocks of 128); gs_record orders slots by
// decreasing step count, so a warp's chains have nearly equal length.  h and
// the checkpoints are step-major over slots (a warp reads 32 consecutive
// elements of a row) and stream into per-thread shared-memory rings with
// cp.async, kV7Ring steps ahead, as in the Tsit5 kernel.
#include "steps.cuh"

namespace gs {

// 4 resident blocks of 128 per SM (125 registers, no spill; 16 warps/SM):
// 9.88-9.91 ms per pass on the 2^20 Lorenz ensemble against 9.91 ms at 3
// blocks (165 registers); the copy rings took 10.17 ms to 9.91 (3 blocks).
#ifndef GS_V7_MINB
#define GS_V7_MINB 4
#endif
#ifndef GS_V7_RING
#define GS_V7_RING 8
#endif
constexpr int kV7Ring = GS_V7_RING;
constexpr int kV7BS = 128;  // threads per block; a thread's ring rows are kV7BS elements apart
static_assert((kV7Ring & (kV7Ring - 1)) == 0 && kV7Ring >= 2, "ring depth: a power of two, at least 2");

template <typename T>
struct Vern7LorenzArgs {
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
  T* loss;          // [n] by trajectory
  T* dp;            // [3][n]
  T* du0;           // [3][n]
  T* ck;            // workspace [smax][3][n] by slot
  T* gsave;         // workspace tail [nsave][3][n] by slot: the save points' loss gradients
};

// dL/dU = J(U)^T nu and pbar += f_p(U)^T nu for Lorenz.
template <typename T>
__device__ __forceinline__ void lorenz_vjp3(const T U[3], T s, T r, T b, const T nu[3], T mu[3], T pb[3]) {
  const T m = s * nu[0];
  mu[0] = fmaT(r - U[2], nu[1], fmaT(U[1], nu[2], -m));
  mu[1] = fmaT(U[0], nu[2], m - nu[1]);
  mu[2] = -fmaT(U[0], nu[1], b * nu[2]);
  pb[0] = fmaT(U[1] - U[0], nu[0], pb[0]);
  pb[1] = fmaT(U[0], nu[1], pb[1]);
  pb[2] = fmaT(-U[2], nu[2], pb[2]);
}

template <typename T>
__global__ void __launch_bounds__(kV7BS, GS_V7_MINB) k_grad_vern7_lorenz(Vern7LorenzArgs<T> a) {
  const int64_t n = a.n;
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
  const int64_t i = a.order[j];
  if (i < 0 || i >= n) return;  // not a permutation entry: nothing to write
  const int S = a.nsteps[j];
  if (a.status[j] != GS_TRAJ_OK || S < 0 || S > a.smax) {
    a.loss[i] = nan;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      a.dp[c * n + i] = nan;
      a.du0[c * n + i] = nan;
    }
    return;
  }
  const T pr[3] = {a.p[i], a.p[n + i], a.p[2 * n + i]};
  const T s = pr[0], r = pr[1], b = pr[2];
  T u[3] = {a.u0[i], a.u0[n + i], a.u0[2 * n + i]};
  const int64_t n3 = 3 * n;
  const T* hp = a.h + j;
  T* cp = a.ck + j;

  // Per-thread copy rings (cp.async into shared memory, each thread waiting
  // on its own copies only): forward, row st % kV7Ring holds h of step st;
  // reverse, rows 4 (st % kV7Ring) + c hold checkpoint row c (c < 3) and h
  // (c = 3) of step st.  Element (row w) of a thread is rg[w * kV7BS]:
  // consecutive threads touch consecutive words.
  extern __shared__ __align__(16) unsigned char v7_ring_raw[];
  T* const rg = reinterpret_cast<T*>(v7_ring_raw) + threadIdx.x;

  // ---------------------------------------------------------------- forward
  {
    auto issue_f = [&](int sf) {
      if (sf < S) cp_async_el(rg + (sf & (kV7Ring - 1)) * kV7BS, hp + (int64_t)sf * n);
      cp_async_commit();
    };
    T k1[3];
    rhs3<T, kSysLorenz>(u, pr, k1);
#pragma unroll
    for (int sf = 0; sf < kV7Ring; ++sf) issue_f(sf);
    cp_async_wait<kV7Ring - 1>();
    T hn = S > 0 ? rg[0] : cst<T>(0.0);
    for (int st = 0; st < S; ++st) {
      const T h = hn;
      cp_async_wait<kV7Ring - 2>();  // the group of step st + 1
      if (st + 1 < S) hn = rg[((st + 1) & (kV7Ring - 1)) * kV7BS];
#pragma unroll
      for (int c = 0; c < 3; ++c) cp[(int64_t)st * n3 + c * n] = u[c];
      T un[3];
      vern7_step3<T, kSysLorenz>(u, pr, h, k1, un, nullptr);
#pragma unroll
      for (int c = 0; c < 3; ++c) u[c] = un[c];
      rhs3<T, kSysLorenz>(u, pr, k1);
      issue_f(st + kV7Ring);  // into the row step st has left
    }
    cp_async_wait<0>();  // the reverse reuses the rows
  }
  // Save points: u(t_k) is the state after step save_idx[k] (its checkpoint,
  // or the final state), taken while the step counts stay in [1, S] and
  // increase; nvalid counts them.  Loss in the contract's order (save
  // points, then components); the loss gradients to the workspace.
  int nvalid = 0;
  {
    const T* lvec = a.loss_kind == GS_LOSS_SUMSQ ? a.target : a.weight;
    T L = cst<T>(0.0);
    int prev = 0;
    for (int k = 0; k < a.nsave && S > 0; ++k) {
      const int sk = a.save_idx[(int64_t)k * n + j];
      if (!(sk > prev && sk <= S)) break;
      prev = sk;
      T uk[3] = {u[0], u[1], u[2]};
      if (sk < S)
#pragma unroll
        for (int c = 0; c < 3; ++c) uk[c] = a.ck[(int64_t)sk * n3 + c * n + j];
      T v[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)}, g[3];
      if (lvec)
#pragma unroll
        for (int c = 0; c < 3; ++c) v[c] = lvec[(int64_t)k * n3 + c * n + i];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        if (a.loss_kind == GS_LOSS_SUMSQ) {
          const T dl = uk[c] - v[c];
          L = fmaT(dl, dl, L);
          g[c] = cst<T>(2.0) * dl;
        } else {
          L = fmaT(v[c], uk[c], L);
          g[c] = v[c];
        }
        a.gsave[(int64_t)k * n3 + c * n + j] = g[c];
      }
      nvalid = k + 1;
    }
    a.loss[i] = L;
  }

  // ---------------------------------------------------------------- reverse
  T lam[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  T pb[3] = {cst<T>(0.0), cst<T>(0.0), cst<T>(0.0)};
  int kk = nvalid - 1;
  int next = kk >= 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
  auto issue_r = [&](int sr) {  // step sr's checkpoint rows and h
    if (sr >= 0 && sr < S) {
      T* d = rg + (sr & (kV7Ring - 1)) * 4 * kV7BS;
#pragma unroll
      for (int c = 0; c < 3; ++c) cp_async_el(d + c * kV7BS, cp + (int64_t)sr * n3 + c * n);
      cp_async_el(d + 3 * kV7BS, hp + (int64_t)sr * n);
    }
    cp_async_commit();
  };
  T cu[3], ch = cst<T>(0.0);
  auto take_r = [&](int sr) {
    const T* d = rg + (sr & (kV7Ring - 1)) * 4 * kV7BS;
#pragma unroll
    for (int c = 0; c < 3; ++c) cu[c] = d[c * kV7BS];
    ch = d[3 * kV7BS];
  };
#pragma unroll
  for (int i2 = 0; i2 < kV7Ring; ++i2) issue_r(S - 1 - i2);
  cp_async_wait<kV7Ring - 1>();
  if (S > 0) take_r(S - 1);
  for (int st = S - 1; st >= 0; --st) {
    // save points reached at u_{st+1} add their loss gradient to lambda
    while (st + 1 == next) {
#pragma unroll
      for (int c = 0; c < 3; ++c) lam[c] += a.gsave[(int64_t)kk * n3 + c * n + j];
      --kk;
      next = kk >= 0 ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
    const T h = ch;
    T U[9][3];
#pragma unroll
    for (int c = 0; c < 3; ++c) U[0][c] = cu[c];
    // recompute the stage states of step st (the forward's arithmetic)
    {
      T k[8][3];
      rhs3<T, kSysLorenz>(U[0], pr, k[0]);
#pragma unroll
      for (int jj = 2; jj <= 9; ++jj) {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          T acc = cst<T>(v7_a(jj, 1)) * k[0][c];
#pragma unroll
          for (int m = 2; m < jj; ++m)
            if (v7_a(jj, m) != 0.0) acc = fmaT(cst<T>(v7_a(jj, m)), k[m - 1][c], acc);
          U[jj - 1][c] = fmaT(h, acc, U[0][c]);
        }
        if (jj < 9) rhs3<T, kSysLorenz>(U[jj - 1], pr, k[jj - 1]);
      }
    }
    // transposed step, stages 9 .. 1
    T mu[9][3];
#pragma unroll
    for (int jj = 9; jj >= 1; --jj) {
      T nu[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        T acc = v7_b(jj) != 0.0 ? cst<T>(v7_b(jj)) * lam[c] : cst<T>(0.0);
#pragma unroll
        for (int m = jj + 1; m <= 9; ++m)
          if (v7_a(m, jj) != 0.0) acc = fmaT(cst<T>(v7_a(m, jj)), mu[m - 1][c], acc);
        nu[c] = h * acc;
      }
      lorenz_vjp3(U[jj - 1], s, r, b, nu, mu[jj - 1], pb);
    }
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      T sum = mu[0][c];
#pragma unroll
      for (int jj = 2; jj <= 9; ++jj) sum += mu[jj - 1][c];
      lam[c] += sum;
    }
    // step st - 1's ring entries, after the transposed step (not live across
    // it); then refill the rows step st has left
    if (st > 0) {
      cp_async_wait<kV7Ring - 2>();  // the group of step st - 1
      take_r(st - 1);
    }
    issue_r(st - kV7Ring);
  }
  cp_async_wait<0>();
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    a.dp[c * n + i] = pb[c];
    a.du0[c * n + i] = lam[c];
  }
}

size_t grad_vern7_lorenz_ws_bytes(int32_t dtype, int64_t n, int32_t smax, int32_t nsave) {
  const size_t tsize = dtype == GS_F64 ? 8 : 4;
  return ((size_t)smax * 3 + (size_t)nsave * 3) * (size_t)n * tsize;
}

template <typename T>
gs_status launch_grad_vern7_lorenz(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp,
                                   void* du0, void* ws, cudaStream_t st) {
  Vern7LorenzArgs<T> a;
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
  a.gsave = (T*)ws + (size_t)M->smax * 3 * (size_t)P->n;
  const int64_t grid = (P->n + kV7BS - 1) / kV7BS;
  const size_t smem = (size_t)kV7Ring * 4 * kV7BS * sizeof(T);  // the larger (reverse) ring
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(k_grad_vern7_lorenz<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return GS_ECUDA;
  k_grad_vern7_lorenz<T><<<(unsigned)grid, kV7BS, smem, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_grad_vern7_lorenz<double>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                    void*, void*, cudaStream_t);
template gs_status launch_grad_vern7_lorenz<float>(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*,
                                                   void*, void*, cudaStream_t);

}  // namespace gs
