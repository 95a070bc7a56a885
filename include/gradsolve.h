/*
 * gradsolve.h -- C ABI of the B200 record-and-replay discrete-adjoint library
 * (libgradsolve.so).
 *
 * The method (GRADSOLVE, arXiv 2609.02876; abstract, and the evolve.pub
 * review's "Summary" and "Strengths: precisely scoped exactness claim"):
 * an adaptive solver runs once per trajectory and records the step sizes it
 * accepts (gs_record); a fixed-step replay of that mesh, the mesh held fixed as
 * data, defines a loss; gs_grad returns the exact derivative of that replay
 * (the discrete adjoint) with respect to each trajectory's parameters and
 * initial state, excluding any derivative of the step-size choices (review FAQ
 * "Is gradsolve's gradient really exact?").  gs_solve is the forward-only
 * replay.  One record serves any number of gs_grad / gs_solve calls: the
 * method is aimed at ensembles whose gradient is taken many times against a
 * single record (abstract).
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" are caller-owned device memory of the current
 *    CUDA device; "host" pointers are read during the call only.  The library
 *    allocates nothing: scratch memory is the caller's workspace, sized by
 *    gs_workspace_bytes.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronize.  Results are valid once the stream reaches
 *    the end of the call's work.
 *  - Outputs are overwritten, never accumulated.
 *  - Argument errors return a negative gs_status before anything is launched.
 *    A launch failure returns GS_ECUDA.  Failures of single trajectories are
 *    not call errors: they are reported per trajectory in mesh.status and the
 *    call returns GS_OK.
 *  - Layouts are structure-of-arrays over the ensemble ("SoA"): element c of
 *    trajectory i of an array shaped [m][n] is at [c * n + i].  Floating-point
 *    arrays have the problem's dtype (float for GS_F32, double for GS_F64).
 *  - Not thread-safe against concurrent calls that share a mesh or workspace.
 */
#ifndef GRADSOLVE_H
#define GRADSOLVE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GS_API __attribute__((visibility("default")))
#else
#define GS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t gs_status;
#define GS_OK 0
#define GS_EINVAL (-1)       /* bad argument (null pointer, size, combination) */
#define GS_ECUDA (-2)        /* a CUDA launch or runtime call failed */
#define GS_EWORKSPACE (-3)   /* workspace pointer null or smaller than required */
#define GS_EUNSUPPORTED (-4) /* valid request this library does not implement */

/* Per-trajectory record status (mesh.status). */
#define GS_TRAJ_OK 0
#define GS_TRAJ_MAXSTEPS 1  /* more than smax accepted steps or smax rejections */
#define GS_TRAJ_DTMIN 2     /* step proposal fell below 16 eps |t| */
#define GS_TRAJ_NONFINITE 3 /* non-finite input, f(u0) or initial step */
#define GS_TRAJ_SINGULAR 4  /* zero or non-finite pivot in the Rosenbrock LU */
#define GS_TRAJ_BADORDER 5  /* gs_record_inplace: the slot's order entry is outside [0, n) */

/* Registered right-hand sides. */
#define GS_LORENZ 1    /* d=3, np=3, p=(sigma, rho, beta): DiffEqGPU "ad" page, Lorenz listing */
#define GS_ROBERTSON 2 /* d=3, np=3, p=(k1, k2, k3): mass-action kinetics A->B, 2B->B+C, B+C->A+C */
#define GS_HIRES 3     /* reserved: not implemented (equations not given by the sources followed) */
#define GS_NODE64 4    /* d=64, np=64 (b_i), shared W [64][64]: f = tanh(W u + b) - u */
/* d=8, np=8 (k1..k8), GS_ROS2 / GS_ROS3 only: kin8, an 8-species stiff
 * mass-action network defined by this library (not a published test problem)
 * that runs the Rosenbrock path at d = 8 (8 x 8 LU in registers):
 *   A1 -> A2 (k1), A2 -> A1 (k2), A2 + A3 -> A4 (k3), A4 -> A3 + A5 (k4),
 *   A5 -> A6 (k5), A6 -> A5 (k6), A6 + A7 -> A8 (k7), A8 -> A7 + A1 (k8);
 * f = N r(u), r = (k1 u1, k2 u2, k3 u2 u3, k4 u4, k5 u5, k6 u6, k7 u6 u7,
 * k8 u8) with N the reactions' stoichiometric matrix. */
#define GS_KIN8 5

/* Integrators. */
#define GS_TSIT5 1 /* Tsitouras 5(4) pair, FSAL, PI step control */
#define GS_ROS2 2  /* Rosenbrock ROS2, gamma = 1 + 1/sqrt(2) (Verwer et al. 1999); d = 3 and kin8 */
/* Rosenbrock ROS3 (Sandu, Verwer, Blom, Spee, Carmichael & Potra 1997): three
 * stages, order 3, L-stable, embedded order 2, controller order q = 3; d = 3
 * and kin8.  Stage form, with J = J(u) and gamma = 0.435866521508459:
 *   M = I/gamma - h J;  M k1 = f(u);  v = u + h k1;  M k2 = f(v) + c21 k1;
 *   M k3 = f(v) + c31 k1 + c32 k2;  u_new = u + h (k1 + m2 k2 + m3 k3);
 *   error estimate h (e1 k1 + e2 k2 + e3 k3).  Higher-order stiff option of
 * GRADSOLVE's explicit and Rosenbrock integrators (abstract), with the
 * higher-order integrators it names as a next step ("Future directions"). */
#define GS_ROS3 3
/* Verner's 7(6) pair (Verner 2010, the "most efficient" 7(6) pair): ten
 * stages, seventh-order propagating weights on stages 1 and 4..9, the
 * sixth-order embedded weights on 1, 4..7 and 10 (stage 10 only for the error
 * estimate; not FSAL), controller order q = 7.  The explicit high-order
 * method the gist.science summary of arXiv 2609.28458 ("Results", "Source of
 * Speed-up") names beside Tsit5.  d = 3 systems, landing records only; the
 * gradient and the forward sensitivities on GS_LORENZ. */
#define GS_VERN7 4

#define GS_F32 1
#define GS_F64 2

/* Losses over the save points k = 0..nsave-1. */
#define GS_LOSS_SUMSQ 1  /* L_i = sum_k ||u_i(t_k) - target_ik||^2  (target NULL = 0) */
#define GS_LOSS_LINEAR 2 /* L_i = sum_k weight_ik . u_i(t_k) */

#define GS_MAX_SAVE 64 /* largest nsave */
#define GS_RECORD_INPLACE_WS 8 /* workspace bytes of gs_record_inplace and gs_solve_adaptive_ordered */

/* workspace operations */
#define GS_OP_RECORD 0
#define GS_OP_GRAD 1

/*
 * An ensemble of n independent trajectories of one registered system.
 *   p       device, [np][n]: per-trajectory parameters.
 *   u0      device, [d][n]:  initial states.
 *   shared  device, GS_NODE64 only: W, [64][64] row-major (row r, column c at
 *           r*64 + c), shared by all trajectories; NULL otherwise.
 *   t0, t1  time span, t0 < t1.
 *   tsave   host, nsave (1..GS_MAX_SAVE) strictly increasing times in (t0, t1]:
 *           the save points of gs_solve and of the loss.  Steps land on them,
 *           unless the record is dense (gs_tol.dense).
 */
typedef struct gs_problem {
  int32_t system, method, dtype, d, np;
  int64_t n;
  const void* p;
  const void* u0;
  const void* shared;
  double t0, t1;
  int32_t nsave;
  const double* tsave;
} gs_problem;

/* Step-size control: accept iff the RMS of e_c / (atol + rtol max(|u_c|, |u'_c|))
 * is <= 1.  h0 > 0 fixes the first proposal; h0 = 0 picks it automatically
 * (Hairer, Norsett & Wanner I, II.4).
 * dense = 0: steps are shortened to land on every save time.  dense = 1 (the
 * d = 3 systems, every method): steps stop only at t1; a save time inside a
 * step is located by its position theta in (0, 1] (gs_mesh.save_theta) and the
 * state there is read off the step's dense output:
 *   Tsit5: its own continuous extension (Tsitouras 2011), fourth order,
 *     u = u_s + h sum_{i=1..7} b_i(theta) k_i  (k_7 = f(u_{s+1})),
 *     b_i(theta) a quartic in theta with b_i(0) = 0, b_i(1) = b_i;
 *   ROS2, ROS3: the cubic Hermite interpolant on the end states and slopes,
 *     u = H00 u_s + H01 u_{s+1} + h (H10 f(u_s) + H11 f(u_{s+1})),
 *     H01 = theta^2 (3 - 2 theta), H00 = 1 - H01, H10 = theta (1 - theta)^2,
 *     H11 = -theta^2 (1 - theta).
 * The loss and its derivative then pass through that dense output (theta,
 * like h, is data).  Dense output (save times interpolated instead of
 * stepped onto: the gist.science summary of arXiv 2609.28458, "Methodology",
 * "Dense Output") names no interpolant; the method's own is the reading for
 * Tsit5, and the Rosenbrock methods take the Hermite one. */
typedef struct gs_tol {
  double rtol, atol, h0;
  int32_t dense;
} gs_tol;

/*
 * The record (the mesh), all device arrays, all indexed by SLOT, not by
 * trajectory: slot j holds trajectory order[j].  gs_record orders slots by
 * decreasing step count (ties by trajectory index) so that the threads of a
 * warp replay chains of nearly equal length; any permutation is valid input to
 * gs_grad / gs_solve (e.g. a mesh built elsewhere, with order = identity).
 *   smax      capacity in steps (rows of h).
 *   nsave     must equal the problem's nsave.
 *   h         [smax][n] dtype, step-major: step s of slot j at s*n + j;
 *             rows s >= nsteps[j] are zero.
 *   order     [n] int32, a permutation of 0..n-1.
 *   nsteps    [n] int32, accepted steps of slot j.
 *   save_idx  [nsave][n] int32, number of steps taken when t reached tsave[k]
 *             (1..nsteps[j]).
 *   status    [n] int32, GS_TRAJ_* of slot j.
 *   nreject   [n] int32, rejected attempts of slot j (diagnostic).
 *   save_theta [nsave][n] dtype, or NULL: for a dense record, the position of
 *             save time k inside step save_idx - 1, in (0, 1]; NULL means the
 *             save points are step ends (theta = 1).  gs_record writes it when
 *             gs_tol.dense is set (and then requires it).
 */
typedef struct gs_mesh {
  int32_t smax, nsave;
  void* h;
  int32_t* order;
  int32_t* nsteps;
  int32_t* save_idx;
  int32_t* status;
  int32_t* nreject;
  void* save_theta;
} gs_mesh;

/* Loss description.  target / weight: device, [nsave][d][n] dtype, indexed by
 * trajectory.  SUMSQ reads target (NULL = zero target); LINEAR reads weight. */
typedef struct gs_loss {
  int32_t kind;
  const void* target;
  const void* weight;
} gs_loss;

/*
 * Workspace (scratch) bytes that op (GS_OP_RECORD / GS_OP_GRAD) needs for this
 * problem and mesh capacity: record -- step counts of the sizing pass and the
 * slot-ordering histograms; grad -- one checkpointed state per step and slot,
 * [smax][d][n] dtype (plus the d=64 weight-gradient partials; for Tsit5 and
 * Verner 7 on Lorenz plus 3 values per save point and slot, 9 for a dense
 * Tsit5 mesh).  Returns
 * 0 for an invalid request.  Host function; no device work.
 */
GS_API size_t gs_workspace_bytes(const gs_problem* prob, const gs_mesh* mesh, int32_t op);

/*
 * Sizing pass: runs the adaptive solve of every trajectory without storing a
 * mesh and writes, indexed by TRAJECTORY, the accepted step count (nsteps) and
 * status (both device [n] int32; status may be NULL).  smax caps the count
 * (GS_TRAJ_MAXSTEPS beyond it).  Use it to pick the mesh capacity.
 * (The recorder of the gptget summary, "Methodology", without its stores.)
 */
GS_API gs_status gs_count(const gs_problem* prob, const gs_tol* tol, int32_t smax, int32_t* nsteps, int32_t* status,
                   void* stream);

/*
 * Record: adaptive solve of every trajectory (Tsit5, Verner 7, ROS2 or ROS3 per prob->method)
 * into the caller's mesh, slots ordered by decreasing step count.  Fills every
 * mesh array.  Trajectories that fail keep a status != 0 and a truncated mesh.
 * Runs the adaptive pass into the workspace (trajectory order), the slot
 * ordering and a gather into slot order, all on stream.  Built for GS_LORENZ
 * and GS_ROBERTSON with GS_TSIT5, GS_VERN7, GS_ROS2 or GS_ROS3, GS_KIN8 with
 * GS_ROS2 or GS_ROS3 (fp64 and fp32), and GS_NODE64 with GS_TSIT5 in fp32;
 * dense records for GS_TSIT5, GS_ROS2 and GS_ROS3 on the d = 3 systems.  gs_count, gs_solve and gs_solve_adaptive
 * take the same combinations.  (Evolve.pub review, "Summary": the adaptive
 * solve happens once and keeps each trajectory's accepted step sizes.)
 */
GS_API gs_status gs_record(const gs_problem* prob, const gs_tol* tol, const gs_mesh* mesh, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * Re-record in place: the adaptive solve of every trajectory, as gs_record
 * runs it, into a mesh whose slot order an earlier record of this ensemble
 * (gs_record, or this call) set.  The order is kept: mesh->order is read, not
 * written, and must be a permutation of 0..n-1 (an entry outside [0, n) gives
 * its slot GS_TRAJ_BADORDER and no steps; duplicates are not detected).  Each
 * slot's steps, count, status, rejections, save indices (and save positions
 * of a dense record) are written straight into the slot, with no workspace
 * copy, sort or gather; h rows from the slot's new count up to its previous
 * count (mesh->nsteps on entry, clamped to [0, smax]) are zeroed, so a mesh
 * that was zero padded stays so.  Slots run in groups of 32 in slot order, so
 * an order sorted by step count (what gs_record leaves) keeps the lanes of a
 * warp on chains of about equal length.  When the trajectories' step counts
 * changed since the order was set, the mesh is still exact, only less well
 * sorted for gs_grad; gs_record sorts afresh.
 *   ws        device, at least GS_RECORD_INPLACE_WS bytes, 8-byte aligned
 *             (a work counter; gs_workspace_bytes(GS_OP_RECORD) is enough).
 * Values equal gs_record's bit for bit (each trajectory's arithmetic does not
 * depend on where it runs).  Same systems, methods and precisions as
 * gs_record except GS_NODE64 (GS_EUNSUPPORTED).  (Evolve.pub review,
 * "Summary": the mesh stays fixed between re-records; this is the
 * re-record.)
 */
GS_API gs_status gs_record_inplace(const gs_problem* prob, const gs_tol* tol, const gs_mesh* mesh, void* ws,
                                   size_t ws_bytes, void* stream);

/*
 * Forward-only replay on the mesh: u_save, device [nsave][d][n] dtype, indexed
 * by trajectory, receives the state at each save point.  Slots with status != 0
 * get NaN.  (The forward-only solver use of the abstract.)
 */
GS_API gs_status gs_solve(const gs_problem* prob, const gs_mesh* mesh, void* u_save, void* stream);

/*
 * Adaptive forward-only solve: the recorder's adaptive iteration (same
 * controller, same stops at the save times) with no mesh stored, returning
 * the accepted state at each save time.
 *   smax     cap on accepted steps and on rejections (GS_TRAJ_MAXSTEPS beyond)
 *   u_save   device [nsave][d][n] dtype, by trajectory; NaN at every save point
 *            of a trajectory whose status is not GS_TRAJ_OK
 *   nsteps   device [n] int32 accepted steps, by trajectory; may be NULL
 *   status   device [n] int32, by trajectory; may be NULL
 * Needs no workspace.  The states equal, bit for bit, those that gs_record
 * followed by gs_solve returns for the same problem and tolerances: the
 * recorder and the replay take each step with the same operations.
 * (GRADSOLVE abstract: the forward-only kernel, the library's second headline
 * use besides gradients.)
 */
GS_API gs_status gs_solve_adaptive(const gs_problem* prob, const gs_tol* tol, int32_t smax, void* u_save,
                                   int32_t* nsteps, int32_t* status, void* stream);

/*
 * gs_solve_adaptive in a given trajectory order: groups of 32 consecutive
 * entries of order (device [n] int32, a permutation of 0..n-1, e.g. the slot
 * order of an earlier gs_record of the ensemble) run side by side in a warp,
 * so an order sorted by step count keeps a warp's lanes on chains of about
 * equal length.  Outputs as gs_solve_adaptive's, indexed by trajectory, bit
 * for bit the same; an entry outside [0, n) is skipped (a trajectory that no
 * entry names gets no output).  ws: device, at least GS_RECORD_INPLACE_WS
 * bytes, 8-byte aligned (a work counter).  Not for GS_NODE64
 * (GS_EUNSUPPORTED).  (The forward-only solver use of the GRADSOLVE
 * abstract, as gs_solve_adaptive.)
 */
GS_API gs_status gs_solve_adaptive_ordered(const gs_problem* prob, const gs_tol* tol, int32_t smax,
                                           const int32_t* order, void* u_save, int32_t* nsteps, int32_t* status,
                                           void* ws, size_t ws_bytes, void* stream);

/*
 * Fused replay + reverse sweep: for every trajectory, the loss of the
 * fixed-step replay on the mesh and its exact discrete adjoint.
 *   loss     device [n] dtype       L_i
 *   dp       device [np][n] dtype   dL_i/dp_i   (GS_NODE64: dL_i/db_i)
 *   du0      device [d][n] dtype    dL_i/du0_i
 *   dshared  device [64][64] dtype, GS_NODE64: sum_i dL_i/dW; else NULL
 *   ws       workspace of gs_workspace_bytes(prob, mesh, GS_OP_GRAD) bytes
 * All indexed by trajectory.  Slots with status != 0 get NaN loss/dp/du0 and
 * do not contribute to dshared.  Built for GS_LORENZ with GS_TSIT5, GS_ROS2
 * or GS_ROS3; GS_ROBERTSON with GS_ROS2 or GS_ROS3 (dense save points
 * included for all of these); GS_LORENZ with GS_VERN7 (landing save points);
 * GS_KIN8 with GS_ROS2 or GS_ROS3 (fp64 and fp32 for all of these);
 * GS_NODE64 with GS_TSIT5
 * in fp32.  Other combinations return GS_EUNSUPPORTED.  (Evolve.pub review,
 * "Summary": the replay is a fixed-length chain without branches, and its
 * backward sweep is the exact discrete adjoint.)
 */
GS_API gs_status gs_grad(const gs_problem* prob, const gs_mesh* mesh, const gs_loss* loss_desc, void* loss, void* dp,
                  void* du0, void* dshared, void* ws, size_t ws_bytes, void* stream);

/*
 * Forward sensitivities on the mesh: the tangent of the fixed-step replay
 * along every input direction -- the np parameters, then the d initial-state
 * components -- integrated alongside the state (forward mode).  The same
 * derivative as gs_grad (of the replay, the mesh held as data), and besides
 * the loss gradient the whole sensitivity matrix at every save point:
 *   sens     device [nsave][d][np + d][n] dtype, by trajectory:
 *            sens[k][c][j][i] = d u_c(t_k) / d theta_j for trajectory i, with
 *            theta = (p_0 .. p_{np-1}, u0_0 .. u0_{d-1}); may be NULL
 *   loss, dp, du0: as gs_grad (dL/dp and dL/du0 by the chain rule through the
 *            tangents)
 * Needs no workspace.  Slots with status != 0 (or whose Rosenbrock matrix
 * turns singular) get NaN everywhere.  Built for GS_LORENZ with GS_TSIT5, and
 * for GS_LORENZ and GS_ROBERTSON with GS_ROS2 or GS_ROS3 (np + d = 6), fp64
 * and fp32, on landing and dense meshes (at a dense save point the matrix is
 * the tangent of the step's dense output); for GS_LORENZ with GS_VERN7 on
 * landing meshes; for GS_KIN8 with GS_ROS2 or GS_ROS3 (np + d = 16) on
 * landing meshes; other problems return
 * GS_EUNSUPPORTED.  (The few-parameter forward-sensitivity
 * route that the gptget summary sets beside the adjoint.)
 */
GS_API gs_status gs_sens(const gs_problem* prob, const gs_mesh* mesh, const gs_loss* loss_desc, void* loss, void* dp,
                         void* du0, void* sens, void* stream);

/*
 * gs_grad without a caller workspace, for callers that cannot allocate device
 * memory (a plugin whose host application owns all device memory, a real-time
 * loop that may not call cudaMalloc, a C host without an allocator).  Same
 * arguments, results and validation as gs_grad, minus ws / ws_bytes: the
 * checkpoints go to a library-owned device array of GS_STATIC_SCRATCH_BYTES
 * (32 MiB), which every GPU that loads the library holds until exit.
 *  - Problems whose gs_grad workspace exceeds GS_STATIC_SCRATCH_BYTES return
 *    GS_EWORKSPACE (d=3, fp64: (smax + nsave) * n <= 1,398,101 for Tsit5 on
 *    Lorenz, (smax + 3 nsave) * n for a dense mesh, smax * n <= 1,398,101 for
 *    the Rosenbrock methods; e.g. 1,024 trajectories of up to 1,355 steps
 *    with 10 save points).
 *  - All calls share the array: calls that overlap on the GPU race.  It keeps
 *    the last call's contents; nothing in it needs clearing between calls.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress)
 *    with the caller's device current, so a context reset between calls is
 *    safe.  The first call on a device also loads the library's module there;
 *    make that first call before any stream capture.
 * No counterpart in the paper.
 */
#define GS_STATIC_SCRATCH_BYTES (32u << 20)
GS_API gs_status gs_grad_static(const gs_problem* prob, const gs_mesh* mesh, const gs_loss* loss_desc, void* loss,
                                void* dp, void* du0, void* dshared, void* stream);

/*
 * Process-wide options (not thread-safe against concurrent calls).
 *   GS_OPT_NODE64_TENSOR_CORES  1 (default): the d = 64 recorder, replay and
 *       gradient compute W U, W^T g and g U^T on the tensor cores (tcgen05,
 *       tf32 with a 3xTF32 split: fp32 accuracy; 128 trajectories per CTA,
 *       one TMEM lane each); 0: with FP32 SIMT products.  Within either form
 *       the recorder and the replay share their arithmetic, so a replay
 *       repeats the recorded states bit for bit; the two forms agree to fp32
 *       rounding (a mesh recorded with one and replayed with the other is
 *       still a valid mesh: the replay is what is differentiated).
 * Returns GS_EINVAL for an unknown option or value.
 */
#define GS_OPT_NODE64_TENSOR_CORES 1
GS_API gs_status gs_set_option(int32_t option, int32_t value);

/* Static description of a status code. */
GS_API const char* gs_status_string(gs_status status);

/* Number of kernels this library has launched since it was loaded
 * (diagnostic for launch accounting; monotone, process-wide). */
GS_API int64_t gs_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GRADSOLVE_H */
