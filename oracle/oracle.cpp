// oracle.cpp -- plain, slow CPU oracle for record-and-replay discrete adjoints.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
// call this file.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
// baseline / reference leg load the shared library built from it.  It shares no
// code with the CUDA library: the step formulas below are written out a second
// time from the method's definition and from the floating-point contract (the
// operation order that both sides follow), not from the kernels.
//
// What it computes (GRADSOLVE, arXiv 2609.02876, abstract and the evolve.pub
// review "Summary" / "Strengths: precisely scoped exactness claim"): an adaptive
// solver records the step sizes it accepts; a fixed-step replay of those steps,
// with the mesh held as data, defines the loss; the gradient is the exact
// derivative of that replay (the discrete adjoint), excluding any derivative of
// the step-size choices.
//
//   record()   the adaptive solve, step by step, plain scalar arithmetic.
//   replay<S>  fixed-step replay over a recorded mesh, generic in the scalar S.
//   grad       reverse-mode AD of replay<S> with a small operator-overloading
//              tape (S = Rv<T>), i.e. the definition "derivative of the replay"
//              written out, not a hand-derived adjoint.
//   dirderiv   forward-mode dual numbers (S = Dv<T>) through the same replay:
//              an independent second route to the same derivative.
//   flops      a counting scalar (S = Cn) to count the replay's operations.
//
// Integrators: Tsitouras' 5(4) pair (Tsit5, Tsitouras 2011), Verner's 7(6)
// pair (Verner 2010), the second-order Rosenbrock method ROS2 of Verwer,
// Spee, Blom & Hundsdorfer (1999) with gamma = 1 + 1/sqrt(2), and the
// third-order Rosenbrock method ROS3 of Sandu, Verwer, Blom, Spee, Carmichael
// & Potra (1997).  Systems: Lorenz (DiffEqGPU "ad" example,
// "Forward-mode automatic differentiation" listing), Robertson kinetics
// (mass-action form of the reaction scheme A->B (k1), 2B->B+C (k2),
// B+C->A+C (k3)), the d=64 shared-weight system tanh(W u + b) - u, and kin8,
// an 8-species stiff mass-action network defined in this library (below; not a
// published test problem) that exercises the Rosenbrock path at d = 8.
//
// Parity pins for every function here live in tests/test_oracle_*.py.
#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <type_traits>
#include <vector>

namespace orc {

// ---------------------------------------------------------------------------
// Scalar types.  Every overload computes its VALUE with exactly the plain-T
// operation (one rounding per +,-,*,/, one per fma), so replay<Rv<T>>,
// replay<Dv<T>> and replay<T> produce bitwise identical forward values.
// ---------------------------------------------------------------------------

// ---- reverse mode: tape of nodes, each with up to three parents -----------
template <class T>
struct Node {
  T v;
  int32_t a, b, c;
  T da, db, dc;
};

template <class T>
struct Tape {
  std::vector<Node<T>> nodes;
  int32_t push(T v, int32_t a = -1, T da = 0, int32_t b = -1, T db = 0, int32_t c = -1, T dc = 0) {
    nodes.push_back(Node<T>{v, a, b, c, da, db, dc});
    return (int32_t)nodes.size() - 1;
  }
};

template <class T>
Tape<T>& tape() {
  static thread_local Tape<T> t;
  return t;
}

// A reverse-mode variable: value plus tape index (-1 = constant, no node).
template <class T>
struct Rv {
  T v;
  int32_t id;
  Rv() : v(0), id(-1) {}
  Rv(T x) : v(x), id(-1) {}  // constants carry no node
  Rv(T x, int32_t i) : v(x), id(i) {}
};

template <class T>
Rv<T> rv_node(T v, int32_t a, T da, int32_t b = -1, T db = 0, int32_t c = -1, T dc = 0) {
  if (a < 0 && b < 0 && c < 0) return Rv<T>(v);
  return Rv<T>(v, tape<T>().push(v, a, da, b, db, c, dc));
}
template <class T> Rv<T> operator+(Rv<T> x, Rv<T> y) { return rv_node<T>(x.v + y.v, x.id, 1, y.id, 1); }
template <class T> Rv<T> operator-(Rv<T> x, Rv<T> y) { return rv_node<T>(x.v - y.v, x.id, 1, y.id, -1); }
template <class T> Rv<T> operator*(Rv<T> x, Rv<T> y) { return rv_node<T>(x.v * y.v, x.id, y.v, y.id, x.v); }
template <class T> Rv<T> operator/(Rv<T> x, Rv<T> y) {
  T q = x.v / y.v;
  return rv_node<T>(q, x.id, T(1) / y.v, y.id, -q / y.v);
}
template <class T> Rv<T> operator-(Rv<T> x) { return rv_node<T>(-x.v, x.id, -1); }
template <class T> Rv<T> fma_(Rv<T> x, Rv<T> y, Rv<T> z) {
  return rv_node<T>(std::fma(x.v, y.v, z.v), x.id, y.v, y.id, x.v, z.id, 1);
}
template <class T> Rv<T> sqrt_(Rv<T> x) {
  T r = std::sqrt(x.v);
  return rv_node<T>(r, x.id, T(0.5) / r);
}
template <class T> Rv<T> tanh_(Rv<T> x) {
  T r = std::tanh(x.v);
  return rv_node<T>(r, x.id, T(1) - r * r);
}
template <class T> T val(Rv<T> x) { return x.v; }

// ---- forward mode: one tangent direction -----------------------------------
template <class T>
struct Dv {
  T v, d;
  Dv() : v(0), d(0) {}
  Dv(T x) : v(x), d(0) {}
  Dv(T x, T dx) : v(x), d(dx) {}
};
template <class T> Dv<T> operator+(Dv<T> x, Dv<T> y) { return Dv<T>(x.v + y.v, x.d + y.d); }
template <class T> Dv<T> operator-(Dv<T> x, Dv<T> y) { return Dv<T>(x.v - y.v, x.d - y.d); }
template <class T> Dv<T> operator*(Dv<T> x, Dv<T> y) { return Dv<T>(x.v * y.v, x.d * y.v + x.v * y.d); }
template <class T> Dv<T> operator/(Dv<T> x, Dv<T> y) {
  T q = x.v / y.v;
  return Dv<T>(q, (x.d - q * y.d) / y.v);
}
template <class T> Dv<T> operator-(Dv<T> x) { return Dv<T>(-x.v, -x.d); }
template <class T> Dv<T> fma_(Dv<T> x, Dv<T> y, Dv<T> z) {
  return Dv<T>(std::fma(x.v, y.v, z.v), x.d * y.v + x.v * y.d + z.d);
}
template <class T> Dv<T> sqrt_(Dv<T> x) {
  T r = std::sqrt(x.v);
  return Dv<T>(r, x.d * (T(0.5) / r));
}
template <class T> Dv<T> tanh_(Dv<T> x) {
  T r = std::tanh(x.v);
  return Dv<T>(r, x.d * (T(1) - r * r));
}
template <class T> T val(Dv<T> x) { return x.v; }

// ---- operation counter ------------------------------------------------------
struct OpCount {
  int64_t add = 0, mul = 0, fma = 0, div = 0, sqrt = 0, tanh = 0;
};
inline OpCount& opcount() {
  static thread_local OpCount c;
  return c;
}
struct Cn {
  double v;
  Cn() : v(0) {}
  Cn(double x) : v(x) {}
};
inline Cn operator+(Cn x, Cn y) { opcount().add++; return Cn(x.v + y.v); }
inline Cn operator-(Cn x, Cn y) { opcount().add++; return Cn(x.v - y.v); }
inline Cn operator*(Cn x, Cn y) { opcount().mul++; return Cn(x.v * y.v); }
inline Cn operator/(Cn x, Cn y) { opcount().div++; return Cn(x.v / y.v); }
inline Cn operator-(Cn x) { return Cn(-x.v); }  // sign flip: not an arithmetic op
inline Cn fma_(Cn x, Cn y, Cn z) { opcount().fma++; return Cn(std::fma(x.v, y.v, z.v)); }
inline Cn sqrt_(Cn x) { opcount().sqrt++; return Cn(std::sqrt(x.v)); }
inline Cn tanh_(Cn x) { opcount().tanh++; return Cn(std::tanh(x.v)); }
inline double val(Cn x) { return x.v; }

// ---- plain scalars -----------------------------------------------------------
inline double fma_(double x, double y, double z) { return std::fma(x, y, z); }
inline float fma_(float x, float y, float z) { return std::fma(x, y, z); }
inline double sqrt_(double x) { return std::sqrt(x); }
inline float sqrt_(float x) { return std::sqrt(x); }
inline double tanh_(double x) { return std::tanh(x); }
inline float tanh_(float x) { return std::tanh(x); }
inline double val(double x) { return x; }
inline float val(float x) { return x; }

template <class S> struct base_of { using type = S; };
template <class T> struct base_of<Rv<T>> { using type = T; };
template <class T> struct base_of<Dv<T>> { using type = T; };
template <> struct base_of<Cn> { using type = double; };

// ---------------------------------------------------------------------------
// Method constants.
// ---------------------------------------------------------------------------
enum { SYS_LORENZ = 1, SYS_ROBERTSON = 2, SYS_HIRES = 3, SYS_NODE64 = 4, SYS_LINEAR = 5, SYS_KIN8 = 6 };
enum { M_TSIT5 = 1, M_ROS2 = 2, M_ROS3 = 3, M_VERN7 = 4 };
enum { DT_F32 = 1, DT_F64 = 2 };
enum { LOSS_SUMSQ = 1, LOSS_LINEAR = 2 };
enum { TRAJ_OK = 0, TRAJ_MAXSTEPS = 1, TRAJ_DTMIN = 2, TRAJ_NONFINITE = 3, TRAJ_SINGULAR = 4 };

// Tsitouras (2011) 5(4) pair.  Row j of TS_A holds a_{j+1, m+1}; row 6 is the
// propagating weight vector b (the method is FSAL: stage 7 is f(u_{n+1})).
// TS_BT holds b - bhat, the weights of the embedded error estimate.
static const double TS_C[7] = {0.0, 0.161, 0.327, 0.9, 0.9800255409045097, 1.0, 1.0};
static const double TS_A[7][6] = {
    {0, 0, 0, 0, 0, 0},
    {0.161, 0, 0, 0, 0, 0},
    {-0.008480655492356989, 0.335480655492357, 0, 0, 0, 0},
    {2.897153057105493, -6.359448489975075, 4.3622954328695815, 0, 0, 0},
    {5.325864828439257, -11.748883564062828, 7.4955393428898365, -0.09249506636175525, 0, 0},
    {5.86145544294642, -12.92096931784711, 8.159367898576159, -0.071584973281401, -0.028269050394068383, 0},
    {0.09646076681806523, 0.01, 0.4798896504144996, 1.379008574103742, -3.290069515436081, 2.324710524099774}};
static const double TS_BT[7] = {-0.00178001105222577714, -0.0008164344596567469, 0.007880878010261995,
                                -0.1447110071732629,     0.5823571654525552,     -0.45808210592918697,
                                1.0 / 66.0};

// Tsitouras' continuous extension of the pair, the dense output of Tsit5
// (save times read off an interpolant instead of being stepped onto: the
// gist.science summary of arXiv 2609.28458, "Methodology", "Dense Output";
// the pages name no interpolant, so the method's own is the reading): the
// state at t_s + theta h is u_s + h sum_i b_i(theta) k_i over the seven
// stages (k_7 = f(u_{s+1})), b_i(theta) = sum_{m=1..4} TS_R[i][m-1] theta^m.
// The values are recalled, not taken from the pages; the pins check that they
// satisfy every fourth-order condition for all theta, equal b at theta = 1
// and make the interpolant C1 across steps (b'(0) = e_1, b'(1) = e_7).
static const double TS_R[7][4] = {
    {1.0, -2.763706197274826, 2.9132554618219126, -1.0530884977290216},
    {0.0, 0.13169999999999998, -0.2234, 0.1017},
    {0.0, 3.9302962368947516, -5.941033872131505, 2.490627285651253},
    {0.0, -12.411077166933676, 30.33818863028232, -16.548102889244902},
    {0.0, 37.50931341651104, -88.1789048947664, 47.37952196281928},
    {0.0, -27.896526289197286, 65.09189467479366, -34.87065786149660},
    {0.0, 1.5, -4.0, 2.5}};

// ROS2 (Verwer et al. 1999): gamma = 1 + 1/sqrt(2), L-stable choice.
static const double ROS2_GAMMA = 1.7071067811865475;  // 1 + 1/sqrt(2) rounded to double

// ROS3 (Sandu et al. 1997, "Benchmarking stiff ODE solvers for atmospheric
// chemistry problems II: Rosenbrock solvers", method ROS3): three stages,
// order 3, L-stable, with an embedded second-order solution.  gamma is the
// root in (1/6, 1/2) of x^3 - 3x^2 + 3/2 x - 1/6.  The coefficients are those
// of the transformed stage form (a_ij, c_ij / h, m_i, e_i); a21 = a31 = 1,
// a32 = 0 and m1 = 1.  Each is the published value rounded to double; 1/gamma
// is rounded once from the exact quotient.
static const double ROS3_GAMMA = 0.435866521508459;
static const double ROS3_INV_GAMMA = 2.294280360279042;
static const double ROS3_C21 = -1.0156171083877703;
static const double ROS3_C31 = 4.07599564525377;
static const double ROS3_C32 = 9.20767942983308;
static const double ROS3_M2 = 6.1697947043828245;
static const double ROS3_M3 = -0.42772256543218573;
static const double ROS3_E1 = 0.5;
static const double ROS3_E2 = -2.907955871680547;
static const double ROS3_E3 = 0.2235406989781157;

// Verner's 7(6) pair (J. H. Verner, "Numerically optimal Runge-Kutta pairs
// with interpolants", Numer. Algorithms 53 (2010); its "most efficient" 7(6)
// pair): ten stages, the seventh-order weights b on stages 1 and 4..9, the
// sixth-order embedded weights bhat on 1, 4..7 and 10 (stage 10 serves only
// the error estimate; the pair is not FSAL).  Row j of V7_A holds a_{j+1, m+1}
// (zeros where the pair has none).  The values are recalled, not taken from
// the pages (the gist.science summary of arXiv 2609.28458, "Results", names
// "Verner 7" beside Tsit5 as the methods compared); the pins check every
// order condition up to order 7 for b and 6 for bhat from these values.
static const double V7_C[10] = {0.0, 0.005, 0.10888888888888888, 0.16333333333333333, 0.4555,
                                0.6095094489978381, 0.884, 0.925, 1.0, 1.0};
static const double V7_A[10][9] = {
    {0, 0, 0, 0, 0, 0, 0, 0, 0},
    {0.005, 0, 0, 0, 0, 0, 0, 0, 0},
    {-1.07679012345679, 1.185679012345679, 0, 0, 0, 0, 0, 0, 0},
    {0.04083333333333333, 0, 0.1225, 0, 0, 0, 0, 0, 0},
    {0.6389139236255726, 0, -2.455672638223657, 2.272258714598084, 0, 0, 0, 0, 0},
    {-2.6615773750187572, 0, 10.804513886456137, -8.3539146573962, 0.820487594956657, 0, 0, 0, 0},
    {6.067741434696772, 0, -24.711273635911088, 20.427517930788895, -1.9061579788166472, 1.006172249242068, 0, 0,
     0},
    {12.054670076253203, 0, -49.75478495046899, 41.142888638604674, -4.461760149974004, 2.042334822239175,
     -0.09834843665406107, 0, 0},
    {10.138146522881808, 0, -42.6411360317175, 35.76384003992257, -4.3480228403929075, 2.0098622683770357,
     0.3487490460338272, -0.27143900510483127, 0},
    {-45.030072034298676, 0, 187.3272437654589, -154.02882369350186, 18.56465306347536, -7.141809679295079,
     1.3088085781613787, 0, 0}};
static const double V7_B[10] = {0.04715561848627222, 0, 0, 0.25750564298434153, 0.26216653977412624,
                                0.15216092656738558, 0.4939969170032485, -0.29430311714032503,
                                0.08131747232495111, 0};
static const double V7_BH[10] = {0.044608606606341174, 0, 0, 0.26716403785713727, 0.22010183001772932,
                                 0.2188431703143157, 0.22898717054112028, 0, 0, 0.02029518466335628};

// Error order q of the step-size controller: the local error estimate of
// Tsit5 is O(h^5), of ROS2 O(h^2), of ROS3 O(h^3), of Verner's 7(6) pair O(h^7).
inline int method_order(int method) {
  return method == M_TSIT5 ? 5 : (method == M_ROS3 ? 3 : (method == M_VERN7 ? 7 : 2));
}

constexpr int DMAX = 64;

// ---------------------------------------------------------------------------
// Right-hand sides.  u: state (d), p: per-trajectory parameters (np),
// W: shared weights (NODE64 only, row-major 64x64).
// ---------------------------------------------------------------------------
template <class S>
void rhs(int sys, const S* u, const S* p, const S* W, S* out) {
  if (sys == SYS_LORENZ) {
    // du1 = sigma (u2 - u1); du2 = u1 (rho - u3) - u2; du3 = u1 u2 - beta u3
    out[0] = p[0] * (u[1] - u[0]);
    out[1] = fma_(u[0], p[1] - u[2], -u[1]);
    out[2] = fma_(u[0], u[1], -(p[2] * u[2]));
  } else if (sys == SYS_ROBERTSON) {
    // rates r1 = k1 y1, r2 = k2 y2^2, r3 = k3 y2 y3
    S r1 = p[0] * u[0];
    S r2 = p[1] * (u[1] * u[1]);
    S r3 = p[2] * (u[1] * u[2]);
    out[0] = r3 - r1;
    out[1] = (r1 - r3) - r2;
    out[2] = r2;
  } else if (sys == SYS_LINEAR) {
    // scalar test equation u' = p u (pins only: closed forms exist)
    out[0] = p[0] * u[0];
  } else if (sys == SYS_KIN8) {
    // kin8: species A1..A8 (u[0..7]), rate constants p[0..7], mass action for
    //   A1 -> A2, A2 -> A1, A2 + A3 -> A4, A4 -> A3 + A5,
    //   A5 -> A6, A6 -> A5, A6 + A7 -> A8, A8 -> A7 + A1,
    // i.e. f = N r(u) with the stoichiometric matrix N of these eight
    // reactions.  u1+u2+u4+u5+u6+u8, u3+u4 and u7+u8 are conserved.
    S r1 = p[0] * u[0];
    S r2 = p[1] * u[1];
    S r3 = p[2] * (u[1] * u[2]);
    S r4 = p[3] * u[3];
    S r5 = p[4] * u[4];
    S r6 = p[5] * u[5];
    S r7 = p[6] * (u[5] * u[6]);
    S r8 = p[7] * u[7];
    out[0] = (r2 - r1) + r8;
    out[1] = (r1 - r2) - r3;
    out[2] = r4 - r3;
    out[3] = r3 - r4;
    out[4] = (r4 - r5) + r6;
    out[5] = (r5 - r6) - r7;
    out[6] = r8 - r7;
    out[7] = r7 - r8;
  } else if (sys == SYS_NODE64) {
    for (int r = 0; r < 64; ++r) {
      S acc = p[r];
      for (int c = 0; c < 64; ++c) acc = fma_(W[r * 64 + c], u[c], acc);
      out[r] = tanh_(acc) - u[r];
    }
  }
}

// Analytic Jacobian df/du, row-major d x d (Rosenbrock path).
template <class S>
void jac(int sys, const S* u, const S* p, S* J) {
  if (sys == SYS_ROBERTSON) {
    S a = p[2] * u[2];           // k3 y3
    S b = p[2] * u[1];           // k3 y2
    S c = S(2) * (p[1] * u[1]);  // 2 k2 y2
    J[0] = -p[0];
    J[1] = a;
    J[2] = b;
    J[3] = p[0];
    J[4] = -(a + c);
    J[5] = -b;
    J[6] = S(0);
    J[7] = c;
    J[8] = S(0);
  } else if (sys == SYS_LINEAR) {
    J[0] = p[0];
  } else if (sys == SYS_KIN8) {
    for (int q = 0; q < 64; ++q) J[q] = S(0);
    S a = p[2] * u[2];  // k3 y3
    S b = p[2] * u[1];  // k3 y2
    S c = p[6] * u[6];  // k7 y7
    S e = p[6] * u[5];  // k7 y6
    J[0 * 8 + 0] = -p[0];
    J[0 * 8 + 1] = p[1];
    J[0 * 8 + 7] = p[7];
    J[1 * 8 + 0] = p[0];
    J[1 * 8 + 1] = -(p[1] + a);
    J[1 * 8 + 2] = -b;
    J[2 * 8 + 1] = -a;
    J[2 * 8 + 2] = -b;
    J[2 * 8 + 3] = p[3];
    J[3 * 8 + 1] = a;
    J[3 * 8 + 2] = b;
    J[3 * 8 + 3] = -p[3];
    J[4 * 8 + 3] = p[3];
    J[4 * 8 + 4] = -p[4];
    J[4 * 8 + 5] = p[5];
    J[5 * 8 + 4] = p[4];
    J[5 * 8 + 5] = -(p[5] + c);
    J[5 * 8 + 6] = -e;
    J[6 * 8 + 5] = -c;
    J[6 * 8 + 6] = -e;
    J[6 * 8 + 7] = p[7];
    J[7 * 8 + 5] = c;
    J[7 * 8 + 6] = e;
    J[7 * 8 + 7] = -p[7];
  } else if (sys == SYS_LORENZ) {
    J[0] = -p[0];
    J[1] = p[0];
    J[2] = S(0);
    J[3] = p[1] - u[2];
    J[4] = S(-1);
    J[5] = -u[0];
    J[6] = u[1];
    J[7] = u[0];
    J[8] = -p[2];
  }
}

// ---------------------------------------------------------------------------
// One Tsit5 step of size h from u.  Stage j state: acc = a_j1 k1 + sum a_jm k_m
// (an fma chain in increasing m), U_j = fma(h, acc, u).  u_new is stage 7.
// If err != nullptr also returns the embedded error e = h * sum bt_j k_j.
// ---------------------------------------------------------------------------
template <class S>
void tsit5_step(int sys, int d, const S* u, const S* p, const S* W, S h, S* unew, S* err) {
  using T = typename base_of<S>::type;
  S k[7][DMAX];
  S U[DMAX];
  rhs<S>(sys, u, p, W, k[0]);
  for (int j = 1; j < 7; ++j) {
    for (int c = 0; c < d; ++c) {
      S acc = S(T(TS_A[j][0])) * k[0][c];
      for (int m = 1; m < j; ++m) acc = fma_(S(T(TS_A[j][m])), k[m][c], acc);
      U[c] = fma_(h, acc, u[c]);
    }
    if (j == 6) {
      for (int c = 0; c < d; ++c) unew[c] = U[c];
      if (!err) return;  // replay: the FSAL stage is the next step's first stage
    }
    rhs<S>(sys, U, p, W, k[j]);
  }
  for (int c = 0; c < d; ++c) {
    S acc = S(T(TS_BT[0])) * k[0][c];
    for (int m = 1; m < 7; ++m) acc = fma_(S(T(TS_BT[m])), k[m][c], acc);
    err[c] = h * acc;
  }
}

// ---------------------------------------------------------------------------
// LU with partial pivoting (largest |entry|, ties to the lowest row), Doolittle
// right-looking order; multipliers stored below the diagonal.  Each pivot's
// reciprocal is formed once (one division) and the multipliers and the back
// substitution multiply by it.  Returns false on an exactly zero or
// non-finite pivot.
// ---------------------------------------------------------------------------
template <class S>
bool lu_factor(int d, S* M, int* P, S* R) {
  using T = typename base_of<S>::type;
  for (int i = 0; i < d; ++i) P[i] = i;
  for (int k = 0; k < d; ++k) {
    int piv = k;
    for (int i = k + 1; i < d; ++i)
      if (std::fabs(val(M[i * d + k])) > std::fabs(val(M[piv * d + k]))) piv = i;
    if (piv != k) {
      for (int j = 0; j < d; ++j) std::swap(M[k * d + j], M[piv * d + j]);
      std::swap(P[k], P[piv]);
    }
    T pv = val(M[k * d + k]);
    if (pv == T(0) || !std::isfinite(pv)) return false;
    R[k] = S(T(1)) / M[k * d + k];
    for (int i = k + 1; i < d; ++i) {
      S l = M[i * d + k] * R[k];
      M[i * d + k] = l;
      for (int j = k + 1; j < d; ++j) M[i * d + j] = fma_(-l, M[k * d + j], M[i * d + j]);
    }
  }
  return true;
}

template <class S>
void lu_solve(int d, const S* LU, const int* P, const S* R, const S* b, S* x) {
  for (int i = 0; i < d; ++i) x[i] = b[P[i]];
  for (int i = 1; i < d; ++i)
    for (int j = 0; j < i; ++j) x[i] = fma_(-LU[i * d + j], x[j], x[i]);
  for (int i = d - 1; i >= 0; --i) {
    for (int j = i + 1; j < d; ++j) x[i] = fma_(-LU[i * d + j], x[j], x[i]);
    x[i] = x[i] * R[i];
  }
}

// ---------------------------------------------------------------------------
// One ROS2 step (Verwer et al. 1999):
//   M = I - gamma h J(u);  M k1 = f(u);  M k2 = f(u + h k1) - 2 k1;
//   u_new = u + h (3/2 k1 + 1/2 k2);  error e = h/2 (k1 + k2)
// (difference to the embedded first-order solution u + h k1).
// Returns false when M is singular.
// ---------------------------------------------------------------------------
template <class S>
bool ros2_step(int sys, int d, const S* u, const S* p, S h, S* unew, S* err) {
  using T = typename base_of<S>::type;
  S J[64];
  S M[64], R[8];
  int P[8];
  jac<S>(sys, u, p, J);
  S gh = S(T(ROS2_GAMMA)) * h;
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) M[i * d + j] = fma_(-gh, J[i * d + j], S(T(i == j ? 1 : 0)));
  if (!lu_factor<S>(d, M, P, R)) return false;
  S f0[8] = {}, k1[8] = {}, v[8] = {}, f1[8] = {}, r[8] = {}, k2[8] = {};
  rhs<S>(sys, u, p, nullptr, f0);
  lu_solve<S>(d, M, P, R, f0, k1);
  for (int c = 0; c < d; ++c) v[c] = fma_(h, k1[c], u[c]);
  rhs<S>(sys, v, p, nullptr, f1);
  for (int c = 0; c < d; ++c) r[c] = fma_(S(T(-2)), k1[c], f1[c]);
  lu_solve<S>(d, M, P, R, r, k2);
  for (int c = 0; c < d; ++c) {
    S acc = S(T(1.5)) * k1[c];
    acc = fma_(S(T(0.5)), k2[c], acc);
    unew[c] = fma_(h, acc, u[c]);
  }
  if (err)
    for (int c = 0; c < d; ++c) err[c] = (h * S(T(0.5))) * (k1[c] + k2[c]);
  return true;
}

// ---------------------------------------------------------------------------
// One ROS3 step (Sandu et al. 1997), with k_i = K_i / h of the paper's
// transformed form (K_i are the paper's stage increments):
//   M = I/gamma - h J(u);  M k1 = f(u);  v = u + h k1;
//   M k2 = f(v) + c21 k1;  M k3 = f(v) + c31 k1 + c32 k2
//   (a31 = a21 = 1 and a32 = 0, so stage 3 evaluates f at the same point as
//   stage 2);  u_new = u + h (k1 + m2 k2 + m3 k3);
//   error e = h (e1 k1 + e2 k2 + e3 k3)  (u_new minus the embedded solution).
// Returns false when M is singular.
// ---------------------------------------------------------------------------
template <class S>
bool ros3_step(int sys, int d, const S* u, const S* p, S h, S* unew, S* err) {
  using T = typename base_of<S>::type;
  S J[64];
  S M[64], R[8];
  int P[8];
  jac<S>(sys, u, p, J);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) M[i * d + j] = fma_(-h, J[i * d + j], S(T(i == j ? ROS3_INV_GAMMA : 0.0)));
  if (!lu_factor<S>(d, M, P, R)) return false;
  S f0[8] = {}, k1[8] = {}, v[8] = {}, f1[8] = {}, r[8] = {}, k2[8] = {}, k3[8] = {};
  rhs<S>(sys, u, p, nullptr, f0);
  lu_solve<S>(d, M, P, R, f0, k1);
  for (int c = 0; c < d; ++c) v[c] = fma_(h, k1[c], u[c]);
  rhs<S>(sys, v, p, nullptr, f1);
  for (int c = 0; c < d; ++c) r[c] = fma_(S(T(ROS3_C21)), k1[c], f1[c]);
  lu_solve<S>(d, M, P, R, r, k2);
  for (int c = 0; c < d; ++c) r[c] = fma_(S(T(ROS3_C32)), k2[c], fma_(S(T(ROS3_C31)), k1[c], f1[c]));
  lu_solve<S>(d, M, P, R, r, k3);
  for (int c = 0; c < d; ++c) {
    S acc = fma_(S(T(ROS3_M3)), k3[c], fma_(S(T(ROS3_M2)), k2[c], k1[c]));
    unew[c] = fma_(h, acc, u[c]);
  }
  if (err)
    for (int c = 0; c < d; ++c)
      err[c] = h * fma_(S(T(ROS3_E3)), k3[c], fma_(S(T(ROS3_E2)), k2[c], S(T(ROS3_E1)) * k1[c]));
  return true;
}

// One step of Verner's 7(6) pair of size h from u.  Stage j state:
// acc = a_j1 k1, then acc = fma(a_jm, k_m, acc) over the nonzero a_jm in
// increasing m, U_j = fma(h, acc, u); u_new the same over the nonzero b_m.
// If err != nullptr, stage 10 is formed too and the embedded error is
// e = h * (E_1 k_1 + sum over the nonzero E_m, increasing m), E = b - bhat
// (each a double difference of the two stored weights).
template <class S>
void vern7_step(int sys, int d, const S* u, const S* p, const S* W, S h, S* unew, S* err) {
  using T = typename base_of<S>::type;
  S k[10][DMAX];
  S U[DMAX];
  rhs<S>(sys, u, p, W, k[0]);
  const int nst = err ? 10 : 9;
  for (int j = 1; j < nst; ++j) {
    for (int c = 0; c < d; ++c) {
      S acc = S(T(V7_A[j][0])) * k[0][c];
      for (int m = 1; m < j; ++m)
        if (V7_A[j][m] != 0.0) acc = fma_(S(T(V7_A[j][m])), k[m][c], acc);
      U[c] = fma_(h, acc, u[c]);
    }
    rhs<S>(sys, U, p, W, k[j]);
  }
  for (int c = 0; c < d; ++c) {
    S acc = S(T(V7_B[0])) * k[0][c];
    for (int m = 1; m < 9; ++m)
      if (V7_B[m] != 0.0) acc = fma_(S(T(V7_B[m])), k[m][c], acc);
    unew[c] = fma_(h, acc, u[c]);
  }
  if (!err) return;
  for (int c = 0; c < d; ++c) {
    S acc = S(T(V7_B[0] - V7_BH[0])) * k[0][c];
    for (int m = 1; m < 10; ++m) {
      const double e = V7_B[m] - V7_BH[m];
      if (e != 0.0) acc = fma_(S(T(e)), k[m][c], acc);
    }
    err[c] = h * acc;
  }
}

// One step of the given method (Tsit5 never fails).
template <class S>
bool method_step(int sys, int method, int d, const S* u, const S* p, const S* W, S h, S* unew, S* err) {
  if (method == M_TSIT5) {
    tsit5_step<S>(sys, d, u, p, W, h, unew, err);
    return true;
  }
  if (method == M_VERN7) {
    vern7_step<S>(sys, d, u, p, W, h, unew, err);
    return true;
  }
  if (method == M_ROS3) return ros3_step<S>(sys, d, u, p, h, unew, err);
  return ros2_step<S>(sys, d, u, p, h, unew, err);
}

// ---------------------------------------------------------------------------
// Logarithm and exponential for the step-size controller, computed from IEEE
// +, -, *, /, fma and the exact frexp / ldexp / rint only, so that any
// implementation keeping this operation order gets the same bits (a library
// pow may differ by an ulp, and the embedded error estimate amplifies such
// differences within a few steps).  The controller's powers are
// x^y = ctrl_exp(y ctrl_ln(x)).
//   ln x : x = m 2^e with m in [sqrt(1/2), sqrt(2)); ln m = 2 atanh(s),
//          s = (m-1)/(m+1), by the series s (1 + z/3 + ... + z^12/25), z = s^2.
//   exp w: Cody & Waite reduction w = k ln2 + r (ln2 split in a 21-bit head and
//          a tail), |r| <= ln2/2, Taylor polynomial to r^14, then 2^k exactly.
// Both polynomials are evaluated by Horner's rule with fused multiply-adds.
// ---------------------------------------------------------------------------
static const double CP_LN2_HI = 0.6931467056274414;      // ln 2, 21 significant bits
static const double CP_LN2_LO = 4.7493250390316726e-07;  // ln 2 - CP_LN2_HI
static const double CP_INV_LN2 = 1.4426950408889634;
static const double CP_SQRT_HALF = 0.7071067811865476;

template <class T>
T ctrl_ln(T x) {  // x > 0 finite
  int e = 0;
  T m = std::frexp(x, &e);
  if (m < T(CP_SQRT_HALF)) {
    m = m + m;
    e = e - 1;
  }
  T s = (m - T(1)) / (m + T(1));
  T z = s * s;
  // sum_{k=0..12} z^k / (2k+1) by Estrin's scheme: pairs in z, then z^2,
  // z^4, z^8 (four dependent levels instead of twelve)
  auto c = [](int k) { return T(1.0 / double(2 * k + 1)); };
  const T z2 = z * z, z4 = z2 * z2, z8 = z4 * z4;
  const T q0 = std::fma(c(1), z, c(0)), q1 = std::fma(c(3), z, c(2)), q2 = std::fma(c(5), z, c(4));
  const T q3 = std::fma(c(7), z, c(6)), q4 = std::fma(c(9), z, c(8)), q5 = std::fma(c(11), z, c(10));
  const T r0 = std::fma(q1, z2, q0), r1 = std::fma(q3, z2, q2), r2 = std::fma(q5, z2, q4);
  const T s0 = std::fma(r1, z4, r0), s1 = std::fma(c(12), z4, r2);
  T poly = std::fma(s1, z8, s0);
  T lnm = (s + s) * poly;
  return std::fma(T(e), T(CP_LN2_HI), std::fma(T(e), T(CP_LN2_LO), lnm));
}

template <class T>
T ctrl_exp(T w) {
  if (std::isnan(w)) return w;
  T kf = std::rint(w * T(CP_INV_LN2));
  if (kf > T(2000)) return std::numeric_limits<T>::infinity();
  if (kf < T(-2000)) return T(0);
  T r = std::fma(-kf, T(CP_LN2_HI), w);
  r = std::fma(-kf, T(CP_LN2_LO), r);
  // sum_{j=0..14} r^j / j! by Estrin's scheme: pairs in r, then r^2, r^4,
  // r^8 (four dependent levels instead of fourteen); j! is exact in double
  auto d = [](int j) {
    double f = 1.0;
    for (int i = 2; i <= j; ++i) f *= double(i);
    return T(1.0 / f);
  };
  const T r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
  T q[7];
  for (int i = 0; i < 7; ++i) q[i] = std::fma(d(2 * i + 1), r, d(2 * i));
  const T t0 = std::fma(q[1], r2, q[0]), t1 = std::fma(q[3], r2, q[2]), t2 = std::fma(q[5], r2, q[4]);
  const T t3 = std::fma(d(14), r2, q[6]);
  const T u0 = std::fma(t1, r4, t0), u1 = std::fma(t3, r4, t2);
  const T p = std::fma(u1, r8, u0);
  return std::ldexp(p, int(kf));
}

template <class T>
T ctrl_pow(T x, T y) {
  if (std::isnan(x) || std::isnan(y)) return std::numeric_limits<T>::quiet_NaN();
  if (x == T(0)) return y > T(0) ? T(0) : (y < T(0) ? std::numeric_limits<T>::infinity() : T(1));
  if (std::isinf(x)) return y > T(0) ? x : (y < T(0) ? T(0) : T(1));
  return ctrl_exp<T>(y * ctrl_ln<T>(x));
}

// ---------------------------------------------------------------------------
// Adaptive recorder (plain scalar T).
//
// Error norm: err = sqrt( (1/d) sum_c (e_c / sc_c)^2 ), sc_c = atol + rtol *
// max(|u_c|, |u_new_c|), accept iff err <= 1.  PI controller with error order
// q (5 for Tsit5, 2 for ROS2, 3 for ROS3): accepted -> fac = 0.9 err^(-0.7/q)
// errprev^(0.4/q) clipped to [0.2, 10] (10 if err == 0), capped at 1 after a
// rejection, errprev <- max(err, 1e-4); rejected -> fac = max(0.2, 0.9
// err^(-1/q)) (0.2 if err is NaN or infinite).  The next proposal is fac * h_prop, where
// h_prop is the unclipped proposal.  Steps are shortened to land exactly on
// every save time and on t1; save_idx[k] is the number of accepted steps taken
// when t reached tsave[k].  Starting step: Hairer, Norsett & Wanner I, II.4.
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Dense output of the Rosenbrock methods between the ends of one step (save
// points that steps do not land on): the cubic Hermite interpolant on
// [t_s, t_s + h] at theta in (0, 1],
//   u(theta) = H00 u_s + H01 u_{s+1} + h (H10 f(u_s) + H11 f(u_{s+1})),
//   H01 = theta^2 (3 - 2 theta),  H00 = 1 - H01,
//   H10 = theta (1 - theta)^2,    H11 = -theta^2 (1 - theta),
// the weights and the combination in this operation order.  theta is data
// (no derivative), like h.
// ---------------------------------------------------------------------------
template <class S>
void hermite(int d, const S* us, const S* un, const S* fs, const S* fn, S h, double theta, S* out) {
  using T = typename base_of<S>::type;
  const T th = T(theta);
  const T t2 = th * th, om = T(1) - th;
  const T H01 = t2 * std::fma(T(-2), th, T(3));
  const T H00 = T(1) - H01;
  const T H10 = (th * om) * om;
  const T H11 = -(t2 * om);
  for (int c = 0; c < d; ++c) out[c] = fma_(S(H00), us[c], fma_(S(H01), un[c], h * fma_(S(H10), fs[c], S(H11) * fn[c])));
}

// Tsit5's dense output at theta in (0, 1) inside a step of size h from u_s:
// the stages are recomputed from u_s exactly as tsit5_step forms them (stage 7
// is the step's end u_{s+1}, k_7 = f(u_{s+1})), then
//   b_1 = fma(theta^2, P_1, theta),  b_i = theta^2 P_i (i >= 2),
//   P_i = fma(fma(r_i4, theta, r_i3), theta, r_i2),
//   u(theta) = fma(h, b_1 k_1 + b_2 k_2 + ... + b_7 k_7, u_s),
// the weights in T and the sum an fma chain in increasing i.  theta is data.
template <class T>
void tsit5_dense_weights(T th, T* bw) {
  const T t2 = th * th;
  for (int i = 0; i < 7; ++i) {
    const T P = std::fma(std::fma(T(TS_R[i][3]), th, T(TS_R[i][2])), th, T(TS_R[i][1]));
    bw[i] = i == 0 ? std::fma(t2, P, th) : t2 * P;
  }
}

template <class S>
void tsit5_dense(int sys, int d, const S* us, const S* p, const S* W, S h, double theta, S* out) {
  using T = typename base_of<S>::type;
  T bw[7];
  tsit5_dense_weights<T>(T(theta), bw);
  S k[7][DMAX];
  S U[DMAX];
  rhs<S>(sys, us, p, W, k[0]);
  for (int j = 1; j < 7; ++j) {
    for (int c = 0; c < d; ++c) {
      S acc = S(T(TS_A[j][0])) * k[0][c];
      for (int m = 1; m < j; ++m) acc = fma_(S(T(TS_A[j][m])), k[m][c], acc);
      U[c] = fma_(h, acc, us[c]);
    }
    rhs<S>(sys, U, p, W, k[j]);
  }
  for (int c = 0; c < d; ++c) {
    S acc = S(bw[0]) * k[0][c];
    for (int m = 1; m < 7; ++m) acc = fma_(S(bw[m]), k[m][c], acc);
    out[c] = fma_(h, acc, us[c]);
  }
}

// The dense output of a step of the given method at theta in (0, 1): Tsit5's
// own continuous extension, the cubic Hermite interpolant for the Rosenbrock
// methods (f evaluated at both ends).
template <class S>
void dense_value(int sys, int method, int d, const S* us, const S* un, const S* p, const S* W, S h, double theta,
                 S* out) {
  if (method == M_TSIT5) {
    tsit5_dense<S>(sys, d, us, p, W, h, theta, out);
    return;
  }
  S fs[DMAX], fn[DMAX];
  rhs<S>(sys, us, p, W, fs);
  rhs<S>(sys, un, p, W, fn);
  hermite<S>(d, us, un, fs, fn, h, theta, out);
}

template <class T>
struct RecordOut {
  std::vector<T> h;
  int nsteps = 0, nreject = 0, status = TRAJ_OK;
  std::vector<int> save_idx;
  std::vector<T> usave;  // [nsave][d]: the accepted state at each save time (the forward-only solve)
  std::vector<T> theta;  // [nsave]: dense mode, position of each save time inside its step (else 1)
};

template <class T>
T rms_scaled(int d, const T* x, const T* sc) {
  T s = 0;
  for (int c = 0; c < d; ++c) {
    T q = x[c] / sc[c];
    s = std::fma(q, q, s);
  }
  return std::sqrt(s / T(d));
}

template <class T>
T initial_step(int sys, int method, int d, const T* u0, const T* p, const T* W, T t0, T t1, T rtol,
               T atol) {
  T q = T(method_order(method));
  T sc[DMAX] = {}, f0[DMAX] = {}, u1[DMAX] = {}, f1[DMAX] = {}, df[DMAX] = {};
  for (int c = 0; c < d; ++c) sc[c] = std::fma(rtol, std::fabs(u0[c]), atol);
  rhs<T>(sys, u0, p, W, f0);
  T d0 = rms_scaled<T>(d, u0, sc);
  T d1 = rms_scaled<T>(d, f0, sc);
  T h0 = (d0 < T(1e-5) || d1 < T(1e-5)) ? T(1e-6) : T(0.01) * (d0 / d1);
  h0 = std::min(h0, t1 - t0);
  for (int c = 0; c < d; ++c) u1[c] = std::fma(h0, f0[c], u0[c]);
  rhs<T>(sys, u1, p, W, f1);
  for (int c = 0; c < d; ++c) df[c] = f1[c] - f0[c];
  T d2 = rms_scaled<T>(d, df, sc) / h0;
  T dm = std::max(d1, d2);
  T h1 = dm <= T(1e-15) ? std::max(T(1e-6), h0 * T(1e-3)) : ctrl_pow<T>(T(0.01) / dm, T(1) / q);
  return std::min(std::min(T(100) * h0, h1), t1 - t0);
}

// The PI factor after an accepted step with scaled error err (error order q):
// 0.9 exp(-(0.7/q) ln err + (0.4/q) ln errprev) clipped to [0.2, 10], 10 if
// err == 0; lnprev carries ln(errprev) (errprev floored at 1e-4) and is
// updated here.  The cap at 1 after a rejection is the caller's.
template <class T>
T accept_factor(T err, T q, T& lnprev) {
  const T ln_floor = ctrl_ln<T>(T(1e-4));
  T fac, lnerr = ln_floor;
  if (err == T(0)) {
    fac = T(10);
  } else {
    lnerr = ctrl_ln<T>(err);
    fac = T(0.9) * ctrl_exp<T>(std::fma(-T(0.7) / q, lnerr, (T(0.4) / q) * lnprev));
    fac = std::min(T(10), std::max(T(0.2), fac));
  }
  lnprev = err < T(1e-4) ? ln_floor : lnerr;
  return fac;
}

template <class T>
RecordOut<T> record_one(int sys, int method, int d, const T* u0, const T* p, const T* W, T t0, T t1,
                        int nsave, const T* tsave, T rtol, T atol, T h0user, int smax, bool dense = false) {
  // dense: steps stop only at t1; a save time inside a step is located by its
  // position theta in (0, 1] and read off the step's dense output
  RecordOut<T> out;
  out.save_idx.assign(nsave, 0);
  out.theta.assign(nsave, T(1));
  out.usave.assign((size_t)nsave * d, std::numeric_limits<T>::quiet_NaN());
  const T eps = std::numeric_limits<T>::epsilon();
  const T q = T(method_order(method));
  T u[DMAX], un[DMAX], e[DMAX], sc[DMAX], f0[DMAX];
  for (int c = 0; c < d; ++c) u[c] = u0[c];
  rhs<T>(sys, u, p, W, f0);
  for (int c = 0; c < d; ++c)
    if (!std::isfinite(f0[c]) || !std::isfinite(u[c])) {
      out.status = TRAJ_NONFINITE;
      return out;
    }
  T hprop = h0user > T(0) ? h0user : initial_step<T>(sys, method, d, u0, p, W, t0, t1, rtol, atol);
  if (!(hprop > T(0)) || !std::isfinite(hprop)) {
    out.status = TRAJ_NONFINITE;
    return out;
  }
  // the controller carries ln(errprev); errprev starts at 1 and is floored at 1e-4
  T t = t0, lnprev = T(0);
  bool prev_rej = false;
  int kk = 0;
  while (true) {
    T tstop = (kk < nsave && !dense) ? tsave[kk] : t1;
    if (hprop < T(16) * eps * std::fabs(t)) {
      out.status = TRAJ_DTMIN;
      return out;
    }
    // a step that would end at or within 4 eps of the next stop lands on it
    T tn = t + hprop;
    bool clipped = tn >= tstop - T(4) * eps * std::fabs(tstop);
    T h = clipped ? tstop - t : hprop;
    bool ok = method_step<T>(sys, method, d, u, p, W, h, un, e);
    if (!ok) {
      out.status = TRAJ_SINGULAR;
      return out;
    }
    for (int c = 0; c < d; ++c) sc[c] = std::fma(rtol, std::max(std::fabs(u[c]), std::fabs(un[c])), atol);
    T err = rms_scaled<T>(d, e, sc);
    if (err <= T(1)) {
      if (out.nsteps >= smax) {
        out.status = TRAJ_MAXSTEPS;
        return out;
      }
      out.h.push_back(h);
      out.nsteps++;
      const T tprev = t;
      t = clipped ? tstop : tn;
      if (dense) {
        while (kk < nsave && tsave[kk] <= t) {
          const T th = (tsave[kk] - tprev) / h;
          out.theta[kk] = th;
          T ut[DMAX] = {};
          if (th != T(1)) dense_value<T>(sys, method, d, u, un, p, W, h, double(th), ut);
          for (int c = 0; c < d; ++c) out.usave[(size_t)kk * d + c] = th == T(1) ? un[c] : ut[c];
          out.save_idx[kk++] = out.nsteps;
        }
      }
      for (int c = 0; c < d; ++c) u[c] = un[c];
      while (!dense && kk < nsave && t == tsave[kk]) {
        for (int c = 0; c < d; ++c) out.usave[(size_t)kk * d + c] = u[c];
        out.save_idx[kk++] = out.nsteps;
      }
      // fac = 0.9 err^(-0.7/q) errprev^(0.4/q) = 0.9 exp(-(0.7/q) ln err + (0.4/q) ln errprev)
      T fac = accept_factor<T>(err, q, lnprev);
      if (prev_rej) fac = std::min(fac, T(1));
      prev_rej = false;
      hprop = fac * hprop;
      if (t >= t1) return out;  // the last step lands exactly on t1
    } else {
      out.nreject++;
      if (out.nreject > smax) {
        out.status = TRAJ_MAXSTEPS;
        return out;
      }
      T fac = !std::isfinite(err) ? T(0.2)
                                  : std::max(T(0.2), T(0.9) * ctrl_exp<T>((-T(1) / q) * ctrl_ln<T>(err)));
      hprop = fac * hprop;
      prev_rej = true;
    }
  }
}

// ---------------------------------------------------------------------------
// Fixed-step replay over a recorded mesh, returning the loss.
//   SUMSQ:  L = sum_k sum_c (u_c(t_k) - target_kc)^2    (target NULL -> 0)
//   LINEAR: L = sum_k sum_c w_kc u_c(t_k)
// accumulated as an fma chain in (k, c) order.  The mesh h is data: no
// derivative flows through it.
// ---------------------------------------------------------------------------
template <class S>
S replay_loss(int sys, int method, int d, const S* u0, const S* p, const S* W, const double* h, int nsteps,
              int nsave, const int* save_idx, int loss_kind, const double* tgt /*[nsave][d] or null*/,
              const double* wgt /*[nsave][d]*/, S* u_save /*[nsave][d] or null*/,
              const double* theta = nullptr /*[nsave] or null: save points at step ends*/) {
  using T = typename base_of<S>::type;
  S u[DMAX], un[DMAX], up[DMAX];
  for (int c = 0; c < d; ++c) u[c] = u0[c];
  S L = S(T(0));
  int kk = 0;
  // save points reached when s steps are taken; up = u_{s-1}, hs = h[s-1]
  auto visit = [&](int s, S hs) {
    while (kk < nsave && save_idx[kk] == s) {
      S ut[DMAX];
      const S* uk = u;
      if (theta && theta[kk] != 1.0 && s > 0) {
        dense_value<S>(sys, method, d, up, u, p, W, hs, theta[kk], ut);
        uk = ut;
      }
      for (int c = 0; c < d; ++c) {
        if (u_save) u_save[kk * d + c] = uk[c];
        if (loss_kind == LOSS_SUMSQ) {
          S dlt = tgt ? uk[c] - S(T(tgt[kk * d + c])) : uk[c];
          L = fma_(dlt, dlt, L);
        } else {
          L = fma_(S(T(wgt[kk * d + c])), uk[c], L);
        }
      }
      kk++;
    }
  };
  visit(0, S(T(0)));
  for (int s = 0; s < nsteps; ++s) {
    S hs = S(T(h[s]));
    method_step<S>(sys, method, d, u, p, W, hs, un, nullptr);
    for (int c = 0; c < d; ++c) {
      up[c] = u[c];
      u[c] = un[c];
    }
    visit(s + 1, hs);
  }
  return L;
}

// ---------------------------------------------------------------------------
// Problem description shared by the entry points below.
// ---------------------------------------------------------------------------
struct Prob {
  int sys, method, dtype, d, np;
  int64_t n;
  const double *p, *u0, *W;  // [np][n], [d][n], [64*64]
};

struct Mesh {
  int smax, nsave;
  const double* h;      // [n][smax]
  const int* nsteps;    // [n]
  const int* save_idx;  // [n][nsave]
  const double* theta = nullptr;  // [n][nsave] dense-output positions, or null (save points at step ends)
  const double* theta_of(int64_t i) const { return theta ? theta + i * nsave : nullptr; }
};

struct Loss {
  int kind;
  const double *target, *weight;  // [nsave][d][n] each (target may be null)
};

template <class F>
void parallel_for(int64_t n, int nthreads, F fn) {
  if (nthreads <= 1 || n < 2) {
    fn(0, (int64_t)0, n);
    return;
  }
  nthreads = (int)std::min<int64_t>(nthreads, n);
  std::vector<std::thread> th;
  int64_t chunk = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    int64_t a = t * chunk, b = std::min(n, a + chunk);
    if (a >= b) break;
    th.emplace_back([=] { fn(t, a, b); });
  }
  for (auto& x : th) x.join();
}

// Per-trajectory gathers of target/weight rows into [nsave][d].
inline void gather_kd(const double* src, int nsave, int d, int64_t n, int64_t i, double* dst) {
  for (int k = 0; k < nsave; ++k)
    for (int c = 0; c < d; ++c) dst[k * d + c] = src[((int64_t)k * d + c) * n + i];
}

// Reverse-mode gradient of one trajectory with the tape.  Outputs: loss, dp
// (np), du0 (d) and, for NODE64, accumulates dW (64*64) into dW_acc.
// A = the type the reverse sweep accumulates adjoints in (T, or long double
// for a reference with 11 more bits; the tape's partials are the same).
// FUSED: each adjoint update adj[parent] += partial * adj[node] as one fused
// multiply-add (one rounding instead of two): the same derivative evaluated
// with different rounding, a third plain-precision route beside the tape and
// the dual numbers (used to gauge how much rounding costs on a trajectory).
template <class T, class A = T, bool FUSED = false>
void grad_one_tape(const Prob& P, const Mesh& Mh, const Loss& Ls, int64_t i, double* loss, double* dp,
                   double* du0, double* dW_acc) {
  using R = Rv<T>;
  auto& tp = tape<T>();
  tp.nodes.clear();
  int d = P.d, np = P.np;
  std::vector<R> u0(d), p(np), W;
  for (int c = 0; c < d; ++c) {
    T v = T(P.u0[(int64_t)c * P.n + i]);
    u0[c] = R(v, tp.push(v));
  }
  for (int c = 0; c < np; ++c) {
    T v = T(P.p[(int64_t)c * P.n + i]);
    p[c] = R(v, tp.push(v));
  }
  if (P.sys == SYS_NODE64) {
    W.resize(64 * 64);
    for (int c = 0; c < 64 * 64; ++c) {
      T v = T(P.W[c]);
      W[c] = R(v, tp.push(v));
    }
  }
  std::vector<double> tg(Mh.nsave * d, 0.0), wg(Mh.nsave * d, 0.0);
  if (Ls.target) gather_kd(Ls.target, Mh.nsave, d, P.n, i, tg.data());
  if (Ls.weight) gather_kd(Ls.weight, Mh.nsave, d, P.n, i, wg.data());
  R L = replay_loss<R>(P.sys, P.method, d, u0.data(), p.data(), W.empty() ? nullptr : W.data(),
                       Mh.h + i * Mh.smax, Mh.nsteps[i], Mh.nsave, Mh.save_idx + i * Mh.nsave, Ls.kind,
                       Ls.target ? tg.data() : nullptr, wg.data(), nullptr, Mh.theta_of(i));
  *loss = double(L.v);
  std::vector<A> adj(tp.nodes.size(), A(0));
  if (L.id >= 0) adj[L.id] = A(1);
  for (int64_t k = (int64_t)tp.nodes.size() - 1; k >= 0; --k) {
    const Node<T>& nd = tp.nodes[k];
    A a = adj[k];
    if (a == A(0)) continue;
    if (FUSED) {
      if (nd.a >= 0) adj[nd.a] = std::fma(A(nd.da), a, adj[nd.a]);
      if (nd.b >= 0) adj[nd.b] = std::fma(A(nd.db), a, adj[nd.b]);
      if (nd.c >= 0) adj[nd.c] = std::fma(A(nd.dc), a, adj[nd.c]);
    } else {
      if (nd.a >= 0) adj[nd.a] += A(nd.da) * a;
      if (nd.b >= 0) adj[nd.b] += A(nd.db) * a;
      if (nd.c >= 0) adj[nd.c] += A(nd.dc) * a;
    }
  }
  for (int c = 0; c < d; ++c) du0[c] = double(u0[c].id >= 0 ? adj[u0[c].id] : A(0));
  for (int c = 0; c < np; ++c) dp[c] = double(p[c].id >= 0 ? adj[p[c].id] : A(0));
  if (dW_acc)
    for (int c = 0; c < 64 * 64; ++c) dW_acc[c] += double(adj[W[c].id]);
}

// Forward-mode directional derivative of one trajectory's loss along
// (dir_p, dir_u0, dir_W).
// dir_p_i[np], dir_u0_i[d]: this trajectory's direction (null = zero).
template <class T>
double dirderiv_one(const Prob& P, const Mesh& Mh, const Loss& Ls, int64_t i, const double* dir_p_i,
                    const double* dir_u0_i, const double* dir_W) {
  using D = Dv<T>;
  int d = P.d, np = P.np;
  std::vector<D> u0(d), p(np), W;
  for (int c = 0; c < d; ++c) u0[c] = D(T(P.u0[(int64_t)c * P.n + i]), dir_u0_i ? T(dir_u0_i[c]) : T(0));
  for (int c = 0; c < np; ++c) p[c] = D(T(P.p[(int64_t)c * P.n + i]), dir_p_i ? T(dir_p_i[c]) : T(0));
  if (P.sys == SYS_NODE64) {
    W.resize(64 * 64);
    for (int c = 0; c < 64 * 64; ++c) W[c] = D(T(P.W[c]), dir_W ? T(dir_W[c]) : T(0));
  }
  std::vector<double> tg(Mh.nsave * d, 0.0), wg(Mh.nsave * d, 0.0);
  if (Ls.target) gather_kd(Ls.target, Mh.nsave, d, P.n, i, tg.data());
  if (Ls.weight) gather_kd(Ls.weight, Mh.nsave, d, P.n, i, wg.data());
  D L = replay_loss<D>(P.sys, P.method, d, u0.data(), p.data(), W.empty() ? nullptr : W.data(),
                       Mh.h + i * Mh.smax, Mh.nsteps[i], Mh.nsave, Mh.save_idx + i * Mh.nsave, Ls.kind,
                       Ls.target ? tg.data() : nullptr, wg.data(), nullptr, Mh.theta_of(i));
  return double(L.d);
}

// Forward sensitivities of one trajectory: the dual-number replay once per
// input direction (the np parameters, then the d initial-state components),
// keeping the tangent of the state at each save point.  sens [nsave][d][np+d]
// (column j = d u / d theta_j).
template <class T>
void sens_one(const Prob& P, const Mesh& Mh, int64_t i, double* sens) {
  using D = Dv<T>;
  const int d = P.d, np = P.np, m = np + d;
  std::vector<D> u0(d), p(np), us(Mh.nsave * d);
  std::vector<double> wg(Mh.nsave * d, 0.0);
  for (int j = 0; j < m; ++j) {
    for (int c = 0; c < d; ++c) u0[c] = D(T(P.u0[(int64_t)c * P.n + i]), T(j == np + c ? 1 : 0));
    for (int c = 0; c < np; ++c) p[c] = D(T(P.p[(int64_t)c * P.n + i]), T(j == c ? 1 : 0));
    replay_loss<D>(P.sys, P.method, d, u0.data(), p.data(), nullptr, Mh.h + i * Mh.smax, Mh.nsteps[i], Mh.nsave,
                   Mh.save_idx + i * Mh.nsave, LOSS_LINEAR, nullptr, wg.data(), us.data(), Mh.theta_of(i));
    for (int k = 0; k < Mh.nsave; ++k)
      for (int c = 0; c < d; ++c) sens[((int64_t)k * d + c) * m + j] = double(us[k * d + c].d);
  }
}

template <class T>
double loss_one(const Prob& P, const Mesh& Mh, const Loss& Ls, int64_t i, double* u_save) {
  int d = P.d, np = P.np;
  std::vector<T> u0(d), p(np), W, us(Mh.nsave * d);
  for (int c = 0; c < d; ++c) u0[c] = T(P.u0[(int64_t)c * P.n + i]);
  for (int c = 0; c < np; ++c) p[c] = T(P.p[(int64_t)c * P.n + i]);
  if (P.sys == SYS_NODE64) {
    W.resize(64 * 64);
    for (int c = 0; c < 64 * 64; ++c) W[c] = T(P.W[c]);
  }
  std::vector<double> tg(Mh.nsave * d, 0.0), wg(Mh.nsave * d, 0.0);
  if (Ls.target) gather_kd(Ls.target, Mh.nsave, d, P.n, i, tg.data());
  if (Ls.weight) gather_kd(Ls.weight, Mh.nsave, d, P.n, i, wg.data());
  T L = replay_loss<T>(P.sys, P.method, d, u0.data(), p.data(), W.empty() ? nullptr : W.data(),
                       Mh.h + i * Mh.smax, Mh.nsteps[i], Mh.nsave, Mh.save_idx + i * Mh.nsave, Ls.kind,
                       Ls.target ? tg.data() : nullptr, wg.data(), us.data(), Mh.theta_of(i));
  if (u_save)
    for (int k = 0; k < Mh.nsave; ++k)
      for (int c = 0; c < d; ++c) u_save[((int64_t)k * d + c) * P.n + i] = double(us[k * d + c]);
  return double(L);
}

int check_prob(const Prob& P) {
  if (P.n < 0) return -1;
  if (P.sys == SYS_LORENZ && (P.d != 3 || P.np != 3)) return -1;
  if (P.sys == SYS_ROBERTSON && (P.d != 3 || P.np != 3)) return -1;
  if (P.sys == SYS_NODE64 && (P.d != 64 || P.np != 64 || !P.W)) return -1;
  if (P.sys == SYS_HIRES) return -4;  // not built: equations not available here
  if (P.sys == SYS_LINEAR && (P.d != 1 || P.np != 1)) return -1;
  if (P.sys == SYS_KIN8 && (P.d != 8 || P.np != 8)) return -1;
  if (P.sys < 1 || P.sys > 6) return -1;
  if (P.method != M_TSIT5 && P.method != M_ROS2 && P.method != M_ROS3 && P.method != M_VERN7) return -1;
  if (P.method != M_TSIT5 && P.d > 8) return -4;
  if (P.method != M_TSIT5 && P.sys == SYS_NODE64) return -4;
  if (P.method == M_VERN7 && P.sys == SYS_KIN8) return -4;
  if (P.dtype != DT_F32 && P.dtype != DT_F64) return -1;
  return 0;
}

}  // namespace orc

using namespace orc;

extern "C" {

// Adaptive record.  Mesh outputs are trajectory-major: h[n][smax] (zero padded,
// values widened to double), save_idx[n][nsave].
int or_record(int sys, int method, int dtype, int64_t n, int d, int np, const double* p, const double* u0,
              const double* W, double t0, double t1, int nsave, const double* tsave, double rtol, double atol,
              double h0, int smax, double* h, int* nsteps, int* save_idx, int* status, int* nreject,
              int dense, double* theta, int nthreads) {
  Prob P{sys, method, dtype, d, np, n, p, u0, W};
  int rc = check_prob(P);
  if (rc) return rc;
  parallel_for(n, nthreads, [&](int, int64_t a, int64_t b) {
    auto run = [&](auto tag) {
      using T = decltype(tag);
      std::vector<T> uu(d), pp(np), WW, ts(nsave);
      for (int k = 0; k < nsave; ++k) ts[k] = T(tsave[k]);
      if (sys == SYS_NODE64) {
        WW.resize(4096);
        for (int c = 0; c < 4096; ++c) WW[c] = T(W[c]);
      }
      for (int64_t i = a; i < b; ++i) {
        for (int c = 0; c < d; ++c) uu[c] = T(u0[(int64_t)c * n + i]);
        for (int c = 0; c < np; ++c) pp[c] = T(p[(int64_t)c * n + i]);
        RecordOut<T> r = record_one<T>(sys, method, d, uu.data(), pp.data(), WW.empty() ? nullptr : WW.data(),
                                       T(t0), T(t1), nsave, ts.data(), T(rtol), T(atol), T(h0), smax, dense != 0);
        nsteps[i] = r.nsteps;
        status[i] = r.status;
        nreject[i] = r.nreject;
        if (theta)
          for (int k = 0; k < nsave; ++k) theta[i * nsave + k] = double(r.theta[k]);
        for (int s = 0; s < smax; ++s) h[i * smax + s] = s < r.nsteps ? double(r.h[s]) : 0.0;
        for (int k = 0; k < nsave; ++k) save_idx[i * nsave + k] = r.save_idx[k];
      }
    };
    if (dtype == DT_F64) run(double(0)); else run(float(0));
  });
  return 0;
}

// Adaptive forward-only solve (GRADSOLVE abstract: the forward-only solver):
// the recorder's own iteration, returning the accepted state at each save time
// instead of the mesh.  u_save [nsave][d][n] (NaN for every save point of a
// trajectory with status != 0), nsteps and status [n].
int or_solve_adaptive(int sys, int method, int dtype, int64_t n, int d, int np, const double* p, const double* u0,
                      const double* W, double t0, double t1, int nsave, const double* tsave, double rtol,
                      double atol, double h0, int smax, int dense, double* u_save, int* nsteps, int* status,
                      int nthreads) {
  Prob P{sys, method, dtype, d, np, n, p, u0, W};
  int rc = check_prob(P);
  if (rc) return rc;
  parallel_for(n, nthreads, [&](int, int64_t a, int64_t b) {
    auto run = [&](auto tag) {
      using T = decltype(tag);
      std::vector<T> uu(d), pp(np), WW, ts(nsave);
      for (int k = 0; k < nsave; ++k) ts[k] = T(tsave[k]);
      if (sys == SYS_NODE64) {
        WW.resize(4096);
        for (int c = 0; c < 4096; ++c) WW[c] = T(W[c]);
      }
      for (int64_t i = a; i < b; ++i) {
        for (int c = 0; c < d; ++c) uu[c] = T(u0[(int64_t)c * n + i]);
        for (int c = 0; c < np; ++c) pp[c] = T(p[(int64_t)c * n + i]);
        RecordOut<T> r = record_one<T>(sys, method, d, uu.data(), pp.data(), WW.empty() ? nullptr : WW.data(),
                                       T(t0), T(t1), nsave, ts.data(), T(rtol), T(atol), T(h0), smax, dense != 0);
        nsteps[i] = r.nsteps;
        status[i] = r.status;
        for (int k = 0; k < nsave; ++k)
          for (int c = 0; c < d; ++c)
            u_save[((int64_t)k * d + c) * n + i] =
                r.status == TRAJ_OK ? double(r.usave[(size_t)k * d + c]) : std::numeric_limits<double>::quiet_NaN();
      }
    };
    if (dtype == DT_F64) run(double(0)); else run(float(0));
  });
  return 0;
}

// Gradient of the replay loss.  mode 0: reverse-mode tape.  mode 1: forward
// mode, one dual-number pass per input direction (p and u0 only; not NODE64).
// mode 2: the tape with adjoints accumulated in a wider type (long double for
// fp64 runs, double for fp32 runs): same forward values and partials, less
// rounding in the reverse sweep.  mode 3: the tape with fused adjoint updates
// (plain precision, rounded differently from mode 0).
// Trajectories with status != 0 get NaN outputs.  dW (NODE64) is the sum over
// trajectories, accumulated per thread chunk and then in chunk order.
int or_grad(int sys, int method, int dtype, int64_t n, int d, int np, const double* p, const double* u0,
            const double* W, int smax, int nsave, const double* h, const int* nsteps, const int* save_idx,
            const double* theta, const int* status, int loss_kind, const double* target, const double* weight,
            int mode, double* loss, double* dp, double* du0, double* dW, int nthreads) {
  Prob P{sys, method, dtype, d, np, n, p, u0, W};
  int rc = check_prob(P);
  if (rc) return rc;
  if (mode == 1 && sys == SYS_NODE64) return -4;
  if (mode < 0 || mode > 3) return -1;
  Mesh Mh{smax, nsave, h, nsteps, save_idx, theta};
  Loss Ls{loss_kind, target, weight};
  int nt = std::max(1, nthreads);
  std::vector<std::vector<double>> dWp(sys == SYS_NODE64 ? nt : 0, std::vector<double>(4096, 0.0));
  const double nan = std::numeric_limits<double>::quiet_NaN();
  parallel_for(n, nt, [&](int tid, int64_t a, int64_t b) {
    std::vector<double> gp(np), gu(d), e_p(np), e_u(d);
    for (int64_t i = a; i < b; ++i) {
      if (status && status[i] != 0) {
        loss[i] = nan;
        for (int c = 0; c < np; ++c) dp[(int64_t)c * n + i] = nan;
        for (int c = 0; c < d; ++c) du0[(int64_t)c * n + i] = nan;
        continue;
      }
      double L;
      if (mode == 3) {
        double* acc = sys == SYS_NODE64 ? dWp[tid].data() : nullptr;
        if (dtype == DT_F64)
          grad_one_tape<double, double, true>(P, Mh, Ls, i, &L, gp.data(), gu.data(), acc);
        else
          grad_one_tape<float, float, true>(P, Mh, Ls, i, &L, gp.data(), gu.data(), acc);
      } else if (mode == 0 || mode == 2) {
        double* acc = sys == SYS_NODE64 ? dWp[tid].data() : nullptr;
        if (dtype == DT_F64 && mode == 0)
          grad_one_tape<double>(P, Mh, Ls, i, &L, gp.data(), gu.data(), acc);
        else if (dtype == DT_F64)
          grad_one_tape<double, long double>(P, Mh, Ls, i, &L, gp.data(), gu.data(), acc);
        else if (mode == 0)
          grad_one_tape<float>(P, Mh, Ls, i, &L, gp.data(), gu.data(), acc);
        else
          grad_one_tape<float, double>(P, Mh, Ls, i, &L, gp.data(), gu.data(), acc);
      } else {
        // unit directions: the basis vectors of p, then of u0
        L = dtype == DT_F64 ? loss_one<double>(P, Mh, Ls, i, nullptr) : loss_one<float>(P, Mh, Ls, i, nullptr);
        for (int c = 0; c < np + d; ++c) {
          std::fill(e_p.begin(), e_p.end(), 0.0);
          std::fill(e_u.begin(), e_u.end(), 0.0);
          (c < np ? e_p[c] : e_u[c - np]) = 1.0;
          double g = dtype == DT_F64 ? dirderiv_one<double>(P, Mh, Ls, i, e_p.data(), e_u.data(), nullptr)
                                     : dirderiv_one<float>(P, Mh, Ls, i, e_p.data(), e_u.data(), nullptr);
          (c < np ? gp[c] : gu[c - np]) = g;
        }
      }
      loss[i] = L;
      for (int c = 0; c < np; ++c) dp[(int64_t)c * n + i] = gp[c];
      for (int c = 0; c < d; ++c) du0[(int64_t)c * n + i] = gu[c];
    }
  });
  if (dW && sys == SYS_NODE64) {
    for (int c = 0; c < 4096; ++c) dW[c] = 0.0;
    for (int t = 0; t < nt; ++t)
      for (int c = 0; c < 4096; ++c) dW[c] += dWp[t][c];
  }
  return 0;
}

// Forward-mode directional derivative of each trajectory's loss along the
// given input directions (any may be null = zero).  out[n].
int or_dirderiv(int sys, int method, int dtype, int64_t n, int d, int np, const double* p, const double* u0,
                const double* W, int smax, int nsave, const double* h, const int* nsteps, const int* save_idx,
                const double* theta, int loss_kind, const double* target, const double* weight, const double* dir_p,
                const double* dir_u0, const double* dir_W, double* out, int nthreads) {
  Prob P{sys, method, dtype, d, np, n, p, u0, W};
  int rc = check_prob(P);
  if (rc) return rc;
  Mesh Mh{smax, nsave, h, nsteps, save_idx, theta};
  Loss Ls{loss_kind, target, weight};
  parallel_for(n, nthreads, [&](int, int64_t a, int64_t b) {
    std::vector<double> dpi(np, 0.0), dui(d, 0.0);
    for (int64_t i = a; i < b; ++i) {
      for (int c = 0; c < np; ++c) dpi[c] = dir_p ? dir_p[(int64_t)c * n + i] : 0.0;
      for (int c = 0; c < d; ++c) dui[c] = dir_u0 ? dir_u0[(int64_t)c * n + i] : 0.0;
      out[i] = dtype == DT_F64 ? dirderiv_one<double>(P, Mh, Ls, i, dpi.data(), dui.data(), dir_W)
                               : dirderiv_one<float>(P, Mh, Ls, i, dpi.data(), dui.data(), dir_W);
    }
  });
  return 0;
}

// Forward sensitivities d u(t_k) / d (p, u0) of the fixed-step replay, by
// forward-mode dual numbers (one pass per input direction).  sens
// [nsave][d][np+d][n]; NaN for trajectories with status != 0 (status may be
// null).  Not for NODE64 (its W directions are not inputs of this product).
int or_sens(int sys, int method, int dtype, int64_t n, int d, int np, const double* p, const double* u0, int smax,
            int nsave, const double* h, const int* nsteps, const int* save_idx, const double* theta,
            const int* status, double* sens, int nthreads) {
  Prob P{sys, method, dtype, d, np, n, p, u0, nullptr};
  int rc = check_prob(P);
  if (rc) return rc;
  if (sys == SYS_NODE64) return -4;
  Mesh Mh{smax, nsave, h, nsteps, save_idx, theta};
  const int m = np + d;
  parallel_for(n, nthreads, [&](int, int64_t a, int64_t b) {
    std::vector<double> si((size_t)nsave * d * m);
    for (int64_t i = a; i < b; ++i) {
      if (status && status[i] != TRAJ_OK) {
        std::fill(si.begin(), si.end(), std::numeric_limits<double>::quiet_NaN());
      } else if (dtype == DT_F64) {
        sens_one<double>(P, Mh, i, si.data());
      } else {
        sens_one<float>(P, Mh, i, si.data());
      }
      for (size_t q = 0; q < si.size(); ++q) sens[(int64_t)q * n + i] = si[q];
    }
  });
  return 0;
}

// Plain replay: loss[n] and, if u_save != null, the states at the save
// points, u_save[nsave][d][n].
int or_replay(int sys, int method, int dtype, int64_t n, int d, int np, const double* p, const double* u0,
              const double* W, int smax, int nsave, const double* h, const int* nsteps, const int* save_idx,
              const double* theta, int loss_kind, const double* target, const double* weight, double* loss,
              double* u_save, int nthreads) {
  Prob P{sys, method, dtype, d, np, n, p, u0, W};
  int rc = check_prob(P);
  if (rc) return rc;
  Mesh Mh{smax, nsave, h, nsteps, save_idx, theta};
  Loss Ls{loss_kind, target, weight};
  parallel_for(n, nthreads, [&](int, int64_t a, int64_t b) {
    for (int64_t i = a; i < b; ++i)
      loss[i] = dtype == DT_F64 ? loss_one<double>(P, Mh, Ls, i, u_save) : loss_one<float>(P, Mh, Ls, i, u_save);
  });
  return 0;
}

// Operation counts of one fixed step of the given system/method, for the
// roofline's algorithmic-work figure: out = {add, mul, fma, div, sqrt, tanh}.
int or_count_step(int sys, int method, int d, int np, double* out6) {
  std::vector<Cn> u(d, Cn(0.5)), p(np, Cn(1.0)), un(d), W;
  if (sys == SYS_NODE64) W.assign(4096, Cn(0.01));
  opcount() = OpCount();
  Cn h(0.01);
  method_step<Cn>(sys, method, d, u.data(), p.data(), W.empty() ? nullptr : W.data(), h, un.data(), nullptr);
  OpCount c = opcount();
  out6[0] = double(c.add);
  out6[1] = double(c.mul);
  out6[2] = double(c.fma);
  out6[3] = double(c.div);
  out6[4] = double(c.sqrt);
  out6[5] = double(c.tanh);
  return 0;
}

// Low-level access for pins: one step of the method in double or float.
int or_step(int sys, int method, int dtype, int d, const double* u, const double* p, const double* W, double h,
            double* unew, double* err) {
  auto run = [&](auto tag) {
    using T = decltype(tag);
    std::vector<T> uu(d), pp(64), WW, un(d), e(d);
    for (int c = 0; c < d; ++c) uu[c] = T(u[c]);
    for (int c = 0; c < 64; ++c) pp[c] = p ? T(p[c]) : T(0);
    if (W) {
      WW.resize(4096);
      for (int c = 0; c < 4096; ++c) WW[c] = T(W[c]);
    }
    bool ok = method_step<T>(sys, method, d, uu.data(), pp.data(), WW.empty() ? nullptr : WW.data(), T(h), un.data(),
                             e.data());
    for (int c = 0; c < d; ++c) {
      unew[c] = double(un[c]);
      if (err) err[c] = double(e[c]);
    }
    return ok ? 0 : 4;
  };
  return dtype == DT_F64 ? run(double(0)) : run(float(0));
}

// splitmix64 (Steele, Lea & Flood 2014): a counter-based 64-bit mixer, used
// only to draw the perturbations of or_step_errors.
static inline uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

// The recorder's view of a given mesh: trajectory i replayed over h[i][0..
// nsteps[i]) (no landing logic: the steps are data), and for every step s its
// scaled error err[i][s] (the recorder's error norm on that step's embedded
// estimate) and the PI factor fac[i][s] that accepting it gives (the cap after
// a rejection not applied: the mesh does not show rejections).  On a mesh the
// recorder wrote in the same precision, the proposal chain fac * h_prop
// reproduces its steps.  Outputs [n][smax], zero past nsteps; a trajectory
// whose status is not 0 is skipped (zeros).
// nperturb > 0: fac_draws[k][n][smax] receives the same factors evaluated
// again with every step's start state multiplied by 1 + r eps (r uniform in
// [-1, 1) per component, draw, step and trajectory; eps of the precision),
// each draw carrying its own errprev: the spread of the draws shows how far
// rounding at the precision's level moves each factor (the embedded estimate
// is a sum with cancellation, so a small error carries a large relative
// rounding noise).
int or_step_errors(int sys, int method, int dtype, int64_t n, int d, int np, const double* p, const double* u0,
                   const double* W, int smax, const double* h, const int* nsteps, const int* status, double rtol,
                   double atol, double* err, double* fac, int nperturb, double* fac_draws, int nthreads) {
  Prob P{sys, method, dtype, d, np, n, p, u0, W};
  int rc = check_prob(P);
  if (rc) return rc;
  parallel_for(n, nthreads, [&](int, int64_t a, int64_t b) {
    auto run = [&](auto tag) {
      using T = decltype(tag);
      const T q = T(method_order(method));
      std::vector<T> u(d), un(d), e(d), sc(d), pp(np), WW;
      if (sys == SYS_NODE64) {
        WW.resize(4096);
        for (int c = 0; c < 4096; ++c) WW[c] = T(W[c]);
      }
      for (int64_t i = a; i < b; ++i) {
        for (int s = 0; s < smax; ++s) err[i * smax + s] = fac[i * smax + s] = 0.0;
        if (status && status[i] != TRAJ_OK) continue;
        for (int c = 0; c < d; ++c) u[c] = T(u0[(int64_t)c * n + i]);
        for (int c = 0; c < np; ++c) pp[c] = T(p[(int64_t)c * n + i]);
        for (int k = 0; k < nperturb; ++k)
          for (int s = 0; s < smax; ++s) fac_draws[((int64_t)k * n + i) * smax + s] = 0.0;
        const int S = std::min(nsteps[i], smax);
        T lnprev = T(0);
        std::vector<T> lnprev_k(nperturb, T(0)), up(d), unp(d), ep(d), scp(d);
        for (int s = 0; s < S; ++s) {
          const T hs = T(h[i * smax + s]);
          const T* Wp = WW.empty() ? nullptr : WW.data();
          method_step<T>(sys, method, d, u.data(), pp.data(), Wp, hs, un.data(), e.data());
          for (int c = 0; c < d; ++c) sc[c] = std::fma(T(rtol), std::max(std::fabs(u[c]), std::fabs(un[c])), T(atol));
          const T er = rms_scaled<T>(d, e.data(), sc.data());
          err[i * smax + s] = double(er);
          fac[i * smax + s] = double(accept_factor<T>(er, q, lnprev));
          for (int k = 0; k < nperturb; ++k) {
            for (int c = 0; c < d; ++c) {
              const uint64_t r = splitmix64(((((uint64_t)i * 4096 + (uint64_t)s) * 64 + (uint64_t)k) << 8) + c);
              const T rho = T(double(r >> 11) * 0x1.0p-52 - 1.0);  // uniform in [-1, 1)
              up[c] = u[c] * (T(1) + rho * std::numeric_limits<T>::epsilon());
            }
            method_step<T>(sys, method, d, up.data(), pp.data(), Wp, hs, unp.data(), ep.data());
            for (int c = 0; c < d; ++c)
              scp[c] = std::fma(T(rtol), std::max(std::fabs(up[c]), std::fabs(unp[c])), T(atol));
            const T erk = rms_scaled<T>(d, ep.data(), scp.data());
            fac_draws[((int64_t)k * n + i) * smax + s] = double(accept_factor<T>(erk, q, lnprev_k[k]));
          }
          for (int c = 0; c < d; ++c) u[c] = un[c];
        }
      }
    };
    if (dtype == DT_F64) run(double(0)); else run(float(0));
  });
  return 0;
}

// The right-hand side and its analytic Jacobian at one point (double).
int or_rhs(int sys, int d, const double* u, const double* p, const double* W, double* f, double* J) {
  (void)d;
  rhs<double>(sys, u, p, W, f);
  if (J) jac<double>(sys, u, p, J);
  return 0;
}

// Verner 7(6) tableau export for the order-condition pins: c[10], A[10][9],
// b[10], bhat[10].
void or_vern7_tableau(double* c, double* A, double* b, double* bh) {
  for (int i = 0; i < 10; ++i) {
    c[i] = V7_C[i];
    b[i] = V7_B[i];
    bh[i] = V7_BH[i];
    for (int j = 0; j < 9; ++j) A[i * 9 + j] = V7_A[i][j];
  }
}

// The continuous extension's coefficients for the pins: r[7][4], b_i(theta) =
// sum_m r[i][m-1] theta^m; and its weights at theta as the dense output forms
// them (dtype 2: double, 1: float).
void or_tsit5_dense_coeffs(double* r) {
  for (int i = 0; i < 7; ++i)
    for (int m = 0; m < 4; ++m) r[i * 4 + m] = TS_R[i][m];
}

void or_tsit5_dense_weights(int dtype, double theta, double* bw) {
  if (dtype == DT_F32) {
    float w[7];
    tsit5_dense_weights<float>(float(theta), w);
    for (int i = 0; i < 7; ++i) bw[i] = w[i];
  } else {
    tsit5_dense_weights<double>(theta, bw);
  }
}

// Tableau export for the order-condition pins: c[7], A[7][6], bt[7].
void or_tsit5_tableau(double* c, double* A, double* bt) {
  for (int i = 0; i < 7; ++i) {
    c[i] = TS_C[i];
    bt[i] = TS_BT[i];
    for (int j = 0; j < 6; ++j) A[i * 6 + j] = TS_A[i][j];
  }
}

double or_ros2_gamma(void) { return ROS2_GAMMA; }

// ROS3 coefficients for the order-condition pins: {gamma, 1/gamma, c21, c31,
// c32, m2, m3, e1, e2, e3}.
void or_ros3_coeffs(double* out10) {
  const double v[10] = {ROS3_GAMMA, ROS3_INV_GAMMA, ROS3_C21, ROS3_C31, ROS3_C32,
                        ROS3_M2,    ROS3_M3,        ROS3_E1,  ROS3_E2,  ROS3_E3};
  for (int i = 0; i < 10; ++i) out10[i] = v[i];
}

// The controller's power function, element-wise (dtype 2: double, 1: float).
void or_ctrl_pow(int dtype, int64_t n, const double* x, const double* y, double* out) {
  for (int64_t i = 0; i < n; ++i)
    out[i] = dtype == DT_F64 ? ctrl_pow<double>(x[i], y[i]) : double(ctrl_pow<float>(float(x[i]), float(y[i])));
}

}  // extern "C"
