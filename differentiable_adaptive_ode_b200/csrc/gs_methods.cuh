// gs_methods.cuh -- the one-step maps on the device: Tsit5 trial step (record / forward),
// Tsit5 replay-adjoint step, ROS34PW2 trial step and its replay-adjoint step.
//
// Method structure: "gradsolve: fast exact gradients for ODE ensembles on GPUs" §2.1 (embedded
// explicit pair with first-same-as-last reuse; RMS error test), §3 (replay map Phi with the
// recorded step size as data; its reverse-mode derivative), §3.2 (Rosenbrock stage solves with
// I - gamma h J; the backward pass needs one solve with the transpose and differentiates J).
// Coefficients (not printed on the pages): Tsitouras (2011) for Tsit5, Rang & Angermann (2005)
// for ROS34PW2 -- the published decimals, rounded to the working precision at compile time.
#pragma once
#include <type_traits>

#include "gs_dual.cuh"
#include "gs_fields.cuh"

namespace gs {

// The step's scaled RMS error sqrt(mean_c (e_c / sc_c)^2) (the accept test of an embedded pair).
template <class R, int D>
__device__ __forceinline__ R scaled_rms(const R (&e)[D], const R (&sc)[D]) {
  R s2 = R(0);
#pragma unroll
  for (int c = 0; c < D; ++c) {
    const R q = e[c] / sc[c];
    s2 = fma(q, q, s2);
  }
  return sqrt(s2 / R(D));
}
// fp64: the D reciprocals 1/sc_c from ONE division by Montgomery's simultaneous inversion
// (P. L. Montgomery, "Speeding the Pollard and elliptic curve methods of factorization", Math.
// Comp. 48, 1987): prefix products P_c = sc_0 ... sc_c, one reciprocal of P_{D-1}, then backwards
// 1/sc_c = P_{c-1} / P_c and 1/P_{c-1} = sc_c / P_c.  Each reciprocal carries at most about 3D
// roundings (below 1e-14 relative for D <= 8), far below what the step control resolves.  Where
// a prefix product leaves the normal range (scales near 0 or huge, non-finite values) the step
// takes the per-component divisions instead, so those cases behave exactly as before.
template <int D>
__device__ __forceinline__ double scaled_rms(const double (&e)[D], const double (&sc)[D]) {
  constexpr double lo = 2.2250738585072014e-308, hi = 1.7976931348623157e308;  // normal range
  double P[D];
  P[0] = sc[0];
  bool ok = (P[0] >= lo) && (P[0] <= hi);
#pragma unroll
  for (int c = 1; c < D; ++c) {
    P[c] = P[c - 1] * sc[c];
    ok = ok && (P[c] >= lo) && (P[c] <= hi);
  }
  double s2 = 0.0;
  if (ok) {
    double inv = 1.0 / P[D - 1];
#pragma unroll
    for (int c = D - 1; c > 0; --c) {
      const double q = e[c] * (inv * P[c - 1]);
      inv = inv * sc[c];
      s2 = fma(q, q, s2);
    }
    const double q0 = e[0] * inv;
    s2 = fma(q0, q0, s2);
  } else {
#pragma unroll
    for (int c = 0; c < D; ++c) {
      const double q = e[c] / sc[c];
      s2 = fma(q, q, s2);
    }
  }
  return sqrt(s2 * (1.0 / D));
}

struct Tsit5 {
  static constexpr int order = 5, err_order = 5;
  // a_ij, i = 2..7, j < i; row 7 equals b (b_7 = 0).
  static constexpr double a21 = 0.161;
  static constexpr double a31 = -0.008480655492356989, a32 = 0.335480655492357;
  static constexpr double a41 = 2.897153057105493, a42 = -6.359448489975075,
                          a43 = 4.3622954328695815;
  static constexpr double a51 = 5.325864828439257, a52 = -11.748883564062828,
                          a53 = 7.4955393428898365, a54 = -0.09249506636175525;
  static constexpr double a61 = 5.86145544294642, a62 = -12.92096931784711,
                          a63 = 8.159367898576159, a64 = -0.071584973281401,
                          a65 = -0.028269050394068383;
  static constexpr double b1 = 0.09646076681806523, b2 = 0.01, b3 = 0.4798896504144996,
                          b4 = 1.379008574103742, b5 = -3.290069515436081,
                          b6 = 2.324710524099774;
  // error weights b - b_hat
  static constexpr double e1 = -0.00178001105222577714, e2 = -0.0008164344596567469,
                          e3 = 0.007880878010261995, e4 = -0.1447110071732629,
                          e5 = 0.5823571654525552, e6 = -0.45808210592918697,
                          e7 = 0.015151515151515152;
};

// Verner's 7(6) pair ("most efficient" IIa, Verner 2010): the seventh-order pair offered next to
// Tsit5 ("gradsolve: fast exact gradients for ODE ensembles on GPUs" §3.1).  10 stages, not
// first-same-as-last; b_2 = b_3 = b_10 = 0 and the tenth stage serves only the error estimate.
// Published decimals.  Zero entries are skipped at compile time in the unrolled stage loops.
struct Vern7 {
  static constexpr int order = 7, err_order = 7;
};
__host__ __device__ constexpr double vern7_a(int i, int j) {
  constexpr double A[10][9] = {
      {0, 0, 0, 0, 0, 0, 0, 0, 0},
      {0.005, 0, 0, 0, 0, 0, 0, 0, 0},
      {-1.0767901234567902, 1.185679012345679, 0, 0, 0, 0, 0, 0, 0},
      {0.04083333333333333, 0, 0.1225, 0, 0, 0, 0, 0, 0},
      {0.6389139236255726, 0, -2.455672638223657, 2.272258714598084, 0, 0, 0, 0, 0},
      {-2.6615773750187572, 0, 10.804513886456137, -8.3539146573962, 0.820487594956657, 0, 0,
       0, 0},
      {6.067741434696772, 0, -24.711273635911088, 20.427517930788895, -1.9061579788166472,
       1.006172249242068, 0, 0, 0},
      {12.054670076253203, 0, -49.75478495046899, 41.142888638604674, -4.461760149974004,
       2.042334822239175, -0.09834843665406107, 0, 0},
      {10.138146522881808, 0, -42.6411360317175, 35.76384003992257, -4.3480228403929075,
       2.009862268377035, 0.3487490460338272, -0.27143900510483127, 0},
      {-45.030072034298676, 0, 187.3272437654589, -154.02882369350186, 18.56465306347536,
       -7.141809679295079, 1.3088085781613787, 0, 0}};
  return A[i][j];
}
__host__ __device__ constexpr double vern7_b(int i) {
  constexpr double B[10] = {0.04715561848627222, 0, 0, 0.25750564298434153, 0.26216653977412624,
                            0.15216092656738558, 0.4939969170032485, -0.29430311714032503,
                            0.08131747232495111, 0};
  return B[i];
}
// b - b_hat
__host__ __device__ constexpr double vern7_e(int i) {
  constexpr double BH[10] = {0.044608606606341174, 0, 0, 0.26716403785713727,
                             0.22010183001772932, 0.2188431703143157, 0.22898717054112028, 0, 0,
                             0.02029518466335628};
  return vern7_b(i) - BH[i];
}

// A[i][j] of the explicit stages as a device-evaluable table (i = 0..5 stage index, j < i).
template <class R> __device__ __forceinline__ R ta(int i, int j) {
  // Resolved at compile time inside fully unrolled loops.
  constexpr double A[6][5] = {
      {0, 0, 0, 0, 0},
      {Tsit5::a21, 0, 0, 0, 0},
      {Tsit5::a31, Tsit5::a32, 0, 0, 0},
      {Tsit5::a41, Tsit5::a42, Tsit5::a43, 0, 0},
      {Tsit5::a51, Tsit5::a52, Tsit5::a53, Tsit5::a54, 0},
      {Tsit5::a61, Tsit5::a62, Tsit5::a63, Tsit5::a64, Tsit5::a65}};
  return R(A[i][j]);
}
template <class R> __device__ __forceinline__ R tb(int i) {
  constexpr double B[6] = {Tsit5::b1, Tsit5::b2, Tsit5::b3, Tsit5::b4, Tsit5::b5, Tsit5::b6};
  return R(B[i]);
}
template <class R> __device__ __forceinline__ R te(int i) {
  constexpr double E[7] = {Tsit5::e1, Tsit5::e2, Tsit5::e3, Tsit5::e4,
                           Tsit5::e5, Tsit5::e6, Tsit5::e7};
  return R(E[i]);
}

// The same tables in constant memory, 1-based stage indices, zero-padded, for the rolled stage
// loop below (the loop index selects the coefficients, so one copy of f serves every stage):
//   fwd[i][m] = a_{i+1+m, i}  (stage i's slope into the stage states still open, m = 0..5)
//   rev[i][m] = a_{i, i-1-m}  (stage i's cotangent into the earlier stages, m = 0..4)
//   b[i] = b_i,  e[i] = b_i - bh_i.
struct Tsit5Rolled {
  double fwd[8][6], rev[8][5], b[8], e[8];
};
constexpr double tsit5_a1(int i, int j) {
  // a_ij, 1-based, i = 2..7 (row 7 = b), j < i; 0 elsewhere
  constexpr double A[8][8] = {
      {0, 0, 0, 0, 0, 0, 0, 0},
      {0, 0, 0, 0, 0, 0, 0, 0},
      {0, Tsit5::a21, 0, 0, 0, 0, 0, 0},
      {0, Tsit5::a31, Tsit5::a32, 0, 0, 0, 0, 0},
      {0, Tsit5::a41, Tsit5::a42, Tsit5::a43, 0, 0, 0, 0},
      {0, Tsit5::a51, Tsit5::a52, Tsit5::a53, Tsit5::a54, 0, 0, 0},
      {0, Tsit5::a61, Tsit5::a62, Tsit5::a63, Tsit5::a64, Tsit5::a65, 0, 0},
      {0, Tsit5::b1, Tsit5::b2, Tsit5::b3, Tsit5::b4, Tsit5::b5, Tsit5::b6, 0}};
  return (i >= 0 && i < 8 && j >= 0 && j < 8) ? A[i][j] : 0.0;
}
constexpr Tsit5Rolled make_tsit5_rolled() {
  Tsit5Rolled t{};
  const double B[8] = {0, Tsit5::b1, Tsit5::b2, Tsit5::b3, Tsit5::b4, Tsit5::b5, Tsit5::b6, 0};
  const double E[8] = {0, Tsit5::e1, Tsit5::e2, Tsit5::e3, Tsit5::e4, Tsit5::e5, Tsit5::e6, Tsit5::e7};
  for (int i = 0; i < 8; ++i) {
    t.b[i] = B[i];
    t.e[i] = E[i];
    for (int m = 0; m < 6; ++m) t.fwd[i][m] = (i >= 1 && i + 1 + m <= 7) ? tsit5_a1(i + 1 + m, i) : 0.0;
    for (int m = 0; m < 5; ++m) t.rev[i][m] = (i - 1 - m >= 1) ? tsit5_a1(i, i - 1 - m) : 0.0;
  }
  return t;
}
static __constant__ Tsit5Rolled c_tsit5_d = make_tsit5_rolled();
struct Tsit5RolledF {
  float fwd[8][6], rev[8][5], b[8], e[8];
};
constexpr Tsit5RolledF make_tsit5_rolled_f() {
  Tsit5RolledF t{};
  const Tsit5Rolled d = make_tsit5_rolled();
  for (int i = 0; i < 8; ++i) {
    t.b[i] = float(d.b[i]);
    t.e[i] = float(d.e[i]);
    for (int m = 0; m < 6; ++m) t.fwd[i][m] = float(d.fwd[i][m]);
    for (int m = 0; m < 5; ++m) t.rev[i][m] = float(d.rev[i][m]);
  }
  return t;
}
static __constant__ Tsit5RolledF c_tsit5_f = make_tsit5_rolled_f();
template <class R> __device__ __forceinline__ const auto& tsit5_tab();
template <> __device__ __forceinline__ const auto& tsit5_tab<double>() { return c_tsit5_d; }
template <> __device__ __forceinline__ const auto& tsit5_tab<float>() { return c_tsit5_f; }

// Tsit5 trial with the stage loop rolled: the open stage states are kept as running sums
// acc[m] = partial Y_{i+m} (all slopes k_l, l < i, already added), so the loop body holds a
// single copy of f.  Same result as tsit5_trial up to the order of the roundings; the products
// are fused explicitly so that every kernel using it rounds identically.
template <class F, class R>
__device__ __forceinline__ R tsit5_trial_rolled(const R (&y)[F::D], R h,
                                                const typename F::template Theta<R>& th,
                                                const R (&k1)[F::D], R (&ynew)[F::D],
                                                R (&k7)[F::D], R rtol, R atol) {
  constexpr int D = F::D;
  const auto& T = tsit5_tab<R>();
  R acc[6][D], er[D], hc1[6];
#pragma unroll
  for (int m = 0; m < 6; ++m) hc1[m] = h * T.fwd[1][m];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    const R yc = y[c], kc = k1[c];
#pragma unroll
    for (int m = 0; m < 6; ++m) acc[m][c] = fma(hc1[m], kc, yc);
    er[c] = T.e[1] * kc;
  }
  // The last stage (i = 7) evaluates f at y_new itself and opens no further stage, so the loop
  // leaves with acc[0] = y_new and kk = f(y_new), copied out after it: no value other than acc
  // and er is carried from one pass of the body to the next.  (Copying them out inside the loop,
  // on its last pass, kept y_new and k7 live across every pass: the stellar record kernel spilled
  // at 168 registers, and ran 15.1 ms against 13.3 ms this way at 2^20 trajectories.)
  R kk[D];
#pragma unroll 1
  for (int i = 2; i <= 7; ++i) {
    F::f(acc[0], th, kk);
    const R ei = T.e[i];
#pragma unroll
    for (int c = 0; c < D; ++c) er[c] = fma(ei, kk[c], er[c]);
    if (i == 7) break;
#pragma unroll
    for (int m = 0; m < 5; ++m) {
      const R hc = h * T.fwd[i][m];
#pragma unroll
      for (int c = 0; c < D; ++c) acc[m][c] = fma(hc, kk[c], acc[m + 1][c]);
    }
  }
#pragma unroll
  for (int c = 0; c < D; ++c) { ynew[c] = acc[0][c]; k7[c] = kk[c]; }
  R ev[D], sc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    const R yc = y[c];
    ev[c] = h * er[c];
    sc[c] = fma(rtol, fmax(fabs(yc), fabs(ynew[c])), atol);
  }
  return scaled_rms(ev, sc);
}

// One Tsit5 trial from y with step h; k1 = f(y) is carried (first-same-as-last).  Produces the
// step result ynew, its slope k7 = f(ynew) (the next k1) and the scaled RMS error
//   err = sqrt(mean_i (e_i / (atol + rtol max(|y_i|, |ynew_i|)))^2),  e = h sum_j (b_j - bh_j) k_j.
template <class F, class R>
__device__ __forceinline__ R tsit5_trial(const R (&y)[F::D], R h, const typename F::template Theta<R>& th,
                                         const R (&k1)[F::D], R (&ynew)[F::D], R (&k7)[F::D],
                                         R rtol, R atol) {
  constexpr int D = F::D;
  R k[6][D];
#pragma unroll
  for (int c = 0; c < D; ++c) k[0][c] = k1[c];
#pragma unroll
  for (int i = 1; i < 6; ++i) {
    R Y[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R s = ta<R>(i, 0) * k[0][c];
#pragma unroll
      for (int j = 1; j < i; ++j) s += ta<R>(i, j) * k[j][c];
      Y[c] = y[c] + h * s;
    }
    F::f(Y, th, k[i]);
  }
#pragma unroll
  for (int c = 0; c < D; ++c) {
    R s = tb<R>(0) * k[0][c];
#pragma unroll
    for (int j = 1; j < 6; ++j) s += tb<R>(j) * k[j][c];
    ynew[c] = y[c] + h * s;
  }
  F::f(ynew, th, k7);
  R ev[D], sc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    R s = te<R>(0) * k[0][c];
#pragma unroll
    for (int j = 1; j < 6; ++j) s += te<R>(j) * k[j][c];
    s += te<R>(6) * k7[c];
    const R e = h * s;
    ev[c] = e;
    sc[c] = atol + rtol * fmax(fabs(y[c]), fabs(ynew[c]));
  }
  return scaled_rms(ev, sc);
}

// The Tsit5 replay map Phi(y, h) = y + h sum_{i<=6} b_i k_i with k_1 = f(y) (no error estimate).
template <class F, class R>
__device__ __forceinline__ void tsit5_replay_step(const R (&y)[F::D], R h,
                                                  const typename F::template Theta<R>& th,
                                                  R (&ynew)[F::D]) {
  constexpr int D = F::D;
  R k[6][D];
  F::f(y, th, k[0]);
#pragma unroll
  for (int i = 1; i < 6; ++i) {
    R Y[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R s = ta<R>(i, 0) * k[0][c];
#pragma unroll
      for (int j = 1; j < i; ++j) s += ta<R>(i, j) * k[j][c];
      Y[c] = y[c] + h * s;
    }
    F::f(Y, th, k[i]);
  }
#pragma unroll
  for (int c = 0; c < D; ++c) {
    R s = tb<R>(0) * k[0][c];
#pragma unroll
    for (int j = 1; j < 6; ++j) s += tb<R>(j) * k[j][c];
    ynew[c] = y[c] + h * s;
  }
}

// TAPE of a field: how many transcendental intermediates of f one stage keeps for its VJP
// (0 when the field declares none).
template <class F, class = void> struct TapeOf { static constexpr int value = 0; };
template <class F> struct TapeOf<F, std::void_t<decltype(F::TAPE)>> {
  static constexpr int value = F::TAPE;
};

// ----------------------------------------------------------------------------------------------
// Verner 7 one-step maps.  Stage states Y_i = y + h sum_{j<i} a_ij k_j, k_i = f(Y_i).
// ----------------------------------------------------------------------------------------------
// Stages 2..NS from y with k1 = f(y) given; k[i] holds slope i (0-based).
template <class F, class R, int NS>
__device__ __forceinline__ void vern7_stages(const R (&y)[F::D], R h,
                                             const typename F::template Theta<R>& th,
                                             R (&k)[10][F::D]) {
  constexpr int D = F::D;
#pragma unroll
  for (int i = 1; i < NS; ++i) {
    R Y[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R s = R(vern7_a(i, 0)) * k[0][c];
#pragma unroll
      for (int j = 1; j < i; ++j)
        if (vern7_a(i, j) != 0.0) s += R(vern7_a(i, j)) * k[j][c];
      Y[c] = y[c] + h * s;
    }
    F::f(Y, th, k[i]);
  }
}

// One Verner 7 trial from y with step h; k1 = f(y) is carried (valid across a rejected trial, and
// evaluated afresh at the new state after an accepted one: the pair is not first-same-as-last).
// Returns the scaled RMS error of e = h sum_i (b_i - bh_i) k_i; ynew = y + h sum_i b_i k_i.
template <class F, class R>
__device__ __forceinline__ R vern7_trial(const R (&y)[F::D], R h,
                                         const typename F::template Theta<R>& th,
                                         const R (&k1)[F::D], R (&ynew)[F::D], R rtol, R atol) {
  constexpr int D = F::D;
  R k[10][D];
#pragma unroll
  for (int c = 0; c < D; ++c) k[0][c] = k1[c];
  vern7_stages<F, R, 10>(y, h, th, k);
  R ev[D], sc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    R s = R(vern7_b(0)) * k[0][c];
#pragma unroll
    for (int j = 1; j < 9; ++j)
      if (vern7_b(j) != 0.0) s += R(vern7_b(j)) * k[j][c];
    ynew[c] = y[c] + h * s;
    R es = R(vern7_e(0)) * k[0][c];
#pragma unroll
    for (int j = 1; j < 10; ++j)
      if (vern7_e(j) != 0.0) es += R(vern7_e(j)) * k[j][c];
    const R e = h * es;
    ev[c] = e;
    sc[c] = atol + rtol * fmax(fabs(y[c]), fabs(ynew[c]));
  }
  return scaled_rms(ev, sc);
}

// The Verner 7 replay map Phi(y, h) = y + h sum_{i<=9} b_i k_i with k_1 = f(y).
template <class F, class R>
__device__ __forceinline__ void vern7_replay_step(const R (&y)[F::D], R h,
                                                  const typename F::template Theta<R>& th,
                                                  R (&ynew)[F::D]) {
  constexpr int D = F::D;
  R k[10][D];
  F::f(y, th, k[0]);
  vern7_stages<F, R, 9>(y, h, th, k);
#pragma unroll
  for (int c = 0; c < D; ++c) {
    R s = R(vern7_b(0)) * k[0][c];
#pragma unroll
    for (int j = 1; j < 9; ++j)
      if (vern7_b(j) != 0.0) s += R(vern7_b(j)) * k[j][c];
    ynew[c] = y[c] + h * s;
  }
}

// Reverse-mode step of the Verner 7 replay map with h fixed (the same rule as the Tsit5 step,
// nine stages): recompute the stage states from the recorded y_n, then for i = 9..1
//   kb_i = h (b_i lam + G_i),  Yb_i = J_y(Y_i)^T kb_i,  thb += J_th(Y_i)^T kb_i,
//   G_j += a_ij Yb_i (j < i),   and finally lam <- lam + sum_i Yb_i.
// Fields that declare TAPE > 0 keep the transcendental part of f at each of the nine stages in
// the per-lane shared-memory tape (slot (i, v) at tape[(i * TAPE + v) * tstride]) for the VJPs.
template <class F, class R>
__device__ __forceinline__ void vern7_adjoint_step(const R (&y)[F::D], R h,
                                                   const typename F::template Theta<R>& th,
                                                   R (&lam)[F::D], R (&thb)[F::M],
                                                   R* tape = nullptr, int tstride = 0) {
  constexpr int D = F::D;
  constexpr int TP = TapeOf<F>::value;
  R Y[9][D];
  {
    R k[10][D];
#pragma unroll
    for (int c = 0; c < D; ++c) Y[0][c] = y[c];
    if constexpr (TP > 0) {
      R tp[TP > 0 ? TP : 1];
      F::f_tape(Y[0], th, k[0], tp);
#pragma unroll
      for (int v = 0; v < TP; ++v) tape[v * tstride] = tp[v];
    } else {
      F::f(y, th, k[0]);
    }
#pragma unroll
    for (int i = 1; i < 9; ++i) {
#pragma unroll
      for (int c = 0; c < D; ++c) {
        R s = R(vern7_a(i, 0)) * k[0][c];
#pragma unroll
        for (int j = 1; j < i; ++j)
          if (vern7_a(i, j) != 0.0) s += R(vern7_a(i, j)) * k[j][c];
        Y[i][c] = y[c] + h * s;
      }
      if constexpr (TP > 0) {
        R tp[TP > 0 ? TP : 1];
        if (i < 8) F::f_tape(Y[i], th, k[i], tp);
        else F::inter_tape(Y[i], th, tp);
#pragma unroll
        for (int v = 0; v < TP; ++v) tape[(i * TP + v) * tstride] = tp[v];
      } else {
        if (i < 8) F::f(Y[i], th, k[i]);
      }
    }
  }
  R G[8][D], dl[D];
#pragma unroll
  for (int c = 0; c < D; ++c) dl[c] = R(0);
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < D; ++c) G[i][c] = R(0);
#pragma unroll
  for (int i = 8; i >= 0; --i) {
    R kb[D], Yb[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R s = (vern7_b(i) != 0.0) ? R(vern7_b(i)) * lam[c] : R(0);
      if (i < 8) s += G[i][c];
      kb[c] = h * s;
    }
    if constexpr (TP > 0) {
      R tp[TP > 0 ? TP : 1];
#pragma unroll
      for (int v = 0; v < TP; ++v) tp[v] = tape[(i * TP + v) * tstride];
      F::vjp_tape(Y[i], th, tp, kb, Yb, thb);
    } else {
      F::vjp(Y[i], th, kb, Yb, thb);
    }
#pragma unroll
    for (int c = 0; c < D; ++c) {
      dl[c] += Yb[c];
#pragma unroll
      for (int j = 0; j < i; ++j)
        if (vern7_a(i, j) != 0.0) G[j][c] += R(vern7_a(i, j)) * Yb[c];
    }
  }
#pragma unroll
  for (int c = 0; c < D; ++c) lam[c] += dl[c];
}

// Tangent of one Tsit5 step with h fixed, along the input direction (yd, thd.d):
//   Yd_i = yd + h sum_{j<i} a_ij Kd_j,   Kd_i = J_y(Y_i) Yd_i + J_theta(Y_i) thd,
//   yd_new = yd + h sum_{i<=6} b_i Kd_i
// -- the forward-mode derivative of Phi(y, h; theta), i.e. the same Tsit5 step applied to the
// sensitivity equations S' = J_y S + J_theta.  Each Kd_i comes from f evaluated on dual numbers
// (value and derivative together), so the stage values Y_i are recomputed alongside.
template <class F, class R>
__device__ __forceinline__ void tsit5_tangent_step(const R (&y)[F::D], R h,
                                                   const typename F::template Theta<Dl<R>>& thd,
                                                   R (&yd)[F::D]) {
  constexpr int D = F::D;
  Dl<R> k[6][D];
  {
    Dl<R> Y[D];
#pragma unroll
    for (int c = 0; c < D; ++c) Y[c] = Dl<R>(y[c], yd[c]);
    F::f(Y, thd, k[0]);
  }
#pragma unroll
  for (int i = 1; i < 6; ++i) {
    Dl<R> Y[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R sv = ta<R>(i, 0) * k[0][c].v, sd = ta<R>(i, 0) * k[0][c].d;
#pragma unroll
      for (int j = 1; j < i; ++j) {
        sv += ta<R>(i, j) * k[j][c].v;
        sd += ta<R>(i, j) * k[j][c].d;
      }
      Y[c] = Dl<R>(y[c] + h * sv, yd[c] + h * sd);
    }
    F::f(Y, thd, k[i]);
  }
#pragma unroll
  for (int c = 0; c < D; ++c) {
    R sd = tb<R>(0) * k[0][c].d;
#pragma unroll
    for (int j = 1; j < 6; ++j) sd += tb<R>(j) * k[j][c].d;
    yd[c] = yd[c] + h * sd;
  }
}

// Reverse-mode step of the Tsit5 replay map y_{n+1} = y_n + h sum_{i<=6} b_i k_i with h fixed:
// recompute the stages from the recorded y_n, then sweep them backwards.
//   kb_i = h (b_i lam + sum_{j>i} a_ji Yb_j),  Yb_i = J_y(Y_i)^T kb_i,  thb += J_th(Y_i)^T kb_i,
//   lam <- lam + sum_i Yb_i.   (b_7 = 0, so the seventh stage never enters the replay map.)
// Fields that declare TAPE > 0 hand the reverse sweep the transcendental part of f at each stage
// (kept in a per-lane shared-memory tape) instead of recomputing it in the VJP.

// tape: this lane's slot 0; slot (i, v) at tape[(i * TAPE + v) * tstride] (shared memory).
template <class F, class R>
__device__ __forceinline__ void tsit5_adjoint_step(const R (&y)[F::D], R h,
                                                   const typename F::template Theta<R>& th,
                                                   R (&lam)[F::D], R (&thb)[F::M],
                                                   R* tape = nullptr, int tstride = 0) {
  constexpr int D = F::D;
  constexpr int TP = TapeOf<F>::value;
  R Y[6][D];
  {
    R k[5][D];
#pragma unroll
    for (int c = 0; c < D; ++c) Y[0][c] = y[c];
    if constexpr (TP > 0) {
      R tp[TP > 0 ? TP : 1];
      F::f_tape(Y[0], th, k[0], tp);
#pragma unroll
      for (int v = 0; v < TP; ++v) tape[v * tstride] = tp[v];
    } else {
      F::f(Y[0], th, k[0]);
    }
#pragma unroll
    for (int i = 1; i < 6; ++i) {
#pragma unroll
      for (int c = 0; c < D; ++c) {
        R s = ta<R>(i, 0) * k[0][c];
#pragma unroll
        for (int j = 1; j < i; ++j) s += ta<R>(i, j) * k[j][c];
        Y[i][c] = y[c] + h * s;
      }
      if constexpr (TP > 0) {
        R tp[TP > 0 ? TP : 1];
        if (i < 5) F::f_tape(Y[i], th, k[i], tp);
        else F::inter_tape(Y[i], th, tp);
#pragma unroll
        for (int v = 0; v < TP; ++v) tape[(i * TP + v) * tstride] = tp[v];
      } else {
        if (i < 5) F::f(Y[i], th, k[i]);
      }
    }
  }
  // Reverse sweep.  Yb_j is kept for the stages j > i still to be visited, so that at every
  // point only six stage vectors are live (the Y_i not yet consumed plus the Yb_j already made).
  R Yb[6][D];
  R lnew[D];
#pragma unroll
  for (int c = 0; c < D; ++c) lnew[c] = lam[c];
#pragma unroll
  for (int i = 5; i >= 0; --i) {
    R kb[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R g = R(0);
#pragma unroll
      for (int j = i + 1; j < 6; ++j) g += ta<R>(j, i) * Yb[j][c];
      kb[c] = h * (tb<R>(i) * lam[c] + g);
    }
    if constexpr (TP > 0) {
      R tp[TP > 0 ? TP : 1];
#pragma unroll
      for (int v = 0; v < TP; ++v) tp[v] = tape[(i * TP + v) * tstride];
      F::vjp_tape(Y[i], th, tp, kb, Yb[i], thb);
    } else {
      F::vjp(Y[i], th, kb, Yb[i], thb);
    }
#pragma unroll
    for (int c = 0; c < D; ++c) lnew[c] += Yb[i][c];
  }
#pragma unroll
  for (int c = 0; c < D; ++c) lam[c] = lnew[c];
}

// ------------------------------------------------------------------------------------------------
// ROS34PW2: (I - gamma h J) k_i = h f(y + sum_{j<i} alpha_ij k_j) + h J sum_{j<i} gamma_ij k_j,
// y_{n+1} = y + sum b_i k_i, e = sum (b_i - bh_i) k_i, J = f_y(y_n) exact.
// ------------------------------------------------------------------------------------------------
struct Ros34pw2 {
  static constexpr int order = 3, err_order = 3;
  static constexpr double gamma = 0.435866521508459;
};
template <class R> __device__ __forceinline__ R ral(int i, int j) {
  constexpr double A[4][3] = {{0, 0, 0},
                              {0.87173304301691801, 0, 0},
                              {0.84457060015369423, -0.11299064236484185, 0},
                              {0, 0, 1.0}};
  return R(A[i][j]);
}
template <class R> __device__ __forceinline__ R rga(int i, int j) {
  constexpr double G[4][3] = {{0, 0, 0},
                              {-0.87173304301691801, 0, 0},
                              {-0.90338057013044082, 0.054180672388095326, 0},
                              {0.24212380706095346, -1.2232505839045147, 0.54526025533510214}};
  return R(G[i][j]);
}
template <class R> __device__ __forceinline__ R rb(int i) {
  constexpr double B[4] = {0.24212380706095346, -1.2232505839045147, 1.5452602553351020,
                           0.435866521508459};
  return R(B[i]);
}
// b_i - bhat_i
template <class R> __device__ __forceinline__ R rbe(int i) {
  constexpr double B[4] = {0.24212380706095346, -1.2232505839045147, 1.5452602553351020,
                           0.435866521508459};
  constexpr double BH[4] = {0.37810903145819369, -0.096042292212423178, 0.5, 0.2179332607542295};
  return R(B[i]) - R(BH[i]);
}

// Structural nonzeros of a field's Jacobian: every entry, unless the field declares its pattern
// with jac_nz(r, c) (false: J[r][c] is zero for every state and parameter).
template <class F, class = void>
struct JacPattern {
  static constexpr bool dense = true;
  GS_HD static constexpr bool nz(int, int) { return true; }
};
template <class F>
struct JacPattern<F, std::void_t<decltype(F::jac_nz(0, 0))>> {
  static constexpr bool dense = false;
  GS_HD static constexpr bool nz(int r, int c) { return F::jac_nz(r, c); }
};
// Entries of the LU factors of I - c J that elimination without row exchanges can make nonzero:
// J's pattern with the diagonal, closed under elimination (fill-in).
template <int D, class P>
GS_HD constexpr bool lu_nz(int r, int c) {
  bool f[D][D] = {};
  for (int i = 0; i < D; ++i)
    for (int j = 0; j < D; ++j) f[i][j] = i == j || P::nz(i, j);
  for (int col = 0; col < D; ++col)
    for (int i = col + 1; i < D; ++i)
      if (f[i][col])
        for (int j = col + 1; j < D; ++j)
          if (f[col][j]) f[i][j] = true;
  return f[r][c];
}
// fn(std::integral_constant<int, i>{}) for i = 0 .. N-1: loop indices usable in constant
// expressions (if constexpr on the pattern).
template <class Fn, int... I>
__device__ __forceinline__ void static_for_seq(Fn& fn, std::integer_sequence<int, I...>) {
  (fn(std::integral_constant<int, I>{}), ...);
}
template <int N, class Fn>
__device__ __forceinline__ void static_for(Fn&& fn) {
  static_for_seq(fn, std::make_integer_sequence<int, N>{});
}

// In-register LU of a D x D matrix with partial pivoting (largest |entry|, ties to the lowest
// row).  The permutation is kept as a row map p[] so that solves index without data movement.
// The pivots' reciprocals are formed once (the factorisation needs them anyway) and every solve
// multiplies by them: a Rosenbrock step solves three or four times with one factorisation, and
// an fp64 division costs several times a multiply on the FP64 pipe.
// The row exchanges are register-resident selects over whole rows (about 900 of them for an
// 8 x 8 matrix), so a column whose diagonal already holds the largest entry -- where partial
// pivoting exchanges nothing -- skips them after one comparison per row; and solves skip the
// row map while no exchange has been made.  The iteration matrices I - gamma h J of the stiff
// fields nearly never need one (none in 6,500 sampled steps of HIRES and Robertson, which keep
// their diagonal dominant), and the results are those of the exchanging code in every case.
// Every update is an explicit FMA, so that all kernels using it round alike.
// With a declared Jacobian pattern P (HIRES: 25 of 64 entries), factor_shifted takes the entries
// of the factors that can be nonzero only (the fill-in known at compile time, every loop index a
// constant): about a tenth of the dense elimination's operations for HIRES and a third of the
// solves', and a fraction of the registers.  It makes no row exchange: should partial pivoting
// want one at some column, ok turns false and the caller makes that step again with the dense
// LU (with_field_lu below) -- the same results as the dense code either way.
template <class R, int D, class P = JacPattern<void>>
struct SmallLU {
  R lu[D][D];
  R dinv[D];  // reciprocals of U's diagonal, formed once by factor(): the solves multiply
  int p[D];
  bool swapped;  // some row exchange was made: p is not the identity
  bool ok;  // patterned factorisation: no row exchange was wanted (always true when dense)

  // factors I - c J (J row-major, D x D)
  __device__ __forceinline__ void factor_shifted(const R (&J)[D * D], R c) {
    if constexpr (P::dense) {
      R A[D][D];
#pragma unroll
      for (int r = 0; r < D; ++r)
#pragma unroll
        for (int q = 0; q < D; ++q) A[r][q] = fma(-c, J[r * D + q], r == q ? R(1) : R(0));
      factor(A);
      ok = true;
    } else {
      static_for<D>([&](auto ri) {
        constexpr int r = decltype(ri)::value;
        static_for<D>([&](auto qi) {
          constexpr int q = decltype(qi)::value;
          if constexpr (lu_nz<D, P>(r, q)) {
            if constexpr (r == q || P::nz(r, q))
              lu[r][q] = fma(-c, J[r * D + q], r == q ? R(1) : R(0));
            else
              lu[r][q] = R(0);  // fill-in
          }
        });
      });
      bool need = false;
      static_for<D>([&](auto ci) {
        constexpr int col = decltype(ci)::value;
        static_for<D>([&](auto ri) {
          constexpr int r = decltype(ri)::value;
          if constexpr (r > col && lu_nz<D, P>(r, col))
            need = need || (fabs(lu[r][col]) > fabs(lu[col][col]));
        });
        const R inv = R(1) / lu[col][col];
        dinv[col] = inv;
        static_for<D>([&](auto ri) {
          constexpr int r = decltype(ri)::value;
          if constexpr (r > col && lu_nz<D, P>(r, col)) {
            const R l = lu[r][col] * inv;
            lu[r][col] = l;
            static_for<D>([&](auto qi) {
              constexpr int q = decltype(qi)::value;
              if constexpr (q > col && lu_nz<D, P>(col, q))
                lu[r][q] = fma(-l, lu[col][q], lu[r][q]);
            });
          }
        });
      });
      ok = !need;
    }
  }
  __device__ __forceinline__ void factor(const R (&A)[D][D]) {
    swapped = false;
#pragma unroll
    for (int r = 0; r < D; ++r) {
      p[r] = r;
#pragma unroll
      for (int c = 0; c < D; ++c) lu[r][c] = A[r][c];
    }
#pragma unroll
    for (int col = 0; col < D; ++col) {
      // choose the pivot among rows col..D-1 and swap it into place (register-resident selects),
      // only when some row below beats the diagonal
      bool need = false;
#pragma unroll
      for (int r = col + 1; r < D; ++r) need = need || (fabs(lu[r][col]) > fabs(lu[col][col]));
      if (need) {
        swapped = true;
#pragma unroll
        for (int r = col + 1; r < D; ++r) {
          if (fabs(lu[r][col]) > fabs(lu[col][col])) {
#pragma unroll
            for (int c = 0; c < D; ++c) { R tmp = lu[r][c]; lu[r][c] = lu[col][c]; lu[col][c] = tmp; }
            int t = p[r]; p[r] = p[col]; p[col] = t;
          }
        }
      }
      const R inv = R(1) / lu[col][col];
      dinv[col] = inv;
#pragma unroll
      for (int r = col + 1; r < D; ++r) {
        const R l = lu[r][col] * inv;
        lu[r][col] = l;
#pragma unroll
        for (int c = col + 1; c < D; ++c) lu[r][c] = fma(-l, lu[col][c], lu[r][c]);
      }
    }
  }
  // x = A^{-1} b   (P A = L U)
  __device__ __forceinline__ void solve(const R (&bb)[D], R (&x)[D]) const {
    if constexpr (!P::dense) {
#pragma unroll
      for (int r = 0; r < D; ++r) x[r] = bb[r];
      static_for<D>([&](auto ri) {
        constexpr int r = decltype(ri)::value;
        static_for<D>([&](auto qi) {
          constexpr int q = decltype(qi)::value;
          if constexpr (q < r && lu_nz<D, P>(r, q)) x[r] = fma(-lu[r][q], x[q], x[r]);
        });
      });
      static_for<D>([&](auto ki) {
        constexpr int r = D - 1 - decltype(ki)::value;
        static_for<D>([&](auto qi) {
          constexpr int q = decltype(qi)::value;
          if constexpr (q > r && lu_nz<D, P>(r, q)) x[r] = fma(-lu[r][q], x[q], x[r]);
        });
        x[r] = x[r] * dinv[r];
      });
    } else {
      if (swapped) {
#pragma unroll
        for (int r = 0; r < D; ++r) {
          R v = R(0);
#pragma unroll
          for (int s = 0; s < D; ++s) v = (p[r] == s) ? bb[s] : v;
          x[r] = v;
        }
      } else {
#pragma unroll
        for (int r = 0; r < D; ++r) x[r] = bb[r];
      }
#pragma unroll
      for (int r = 1; r < D; ++r)
#pragma unroll
        for (int c = 0; c < r; ++c) x[r] = fma(-lu[r][c], x[c], x[r]);
#pragma unroll
      for (int r = D - 1; r >= 0; --r) {
#pragma unroll
        for (int c = r + 1; c < D; ++c) x[r] = fma(-lu[r][c], x[c], x[r]);
        x[r] = x[r] * dinv[r];
      }
    }
  }
  // x = A^{-T} b:  A^T = U^T L^T P, so solve U^T z = b, L^T w = z, x = P^T w.
  __device__ __forceinline__ void solve_t(const R (&bb)[D], R (&x)[D]) const {
    if constexpr (!P::dense) {
      static_for<D>([&](auto ri) {
        constexpr int r = decltype(ri)::value;
        R v = bb[r];
        static_for<D>([&](auto qi) {
          constexpr int q = decltype(qi)::value;
          if constexpr (q < r && lu_nz<D, P>(q, r)) v = fma(-lu[q][r], x[q], v);
        });
        x[r] = v * dinv[r];
      });
      static_for<D>([&](auto ki) {
        constexpr int r = D - 1 - decltype(ki)::value;
        static_for<D>([&](auto qi) {
          constexpr int q = decltype(qi)::value;
          if constexpr (q > r && lu_nz<D, P>(q, r)) x[r] = fma(-lu[q][r], x[q], x[r]);
        });
      });
    } else {
      R z[D];
#pragma unroll
      for (int r = 0; r < D; ++r) {
        R v = bb[r];
#pragma unroll
        for (int c = 0; c < r; ++c) v = fma(-lu[c][r], z[c], v);
        z[r] = v * dinv[r];
      }
#pragma unroll
      for (int r = D - 1; r >= 0; --r)
#pragma unroll
        for (int c = r + 1; c < D; ++c) z[r] = fma(-lu[c][r], z[c], z[r]);
      if (swapped) {
#pragma unroll
        for (int s = 0; s < D; ++s) {
          R v = R(0);
#pragma unroll
          for (int r = 0; r < D; ++r) v = (p[r] == s) ? z[r] : v;
          x[s] = v;
        }
      } else {
#pragma unroll
        for (int s = 0; s < D; ++s) x[s] = z[s];
      }
    }
  }
};

// Runs step(lu) -- a Rosenbrock step that factors its iteration matrix into lu first and returns
// false, before writing any output, when lu reports that partial pivoting would exchange rows --
// with the LU of the field's Jacobian pattern, and again with the dense LU when that one would
// have exchanged rows.  Fields without a declared pattern take the dense LU only.
template <class F, class R, class Step>
__device__ __forceinline__ void with_field_lu(Step&& step) {
  if constexpr (JacPattern<F>::dense) {
    SmallLU<R, F::D> lu;
    step(lu);
  } else {
    SmallLU<R, F::D, JacPattern<F>> lu;
    if (!step(lu)) {
      SmallLU<R, F::D> ld;
      step(ld);
    }
  }
}

template <class F, class R, class LU>
__device__ __forceinline__ void ros_stages(const R (&y)[F::D], R h,
                                           const typename F::template Theta<R>& th,
                                           const R (&J)[F::D * F::D], const LU& lu,
                                           R (&k)[4][F::D]) {
  constexpr int D = F::D;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    R Y[D], G[D], fy[D], r[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R u = R(0), g = R(0);
#pragma unroll
      for (int j = 0; j < i; ++j) {
        u += ral<R>(i, j) * k[j][c];
        g += rga<R>(i, j) * k[j][c];
      }
      Y[c] = y[c] + u;
      G[c] = g;
    }
    F::f(Y, th, fy);
#pragma unroll
    for (int rr = 0; rr < D; ++rr) {
      R jg = R(0);
#pragma unroll
      for (int c = 0; c < D; ++c) jg += J[rr * D + c] * G[c];
      r[rr] = h * fy[rr] + h * jg;
    }
    lu.solve(r, k[i]);
  }
}

template <class F, class R, class LU>
__device__ __forceinline__ void ros_matrix(const R (&y)[F::D], R h,
                                           const typename F::template Theta<R>& th,
                                           R (&J)[F::D * F::D], LU& lu) {
  F::jac(y, th, J);
  lu.factor_shifted(J, R(Ros34pw2::gamma) * h);
}

template <class F, class R>
__device__ __forceinline__ R ros_trial(const R (&y)[F::D], R h,
                                       const typename F::template Theta<R>& th,
                                       R (&ynew)[F::D], R rtol, R atol) {
  constexpr int D = F::D;
  R err_out = R(0);
  with_field_lu<F, R>([&](auto& lu) {
    R J[D * D];
    ros_matrix<F, R>(y, h, th, J, lu);
    if (!lu.ok) return false;
    R k[4][D];
    ros_stages<F, R>(y, h, th, J, lu, k);
    R ev[D], sc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R s = rb<R>(0) * k[0][c];
      R e = rbe<R>(0) * k[0][c];
#pragma unroll
      for (int i = 1; i < 4; ++i) {
        s += rb<R>(i) * k[i][c];
        e += rbe<R>(i) * k[i][c];
      }
      ynew[c] = y[c] + s;
      ev[c] = e;
      sc[c] = atol + rtol * fmax(fabs(y[c]), fabs(ynew[c]));
    }
    err_out = scaled_rms(ev, sc);
    return true;
  });
  return err_out;
}

// The ROS34PW2 replay map (no error estimate).
template <class F, class R>
__device__ __forceinline__ void ros_replay_step(const R (&y)[F::D], R h,
                                                const typename F::template Theta<R>& th,
                                                R (&ynew)[F::D]) {
  constexpr int D = F::D;
  with_field_lu<F, R>([&](auto& lu) {
    R J[D * D];
    ros_matrix<F, R>(y, h, th, J, lu);
    if (!lu.ok) return false;
    R k[4][D];
    ros_stages<F, R>(y, h, th, J, lu, k);
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R s = rb<R>(0) * k[0][c];
#pragma unroll
      for (int i = 1; i < 4; ++i) s += rb<R>(i) * k[i][c];
      ynew[c] = y[c] + s;
    }
    return true;
  });
}

// ----------------------------------------------------------------------------------------------
// Rosenbrock23 (Shampine & Reichelt 1997, the pair of MATLAB's ode23s; "gradsolve: fast exact
// gradients for ODE ensembles on GPUs" §3.1: the second-order linearly implicit method of the
// fused stiff kernels), autonomous form with the exact J = f_y(y_n), d = 1/(2 + sqrt 2):
//   W = I - h d J;  F0 = f(y_n);  k1 = W^{-1} F0;  F1 = f(y_n + h k1/2);
//   k2 = W^{-1} (F1 - k1) + k1;  y_{n+1} = y_n + h k2;
//   F2 = f(y_{n+1});  k3 = W^{-1} (F2 - e32 (k2 - F1) - 2 (k1 - F0));  e = h (k1 - 2 k2 + k3)/6.
// F2 is the next step's F0 (first-same-as-last).
// ----------------------------------------------------------------------------------------------
struct Rb23 {
  static constexpr int order = 2, err_order = 3;
  static constexpr double d = 0.29289321881345248;    // 1 / (2 + sqrt 2)
  static constexpr double e32 = 7.4142135623730951;   // 6 + sqrt 2
};

template <class F, class R, class LU>
__device__ __forceinline__ void rb23_matrix(const R (&y)[F::D], R h,
                                            const typename F::template Theta<R>& th,
                                            R (&J)[F::D * F::D], LU& lu) {
  F::jac(y, th, J);
  lu.factor_shifted(J, h * R(Rb23::d));
}

// k1, F1 and k2 of the step from y (F0 = f(y) given).
template <class F, class R, class LU>
__device__ __forceinline__ void rb23_stages(const R (&y)[F::D], R h,
                                            const typename F::template Theta<R>& th,
                                            const LU& lu, const R (&F0)[F::D],
                                            R (&k1)[F::D], R (&F1)[F::D], R (&k2)[F::D]) {
  constexpr int D = F::D;
  lu.solve(F0, k1);
  R Y1[D], r[D];
#pragma unroll
  for (int c = 0; c < D; ++c) Y1[c] = y[c] + R(0.5) * h * k1[c];
  F::f(Y1, th, F1);
#pragma unroll
  for (int c = 0; c < D; ++c) r[c] = F1[c] - k1[c];
  lu.solve(r, k2);
#pragma unroll
  for (int c = 0; c < D; ++c) k2[c] = k2[c] + k1[c];
}

// One Rosenbrock23 trial from y with F0 = f(y) carried; returns the scaled RMS error and
// F2 = f(y_new) (the next F0 when the step is accepted).
template <class F, class R>
__device__ __forceinline__ R rb23_trial(const R (&y)[F::D], R h,
                                        const typename F::template Theta<R>& th,
                                        const R (&F0)[F::D], R (&ynew)[F::D], R (&F2)[F::D],
                                        R rtol, R atol) {
  constexpr int D = F::D;
  R err_out = R(0);
  with_field_lu<F, R>([&](auto& lu) {
    R J[D * D];
    rb23_matrix<F, R>(y, h, th, J, lu);
    if (!lu.ok) return false;
    R k1[D], F1[D], k2[D];
    rb23_stages<F, R>(y, h, th, lu, F0, k1, F1, k2);
#pragma unroll
    for (int c = 0; c < D; ++c) ynew[c] = y[c] + h * k2[c];
    F::f(ynew, th, F2);
    R r[D], k3[D];
#pragma unroll
    for (int c = 0; c < D; ++c)
      r[c] = F2[c] - R(Rb23::e32) * (k2[c] - F1[c]) - R(2) * (k1[c] - F0[c]);
    lu.solve(r, k3);
    R ev[D], sc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      const R e = h * (k1[c] - R(2) * k2[c] + k3[c]) * R(1.0 / 6.0);
      ev[c] = e;
      sc[c] = atol + rtol * fmax(fabs(y[c]), fabs(ynew[c]));
    }
    err_out = scaled_rms(ev, sc);
    return true;
  });
  return err_out;
}

// The Rosenbrock23 replay map y + h k2 (no error estimate).
template <class F, class R>
__device__ __forceinline__ void rb23_replay_step(const R (&y)[F::D], R h,
                                                 const typename F::template Theta<R>& th,
                                                 R (&ynew)[F::D]) {
  constexpr int D = F::D;
  with_field_lu<F, R>([&](auto& lu) {
    R J[D * D];
    rb23_matrix<F, R>(y, h, th, J, lu);
    if (!lu.ok) return false;
    R F0[D], k1[D], F1[D], k2[D];
    F::f(y, th, F0);
    rb23_stages<F, R>(y, h, th, lu, F0, k1, F1, k2);
#pragma unroll
    for (int c = 0; c < D; ++c) ynew[c] = y[c] + h * k2[c];
    return true;
  });
}

// Reverse-mode step of the Rosenbrock23 replay map with h fixed.  With u = k2 - k1
// (W u = F1 - k1) and lam the cotangent of y_{n+1}:
//   k2b = h lam;  mu2 = W^{-T} k2b;  F1b = mu2;  k1b = k2b - mu2;  Jb = h d mu2 u^T
//   Y1b = J_y(Y1)^T mu2 (thb += J_th(Y1)^T mu2);  yb = lam + Y1b;  k1b += h Y1b / 2
//   mu1 = W^{-T} k1b;  Jb += h d mu1 k1^T;  yb += J_y(y)^T mu1 (thb += J_th(y)^T mu1)
//   yb += Jb : dJ/dy,  thb += Jb : dJ/dtheta;   lam <- yb.
template <class F, class R>
__device__ __forceinline__ void rb23_adjoint_step(const R (&y)[F::D], R h,
                                                  const typename F::template Theta<R>& th,
                                                  R (&lam)[F::D], R (&thb)[F::M]) {
  constexpr int D = F::D;
  with_field_lu<F, R>([&](auto& lu) {
    R J[D * D];
    rb23_matrix<F, R>(y, h, th, J, lu);
    if (!lu.ok) return false;
    R F0[D], k1[D], F1[D], k2[D];
    F::f(y, th, F0);
    rb23_stages<F, R>(y, h, th, lu, F0, k1, F1, k2);
    const R hd = h * R(Rb23::d);
    R Jb[D * D], yb[D], k2b[D], mu[D], k1b[D], tmp[D];
#pragma unroll
    for (int c = 0; c < D; ++c) { yb[c] = lam[c]; k2b[c] = h * lam[c]; }
    lu.solve_t(k2b, mu);                               // mu2
#pragma unroll
    for (int r = 0; r < D; ++r)
#pragma unroll
      for (int c = 0; c < D; ++c) Jb[r * D + c] = hd * mu[r] * (k2[c] - k1[c]);
    R Y1[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      k1b[c] = k2b[c] - mu[c];
      Y1[c] = y[c] + R(0.5) * h * k1[c];
    }
    F::vjp(Y1, th, mu, tmp, thb);                      // Y1b
#pragma unroll
    for (int c = 0; c < D; ++c) {
      yb[c] += tmp[c];
      k1b[c] += R(0.5) * h * tmp[c];
    }
    lu.solve_t(k1b, mu);                               // mu1
#pragma unroll
    for (int r = 0; r < D; ++r)
#pragma unroll
      for (int c = 0; c < D; ++c) Jb[r * D + c] += hd * mu[r] * k1[c];
    F::vjp(y, th, mu, tmp, thb);
#pragma unroll
    for (int c = 0; c < D; ++c) yb[c] += tmp[c];
    F::jac_vjp(y, th, Jb, yb, thb);
#pragma unroll
    for (int c = 0; c < D; ++c) lam[c] = yb[c];
    return true;
  });
}

// Reverse-mode step of the ROS34PW2 replay map with h fixed.  With M = I - gamma h J,
// r_i = h f(Y_i) + h J G_i, M k_i = r_i, the backward pass for stage i = 4..1 is
//   mu_i = M^{-T} kb_i                          (one transpose solve, same LU)
//   Jb  += gamma h mu_i k_i^T + h mu_i G_i^T     (M depends on J; r_i depends on J)
//   fb_i = h mu_i -> Yb_i = J_y(Y_i)^T fb_i, thb += J_th(Y_i)^T fb_i
//   kb_j += alpha_ij Yb_i + gamma_ij h J^T mu_i   for j < i
//   yb  += Yb_i
// and finally yb += Jb : dJ/dy, thb += Jb : dJ/dtheta; lam <- yb (with yb starting at lam).
template <class F, class R>
__device__ __forceinline__ void ros_adjoint_step(const R (&y)[F::D], R h,
                                                 const typename F::template Theta<R>& th,
                                                 R (&lam)[F::D], R (&thb)[F::M]) {
  constexpr int D = F::D;
  with_field_lu<F, R>([&](auto& lu) {
    R J[D * D];
    ros_matrix<F, R>(y, h, th, J, lu);
    if (!lu.ok) return false;
    R k[4][D];
    ros_stages<F, R>(y, h, th, J, lu, k);
    R kb[4][D], Jb[D * D], yb[D];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < D; ++c) kb[i][c] = rb<R>(i) * lam[c];
#pragma unroll
    for (int i = 0; i < D * D; ++i) Jb[i] = R(0);
#pragma unroll
    for (int c = 0; c < D; ++c) yb[c] = lam[c];
    const R gh = R(Ros34pw2::gamma) * h;
#pragma unroll
    for (int i = 3; i >= 0; --i) {
      R mu[D];
      lu.solve_t(kb[i], mu);
      R Y[D], G[D];
#pragma unroll
      for (int c = 0; c < D; ++c) {
        R u = R(0), g = R(0);
#pragma unroll
        for (int j = 0; j < i; ++j) {
          u += ral<R>(i, j) * k[j][c];
          g += rga<R>(i, j) * k[j][c];
        }
        Y[c] = y[c] + u;
        G[c] = g;
      }
#pragma unroll
      for (int r = 0; r < D; ++r)
#pragma unroll
        for (int c = 0; c < D; ++c) Jb[r * D + c] += mu[r] * (gh * k[i][c] + h * G[c]);
      R fb[D], Yb[D];
#pragma unroll
      for (int c = 0; c < D; ++c) fb[c] = h * mu[c];
      F::vjp(Y, th, fb, Yb, thb);
      if (i > 0) {
        R Jtmu[D];
#pragma unroll
        for (int c = 0; c < D; ++c) {
          R s = R(0);
#pragma unroll
          for (int r = 0; r < D; ++r) s += J[r * D + c] * mu[r];
          Jtmu[c] = h * s;
        }
#pragma unroll
        for (int j = 0; j < i; ++j)
#pragma unroll
          for (int c = 0; c < D; ++c)
            kb[j][c] += ral<R>(i, j) * Yb[c] + rga<R>(i, j) * Jtmu[c];
      }
#pragma unroll
      for (int c = 0; c < D; ++c) yb[c] += Yb[c];
    }
    F::jac_vjp(y, th, Jb, yb, thb);
#pragma unroll
    for (int c = 0; c < D; ++c) lam[c] = yb[c];
    return true;
  });
}

}  // namespace gs
