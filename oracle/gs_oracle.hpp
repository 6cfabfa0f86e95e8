// gs_oracle.hpp -- the CPU oracle: a plain, slow, obviously correct statement of what the
// record-and-replay discrete adjoint computes.  TEST INFRASTRUCTURE ONLY: the test suite, the
// smoke check and the benchmark's CPU-baseline leg are the only callers.  It shares no code,
// header, table or helper with the CUDA library; the two meet only through seeded input arrays.
//
// Sources (cited as "page title, section"):
//   [GS]  "gradsolve: fast exact gradients for ODE ensembles on GPUs"
//         §2.1 adaptive solve (embedded pair, RMS error test, reject-and-retry),
//         §2.2 scalar loss whose parameter gradient flows only through the solves,
//         §3   record (accepted step sizes) and replay (fixed-step chain Psi, Eq. 4) with the
//              stop-gradient mesh; §3.2 Rosenbrock one-step map (I - gamma h J) and the
//              transpose-solve rule; §3.3 in-kernel adjoint keeps one accepted state per step.
//   [DA]  "Differentiable astrophysics at scale", §3 stellar orbits (energy / angular momentum
//         conservation as a check).
//   Coefficients that the pages do not print come from the published methods they name:
//   Tsitouras (2011), Comput. Math. Appl. 62, 770 (Tsit5 pair); Rang & Angermann (2005),
//   BIT 45, 761 (ROS34PW2); Hairer, Norsett & Wanner, Solving ODEs I, §II.4 (starting step).
//
// What each routine is:
//   * fields            : the right-hand sides f(y; theta), written once, templated on the scalar
//                         so that they run in double, float, dual numbers and an op counter.
//   * tsit5_trial/ros_trial : one trial step of the method in the method's own textbook form.
//   * solve             : the adaptive loop (initial step, RMS test, I-controller, reject/retry),
//                         keeping the accepted (t_n, h_n, y_n): the record.
//   * replay            : the chain of one-step maps over a given mesh h_0..h_{S-1}.
//   * replay_grad       : the gradient of the replay by its plain definition -- the Jacobian of
//                         y_S with respect to (y0, theta), obtained by pushing forward-mode dual
//                         numbers through the replay, contracted with dL/dy_S.  This is not the
//                         reverse sweep the GPU runs; it reaches the same number by another road.
// Every routine here is pinned by the tests in tests/test_oracle_*.py against closed forms,
// order conditions, invariants, brute force and finite differences.
#pragma once
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <limits>
#include <type_traits>
#include <vector>

namespace orc {

// ------------------------------------------------------------------------------------------
// Scalars.  Dual<R,P> carries a value and P directional derivatives (forward-mode AD).
// ------------------------------------------------------------------------------------------
template <class R, int P>
struct Dual {
  R v;
  R g[P];
  Dual() : v(0) { for (int i = 0; i < P; ++i) g[i] = 0; }
  Dual(R x) : v(x) { for (int i = 0; i < P; ++i) g[i] = 0; }
};

template <class T> struct base_of { using type = T; };
template <class R, int P> struct base_of<Dual<R, P>> { using type = R; };

template <class R, int P>
inline Dual<R, P> operator+(const Dual<R, P>& a, const Dual<R, P>& b) {
  Dual<R, P> c;
  c.v = a.v + b.v;
  for (int i = 0; i < P; ++i) c.g[i] = a.g[i] + b.g[i];
  return c;
}
template <class R, int P>
inline Dual<R, P> operator-(const Dual<R, P>& a, const Dual<R, P>& b) {
  Dual<R, P> c;
  c.v = a.v - b.v;
  for (int i = 0; i < P; ++i) c.g[i] = a.g[i] - b.g[i];
  return c;
}
template <class R, int P>
inline Dual<R, P> operator-(const Dual<R, P>& a) {
  Dual<R, P> c;
  c.v = -a.v;
  for (int i = 0; i < P; ++i) c.g[i] = -a.g[i];
  return c;
}
template <class R, int P>
inline Dual<R, P> operator*(const Dual<R, P>& a, const Dual<R, P>& b) {
  Dual<R, P> c;
  c.v = a.v * b.v;
  for (int i = 0; i < P; ++i) c.g[i] = a.g[i] * b.v + a.v * b.g[i];
  return c;
}
template <class R, int P>
inline Dual<R, P> operator/(const Dual<R, P>& a, const Dual<R, P>& b) {
  Dual<R, P> c;
  c.v = a.v / b.v;
  for (int i = 0; i < P; ++i) c.g[i] = (a.g[i] - c.v * b.g[i]) / b.v;
  return c;
}
// d sqrt(u) = du / (2 sqrt(u)),  d log1p(u) = du / (1 + u),  d tanh(u) = (1 - tanh(u)^2) du.
template <class R, int P>
inline Dual<R, P> sqrt(const Dual<R, P>& a) {
  Dual<R, P> c;
  using std::sqrt;  // plain scalars, or the op counter through argument lookup
  c.v = sqrt(a.v);
  const R d = R(1) / (R(2) * c.v);
  for (int i = 0; i < P; ++i) c.g[i] = a.g[i] * d;
  return c;
}
template <class R, int P>
inline Dual<R, P> log1p(const Dual<R, P>& a) {
  Dual<R, P> c;
  using std::log1p;  // plain scalars, or the op counter through argument lookup
  c.v = log1p(a.v);
  const R d = R(1) / (R(1) + a.v);
  for (int i = 0; i < P; ++i) c.g[i] = a.g[i] * d;
  return c;
}
template <class R, int P>
inline Dual<R, P> tanh(const Dual<R, P>& a) {
  Dual<R, P> c;
  using std::tanh;  // plain scalars, or the op counter through argument lookup
  c.v = tanh(a.v);
  const R d = R(1) - c.v * c.v;
  for (int i = 0; i < P; ++i) c.g[i] = a.g[i] * d;
  return c;
}
template <class R, int P> inline R value_of(const Dual<R, P>& a) { return a.v; }
inline double value_of(double a) { return a; }
inline float value_of(float a) { return a; }

using std::log1p;
using std::sqrt;
using std::tanh;

// A coefficient given as a decimal is first rounded to the working precision R, then lifted.
template <class T> inline T cst(double c) { return T(typename base_of<T>::type(c)); }

// ------------------------------------------------------------------------------------------
// Op counter: a double that counts the arithmetic done on it (used to state algorithmic flops).
// ------------------------------------------------------------------------------------------
struct OpTally { long long add = 0, mul = 0, div = 0, sqrt = 0, log1p = 0, tanh = 0; };
inline OpTally& tally() { static thread_local OpTally t; return t; }
struct Cnt {
  double v;
  Cnt() : v(0) {}
  Cnt(double x) : v(x) {}
};
template <> struct base_of<Cnt> { using type = double; };
inline Cnt operator+(Cnt a, Cnt b) { tally().add++; return Cnt(a.v + b.v); }
inline Cnt operator-(Cnt a, Cnt b) { tally().add++; return Cnt(a.v - b.v); }
inline Cnt operator-(Cnt a) { return Cnt(-a.v); }
inline Cnt operator*(Cnt a, Cnt b) { tally().mul++; return Cnt(a.v * b.v); }
inline Cnt operator/(Cnt a, Cnt b) { tally().div++; return Cnt(a.v / b.v); }
inline Cnt sqrt(Cnt a) { tally().sqrt++; return Cnt(std::sqrt(a.v)); }
inline Cnt log1p(Cnt a) { tally().log1p++; return Cnt(std::log1p(a.v)); }
inline Cnt tanh(Cnt a) { tally().tanh++; return Cnt(std::tanh(a.v)); }
inline double value_of(Cnt a) { return a.v; }

// ------------------------------------------------------------------------------------------
// Reverse-mode tape: a double that records every operation whose result depends on a marked
// input, so that the work of a plain reverse sweep (the definitional pullback of f, adjoints
// accumulated into zero-initialised slots) can be tallied.  Used to bound the operation count of
// a vector-Jacobian product independently of any hand-written one.
// ------------------------------------------------------------------------------------------
enum TapOp { TAP_LEAF, TAP_ADD, TAP_SUB, TAP_NEG, TAP_MUL, TAP_DIV, TAP_SQRT, TAP_LOG1P, TAP_TANH };
struct TapNode { TapOp op; int a, b; };
inline std::vector<TapNode>& tape() { static thread_local std::vector<TapNode> t; return t; }
struct Tap {
  double v;
  int id;  // node on the tape, -1 for a value that depends on no marked input
  Tap() : v(0), id(-1) {}
  Tap(double x) : v(x), id(-1) {}
  static Tap leaf(double x) {
    tape().push_back({TAP_LEAF, -1, -1});
    Tap t(x);
    t.id = (int)tape().size() - 1;
    return t;
  }
};
template <> struct base_of<Tap> { using type = double; };
inline Tap tap_node(double v, TapOp op, int a, int b) {
  Tap t(v);
  if (a < 0 && b < 0) return t;
  tape().push_back({op, a, b});
  t.id = (int)tape().size() - 1;
  return t;
}
inline Tap operator+(Tap a, Tap b) { return tap_node(a.v + b.v, TAP_ADD, a.id, b.id); }
inline Tap operator-(Tap a, Tap b) { return tap_node(a.v - b.v, TAP_SUB, a.id, b.id); }
inline Tap operator-(Tap a) { return tap_node(-a.v, TAP_NEG, a.id, -1); }
inline Tap operator*(Tap a, Tap b) { return tap_node(a.v * b.v, TAP_MUL, a.id, b.id); }
inline Tap operator/(Tap a, Tap b) { return tap_node(a.v / b.v, TAP_DIV, a.id, b.id); }
inline Tap sqrt(Tap a) { return tap_node(std::sqrt(a.v), TAP_SQRT, a.id, -1); }
inline Tap log1p(Tap a) { return tap_node(std::log1p(a.v), TAP_LOG1P, a.id, -1); }
inline Tap tanh(Tap a) { return tap_node(std::tanh(a.v), TAP_TANH, a.id, -1); }
inline double value_of(Tap a) { return a.v; }

// Operations of the reverse sweep over the tape, from the given output nodes back to the leaves,
// for the nodes on a path between them.  Per node, with z its result and zb its adjoint:
//   z = a +- b:  ab += zb, bb +-= zb                  1 add per marked operand
//   z = -a:      ab -= zb                             1 add
//   z = a b:     ab += zb b, bb += zb a               1 mul + 1 add per marked operand
//   z = a / b:   t = zb / b;  ab += t;  bb -= t z     1 div, + 1 add (a), + 1 mul + 1 add (b)
//   z = sqrt a:  ab += 0.5 (zb / z)                   1 div + 1 mul + 1 add
//   z = log1p a: ab += zb / (1 + a)                   2 add + 1 div
//   z = tanh a:  ab += zb (1 - z z)                   2 mul + 2 add
inline OpTally tally_reverse_sweep(const int* outputs, int nout) {
  const std::vector<TapNode>& t = tape();
  std::vector<char> live(t.size(), 0);
  for (int i = 0; i < nout; ++i)
    if (outputs[i] >= 0) live[outputs[i]] = 1;
  OpTally c;
  for (int n = (int)t.size() - 1; n >= 0; --n) {
    if (!live[n]) continue;
    const TapNode& d = t[n];
    const bool ua = d.a >= 0, ub = d.b >= 0;
    if (ua) live[d.a] = 1;
    if (ub) live[d.b] = 1;
    switch (d.op) {
      case TAP_LEAF: break;
      case TAP_ADD: case TAP_SUB: c.add += ua + ub; break;
      case TAP_NEG: c.add += 1; break;
      case TAP_MUL: c.mul += ua + ub; c.add += ua + ub; break;
      case TAP_DIV: c.div += 1; c.add += ua + ub; c.mul += ub; break;
      case TAP_SQRT: c.div += 1; c.mul += 1; c.add += 1; break;
      case TAP_LOG1P: c.add += 2; c.div += 1; break;
      case TAP_TANH: c.mul += 2; c.add += 2; break;
    }
  }
  return c;
}

// ------------------------------------------------------------------------------------------
// Fields.  Each is autonomous: dy/dt = f(y; theta).  D = state size, M = parameter count.
// ------------------------------------------------------------------------------------------

// Lotka-Volterra, theta = (alpha, beta, gamma, delta):  x' = alpha x - beta x y,
// y' = delta x y - gamma y.
struct LotkaVolterra {
  static constexpr int D = 2, M = 4;
  template <class T> static void f(const T* y, const T* th, T* dy) {
    dy[0] = th[0] * y[0] - th[1] * y[0] * y[1];
    dy[1] = th[3] * y[0] * y[1] - th[2] * y[1];
  }
};

// Lorenz-63 ([GS] §4.3 benchmark system), theta = (sigma, rho, beta).
struct Lorenz63 {
  static constexpr int D = 3, M = 3;
  template <class T> static void f(const T* y, const T* th, T* dy) {
    dy[0] = th[0] * (y[1] - y[0]);
    dy[1] = y[0] * (th[1] - y[2]) - y[1];
    dy[2] = y[0] * y[1] - th[2] * y[2];
  }
};

// Robertson kinetics ([GS] §4.2, §4.5 stiff system), theta = (k1, k2, k3).
struct Robertson {
  static constexpr int D = 3, M = 3;
  template <class T> static void f(const T* y, const T* th, T* dy) {
    dy[0] = -(th[0] * y[0]) + th[2] * y[1] * y[2];
    dy[1] = th[0] * y[0] - th[1] * y[1] * y[1] - th[2] * y[1] * y[2];
    dy[2] = th[1] * y[1] * y[1];
  }
  // J = df/dy, row-major J[r*D + c] = d f_r / d y_c (written out from f above).
  template <class T> static void jac(const T* y, const T* th, T* J) {
    J[0] = -th[0];  J[1] = th[2] * y[2];                              J[2] = th[2] * y[1];
    J[3] = th[0];   J[4] = -(cst<T>(2.0) * th[1] * y[1]) - th[2] * y[2]; J[5] = -(th[2] * y[1]);
    J[6] = T(0);    J[7] = cst<T>(2.0) * th[1] * y[1];                 J[8] = T(0);
  }
};

// HIRES (Schaefer 1975; Hairer & Wanner II, §IV.10: "high irradiance responses" of
// photomorphogenesis), the stiff eight-component system of [GS] §4.5 / §4.6.  The twelve rate
// constants are the parameters, theta = (k1..k12), nominal
//   (1.71, 0.43, 8.32, 0.0007, 8.75, 10.03, 0.035, 1.12, 1.745, 280, 0.69, 1.81):
//   y1' = -k1 y1 + k2 y2 + k3 y3 + k4
//   y2' =  k1 y1 - k5 y2
//   y3' = -k6 y3 + k2 y4 + k7 y5
//   y4' =  k3 y2 + k1 y3 - k8 y4
//   y5' = -k9 y5 + k2 y6 + k2 y7
//   y6' = -k10 y6 y8 + k11 y4 + k1 y5 - k2 y6 + k11 y7
//   y7' =  k10 y6 y8 - k12 y7
//   y8' = -k10 y6 y8 + k12 y7
struct Hires {
  static constexpr int D = 8, M = 12;
  template <class T> static void f(const T* y, const T* k, T* dy) {
    const T r = k[9] * y[5] * y[7];
    dy[0] = -(k[0] * y[0]) + k[1] * y[1] + k[2] * y[2] + k[3];
    dy[1] = k[0] * y[0] - k[4] * y[1];
    dy[2] = -(k[5] * y[2]) + k[1] * y[3] + k[6] * y[4];
    dy[3] = k[2] * y[1] + k[0] * y[2] - k[7] * y[3];
    dy[4] = -(k[8] * y[4]) + k[1] * y[5] + k[1] * y[6];
    dy[5] = -r + k[10] * y[3] + k[0] * y[4] - k[1] * y[5] + k[10] * y[6];
    dy[6] = r - k[11] * y[6];
    dy[7] = -r + k[11] * y[6];
  }
  // J = df/dy, row-major, written out from f above.
  template <class T> static void jac(const T* y, const T* k, T* J) {
    for (int i = 0; i < 64; ++i) J[i] = T(0);
    J[0 * 8 + 0] = -k[0]; J[0 * 8 + 1] = k[1];  J[0 * 8 + 2] = k[2];
    J[1 * 8 + 0] = k[0];  J[1 * 8 + 1] = -k[4];
    J[2 * 8 + 2] = -k[5]; J[2 * 8 + 3] = k[1];  J[2 * 8 + 4] = k[6];
    J[3 * 8 + 1] = k[2];  J[3 * 8 + 2] = k[0];  J[3 * 8 + 3] = -k[7];
    J[4 * 8 + 4] = -k[8]; J[4 * 8 + 5] = k[1];  J[4 * 8 + 6] = k[1];
    J[5 * 8 + 3] = k[10]; J[5 * 8 + 4] = k[0];  J[5 * 8 + 5] = -(k[9] * y[7]) - k[1];
    J[5 * 8 + 6] = k[10]; J[5 * 8 + 7] = -(k[9] * y[5]);
    J[6 * 8 + 5] = k[9] * y[7]; J[6 * 8 + 6] = -k[11]; J[6 * 8 + 7] = k[9] * y[5];
    J[7 * 8 + 5] = -(k[9] * y[7]); J[7 * 8 + 6] = k[11]; J[7 * 8 + 7] = -(k[9] * y[5]);
  }
};

// Test particle in an NFW halo plus a Miyamoto-Nagai disk, G = 1; state (x, y, z, vx, vy, vz),
// theta = (M_h, r_s, M_d, a, b).
//   Phi = -M_h ln(1 + r/r_s)/r  -  M_d / sqrt(R^2 + (a + sqrt(z^2 + b^2))^2),  x'' = -grad Phi.
// The NFW radial force written out:  -grad Phi_NFW = -M_h [ln(1+r/r_s)/r^3 - 1/(r^2 (r_s+r))] x.
// The Miyamoto-Nagai force:  -grad Phi_MN = -M_d/D^3 (x, y, z (a+B)/B),  B = sqrt(z^2+b^2),
// D^2 = R^2 + (a+B)^2.  (Stellar-orbit workload shaped like [DA] §3, with the potential of the
// benchmark configuration.)
struct NfwMiyamotoNagai {
  static constexpr int D = 6, M = 5;
  template <class T> static void f(const T* y, const T* th, T* dy) {
    const T x = y[0], yy = y[1], z = y[2];
    const T Mh = th[0], rs = th[1], Md = th[2], a = th[3], b = th[4];
    const T R2 = x * x + yy * yy;
    const T r2 = R2 + z * z;
    const T r = sqrt(r2);
    const T gN = Mh * (log1p(r / rs) / (r2 * r) - T(1) / (r2 * (rs + r)));
    const T B = sqrt(z * z + b * b);
    const T apB = a + B;
    const T D2 = R2 + apB * apB;
    const T D = sqrt(D2);
    const T gM = Md / (D2 * D);
    dy[0] = y[3];
    dy[1] = y[4];
    dy[2] = y[5];
    dy[3] = -((gN + gM) * x);
    dy[4] = -((gN + gM) * yy);
    dy[5] = -((gN + gM * apB / B) * z);
  }
};

// Test particle in an axisymmetric flattened logarithmic halo ([DA] §3; the same potential as
// the halo-flattening study of [GS] §4.5):  Phi = (1/2) v_c^2 ln(R_c^2 + x^2 + y^2 + z^2/q^2),
// state (x, y, z, vx, vy, vz), theta = (v_c, q) shared by the stars, core radius R_c = 0.2 fixed
// (the pages' value; the two differentiated parameters are v_c and q).  -grad Phi written out:
//   -v_c^2 (x, y, z/q^2) / (R_c^2 + x^2 + y^2 + z^2/q^2).
struct LogHalo {
  static constexpr int D = 6, M = 2;
  static constexpr double Rc = 0.2;
  template <class T> static void f(const T* y, const T* th, T* dy) {
    const T x = y[0], yy = y[1], z = y[2];
    const T vc = th[0], q = th[1];
    const T zq = z / q;
    const T Q = cst<T>(Rc * Rc) + x * x + yy * yy + zq * zq;
    const T g = vc * vc / Q;
    dy[0] = y[3];
    dy[1] = y[4];
    dy[2] = y[5];
    dy[3] = -(g * x);
    dy[4] = -(g * yy);
    dy[5] = -(g * (zq / q));
  }
};

// Neural right-hand side: f(y) = W3 tanh(W2 tanh(W1 y + b1) + b2) + b3, sizes 4 -> 32 -> 32 -> 4,
// all layers with biases ([GS] §2.2: m runs to thousands of weights for a neural RHS).
// Parameter vector layout (row-major, W[out][in]):
//   W1 at 0 (32x4), b1 at 128, W2 at 160 (32x32), b2 at 1184, W3 at 1216 (4x32), b3 at 1344.
struct Mlp4x32x32x4 {
  static constexpr int D = 4, H = 32, M = 1348;
  static constexpr int oW1 = 0, ob1 = 128, oW2 = 160, ob2 = 1184, oW3 = 1216, ob3 = 1344;
  template <class T> static void f(const T* y, const T* th, T* dy) {
    T h1[H], h2[H];
    for (int i = 0; i < H; ++i) {
      T acc = th[ob1 + i];
      for (int j = 0; j < D; ++j) acc = acc + th[oW1 + i * D + j] * y[j];
      h1[i] = tanh(acc);
    }
    for (int i = 0; i < H; ++i) {
      T acc = th[ob2 + i];
      for (int j = 0; j < H; ++j) acc = acc + th[oW2 + i * H + j] * h1[j];
      h2[i] = tanh(acc);
    }
    for (int i = 0; i < D; ++i) {
      T acc = th[ob3 + i];
      for (int j = 0; j < H; ++j) acc = acc + th[oW3 + i * H + j] * h2[j];
      dy[i] = acc;
    }
  }
};

// Linear test family y' = A y with theta = A (row-major, DxD); its Jacobian is A itself.
// ([GS] §4.6-4.7: the linear family with a closed-form sensitivity.)
template <int DD>
struct Linear {
  static constexpr int D = DD, M = DD * DD;
  template <class T> static void f(const T* y, const T* th, T* dy) {
    for (int r = 0; r < D; ++r) {
      T acc = T(0);
      for (int c = 0; c < D; ++c) acc = acc + th[r * D + c] * y[c];
      dy[r] = acc;
    }
  }
  template <class T> static void jac(const T* /*y*/, const T* th, T* J) {
    for (int i = 0; i < D * D; ++i) J[i] = th[i];
  }
};

// ------------------------------------------------------------------------------------------
// Tsit5 (Tsitouras 2011, 5(4) pair, 7 stages, first-same-as-last).  The pages fix the
// structure ([GS] §2.1 and §3: s = 7, the last stage reused as the next first stage); the
// decimals are the published ones.  A[i][j] for stage i (0-based) from stage j < i; the last
// row equals b (stiffly the step result); BT = b - b_hat gives the error estimate e.
// ------------------------------------------------------------------------------------------
struct Tsit5Tab {
  static constexpr int S = 7;
  static constexpr int order = 5;       // order used by the starting-step rule
  static constexpr int err_order = 5;   // embedded order + 1, the controller's q
  static constexpr double C[7] = {0.0, 0.161, 0.327, 0.9, 0.9800255409045097, 1.0, 1.0};
  static constexpr double A[7][6] = {
      {0, 0, 0, 0, 0, 0},
      {0.161, 0, 0, 0, 0, 0},
      {-0.008480655492356989, 0.335480655492357, 0, 0, 0, 0},
      {2.897153057105493, -6.359448489975075, 4.3622954328695815, 0, 0, 0},
      {5.325864828439257, -11.748883564062828, 7.4955393428898365, -0.09249506636175525, 0, 0},
      {5.86145544294642, -12.92096931784711, 8.159367898576159, -0.071584973281401,
       -0.028269050394068383, 0},
      {0.09646076681806523, 0.01, 0.4798896504144996, 1.379008574103742, -3.290069515436081,
       2.324710524099774}};
  static constexpr double B[7] = {0.09646076681806523, 0.01, 0.4798896504144996,
                                  1.379008574103742, -3.290069515436081, 2.324710524099774, 0.0};
  static constexpr double BT[7] = {-0.00178001105222577714, -0.0008164344596567469,
                                   0.007880878010261995, -0.1447110071732629,
                                   0.5823571654525552, -0.45808210592918697,
                                   0.015151515151515152};  // last entry 1/66
};

// ROS34PW2 (Rang & Angermann 2005): 4 stages, order 3, embedded order 2, L-stable,
// stiffly accurate.  Hairer-Wanner form with exact J = f_y(y_n):
//   (I - gamma h J) k_i = h f(y_n + sum_{j<i} ALPHA_ij k_j) + h J sum_{j<i} GAMMA_ij k_j,
//   y_{n+1} = y_n + sum_i B_i k_i,   e = sum_i (B_i - BHAT_i) k_i.
struct Ros34pw2Tab {
  static constexpr int S = 4;
  static constexpr int order = 3;
  static constexpr int err_order = 3;
  static constexpr double gamma = 0.435866521508459;
  static constexpr double ALPHA[4][3] = {{0, 0, 0},
                                         {0.87173304301691801, 0, 0},
                                         {0.84457060015369423, -0.11299064236484185, 0},
                                         {0, 0, 1.0}};
  static constexpr double GAMMA[4][3] = {{0, 0, 0},
                                         {-0.87173304301691801, 0, 0},
                                         {-0.90338057013044082, 0.054180672388095326, 0},
                                         {0.24212380706095346, -1.2232505839045147,
                                          0.54526025533510214}};
  static constexpr double B[4] = {0.24212380706095346, -1.2232505839045147, 1.5452602553351020,
                                  0.435866521508459};
  static constexpr double BHAT[4] = {0.37810903145819369, -0.096042292212423178, 0.5,
                                     0.2179332607542295};
};

// ------------------------------------------------------------------------------------------
// Verner's 7(6) pair ("most efficient" IIa, Verner 2010; the seventh-order Verner pair that
// [GS] §3.1 offers besides Tsit5 for non-stiff problems): 10 stages, not first-same-as-last.
// b_2 = b_3 = b_10 = 0; the tenth stage enters only the embedded sixth-order solution b_hat.
// The decimals are the published ones (checked by the order conditions in the tests).
// ------------------------------------------------------------------------------------------
struct Vern7Tab {
  static constexpr int S = 10;
  static constexpr int order = 7;
  static constexpr int err_order = 7;   // embedded order 6, plus one
  static constexpr double A[10][9] = {
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
  static constexpr double B[10] = {0.04715561848627222, 0, 0, 0.25750564298434153,
                                   0.26216653977412624, 0.15216092656738558, 0.4939969170032485,
                                   -0.29430311714032503, 0.08131747232495111, 0};
  static constexpr double BH[10] = {0.044608606606341174, 0, 0, 0.26716403785713727,
                                    0.22010183001772932, 0.2188431703143157, 0.22898717054112028,
                                    0, 0, 0.02029518466335628};
};

// One trial step of Verner 7 from y with step h; k1 = f(y) is passed in (it stays valid across a
// rejected trial).  Stage states Y_i = y + h sum_{j<i} A_ij k_j (j ascending), the step result
// y_new = y + h sum_i B_i k_i, the error estimate e = h sum_i (B_i - BH_i) k_i.  With want_err
// false only stages 1..9 are formed (the replay map: B_10 = 0).
template <class F, class T>
void vern7_trial(const T* y, T h, const T* th, const T* k1, T* ynew, T* e, bool want_err) {
  constexpr int D = F::D;
  const int nst = want_err ? 10 : 9;
  T k[10][D];
  for (int c = 0; c < D; ++c) k[0][c] = k1[c];
  for (int i = 1; i < nst; ++i) {
    T Y[D];
    for (int c = 0; c < D; ++c) {
      T s = cst<T>(Vern7Tab::A[i][0]) * k[0][c];
      for (int j = 1; j < i; ++j) s = s + cst<T>(Vern7Tab::A[i][j]) * k[j][c];
      Y[c] = y[c] + h * s;
    }
    F::f(Y, th, k[i]);
  }
  for (int c = 0; c < D; ++c) {
    T s = cst<T>(Vern7Tab::B[0]) * k[0][c];
    for (int j = 1; j < 9; ++j) s = s + cst<T>(Vern7Tab::B[j]) * k[j][c];
    ynew[c] = y[c] + h * s;
  }
  if (!want_err) return;
  for (int c = 0; c < D; ++c) {
    T s = (cst<T>(Vern7Tab::B[0]) - cst<T>(Vern7Tab::BH[0])) * k[0][c];
    for (int j = 1; j < 10; ++j) s = s + (cst<T>(Vern7Tab::B[j]) - cst<T>(Vern7Tab::BH[j])) * k[j][c];
    e[c] = h * s;
  }
}

// ------------------------------------------------------------------------------------------
// One trial step of Tsit5 from y with step h.  k1 = f(y) is passed in (first-same-as-last).
// Writes the step result y_new, the last stage k7 = f(y_new) (the next k1) and the error
// estimate e = h sum_j BT_j k_j.  Stage states: Y_i = y + h sum_{j<i} A_ij k_j, summed j-ascending.
// When want_err is false only y_new is formed (the replay map Phi: k7 is not needed, b7 = 0).
// ------------------------------------------------------------------------------------------
template <class F, class T>
void tsit5_trial(const T* y, T h, const T* th, const T* k1, T* ynew, T* k7, T* e, bool want_err) {
  constexpr int D = F::D;
  T k[7][D];
  for (int c = 0; c < D; ++c) k[0][c] = k1[c];
  T Y[D];
  for (int i = 1; i < 7; ++i) {
    for (int c = 0; c < D; ++c) {
      T s = cst<T>(Tsit5Tab::A[i][0]) * k[0][c];
      for (int j = 1; j < i; ++j) s = s + cst<T>(Tsit5Tab::A[i][j]) * k[j][c];
      Y[c] = y[c] + h * s;
    }
    if (i < 6) {
      F::f(Y, th, k[i]);
    } else {
      for (int c = 0; c < D; ++c) ynew[c] = Y[c];
    }
  }
  if (!want_err) return;
  F::f(ynew, th, k[6]);
  for (int c = 0; c < D; ++c) k7[c] = k[6][c];
  for (int c = 0; c < D; ++c) {
    T s = cst<T>(Tsit5Tab::BT[0]) * k[0][c];
    for (int j = 1; j < 7; ++j) s = s + cst<T>(Tsit5Tab::BT[j]) * k[j][c];
    e[c] = h * s;
  }
}

// Dense LU with partial pivoting (pivot = largest |value|, ties to the lowest row), in place.
template <class T, int D>
void lu_factor(T* Mtx, int* piv) {
  for (int col = 0; col < D; ++col) {
    int p = col;
    auto best = std::fabs(value_of(Mtx[col * D + col]));
    for (int r = col + 1; r < D; ++r) {
      auto v = std::fabs(value_of(Mtx[r * D + col]));
      if (v > best) { best = v; p = r; }
    }
    piv[col] = p;
    if (p != col)
      for (int c = 0; c < D; ++c) std::swap(Mtx[col * D + c], Mtx[p * D + c]);
    for (int r = col + 1; r < D; ++r) {
      T l = Mtx[r * D + col] / Mtx[col * D + col];
      Mtx[r * D + col] = l;
      for (int c = col + 1; c < D; ++c) Mtx[r * D + c] = Mtx[r * D + c] - l * Mtx[col * D + c];
    }
  }
}
template <class T, int D>
void lu_solve(const T* LU, const int* piv, T* x) {
  for (int col = 0; col < D; ++col)
    if (piv[col] != col) std::swap(x[col], x[piv[col]]);
  for (int r = 1; r < D; ++r)
    for (int c = 0; c < r; ++c) x[r] = x[r] - LU[r * D + c] * x[c];
  for (int r = D - 1; r >= 0; --r) {
    for (int c = r + 1; c < D; ++c) x[r] = x[r] - LU[r * D + c] * x[c];
    x[r] = x[r] / LU[r * D + r];
  }
}

// One trial step of ROS34PW2 in the Hairer-Wanner form stated on Ros34pw2Tab ([GS] §3.2:
// each stage solves a linear system with I - gamma h J, J = df/dy).
template <class F, class T>
void ros_trial(const T* y, T h, const T* th, T* ynew, T* e, bool want_err) {
  constexpr int D = F::D;
  T J[D * D], Mtx[D * D];
  int piv[D];
  F::jac(y, th, J);
  const T gh = cst<T>(Ros34pw2Tab::gamma) * h;
  for (int r = 0; r < D; ++r)
    for (int c = 0; c < D; ++c) Mtx[r * D + c] = T(r == c ? 1.0 : 0.0) - gh * J[r * D + c];
  lu_factor<T, D>(Mtx, piv);
  T k[4][D];
  for (int i = 0; i < 4; ++i) {
    T Y[D], G[D], fy[D], r[D];
    for (int c = 0; c < D; ++c) {
      T u = T(0), g = T(0);
      for (int j = 0; j < i; ++j) {
        u = u + cst<T>(Ros34pw2Tab::ALPHA[i][j]) * k[j][c];
        g = g + cst<T>(Ros34pw2Tab::GAMMA[i][j]) * k[j][c];
      }
      Y[c] = y[c] + u;
      G[c] = g;
    }
    F::f(Y, th, fy);
    for (int rr = 0; rr < D; ++rr) {
      T jg = T(0);
      for (int c = 0; c < D; ++c) jg = jg + J[rr * D + c] * G[c];
      r[rr] = h * fy[rr] + h * jg;
    }
    lu_solve<T, D>(Mtx, piv, r);
    for (int c = 0; c < D; ++c) k[i][c] = r[c];
  }
  for (int c = 0; c < D; ++c) {
    T s = cst<T>(Ros34pw2Tab::B[0]) * k[0][c];
    for (int i = 1; i < 4; ++i) s = s + cst<T>(Ros34pw2Tab::B[i]) * k[i][c];
    ynew[c] = y[c] + s;
  }
  if (!want_err) return;
  for (int c = 0; c < D; ++c) {
    T s = (cst<T>(Ros34pw2Tab::B[0]) - cst<T>(Ros34pw2Tab::BHAT[0])) * k[0][c];
    for (int i = 1; i < 4; ++i)
      s = s + (cst<T>(Ros34pw2Tab::B[i]) - cst<T>(Ros34pw2Tab::BHAT[i])) * k[i][c];
    e[c] = s;
  }
}

// Rosenbrock23 (Shampine & Reichelt 1997, the pair of MATLAB's ode23s; [GS] §3.1: the
// second-order linearly implicit method of the fused stiff kernels), autonomous form, exact J:
//   d = 1/(2 + sqrt 2),  W = I - h d J,  J = f_y(y_n)
//   F0 = f(y_n),  k1 = W^{-1} F0,  F1 = f(y_n + h k1 / 2),  k2 = W^{-1} (F1 - k1) + k1,
//   y_{n+1} = y_n + h k2,
//   F2 = f(y_{n+1}),  k3 = W^{-1} (F2 - e32 (k2 - F1) - 2 (k1 - F0)),  e32 = 6 + sqrt 2,
//   error estimate e = h (k1 - 2 k2 + k3) / 6.
struct Rb23Tab {
  static constexpr int order = 2;
  static constexpr int err_order = 3;   // the estimate is the local error of the order-2 step
  static constexpr double d = 0.29289321881345248;    // 1 / (2 + sqrt 2)
  static constexpr double e32 = 7.4142135623730951;   // 6 + sqrt 2
};

template <class F, class T>
void rb23_trial(const T* y, T h, const T* th, T* ynew, T* e, bool want_err) {
  constexpr int D = F::D;
  T J[D * D], W[D * D];
  int piv[D];
  F::jac(y, th, J);
  const T hd = h * cst<T>(Rb23Tab::d);
  for (int r = 0; r < D; ++r)
    for (int c = 0; c < D; ++c) W[r * D + c] = T(r == c ? 1.0 : 0.0) - hd * J[r * D + c];
  lu_factor<T, D>(W, piv);
  T F0[D], k1[D], Y1[D], F1[D], k2[D];
  F::f(y, th, F0);
  for (int c = 0; c < D; ++c) k1[c] = F0[c];
  lu_solve<T, D>(W, piv, k1);
  for (int c = 0; c < D; ++c) Y1[c] = y[c] + cst<T>(0.5) * h * k1[c];
  F::f(Y1, th, F1);
  for (int c = 0; c < D; ++c) k2[c] = F1[c] - k1[c];
  lu_solve<T, D>(W, piv, k2);
  for (int c = 0; c < D; ++c) k2[c] = k2[c] + k1[c];
  for (int c = 0; c < D; ++c) ynew[c] = y[c] + h * k2[c];
  if (!want_err) return;
  T F2[D], k3[D];
  F::f(ynew, th, F2);
  for (int c = 0; c < D; ++c)
    k3[c] = F2[c] - cst<T>(Rb23Tab::e32) * (k2[c] - F1[c]) - cst<T>(2.0) * (k1[c] - F0[c]);
  lu_solve<T, D>(W, piv, k3);
  for (int c = 0; c < D; ++c)
    e[c] = h * (k1[c] - cst<T>(2.0) * k2[c] + k3[c]) / cst<T>(6.0);
}

enum Method { TSIT5 = 0, ROS34PW2 = 1, VERN7 = 2, RB23 = 3 };

inline int method_order(Method m) {
  return m == TSIT5 ? Tsit5Tab::order : m == VERN7 ? Vern7Tab::order
                                      : m == RB23 ? Rb23Tab::order : Ros34pw2Tab::order;
}
inline int method_err_order(Method m) {
  return m == TSIT5 ? Tsit5Tab::err_order : m == VERN7 ? Vern7Tab::err_order
                                          : m == RB23 ? Rb23Tab::err_order
                                                      : Ros34pw2Tab::err_order;
}

// has_jac<F>: stiff fields carry an analytic Jacobian.
template <class F, class = void> struct has_jac : std::false_type {};
template <class F>
struct has_jac<F, std::void_t<decltype(&F::template jac<double>)>> : std::true_type {};


// ------------------------------------------------------------------------------------------
// The adaptive solve ([GS] §2.1) with the record of accepted steps ([GS] §3).
// Readings where the pages are silent (the controller equation is not in the text):
//  * error norm: err = sqrt(mean_i (e_i / sc_i)^2), sc_i = atol + rtol max(|y_i|, |ynew_i|);
//    accept iff err <= 1; a non-finite err is a reject with factor 0.2.
//  * I-controller: fac = 0.9 err^(-1/q), q = embedded order + 1; fac clamped to [0.2, facmax];
//    fac = facmax when err = 0; facmax = 10, except 1 for the first accepted step after a reject.
//  * starting step: Hairer-Norsett-Wanner §II.4 with sc = atol + rtol |y0| and p = method order.
//  * loop: clip h to t1 - t; an accepted step that reaches t1 sets t = t1 exactly; status 1 after
//    max_attempts attempts, status 2 when h < 16 eps max(|t|, |t1 - t0|) or h is not finite
//    (the comparison is written so that NaN fails it), status 3 when y0 or
//    f(y0) is not finite.  Rejected trials leave no trace in the record.
// ------------------------------------------------------------------------------------------
template <class R>
struct Record {
  std::vector<R> t, h, y;  // y is [S][D]
  int S = 0, rejected = 0, status = 0;
  long long attempts = 0;
  std::vector<R> y1;
};

template <class R>
inline R rms_scaled(const R* v, const R* a, const R* b, int D, R rtol, R atol) {
  R s = R(0);
  for (int i = 0; i < D; ++i) {
    R sc = atol + rtol * std::max(std::fabs(a[i]), std::fabs(b[i]));
    R q = v[i] / sc;
    s = s + q * q;
  }
  return std::sqrt(s / R(D));
}

// Dc = number of leading state components the step control sees (all of them unless a
// sensitivity block rides along, see solve_sens).
template <class F, class R>
R initial_step(const R* y0, const R* f0, const R* th, R t0, R t1, R rtol, R atol, int p,
               int Dc = F::D) {
  constexpr int D = F::D;
  R sc[D];
  for (int i = 0; i < D; ++i) sc[i] = atol + rtol * std::fabs(y0[i]);
  auto norm = [&](const R* v) {
    R s = R(0);
    for (int i = 0; i < Dc; ++i) { R q = v[i] / sc[i]; s = s + q * q; }
    return std::sqrt(s / R(Dc));
  };
  const R d0 = norm(y0), d1 = norm(f0);
  R h0 = (d0 < R(1e-5) || d1 < R(1e-5)) ? R(1e-6) : R(0.01) * d0 / d1;
  R y1[D], f1[D], df[D];
  for (int i = 0; i < D; ++i) y1[i] = y0[i] + h0 * f0[i];
  F::f(y1, th, f1);
  for (int i = 0; i < D; ++i) df[i] = f1[i] - f0[i];
  const R d2 = norm(df) / h0;
  const R dm = std::max(d1, d2);
  R h1 = (dm <= R(1e-15)) ? std::max(R(1e-6), h0 * R(1e-3))
                          : std::pow(R(0.01) / dm, R(1) / R(p));
  return std::min(std::min(R(100) * h0, h1), t1 - t0);
}

template <class F, class R>
Record<R> solve(Method method, const R* y0, const R* th, R t0, R t1, R rtol, R atol,
                long long max_attempts, bool keep_record, int Dc = F::D) {
  constexpr int D = F::D;
  Record<R> rec;
  rec.y1.assign(y0, y0 + D);
  R y[D], k1[D];
  for (int i = 0; i < D; ++i) y[i] = y0[i];
  if (!(t1 > t0)) return rec;  // empty interval: no step, y1 = y0
  F::f(y, th, k1);
  for (int i = 0; i < Dc; ++i)
    if (!std::isfinite(y[i]) || !std::isfinite(k1[i])) { rec.status = 3; return rec; }
  const int p = method_order(method);
  const int q = method_err_order(method);
  const R expo = R(-1.0 / double(q));
  const R eps = std::numeric_limits<R>::epsilon();
  R h = initial_step<F, R>(y, k1, th, t0, t1, rtol, atol, p, Dc);
  R t = t0;
  bool last_rejected = false;
  while (t < t1) {
    if (rec.attempts >= max_attempts) { rec.status = 1; break; }
    // a step below 16 ulp of the time scale, or a non-finite step, ends the solve
    if (!(h >= R(16) * eps * std::max(std::fabs(t), std::fabs(t1 - t0)))) { rec.status = 2; break; }
    bool clipped = false;
    if (t + h > t1) { h = t1 - t; clipped = true; }
    rec.attempts++;
    R ynew[D], k7[D], e[D];
    if (method == TSIT5) {
      tsit5_trial<F, R>(y, h, th, k1, ynew, k7, e, true);
    } else if (method == VERN7) {
      vern7_trial<F, R>(y, h, th, k1, ynew, e, true);
    } else if (method == RB23) {
      if constexpr (has_jac<F>::value) rb23_trial<F, R>(y, h, th, ynew, e, true);
    } else {
      if constexpr (has_jac<F>::value) ros_trial<F, R>(y, h, th, ynew, e, true);
    }
    const R err = rms_scaled<R>(e, y, ynew, Dc, rtol, atol);
    if (err <= R(1)) {
      if (keep_record) {
        rec.t.push_back(t);
        rec.h.push_back(h);
        for (int i = 0; i < D; ++i) rec.y.push_back(y[i]);
      }
      rec.S++;
      const R facmax = last_rejected ? R(1) : R(10);
      R fac = (err == R(0)) ? facmax : R(0.9) * std::pow(err, expo);
      fac = std::min(facmax, std::max(R(0.2), fac));
      t = (clipped || t + h >= t1) ? t1 : t + h;
      for (int i = 0; i < D; ++i) y[i] = ynew[i];
      if (method == TSIT5)
        for (int i = 0; i < D; ++i) k1[i] = k7[i];  // first-same-as-last
      else if (method == VERN7)
        F::f(y, th, k1);                             // a fresh first stage at the new state
      h = h * fac;
      last_rejected = false;
    } else {
      rec.rejected++;
      R fac = std::isfinite(err) ? R(0.9) * std::pow(err, expo) : R(0.2);
      fac = std::min(R(10), std::max(R(0.2), fac));
      h = h * fac;
      last_rejected = true;
    }
  }
  for (int i = 0; i < D; ++i) rec.y1[i] = y[i];
  return rec;
}

// One step of the method's one-step map Phi(y, h; theta) (no error estimate): the replay step.
template <class F, class T>
void one_step(Method method, const T* y, const T* th, T h, T* ynew) {
  constexpr int D = F::D;
  if (method == TSIT5 || method == VERN7) {
    T k1[D];
    F::f(y, th, k1);
    if (method == TSIT5) tsit5_trial<F, T>(y, h, th, k1, ynew, nullptr, nullptr, false);
    else vern7_trial<F, T>(y, h, th, k1, ynew, nullptr, false);
  } else if (method == RB23) {
    if constexpr (has_jac<F>::value) rb23_trial<F, T>(y, h, th, ynew, nullptr, false);
  } else {
    if constexpr (has_jac<F>::value) ros_trial<F, T>(y, h, th, ynew, nullptr, false);
  }
}

// ------------------------------------------------------------------------------------------
// Replay ([GS] §3, Eq. 4): y_{n+1} = Phi(y_n, h_n; theta), n = 0..S-1, with the recorded h_n
// as data.  For Tsit5, Phi(y, h) = y + h sum_{i<=6} b_i k_i with k_1 = f(y) evaluated afresh;
// for Verner 7, Phi(y, h) = y + h sum_{i<=9} b_i k_i.
// ------------------------------------------------------------------------------------------
template <class F, class T>
void replay(Method method, T* y, const T* th, const typename base_of<T>::type* H, int S) {
  constexpr int D = F::D;
  for (int n = 0; n < S; ++n) {
    const T h = T(H[n]);
    T ynew[D];
    one_step<F, T>(method, y, th, h, ynew);
    for (int c = 0; c < D; ++c) y[c] = ynew[c];
  }
}

// ------------------------------------------------------------------------------------------
// Gradient of L through the replay, by its plain definition ([GS] §3: the derivative of the
// chain Psi(theta; sg[h]) with h held fixed as data).  The Jacobian of y_S with respect to the
// D + M inputs (y0, theta) is formed column by column with P-direction dual numbers pushed
// through the replay; then dL/d(input j) = sum_c lam_c dy_S,c/d(input j), lam = dL/dy_S.
// ------------------------------------------------------------------------------------------
template <class F, class R>
void replay_grad(Method method, const R* y0, const R* th, const R* H, int S, const R* lam,
                 R* dL_dy0, R* dL_dth) {
  constexpr int D = F::D, M = F::M, P = 16;
  using T = Dual<R, P>;
  const int ninputs = D + M;
  std::vector<T> thd(M);
  for (int base = 0; base < ninputs; base += P) {
    T yd[D];
    for (int c = 0; c < D; ++c) {
      yd[c] = T(y0[c]);
      const int dir = c - base;
      if (dir >= 0 && dir < P) yd[c].g[dir] = R(1);
    }
    for (int j = 0; j < M; ++j) {
      thd[j] = T(th[j]);
      const int dir = D + j - base;
      if (dir >= 0 && dir < P) thd[j].g[dir] = R(1);
    }
    replay<F, T>(method, yd, thd.data(), H, S);
    for (int dir = 0; dir < P && base + dir < ninputs; ++dir) {
      R s = R(0);
      for (int c = 0; c < D; ++c) s = s + lam[c] * yd[c].g[dir];
      const int idx = base + dir;
      if (idx < D) { if (dL_dy0) dL_dy0[idx] = s; }
      else if (dL_dth) dL_dth[idx - D] = s;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Outputs at requested times ([GS] §3.4: the replay takes one extra solver step from the
// preceding mesh point exactly to each requested time, so the state is integrated, not
// interpolated).  Reading: for tau_j (ascending, t0 <= tau_j <= t1) the preceding mesh point is
// the last recorded t_n with t_n <= tau_j and tau_j < t_{n+1} (t_S = t1); the output is
// Phi(y_n, tau_j - t_n), and tau_j = t1 gives y_S.  Tm holds the recorded start times t_n.
// ------------------------------------------------------------------------------------------

template <class F, class T>
void replay_outputs(Method method, const T* y0, const T* th,
                    const typename base_of<T>::type* Tm, const typename base_of<T>::type* H,
                    int S, typename base_of<T>::type t1, int J,
                    const typename base_of<T>::type* tau, T* out) {
  using R = typename base_of<T>::type;
  constexpr int D = F::D;
  T y[D];
  for (int c = 0; c < D; ++c) y[c] = y0[c];
  int j = 0;
  for (int n = 0; n < S; ++n) {
    const R tnext = (n + 1 < S) ? Tm[n + 1] : t1;
    while (j < J && tau[j] < tnext) {
      one_step<F, T>(method, y, th, T(tau[j] - Tm[n]), out + (size_t)j * D);
      ++j;
    }
    T ynew[D];
    one_step<F, T>(method, y, th, T(H[n]), ynew);
    for (int c = 0; c < D; ++c) y[c] = ynew[c];
  }
  for (; j < J; ++j)
    for (int c = 0; c < D; ++c) out[(size_t)j * D + c] = y[c];
}

// Gradient of L = sum_j lam_j . y(tau_j) by its plain definition: forward-mode duals through
// replay_outputs, contracted with the output cotangents lam [J][D].
template <class F, class R>
void replay_outputs_grad(Method method, const R* y0, const R* th, const R* Tm, const R* H, int S,
                         R t1, int J, const R* tau, const R* lam, R* dL_dy0, R* dL_dth) {
  constexpr int D = F::D, M = F::M, P = 16;
  using T = Dual<R, P>;
  const int ninputs = D + M;
  std::vector<T> thd(M), out((size_t)J * D);
  for (int base = 0; base < ninputs; base += P) {
    T yd[D];
    for (int c = 0; c < D; ++c) {
      yd[c] = T(y0[c]);
      const int dir = c - base;
      if (dir >= 0 && dir < P) yd[c].g[dir] = R(1);
    }
    for (int i = 0; i < M; ++i) {
      thd[i] = T(th[i]);
      const int dir = D + i - base;
      if (dir >= 0 && dir < P) thd[i].g[dir] = R(1);
    }
    replay_outputs<F, T>(method, yd, thd.data(), Tm, H, S, t1, J, tau, out.data());
    for (int dir = 0; dir < P && base + dir < ninputs; ++dir) {
      R s = R(0);
      for (int q = 0; q < J * D; ++q) s = s + lam[q] * out[q].g[dir];
      const int idx = base + dir;
      if (idx < D) { if (dL_dy0) dL_dy0[idx] = s; }
      else if (dL_dth) dL_dth[idx - D] = s;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Forward sensitivity along a direction (forward mode through the replay, [GS] §4.4; the
// in-kernel forward sensitivities of [DA] §2, one direction per pass): the tangent of y_S for
// the input direction (ydot0, thdot), by one-direction dual numbers through the same chain.
// ------------------------------------------------------------------------------------------
template <class F, class R>
void replay_jvp(Method method, const R* y0, const R* th, const R* ydot0, const R* thdot,
                const R* H, int S, R* y1, R* ydot1) {
  constexpr int D = F::D, M = F::M;
  using T = Dual<R, 1>;
  T yd[D];
  std::vector<T> thd(M);
  for (int c = 0; c < D; ++c) { yd[c] = T(y0[c]); yd[c].g[0] = ydot0[c]; }
  for (int j = 0; j < M; ++j) { thd[j] = T(th[j]); thd[j].g[0] = thdot[j]; }
  replay<F, T>(method, yd, thd.data(), H, S);
  for (int c = 0; c < D; ++c) { y1[c] = yd[c].v; ydot1[c] = yd[c].g[0]; }
}

// ------------------------------------------------------------------------------------------
// Forward sensitivities in the same solve ([DA] §2 and §3: the sensitivity equations integrated
// together with the orbit, with the step size controlled on the orbit alone).  The augmented
// state is z = (y, S), S = dy/dtheta stored row-major [D][M]; its right-hand side is
//   (f(y; theta),  J_y(y) S + J_theta(y)),
// the second block evaluated as the M directional derivatives of f along (S_{:,p}, e_p) with
// M-direction dual numbers.  Reading: "controlled on the orbit alone" means that the error test,
// the starting step and the finiteness check at the start look at the first D components only,
// so the accepted mesh and y are those of the plain solve.
// ------------------------------------------------------------------------------------------
template <class F>
struct SensAug {
  static constexpr int D0 = F::D, M = F::M, D = F::D * (1 + F::M);
  template <class T> static void f(const T* z, const T* th, T* dz) {
    using DT = Dual<T, M>;
    DT y[D0], t[M], dy[D0];
    for (int c = 0; c < D0; ++c) {
      y[c] = DT(z[c]);
      for (int p = 0; p < M; ++p) y[c].g[p] = z[D0 + c * M + p];
    }
    for (int j = 0; j < M; ++j) { t[j] = DT(th[j]); t[j].g[j] = T(1); }
    F::f(y, t, dy);
    for (int c = 0; c < D0; ++c) {
      dz[c] = dy[c].v;
      for (int p = 0; p < M; ++p) dz[D0 + c * M + p] = dy[c].g[p];
    }
  }
};

template <class F, class R>
Record<R> solve_sens(const R* y0, const R* S0, const R* th, R t0, R t1, R rtol, R atol,
                     long long max_attempts, R* S1) {
  constexpr int D = F::D, M = F::M;
  using A = SensAug<F>;
  R z0[A::D];
  for (int c = 0; c < D; ++c) z0[c] = y0[c];
  for (int i = 0; i < D * M; ++i) z0[D + i] = S0 ? S0[i] : R(0);
  Record<R> za = solve<A, R>(TSIT5, z0, th, t0, t1, rtol, atol, max_attempts, false, D);
  Record<R> rec;
  rec.S = za.S; rec.rejected = za.rejected; rec.status = za.status; rec.attempts = za.attempts;
  rec.y1.assign(za.y1.begin(), za.y1.begin() + D);
  for (int i = 0; i < D * M; ++i) S1[i] = za.y1[D + i];
  return rec;
}

}  // namespace orc
