// Host program that tallies the arithmetic of the device fields' f and vector-Jacobian product
// (add/sub, mul, div, sqrt/rsqrt, log1p per call) by instantiating them with a counting scalar.
// For a field that hands its VJP the intermediates of f (a stage tape), the VJP is counted
// without recomputing them: that recomputation is not part of the pullback.
// Compiled as plain C++ (g++) and run by tests/test_flop_counts.py; prints one JSON object per field.
#include <cmath>
#include <cstdio>
#include <type_traits>

#include "gs_fields.cuh"
#include "gs_dual.cuh"

struct Tally { long add = 0, mul = 0, div = 0, sqrt = 0, log1p = 0; };
static Tally T;
struct Cnt {
  double v;
  Cnt() : v(0) {}
  Cnt(double x) : v(x) {}
  Cnt& operator+=(Cnt o) { T.add++; v += o.v; return *this; }
  Cnt& operator-=(Cnt o) { T.add++; v -= o.v; return *this; }
};
inline Cnt operator+(Cnt a, Cnt b) { T.add++; return Cnt(a.v + b.v); }
inline Cnt operator-(Cnt a, Cnt b) { T.add++; return Cnt(a.v - b.v); }
inline Cnt operator-(Cnt a) { return Cnt(-a.v); }
inline Cnt operator*(Cnt a, Cnt b) { T.mul++; return Cnt(a.v * b.v); }
inline Cnt operator/(Cnt a, Cnt b) { T.div++; return Cnt(a.v / b.v); }
inline Cnt sqrt(Cnt a) { T.sqrt++; return Cnt(std::sqrt(a.v)); }
inline Cnt log1p(Cnt a) { T.log1p++; return Cnt(std::log1p(a.v)); }
// the fields' log1p evaluation given a reciprocal of 1 + x (log1p_q) is one log1p of the formula
inline Cnt log1p_q(Cnt a, Cnt, Cnt) { T.log1p++; return Cnt(std::log1p(a.v)); }
inline Cnt rsqrt(Cnt a) { T.sqrt++; return Cnt(1.0 / std::sqrt(a.v)); }
inline Cnt fma(Cnt a, Cnt b, Cnt c) { T.mul++; T.add++; return Cnt(a.v * b.v + c.v); }

template <class F, class = void> struct has_pullback : std::false_type {};
template <class F>
struct has_pullback<F, std::void_t<decltype(F::TAPE)>> : std::true_type {};

template <class F, class = void> struct has_jac : std::false_type {};
template <class F>
struct has_jac<F, std::void_t<decltype(&F::template jac<double>)>> : std::true_type {};

template <class F>
void run(const char* name, const double* theta, const double* y) {
  Cnt th_src[F::M], yy[F::D], dy[F::D], kb[F::D], yb[F::D], thb[F::M];
  for (int j = 0; j < F::M; ++j) { th_src[j] = Cnt(theta[j]); thb[j] = Cnt(0); }
  for (int c = 0; c < F::D; ++c) { yy[c] = Cnt(y[c]); kb[c] = Cnt(0.1 * (c + 1)); }
  typename F::template Theta<Cnt> th;
  F::load(th, th_src);
  T = Tally();
  F::f(yy, th, dy);
  Tally tf = T;
  Tally tv;
  if constexpr (has_pullback<F>::value) {
    // the pullback proper, given f's intermediates at the stage (which f already computed)
    typename F::template Inter<Cnt> I;
    F::inter(yy, th, I);
    T = Tally();
    F::vjp_from(yy, th, I, kb, yb, thb);
    tv = T;
  } else {
    T = Tally();
    F::vjp(yy, th, kb, yb, thb);
    tv = T;
  }
  // f on one-direction dual numbers (the forward-sensitivity stage): value and tangent together
  using DC = gs::Dl<Cnt>;
  DC dsrc[F::M], dy_[F::D], ddy[F::D];
  for (int j = 0; j < F::M; ++j) dsrc[j] = DC(Cnt(theta[j]), Cnt(j == 0 ? 1.0 : 0.0));
  for (int c = 0; c < F::D; ++c) dy_[c] = DC(Cnt(y[c]), Cnt(0.01 * (c + 1)));
  typename F::template Theta<DC> thd;
  F::load(thd, dsrc);
  T = Tally();
  F::f(dy_, thd, ddy);
  Tally td = T;
  // Jacobian and the contraction of a Jacobian cotangent with its derivatives (stiff fields)
  Tally tj, tjv;
  if constexpr (has_jac<F>::value) {
    Cnt J[F::D * F::D], Jb[F::D * F::D], yb2[F::D], thb2[F::M];
    for (int i = 0; i < F::D * F::D; ++i) Jb[i] = Cnt(0.01 * (i + 1));
    for (int c = 0; c < F::D; ++c) yb2[c] = Cnt(0);
    for (int j = 0; j < F::M; ++j) thb2[j] = Cnt(0);
    T = Tally();
    F::jac(yy, th, J);
    tj = T;
    T = Tally();
    F::jac_vjp(yy, th, Jb, yb2, thb2);
    tjv = T;
  }
  std::printf("{\"jac\": %ld, \"jac_vjp\": %ld, ", tj.add + tj.mul + tj.div + tj.sqrt + tj.log1p,
              tjv.add + tjv.mul + tjv.div + tjv.sqrt + tjv.log1p);
  std::printf("\"field\": \"%s\", \"D\": %d, \"M\": %d, "
              "\"f\": {\"add\": %ld, \"mul\": %ld, \"div\": %ld, \"sqrt\": %ld, \"log1p\": %ld}, "
              "\"vjp\": {\"add\": %ld, \"mul\": %ld, \"div\": %ld, \"sqrt\": %ld, \"log1p\": %ld}, "
              "\"fdual\": {\"add\": %ld, \"mul\": %ld, \"div\": %ld, \"sqrt\": %ld, \"log1p\": %ld}}\n",
              name, F::D, F::M, tf.add, tf.mul, tf.div, tf.sqrt, tf.log1p, tv.add, tv.mul, tv.div,
              tv.sqrt, tv.log1p, td.add, td.mul, td.div, td.sqrt, td.log1p);
}

int main() {
  const double nfw_th[5] = {1, 1, 0.1, 0.3, 0.03}, nfw_y[6] = {0.7, 0.2, 0.1, 0.1, 0.5, 0.05};
  const double lor_th[3] = {10, 28, 8.0 / 3}, lor_y[3] = {1, 1, 1};
  const double lv_th[4] = {1.5, 1, 3, 1}, lv_y[2] = {1, 1};
  const double rob_th[3] = {0.04, 3e7, 1e4}, rob_y[3] = {0.9, 1e-5, 0.1};
  run<gs::FNfwMiyamotoNagai>("nfw_mn", nfw_th, nfw_y);
  run<gs::FLorenz63>("lorenz63", lor_th, lor_y);
  run<gs::FLotkaVolterra>("lotka_volterra", lv_th, lv_y);
  run<gs::FRobertson>("robertson", rob_th, rob_y);
  const double lh_th[2] = {1.0, 0.7}, lh_y[6] = {0.7, 0.2, 0.4, 0.1, 0.5, 0.05};
  run<gs::FLogHalo>("log_halo", lh_th, lh_y);
  const double hi_th[12] = {1.71, 0.43, 8.32, 0.0007, 8.75, 10.03, 0.035, 1.12, 1.745, 280, 0.69,
                            1.81};
  const double hi_y[8] = {0.7, 0.01, 0.02, 0.03, 0.04, 0.05, 0.06, 0.007};
  run<gs::FHires>("hires", hi_th, hi_y);
  return 0;
}
