// gs_oracle.cpp -- C entry points of the CPU oracle (TEST INFRASTRUCTURE ONLY; see
// gs_oracle.hpp).  Plain loops over trajectories, optionally spread over host threads in
// dynamic chunks of 64 trajectories.  Built as oracle/liboracle.so by oracle/build_oracle.py.
//
// Conventions: dtype 0 = double, 1 = float.  Arrays are row-major: theta [N][M] (or [M] when
// theta_shared), y [N][D]; records are padded rectangles [N][Smax] (the pages' own padded
// layout, [GS] §3) with per-trajectory counts S[N].  Return 0 on success, a negative code on a
// bad argument, 1 when some record did not fit in Smax.
#include <atomic>
#include <cstring>
#include <thread>

#include "gs_oracle.hpp"

namespace {

using namespace orc;

enum FieldId { F_LV = 0, F_LORENZ = 1, F_MLP = 2, F_ROBERTSON = 3, F_NFW = 4, F_LIN1 = 5,
               F_LIN2 = 6, F_LIN3 = 7, F_LOGHALO = 8, F_HIRES = 9 };

template <class Fn>
void parallel_for(long long N, int nthreads, Fn fn) {
  if (nthreads <= 1 || N <= 64) {
    for (long long k = 0; k < N; ++k) fn(k);
    return;
  }
  std::atomic<long long> next(0);
  std::vector<std::thread> pool;
  for (int w = 0; w < nthreads; ++w)
    pool.emplace_back([&]() {
      for (;;) {
        long long b = next.fetch_add(64);
        if (b >= N) break;
        long long e = std::min(N, b + 64);
        for (long long k = b; k < e; ++k) fn(k);
      }
    });
  for (auto& t : pool) t.join();
}

struct SolveArgs {
  int method;
  long long N;
  int theta_shared;
  const void* theta;
  const void* y0;
  double t0, t1, rtol, atol;
  long long max_attempts;
  void* y1;
  int* S;
  int* rej;
  int* status;
  long long* attempts;
  int keep_record, Smax;
  void* Tout;
  void* Hout;
  void* Yout;
  int nthreads;
};

template <class F, class R>
int solve_impl(const SolveArgs& a) {
  constexpr int D = F::D, M = F::M;
  const R* th = static_cast<const R*>(a.theta);
  const R* y0 = static_cast<const R*>(a.y0);
  std::atomic<int> overflow(0);
  parallel_for(a.N, a.nthreads, [&](long long k) {
    const R* thk = th + (a.theta_shared ? 0 : k * M);
    Record<R> rec = solve<F, R>(Method(a.method), y0 + k * D, thk, R(a.t0), R(a.t1), R(a.rtol),
                                R(a.atol), a.max_attempts, a.keep_record != 0);
    if (a.y1) for (int c = 0; c < D; ++c) static_cast<R*>(a.y1)[k * D + c] = rec.y1[c];
    if (a.S) a.S[k] = rec.S;
    if (a.rej) a.rej[k] = rec.rejected;
    if (a.status) a.status[k] = rec.status;
    if (a.attempts) a.attempts[k] = rec.attempts;
    if (a.keep_record) {
      if (rec.S > a.Smax) { overflow = 1; return; }
      R* T = static_cast<R*>(a.Tout) + k * (long long)a.Smax;
      R* H = static_cast<R*>(a.Hout) + k * (long long)a.Smax;
      R* Y = static_cast<R*>(a.Yout) + k * (long long)a.Smax * D;
      for (int n = 0; n < rec.S; ++n) {
        T[n] = rec.t[n];
        H[n] = rec.h[n];
        for (int c = 0; c < D; ++c) Y[n * D + c] = rec.y[n * D + c];
      }
    }
  });
  return overflow.load() ? 1 : 0;
}

struct ReplayArgs {
  int method;
  long long N;
  int theta_shared;
  const void* theta;
  const void* y0;
  const void* H;
  const int* S;
  int Smax;
  const void* lam;
  void* y_out;
  void* dL_dy0;
  void* dL_dth;
  int nthreads;
};

template <class F, class R>
int replay_impl(const ReplayArgs& a) {
  constexpr int D = F::D, M = F::M;
  const R* th = static_cast<const R*>(a.theta);
  const R* y0 = static_cast<const R*>(a.y0);
  const R* H = static_cast<const R*>(a.H);
  parallel_for(a.N, a.nthreads, [&](long long k) {
    const R* thk = th + (a.theta_shared ? 0 : k * M);
    R y[D];
    for (int c = 0; c < D; ++c) y[c] = y0[k * D + c];
    replay<F, R>(Method(a.method), y, thk, H + k * (long long)a.Smax, a.S[k]);
    for (int c = 0; c < D; ++c) static_cast<R*>(a.y_out)[k * D + c] = y[c];
  });
  return 0;
}

template <class F, class R>
int grad_impl(const ReplayArgs& a) {
  constexpr int D = F::D, M = F::M;
  const R* th = static_cast<const R*>(a.theta);
  const R* y0 = static_cast<const R*>(a.y0);
  const R* H = static_cast<const R*>(a.H);
  const R* lam = static_cast<const R*>(a.lam);
  parallel_for(a.N, a.nthreads, [&](long long k) {
    const R* thk = th + (a.theta_shared ? 0 : k * M);
    R* gy = a.dL_dy0 ? static_cast<R*>(a.dL_dy0) + k * D : nullptr;
    R* gt = a.dL_dth ? static_cast<R*>(a.dL_dth) + k * M : nullptr;
    replay_grad<F, R>(Method(a.method), y0 + k * D, thk, H + k * (long long)a.Smax, a.S[k],
                      lam + k * D, gy, gt);
  });
  return 0;
}

struct OutArgs {
  int method;
  long long N;
  int theta_shared;
  const void* theta;
  const void* y0;
  const void* T;
  const void* H;
  const int* S;
  int Smax;
  double t1;
  int J;
  const void* tau;
  const void* lam;   // [N][J][D] (gradient only)
  void* out;         // [N][J][D] (outputs only)
  void* dL_dy0;
  void* dL_dth;
  int nthreads;
};

template <class F, class R>
int outputs_impl(const OutArgs& a, bool grad) {
  constexpr int D = F::D, M = F::M;
  const R* th = static_cast<const R*>(a.theta);
  const R* y0 = static_cast<const R*>(a.y0);
  const R* Tm = static_cast<const R*>(a.T);
  const R* H = static_cast<const R*>(a.H);
  const R* tau = static_cast<const R*>(a.tau);
  parallel_for(a.N, a.nthreads, [&](long long k) {
    const R* thk = th + (a.theta_shared ? 0 : k * M);
    const size_t off = (size_t)k * a.Smax;
    if (!grad) {
      replay_outputs<F, R>(Method(a.method), y0 + k * D, thk, Tm + off, H + off, a.S[k], R(a.t1),
                           a.J, tau, static_cast<R*>(a.out) + (size_t)k * a.J * D);
    } else {
      R* gy = a.dL_dy0 ? static_cast<R*>(a.dL_dy0) + k * D : nullptr;
      R* gt = a.dL_dth ? static_cast<R*>(a.dL_dth) + k * M : nullptr;
      replay_outputs_grad<F, R>(Method(a.method), y0 + k * D, thk, Tm + off, H + off, a.S[k],
                                R(a.t1), a.J, tau,
                                static_cast<const R*>(a.lam) + (size_t)k * a.J * D, gy, gt);
    }
  });
  return 0;
}

// Field dispatch: calls fn.template operator()<F>() for the field id; -2 if unknown.
template <class Fn>
int with_field(int field, Fn&& fn) {
  switch (field) {
    case F_LV: return fn(LotkaVolterra{});
    case F_LORENZ: return fn(Lorenz63{});
    case F_MLP: return fn(Mlp4x32x32x4{});
    case F_ROBERTSON: return fn(Robertson{});
    case F_NFW: return fn(NfwMiyamotoNagai{});
    case F_LIN1: return fn(Linear<1>{});
    case F_LIN2: return fn(Linear<2>{});
    case F_LIN3: return fn(Linear<3>{});
    case F_LOGHALO: return fn(LogHalo{});
    case F_HIRES: return fn(Hires{});
    default: return -2;
  }
}

template <class F>
bool method_ok(int method) {
  if (method == TSIT5 || method == VERN7) return true;
  if (method == ROS34PW2 || method == RB23) return has_jac<F>::value;
  return false;
}

}  // namespace

extern "C" {

int orc_field_dims(int field, int* D, int* M) {
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    *D = F::D;
    *M = F::M;
    return 0;
  });
}

int orc_solve(int field, int method, int dtype, long long N, int theta_shared, const void* theta,
              const void* y0, double t0, double t1, double rtol, double atol,
              long long max_attempts, void* y1, int* S, int* rej, int* status,
              long long* attempts, int keep_record, int Smax, void* Tout, void* Hout, void* Yout,
              int nthreads) {
  SolveArgs a{method, N, theta_shared, theta, y0, t0, t1, rtol, atol, max_attempts, y1, S, rej,
              status, attempts, keep_record, Smax, Tout, Hout, Yout, nthreads};
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if (!method_ok<F>(method)) return -3;
    return dtype == 0 ? solve_impl<F, double>(a) : dtype == 1 ? solve_impl<F, float>(a) : -4;
  });
}

int orc_replay(int field, int method, int dtype, long long N, int theta_shared, const void* theta,
               const void* y0, const void* H, const int* S, int Smax, void* y_out, int nthreads) {
  ReplayArgs a{method, N, theta_shared, theta, y0, H, S, Smax, nullptr, y_out, nullptr, nullptr,
               nthreads};
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if (!method_ok<F>(method)) return -3;
    return dtype == 0 ? replay_impl<F, double>(a) : dtype == 1 ? replay_impl<F, float>(a) : -4;
  });
}

// dL_dth is always per trajectory [N][M] here; a caller wanting the shared-theta gradient sums
// the rows (the ensemble loss is a plain sum over trajectories, [GS] §2.2).
int orc_replay_grad(int field, int method, int dtype, long long N, int theta_shared,
                    const void* theta, const void* y0, const void* H, const int* S, int Smax,
                    const void* lam, void* dL_dy0, void* dL_dth, int nthreads) {
  ReplayArgs a{method, N, theta_shared, theta, y0, H, S, Smax, lam, nullptr, dL_dy0, dL_dth,
               nthreads};
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if (!method_ok<F>(method)) return -3;
    return dtype == 0 ? grad_impl<F, double>(a) : dtype == 1 ? grad_impl<F, float>(a) : -4;
  });
}

// States at requested times tau[J] (ascending, in [t0, t1]) over the padded record (T, H, S):
// out [N][J][D]; and the gradient of sum_j lam_j . y(tau_j) (lam [N][J][D]).
int orc_replay_outputs(int field, int method, int dtype, long long N, int theta_shared,
                       const void* theta, const void* y0, const void* T, const void* H,
                       const int* S, int Smax, double t1, int J, const void* tau, void* out,
                       int nthreads) {
  OutArgs a{method, N, theta_shared, theta, y0, T, H, S, Smax, t1, J, tau, nullptr, out,
            nullptr, nullptr, nthreads};
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if (!method_ok<F>(method)) return -3;
    return dtype == 0 ? outputs_impl<F, double>(a, false)
                      : dtype == 1 ? outputs_impl<F, float>(a, false) : -4;
  });
}

int orc_replay_outputs_grad(int field, int method, int dtype, long long N, int theta_shared,
                            const void* theta, const void* y0, const void* T, const void* H,
                            const int* S, int Smax, double t1, int J, const void* tau,
                            const void* lam, void* dL_dy0, void* dL_dth, int nthreads) {
  OutArgs a{method, N, theta_shared, theta, y0, T, H, S, Smax, t1, J, tau, lam, nullptr,
            dL_dy0, dL_dth, nthreads};
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if (!method_ok<F>(method)) return -3;
    return dtype == 0 ? outputs_impl<F, double>(a, true)
                      : dtype == 1 ? outputs_impl<F, float>(a, true) : -4;
  });
}

// Tangent of the replay's final state along (ydot0 [N][D], thdot [N][M] or [M]) over the padded
// mesh: y1 [N][D], ydot1 [N][D].
int orc_replay_jvp(int field, int method, int dtype, long long N, int theta_shared,
                   const void* theta, const void* y0, const void* thdot, const void* ydot0,
                   const void* H, const int* S, int Smax, void* y1, void* ydot1, int nthreads) {
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if (!method_ok<F>(method)) return -3;
    auto run = [&](auto zero) {
      using R = decltype(zero);
      constexpr int D = F::D, M = F::M;
      const R* th = static_cast<const R*>(theta);
      const R* td = static_cast<const R*>(thdot);
      parallel_for(N, nthreads, [&](long long k) {
        const long long to = theta_shared ? 0 : k * M;
        replay_jvp<F, R>(Method(method), static_cast<const R*>(y0) + k * D, th + to,
                         static_cast<const R*>(ydot0) + k * D, td + to,
                         static_cast<const R*>(H) + k * (long long)Smax, S[k],
                         static_cast<R*>(y1) + k * D, static_cast<R*>(ydot1) + k * D);
      });
      return 0;
    };
    return dtype == 0 ? run(0.0) : dtype == 1 ? run(0.0f) : -4;
  });
}

// Orbit plus forward sensitivities S = dy/dtheta [N][D][M] (Tsit5, control on y alone).
// S0 [N][D][M] may be NULL (zero start, theta does not enter y0).
int orc_solve_sens(int field, int dtype, long long N, int theta_shared, const void* theta,
                   const void* y0, const void* S0, double t0, double t1, double rtol, double atol,
                   long long max_attempts, void* y1, void* S1, int* S, int* rej, int* status,
                   int nthreads) {
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if constexpr (F::M > 16) {
      return -3;  // the dual width is the parameter count: kept to small M
    } else {
      auto run = [&](auto zero) {
        using R = decltype(zero);
        constexpr int D = F::D, M = F::M;
        const R* th = static_cast<const R*>(theta);
        parallel_for(N, nthreads, [&](long long k) {
          const R* s0 = S0 ? static_cast<const R*>(S0) + k * D * M : nullptr;
          Record<R> r = solve_sens<F, R>(static_cast<const R*>(y0) + k * D, s0,
                                         th + (theta_shared ? 0 : k * M), R(t0), R(t1), R(rtol),
                                         R(atol), max_attempts,
                                         static_cast<R*>(S1) + k * D * M);
          for (int c = 0; c < D; ++c) static_cast<R*>(y1)[k * D + c] = r.y1[c];
          if (S) S[k] = r.S;
          if (rej) rej[k] = r.rejected;
          if (status) status[k] = r.status;
        });
        return 0;
      };
      return dtype == 0 ? run(0.0) : dtype == 1 ? run(0.0f) : -4;
    }
  });
}

// f(y; theta) for N states (double only; used by field-level checks).
int orc_rhs(int field, long long N, int theta_shared, const double* theta, const double* y,
            double* out) {
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    for (long long k = 0; k < N; ++k)
      F::f(y + k * F::D, theta + (theta_shared ? 0 : k * F::M), out + k * F::D);
    return 0;
  });
}

// Analytic Jacobian df/dy [N][D][D] of the stiff fields (double only).
int orc_jac(int field, long long N, int theta_shared, const double* theta, const double* y,
            double* J) {
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if constexpr (has_jac<F>::value) {
      for (long long k = 0; k < N; ++k)
        F::jac(y + k * F::D, theta + (theta_shared ? 0 : k * F::M), J + k * F::D * F::D);
      return 0;
    } else {
      return -3;
    }
  });
}

// One trial step (double) from (y, h) with its error estimate: ynew[D], e[D].
int orc_trial(int field, int method, const double* theta, const double* y, double h,
              double* ynew, double* e) {
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    if (!method_ok<F>(method)) return -3;
    if (method == TSIT5) {
      double k1[F::D], k7[F::D];
      F::f(y, theta, k1);
      tsit5_trial<F, double>(y, h, theta, k1, ynew, k7, e, true);
    } else if (method == VERN7) {
      double k1[F::D];
      F::f(y, theta, k1);
      vern7_trial<F, double>(y, h, theta, k1, ynew, e, true);
    } else if (method == RB23) {
      if constexpr (has_jac<F>::value) rb23_trial<F, double>(y, h, theta, ynew, e, true);
    } else {
      if constexpr (has_jac<F>::value) ros_trial<F, double>(y, h, theta, ynew, e, true);
    }
    return 0;
  });
}

// Arithmetic tally of one f evaluation (what=0), one Tsit5 trial step with error estimate
// (what=1), one Rosenbrock trial step (what=2), f on one-direction dual numbers (what=3), or the
// reverse sweep of f's vector-Jacobian product with respect to (y, theta) taken by a plain
// reverse-mode pass over f's operations (what=4), at state y and parameters theta.
// counts = {add, mul, div, sqrt, log1p, tanh}.
int orc_count_ops(int field, int what, const double* theta, const double* y, double h,
                  long long* counts) {
  return with_field(field, [&](auto fld) {
    using F = decltype(fld);
    std::vector<Cnt> th(F::M);
    Cnt yy[F::D], out[F::D], k1[F::D], k7[F::D], e[F::D];
    for (int j = 0; j < F::M; ++j) th[j] = Cnt(theta[j]);
    for (int c = 0; c < F::D; ++c) yy[c] = Cnt(y[c]);
    for (int c = 0; c < F::D; ++c) k1[c] = Cnt(0.0);
    tally() = OpTally{};
    if (what == 0) {
      F::f(yy, th.data(), out);
    } else if (what == 3) {
      // f with one tangent direction (forward-mode rules): value + directional derivative
      using DC = Dual<Cnt, 1>;
      std::vector<DC> thd(F::M);
      DC yd[F::D], od[F::D];
      for (int j = 0; j < F::M; ++j) { thd[j] = DC(th[j]); thd[j].g[0] = Cnt(j == 0 ? 1.0 : 0.0); }
      for (int c = 0; c < F::D; ++c) { yd[c] = DC(yy[c]); yd[c].g[0] = Cnt(1.0); }
      tally() = OpTally{};
      F::f(yd, thd.data(), od);
    } else if (what == 4) {
      std::vector<Tap> tht(F::M);
      Tap yt[F::D], ot[F::D];
      tape().clear();
      for (int c = 0; c < F::D; ++c) yt[c] = Tap::leaf(y[c]);
      for (int j = 0; j < F::M; ++j) tht[j] = Tap::leaf(theta[j]);
      F::f(yt, tht.data(), ot);
      int outs[F::D];
      for (int c = 0; c < F::D; ++c) outs[c] = ot[c].id;
      const OpTally t = tally_reverse_sweep(outs, F::D);
      tape().clear();
      counts[0] = t.add; counts[1] = t.mul; counts[2] = t.div;
      counts[3] = t.sqrt; counts[4] = t.log1p; counts[5] = t.tanh;
      return 0;
    } else if (what == 1) {
      tsit5_trial<F, Cnt>(yy, Cnt(h), th.data(), k1, out, k7, e, true);
    } else {
      if constexpr (has_jac<F>::value) ros_trial<F, Cnt>(yy, Cnt(h), th.data(), out, e, true);
      else return -3;
    }
    const OpTally t = tally();
    counts[0] = t.add; counts[1] = t.mul; counts[2] = t.div;
    counts[3] = t.sqrt; counts[4] = t.log1p; counts[5] = t.tanh;
    return 0;
  });
}

// The method tables as the oracle holds them (for the order-condition pins).
void orc_tsit5_tableau(double* C7, double* A49, double* B7, double* BT7) {
  for (int i = 0; i < 7; ++i) {
    C7[i] = Tsit5Tab::C[i];
    B7[i] = Tsit5Tab::B[i];
    BT7[i] = Tsit5Tab::BT[i];
    for (int j = 0; j < 7; ++j) A49[i * 7 + j] = j < 6 ? Tsit5Tab::A[i][j] : 0.0;
  }
}
void orc_vern7_tableau(double* A100, double* B10, double* BH10) {
  for (int i = 0; i < 10; ++i) {
    B10[i] = Vern7Tab::B[i];
    BH10[i] = Vern7Tab::BH[i];
    for (int j = 0; j < 10; ++j) A100[i * 10 + j] = j < 9 ? Vern7Tab::A[i][j] : 0.0;
  }
}
void orc_ros34pw2_tableau(double* gamma, double* ALPHA16, double* GAMMA16, double* B4,
                          double* BHAT4) {
  *gamma = Ros34pw2Tab::gamma;
  for (int i = 0; i < 4; ++i) {
    B4[i] = Ros34pw2Tab::B[i];
    BHAT4[i] = Ros34pw2Tab::BHAT[i];
    for (int j = 0; j < 4; ++j) {
      ALPHA16[i * 4 + j] = j < 3 ? Ros34pw2Tab::ALPHA[i][j] : 0.0;
      GAMMA16[i * 4 + j] = j < 3 ? Ros34pw2Tab::GAMMA[i][j] : 0.0;
    }
  }
}

}  // extern "C"
