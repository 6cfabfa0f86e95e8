// gs_dual.cuh -- one-direction dual numbers for the device: a value and its derivative along one
// input direction.  A field's own f(), evaluated on these, returns f and its directional
// derivative J_y(y) ydot + J_theta(y) thdot in one pass -- the right-hand side of the forward
// sensitivity equations S' = J_y S + J_theta ("Differentiable astrophysics at scale" §2: the
// sensitivities are integrated together with the orbit in the same kernel).
//
// The functions are friends, found by argument-dependent lookup only, so that they do not hide
// the plain double/float math functions inside namespace gs.
#pragma once
// Host-callable too (plain C++), so that the forward-mode rules can be tallied with a counting
// scalar like the fields themselves.
#ifdef __CUDACC__
#include <cuda_runtime.h>
#define GS_DHD __host__ __device__ __forceinline__
#else
#include <cmath>
#define GS_DHD inline
#endif

namespace gs {

template <class R>
struct Dl {
  R v, d;
  GS_DHD Dl() {}
  GS_DHD Dl(R x) : v(x), d(R(0)) {}
  GS_DHD Dl(R x, R dx) : v(x), d(dx) {}

  friend GS_DHD Dl operator+(const Dl& a, const Dl& b) {
    return Dl(a.v + b.v, a.d + b.d);
  }
  friend GS_DHD Dl operator-(const Dl& a, const Dl& b) {
    return Dl(a.v - b.v, a.d - b.d);
  }
  friend GS_DHD Dl operator-(const Dl& a) { return Dl(-a.v, -a.d); }
  friend GS_DHD Dl operator*(const Dl& a, const Dl& b) {
    return Dl(a.v * b.v, fma(a.d, b.v, a.v * b.d));
  }
  friend GS_DHD Dl operator/(const Dl& a, const Dl& b) {
    const R ib = R(1) / b.v;
    const R q = a.v * ib;
    return Dl(q, (a.d - q * b.d) * ib);
  }
  GS_DHD Dl& operator+=(const Dl& b) {
    v += b.v;
    d += b.d;
    return *this;
  }
  // d rsqrt(u) = -u'/(2 u^{3/2}),  d sqrt(u) = u'/(2 sqrt(u)),  d log1p(u) = u'/(1 + u)
  friend GS_DHD Dl rsqrt(const Dl& a) {
    const R r = rsqrt(a.v);
    return Dl(r, R(-0.5) * r * r * r * a.d);
  }
  friend GS_DHD Dl sqrt(const Dl& a) {
    const R s = sqrt(a.v);
    return Dl(s, R(0.5) * a.d / s);
  }
  friend GS_DHD Dl log1p(const Dl& a) {
    return Dl(log1p(a.v), a.d / (R(1) + a.v));
  }
};

}  // namespace gs
