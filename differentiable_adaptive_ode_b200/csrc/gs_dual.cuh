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

#ifdef __CUDACC__
#include "gs_log_table.cuh"
#endif

namespace gs {

#ifdef __CUDACC__
// Natural logarithm of a positive normal x, table-driven (P. T. P. Tang, "Table-driven
// implementation of the logarithm function in IEEE floating-point arithmetic", ACM TOMS 16(4),
// 1990), written here for the stellar field's log(1 + r/r_s), one per stage: x = 2^e m,
// m in [1, 2); c_j = 1 + j/128 the breakpoint nearest m and g_j = RN(1/c_j), so that
//   log x = e ln2 + L_j + log(1 + r),  r = m g_j - 1,  |r| <= 2^-8 + 2^-53,  L_j = -log(g_j),
// with L_j tabulated to about 2^-95 (gs_log_table.cuh, from gen_log_table.py).  The product m g_j
// is split exactly into its rounded value p and its error (an FMA), and p - 1 is exact (p lies
// within 2^-7 of 1), so r = rh + rl exactly.  log(1 + r) = rh + rh^2 P(rh) + rl (1 - rh) to about
// 2^-67: P the Taylor polynomial -1/2 + r/3 - ... + r^5/7, evaluated in two halves.  The head
// e ln2_hi + L_j,hi is exact (both on the 2^-42 grid), its sum with rh is carried with its rounding
// error (Fast2Sum: the head is 0 or at least log(1 + 1/128) > |rh|), and the small terms join
// last: within about half an ulp plus the final rounding (0.52 ulp the largest error seen, against
// 0.53 for CUDA's log on the same arguments).  Every operation is rounded on its own
// (explicit FMAs and _rn intrinsics), so all kernels that inline it round identically.  About 20
// FP64 operations and two table loads (L1-resident, 4 KB), with no branch: the same steps hold
// for every positive normal x (the head is then 0 or larger than |rh| as well), and the other
// arguments are sorted out by integer tests on the bits at the end (+inf -> +inf, +0 -> -inf;
// negative, NaN and subnormal arguments -> NaN).
__device__ __forceinline__ double log_tab(double x) {
  const long long b = __double_as_longlong(x);
  const int e = (int)(b >> 52) - 1023;
  const int j = ((int)((b >> 44) & 0xFF) + 1) >> 1;
  const double m = __longlong_as_double((b & 0x000FFFFFFFFFFFFFLL) | 0x3FF0000000000000LL);
  const double2 gl = __ldg(reinterpret_cast<const double2*>(&c_log_tab[j]));  // g_j, L_j,hi
  const double llo = __ldg(&c_log_tab[j].llo);
  const double p = __dmul_rn(m, gl.x);
  const double rl = fma(m, gl.x, -p);
  const double rh = __dsub_rn(p, 1.0);
  // e as a double with integer arithmetic only: the double 1.5 2^52 + e holds e in its low bits
  const double ed = __dsub_rn(__longlong_as_double(0x4338000000000000LL + e), 0x1.8p52);
  const double A = fma(ed, LOG_LN2_HI, gl.y);
  const double B = fma(ed, LOG_LN2_LO, llo);
  const double r2 = __dmul_rn(rh, rh);
  const double p01 = fma(rh, 1.0 / 3.0, -0.5);
  const double p23 = fma(rh, 0.2, -0.25);
  const double p45 = fma(rh, 1.0 / 7.0, -1.0 / 6.0);
  const double P = fma(r2, fma(r2, p45, p23), p01);
  const double q = __dmul_rn(r2, P);
  const double S = __dadd_rn(A, rh);
  const double z = __dadd_rn(__dsub_rn(A, S), rh);
  const double small = __dadd_rn(fma(-rh, rl, rl), __dadd_rn(B, q));
  const double res = __dadd_rn(S, __dadd_rn(z, small));
  const bool normal = b >= 0x0010000000000000LL && b < 0x7FF0000000000000LL;
  const long long special = b == 0x7FF0000000000000LL ? b                       // +inf
                            : b == 0 ? (long long)0xFFF0000000000000ULL         // -inf
                                     : 0x7FF8000000000000LL;                   // NaN
  return normal ? res : __longlong_as_double(special);
}
#endif

// log(1 + x) for x > -1, given a and b with a * b = 1 / (1 + x) to a few ulps (a reciprocal that
// the caller has at hand).  fp64: w = fl(1 + x) and its rounding error c, 1 + x = w + c exactly
// (Knuth's TwoSum, branch-free); then log(1 + x) = log(w) + c / w up to (c / w)^2 <= 2^-106, and
// 1 / w = a * b to a few ulps suffices for the small correction.  On the device log w is
// log_tab (w >= 1 when x >= 0; within about half an ulp), so the result stays within about an
// ulp at the cost of that log, six adds and a multiply-add, with no division.  The sums are
// rounded one by one on the device, which the exactness of c needs; a
// caller whose x is a product forms it with mul_rn, so that no kernel fuses that product into
// the sums (the forward-only and recording solvers then stay bit-for-bit alike).  fp32 keeps
// log1pf.
GS_DHD double log1p_q(double x, double a, double b) {
#ifdef __CUDA_ARCH__
  const double w = __dadd_rn(1.0, x);
  const double xv = __dsub_rn(w, 1.0);
  const double c = __dadd_rn(__dsub_rn(1.0, __dsub_rn(w, xv)), __dsub_rn(x, xv));
  return fma(c, __dmul_rn(a, b), log_tab(w));
#else
  const double w = 1.0 + x;
  const double xv = w - 1.0;
  const double c = (1.0 - (w - xv)) + (x - xv);
  return fma(c, a * b, log(w));
#endif
}
GS_DHD float log1p_q(float x, float, float) { return log1pf(x); }

// a * b and a + b rounded on their own: on the device the product is never fused into a later
// sum, nor the sum into an earlier product.  Written with these (and explicit fma), an expression
// rounds the same way in every kernel that inlines it, whatever the compiler could otherwise merge
// or fuse around it.
template <class R> GS_DHD R mul_rn(R a, R b) { return a * b; }
template <class R> GS_DHD R add_rn(R a, R b) { return a + b; }
#ifdef __CUDA_ARCH__
template <> GS_DHD double mul_rn<double>(double a, double b) { return __dmul_rn(a, b); }
template <> GS_DHD float mul_rn<float>(float a, float b) { return __fmul_rn(a, b); }
template <> GS_DHD double add_rn<double>(double a, double b) { return __dadd_rn(a, b); }
template <> GS_DHD float add_rn<float>(float a, float b) { return __fadd_rn(a, b); }
#endif

// 1/x and 1/sqrt(x) for normal, positive, finite x: the hardware's approximations
// (rcp.approx.ftz.f64, rsqrt.approx.ftz.f64: relative error near 2^-22) refined by one
// third-order step (the series of (1 - e)^(-1) and (1 - e)^(-1/2) to second order in the
// residual): with e = 1 - x y, 1/x = y (1 + e + e^2 + ...); with e = 1 - x y^2,
// 1/sqrt(x) = y (1 + e/2 + 3 e^2/8 + ...).  The dropped terms are below e^3 <= 2^-63 relative,
// so what remains is the rounding of the few operations: within about an ulp of the exact value
// (checked against long double), without the special-case paths of a general division or rsqrt.
// Other scalar types (float, dual numbers, the counting scalar) take the plain operations.
template <class R> GS_DHD R rsqrt_nr(R x) { return rsqrt(x); }
template <class R> GS_DHD R rcp_nr(R x) { return R(1) / x; }
#ifdef __CUDA_ARCH__
template <> __device__ __forceinline__ double rsqrt_nr<double>(double x) {
  double y;
  asm("rsqrt.approx.ftz.f64 %0, %1;" : "=d"(y) : "d"(x));
  const double e = fma(-x * y, y, 1.0);
  return fma(y * fma(0.375, e, 0.5), e, y);
}
template <> __device__ __forceinline__ double rcp_nr<double>(double x) {
  double y;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(y) : "d"(x));
  const double e = fma(-x, y, 1.0);
  return fma(y, fma(e, e, e), y);
}
#endif

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
  // a b + c: d = a' b + a b' + c'
  friend GS_DHD Dl fma(const Dl& a, const Dl& b, const Dl& c) {
    return Dl(fma(a.v, b.v, c.v), fma(a.d, b.v, fma(a.v, b.d, c.d)));
  }
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
  // d log(1 + x) = dx / (1 + x) = dx * (p * q) when p * q = 1 / (1 + x)
  friend GS_DHD Dl log1p_q(const Dl& x, const Dl& p, const Dl& q) {
    const R iw = p.v * q.v;
    return Dl(log1p_q(x.v, p.v, q.v), x.d * iw);
  }
  friend GS_DHD Dl log1p(const Dl& a) {
    return Dl(log1p(a.v), a.d / (R(1) + a.v));
  }
};

}  // namespace gs
