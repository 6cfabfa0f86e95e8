// gs_fields.cuh -- right-hand sides f(y; theta) and their hand-written vector-Jacobian products
// for the device kernels.  Every field is autonomous.
//
// Interface of a field F (R = double or float):
//   F::D, F::M                       state size, parameter count
//   F::Theta<R>                      per-lane parameters (registers) plus hoisted invariants
//   F::load(Theta&, const R* src)    read M parameters, precompute what depends only on theta
//   F::f(y, th, dy)                  dy = f(y; theta)
//   F::vjp(y, th, kb, yb, thb)       yb = (df/dy)^T kb (overwritten), thb += (df/dtheta)^T kb
// Stiff fields also provide
//   F::jac(y, th, J)                 J = df/dy, row-major D x D
//   F::jac_vjp(y, th, Jb, yb, thb)   yb += sum_rc Jb_rc dJ_rc/dy,  thb += sum_rc Jb_rc dJ_rc/dtheta
//
// The reverse sweep that calls vjp() is the discrete adjoint of "gradsolve: fast exact gradients
// for ODE ensembles on GPUs" §3 (the gradient of the fixed-mesh replay) and §3.2 (the Rosenbrock
// stage also differentiates J, i.e. second derivatives of f).
#pragma once
// Fields are host-callable too (and compile as plain C++) so that their arithmetic can be
// tallied on the host with a counting scalar.
#ifdef __CUDACC__
#include <cuda_runtime.h>
#define GS_HD __host__ __device__ __forceinline__
#else
#include <cmath>
#define GS_HD inline
inline double rsqrt(double x) { return 1.0 / std::sqrt(x); }
inline float rsqrt(float x) { return 1.0f / std::sqrt(x); }
#endif
#include "gs_dual.cuh"

namespace gs {

// ----------------------------------------------------------------------------------------------
// Lotka-Volterra, theta = (alpha, beta, gamma, delta): x' = alpha x - beta x y, y' = delta x y - gamma y
// ----------------------------------------------------------------------------------------------
struct FLotkaVolterra {
  static constexpr int D = 2, M = 4;
  template <class R> struct Theta { R a, b, g, d; };
  template <class R> GS_HD static void load(Theta<R>& t, const R* s) {
    t.a = s[0]; t.b = s[1]; t.g = s[2]; t.d = s[3];
  }
  template <class R> GS_HD static void f(const R* y, const Theta<R>& t, R* dy) {
    const R xy = y[0] * y[1];
    dy[0] = t.a * y[0] - t.b * xy;
    dy[1] = t.d * xy - t.g * y[1];
  }
  template <class R>
  GS_HD static void vjp(const R* y, const Theta<R>& t, const R* kb, R* yb, R* thb) {
    yb[0] = (t.a - t.b * y[1]) * kb[0] + t.d * y[1] * kb[1];
    yb[1] = -(t.b * y[0]) * kb[0] + (t.d * y[0] - t.g) * kb[1];
    const R xy = y[0] * y[1];
    thb[0] += y[0] * kb[0];
    thb[1] -= xy * kb[0];
    thb[2] -= y[1] * kb[1];
    thb[3] += xy * kb[1];
  }
};

// ----------------------------------------------------------------------------------------------
// Lorenz-63, theta = (sigma, rho, beta)
// ----------------------------------------------------------------------------------------------
struct FLorenz63 {
  static constexpr int D = 3, M = 3;
  template <class R> struct Theta { R s, r, b; };
  template <class R> GS_HD static void load(Theta<R>& t, const R* s) {
    t.s = s[0]; t.r = s[1]; t.b = s[2];
  }
  template <class R> GS_HD static void f(const R* y, const Theta<R>& t, R* dy) {
    dy[0] = t.s * (y[1] - y[0]);
    dy[1] = y[0] * (t.r - y[2]) - y[1];
    dy[2] = y[0] * y[1] - t.b * y[2];
  }
  template <class R>
  GS_HD static void vjp(const R* y, const Theta<R>& t, const R* kb, R* yb, R* thb) {
    yb[0] = -t.s * kb[0] + (t.r - y[2]) * kb[1] + y[1] * kb[2];
    yb[1] = t.s * kb[0] - kb[1] + y[0] * kb[2];
    yb[2] = -y[0] * kb[1] - t.b * kb[2];
    thb[0] += (y[1] - y[0]) * kb[0];
    thb[1] += y[0] * kb[1];
    thb[2] -= y[2] * kb[2];
  }
};

// ----------------------------------------------------------------------------------------------
// Robertson kinetics (stiff), theta = (k1, k2, k3)
//   y1' = -k1 y1 + k3 y2 y3,  y2' = k1 y1 - k2 y2^2 - k3 y2 y3,  y3' = k2 y2^2
// ----------------------------------------------------------------------------------------------
struct FRobertson {
  static constexpr int D = 3, M = 3;
  template <class R> struct Theta { R k1, k2, k3; };
  template <class R> GS_HD static void load(Theta<R>& t, const R* s) {
    t.k1 = s[0]; t.k2 = s[1]; t.k3 = s[2];
  }
  template <class R> GS_HD static void f(const R* y, const Theta<R>& t, R* dy) {
    const R a = t.k1 * y[0], b = t.k2 * y[1] * y[1], c = t.k3 * y[1] * y[2];
    dy[0] = -a + c;
    dy[1] = a - b - c;
    dy[2] = b;
  }
  template <class R> GS_HD static void jac(const R* y, const Theta<R>& t, R* J) {
    J[0] = -t.k1; J[1] = t.k3 * y[2];                        J[2] = t.k3 * y[1];
    J[3] = t.k1;  J[4] = -R(2) * t.k2 * y[1] - t.k3 * y[2];  J[5] = -t.k3 * y[1];
    J[6] = R(0);  J[7] = R(2) * t.k2 * y[1];                 J[8] = R(0);
  }
  template <class R>
  GS_HD static void vjp(const R* y, const Theta<R>& t, const R* kb, R* yb, R* thb) {
    // yb = J^T kb
    const R d01 = kb[1] - kb[0];     // k1 y1 leaves y1 and enters y2
    const R d12 = kb[2] - kb[1];     // k2 y2^2 leaves y2 and enters y3
    const R d10 = kb[0] - kb[1];     // k3 y2 y3 leaves y2 and enters y1
    yb[0] = t.k1 * d01;
    yb[1] = R(2) * t.k2 * y[1] * d12 + t.k3 * y[2] * d10;
    yb[2] = t.k3 * y[1] * d10;
    thb[0] += y[0] * d01;
    thb[1] += y[1] * y[1] * d12;
    thb[2] += y[1] * y[2] * d10;
  }
  // J depends on y only through y2, y3 and linearly: the second derivatives are constants.
  template <class R>
  GS_HD static void jac_vjp(const R* y, const Theta<R>& t, const R* Jb, R* yb, R* thb) {
    // dJ12/dy3 = k3, dJ13/dy2 = k3, dJ22/dy2 = -2 k2, dJ22/dy3 = -k3, dJ23/dy2 = -k3, dJ32/dy2 = 2 k2
    yb[1] += t.k3 * (Jb[2] - Jb[5]) + R(2) * t.k2 * (Jb[7] - Jb[4]);
    yb[2] += t.k3 * (Jb[1] - Jb[4]);
    // dJ/dk1: J11 = -k1, J21 = k1;  dJ/dk2: J22 = -2 k2 y2, J32 = 2 k2 y2;
    // dJ/dk3: J12 = k3 y3, J13 = k3 y2, J22 = -k3 y3, J23 = -k3 y2
    thb[0] += Jb[3] - Jb[0];
    thb[1] += R(2) * y[1] * (Jb[7] - Jb[4]);
    thb[2] += y[2] * (Jb[1] - Jb[4]) + y[1] * (Jb[2] - Jb[5]);
  }
};

// ----------------------------------------------------------------------------------------------
// HIRES (Schaefer 1975; Hairer & Wanner II §IV.10), stiff, theta = the twelve rate constants
// k = (1.71, 0.43, 8.32, 0.0007, 8.75, 10.03, 0.035, 1.12, 1.745, 280, 0.69, 1.81) nominal:
//   f0 = -k0 y0 + k1 y1 + k2 y2 + k3          f4 = -k8 y4 + k1 y5 + k1 y6
//   f1 =  k0 y0 - k4 y1                        f5 = -r + k10 y3 + k0 y4 - k1 y5 + k10 y6
//   f2 = -k5 y2 + k1 y3 + k6 y4                f6 =  r - k11 y6
//   f3 =  k2 y1 + k0 y2 - k7 y3                f7 = -r + k11 y6,      r = k9 y5 y7.
// J depends on y only through r (entries (5|6|7, 5|7)), linearly: its derivatives are constants.
// ----------------------------------------------------------------------------------------------
struct FHires {
  static constexpr int D = 8, M = 12;
  template <class R> struct Theta { R k[12]; };
  template <class R> GS_HD static void load(Theta<R>& t, const R* s) {
#pragma unroll
    for (int i = 0; i < 12; ++i) t.k[i] = s[i];
  }
  template <class R> GS_HD static void f(const R* y, const Theta<R>& t, R* dy) {
    const R* k = t.k;
    const R r = k[9] * y[5] * y[7];
    dy[0] = -k[0] * y[0] + k[1] * y[1] + k[2] * y[2] + k[3];
    dy[1] = k[0] * y[0] - k[4] * y[1];
    dy[2] = -k[5] * y[2] + k[1] * y[3] + k[6] * y[4];
    dy[3] = k[2] * y[1] + k[0] * y[2] - k[7] * y[3];
    dy[4] = -k[8] * y[4] + k[1] * y[5] + k[1] * y[6];
    dy[5] = -r + k[10] * y[3] + k[0] * y[4] - k[1] * y[5] + k[10] * y[6];
    dy[6] = r - k[11] * y[6];
    dy[7] = -r + k[11] * y[6];
  }
  // Structural nonzeros of jac: bit c of row r (the iteration matrices' LU skips the rest).
  GS_HD static constexpr bool jac_nz(int r, int c) {
    constexpr unsigned rows[8] = {0x07, 0x03, 0x1C, 0x0E, 0x70, 0xF8, 0xE0, 0xE0};
    return r >= 0 && r < 8 && c >= 0 && c < 8 && ((rows[r] >> c) & 1u) != 0;
  }
  template <class R> GS_HD static void jac(const R* y, const Theta<R>& t, R* J) {
    const R* k = t.k;
#pragma unroll
    for (int i = 0; i < 64; ++i) J[i] = R(0);
    J[0] = -k[0];  J[1] = k[1];  J[2] = k[2];
    J[8] = k[0];   J[9] = -k[4];
    J[18] = -k[5]; J[19] = k[1]; J[20] = k[6];
    J[25] = k[2];  J[26] = k[0]; J[27] = -k[7];
    J[36] = -k[8]; J[37] = k[1]; J[38] = k[1];
    const R a = k[9] * y[7], b = k[9] * y[5];
    J[43] = k[10]; J[44] = k[0]; J[45] = -a - k[1]; J[46] = k[10]; J[47] = -b;
    J[53] = a;     J[54] = -k[11]; J[55] = b;
    J[61] = -a;    J[62] = k[11];  J[63] = -b;
  }
  template <class R>
  GS_HD static void vjp(const R* y, const Theta<R>& t, const R* u, R* yb, R* thb) {
    const R* k = t.k;
    const R w = u[6] - u[5] - u[7];   // cotangent of r
    yb[0] = k[0] * (u[1] - u[0]);
    yb[1] = k[1] * u[0] - k[4] * u[1] + k[2] * u[3];
    yb[2] = k[2] * u[0] - k[5] * u[2] + k[0] * u[3];
    yb[3] = k[1] * u[2] - k[7] * u[3] + k[10] * u[5];
    yb[4] = k[6] * u[2] - k[8] * u[4] + k[0] * u[5];
    yb[5] = k[1] * (u[4] - u[5]) + k[9] * y[7] * w;
    yb[6] = k[1] * u[4] + k[10] * u[5] + k[11] * (u[7] - u[6]);
    yb[7] = k[9] * y[5] * w;
    thb[0] += y[0] * (u[1] - u[0]) + y[2] * u[3] + y[4] * u[5];
    thb[1] += y[1] * u[0] + y[3] * u[2] + (y[5] + y[6]) * u[4] - y[5] * u[5];
    thb[2] += y[2] * u[0] + y[1] * u[3];
    thb[3] += u[0];
    thb[4] -= y[1] * u[1];
    thb[5] -= y[2] * u[2];
    thb[6] += y[4] * u[2];
    thb[7] -= y[3] * u[3];
    thb[8] -= y[4] * u[4];
    thb[9] += y[5] * y[7] * w;
    thb[10] += (y[3] + y[6]) * u[5];
    thb[11] += y[6] * (u[7] - u[6]);
  }
  template <class R>
  GS_HD static void jac_vjp(const R* y, const Theta<R>& t, const R* Jb, R* yb, R* thb) {
    const R* k = t.k;
    const R wa = Jb[53] - Jb[45] - Jb[61];   // entries carrying a = k9 y7
    const R wb = Jb[55] - Jb[47] - Jb[63];   // entries carrying b = k9 y5
    yb[7] += k[9] * wa;
    yb[5] += k[9] * wb;
    thb[0] += Jb[8] - Jb[0] + Jb[26] + Jb[44];
    thb[1] += Jb[1] + Jb[19] + Jb[37] + Jb[38] - Jb[45];
    thb[2] += Jb[2] + Jb[25];
    thb[4] -= Jb[9];
    thb[5] -= Jb[18];
    thb[6] += Jb[20];
    thb[7] -= Jb[27];
    thb[8] -= Jb[36];
    thb[9] += y[7] * wa + y[5] * wb;
    thb[10] += Jb[43] + Jb[46];
    thb[11] += Jb[62] - Jb[54];
  }
};

// ----------------------------------------------------------------------------------------------
// Linear test field y' = A y, theta = A (row-major 3x3); J = A.
// ----------------------------------------------------------------------------------------------
struct FLinear3 {
  static constexpr int D = 3, M = 9;
  template <class R> struct Theta { R A[9]; };
  template <class R> GS_HD static void load(Theta<R>& t, const R* s) {
#pragma unroll
    for (int i = 0; i < 9; ++i) t.A[i] = s[i];
  }
  template <class R> GS_HD static void f(const R* y, const Theta<R>& t, R* dy) {
#pragma unroll
    for (int r = 0; r < 3; ++r) dy[r] = t.A[3 * r] * y[0] + t.A[3 * r + 1] * y[1] + t.A[3 * r + 2] * y[2];
  }
  template <class R> GS_HD static void jac(const R*, const Theta<R>& t, R* J) {
#pragma unroll
    for (int i = 0; i < 9; ++i) J[i] = t.A[i];
  }
  template <class R>
  GS_HD static void vjp(const R* y, const Theta<R>& t, const R* kb, R* yb, R* thb) {
#pragma unroll
    for (int c = 0; c < 3; ++c) yb[c] = t.A[c] * kb[0] + t.A[3 + c] * kb[1] + t.A[6 + c] * kb[2];
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
      for (int c = 0; c < 3; ++c) thb[3 * r + c] += kb[r] * y[c];
  }
  template <class R>
  GS_HD static void jac_vjp(const R*, const Theta<R>&, const R* Jb, R*, R* thb) {
#pragma unroll
    for (int i = 0; i < 9; ++i) thb[i] += Jb[i];
  }
};

// ----------------------------------------------------------------------------------------------
// Test particle in an NFW halo plus a Miyamoto-Nagai disk, G = 1.
// State (x, y, z, vx, vy, vz); theta = (M_h, r_s, M_d, a, b).
//   Phi = -M_h ln(1 + r/r_s)/r - M_d/D,  D^2 = R^2 + (a + B)^2,  B = sqrt(z^2 + b^2)
//   x' = v,  v' = acc = -gN x - gM w,  w = (x, y, z q),  q = (a + B)/B,
//   gN = M_h (L/r^3 - 1/(r^2 (r_s + r))),  L = ln(1 + r/r_s),  gM = M_d / D^3.
// VJP (u = cotangent of v'):
//   d acc/dx = -[gN I + (gN'/r) x x^T] - [gM diag(1, 1, q - a z^2/B^3) - 3 gM/D^2 w w^T]
//   gN'/r = M_h [3/(r^4 (r_s + r)) - 3 L / r^5 + 1/(r^3 (r_s + r)^2)]
//   d acc/dM_h = -(gN/M_h) x,     d acc/dr_s = M_h/(r r_s (r_s + r)^2) x,
//   d acc/dM_d = -w/D^3,
//   d acc/da = 3 gM (a+B)/D^2 w - gM (0, 0, z/B),
//   d acc/db = 3 gM (a+B) b/(B D^2) w + gM (0, 0, a b z/B^3).
// Per-lane invariants of theta (1/r_s, b^2) are hoisted into Theta.
// ----------------------------------------------------------------------------------------------
struct FNfwMiyamotoNagai {
  static constexpr int D = 6, M = 5;
  template <class R> struct Theta { R Mh, rs, Md, a, b, irs, b2; };
  template <class R> GS_HD static void load(Theta<R>& t, const R* s) {
    t.Mh = s[0]; t.rs = s[1]; t.Md = s[2]; t.a = s[3]; t.b = s[4];
    t.irs = R(1) / t.rs;
    t.b2 = t.b * t.b;
  }
  // Quantities of f shared with the VJP; one division, three reciprocal square roots, one log1p.
  // Every rounding is spelled out (explicit fma, mul_rn, add_rn): f is inlined into the solve,
  // record and sensitivity kernels, and must round the same way in each of them.  Its operands
  // are normal and positive (r^2 > 0, z^2 + b^2 >= b^2, r_s + r >= r_s), so the reciprocal and
  // the reciprocal square roots take the refined hardware approximations (rcp_nr, rsqrt_nr):
  // measured on the 2^20 stellar ensemble against CUDA's division and rsqrt, record 16.2 -> 15.1
  // ms, replay adjoint 12.6 -> 11.6 ms.
  template <class R> struct Inter { R R2, r, ir, L, isr, gN, iB, apB, iD, gM; };
  template <class R> GS_HD static void inter(const R* y, const Theta<R>& t, Inter<R>& I) {
    const R x = y[0], yy = y[1], z = y[2];
    I.R2 = fma(x, x, mul_rn(yy, yy));
    const R r2 = fma(z, z, I.R2);
    I.ir = rsqrt_nr(r2);
    I.r = mul_rn(r2, I.ir);
    I.isr = rcp_nr(add_rn(t.rs, I.r));
    I.L = log1p_q(mul_rn(I.r, t.irs), t.rs, I.isr);  // rs / (rs + r) = 1 / (1 + r / rs)
    I.gN = mul_rn(mul_rn(t.Mh, mul_rn(I.ir, I.ir)), fma(I.L, I.ir, -I.isr));
    const R B2 = fma(z, z, t.b2);
    I.iB = rsqrt_nr(B2);
    I.apB = fma(B2, I.iB, t.a);
    I.iD = rsqrt_nr(fma(I.apB, I.apB, I.R2));
    I.gM = mul_rn(t.Md, mul_rn(mul_rn(I.iD, I.iD), I.iD));
  }
  template <class R> GS_HD static void f(const R* y, const Theta<R>& t, R* dy) {
    Inter<R> I;
    inter(y, t, I);
    const R g = add_rn(I.gN, I.gM);
    dy[0] = y[3];
    dy[1] = y[4];
    dy[2] = y[5];
    dy[3] = -mul_rn(g, y[0]);
    dy[4] = -mul_rn(g, y[1]);
    dy[5] = -mul_rn(fma(mul_rn(I.gM, I.apB), I.iB, I.gN), y[2]);
  }
  // Tape of a stage for the reverse sweep: the five transcendental results of f at that stage,
  // so that the VJP recomputes only products and sums.
  static constexpr int TAPE = 5;
  template <class R> GS_HD static void inter_tape(const R* y, const Theta<R>& t, R* tp) {
    Inter<R> I;
    inter(y, t, I);
    tp[0] = I.ir; tp[1] = I.L; tp[2] = I.isr; tp[3] = I.iB; tp[4] = I.iD;
  }
  template <class R>
  GS_HD static void f_tape(const R* y, const Theta<R>& t, R* dy, R* tp) {
    Inter<R> I;
    inter(y, t, I);
    tp[0] = I.ir; tp[1] = I.L; tp[2] = I.isr; tp[3] = I.iB; tp[4] = I.iD;
    const R g = add_rn(I.gN, I.gM);
    dy[0] = y[3];
    dy[1] = y[4];
    dy[2] = y[5];
    dy[3] = -mul_rn(g, y[0]);
    dy[4] = -mul_rn(g, y[1]);
    dy[5] = -mul_rn(fma(mul_rn(I.gM, I.apB), I.iB, I.gN), y[2]);
  }
  template <class R>
  GS_HD static void vjp_tape(const R* y, const Theta<R>& t, const R* tp, const R* kb, R* yb,
                             R* thb) {
    Inter<R> I;
    const R x = y[0], yy = y[1], z = y[2];
    I.R2 = x * x + yy * yy;
    I.ir = tp[0];
    I.r = (I.R2 + z * z) * I.ir;
    I.L = tp[1];
    I.isr = tp[2];
    I.gN = t.Mh * (I.ir * I.ir) * (I.L * I.ir - I.isr);
    I.iB = tp[3];
    I.apB = t.a + (z * z + t.b2) * I.iB;
    I.iD = tp[4];
    I.gM = t.Md * (I.iD * I.iD * I.iD);
    vjp_from(y, t, I, kb, yb, thb);
  }
  template <class R>
  GS_HD static void vjp(const R* y, const Theta<R>& t, const R* kb, R* yb, R* thb) {
    Inter<R> I;
    inter(y, t, I);
    vjp_from(y, t, I, kb, yb, thb);
  }
  template <class R>
  GS_HD static void vjp_from(const R* y, const Theta<R>& t, const Inter<R>& I, const R* kb, R* yb,
                             R* thb) {
    const R x = y[0], yy = y[1], z = y[2];
    const R ux = kb[3], uy = kb[4], uz = kb[5];
    const R ir2 = I.ir * I.ir;
    const R Lir = I.L * I.ir;
    const R gNp_r = t.Mh * ir2 * ir2 * (R(3) * I.isr - R(3) * Lir + I.r * I.isr * I.isr);  // gN'/r
    const R q = I.apB * I.iB;
    const R iD2 = I.iD * I.iD;
    const R wz = z * q;
    const R xu = x * ux + yy * uy + z * uz;
    const R wu = x * ux + yy * uy + wz * uz;
    const R c3 = R(3) * I.gM * iD2 * wu;
    const R hz = q - t.a * z * z * I.iB * I.iB * I.iB;
    yb[0] = -(I.gN * ux + gNp_r * xu * x) - (I.gM * ux - c3 * x);
    yb[1] = -(I.gN * uy + gNp_r * xu * yy) - (I.gM * uy - c3 * yy);
    yb[2] = -(I.gN * uz + gNp_r * xu * z) - (I.gM * hz * uz - c3 * wz);
    yb[3] = kb[0];
    yb[4] = kb[1];
    yb[5] = kb[2];
    thb[0] -= ir2 * (Lir - I.isr) * xu;
    thb[1] += t.Mh * I.ir * t.irs * I.isr * I.isr * xu;
    thb[2] -= iD2 * I.iD * wu;
    thb[3] += I.apB * c3 - I.gM * z * I.iB * uz;
    thb[4] += t.b * I.iB * (I.apB * c3 + I.gM * t.a * z * I.iB * I.iB * uz);
  }
};

// ----------------------------------------------------------------------------------------------
// Test particle in an axisymmetric flattened logarithmic halo ("Differentiable astrophysics at
// scale" §3): Phi = (1/2) v_c^2 ln(R_c^2 + x^2 + y^2 + z^2/q^2), R_c = 0.2, theta = (v_c, q).
//   x' = v,  v' = acc = -g w,  w = (x, y, z/q^2),  g = v_c^2 / Q,  Q = R_c^2 + x^2 + y^2 + z^2/q^2.
// VJP (u = cotangent of v'):  d acc_i/dx_j = (2 g/Q) w_i w_j - g c_j delta_ij, c = (1, 1, 1/q^2);
//   d acc/dv_c = -(2 v_c/Q) w;  d acc/dq = -(2 g z^2/(q^3 Q)) w + g (0, 0, 2 z/q^3).
// ----------------------------------------------------------------------------------------------
struct FLogHalo {
  static constexpr int D = 6, M = 2;
  static constexpr double Rc2 = 0.2 * 0.2;
  template <class R> struct Theta { R vc, q, vc2, iq2; };
  template <class R> GS_HD static void load(Theta<R>& t, const R* s) {
    t.vc = s[0]; t.q = s[1];
    t.vc2 = t.vc * t.vc;
    const R iq = R(1) / t.q;
    t.iq2 = iq * iq;
  }
  template <class R> GS_HD static void f(const R* y, const Theta<R>& t, R* dy) {
    const R wz = y[2] * t.iq2;
    const R Q = R(Rc2) + y[0] * y[0] + y[1] * y[1] + y[2] * wz;
    const R g = mul_rn(t.vc2, rcp_nr(Q));  // Q >= R_c^2 > 0
    dy[0] = y[3];
    dy[1] = y[4];
    dy[2] = y[5];
    dy[3] = -g * y[0];
    dy[4] = -g * y[1];
    dy[5] = -g * wz;
  }
  template <class R>
  GS_HD static void vjp(const R* y, const Theta<R>& t, const R* kb, R* yb, R* thb) {
    const R x = y[0], yy = y[1], z = y[2];
    const R wz = z * t.iq2;
    const R iQ = rcp_nr(R(Rc2) + x * x + yy * yy + z * wz);
    const R g = t.vc2 * iQ;
    const R ux = kb[3], uy = kb[4], uz = kb[5];
    const R uw = ux * x + uy * yy + uz * wz;
    const R c2 = R(2) * g * iQ * uw;
    yb[0] = c2 * x - g * ux;
    yb[1] = c2 * yy - g * uy;
    yb[2] = c2 * wz - g * t.iq2 * uz;
    yb[3] = kb[0];
    yb[4] = kb[1];
    yb[5] = kb[2];
    thb[0] -= R(2) * t.vc * iQ * uw;
    // d/dq: z^2/q^3 = z wz / q and z/q^3 = wz / q
    const R iq = t.iq2 * t.q;
    thb[1] += R(2) * g * wz * iq * (uz - z * iQ * uw);
  }
};

}  // namespace gs
