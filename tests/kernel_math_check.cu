// Accuracy check of the kernels' own fp64 arithmetic helpers against long-double host references:
//  - the step controller's factor 0.9 err^(-1/Q) (gs::ctrl_factor: two Newton steps on
//    err y^Q = 1 from a float estimate, after clamping err to [1e-10, 1e10]), beside CUDA's pow,
//    and the clamp's claim: below (0.09)^Q the factor is at least 10 and above 4.5^Q at most 0.2,
//    so the controller's clamped factor is the same as with the unclamped power;
//  - the refined reciprocal and reciprocal square root (gs::rcp_nr, gs::rsqrt_nr), beside
//    CUDA's division and rsqrt, over normal positive arguments from 2^-1000 to 2^1000;
//  - the LU of a patterned iteration matrix I - c J (gs::SmallLU with HIRES's Jacobian pattern:
//    only the entries the fill-in can reach, no row exchange) against the dense one, on random
//    matrices of that pattern, half of them made to need exchanges: it reports a wanted exchange
//    exactly when the dense LU makes one, its solutions x = W^{-1} b and x = W^{-T} b are the
//    dense ones bit for bit otherwise, and a step run through gs::with_field_lu (the patterned LU,
//    the dense one when an exchange is wanted) gives the dense solution in every case;
//  - the table-driven logarithm (gs::log_tab) beside CUDA's log: positive normal arguments
//    across the whole range, densely over [1, 16] (where the stellar field evaluates it), near 1,
//    next to every breakpoint c_j +- 1/256 of the table, and the special arguments.
//
// Built and run by tests/test_gpu_kernel_math.py.  Prints one JSON object:
//   {"n": ..., "q3": {"ulp": max, "pow_ulp": max, "clamp_ok": 0|1}, "q5": ..., "q7": ...,
//    "rcp": {"ulp": max, "cuda_ulp": max}, "rsqrt": {...},
//    "n_log": ..., "log": {"ulp": max, "cuda_ulp": max, "special_ok": 0|1},
//    "lu": {"n": ..., "fallback": cases that wanted an exchange, "flag_mismatch": ...,
//           "mismatch": ..., "resid": max}}
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <vector>

#include "gs_kernels.cuh"

__global__ void k_recip(const double* __restrict__ x, double* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    out[4 * i + 0] = gs::rcp_nr(x[i]);
    out[4 * i + 1] = 1.0 / x[i];
    out[4 * i + 2] = gs::rsqrt_nr(x[i]);
    out[4 * i + 3] = rsqrt(x[i]);
  }
}

// per case: J (64), c, b (8) in; x, x_dense, xt, xt_dense, x through with_field_lu (5 x 8) and
// two flags out: the patterned LU's ok, and whether the dense LU exchanged rows
__global__ void k_lu(const double* __restrict__ in, double* __restrict__ out, int* __restrict__ fl,
                     int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const double* q = in + (size_t)i * 73;
  double J[64], b[8];
#pragma unroll
  for (int k = 0; k < 64; ++k) J[k] = q[k];
  const double c = q[64];
#pragma unroll
  for (int k = 0; k < 8; ++k) b[k] = q[65 + k];
  gs::SmallLU<double, 8, gs::JacPattern<gs::FHires>> ps;
  gs::SmallLU<double, 8> dn;
  ps.factor_shifted(J, c);
  dn.factor_shifted(J, c);
  double x1[8], x2[8], x3[8], x4[8], x5[8];
  ps.solve(b, x1);
  dn.solve(b, x2);
  ps.solve_t(b, x3);
  dn.solve_t(b, x4);
  gs::with_field_lu<gs::FHires, double>([&](auto& lu) {
    lu.factor_shifted(J, c);
    if (!lu.ok) return false;
    lu.solve(b, x5);
    return true;
  });
  double* o = out + (size_t)i * 40;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    o[k] = x1[k]; o[8 + k] = x2[k]; o[16 + k] = x3[k]; o[24 + k] = x4[k]; o[32 + k] = x5[k];
  }
  fl[2 * i] = ps.ok ? 1 : 0;
  fl[2 * i + 1] = dn.swapped ? 1 : 0;
}

__global__ void k_log(const double* __restrict__ x, double* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    out[2 * i + 0] = gs::log_tab(x[i]);
    out[2 * i + 1] = log(x[i]);
  }
}

template <int Q>
__global__ void k_eval(const double* __restrict__ x, double* __restrict__ f,
                       double* __restrict__ p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    f[i] = gs::ctrl_factor<double, Q>(x[i]);
    p[i] = 0.9 * pow(x[i], -1.0 / Q);
  }
}

static bool ok(cudaError_t e, const char* what) {
  if (e != cudaSuccess) std::fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
  return e == cudaSuccess;
}

template <int Q>
static bool run(const std::vector<double>& x, double* ulp, double* pow_ulp, int* clamp_ok) {
  const int n = int(x.size());
  const size_t bytes = x.size() * sizeof(double);
  double *dx = nullptr, *df = nullptr, *dp = nullptr;
  if (!ok(cudaMalloc(&dx, bytes), "malloc") || !ok(cudaMalloc(&df, bytes), "malloc") ||
      !ok(cudaMalloc(&dp, bytes), "malloc"))
    return false;
  if (!ok(cudaMemcpy(dx, x.data(), bytes, cudaMemcpyHostToDevice), "h2d")) return false;
  k_eval<Q><<<(n + 255) / 256, 256>>>(dx, df, dp, n);
  if (!ok(cudaGetLastError(), "launch") || !ok(cudaDeviceSynchronize(), "sync")) return false;
  std::vector<double> f(x.size()), p(x.size());
  if (!ok(cudaMemcpy(f.data(), df, bytes, cudaMemcpyDeviceToHost), "d2h") ||
      !ok(cudaMemcpy(p.data(), dp, bytes, cudaMemcpyDeviceToHost), "d2h"))
    return false;
  cudaFree(dx); cudaFree(df); cudaFree(dp);
  *ulp = 0;
  *pow_ulp = 0;
  *clamp_ok = 1;
  const long double lo = powl(0.09L, Q), hi = powl(4.5L, Q);
  for (size_t i = 0; i < x.size(); ++i) {
    const long double xi = x[i];
    if (xi < lo) { if (!(f[i] >= 10.0)) *clamp_ok = 0; continue; }
    if (xi > hi) { if (!(f[i] <= 0.2)) *clamp_ok = 0; continue; }
    const long double ref = (long double)0.9 * powl(xi, -1.0L / Q);
    int ex;
    std::frexp(double(ref), &ex);
    const double u = std::ldexp(1.0, ex - 53);
    const double e1 = double(fabsl((long double)f[i] - ref)) / u;
    const double e2 = double(fabsl((long double)p[i] - ref)) / u;
    if (!(e1 <= *ulp)) *ulp = e1;  // NaN propagates as a failure
    if (e2 > *pow_ulp) *pow_ulp = e2;
  }
  return true;
}

static bool run_recip(double* u_rcp, double* c_rcp, double* u_rs, double* c_rs, int* n_out) {
  std::vector<double> x;
  for (int e = -1000; e < 1000; ++e)
    for (int k = 0; k < 64; ++k) x.push_back(std::ldexp(1.0 + k / 64.0 + 1.0 / 4099.0, e));
  const int n = int(x.size());
  *n_out = n;
  double *dx = nullptr, *dout = nullptr;
  if (!ok(cudaMalloc(&dx, n * sizeof(double)), "malloc") ||
      !ok(cudaMalloc(&dout, 4 * n * sizeof(double)), "malloc"))
    return false;
  if (!ok(cudaMemcpy(dx, x.data(), n * sizeof(double), cudaMemcpyHostToDevice), "h2d")) return false;
  k_recip<<<(n + 255) / 256, 256>>>(dx, dout, n);
  if (!ok(cudaGetLastError(), "launch") || !ok(cudaDeviceSynchronize(), "sync")) return false;
  std::vector<double> out(4 * x.size());
  if (!ok(cudaMemcpy(out.data(), dout, 4 * n * sizeof(double), cudaMemcpyDeviceToHost), "d2h"))
    return false;
  cudaFree(dx); cudaFree(dout);
  *u_rcp = *c_rcp = *u_rs = *c_rs = 0;
  auto ulps = [](long double v, long double ref) {
    int ex;
    std::frexp(double(ref), &ex);
    return double(fabsl(v - ref)) / std::ldexp(1.0, ex - 53);
  };
  for (int i = 0; i < n; ++i) {
    const long double xi = x[i];
    const long double r1 = 1.0L / xi, r2 = 1.0L / sqrtl(xi);
    const double a = ulps(out[4 * i], r1), b = ulps(out[4 * i + 1], r1);
    const double c = ulps(out[4 * i + 2], r2), d = ulps(out[4 * i + 3], r2);
    if (!(a <= *u_rcp)) *u_rcp = a;
    if (b > *c_rcp) *c_rcp = b;
    if (!(c <= *u_rs)) *u_rs = c;
    if (d > *c_rs) *c_rs = d;
  }
  return true;
}

static bool run_log(double* u_log, double* c_log, int* special_ok, int* n_out) {
  std::vector<double> x;
  for (int e = -1022; e < 1024; ++e)
    for (int k = 0; k < 64; ++k) x.push_back(std::ldexp(1.0 + k / 64.0 + 1.0 / 7919.0, e));
  for (int k = 0; k < 400000; ++k) x.push_back(1.0 + 15.0 * k / 400000.0 + 1e-9 * (k % 7));
  for (int k = 0; k < 100000; ++k) x.push_back(1.0 + std::ldexp(1.0, -6) * k / 100000.0);
  for (int k = 0; k < 100000; ++k) x.push_back(1.0 - std::ldexp(1.0, -7) * k / 100000.0);
  for (int k = 1; k < 53; ++k) { x.push_back(1.0 + std::ldexp(1.0, -k)); x.push_back(1.0 - std::ldexp(1.0, -k - 1)); }
  for (int e = -2; e < 4; ++e)
    for (int j = 0; j < 256; ++j)
      for (int d = -4; d <= 4; ++d)
        x.push_back(std::ldexp(1.0 + (j + 0.5) / 256.0 + d * 0x1p-52, e));
  x.push_back(2.2250738585072014e-308);
  x.push_back(1.7976931348623157e308);
  const int nreg = int(x.size());
  // special arguments, checked separately: +inf, +0, -1, NaN, a subnormal
  const double specials[] = {HUGE_VAL, 0.0, -1.0, std::nan(""), 4.9e-324};
  for (double v : specials) x.push_back(v);
  const int n = int(x.size());
  *n_out = nreg;
  double *dx = nullptr, *dout = nullptr;
  if (!ok(cudaMalloc(&dx, n * sizeof(double)), "malloc") ||
      !ok(cudaMalloc(&dout, 2 * n * sizeof(double)), "malloc"))
    return false;
  if (!ok(cudaMemcpy(dx, x.data(), n * sizeof(double), cudaMemcpyHostToDevice), "h2d")) return false;
  k_log<<<(n + 255) / 256, 256>>>(dx, dout, n);
  if (!ok(cudaGetLastError(), "launch") || !ok(cudaDeviceSynchronize(), "sync")) return false;
  std::vector<double> out(2 * x.size());
  if (!ok(cudaMemcpy(out.data(), dout, 2 * n * sizeof(double), cudaMemcpyDeviceToHost), "d2h"))
    return false;
  cudaFree(dx); cudaFree(dout);
  *u_log = *c_log = 0;
  for (int i = 0; i < nreg; ++i) {
    const long double ref = logl((long double)x[i]);
    if (ref == 0) {                       // log 1 = 0 exactly
      if (out[2 * i] != 0.0) *u_log = 1e9;
      continue;
    }
    int ex;
    std::frexp(double(ref), &ex);
    const double u = std::ldexp(1.0, ex - 53);
    const double a = double(fabsl((long double)out[2 * i] - ref)) / u;
    const double b = double(fabsl((long double)out[2 * i + 1] - ref)) / u;
    if (!(a <= *u_log)) *u_log = a;       // NaN propagates as a failure
    if (b > *c_log) *c_log = b;
  }
  const double* sp = out.data() + 2 * nreg;
  *special_ok = (sp[0] == HUGE_VAL) && (sp[2] == -HUGE_VAL) && std::isnan(sp[4]) &&
                std::isnan(sp[6]) && std::isnan(sp[8]);
  return true;
}

static bool run_lu(int* n_out, int* fallback, int* flag_mismatch, int* mismatch, double* resid) {
  const int n = 20000;
  std::vector<double> in((size_t)n * 73);
  unsigned long long st = 0x9E3779B97F4A7C15ULL;
  auto uni = [&]() {  // xorshift64*, uniform in [0, 1)
    st ^= st >> 12; st ^= st << 25; st ^= st >> 27;
    return double((st * 0x2545F4914F6CDD1DULL) >> 11) * 0x1p-53;
  };
  for (int i = 0; i < n; ++i) {
    double* q = in.data() + (size_t)i * 73;
    for (int r = 0; r < 8; ++r)
      for (int k = 0; k < 8; ++k) {
        double v = 0.0;
        if (gs::FHires::jac_nz(r, k)) v = (r == k ? -1.0 : 1.0) * (0.05 + uni());
        // odd cases: a large entry below the diagonal, so that pivoting exchanges rows
        if (i % 2 == 1 && r > k && gs::FHires::jac_nz(r, k) && uni() < 0.5) v *= 40.0;
        q[r * 8 + k] = v;
      }
    // even cases: each diagonal entry outweighs the rest of its column, so that I - c J is
    // column diagonally dominant and partial pivoting exchanges nothing
    if (i % 2 == 0)
      for (int k = 0; k < 8; ++k) {
        double sum = 0.0;
        for (int r = 0; r < 8; ++r)
          if (r != k) sum += std::fabs(q[r * 8 + k]);
        q[k * 8 + k] = -(sum + 0.05 + uni());
      }
    q[64] = 0.1 + 10.0 * uni();
    for (int k = 0; k < 8; ++k) q[65 + k] = 2.0 * uni() - 1.0;
  }
  double *din = nullptr, *dout = nullptr;
  int* dfb = nullptr;
  if (!ok(cudaMalloc(&din, in.size() * sizeof(double)), "malloc") ||
      !ok(cudaMalloc(&dout, (size_t)n * 40 * sizeof(double)), "malloc") ||
      !ok(cudaMalloc(&dfb, 2 * n * sizeof(int)), "malloc"))
    return false;
  if (!ok(cudaMemcpy(din, in.data(), in.size() * sizeof(double), cudaMemcpyHostToDevice), "h2d"))
    return false;
  k_lu<<<(n + 127) / 128, 128>>>(din, dout, dfb, n);
  if (!ok(cudaGetLastError(), "launch") || !ok(cudaDeviceSynchronize(), "sync")) return false;
  std::vector<double> out((size_t)n * 40);
  std::vector<int> fb(2 * n);
  if (!ok(cudaMemcpy(out.data(), dout, out.size() * sizeof(double), cudaMemcpyDeviceToHost), "d2h") ||
      !ok(cudaMemcpy(fb.data(), dfb, 2 * n * sizeof(int), cudaMemcpyDeviceToHost), "d2h"))
    return false;
  cudaFree(din); cudaFree(dout); cudaFree(dfb);
  *n_out = n;
  *fallback = *flag_mismatch = *mismatch = 0;
  *resid = 0;
  for (int i = 0; i < n; ++i) {
    const double* q = in.data() + (size_t)i * 73;
    const double* o = out.data() + (size_t)i * 40;
    const bool pat_ok = fb[2 * i] != 0, exchanged = fb[2 * i + 1] != 0;
    *fallback += pat_ok ? 0 : 1;
    if (pat_ok == exchanged) ++*flag_mismatch;  // ok must be false exactly when pivoting exchanges
    for (int k = 0; k < 8; ++k)
      if ((pat_ok && (!(o[k] == o[8 + k]) || !(o[16 + k] == o[24 + k]))) || !(o[32 + k] == o[8 + k])) {
        ++*mismatch;
        break;
      }
    // residuals of W x = b and W^T x = b in long double, relative to |W| |x| + |b|, for the
    // solutions through with_field_lu and the dense transpose solve
    for (int t = 0; t < 2; ++t) {
      const double* x = o + (t == 0 ? 32 : 24);
      for (int r = 0; r < 8; ++r) {
        long double acc = -(long double)q[65 + r], mag = fabsl((long double)q[65 + r]);
        for (int k = 0; k < 8; ++k) {
          const double jv = t == 0 ? q[r * 8 + k] : q[k * 8 + r];
          const long double w = (r == k ? 1.0L : 0.0L) - (long double)q[64] * jv;
          acc += w * x[k];
          mag += fabsl(w * x[k]);
        }
        const double rel = double(fabsl(acc) / mag);
        if (!(rel <= *resid)) *resid = rel;
      }
    }
  }
  return true;
}

int main() {
  // err from 1e-14 to 1e14, 4096 points per decade, plus the clamp's edges
  std::vector<double> x;
  for (int i = 0; i <= 28 * 4096; ++i) x.push_back(std::pow(10.0, -14.0 + i / 4096.0));
  for (double e : {1e-10, 1e10, 0.5, 1.0, 2.0}) x.push_back(e);
  double u3, p3, u5, p5, u7, p7;
  int c3, c5, c7;
  if (!run<3>(x, &u3, &p3, &c3) || !run<5>(x, &u5, &p5, &c5) || !run<7>(x, &u7, &p7, &c7))
    return 1;
  double ur, cr, us, cs;
  int nr;
  if (!run_recip(&ur, &cr, &us, &cs, &nr)) return 1;
  double ul, cl;
  int sl, nl;
  if (!run_log(&ul, &cl, &sl, &nl)) return 1;
  int lun, lufb, lufm, lumm;
  double lures;
  if (!run_lu(&lun, &lufb, &lufm, &lumm, &lures)) return 1;
  std::printf("{\"n\": %d, \"q3\": {\"ulp\": %.4f, \"pow_ulp\": %.4f, \"clamp_ok\": %d}, "
              "\"q5\": {\"ulp\": %.4f, \"pow_ulp\": %.4f, \"clamp_ok\": %d}, "
              "\"q7\": {\"ulp\": %.4f, \"pow_ulp\": %.4f, \"clamp_ok\": %d}, "
              "\"n_recip\": %d, \"rcp\": {\"ulp\": %.4f, \"cuda_ulp\": %.4f}, "
              "\"rsqrt\": {\"ulp\": %.4f, \"cuda_ulp\": %.4f}, "
              "\"n_log\": %d, \"log\": {\"ulp\": %.4f, \"cuda_ulp\": %.4f, \"special_ok\": %d}, "
              "\"lu\": {\"n\": %d, \"fallback\": %d, \"flag_mismatch\": %d, \"mismatch\": %d, "
              "\"resid\": %.3e}}\n",
              int(x.size()), u3, p3, c3, u5, p5, c5, u7, p7, c7, nr, ur, cr, us, cs, nl, ul, cl, sl,
              lun, lufb, lufm, lumm, lures);
  return 0;
}
