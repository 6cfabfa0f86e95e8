// Accuracy check of the device log1p evaluation used by the fields (gs::log1p_q: fp64 by a log of
// the rounded 1 + x plus the first-order correction for its rounding error, fp32 by log1pf)
// against CUDA's own log1p and against a host reference in higher precision (long double for
// fp64 arguments, double for fp32 ones).  The reciprocal 1 / (1 + x) that log1p_q takes is formed
// here by one division, as the stellar field forms it from a quotient it needs anyway.
//
// Built and run by tests/test_gpu_log1p.py.  Prints one JSON object:
//   {"n": ..., "f64": {"field_ulp": max, "cuda_ulp": max}, "f32": {...}}
// where an "ulp" is the spacing of the format at the reference value.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <limits>
#include <vector>

#include "gs_dual.cuh"

template <class R>
__global__ void k_eval(const R* __restrict__ x, R* __restrict__ field, R* __restrict__ cuda, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    field[i] = gs::log1p_q(x[i], R(1), R(1) / (R(1) + x[i]));
    cuda[i] = log1p(x[i]);
  }
}

static bool ok(cudaError_t e, const char* what) {
  if (e != cudaSuccess) std::fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
  return e == cudaSuccess;
}

// Arguments: x = 0, every power-of-two scale from 2^-1000 (fp64) or 2^-120 (fp32) up to 2^20 with
// 64 points per octave, and negatives down to -0.75.
template <class R> static std::vector<R> arguments(int lo_exp) {
  std::vector<R> x{R(0)};
  for (int e = lo_exp; e < 20; ++e)
    for (int k = 0; k < 64; ++k) x.push_back(R(std::ldexp(1.0 + k / 64.0, e)));
  for (int k = 1; k < 4096; ++k) x.push_back(R(-0.75 * k / 4096.0));
  return x;
}

template <class R, class H> static bool run(int lo_exp, double* field_ulp, double* cuda_ulp, int* n) {
  const std::vector<R> x = arguments<R>(lo_exp);
  *n = int(x.size());
  const size_t bytes = x.size() * sizeof(R);
  R *dx = nullptr, *dk = nullptr, *dc = nullptr;
  if (!ok(cudaMalloc(&dx, bytes), "malloc") || !ok(cudaMalloc(&dk, bytes), "malloc") ||
      !ok(cudaMalloc(&dc, bytes), "malloc"))
    return false;
  if (!ok(cudaMemcpy(dx, x.data(), bytes, cudaMemcpyHostToDevice), "h2d")) return false;
  k_eval<R><<<(*n + 255) / 256, 256>>>(dx, dk, dc, *n);
  if (!ok(cudaGetLastError(), "launch") || !ok(cudaDeviceSynchronize(), "sync")) return false;
  std::vector<R> k(x.size()), c(x.size());
  if (!ok(cudaMemcpy(k.data(), dk, bytes, cudaMemcpyDeviceToHost), "d2h") ||
      !ok(cudaMemcpy(c.data(), dc, bytes, cudaMemcpyDeviceToHost), "d2h"))
    return false;
  cudaFree(dx); cudaFree(dk); cudaFree(dc);
  *field_ulp = 0;
  *cuda_ulp = 0;
  for (size_t i = 0; i < x.size(); ++i) {
    const H ref = std::log1p(H(x[i]));
    if (ref == H(0)) {
      if (k[i] != R(0) || c[i] != R(0)) { *field_ulp = 1e30; return true; }
      continue;
    }
    int ex;
    std::frexp(double(ref), &ex);
    const double ulp = std::ldexp(1.0, ex - std::numeric_limits<R>::digits);
    const double ek = double(std::fabs(H(k[i]) - ref)) / ulp;
    const double ec = double(std::fabs(H(c[i]) - ref)) / ulp;
    if (!(ek <= *field_ulp)) *field_ulp = ek;  // NaN propagates as a failure
    if (ec > *cuda_ulp) *cuda_ulp = ec;
  }
  return true;
}

int main() {
  double k64, c64, k32, c32;
  int n64, n32;
  if (!run<double, long double>(-1000, &k64, &c64, &n64)) return 1;
  if (!run<float, double>(-120, &k32, &c32, &n32)) return 1;
  std::printf("{\"n\": %d, \"f64\": {\"field_ulp\": %.4f, \"cuda_ulp\": %.4f}, "
              "\"f32\": {\"field_ulp\": %.4f, \"cuda_ulp\": %.4f}}\n",
              n64 + n32, k64, c64, k32, c32);
  return 0;
}
