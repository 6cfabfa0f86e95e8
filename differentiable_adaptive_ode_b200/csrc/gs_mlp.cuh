// gs_mlp.cuh -- the neural right-hand side f(y) = W3 tanh(W2 tanh(W1 y + b1) + b2) + b3
// (4 -> 32 -> 32 -> 4, theta shared by the ensemble): forward, record, replay and replay-adjoint
// kernels with ONE WARP PER TRAJECTORY.
//
// Layout of theta (row-major W[out][in]): W1 at 0 (32x4), b1 at 128, W2 at 160 (32x32),
// b2 at 1184, W3 at 1216 (4x32), b3 at 1344; 1348 values.
//
// Lane i of a warp owns hidden unit i of both layers: row i of W1, W2 (and column i of W2 for the
// transposed product of the backward pass), column i of W3, and the matching rows/columns of the
// weight cotangent -- all in registers.  The trajectory's state and stages are replicated in all
// lanes (identical arithmetic, identical accept decisions), so the adaptive loop has no intra-warp
// divergence.  A hidden vector is broadcast through a 32-float shared-memory slot per warp; the
// four output sums are butterfly reductions.  The weight cotangent of a stage is the outer product
// z2b h1^T summed over everything the warp integrates; each warp keeps its partial sum in
// registers and the partials are reduced over warps in a fixed order at the end.
//
// Method: "gradsolve: fast exact gradients for ODE ensembles on GPUs" §2.2 (a neural right-hand
// side with thousands of weights: reverse mode is the only practical route), §3 (record, replay,
// discrete adjoint with the mesh held fixed).
#pragma once
#include "gs_kernels.cuh"

namespace gs {

constexpr int MLP_H = 32, MLP_D = 4, MLP_M = 1348;
static_assert(MLP_D == 4, "warp_sum4 reduces the four outputs of the field");
constexpr int MLP_OW1 = 0, MLP_OB1 = 128, MLP_OW2 = 160, MLP_OB2 = 1184, MLP_OW3 = 1216,
              MLP_OB3 = 1344;

template <class R>
struct MlpLane {
  R w1[MLP_D];   // W1[i][:]
  R b1;
  R w2r[MLP_H];  // W2[i][:]
  R w2c[MLP_H];  // W2[:][i]
  R b2;
  R w3c[MLP_D];  // W3[:][i]
  R b3[MLP_D];
  R* bcast;      // this warp's 32-slot shared-memory broadcast buffer

  __device__ void load(const R* th, R* warp_slot) {
    const int i = threadIdx.x & 31;
#pragma unroll
    for (int c = 0; c < MLP_D; ++c) w1[c] = th[MLP_OW1 + i * MLP_D + c];
    b1 = th[MLP_OB1 + i];
#pragma unroll
    for (int j = 0; j < MLP_H; ++j) {
      w2r[j] = th[MLP_OW2 + i * MLP_H + j];
      w2c[j] = th[MLP_OW2 + j * MLP_H + i];
    }
    b2 = th[MLP_OB2 + i];
#pragma unroll
    for (int o = 0; o < MLP_D; ++o) {
      w3c[o] = th[MLP_OW3 + o * MLP_H + i];
      b3[o] = th[MLP_OB3 + o];
    }
    bcast = warp_slot;
  }
};

// The four sums over the warp of four per-lane values, every lane receiving all four.  A
// reduce-scatter butterfly: over the first two exchanges (lane distance 16, then 8) the lanes
// split the four sums between them, each lane keeping one and passing the others on; the last
// three exchanges (4, 2, 1) finish the sum each lane kept; then each sum is broadcast from a lane
// that holds it (lanes 0, 8, 16, 24 hold sums 0, 1, 2, 3).  10 shuffles, where four separate
// butterflies with broadcasts take 24.  Addition being commutative, every lane that finishes a
// sum holds the same bits, and the broadcast gives every lane the same value, so the state that
// the lanes replicate cannot drift between them.
template <class R>
__device__ __forceinline__ void warp_sum4(const R (&v)[4], R (&sum)[4]) {
  const int lane = threadIdx.x & 31;
  const bool up16 = lane & 16, up8 = lane & 8;
  // distance 16: the lower half keeps sums 0 and 1, the upper half sums 2 and 3
  R a0 = up16 ? v[2] : v[0], a1 = up16 ? v[3] : v[1];
  const R s0 = up16 ? v[0] : v[2], s1 = up16 ? v[1] : v[3];
  a0 += __shfl_xor_sync(FULL, s0, 16);
  a1 += __shfl_xor_sync(FULL, s1, 16);
  // distance 8: of its two, a lane keeps the first if bit 3 of its index is clear
  R k = up8 ? a1 : a0;
  k += __shfl_xor_sync(FULL, up8 ? a0 : a1, 8);
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) k += __shfl_xor_sync(FULL, k, o);
#pragma unroll
  for (int c = 0; c < 4; ++c) sum[c] = __shfl_sync(FULL, k, 8 * c);
}

// Broadcast the 32 lane values v through shared memory; out[j] = v of lane j.  The slot is
// 16-byte aligned and read back as 16-byte vectors (every lane reads the same words: a broadcast).
template <class R>
__device__ __forceinline__ void warp_gather(R* slot, R v, R (&out)[MLP_H]) {
  const int i = threadIdx.x & 31;
  __syncwarp();
  slot[i] = v;
  __syncwarp();
  if constexpr (sizeof(R) == 4) {
    const float4* s4 = reinterpret_cast<const float4*>(slot);
#pragma unroll
    for (int q = 0; q < MLP_H / 4; ++q) {
      const float4 t = s4[q];
      out[4 * q] = t.x;
      out[4 * q + 1] = t.y;
      out[4 * q + 2] = t.z;
      out[4 * q + 3] = t.w;
    }
  } else {
    const double2* s2 = reinterpret_cast<const double2*>(slot);
#pragma unroll
    for (int q = 0; q < MLP_H / 2; ++q) {
      const double2 t = s2[q];
      out[2 * q] = t.x;
      out[2 * q + 1] = t.y;
    }
  }
}

template <class R> __device__ __forceinline__ R tanh_r(R x);
template <> __device__ __forceinline__ double tanh_r<double>(double x) { return tanh(x); }
template <> __device__ __forceinline__ float tanh_r<float>(float x) { return tanhf(x); }

// Warp-cooperative f: y replicated in every lane; returns dy replicated; h1, h2 = this lane's
// hidden activations.
template <class R>
__device__ __forceinline__ void mlp_f(const MlpLane<R>& W, const R (&y)[MLP_D], R (&dy)[MLP_D],
                                      R& h1, R& h2) {
  R z1 = W.b1;
#pragma unroll
  for (int c = 0; c < MLP_D; ++c) z1 += W.w1[c] * y[c];
  h1 = tanh_r<R>(z1);
  R hv[MLP_H];
  warp_gather(W.bcast, h1, hv);
  R z2 = W.b2;
#pragma unroll
  for (int j = 0; j < MLP_H; ++j) z2 += W.w2r[j] * hv[j];
  h2 = tanh_r<R>(z2);
  R part[MLP_D], sum[MLP_D];
#pragma unroll
  for (int o = 0; o < MLP_D; ++o) part[o] = W.w3c[o] * h2;
  warp_sum4<R>(part, sum);
#pragma unroll
  for (int o = 0; o < MLP_D; ++o) dy[o] = W.b3[o] + sum[o];
}

// Field adaptor so that the generic Tsit5 trial step can drive the warp-cooperative f.
struct FMlpWarp {
  static constexpr int D = MLP_D, M = MLP_M;
  template <class R> using Theta = MlpLane<R>;
  template <class R> __device__ static void f(const R* y, const MlpLane<R>& W, R* dy) {
    R yy[MLP_D], d[MLP_D], h1, h2;
#pragma unroll
    for (int c = 0; c < MLP_D; ++c) yy[c] = y[c];
    mlp_f<R>(W, yy, d, h1, h2);
#pragma unroll
    for (int c = 0; c < MLP_D; ++c) dy[c] = d[c];
  }
};

// Per-lane share of the warp's weight cotangent (lane i: row i of W1b, W2b; b1b_i, b2b_i;
// column i of W3b; b3b in every lane).
template <class R>
struct MlpBar {
  R w1[MLP_D], b1, w2[MLP_H], b2, w3[MLP_D], b3[MLP_D];
  __device__ void zero() {
#pragma unroll
    for (int c = 0; c < MLP_D; ++c) { w1[c] = R(0); w3[c] = R(0); b3[c] = R(0); }
#pragma unroll
    for (int j = 0; j < MLP_H; ++j) w2[j] = R(0);
    b1 = R(0);
    b2 = R(0);
  }
  // write this warp's partial (M values) to out
  __device__ void store(R* out) const {
    const int i = threadIdx.x & 31;
#pragma unroll
    for (int c = 0; c < MLP_D; ++c) out[MLP_OW1 + i * MLP_D + c] = w1[c];
    out[MLP_OB1 + i] = b1;
#pragma unroll
    for (int j = 0; j < MLP_H; ++j) out[MLP_OW2 + i * MLP_H + j] = w2[j];
    out[MLP_OB2 + i] = b2;
#pragma unroll
    for (int o = 0; o < MLP_D; ++o) out[MLP_OW3 + o * MLP_H + i] = w3[o];
    if (i < MLP_D) out[MLP_OB3 + i] = b3[i];
  }
};

// Reverse-mode Tsit5 replay step for the MLP field (same sweep as tsit5_adjoint_step; the VJP is
// written out for the two tanh layers).  Every lane of the warp executes it; a lane's theta-bar
// share accumulates the weight cotangent.  `active` = false contributes nothing (idle warp).
template <class R>
__device__ __forceinline__ void mlp_adjoint_step(const MlpLane<R>& W, const R (&y)[MLP_D], R h,
                                                 R (&lam)[MLP_D], MlpBar<R>& tb_) {
  constexpr int D = MLP_D;
  R Y[6][D], H1[6], H2[6];
  {
    R k[5][D];
#pragma unroll
    for (int c = 0; c < D; ++c) Y[0][c] = y[c];
    mlp_f<R>(W, Y[0], k[0], H1[0], H2[0]);
#pragma unroll
    for (int i = 1; i < 6; ++i) {
#pragma unroll
      for (int c = 0; c < D; ++c) {
        R s = ta<R>(i, 0) * k[0][c];
#pragma unroll
        for (int j = 1; j < i; ++j) s += ta<R>(i, j) * k[j][c];
        Y[i][c] = y[c] + h * s;
      }
      R dummy[D];
      if (i < 5) mlp_f<R>(W, Y[i], k[i], H1[i], H2[i]);
      else mlp_f<R>(W, Y[i], dummy, H1[i], H2[i]);
    }
  }
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
    // output layer: dy = W3 h2 + b3
    R h2b = R(0);
#pragma unroll
    for (int o = 0; o < D; ++o) {
      h2b += W.w3c[o] * kb[o];
      tb_.w3[o] += kb[o] * H2[i];
      tb_.b3[o] += kb[o];
    }
    const R z2b = h2b * (R(1) - H2[i] * H2[i]);
    tb_.b2 += z2b;
    // W2b[i][:] += z2b h1^T  and  h1b_j = sum_i W2[i][j] z2b_i
    R hv[MLP_H];
    warp_gather(W.bcast, H1[i], hv);
#pragma unroll
    for (int j = 0; j < MLP_H; ++j) tb_.w2[j] += z2b * hv[j];
    R zv[MLP_H];
    warp_gather(W.bcast, z2b, zv);
    R h1b = R(0);
#pragma unroll
    for (int j = 0; j < MLP_H; ++j) h1b += W.w2c[j] * zv[j];
    const R z1b = h1b * (R(1) - H1[i] * H1[i]);
    tb_.b1 += z1b;
    R part[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
      tb_.w1[c] += z1b * Y[i][c];
      part[c] = W.w1[c] * z1b;
    }
    warp_sum4<R>(part, Yb[i]);
#pragma unroll
    for (int c = 0; c < D; ++c) lnew[c] += Yb[i][c];
  }
#pragma unroll
  for (int c = 0; c < D; ++c) lam[c] = lnew[c];
}

// ------------------------------------------------------------------------------------------------
// Forward / record: one warp per trajectory, work taken from a global counter by lane 0.
// The record is written straight into the chunk pool (C steps of E = 2 + 4 reals per chunk);
// lane 0 allocates a chunk every C accepted steps.
// ------------------------------------------------------------------------------------------------
template <class R>
struct MlpLayout {
  static constexpr int E = 2 + MLP_D;
  static constexpr int C = RecLayout<FMlpWarp, R>::C;
};

// fp32: 5 blocks/SM (96 registers, 32-64 B of spills) against 4 (119, none): record kernel 0.1065 ->
// 0.1024 ms, forward-only 0.1030 -> 0.0985 ms on the 16,384-trajectory ensemble (more warps to
// hide the shuffles); fp64 at 5 blocks spills 848 B and keeps its unconstrained allocation.
template <class R, bool REC>
__global__ void __launch_bounds__(128, sizeof(R) == 4 ? 5 : 1) k_solve_mlp(SolveParams<R> p) {
  using L = MlpLayout<R>;
  constexpr int D = MLP_D;
  __shared__ __align__(16) R slots[4][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  MlpLane<R> W;
  W.load(p.theta, slots[warp]);
  const R expo = R(-1.0 / double(Tsit5::err_order));
  const R eps = eps_of<R>();
  const R span = fabs(p.t1 - p.t0);
  constexpr int PARKED = -2;
  for (;;) {
    int q = 0;
    if (lane == 0) q = atomicAdd(p.queue, 1);
    q = __shfl_sync(FULL, q, 0);
    if (q >= p.nqueue) break;
    const int k = p.order ? p.order[q] : q;
    if (k < 0 || k >= p.N) continue;   // an order entry outside the ensemble is skipped
    R y[D], k1[D];
    R t = p.t0, h = R(0);
    int S = 0, Rj = 0, seq = 0, slot = 0, chunk = -1, st = -1;
    long long att = 0;
    bool last_rej = false;
    if (REC && p.resume) {
      // a parked trajectory continues from its parked state (start-up already done)
      const R* pr = p.park_r + (size_t)k * (2 + 2 * D);
      t = pr[0];
      h = pr[1];
#pragma unroll
      for (int c = 0; c < D; ++c) { y[c] = pr[2 + c]; k1[c] = pr[2 + D + c]; }
      const int* pi = p.park_i + (size_t)k * 4;
      S = pi[0]; Rj = pi[1]; seq = pi[2]; last_rej = pi[3] != 0;
      att = p.park_att[k];
    } else {
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = p.y0[(size_t)k * D + c];
      if (!(p.t1 > p.t0)) {
        st = 0;
      } else {
        FMlpWarp::f<R>(y, W, k1);
        bool finite = true;
#pragma unroll
        for (int c = 0; c < D; ++c) finite = finite && isfinite(y[c]) && isfinite(k1[c]);
        if (!finite) st = 3;
        else h = initial_step<FMlpWarp, R>(y, k1, W, p.t0, p.t1, p.rtol, p.atol, Tsit5::order);
      }
    }
    while (st < 0) {
      if (att >= p.max_attempts) { st = 1; break; }
      if (!(h >= R(16) * eps * fmax(fabs(t), span))) { st = 2; break; }
      if (REC && chunk < 0) {
        // the chunk for the next accepted steps is taken before the attempt; when the pool is
        // exhausted the trajectory is parked here, every accepted step so far written
        int ch = 0;
        if (lane == 0) ch = atomicAdd(p.chunk_count, 1);
        ch = __shfl_sync(FULL, ch, 0);
        if (ch < p.pool_chunks) {
          chunk = ch;
          if (lane == 0) { p.chunk_traj[chunk] = k; p.chunk_seq[chunk] = seq; }
          ++seq;
        } else {
          if (lane == 0) {
            const int at = atomicAdd(p.park_count, 1);
            p.park_list[at] = k;
            R* pr = p.park_r + (size_t)k * (2 + 2 * D);
            pr[0] = t;
            pr[1] = h;
#pragma unroll
            for (int c = 0; c < D; ++c) { pr[2 + c] = y[c]; pr[2 + D + c] = k1[c]; }
            int* pi = p.park_i + (size_t)k * 4;
            pi[0] = S; pi[1] = Rj; pi[2] = seq; pi[3] = last_rej ? 1 : 0;
            p.park_att[k] = att;
          }
          st = PARKED;
          break;
        }
      }
      bool clipped = false;
      if (t + h > p.t1) { h = p.t1 - t; clipped = true; }
      ++att;
      R ynew[D], k7[D];
      const R err = tsit5_trial<FMlpWarp, R>(y, h, W, k1, ynew, k7, p.rtol, p.atol);
      if (err <= R(1)) {
        if (REC) {
          R* e = p.pool + ((size_t)chunk * L::C + slot) * L::E;
          R v = (lane == 0) ? t : h;
#pragma unroll
          for (int c = 0; c < D; ++c) v = (lane == 2 + c) ? y[c] : v;
          if (lane < L::E) e[lane] = v;
          slot = (slot + 1 == L::C) ? 0 : slot + 1;
          if (slot == 0) chunk = -1;
        }
        ++S;
        const R facmax = last_rej ? R(1) : R(10);
        R fac = (err == R(0)) ? facmax : R(0.9) * pw<R>(err, expo);
        fac = fmin(facmax, fmax(R(0.2), fac));
        t = (clipped || t + h >= p.t1) ? p.t1 : t + h;
#pragma unroll
        for (int c = 0; c < D; ++c) { y[c] = ynew[c]; k1[c] = k7[c]; }
        h = h * fac;
        last_rej = false;
        if (t == p.t1) st = 0;
      } else {
        ++Rj;
        R fac = isfinite(err) ? R(0.9) * pw<R>(err, expo) : R(0.2);
        fac = fmin(R(10), fmax(R(0.2), fac));
        h = h * fac;
        last_rej = true;
      }
    }
    if (st == PARKED) continue;
    // a chunk taken for an attempt that was never accepted is marked unused
    if (REC && chunk >= 0 && slot == 0 && lane == 0) p.chunk_traj[chunk] = -1;
    if (lane < D) p.y1[(size_t)k * D + lane] = y[lane];
    if (lane == 0) {
      if (p.nsteps) p.nsteps[k] = S;
      if (p.nrejected) p.nrejected[k] = Rj;
      if (p.status) p.status[k] = st;
    }
  }
}

// One Tsit5 step of the replay map for the MLP field: every lane of the warp, y replicated.
template <class R>
__device__ __forceinline__ void mlp_replay_step(const MlpLane<R>& W, const R (&y)[MLP_D], R h,
                                                R (&ynew)[MLP_D]) {
  constexpr int D = MLP_D;
  R kk[6][D], Y[D];
  FMlpWarp::f<R>(y, W, kk[0]);
#pragma unroll
  for (int i = 1; i < 6; ++i) {
#pragma unroll
    for (int c = 0; c < D; ++c) {
      R s = ta<R>(i, 0) * kk[0][c];
#pragma unroll
      for (int j = 1; j < i; ++j) s += ta<R>(i, j) * kk[j][c];
      Y[c] = y[c] + h * s;
    }
    FMlpWarp::f<R>(Y, W, kk[i]);
  }
#pragma unroll
  for (int c = 0; c < D; ++c) {
    R s = tb<R>(0) * kk[0][c];
#pragma unroll
    for (int j = 1; j < 6; ++j) s += tb<R>(j) * kk[j][c];
    ynew[c] = y[c] + h * s;
  }
}

// Lane c (< D) writes component c of a vector that every lane holds.
template <class R>
__device__ __forceinline__ void mlp_lane_store(R* out, const R (&v)[MLP_D]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < MLP_D; ++c)
    if (lane == c) out[c] = v[c];
}

// Forward replay over the recorded mesh (rewrites the stored y_n), one warp per trajectory.
template <class R>
__global__ void __launch_bounds__(128) k_replay_forward_mlp(ReplayParams<R> p) {
  using L = MlpLayout<R>;
  constexpr int D = MLP_D;
  __shared__ __align__(16) R slots[4][32];
  if (p.gate && *p.gate == 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  MlpLane<R> W;
  W.load(p.theta, slots[warp]);
  for (;;) {
    int id = 0;
    if (lane == 0) id = atomicAdd(p.queue, 1);
    id = __shfl_sync(FULL, id, 0);
    if (id >= p.N) break;
    const int k = p.perm ? p.perm[id] : id;
    const int S = p.nsteps[k];
    const long long cbase = p.choff[k];
    R y[D];
    if (p.y0) {
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = p.y0[(size_t)k * D + c];
    } else {
      if (S == 0) continue;  // nothing stored and nothing to rewrite
      const R* e0 = chunk_entry<L>(p.pool, chunk_at(p.chunk_table, cbase, p.bounds), 0, p.bounds);
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = e0[2 + c];
    }
    for (int n = 0; n < S; ++n) {
      R* e = chunk_entry<L>(p.pool, chunk_at(p.chunk_table, cbase + n / L::C, p.bounds), n,
                            p.bounds);
      const R h = e[1];
      __syncwarp();
      if (lane < D) e[2 + lane] = y[lane];
      R ynew[D];
      mlp_replay_step<R>(W, y, h, ynew);
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = ynew[c];
    }
    if (p.y1 && lane < D) p.y1[(size_t)k * D + lane] = y[lane];
  }
}

// Replay adjoint: warp w visits the trajectories perm[w], perm[w + nwarps], ... (longest records
// first, dealt round-robin: a fixed assignment, so every warp partial -- and the ensemble sum made
// from the partials in warp order -- is bitwise reproducible).
template <class R>
struct MlpAdjParams {
  int N;
  const R* theta;
  const R* dL_dy1;
  R* dL_dy0;          // nullable
  R* partials;        // [nwarps][M] or nullptr
  const int* nsteps;
  const long long* choff;
  const int* chunk_table;
  const R* pool;
  const int* perm;
  RecBounds bounds;
};

template <class R>
__global__ void __launch_bounds__(128) k_adjoint_mlp(MlpAdjParams<R> p) {
  using L = MlpLayout<R>;
  constexpr int D = MLP_D;
  __shared__ __align__(16) R slots[4][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gw = blockIdx.x * 4 + warp;
  const int nwarps = gridDim.x * 4;
  MlpLane<R> W;
  W.load(p.theta, slots[warp]);
  MlpBar<R> bar;
  bar.zero();
  for (int id = gw; id < p.N; id += nwarps) {
    const int k = p.perm ? p.perm[id] : id;
    R lam[D];
#pragma unroll
    for (int c = 0; c < D; ++c) lam[c] = p.dL_dy1[(size_t)k * D + c];
    const long long cbase = p.choff[k];
    for (int n = p.nsteps[k] - 1; n >= 0; --n) {
      const R* e = chunk_entry<L>(p.pool, chunk_at(p.chunk_table, cbase + n / L::C, p.bounds),
                                  n, p.bounds);
      const R h = e[1];
      R y[D];
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = e[2 + c];
      mlp_adjoint_step<R>(W, y, h, lam, bar);
    }
    if (p.dL_dy0 && lane < D) p.dL_dy0[(size_t)k * D + lane] = lam[lane];
  }
  if (p.partials) bar.store(p.partials + (size_t)gw * MLP_M);
}

// ------------------------------------------------------------------------------------------------
// Outputs at requested times and their gradient ("gradsolve: fast exact gradients for ODE
// ensembles on GPUs" §3.4: one extra solver step from the preceding mesh point exactly to each
// requested time), one warp per trajectory.  The rule is the other fields' (k_replay_outputs,
// k_adjoint_outputs): output j < jS is one step of size tau_j - t_n from the recorded y_n of its
// step n (output_step), the rest are the final state, and y0 when nothing is recorded.  Warp w
// takes trajectories w, w + nwarps, ...; every lane takes the same search and steps, so the warp
// stays converged for the field's shuffles.
// ------------------------------------------------------------------------------------------------
template <class R>
__global__ void __launch_bounds__(128) k_replay_outputs_mlp(OutParams<R> q) {
  constexpr int D = MLP_D;
  __shared__ __align__(16) R slots[4][32];
  const ReplayParams<R>& p = q.rp;
  const int warp = threadIdx.x >> 5;
  const int J = q.ot.J, jS = q.jS;
  MlpLane<R> W;
  W.load(p.theta, slots[warp]);
  for (int k = blockIdx.x * 4 + warp; k < p.N; k += gridDim.x * 4) {
    const int S = p.nsteps[k];
    R* out = q.y_out + (size_t)k * J * D;
    if (S == 0) {
      R y[D];
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = p.y0[(size_t)k * D + c];
      for (int j = 0; j < J; ++j) mlp_lane_store<R>(out + (size_t)j * D, y);
      continue;
    }
    const long long cbase = p.choff[k];
    int n = 0;
    for (int j = 0; j < jS; ++j) {
      const R tau = q.ot.tau[j];
      n = output_step<FMlpWarp, R>(p, cbase, n, S, tau);
      const R* e = rec_entry<FMlpWarp, R>(p, cbase, n);
      R y[D], yo[D];
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = e[2 + c];
      mlp_replay_step<R>(W, y, tau - e[0], yo);
      mlp_lane_store<R>(out + (size_t)j * D, yo);
    }
    if (jS < J) {
      const R* e = rec_entry<FMlpWarp, R>(p, cbase, S - 1);
      R y[D], yS[D];
#pragma unroll
      for (int c = 0; c < D; ++c) y[c] = e[2 + c];
      mlp_replay_step<R>(W, y, e[1], yS);
      for (int j = jS; j < J; ++j) mlp_lane_store<R>(out + (size_t)j * D, yS);
    }
  }
}

template <class R>
struct MlpOutAdjParams {
  MlpAdjParams<R> ap;   // dL_dy1 may be null here
  const R* dL_dyout;    // [N][J][D]
  OutTimes<R> ot;
  int jS;               // outputs 0 .. jS - 1 are before t1
};

// Gradient: k_adjoint_mlp's walk from dL/dy1 plus the cotangents of the outputs at or after t1;
// after the pullback of a step that holds outputs, each of them is pulled back through its extra
// step from the same y_n and added.  A warp works on one trajectory, so the extra pullbacks leave
// no lane idle.
template <class R>
__global__ void __launch_bounds__(128) k_adjoint_outputs_mlp(MlpOutAdjParams<R> q) {
  constexpr int D = MLP_D;
  __shared__ __align__(16) R slots[4][32];
  const MlpAdjParams<R>& p = q.ap;
  const int warp = threadIdx.x >> 5;
  const int gw = blockIdx.x * 4 + warp;
  const int nwarps = gridDim.x * 4;
  const int J = q.ot.J, jS = q.jS;
  MlpLane<R> W;
  W.load(p.theta, slots[warp]);
  MlpBar<R> bar;
  bar.zero();
  for (int id = gw; id < p.N; id += nwarps) {
    const int k = p.perm ? p.perm[id] : id;
    const int S = p.nsteps[k];
    const R* lo = q.dL_dyout + (size_t)k * J * D;
    R lam[D];
#pragma unroll
    for (int c = 0; c < D; ++c) lam[c] = p.dL_dy1 ? p.dL_dy1[(size_t)k * D + c] : R(0);
    int jcur = S == 0 ? 0 : jS;
    for (int jj = jcur; jj < J; ++jj)
#pragma unroll
      for (int c = 0; c < D; ++c) lam[c] += lo[(size_t)jj * D + c];
    const long long cbase = p.choff[k];
    // one adjoint step per pass: step n itself, or (r >= jlo) the extra step of output r from the
    // same y_n; one call site keeps one copy of the step in the kernel
    int n = S - 1, r = -1, jlo = jcur;
    while (n >= 0) {
      const R* e = rec_entry<FMlpWarp, R>(p, cbase, n);
      const R t = e[0];
      const bool out = r >= 0;
      R y[D], v[D];
#pragma unroll
      for (int c = 0; c < D; ++c) {
        y[c] = e[2 + c];
        v[c] = out ? lo[(size_t)r * D + c] : lam[c];
      }
      mlp_adjoint_step<R>(W, y, out ? q.ot.tau[r] - t : e[1], v, bar);
      if (out) {
#pragma unroll
        for (int c = 0; c < D; ++c) lam[c] += v[c];
        if (--r < jlo) {  // the step's outputs are taken: on to step n - 1
          jcur = jlo;
          r = -1;
          --n;
        }
      } else {
#pragma unroll
        for (int c = 0; c < D; ++c) lam[c] = v[c];
        jlo = jcur;
        while (jlo > 0 && (n == 0 || q.ot.tau[jlo - 1] >= t)) --jlo;
        if (jlo < jcur) r = jcur - 1;
        else --n;
      }
    }
    if (p.dL_dy0) mlp_lane_store<R>(p.dL_dy0 + (size_t)k * D, lam);
  }
  if (p.partials) bar.store(p.partials + (size_t)gw * MLP_M);
}

}  // namespace gs
