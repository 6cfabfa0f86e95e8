// gs_kernels.cuh -- the ensemble kernels.
//
//  k_solve<F,R,Method,REC>   one trajectory per lane, state in registers; persistent grid whose
//                            warps refill retired lanes from a global work counter (one ballot +
//                            one atomicAdd per warp per refill).  REC = true also keeps the record:
//                            each accepted step (t_n, h_n, y_n) is staged in shared memory and a
//                            full chunk of C steps is written by the whole warp as one contiguous,
//                            coalesced block of the record pool.
//  k_adjoint<F,R,Method>     the replay-adjoint: each lane walks its trajectory's record from the
//                            last accepted step back to the first, recomputes the stages from the
//                            recorded y_n, and pulls lambda and theta-bar back through each step.
//  k_scan_*, k_chunk_table   record finalisation: prefix offsets and the per-trajectory chunk table.
//  k_reduce_theta            deterministic ensemble sum of theta-bar for a shared theta.
//
// Source of the method: "gradsolve: fast exact gradients for ODE ensembles on GPUs" -- §2.1
// (adaptive loop, RMS test, reject-and-retry), §2.4 (one thread per trajectory with its state
// in registers), §3 (record of accepted steps; replay with the mesh as data; exact reverse-mode
// derivative of the replay), §3.3 (the adjoint keeps one accepted state per step and recomputes
// the stages from it).
#pragma once
#include <cstdint>
#include <type_traits>

#include "gs_methods.cuh"

namespace gs {

constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------------------------------------
// Bounds of a record's device arrays, for the checked build (-DGS_CHECKED): every access through
// the chunk table is checked against the allocated sizes; an out-of-range index is counted in
// g_gs_violations and the access is redirected to a small scratch entry, so the kernel stays in
// bounds and finishes (the result is then wrong and the count says so).  The normal build
// compiles the checks away.
// ---------------------------------------------------------------------------------------------
struct RecBounds {
  long long table_cap;   // entries allocated for the chunk table
  long long pool_chunks; // chunks allocated in the pool
};
#ifdef GS_CHECKED
__device__ unsigned long long g_gs_violations;
__device__ __align__(16) double g_gs_scratch_entry[64];  // 16-byte loads and stores of entries
__device__ __forceinline__ void gs_violation() { atomicAdd(&g_gs_violations, 1ull); }
#endif

// Chunk id at chunk-table position ti (checked build: -1 when ti is outside the table).
__device__ __forceinline__ int chunk_at(const int* table, long long ti, const RecBounds& b) {
#ifdef GS_CHECKED
  if (ti < 0 || ti >= b.table_cap) {
    gs_violation();
    return -1;
  }
#endif
  return __ldg(table + ti);
}
// Entry of step n (slot n % C) in chunk ch (checked build: the scratch entry when ch is not a
// chunk of the pool).
template <class L, class R>
__device__ __forceinline__ R* chunk_entry(R* pool, int ch, int n, const RecBounds& b) {
#ifdef GS_CHECKED
  if (ch < 0 || ch >= b.pool_chunks) {
    gs_violation();
    return reinterpret_cast<R*>(g_gs_scratch_entry);
  }
#endif
  return pool + ((size_t)ch * L::C + (n % L::C)) * L::E;
}

// Record writes, two forms.  Direct: each accepted step's entry goes straight from the lane's
// registers into its current chunk (taken from the warp's block before the attempt), with no
// staging and no flush.  Staged: the entry is staged in shared memory and a full chunk is
// copied out by the whole warp as one coalesced block.  Measured on B200 at 2^20 trajectories
// (record call): the stellar field, whose step is long, 24.8 -> 22.1 ms direct (fp32 3.21 ->
// 2.89); Lorenz-63, whose step is short and whose record rate is high, 5.44 staged against 6.13
// direct.  Fields with long steps take the direct form.
template <class F, class R> struct RecDirect { static constexpr bool value = false; };
template <class R> struct RecDirect<FNfwMiyamotoNagai, R> { static constexpr bool value = true; };
template <class R> struct RecDirect<FHires, R> { static constexpr bool value = true; };

// Record chunk: C accepted steps of one trajectory, entry = (t, h, y[0..D-1]) contiguous: 8 steps
// for entries under 48 bytes, and for direct fields while the chunk stays within 512 bytes (no
// shared-memory stage to hold it; half the chunks to hand out, label and list in the chunk table
// and half the chunk changes of the replay kernels: the stellar step 24.33 -> 24.12 ms at 2^20);
// 4 otherwise (HIRES's 80-byte entries: 8 measured slower in its record kernel, 8.45 -> 8.79 ms).
template <class F, class R>
struct RecLayout {
  static constexpr int E = 2 + F::D;                                     // reals per step
  static constexpr int C = (E * int(sizeof(R)) < 48 ||
                            (RecDirect<F, R>::value && 8 * E * int(sizeof(R)) <= 512))
                               ? 8
                               : 4;                                      // steps per chunk
  static constexpr int STAGE_STRIDE = C * E + 1;                         // per-lane smem stride
};

template <class R>
struct SolveParams {
  int N;
  const R* theta;
  int theta_stride;  // 0 when theta is shared by the ensemble
  const R* y0;
  R t0, t1, rtol, atol;
  long long max_attempts;
  R* y1;
  int* nsteps;
  int* nrejected;
  int* status;
  int* queue;        // work counter
  const int* order;  // trajectory visited at queue position q (null: q itself)
  int nqueue;        // queue positions to visit: N, or the number of parked trajectories resumed
  // record (REC only)
  R* pool;
  int* chunk_traj;
  int* chunk_seq;
  int pool_chunks;   // capacity in chunks
  int* chunk_count;  // bump allocator
  // Trajectories that found the pool exhausted are parked before their next attempt, with every
  // accepted step so far written: their ids go to park_list (park_count of them) and their state
  // to the per-trajectory park arrays.  A pass with resume = 1 visits park_list entries (order)
  // and continues each from its parked state instead of starting it.
  int* park_count;
  int* park_list;      // [N]
  R* park_r;           // [N][2 + 2D]: t, h, y, the slope f(y) carried into the next attempt
  int* park_i;         // [N][4]: accepted steps, rejected trials, next chunk sequence, last rejected
  long long* park_att; // [N] attempts so far
  int resume;
  // > 0: a trajectory that has made this many attempts in the pass is parked at its next chunk
  // boundary (a first slice of every trajectory, whose progress orders the rest of the record)
  int slice;
  // forward sensitivities (SENS only): S = dy/dtheta, [N][D][M]; sens0 may be null (zero start)
  const R* sens0;
  R* sens1;
};

template <class R> __device__ __forceinline__ R pw(R x, R e);
template <> __device__ __forceinline__ double pw<double>(double x, double e) { return pow(x, e); }
template <> __device__ __forceinline__ float pw<float>(float x, float e) { return powf(x, e); }
// y^Q for a small positive integer Q, by repeated multiplication
template <int Q>
__device__ __forceinline__ double ipow(double y) {
  if constexpr (Q == 1) return y;
  else if constexpr (Q % 2 == 0) { const double h = ipow<Q / 2>(y); return h * h; }
  else return ipow<Q - 1>(y) * y;
}

// The step controller's factor 0.9 err^(-1/Q), which the controller clamps to [0.2, 10] (or to
// [0.2, 1] right after a reject): only err within [(0.09)^Q, 4.5^Q] -- inside [1e-10, 1e10] for
// Q <= 7 -- reaches the clamp's interior, so err is clamped to [1e-10, 1e10] first, which leaves
// every clamped factor as it was (non-finite and zero err never use this value).  fp64: Newton's
// iteration on g(y) = err y^Q - 1, y <- y + (y / Q)(1 - err y^Q), from a float estimate good to
// ~1e-7; quadratic convergence takes two steps below the double rounding, so the factor is within
// about an ulp of the exactly rounded power, for a dozen FP64 operations instead of a general
// power function.  fp32 keeps powf.
template <class R, int Q> __device__ __forceinline__ R ctrl_factor(R err);
template <int Q>
__device__ __forceinline__ double ctrl_factor_d(double err) {
  const double x = fmin(fmax(err, 1e-10), 1e10);
  double y = (double)exp2f(-__log2f((float)x) / float(Q));
#pragma unroll
  for (int it = 0; it < 2; ++it) y = fma(y * (1.0 / Q), fma(-x, ipow<Q>(y), 1.0), y);
  return 0.9 * y;
}
template <> __device__ __forceinline__ double ctrl_factor<double, 3>(double e) { return ctrl_factor_d<3>(e); }
template <> __device__ __forceinline__ double ctrl_factor<double, 5>(double e) { return ctrl_factor_d<5>(e); }
template <> __device__ __forceinline__ double ctrl_factor<double, 7>(double e) { return ctrl_factor_d<7>(e); }
template <> __device__ __forceinline__ float ctrl_factor<float, 3>(float e) { return 0.9f * powf(e, float(-1.0 / 3)); }
template <> __device__ __forceinline__ float ctrl_factor<float, 5>(float e) { return 0.9f * powf(e, float(-1.0 / 5)); }
template <> __device__ __forceinline__ float ctrl_factor<float, 7>(float e) { return 0.9f * powf(e, float(-1.0 / 7)); }

template <class R> __device__ __forceinline__ R eps_of();
template <> __device__ __forceinline__ double eps_of<double>() { return 2.220446049250313e-16; }
template <> __device__ __forceinline__ float eps_of<float>() { return 1.1920929e-07f; }

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Warp-aggregated draw from the work counter: every lane with `need` receives the next id.
__device__ __forceinline__ int warp_take(bool need, int* counter) {
  const unsigned m = __ballot_sync(FULL, need);
  if (m == 0) return -1;
  const int leader = __ffs(m) - 1;
  const int lane = threadIdx.x & 31;
  int base = 0;
  if (lane == leader) base = atomicAdd(counter, __popc(m));
  base = __shfl_sync(FULL, base, leader);
  return need ? base + __popc(m & lanemask_lt()) : -1;
}

// Hairer-Norsett-Wanner starting step (Solving ODEs I, §II.4), RMS norm with sc = atol + rtol|y0|.
template <class F, class R>
__device__ R initial_step(const R (&y0)[F::D], const R (&f0)[F::D],
                          const typename F::template Theta<R>& th, R t0, R t1, R rtol, R atol,
                          int p) {
  constexpr int D = F::D;
  // roundings spelled out (explicit fma, mul_rn, add_rn) so that every kernel starts alike
  R s0 = R(0), s1 = R(0), sc[D];
#pragma unroll
  for (int i = 0; i < D; ++i) {
    sc[i] = add_rn(atol, mul_rn(rtol, fabs(y0[i])));
    const R a = y0[i] / sc[i], b = f0[i] / sc[i];
    s0 = fma(a, a, s0);
    s1 = fma(b, b, s1);
  }
  const R d0 = sqrt(s0 / R(D)), d1 = sqrt(s1 / R(D));
  const R h0 = (d0 < R(1e-5) || d1 < R(1e-5)) ? R(1e-6) : mul_rn(R(0.01), d0) / d1;
  R y1[D], f1[D];
#pragma unroll
  for (int i = 0; i < D; ++i) y1[i] = fma(h0, f0[i], y0[i]);
  F::f(y1, th, f1);
  R s2 = R(0);
#pragma unroll
  for (int i = 0; i < D; ++i) {
    const R q = add_rn(f1[i], -f0[i]) / sc[i];
    s2 = fma(q, q, s2);
  }
  const R d2 = sqrt(s2 / R(D)) / h0;
  const R dm = d1 > d2 ? d1 : d2;   // same selection as max(d1, d2) with d1 first
  const R h1 = (dm <= R(1e-15)) ? fmax(R(1e-6), h0 * R(1e-3)) : pw<R>(R(0.01) / dm, R(1) / R(p));
  R h = R(100) * h0;
  h = h1 < h ? h1 : h;
  h = (t1 - t0) < h ? (t1 - t0) : h;
  return h;
}

constexpr int M_TSIT5 = 0, M_ROS = 1, M_VERN7 = 2, M_RB23 = 3;
template <int METHOD> struct MethodOrder;
template <> struct MethodOrder<M_TSIT5> { static constexpr int p = Tsit5::order, q = Tsit5::err_order; };
template <> struct MethodOrder<M_ROS> { static constexpr int p = Ros34pw2::order, q = Ros34pw2::err_order; };
template <> struct MethodOrder<M_VERN7> { static constexpr int p = Vern7::order, q = Vern7::err_order; };
template <> struct MethodOrder<M_RB23> { static constexpr int p = Rb23::order, q = Rb23::err_order; };

// Minimum resident 128-thread blocks per SM asked of the compiler (register cap 65536 / (128 b)).
// Measured on B200 for the stellar field in double precision: the replay adjoint runs 13 % faster
// at 3 blocks (168 registers, a few spilled) than unconstrained (2 blocks, 236 registers).
template <class F, class R> struct Tune { static constexpr int adj_blocks = 1, solve_blocks = 1; };
// Fields whose f is large (transcendentals) run the Tsit5 trial with the stage loop rolled: one
// copy of f in the kernel instead of six keeps the hot loop inside the instruction cache (the
// record pass of the stellar field: 35.1 -> 30.6 ms at 2^20).  The reverse sweep stays unrolled,
// which measured faster (20.2 vs 23.0 ms).
template <class F, class R> struct Roll { static constexpr bool value = false; };
template <class R> struct Roll<FNfwMiyamotoNagai, R> { static constexpr bool value = true; };
// The rolled forward/record kernel of the same field: 3 blocks (170 registers) is 13 % faster on
// the record pass than unconstrained.  (Verner 7 kernels keep nine stage vectors live and are
// left unconstrained.)
template <> struct Tune<FNfwMiyamotoNagai, double> {
  static constexpr int adj_blocks = 3, solve_blocks = 3;
};
// fp32: the reverse sweep at 4 blocks/SM (128 registers, from 141) 1.60 -> 1.45 ms at 2^20; the
// solve kernels (112 registers, 4 blocks already) lose at 5 (2.91 -> 3.02 ms record), and 4
// blocks of the fp64 kernels (spilling) lose too (record 20.4 -> 24.4, adjoint 13.6 -> 15.0).
template <> struct Tune<FNfwMiyamotoNagai, float> {
  static constexpr int adj_blocks = 4, solve_blocks = 1;
};
// The forward-sensitivity solve of the logarithmic halo in double precision: 3 blocks/SM
// (168 registers) against 2 unconstrained (228): 31.5 -> 28.7 ms at 2^20 orbits.
template <> struct Tune<FLogHalo, double> {
  static constexpr int adj_blocks = 1, solve_blocks = 3;
};

// Record chunks are reserved from the global bump counter CHUNK_BATCH at a time per warp.
constexpr int CHUNK_BATCH = 32;
// One record entry (t, h, y) written from a lane's registers.  When the entry fills whole
// 16-byte words (the pool is 256-byte aligned and entries are contiguous), it goes out as 16-byte
// vector stores: half (fp64) or a quarter (fp32) of the store instructions, and of the requests
// that the L1 must process for a warp whose 32 lanes write 32 different chunks.
template <class R, int E>
__device__ __forceinline__ void store_entry(R* e, R t, R h, const R (&y)[E - 2]) {
  if constexpr (E * sizeof(R) % 16 == 0 && sizeof(R) == 8) {
    double2* v = reinterpret_cast<double2*>(e);
    v[0] = make_double2(t, h);
#pragma unroll
    for (int c = 0; c < (E - 2) / 2; ++c) v[1 + c] = make_double2(y[2 * c], y[2 * c + 1]);
  } else if constexpr (E * sizeof(R) % 16 == 0 && sizeof(R) == 4 && E % 4 == 0) {
    float4* v = reinterpret_cast<float4*>(e);
    v[0] = make_float4(t, h, y[0], y[1]);
#pragma unroll
    for (int c = 0; c < (E - 4) / 4; ++c)
      v[1 + c] = make_float4(y[2 + 4 * c], y[3 + 4 * c], y[4 + 4 * c], y[5 + 4 * c]);
  } else {
    e[0] = t;
    e[1] = h;
#pragma unroll
    for (int c = 0; c < E - 2; ++c) e[2 + c] = y[c];
  }
}

// One record entry's step size and state read by a replay kernel (read-only path): as 16-byte
// loads when the entry fills whole 16-byte words (fp64 entries of an even number of reals), the
// counterpart of store_entry.
template <class R, int E>
__device__ __forceinline__ void load_entry(const R* e, R& t, R& h, R (&y)[E - 2]) {
  if constexpr (E * sizeof(R) % 16 == 0 && sizeof(R) == 8) {
    const double2* v = reinterpret_cast<const double2*>(e);
    const double2 th = __ldg(v);
    t = th.x;
    h = th.y;
#pragma unroll
    for (int c = 0; c < (E - 2) / 2; ++c) {
      const double2 w = __ldg(v + 1 + c);
      y[2 * c] = w.x;
      y[2 * c + 1] = w.y;
    }
  } else {
    t = __ldg(e);
    h = __ldg(e + 1);
#pragma unroll
    for (int c = 0; c < E - 2; ++c) y[c] = __ldg(e + 2 + c);
  }
}
template <class R, int E>
__device__ __forceinline__ void load_entry(const R* e, R& h, R (&y)[E - 2]) {
  R t;
  load_entry<R, E>(e, t, h, y);
}

// Per-warp ring of trajectories whose start-up is done (id, status, starting step, f(y0)).
constexpr int START_RING = 64;
template <class F, class R>
struct StartRing {
  R f0[F::D][START_RING];
  R h0[START_RING];
  int id[START_RING];
  int st[START_RING];
};
template <class F, class R>
__host__ __device__ constexpr size_t solve_stage_bytes() {
  return (size_t)4 * 32 * RecLayout<F, R>::STAGE_STRIDE * sizeof(R);
}
// Per-lane sensitivity matrices of a 128-thread block, entry (c, j) of lane l at
// [(c * M + j) * 128 + l] (consecutive lanes in consecutive words).
template <class F, class R>
__host__ __device__ constexpr size_t solve_sens_bytes() {
  return (size_t)F::D * F::M * 128 * sizeof(R);
}
template <class F, class R, bool REC, bool SENS = false>
__host__ __device__ constexpr size_t solve_smem_bytes() {
  return ((REC && !RecDirect<F, R>::value) ? solve_stage_bytes<F, R>() : 0) +
         (SENS ? solve_sens_bytes<F, R>() : 0) + 4 * sizeof(StartRing<F, R>);
}

// Parks trajectory k: its id goes to the park list and its state (everything the next attempt
// needs) to the park arrays, from which a later record pass resumes it.
template <class F, class R>
__device__ __forceinline__ void park_state(const SolveParams<R>& p, int k, R t, R h,
                                           const R (&y)[F::D], const R (&k1)[F::D], int S, int Rj,
                                           int seq, bool last_rej, long long att) {
  constexpr int D = F::D;
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

// SENS = true (Tsit5, no record): the forward sensitivities S = dy/dtheta ride along with the
// orbit ("Differentiable astrophysics at scale" §2-§3: sensitivity equations integrated in the
// same kernel, step size controlled on the orbit alone).  The trial, the error test and the
// controller are exactly those of the plain solve, so the accepted mesh and y1 are the forward
// solve's; on each accepted step every column S_{:,j} takes the tangent step of that step along
// (S_{:,j}, e_j).  S lives in shared memory (indexed by the column loop), one slab per lane.
template <class F, class R, int METHOD, bool REC, bool SENS = false>
__global__ void __launch_bounds__(128, METHOD == M_VERN7 ? 1 : Tune<F, R>::solve_blocks)
    k_solve(SolveParams<R> p) {
  using L = RecLayout<F, R>;
  constexpr int D = F::D;
  constexpr int order = MethodOrder<METHOD>::p;
  constexpr int qerr = MethodOrder<METHOD>::q;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // shared memory: [record staging, staged REC only][sensitivities, SENS only]
  //                [start-up ring of this block's warps]
  constexpr bool DIRECT = REC && RecDirect<F, R>::value;
  constexpr bool STAGED = REC && !DIRECT;
  constexpr size_t stage_bytes = STAGED ? solve_stage_bytes<F, R>() : 0;
  R* stage = STAGED ? reinterpret_cast<R*>(smem_raw) + (size_t)warp * 32 * L::STAGE_STRIDE
                    : nullptr;
  R* mystage = STAGED ? stage + lane * L::STAGE_STRIDE : nullptr;
  R* sens = SENS ? reinterpret_cast<R*>(smem_raw + stage_bytes) + threadIdx.x : nullptr;
  StartRing<F, R>* ring =
      reinterpret_cast<StartRing<F, R>*>(smem_raw + stage_bytes +
                                         (SENS ? solve_sens_bytes<F, R>() : 0)) +
      warp;
  int cur = -1;               // direct record: chunk receiving this lane's next entries
  constexpr int SM = F::M;

  const R eps = eps_of<R>();
  const R span = fabs(p.t1 - p.t0);

  int k = -1;                 // current trajectory, -1 when the lane needs work
  int head = 0, tail = 0;     // this warp's start-up ring (warp-uniform)
  int cnext = 0, cend = 0;    // this warp's reserved record chunks [cnext, cend) (warp-uniform)
  bool exhausted = false;     // the work counter has run past N (warp-uniform)
  R t = R(0), h = R(0);
  R y[D], k1[D];
  typename F::template Theta<R> th;
  int S = 0, Rj = 0, ns = 0, seq = 0;
  long long att = 0;
  bool last_rej = false;

#pragma unroll
  for (int c = 0; c < D; ++c) { y[c] = R(0); k1[c] = R(0); }

  for (;;) {
    // ---- refill retired lanes from the warp's start-up ring.  When the ring cannot serve every
    // lane that needs work, the whole warp takes the next 32 trajectories from the work counter
    // and runs their start-up (f(y0), finiteness, starting step) together, one per lane -- so
    // that start-up is paid once per 32 trajectories instead of stalling the warp on one lane.
    const bool need = k < 0 && !(exhausted && head == tail);
    const unsigned nm = __ballot_sync(FULL, need);
    if (nm) {
      const int want = __popc(nm);
      if (!exhausted && tail - head < want) {
        int base = 0;
        if (lane == 0) base = atomicAdd(p.queue, 32);
        base = __shfl_sync(FULL, base, 0);
        if (base + 32 >= p.nqueue) exhausted = true;
        const int q = base + lane;
        int id = q;
        bool valid = q < p.nqueue;
        if (valid && p.order) {
          id = p.order[q];
          valid = id >= 0 && id < p.N;   // a caller's order entry outside the ensemble is skipped
        }
        int st = -1;
        R h0 = R(0), f0[D];
#pragma unroll
        for (int c = 0; c < D; ++c) f0[c] = R(0);
        if (REC && valid && p.resume) {
          // a parked trajectory: its start-up is done; it brings its step and carried slope
          const R* pr = p.park_r + (size_t)id * (2 + 2 * D);
          h0 = pr[1];
#pragma unroll
          for (int c = 0; c < D; ++c) f0[c] = pr[2 + D + c];
        } else if (valid) {
          typename F::template Theta<R> th0;
          F::load(th0, p.theta + (size_t)p.theta_stride * id);
          R yy[D];
#pragma unroll
          for (int c = 0; c < D; ++c) yy[c] = p.y0[(size_t)id * D + c];
          if (!(p.t1 > p.t0)) {
            st = 0;
          } else {
            F::f(yy, th0, f0);
            bool finite = true;
#pragma unroll
            for (int c = 0; c < D; ++c) finite = finite && isfinite(yy[c]) && isfinite(f0[c]);
            if (!finite) st = 3;
            else h0 = initial_step<F, R>(yy, f0, th0, p.t0, p.t1, p.rtol, p.atol, order);
          }
        }
        const unsigned vm = __ballot_sync(FULL, valid);
        if (valid) {
          const int slot = (tail + __popc(vm & lanemask_lt())) & (START_RING - 1);
          ring->id[slot] = id;
          ring->st[slot] = st;
          ring->h0[slot] = h0;
#pragma unroll
          for (int c = 0; c < D; ++c) ring->f0[c][slot] = f0[c];
        }
        tail += __popc(vm);
        __syncwarp();
      }
      const int avail = tail - head;
      const int rank = __popc(nm & lanemask_lt());
      if (need && rank < avail) {
        const int slot = (head + rank) & (START_RING - 1);
        k = ring->id[slot];
        const int st = ring->st[slot];
        h = ring->h0[slot];
#pragma unroll
        for (int c = 0; c < D; ++c) k1[c] = ring->f0[c][slot];
        F::load(th, p.theta + (size_t)p.theta_stride * k);
        ns = 0;
        if (REC && p.resume) {
          const R* pr = p.park_r + (size_t)k * (2 + 2 * D);
          t = pr[0];
#pragma unroll
          for (int c = 0; c < D; ++c) y[c] = pr[2 + c];
          const int* pi = p.park_i + (size_t)k * 4;
          S = pi[0]; Rj = pi[1]; seq = pi[2]; last_rej = pi[3] != 0;
          att = p.park_att[k];
        } else {
#pragma unroll
          for (int c = 0; c < D; ++c) y[c] = p.y0[(size_t)k * D + c];
          t = p.t0;
          S = 0; Rj = 0; att = 0; last_rej = false; seq = 0;
        }
        if constexpr (SENS) {
          for (int i = 0; i < D * SM; ++i)
            sens[i * 128] = p.sens0 ? p.sens0[(size_t)k * D * SM + i] : R(0);
        }
        if (st >= 0) {  // finished at start-up: empty interval or non-finite y0 / f(y0)
          if constexpr (SENS)
            for (int i = 0; i < D * SM; ++i) p.sens1[(size_t)k * D * SM + i] = sens[i * 128];
#pragma unroll
          for (int c = 0; c < D; ++c) p.y1[(size_t)k * D + c] = y[c];
          if (p.nsteps) p.nsteps[k] = 0;
          if (p.nrejected) p.nrejected[k] = 0;
          if (p.status) p.status[k] = st;
          k = -1;
        }
      }
      head += want < avail ? want : avail;
      __syncwarp();
    }
    if (!__any_sync(FULL, k >= 0) && exhausted && head == tail) break;

    // ---- record: a lane about to attempt a step without a chunk takes one from this warp's
    // reserved block (a new block of CHUNK_BATCH from the global bump counter only when the
    // current one runs out) and labels it with its trajectory and sequence number.  When the pool
    // is exhausted the trajectory is parked instead, before the attempt: every step it accepted
    // so far is in its chunks, and its state goes to the park arrays for a later pass.
    if constexpr (REC) {
      // the slice of the first pass: a trajectory with p.slice attempts made is parked instead
      // of taking a chunk (first passes start every trajectory afresh, so attempts count from 0)
      const bool sliced = p.slice > 0 && att >= p.slice;
      const bool needc = k >= 0 && cur < 0 && !sliced;
      const unsigned cm = __ballot_sync(FULL, needc);
      if (cm) {
        const int nwant = __popc(cm), rank = __popc(cm & lanemask_lt());
        const int avail = cend - cnext;
        int mychunk;
        if (nwant > avail) {
          int nb = 0;
          if (lane == 0) nb = atomicAdd(p.chunk_count, CHUNK_BATCH);
          nb = __shfl_sync(FULL, nb, 0);
          mychunk = rank < avail ? cnext + rank : nb + (rank - avail);
          cnext = nb + (nwant - avail);
          cend = nb + CHUNK_BATCH;
        } else {
          mychunk = cnext + rank;
          cnext += nwant;
        }
        if (needc) {
          if (mychunk < p.pool_chunks) {
            cur = mychunk;
            p.chunk_traj[cur] = k;
            p.chunk_seq[cur] = seq;
          } else {
            park_state<F, R>(p, k, t, h, y, k1, S, Rj, seq, last_rej, att);
            k = -1;
          }
        }
      }
      if (k >= 0 && cur < 0 && sliced) {
        park_state<F, R>(p, k, t, h, y, k1, S, Rj, seq, last_rej, att);
        k = -1;
      }
    }

    // ---- one attempted step per active lane
    bool finishing = false;
    if (k >= 0) {
      int st = -1;
      if (att >= p.max_attempts) {
        st = 1;
      } else if (!(h >= R(16) * eps * fmax(fabs(t), span))) {
        st = 2;
      } else {
        bool clipped = false;
        if (t + h > p.t1) { h = p.t1 - t; clipped = true; }
        ++att;
        R ynew[D];
        R err;
        if constexpr (METHOD == M_TSIT5) {
          R k7[D];
          if constexpr (Roll<F, R>::value)
            err = tsit5_trial_rolled<F, R>(y, h, th, k1, ynew, k7, p.rtol, p.atol);
          else
            err = tsit5_trial<F, R>(y, h, th, k1, ynew, k7, p.rtol, p.atol);
          if (err <= R(1)) {
#pragma unroll
            for (int c = 0; c < D; ++c) k1[c] = k7[c];
          }
        } else if constexpr (METHOD == M_VERN7) {
          err = vern7_trial<F, R>(y, h, th, k1, ynew, p.rtol, p.atol);
        } else if constexpr (METHOD == M_RB23) {
          R F2[D];
          err = rb23_trial<F, R>(y, h, th, k1, ynew, F2, p.rtol, p.atol);
          if (err <= R(1)) {
#pragma unroll
            for (int c = 0; c < D; ++c) k1[c] = F2[c];   // first-same-as-last
          }
        } else {
          err = ros_trial<F, R>(y, h, th, ynew, p.rtol, p.atol);
        }
        // the controller's factor 0.9 err^(-1/q), formed once for both outcomes: when a warp holds
        // accepted and rejected lanes together (nearly always) it would otherwise run the power
        // function on both paths
        const R fpow = ctrl_factor<R, qerr>(err);
        if (err <= R(1)) {
          if constexpr (DIRECT) {
            if (cur < p.pool_chunks) {
              R* e = p.pool + ((size_t)cur * L::C + ns) * L::E;
              store_entry<R, L::E>(e, t, h, y);
            }
            if (++ns == L::C) {   // chunk full: the next attempt takes a new one
              ++seq;
              ns = 0;
              cur = -1;
            }
          } else if constexpr (STAGED) {
            R* e = mystage + ns * L::E;
            e[0] = t;
            e[1] = h;
#pragma unroll
            for (int c = 0; c < D; ++c) e[2 + c] = y[c];
            ++ns;
          }
          if constexpr (SENS && METHOD == M_TSIT5) {
            // tangent step of the accepted step for each column j, direction (S_{:,j}, e_j)
            const R* thk = p.theta + (size_t)p.theta_stride * k;
#pragma unroll 1
            for (int j = 0; j < SM; ++j) {
              Dl<R> src[SM];
#pragma unroll
              for (int i = 0; i < SM; ++i) src[i] = Dl<R>(thk[i], i == j ? R(1) : R(0));
              typename F::template Theta<Dl<R>> thd;
              F::load(thd, src);
              R col[D];
#pragma unroll
              for (int c = 0; c < D; ++c) col[c] = sens[(c * SM + j) * 128];
              tsit5_tangent_step<F, R>(y, h, thd, col);
#pragma unroll
              for (int c = 0; c < D; ++c) sens[(c * SM + j) * 128] = col[c];
            }
          }
          ++S;
          const R facmax = last_rej ? R(1) : R(10);
          R fac = (err == R(0)) ? facmax : fpow;
          fac = fmin(facmax, fmax(R(0.2), fac));
          t = (clipped || t + h >= p.t1) ? p.t1 : t + h;
#pragma unroll
          for (int c = 0; c < D; ++c) y[c] = ynew[c];
          if constexpr (METHOD == M_VERN7) F::f(y, th, k1);   // fresh first stage (no FSAL)
          h = h * fac;
          last_rej = false;
          if (t == p.t1) st = 0;
        } else {
          ++Rj;
          R fac = isfinite(err) ? fpow : R(0.2);
          fac = fmin(R(10), fmax(R(0.2), fac));
          h = h * fac;
          last_rej = true;
        }
      }
      if (st >= 0) {
        if constexpr (REC) {
          // a chunk taken for an attempt that never came to be accepted is marked unused; a
          // partly filled one keeps its entries (staged ones are flushed into it below)
          if (cur >= 0 && ns == 0) p.chunk_traj[cur] = -1;
          if (DIRECT || ns == 0) {
            cur = -1;
            ns = 0;
            seq = 0;
          }
        }
        if constexpr (SENS)
          for (int i = 0; i < D * SM; ++i) p.sens1[(size_t)k * D * SM + i] = sens[i * 128];
#pragma unroll
        for (int c = 0; c < D; ++c) p.y1[(size_t)k * D + c] = y[c];
        if (p.nsteps) p.nsteps[k] = S;
        if (p.nrejected) p.nrejected[k] = Rj;
        if (p.status) p.status[k] = st;
        finishing = true;
        k = -1;
      }
    }

    // ---- staged record: flush full (or final partial) chunks into their lanes' chunks, one
    // warp-wide coalesced copy each
    if constexpr (STAGED) {
      const bool want = (ns == L::C) || (finishing && ns > 0);
      unsigned fm = __ballot_sync(FULL, want);
      if (fm) {
        __syncwarp();
        while (fm) {
          const int src = __ffs(fm) - 1;
          fm &= fm - 1;
          const int ch = __shfl_sync(FULL, cur, src);
          const int cnt = __shfl_sync(FULL, ns, src);
          if (ch >= 0 && ch < p.pool_chunks) {
            R* dst = p.pool + (size_t)ch * (L::C * L::E);
            const R* s = stage + src * L::STAGE_STRIDE;
            for (int i = lane; i < cnt * L::E; i += 32) dst[i] = s[i];
          }
        }
        __syncwarp();
        if (want) {
          ++seq;
          ns = 0;
          cur = -1;
          if (finishing) seq = 0;
        }
      }
    }
  }
  // chunks reserved but never filled are marked unused for the chunk-table pass
  if (REC)
    for (int c = cnext + lane; c < cend; c += 32)
      if (c < p.pool_chunks) p.chunk_traj[c] = -1;
}

template <class R>
struct AdjointParams {
  int N;
  const R* theta;
  int theta_stride;
  const R* dL_dy1;
  R* dL_dy0;        // nullable
  R* dL_dtheta;     // [N][M] per trajectory (or scratch for the shared reduction); nullable
  const int* nsteps;
  const long long* choff;   // chunk offsets [N+1]
  const int* chunk_table;
  const R* pool;
  int* queue;
  const int* perm;          // visiting order (longest records first); nullable = identity
  RecBounds bounds;
};

template <class F, class R, int METHOD>
__global__ void __launch_bounds__(128, METHOD == M_VERN7 ? 1 : Tune<F, R>::adj_blocks)
    k_adjoint(AdjointParams<R> p) {
  using L = RecLayout<F, R>;
  constexpr int D = F::D, M = F::M;
  extern __shared__ __align__(16) unsigned char adj_smem[];
  R* tape = reinterpret_cast<R*>(adj_smem) + threadIdx.x;  // per-lane stage tape (TAPE fields)
  int k = -1;
  bool alive = true;
  int n = 0, first_n = -1, cur_ch = 0, next_ch = -1;
  bool pf_pending = false;
  long long cbase = 0;
  R lam[D], thb[M];
  typename F::template Theta<R> th;
#pragma unroll
  for (int c = 0; c < D; ++c) lam[c] = R(0);
#pragma unroll
  for (int j = 0; j < M; ++j) thb[j] = R(0);

  for (;;) {
    const bool need = alive && k < 0;
    if (__any_sync(FULL, need)) {
      const int id = warp_take(need, p.queue);
      if (need) {
        if (id < p.N) {
          k = p.perm ? p.perm[id] : id;
          F::load(th, p.theta + (size_t)p.theta_stride * k);
#pragma unroll
          for (int c = 0; c < D; ++c) lam[c] = p.dL_dy1[(size_t)k * D + c];
#pragma unroll
          for (int j = 0; j < M; ++j) thb[j] = R(0);
          n = p.nsteps[k] - 1;
          first_n = n;
          cbase = p.choff[k];
        } else {
          alive = false;
        }
      }
    }
    if (!__any_sync(FULL, k >= 0 || alive)) break;
    if (k >= 0) {
      if (n >= 0) {
        // chunk of step n; on entering a chunk, fetch the id of the next chunk to be visited and
        // prefetch its lines one step later (the id load then has had a whole step to land)
        if (n == first_n || n % L::C == L::C - 1) {
          cur_ch = chunk_at(p.chunk_table, cbase + n / L::C, p.bounds);
          next_ch = (n / L::C >= 1) ? chunk_at(p.chunk_table, cbase + n / L::C - 1, p.bounds) : -1;
#ifdef GS_CHECKED
          if (next_ch >= p.bounds.pool_chunks) next_ch = -1;
#endif
          pf_pending = next_ch >= 0;
        } else if (pf_pending) {
          const R* q = p.pool + (size_t)next_ch * L::C * L::E;
#pragma unroll
          for (int b = 0; b < L::C * L::E * (int)sizeof(R); b += 128)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const char*>(q) + b));
          pf_pending = false;
        }
        const R* e = chunk_entry<L>(p.pool, cur_ch, n, p.bounds);
        R h, y[D];
        load_entry<R, L::E>(e, h, y);
        if constexpr (METHOD == M_TSIT5) tsit5_adjoint_step<F, R>(y, h, th, lam, thb, tape, blockDim.x);
        else if constexpr (METHOD == M_VERN7) vern7_adjoint_step<F, R>(y, h, th, lam, thb, tape, blockDim.x);
        else if constexpr (METHOD == M_RB23) rb23_adjoint_step<F, R>(y, h, th, lam, thb);
        else ros_adjoint_step<F, R>(y, h, th, lam, thb);
        --n;
      }
      if (n < 0) {
        if (p.dL_dy0)
#pragma unroll
          for (int c = 0; c < D; ++c) p.dL_dy0[(size_t)k * D + c] = lam[c];
        if (p.dL_dtheta)
#pragma unroll
          for (int j = 0; j < M; ++j) p.dL_dtheta[(size_t)k * M + j] = thb[j];
        k = -1;
      }
    }
  }
}

// Forward replay over the recorded mesh at (possibly new) parameters: y_{n+1} = Phi(y_n, h_n),
// rewriting the stored y_n of every step so that a following k_adjoint differentiates the replay
// at these parameters; writes y_S to y1.  t_n and h_n are left as recorded.
// One step of the method's replay map Phi(y, h; theta).
template <class F, class R, int METHOD>
__device__ __forceinline__ void replay_step(const R (&y)[F::D], R h,
                                            const typename F::template Theta<R>& th,
                                            R (&ynew)[F::D]) {
  if constexpr (METHOD == M_TSIT5) tsit5_replay_step<F, R>(y, h, th, ynew);
  else if constexpr (METHOD == M_VERN7) vern7_replay_step<F, R>(y, h, th, ynew);
  else if constexpr (METHOD == M_RB23) rb23_replay_step<F, R>(y, h, th, ynew);
  else ros_replay_step<F, R>(y, h, th, ynew);
}

template <class R>
struct ReplayParams {
  int N;
  const R* theta;
  int theta_stride;
  const R* y0;              // null: each trajectory starts from its stored y_0 (entry 0)
  R* y1;                    // nullable
  const int* nsteps;
  const long long* choff;
  const int* chunk_table;
  R* pool;
  int* queue;
  const int* perm;
  RecBounds bounds;
  const int* gate = nullptr;  // k_replay_forward*: when set and *gate == 0 the kernel does nothing
};

template <class F, class R, int METHOD>
__global__ void __launch_bounds__(128) k_replay_forward(ReplayParams<R> p) {
  using L = RecLayout<F, R>;
  constexpr int D = F::D;
  if (p.gate && *p.gate == 0) return;
  int k = -1, n = 0, S = 0;
  bool alive = true;
  long long cbase = 0;
  R y[D];
  typename F::template Theta<R> th;
#pragma unroll
  for (int c = 0; c < D; ++c) y[c] = R(0);
  for (;;) {
    const bool need = alive && k < 0;
    if (__any_sync(FULL, need)) {
      const int id = warp_take(need, p.queue);
      if (need) {
        if (id < p.N) {
          k = p.perm ? p.perm[id] : id;
          F::load(th, p.theta + (size_t)p.theta_stride * k);
          n = 0;
          S = p.nsteps[k];
          cbase = p.choff[k];
          if (p.y0) {
#pragma unroll
            for (int c = 0; c < D; ++c) y[c] = p.y0[(size_t)k * D + c];
          } else if (S > 0) {
            const R* e0 = chunk_entry<L>(p.pool, chunk_at(p.chunk_table, cbase, p.bounds), 0,
                                         p.bounds);
#pragma unroll
            for (int c = 0; c < D; ++c) y[c] = e0[2 + c];
          }
        } else {
          alive = false;
        }
      }
    }
    if (!__any_sync(FULL, k >= 0 || alive)) break;
    if (k >= 0) {
      if (n < S) {
        R* e = chunk_entry<L>(p.pool, chunk_at(p.chunk_table, cbase + n / L::C, p.bounds), n,
                              p.bounds);
        const R h = e[1];
#pragma unroll
        for (int c = 0; c < D; ++c) e[2 + c] = y[c];
        R ynew[D];
        replay_step<F, R, METHOD>(y, h, th, ynew);
#pragma unroll
        for (int c = 0; c < D; ++c) y[c] = ynew[c];
        ++n;
      }
      if (n >= S) {
        if (p.y1)
#pragma unroll
          for (int c = 0; c < D; ++c) p.y1[(size_t)k * D + c] = y[c];
        k = -1;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Outputs at requested times ("gradsolve: fast exact gradients for ODE ensembles on GPUs" §3.4:
// one extra solver step from the preceding mesh point exactly to each requested time -- the state
// is integrated, not interpolated).  For ascending tau_j: the output is Phi(y_n, tau_j - t_n) for
// the first n with tau_j < t_{n+1} (t_S = t1), and y_S when tau_j >= t1.  The requested times
// travel by value in the kernel parameters.
// ---------------------------------------------------------------------------------------------
constexpr int MAX_OUT = 256;
template <class R>
struct OutTimes {
  int J;
  R t1;
  R tau[MAX_OUT];
};

template <class R>
struct OutParams {
  ReplayParams<R> rp;   // theta, y0, record (y1, queue and perm unused)
  R* y_out;             // [N][J][D]
  OutTimes<R> ot;
  int jS;               // outputs 0 .. jS - 1 are before t1 (the rest are the final state)
};


template <class F, class R, class P>
__device__ __forceinline__ const R* rec_entry(const P& p, long long cbase, int n) {
  using L = RecLayout<F, R>;
  return chunk_entry<L>(p.pool, chunk_at(p.chunk_table, cbase + n / L::C, p.bounds), n,
                        p.bounds);
}

// The recorded step output time tau is taken from: the last step n in [from, S) with
// t_n <= tau, or `from` when there is none (from = 0: a time before t0 is taken from step 0).
// Binary search over the recorded times, which ascend with n; the caller passes, as `from`, the
// step of an earlier (not later) time, whose t_n <= tau.
template <class F, class R, class P>
__device__ __forceinline__ int output_step(const P& p, long long cbase, int from, int S, R tau) {
  int a = from, b = S - 1;
  while (a < b) {
    const int m = (a + b + 1) >> 1;
    if (rec_entry<F, R>(p, cbase, m)[0] <= tau) a = m;
    else b = m - 1;
  }
  return a;
}

// States at requested times.  Output j of trajectory k with tau_j < t1 is one extra step, of size
// tau_j - t_n, from the recorded state y_n of its step n (output_step); the outputs at or after t1
// are the final state, one step of size h_{S-1} from y_{S-1}; with no recorded step every output
// is y0.  The record keeps every y_n, so no walk over it is needed: each output reads one entry
// after its search.  Every lane takes the same jS extra steps (the times are shared), so a warp
// takes them in lockstep.  One lane per trajectory.
template <class F, class R, int METHOD>
__global__ void __launch_bounds__(128) k_replay_outputs(OutParams<R> q) {
  using L = RecLayout<F, R>;
  constexpr int D = F::D;
  const ReplayParams<R>& p = q.rp;
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= p.N) return;
  const int J = q.ot.J, jS = q.jS;
  const int S = p.nsteps[k];
  R* out = q.y_out + (size_t)k * J * D;
  if (S == 0) {
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int c = 0; c < D; ++c) out[(size_t)j * D + c] = p.y0[(size_t)k * D + c];
    return;
  }
  typename F::template Theta<R> th;
  F::load(th, p.theta + (size_t)p.theta_stride * k);
  const long long cbase = p.choff[k];
  int n = 0;
  for (int j = 0; j < jS; ++j) {
    const R tau = q.ot.tau[j];
    n = output_step<F, R>(p, cbase, n, S, tau);
    R t, h, y[D], yo[D];
    load_entry<R, L::E>(rec_entry<F, R>(p, cbase, n), t, h, y);
    replay_step<F, R, METHOD>(y, tau - t, th, yo);
#pragma unroll
    for (int c = 0; c < D; ++c) out[(size_t)j * D + c] = yo[c];
  }
  if (jS < J) {
    R t, h, y[D], yS[D];
    load_entry<R, L::E>(rec_entry<F, R>(p, cbase, S - 1), t, h, y);
    replay_step<F, R, METHOD>(y, h, th, yS);
    for (int j = jS; j < J; ++j)
#pragma unroll
      for (int c = 0; c < D; ++c) out[(size_t)j * D + c] = yS[c];
  }
}

// One step of the method's replay adjoint: lam <- the pullback of lam through the step from y
// with size h, theta-bar accumulated (the tape is the Tsit5 and Verner 7 stage tape).
template <class F, class R, int METHOD>
__device__ __forceinline__ void adjoint_step(const R (&y)[F::D], R h,
                                             const typename F::template Theta<R>& th,
                                             R (&lam)[F::D], R (&thb)[F::M], R* tape) {
  if constexpr (METHOD == M_TSIT5) tsit5_adjoint_step<F, R>(y, h, th, lam, thb, tape, blockDim.x);
  else if constexpr (METHOD == M_VERN7) vern7_adjoint_step<F, R>(y, h, th, lam, thb, tape, blockDim.x);
  else if constexpr (METHOD == M_RB23) rb23_adjoint_step<F, R>(y, h, th, lam, thb);
  else ros_adjoint_step<F, R>(y, h, th, lam, thb);
}

template <class R>
struct AdjOutParams {
  AdjointParams<R> ap;  // dL_dy1 may be null here
  const R* dL_dyout;    // [N][J][D]
  OutTimes<R> ot;
  int jS;               // outputs 0 .. jS - 1 are before t1 (the rest are the final state)
};

// Replay adjoint with outputs at requested times ("gradsolve: fast exact gradients for ODE
// ensembles on GPUs" §3.4).  Output j < jS of trajectory k is one extra step, of size tau_j - t_n,
// from the recorded state y_n of the first step n (going down the record) with t_n <= tau_j, and
// of step 0 if there is none; the outputs at or after t1 are the final state.  So the cotangent of
// y_n is the pullback of the later steps' cotangent through step n, plus, for each output of that
// step, the pullback of the output's cotangent through its extra step.
//
// The walk of k_adjoint (one pullback per active lane per pass of the loop, a lane refilled with
// the next trajectory, longest records first, as soon as its own is done), in which a lane's pass
// pulls back either its next recorded step or, after a step that holds outputs, one of those
// outputs' extra steps.  Both are the same adjoint step of the same y_n with another step size and
// cotangent, so the warp takes them together in one call: a lane that meets an output costs the
// others nothing, where an extra call for it would stall the warp on nearly every pass (with 8
// outputs over about 130 steps, some lane of a 32-lane warp meets one on most passes).  During an
// output's pass the lane's cotangent waits in its shared-memory slot and the output's cotangent
// takes its place in the call; the result is added to it afterwards.
template <class F, class R, int METHOD>
__global__ void __launch_bounds__(128, METHOD == M_VERN7 ? 1 : Tune<F, R>::adj_blocks)
    k_adjoint_outputs(AdjOutParams<R> q) {
  using L = RecLayout<F, R>;
  constexpr int D = F::D, M = F::M;
  extern __shared__ __align__(16) unsigned char adj_smem[];
  R* tape = reinterpret_cast<R*>(adj_smem) + threadIdx.x;
  // after the stage tape of the Tsit5 and Verner 7 sweeps (TAPE reals per stage and lane), this
  // lane's cotangent slot: D reals at stride blockDim.x
  constexpr int TAPE_REALS = (METHOD == M_VERN7 ? 9 : (METHOD == M_TSIT5 ? 6 : 0)) * TapeOf<F>::value;
  R* stash = reinterpret_cast<R*>(adj_smem) + TAPE_REALS * blockDim.x + threadIdx.x;
  const AdjointParams<R>& p = q.ap;
  const int J = q.ot.J, jS = q.jS;
  // per lane: trajectory k, step n; the outputs jcur .. J - 1 are taken; after the pullback of a
  // step that holds outputs jlo .. jcur - 1, r counts them down (r >= jlo: output r is next)
  int k = -1, n = -1, first_n = -1, jcur = 0, jlo = 0, r = -1, cur_ch = 0, next_ch = -1;
  bool alive = true, pf_pending = false;
  long long cbase = 0;
  const R* lo = nullptr;
  R tau_next = R(0);  // tau[jcur - 1]: the time of the next output going down (jcur > 0)
  R lam[D], thb[M];
  typename F::template Theta<R> th;
#pragma unroll
  for (int c = 0; c < D; ++c) lam[c] = R(0);
#pragma unroll
  for (int i = 0; i < M; ++i) thb[i] = R(0);
  for (;;) {
    const bool need = alive && k < 0;
    if (__any_sync(FULL, need)) {
      const int id = warp_take(need, p.queue);
      if (need) {
        if (id < p.N) {
          k = p.perm ? p.perm[id] : id;
          F::load(th, p.theta + (size_t)p.theta_stride * k);
          lo = q.dL_dyout + (size_t)k * J * D;
#pragma unroll
          for (int c = 0; c < D; ++c) lam[c] = p.dL_dy1 ? p.dL_dy1[(size_t)k * D + c] : R(0);
#pragma unroll
          for (int i = 0; i < M; ++i) thb[i] = R(0);
          const int S = p.nsteps[k];
          jcur = S == 0 ? 0 : jS;
          for (int jj = jcur; jj < J; ++jj)
#pragma unroll
            for (int c = 0; c < D; ++c) lam[c] += lo[(size_t)jj * D + c];
          tau_next = jcur > 0 ? q.ot.tau[jcur - 1] : R(0);
          n = S - 1;
          first_n = n;
          r = -1;
          cbase = p.choff[k];
        } else {
          alive = false;
        }
      }
    }
    if (!__any_sync(FULL, k >= 0 || alive)) break;
    if (k >= 0) {
      if (n >= 0) {
        const bool out = r >= 0;  // this pass: output r's extra step from y_n
        if (!out) {
          // chunk of step n, and the next chunk's lines prefetched one step after entering one
          if (n == first_n || n % L::C == L::C - 1) {
            cur_ch = chunk_at(p.chunk_table, cbase + n / L::C, p.bounds);
            next_ch = (n / L::C >= 1) ? chunk_at(p.chunk_table, cbase + n / L::C - 1, p.bounds) : -1;
#ifdef GS_CHECKED
            if (next_ch >= p.bounds.pool_chunks) next_ch = -1;
#endif
            pf_pending = next_ch >= 0;
          } else if (pf_pending) {
            const R* pq = p.pool + (size_t)next_ch * L::C * L::E;
#pragma unroll
            for (int b = 0; b < L::C * L::E * (int)sizeof(R); b += 128)
              asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const char*>(pq) + b));
            pf_pending = false;
          }
        }
        const R* e = chunk_entry<L>(p.pool, cur_ch, n, p.bounds);
        R t, h, y[D];
        load_entry<R, L::E>(e, t, h, y);
        if (out) {
#pragma unroll
          for (int c = 0; c < D; ++c) {
            stash[c * blockDim.x] = lam[c];
            lam[c] = lo[(size_t)r * D + c];
          }
          h = q.ot.tau[r] - t;
        }
        adjoint_step<F, R, METHOD>(y, h, th, lam, thb, tape);
        if (out) {
#pragma unroll
          for (int c = 0; c < D; ++c) lam[c] += stash[c * blockDim.x];
          if (--r < jlo) {  // the step's outputs are taken: on to step n - 1
            jcur = jlo;
            tau_next = jcur > 0 ? q.ot.tau[jcur - 1] : R(0);
            r = -1;
            --n;
          }
        } else if (jcur > 0 && (n == 0 || tau_next >= t)) {  // the step holds outputs
          jlo = jcur - 1;
          while (jlo > 0 && (n == 0 || q.ot.tau[jlo - 1] >= t)) --jlo;
          r = jcur - 1;
        } else {
          --n;
        }
      }
      if (n < 0) {
        if (p.dL_dy0)
#pragma unroll
          for (int c = 0; c < D; ++c) p.dL_dy0[(size_t)k * D + c] = lam[c];
        if (p.dL_dtheta)
#pragma unroll
          for (int i = 0; i < M; ++i) p.dL_dtheta[(size_t)k * M + i] = thb[i];
        k = -1;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Record finalisation.
// ---------------------------------------------------------------------------------------------
// Block-wide exclusive scan of per-trajectory counts (steps, or chunks = ceil(steps / C)).
// Pass 1: each block scans its tile and writes the tile total; pass 2: one block scans the tile
// totals; pass 3: add the tile base.  Deterministic; int64 outputs.
constexpr int SCAN_BLOCK = 1024;

template <int MODE>  // 0: steps, 1: chunks of C
__device__ __forceinline__ long long scan_value(const int* S, int i, int N, int C) {
  if (i >= N) return 0;
  const int s = S[i];
  return MODE == 0 ? (long long)s : (long long)((s + C - 1) / C);
}

__device__ __forceinline__ long long block_exclusive_scan(long long v, long long* total) {
  __shared__ long long warp_sums[SCAN_BLOCK / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(FULL, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = (lane < SCAN_BLOCK / 32) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(FULL, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const long long before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[SCAN_BLOCK / 32 - 1];
  __syncthreads();
  return before;
}

template <int MODE>
__global__ void __launch_bounds__(SCAN_BLOCK) k_scan_tiles(const int* S, int N, int C,
                                                           long long* out, long long* tile_tot) {
  const int i = blockIdx.x * SCAN_BLOCK + threadIdx.x;
  long long tot;
  const long long ex = block_exclusive_scan(scan_value<MODE>(S, i, N, C), &tot);
  if (i < N) out[i] = ex;
  if (threadIdx.x == 0) tile_tot[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(SCAN_BLOCK) k_scan_totals(long long* tile_tot, int ntiles,
                                                            long long* grand) {
  long long carry = 0;
  for (int b0 = 0; b0 < ntiles; b0 += SCAN_BLOCK) {
    const int i = b0 + threadIdx.x;
    long long tot;
    const long long v = i < ntiles ? tile_tot[i] : 0;
    const long long ex = block_exclusive_scan(v, &tot);
    if (i < ntiles) tile_tot[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) *grand = carry;
}

// Exclusive scan of n counts by one block, tile after tile with a carry: out[0..n), out[n] = the
// total.  For short arrays (the length bins of the longest-first order), one launch instead of
// three.
__global__ void __launch_bounds__(SCAN_BLOCK) k_scan_one_block(const int* in, int n,
                                                               long long* out) {
  long long carry = 0;
  for (int b0 = 0; b0 < n; b0 += SCAN_BLOCK) {
    const int i = b0 + threadIdx.x;
    long long tot;
    const long long ex = block_exclusive_scan(i < n ? (long long)in[i] : 0LL, &tot);
    if (i < n) out[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) out[n] = carry;
}

__global__ void k_scan_add(long long* out, int N, const long long* tile_base,
                           const long long* grand) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < N) out[i] += tile_base[i / SCAN_BLOCK];
  if (i == 0) out[N] = *grand;
}

// The summary of a record pass in one three-kernel scan: the exclusive scans of the step counts
// (step offsets) and of the chunk counts ceil(S / C) (chunk offsets) side by side, and the largest
// step count and status (atomicMax into maxes[0] and maxes[1], which the caller zeroes).  The tile
// scratch holds two halves of ntiles + 2: tile totals, then the grand total.
__global__ void __launch_bounds__(SCAN_BLOCK) k_summary_tiles(const int* S, const int* status,
                                                              int N, int C, long long* off,
                                                              long long* choff, long long* tiles,
                                                              int* maxes) {
  const int i = blockIdx.x * SCAN_BLOCK + threadIdx.x;
  const int ntiles = gridDim.x;
  const int sv = i < N ? S[i] : 0;
  long long tot_s, tot_c;
  const long long ex_s = block_exclusive_scan((long long)sv, &tot_s);
  const long long ex_c = block_exclusive_scan((long long)((sv + C - 1) / C), &tot_c);
  if (i < N) {
    off[i] = ex_s;
    choff[i] = ex_c;
  }
  if (threadIdx.x == 0) {
    tiles[blockIdx.x] = tot_s;
    tiles[ntiles + 2 + blockIdx.x] = tot_c;
  }
  int ms = sv, mt = i < N ? status[i] : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ms = max(ms, __shfl_xor_sync(FULL, ms, o));
    mt = max(mt, __shfl_xor_sync(FULL, mt, o));
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMax(maxes, ms);
    atomicMax(maxes + 1, mt);
  }
}

__global__ void __launch_bounds__(SCAN_BLOCK) k_summary_totals(long long* tiles, int ntiles) {
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    long long* t = tiles + h * (ntiles + 2);
    long long carry = 0;
    for (int b0 = 0; b0 < ntiles; b0 += SCAN_BLOCK) {
      const int i = b0 + threadIdx.x;
      long long tot;
      const long long v = i < ntiles ? t[i] : 0;
      const long long ex = block_exclusive_scan(v, &tot);
      if (i < ntiles) t[i] = carry + ex;
      carry += tot;
    }
    if (threadIdx.x == 0) t[ntiles] = carry;
  }
}

__global__ void k_summary_add(long long* off, long long* choff, int N, const long long* tiles,
                              int ntiles) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const long long* tc = tiles + ntiles + 2;
  if (i < N) {
    off[i] += tiles[i / SCAN_BLOCK];
    choff[i] += tc[i / SCAN_BLOCK];
  }
  if (i == 0) {
    off[N] = tiles[ntiles];
    choff[N] = tc[ntiles];
  }
}

// chunk_table[choff[traj] + seq] = chunk (reserved-but-unused chunks carry traj = -1)
__global__ void k_chunk_table(const int* chunk_traj, const int* chunk_seq, int nchunks,
                              const long long* choff, int* table, RecBounds b) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < nchunks) {
    const int k = chunk_traj[c];
    if (k >= 0) {
      const long long ti = choff[k] + chunk_seq[c];
#ifdef GS_CHECKED
      if (ti < 0 || ti >= b.table_cap) {
        gs_violation();
        return;
      }
#endif
      table[ti] = c;
    }
  }
}

// Chunks the parked trajectories of a record pass still need, estimated from their progress:
// a trajectory parked at time t after S accepted steps needs about S (t1 - t) / (t - t0) more
// (at most 128 S; taken with a 25 % margin); out[1] counts those parked before their first step.  With `keys`,
// keys[i] = that estimate of the remaining steps of list[i], capped at kmax (kmax for a
// trajectory without progress): the order in which the next pass takes them, largest first.
template <class R>
__global__ void k_park_estimate(const int* list, int P, const int* count, const R* park_r,
                                const int* park_i, int D, R t0, R t1, int C,
                                unsigned long long* out, int* keys, int kmax) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  unsigned long long chunks = 0, fresh = 0;
  // the number of parked trajectories: P, or (count non-null) read on the device by a launch
  // sized for at most P, queued behind the pass before the host has read it
  const int n = count ? min(*count, P) : P;
  if (i < n) {
    const int k = list[i];
    const R t = park_r[(size_t)k * (2 + 2 * D)];
    const int S = park_i[(size_t)k * 4];
    if (t > t0) {
      // progress in time is a poor guide after a stiff start (tiny early steps): at most 128
      // times the steps taken so far
      const double rem = fmin(double(S + 1) * double(t1 - t) / double(t - t0), 128.0 * (S + 1));
      chunks = (unsigned long long)fmin(1.25 * rem / C + 2.0, double(1 << 20));
      if (keys) keys[i] = (int)fmin(rem, double(kmax));
    } else {
      fresh = 1;
      if (keys) keys[i] = kmax;
    }
  }
  // one atomic per warp for each sum (the block is a whole number of warps)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    chunks += __shfl_xor_sync(FULL, chunks, o);
    fresh += __shfl_xor_sync(FULL, fresh, o);
  }
  if ((threadIdx.x & 31) == 0) {
    if (chunks) atomicAdd(out, chunks);
    if (fresh) atomicAdd(out + 1, fresh);
  }
}

// *p = v, queued on a stream (no host buffer to keep alive until the copy has run).
__global__ void k_set_int(int* p, int v) { *p = v; }

// The stored states of a record belong to the theta kept beside them.  Compares the caller's
// theta with that copy bit for bit; any difference sets *stale (the caller zeroes it, or sets it
// to force a replay) and the copy takes the caller's values.
template <class R>
__global__ void k_theta_check(const R* theta, R* kept, long long count, int* stale) {
  using U = typename std::conditional<sizeof(R) == 8, unsigned long long, unsigned>::type;
  const U* a = reinterpret_cast<const U*>(theta);
  U* b = reinterpret_cast<U*>(kept);
  bool diff = false;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count;
       i += (long long)gridDim.x * blockDim.x) {
    const U v = a[i];
    if (v != b[i]) {
      b[i] = v;
      diff = true;
    }
  }
  if (__any_sync(FULL, diff) && (threadIdx.x & 31) == 0) *stale = 1;
}

// max over S (int), via warp reduce + atomicMax
__global__ void k_max_int(const int* S, int N, int* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  int v = i < N ? S[i] : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(FULL, v, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, v);
}

// Export: write the record as contiguous ragged arrays T[tot], H[tot], Y[tot][D] in
// trajectory-major order (offsets = prefix sums of S).  One thread per trajectory-step.
template <class R>
__global__ void k_export(const R* pool, const int* table, const long long* choff,
                         const long long* offsets, int N, int D, int C, long long total, R* T,
                         R* H, R* Y, RecBounds b) {
  const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= total) return;
  // binary search the trajectory owning step g
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= g) lo = mid; else hi = mid - 1;
  }
  const int k = lo;
  const long long n = g - offsets[k];
  const int E = 2 + D;
  const long long ti = choff[k] + n / C;
  const int ch = table[ti];
  const R* e = pool + ((size_t)ch * C + (n % C)) * E;
#ifdef GS_CHECKED
  if (ti < 0 || ti >= b.table_cap || ch < 0 || ch >= b.pool_chunks) {
    gs_violation();
    return;
  }
#endif
  if (T) T[g] = e[0];
  if (H) H[g] = e[1];
  if (Y) for (int c = 0; c < D; ++c) Y[g * D + c] = e[2 + c];
}

// Import: inverse of export into a pool whose chunks are laid out trajectory by trajectory
// (chunk id = choff[k] + n / C, so chunk_table is the identity).
template <class R>
__global__ void k_import(R* pool, const long long* choff, const long long* offsets, int N, int D,
                         int C, long long total, const R* T, const R* H, const R* Y,
                         RecBounds b) {
  const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= total) return;
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= g) lo = mid; else hi = mid - 1;
  }
  const int k = lo;
  const long long n = g - offsets[k];
  const int E = 2 + D;
  const long long ch = choff[k] + n / C;
#ifdef GS_CHECKED
  if (ch < 0 || ch >= b.pool_chunks) {
    gs_violation();
    return;
  }
#endif
  R* e = pool + ((size_t)ch * C + (n % C)) * E;
  e[0] = T ? T[g] : R(0);
  e[1] = H[g];
  for (int c = 0; c < D; ++c) e[2 + c] = Y[g * D + c];
}

// Visiting order for the replay kernels: trajectories sorted by decreasing record length
// (counting sort on S; bin b holds S = smax - b), so that the work queue hands out the longest
// records first and the tail of the launch is made of the shortest ones.
__global__ void k_bin_count(const int* S, int N, int smax, int* bins) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < N) atomicAdd(&bins[smax - S[i]], 1);
}
// The same counts through a per-block histogram in shared memory ([smax + 1] ints), added to the
// global one once per nonzero bin: a handful of hot bins no longer serialise every element's
// atomic in L2.
__global__ void k_bin_count_smem(const int* S, int N, int smax, int* bins) {
  extern __shared__ int hist[];
  for (int j = threadIdx.x; j <= smax; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < N) atomicAdd(&hist[smax - S[i]], 1);
  __syncthreads();
  for (int j = threadIdx.x; j <= smax; j += blockDim.x)
    if (hist[j]) atomicAdd(&bins[j], hist[j]);
}
// perm[position] = i (or ids[i] when ids is given), positions by decreasing S[i]
__global__ void k_bin_scatter(const int* S, int N, int smax, const long long* binoff, int* cursor,
                              int* perm, const int* ids) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < N) {
    const int b = smax - S[i];
    perm[binoff[b] + atomicAdd(&cursor[b], 1)] = ids ? ids[i] : i;
  }
}
// The same scatter with one global reservation per block and nonzero bin: ranks within the block
// from a shared-memory histogram ([2 (smax + 1)] ints: counts, then the block's bases).
__global__ void k_bin_scatter_smem(const int* S, int N, int smax, const long long* binoff,
                                   int* cursor, int* perm, const int* ids) {
  extern __shared__ int hist[];
  int* base = hist + smax + 1;
  for (int j = threadIdx.x; j <= smax; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  int b = 0, rank = 0;
  if (i < N) {
    b = smax - S[i];
    rank = atomicAdd(&hist[b], 1);
  }
  __syncthreads();
  for (int j = threadIdx.x; j <= smax; j += blockDim.x)
    if (hist[j]) base[j] = atomicAdd(&cursor[j], hist[j]);
  __syncthreads();
  if (i < N) perm[binoff[b] + base[b] + rank] = ids ? ids[i] : i;
}

__global__ void k_iota(int* a, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) a[i] = i;
}

// ---------------------------------------------------------------------------------------------
// Shared-theta reduction: out[j] = sum_k part[k][j] in a fixed order.  Each block reduces a fixed
// contiguous slice of trajectories (warp shuffles, then shared memory), writes its partial; a
// second launch with one block sums the partials in block order.  Bitwise reproducible.
// ---------------------------------------------------------------------------------------------
constexpr int RED_BLOCK = 256;

template <class R>
__global__ void __launch_bounds__(RED_BLOCK) k_reduce_theta(const R* part, int N, int M,
                                                            int per_block, R* partials) {
  __shared__ R warp_acc[RED_BLOCK / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k0 = blockIdx.x * per_block;
  const int k1 = min(N, k0 + per_block);
  for (int j = 0; j < M; ++j) {
    R acc = R(0);
    for (int k = k0 + threadIdx.x; k < k1; k += RED_BLOCK) acc += part[(size_t)k * M + j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
    if (lane == 0) warp_acc[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      R s = R(0);
      for (int w = 0; w < RED_BLOCK / 32; ++w) s += warp_acc[w];
      partials[(size_t)blockIdx.x * M + j] = s;
    }
    __syncthreads();
  }
}

template <class R>
__global__ void k_reduce_partials(const R* partials, int nblocks, int M, R* out) {
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < M; j += gridDim.x * blockDim.x) {
    R s = R(0);
    for (int b = 0; b < nblocks; ++b) s += partials[(size_t)b * M + j];
    out[j] = s;
  }
}

}  // namespace gs
