/* gradsolve_b200.h -- C ABI of the B200 record-and-replay discrete-adjoint library.
 *
 * What it computes ("gradsolve: fast exact gradients for ODE ensembles on GPUs"):
 *   An ensemble of N independent trajectories dy/dt = f(y; theta_k), y(t0) = y0_k, is solved with
 *   an adaptive embedded pair (§2.1: trial steps, RMS error test
 *   RMS(e / (atol + rtol max(|y|, |y_new|))) <= 1, reject and retry from the same (t, y)).
 *   The record pass keeps each trajectory's accepted steps (§3, Fig. 2: the mesh h = R(theta0);
 *   rejected trials leave no trace), and the replay gradient is the exact reverse-mode derivative of
 *   the fixed-step replay over that mesh with the mesh held fixed as data (§3: d Psi(theta;
 *   sg[R(theta0)]) / d theta, Eq. 4), with respect to theta, y0 or both.  The loss is a scalar
 *   L = sum_k l(y_k(t1; theta)) (§2.2), so the caller passes dL/dy1 and receives the pull-back.
 *   Non-stiff problems use the Tsit5 5(4) pair with first-same-as-last reuse (§2.1, §3.1) or
 *   Verner's 7(6) pair; stiff problems a linearly implicit Rosenbrock-Wanner step (ROS34PW2 or
 *   Rosenbrock23), whose stages solve with I - gamma h J and whose backward pass uses transpose
 *   solves with the same factorisation and differentiates J (§3.2).  One GPU thread integrates
 *   one trajectory with its state in registers (§2.4, §4.1); the neural field takes one warp.
 *   gs_solve_forward_sens integrates forward sensitivities dy/dtheta with the orbit instead
 *   ([DA] = "Differentiable astrophysics at scale", §2-§3).
 *
 * Conventions (all entry points):
 *   - Real arrays are double (GS_F64) or float (GS_F32) per gs_system.dtype, row-major:
 *     y0, y1, dL_dy1, dL_dy0: [N][d];  theta, dL_dtheta: [N][m], or [m] when theta_shared.
 *   - Array pointers are DEVICE pointers owned by the caller, unless stated otherwise.  The record
 *     (gs_record) is owned by the library and freed by gs_record_destroy.  Before launching, the
 *     entry points ask the runtime what each array is and return GS_ERR_INVALID_ARG for plain
 *     (unregistered) host memory or another device's memory, which a kernel could not read;
 *     device, managed and page-locked host memory pass.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued on it; calls
 *     return when the work is enqueued, except where a host synchronisation is stated.  Calls on
 *     one record use its device storage and must be ordered: on one stream, or with the caller
 *     synchronising between streams.
 *   - Errors: every entry point returns a gs_status and never aborts or exits; gs_last_error()
 *     returns a message for the calling thread's most recent failure.
 *   - Per-trajectory status codes (status arrays): 0 ok; 1 max_attempts reached; 2 step size
 *     underflow (h < 16 eps max(|t|, |t1 - t0|) or h not finite); 3 y0 or f(y0) not finite.  A
 *     failed trajectory's record ends at its last accepted step and y1 holds its state there.
 *   - Sizes: N <= 2^31 - 1; the record holds at most 2^31 - 1 chunks.
 */
#ifndef GRADSOLVE_B200_H
#define GRADSOLVE_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GS_OK = 0,
  GS_ERR_INVALID_ARG = 1,  /* bad pointer, size, enum or inconsistent d/m */
  GS_ERR_CUDA = 2,         /* a CUDA call failed; see gs_last_error() */
  GS_ERR_CAPACITY = 3,     /* a size limit of the library was exceeded */
  GS_ERR_UNSUPPORTED = 4,  /* field/method/dtype combination not built */
  GS_ERR_TRAJ_FAILED = 5   /* gs_solve_record only: some trajectory status != 0 */
} gs_status;

typedef enum { GS_F64 = 0, GS_F32 = 1 } gs_dtype;
/* GS_TSIT5: Tsitouras 5(4), 7 stages, first-same-as-last ([GS] §2.1, the default explicit pair).
 * GS_ROS34PW2: Rang & Angermann's 4-stage Rosenbrock-Wanner method, order 3(2), for stiff fields.
 * GS_VERN7: Verner's 7(6) pair, 10 stages, for tight tolerances ([GS] §3.1: the seventh-order
 * Verner pair offered next to Tsit5); every explicit field except GS_MLP_4_32_32_4.
 * GS_ROSENBROCK23: Shampine & Reichelt's linearly implicit order-2(3) pair ([GS] §3.1: the
 * second-order Rosenbrock23 method of the fused stiff kernels), for the stiff fields. */
typedef enum { GS_TSIT5 = 0, GS_ROS34PW2 = 1, GS_VERN7 = 2, GS_ROSENBROCK23 = 3 } gs_method;

/* Built-in fields (all autonomous).  d = state size, m = parameters per trajectory.
 *   GS_LOTKA_VOLTERRA  d=2 m=4     theta = (alpha, beta, gamma, delta)
 *   GS_LORENZ63        d=3 m=3     theta = (sigma, rho, beta)            ([GS] §4.3)
 *   GS_MLP_4_32_32_4   d=4 m=1348  tanh MLP 4->32->32->4, theta = (W1,b1,W2,b2,W3,b3), shared
 *   GS_ROBERTSON       d=3 m=3     theta = (k1, k2, k3), stiff          ([GS] §4.2, §4.5)
 *   GS_NFW_MN          d=6 m=5     test particle in NFW halo + Miyamoto-Nagai disk,
 *                                  theta = (M_h, r_s, M_d, a, b), G = 1
 *   GS_LINEAR          d=3 m=9     y' = A y, theta = A row-major         ([GS] §4.6-4.7)
 *   GS_LOG_HALO        d=6 m=2     test particle in the flattened logarithmic halo
 *                                  Phi = v_c^2/2 ln(R_c^2 + x^2 + y^2 + z^2/q^2), R_c = 0.2,
 *                                  theta = (v_c, q)                     ([DA] §3)
 *   GS_HIRES           d=8 m=12    stiff HIRES kinetics, theta = the 12 rate constants
 *                                  (1.71, 0.43, 8.32, 7e-4, 8.75, 10.03, 0.035, 1.12, 1.745,
 *                                  280, 0.69, 1.81 nominal)             ([GS] §4.5-4.6)
 * [DA] = "Differentiable astrophysics at scale: solving and differentiating ODE ensembles on the
 * GPU". */
typedef enum {
  GS_LOTKA_VOLTERRA = 0,
  GS_LORENZ63 = 1,
  GS_MLP_4_32_32_4 = 2,
  GS_ROBERTSON = 3,
  GS_NFW_MN = 4,
  GS_LINEAR = 5,
  GS_LOG_HALO = 6,
  GS_HIRES = 7
} gs_field;

typedef struct {
  int32_t field;        /* gs_field */
  int32_t method;       /* gs_method: GS_TSIT5 or GS_VERN7 for non-stiff fields, GS_ROS34PW2 or
                           GS_ROSENBROCK23 for stiff ones */
  int32_t dtype;        /* gs_dtype */
  int32_t d, m;         /* must equal the field's sizes (checked) */
  int32_t theta_shared; /* 1: theta is [m] shared by all trajectories; 0: [N][m] */
} gs_system;

typedef struct {
  int64_t max_attempts;          /* per trajectory; <= 0 means the default 100000 */
  int64_t record_capacity_steps; /* initial record pool size in steps; 0 = automatic */
  const int32_t* start_order;    /* device [N] or NULL: trajectory started at queue position q
                                    is start_order[q].  Scheduling only (results do not depend
                                    on it): a permutation that starts long trajectories first
                                    shortens the tail of a launch.  Entries outside [0, N) are
                                    skipped; a non-permutation leaves some outputs unwritten.
                                    gs_solve_record falls back to the previous record's
                                    longest-first order when NULL (see there). */
} gs_options;

typedef struct gs_record gs_record; /* opaque, library-owned, device resident */

typedef struct {
  int64_t N;
  int64_t total_steps;      /* sum of accepted steps over the ensemble */
  int32_t max_steps;        /* longest record */
  int32_t chunk_steps;      /* C: steps per pool chunk */
  int32_t entry_reals;      /* E = 2 + d: reals per recorded step (t_n, h_n, y_n[0..d-1]) */
  int32_t dtype;
  int64_t nchunks;          /* chunks handed out from the pool (a few may be reserved but
                               unused; the chunk table lists the used ones) */
  int64_t pool_bytes;       /* device bytes of the step pool */
  /* device pointers owned by the record */
  const int32_t* nsteps;        /* [N] accepted steps S_k */
  const int32_t* status;        /* [N] per-trajectory status */
  const int64_t* offsets;       /* [N+1] exclusive prefix sum of S_k (ragged-array offsets) */
  const int64_t* chunk_offsets; /* [N+1] exclusive prefix sum of ceil(S_k / C) */
  const int32_t* chunk_table;   /* [nchunks]: chunk id of trajectory k's j-th chunk at
                                   chunk_offsets[k] + j */
  const void* pool;             /* chunk c holds steps of one trajectory at
                                   pool + (c*C + slot)*E reals, entry = (t, h, y[0..d-1]) */
  double solve_ms;              /* device time of the solve kernel(s) of the last
                                   gs_solve_record (CUDA events around the launch), 0 if none */
  const int32_t* order;          /* [N] trajectories by decreasing accepted-step count (the
                                   replay's visiting order); usable as gs_options.start_order
                                   for later solves of the same ensemble */
} gs_record_info_t;

/* Forward-only solve ([GS] §4.1: one thread per trajectory, final state only).
 * In:  theta, y0 (device), t0 < t1 (t1 <= t0 returns y1 = y0 with 0 steps), rtol, atol > 0.
 * Out: y1 [N][d]; nsteps, nrejected, status [N] (int32, each nullable).
 * Asynchronous: no host synchronisation; per-trajectory failures appear only in `status`. */
gs_status gs_solve_forward(const gs_system* sys, const gs_options* opt, int64_t N,
                           const void* theta, const void* y0, double t0, double t1, double rtol,
                           double atol, void* y1, int32_t* nsteps, int32_t* nrejected,
                           int32_t* status, void* stream);

/* Forward solve with forward sensitivities ([DA] §2-§3: the sensitivity equations
 * S' = J_y(y) S + J_theta(y), S = dy/dtheta, integrated in the same kernel as the orbit, with the
 * step size controlled on the orbit alone).  The trial steps, error test and controller are those
 * of gs_solve_forward, so y1, nsteps, nrejected and status are identical to its results; on every
 * accepted step each column S_{:,j} takes the same Tsit5 step of the sensitivity equations along
 * (S_{:,j}, e_j).  The result is therefore the exact derivative of the discrete solution on the
 * accepted mesh (the mesh held fixed, as in [GS] §3).
 * In:  as gs_solve_forward, plus S0 [N][d][m] (device, nullable: zero, i.e. y0 independent of
 * theta).  For a shared theta, S is still per trajectory: [N][d][m].
 * Out: y1 [N][d]; S1 [N][d][m] (device, required); nsteps, nrejected, status (nullable).
 * Built for GS_TSIT5 and every Tsit5 field except GS_MLP_4_32_32_4 (GS_ERR_UNSUPPORTED otherwise).
 * A non-finite S does not change a trajectory's status (the controller does not see S).
 * Asynchronous. */
gs_status gs_solve_forward_sens(const gs_system* sys, const gs_options* opt, int64_t N,
                                const void* theta, const void* y0, const void* S0, double t0,
                                double t1, double rtol, double atol, void* y1, void* S1,
                                int32_t* nsteps, int32_t* nrejected, int32_t* status,
                                void* stream);

/* Record pass ([GS] §3, Fig. 2): the same adaptive solve, keeping each accepted step
 * (t_n, h_n, y_n) = (start time, step size used, state at the start of the step), n < S_k.
 * *rec: if NULL on entry a new record is created; otherwise its storage is reused (grown when
 * needed) and its contents replaced.  y1 [N][d] (device, required), status [N] (nullable).
 * Synchronises the stream once to size the record; if the pool was too small the solve is run
 * again with exactly the needed size.  A record made again for an ensemble of the same size
 * starts its trajectories in the previous solve's longest-first order (scheduling only: results
 * do not depend on the order).  Returns GS_ERR_TRAJ_FAILED (with the record complete)
 * when some trajectory status != 0. */
gs_status gs_solve_record(const gs_system* sys, const gs_options* opt, int64_t N,
                          const void* theta, const void* y0, double t0, double t1, double rtol,
                          double atol, gs_record** rec, void* y1, int32_t* status, void* stream);

/* Replay gradient ([GS] §3): the exact reverse-mode derivative of the replay over the recorded
 * mesh with the mesh held fixed as data, at `theta`: d Psi(theta; sg[R(theta0)]) / d theta, where
 * R(theta0) is the recorded mesh, for `theta` equal to the recorded theta0 or not ([GS] §3; §4.8:
 * one mesh serves the gradients of a whole fit).  The backward sweep recomputes each step's stages
 * from the state stored for that step ([GS] §3.3: one accepted state kept per step).  The record
 * keeps the theta its stored states were made at (the record pass's, or the latest
 * gs_replay_forward's); the call compares it with `theta` bit for bit on the device and, when they
 * differ, first replays the mesh forward at `theta` from the stored y_0, rewriting the stored
 * states in place (t_n, h_n kept; nothing allocated).  Calls on one record must be ordered on one
 * stream (they share its states).
 * In:  theta (as for the solve), dL_dy1 [N][d].  Out (each nullable, at least one non-NULL):
 * dL_dy0 [N][d]; dL_dtheta [N][m], or [m] = sum over the ensemble when theta is shared (summed in
 * a fixed order: bitwise reproducible).  Asynchronous. */
gs_status gs_replay_grad(const gs_record* rec, const void* theta, const void* dL_dy1,
                         void* dL_dtheta, void* dL_dy0, void* stream);

/* Forward replay ([GS] §3, Eq. 4): y_{n+1} = Phi(y_n, h_n; theta) over the recorded mesh from y0,
 * storing each y_n in the record (t_n and h_n are kept) and y_S in y1 [N][d] (device, nullable);
 * the record then holds the states of `theta` (and of this y0).  Asynchronous. */
gs_status gs_replay_forward(gs_record* rec, const void* theta, const void* y0, void* y1,
                            void* stream);

/* States at requested times ([GS] §3.4: one extra solver step from the preceding mesh point
 * exactly to each requested time -- the returned state is integrated, not interpolated).
 * tau: HOST array of J times (1 <= J <= GS_MAX_OUTPUT_TIMES), ascending; for tau_j the output is
 * Phi(y_n, tau_j - t_n) with n the first recorded step with tau_j < t_{n+1} (t_S = t1), and the
 * final state for tau_j >= t1 (times before t0 are integrated backwards from y0).  Uses the
 * record's stored states, replayed first when `theta` is not the theta they were made at (as
 * gs_replay_grad); y0 [N][d] (device) is the initial state, read for trajectories with no
 * recorded step.  y_out [N][J][d] (device).  Every field, the MLP field included.
 * Asynchronous. */
#define GS_MAX_OUTPUT_TIMES 256
gs_status gs_replay_outputs(const gs_record* rec, const void* theta, const void* y0, int32_t J,
                            const double* tau, void* y_out, void* stream);

/* Gradient of a loss on the outputs at requested times (and optionally on the final state):
 * dL_dyout [N][J][d] (device), dL_dy1 [N][d] (device, nullable); outputs as gs_replay_grad.
 * Each output's cotangent is pulled back through its extra step from y_n and added to the
 * cotangent of y_n.  The stored states follow `theta` as in gs_replay_grad.  Asynchronous. */
gs_status gs_replay_grad_outputs(const gs_record* rec, const void* theta, int32_t J,
                                 const double* tau, const void* dL_dyout, const void* dL_dy1,
                                 void* dL_dtheta, void* dL_dy0, void* stream);

/* Replay gradient that allocates no device memory.  The paper has no counterpart: this entry
 * point exists for callers that must not allocate at the moment they ask for a gradient -- code
 * that runs while a stream is being captured into a CUDA graph (allocation is not a capturable
 * operation), code living under an allocator that forbids driver allocations, or a time-critical
 * loop in which cudaMalloc/cudaFree would synchronise the device.  gs_replay_grad, by contrast,
 * may allocate on its first use (work counters, and for a shared theta its per-trajectory
 * scratch).
 * Same arguments and result as gs_replay_grad, for every field except GS_MLP_4_32_32_4
 * (GS_ERR_UNSUPPORTED).  Its scratch -- a work counter and, when theta is shared, the
 * per-trajectory theta-bar [N][m] plus the block partials of the ensemble sum -- lives in one
 * fixed array of GS_NOALLOC_SCRATCH_BYTES (8 MiB) inside the library, held by every GPU that
 * loads the library until the process exits.  A record whose shared-theta scratch would not fit
 * (about N*m <= 1.04e6 in double, 2.09e6 in float) is rejected with GS_ERR_CAPACITY.
 * Like gs_replay_grad it differentiates at `theta` even when the stored states were made at
 * another theta, replaying them into the record's own slots first.
 * The first call on a device looks up that array's device address (a one-time set-up per
 * device), and the first call for each (field, method, dtype) combination loads that
 * combination's kernels; make those first calls before any stream capture begins.  All calls
 * share the one array and its work counters are cleared at the start of each call: calls that
 * overlap on the GPU (on different streams, or from different threads) race and must not be
 * issued.  Asynchronous. */
#define GS_NOALLOC_SCRATCH_BYTES (8u << 20)
gs_status gs_replay_grad_noalloc(const gs_record* rec, const void* theta, const void* dL_dy1,
                                 void* dL_dtheta, void* dL_dy0, void* stream);

/* Checked build (compiled with -DGS_CHECKED into libgradsolve_b200_checked.so): every access
 * through a record's chunk table is checked against the allocated pool and table, and an
 * out-of-range one is counted and redirected to scratch memory instead of touching memory
 * outside the record.  Returns, in *count, the number counted since the previous call (the
 * counter is then reset).  Synchronises the device.  The normal build returns GS_ERR_UNSUPPORTED. */
gs_status gs_checked_violations(int64_t* count);

/* Sizes and device pointers of a record (no synchronisation). */
gs_status gs_record_info(const gs_record* rec, gs_record_info_t* out);

/* Copy the record out as contiguous ragged arrays in trajectory order: T[total], H[total],
 * Y[total][d] (device, each nullable) and offsets [N+1] (device int64, nullable). */
gs_status gs_record_export(const gs_record* rec, void* T, void* H, void* Y, int64_t* offsets,
                           void* stream);

/* Build a record from contiguous ragged arrays (device): nsteps [N] int32, T [total] (nullable,
 * zeros when NULL), H [total], Y [total][d] with total = sum nsteps.  Lets one mesh be replayed
 * by another producer's record or reused across many gradients ([GS] §4.8).  The theta of the
 * imported states is unknown to the library, so the first call that takes a theta replays them
 * from each trajectory's first state Y[offsets[k]].  Synchronises once. */
gs_status gs_record_import(const gs_system* sys, int64_t N, const int32_t* nsteps, const void* T,
                           const void* H, const void* Y, gs_record** rec, void* stream);

/* Free a record (NULL is ignored).  Synchronises the record's device.  The record's device
 * storage goes to the device's cache of record storage, where the next records take it (see
 * gs_memory_trim). */
void gs_record_destroy(gs_record* rec);

/* Records keep their device storage in a cache per device: storage released by a destroyed record
 * (or by a record that grew) stays reserved for later records instead of going back to the
 * device, so a new record costs no allocation and destroying one no cudaFree.  New storage comes
 * from cudaMalloc; when the device runs out of memory the cache is handed back first.
 * gs_memory_trim(keep_bytes) hands cached storage beyond keep_bytes back to the current device
 * (storage of live records is not touched).  Synchronises the device.  Not part of the method
 * ([GS] has no counterpart): memory management of the library. */
gs_status gs_memory_trim(int64_t keep_bytes);

/* Message of the calling thread's last failure ("" if none). */
const char* gs_last_error(void);

/* Library version string. */
const char* gs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GRADSOLVE_B200_H */
