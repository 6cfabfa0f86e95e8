"""Seeded synthetic ensembles: the inputs both the CUDA library and the CPU oracle consume.

This module holds random-number generation and the shapes of the benchmark ensembles, and none
of the solver's arithmetic.  Every array is generated on the host in float64 from a
counter-based SplitMix64 stream (Steele, Lea & Flood 2014: state advance by the golden-ratio
increment, then the two xor-shift-multiply finalisation rounds), so an array depends only on
(seed, stream, index) and any sub-range can be regenerated alone.  Uniforms take the top 53
bits; normals use the Box-Muller transform.

The five ensembles (sizes, distributions and tolerances as stated for the benchmark; the pages'
own workloads -- Lorenz, Robertson, stellar orbits -- are described in "gradsolve: fast exact
gradients for ODE ensembles on GPUs" §4 and "Differentiable astrophysics at scale" §3):

  lotka_volterra  N=1024,   d=2, m=4, fp64, Tsit5,    t in [0,10],  rtol 1e-6, atol 1e-8
  lorenz63        N=65536,  d=3, m=3, fp64, Tsit5,    t in [0,1],   rtol 1e-8, atol 1e-10
  mlp             N=16384,  d=4, M=1348 shared, fp32, Tsit5, t in [0,1], rtol 1e-5, atol 1e-6
  robertson       N=65536,  d=3, m=3, fp64, ROS34PW2, t in [0,1e4], rtol 1e-6, atol 1e-10
  nfw_mn          N=2^20,   d=6, m=5, fp64 (fp32 variant at rtol 1e-5, atol 1e-6), Tsit5,
                  t in [0,20], rtol 1e-8, atol 1e-10
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z):
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        return _mix(np.uint64(seed) * _GOLDEN + np.uint64(stream) + np.uint64(1))


def uniform(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """n uniforms in [0, 1) from the counter-based stream (seed, stream), indices start..start+n."""
    idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix(_key(seed, stream) + idx * _GOLDEN)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, stream: int, n: int) -> np.ndarray:
    """n standard normals by Box-Muller from 2n uniforms of the stream."""
    u = uniform(seed, stream, 2 * n)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)


# stream ids: one per quantity so that changing N never shifts another quantity's draws
S_THETA, S_Y0, S_TARGET, S_DIR, S_VEL, S_TEACHER, S_STUDENT = 1, 2, 3, 4, 5, 6, 7

MLP_SIZES = (4, 32, 32, 4)
# parameter layout of the 4->32->32->4 tanh MLP (row-major W[out][in]; all layers biased)
MLP_LAYOUT = (("W1", 0, (32, 4)), ("b1", 128, (32,)), ("W2", 160, (32, 32)),
              ("b2", 1184, (32,)), ("W3", 1216, (4, 32)), ("b3", 1344, (4,)))
MLP_M = 1348


@dataclass
class Workload:
    name: str
    field: str                 # lotka_volterra | lorenz63 | mlp | robertson | nfw_mn | log_halo
    method: str                # tsit5 | ros34pw2
    dtype: type                # np.float64 | np.float32
    N: int
    d: int
    m: int
    theta_shared: bool
    theta: np.ndarray          # [N, m] or [m]
    y0: np.ndarray             # [N, d]
    t0: float
    t1: float
    rtol: float
    atol: float
    seed: int
    target: Optional[np.ndarray] = None   # [N, d] when drawn directly
    target_kind: str = "given"            # given | nominal_solve | teacher_solve | nominal_y0
    nominal_theta: Optional[np.ndarray] = None
    loss_mask: Optional[np.ndarray] = None  # components of y entering the loss (1) or not (0)
    loss_scale: float = 1.0               # L = loss_scale * sum_k |mask*(y_k - target_k)|^2
    notes: dict = field(default_factory=dict)


def _scaled(nominal, lo, hi, seed, N):
    m = len(nominal)
    u = uniform(seed, S_THETA, N * m).reshape(N, m)
    return np.asarray(nominal)[None, :] * (lo + (hi - lo) * u)


def lotka_volterra(N=1024, seed=0):
    nominal = np.array([1.5, 1.0, 3.0, 1.0])
    return Workload("lotka_volterra", "lotka_volterra", "tsit5", np.float64, N, 2, 4, False,
                    _scaled(nominal, 0.9, 1.1, seed, N), np.ones((N, 2)), 0.0, 10.0, 1e-6, 1e-8,
                    seed, target_kind="nominal_solve", nominal_theta=nominal)


def lorenz63(N=65536, seed=1):
    nominal = np.array([10.0, 28.0, 8.0 / 3.0])
    y0 = 1.0 + 0.1 * normal(seed, S_Y0, N * 3).reshape(N, 3)
    target = normal(seed, S_TARGET, N * 3).reshape(N, 3)
    return Workload("lorenz63", "lorenz63", "tsit5", np.float64, N, 3, 3, False,
                    _scaled(nominal, 0.95, 1.05, seed, N), y0, 0.0, 1.0, 1e-8, 1e-10, seed,
                    target=target)


def glorot_mlp(seed: int, stream: int) -> np.ndarray:
    """Glorot-uniform weights U(+-sqrt(6/(fan_in+fan_out))), zero biases, in the MLP layout."""
    th = np.zeros(MLP_M)
    u = uniform(seed, stream, MLP_M)
    for name, off, shape in MLP_LAYOUT:
        if name.startswith("W"):
            fan_out, fan_in = shape
            lim = np.sqrt(6.0 / (fan_in + fan_out))
            n = fan_out * fan_in
            th[off:off + n] = -lim + 2.0 * lim * u[off:off + n]
    return th


def mlp(N=16384, seed=2):
    student = glorot_mlp(seed, S_STUDENT)
    teacher = glorot_mlp(seed + 1, S_TEACHER)
    y0 = normal(seed, S_Y0, N * 4).reshape(N, 4)
    return Workload("mlp", "mlp", "tsit5", np.float32, N, 4, MLP_M, True, student, y0, 0.0, 1.0,
                    1e-5, 1e-6, seed, target_kind="teacher_solve", nominal_theta=teacher,
                    loss_scale=1.0 / (4.0 * N))


def robertson(N=65536, seed=3):
    nominal = np.array([0.04, 3e7, 1e4])
    u = uniform(seed, S_THETA, N * 3).reshape(N, 3)
    theta = nominal[None, :] * np.exp(np.log(0.8) + (np.log(1.25) - np.log(0.8)) * u)
    y0 = np.tile(np.array([1.0, 0.0, 0.0]), (N, 1))
    return Workload("robertson", "robertson", "ros34pw2", np.float64, N, 3, 3, False, theta, y0,
                    0.0, 1e4, 1e-6, 1e-10, seed, target_kind="nominal_solve",
                    nominal_theta=nominal)


def _shell_points(seed, stream, N, rmin=0.5, rmax=2.0):
    """Points uniform in volume in the shell rmin <= r <= rmax, isotropic direction."""
    u = uniform(seed, stream, 3 * N).reshape(N, 3)
    r = (rmin ** 3 + u[:, 0] * (rmax ** 3 - rmin ** 3)) ** (1.0 / 3.0)
    cth = 2.0 * u[:, 1] - 1.0
    sth = np.sqrt(np.maximum(0.0, 1.0 - cth * cth))
    ph = 2.0 * np.pi * u[:, 2]
    return np.stack([r * sth * np.cos(ph), r * sth * np.sin(ph), r * cth], axis=1)


def nfw_mn(N=1 << 20, seed=4, dtype=np.float64, theta_shared=False):
    nominal = np.array([1.0, 1.0, 0.1, 0.3, 0.03])
    x = _shell_points(seed, S_Y0, N)
    v = 0.3 * normal(seed, S_VEL, 3 * N).reshape(N, 3)
    y0 = np.concatenate([x, v], axis=1)
    target = np.zeros((N, 6))
    target[:, :3] = _shell_points(seed, S_TARGET, N)
    theta = nominal.copy() if theta_shared else _scaled(nominal, 0.9, 1.1, seed, N)
    if dtype == np.float32:
        rtol, atol = 1e-5, 1e-6
    else:
        rtol, atol = 1e-8, 1e-10
    mask = np.array([1, 1, 1, 0, 0, 0], np.float64)
    return Workload("nfw_mn" + ("_f32" if dtype == np.float32 else ""), "nfw_mn", "tsit5", dtype,
                    N, 6, 5, theta_shared, theta, y0, 0.0, 20.0, rtol, atol, seed, target=target,
                    loss_mask=mask)


HIRES_K = np.array([1.71, 0.43, 8.32, 0.0007, 8.75, 10.03, 0.035, 1.12, 1.745, 280.0, 0.69, 1.81])


def hires(N=65536, seed=6):
    """HIRES (8 components, stiff), rate constants shared at their nominal values; the ensemble
    varies the initial state (the gradient of interest is with respect to y0):
    y0 = (u1, 0, 0, 0, 0, 0, 0, 0.0057 u8), u ~ U(0.8, 1.2); t in [0, 321.8122];
    Rosenbrock23, rtol 1e-6, atol 1e-10.  Loss targets: the final state of the nominal y0."""
    u = uniform(seed, S_Y0, 2 * N).reshape(N, 2)
    y0 = np.zeros((N, 8))
    y0[:, 0] = 0.8 + 0.4 * u[:, 0]
    y0[:, 7] = 0.0057 * (0.8 + 0.4 * u[:, 1])
    nominal_y0 = np.array([1.0, 0, 0, 0, 0, 0, 0, 0.0057])
    w = Workload("hires", "hires", "rosenbrock23", np.float64, N, 8, 12, True, HIRES_K.copy(), y0,
                 0.0, 321.8122, 1e-6, 1e-10, seed, target_kind="nominal_y0",
                 nominal_theta=HIRES_K.copy())
    w.notes["nominal_y0"] = nominal_y0
    return w


LOG_HALO_RC = 0.2


def log_halo_vcirc(r, vc=1.0):
    """Circular speed v_c r / sqrt(R_c^2 + r^2) of the logarithmic halo at radius r (in the plane;
    used as the velocity scale at any position)."""
    return vc * r / np.sqrt(LOG_HALO_RC ** 2 + r * r)


def log_halo_t1():
    """3.7 circular periods 2 pi r_m / v_circ(r_m) at the median radius r_m of the shell
    0.5 <= r <= 2 (uniform in volume): the pages' median of 3.7 orbital periods per orbit."""
    rm = ((0.5 ** 3 + 2.0 ** 3) / 2.0) ** (1.0 / 3.0)
    return 3.7 * 2.0 * np.pi * rm / log_halo_vcirc(rm)


def log_halo(N=1 << 20, seed=5, dtype=np.float64):
    """Stars in the flattened logarithmic halo, theta = (v_c, q) = (1, 0.7) shared, R_c = 0.2.
    Positions uniform in volume in 0.5 <= r <= 2 with an isotropic direction; velocity
    v_circ(r) (eta t + xi r_hat), t a unit vector perpendicular to r_hat at a uniform angle (orbits
    in and out of the plane), eta ~ U(0.05, 1) (nearly radial to near-circular), xi ~ U(-0.2, 0.2).
    rtol = atol = 3.16e-7; t in [0, 3.7 circular periods at the median radius]."""
    x = _shell_points(seed, S_Y0, N)
    u = uniform(seed, S_VEL, 3 * N).reshape(N, 3)
    r = np.linalg.norm(x, axis=1)
    rh = x / r[:, None]
    # an orthonormal pair perpendicular to r_hat: e1 = normalise(z_hat x r_hat) (or x_hat when
    # r_hat is along z), e2 = r_hat x e1
    e1 = np.cross(np.array([0.0, 0.0, 1.0])[None, :], rh)
    n1 = np.linalg.norm(e1, axis=1)
    bad = n1 < 1e-12
    e1[bad] = np.array([1.0, 0.0, 0.0])
    n1[bad] = 1.0
    e1 /= n1[:, None]
    e2 = np.cross(rh, e1)
    psi = 2.0 * np.pi * u[:, 0]
    t = np.cos(psi)[:, None] * e1 + np.sin(psi)[:, None] * e2
    eta = 0.05 + 0.95 * u[:, 1]
    xi = -0.2 + 0.4 * u[:, 2]
    v = log_halo_vcirc(r)[:, None] * (eta[:, None] * t + xi[:, None] * rh)
    y0 = np.concatenate([x, v], axis=1).astype(dtype)
    theta = np.array([1.0, 0.7], dtype)
    target = np.zeros((N, 6))
    target[:, :3] = _shell_points(seed, S_TARGET, N)
    mask = np.array([1, 1, 1, 0, 0, 0], np.float64)
    return Workload("log_halo" + ("_f32" if dtype == np.float32 else ""), "log_halo", "tsit5",
                    dtype, N, 6, 2, True, theta, y0, 0.0, float(log_halo_t1()), 3.16e-7, 3.16e-7,
                    seed, target=target, loss_mask=mask)


def by_name(name: str, N: Optional[int] = None, **kw) -> Workload:
    table = {"lotka_volterra": lotka_volterra, "lorenz63": lorenz63, "mlp": mlp,
             "robertson": robertson, "nfw_mn": nfw_mn, "log_halo": log_halo, "hires": hires}
    if name == "nfw_mn_f32":
        return nfw_mn(N=N if N else 1 << 20, dtype=np.float32, **kw)
    for suffix, method in (("_vern7", "vern7"), ("_rb23", "rosenbrock23"),
                           ("_ros34pw2", "ros34pw2")):
        if name.endswith(suffix):
            # the same ensemble integrated with another method of the same kind
            w = by_name(name[:-len(suffix)], N=N, **kw)
            w.name, w.method = name, method
            return w
    fn = table[name]
    return fn(N=N, **kw) if N else fn(**kw)


def subset(w: Workload, idx) -> Workload:
    """The same ensemble restricted to trajectories idx (the draws are per-index, so a subset is
    exactly the corresponding rows of the full ensemble)."""
    import copy
    s = copy.copy(w)
    idx = np.asarray(idx)
    s.N = len(idx)
    s.y0 = w.y0[idx]
    if not w.theta_shared:
        s.theta = w.theta[idx]
    if w.target is not None:
        s.target = w.target[idx]
    if w.loss_scale != 1.0 and w.name == "mlp":
        s.loss_scale = w.loss_scale  # the scale stays that of the full ensemble
    return s


def loss_cotangent(w: Workload, y1: np.ndarray, target: np.ndarray) -> np.ndarray:
    """dL/dy1 of L = loss_scale * sum_k |mask (y1_k - target_k)|^2 (the caller's loss, [GS] §2.2:
    a scalar built from the final states; the library only sees this cotangent)."""
    g = 2.0 * w.loss_scale * (np.asarray(y1, np.float64) - np.asarray(target, np.float64))
    if w.loss_mask is not None:
        g = g * w.loss_mask[None, :]
    return g
