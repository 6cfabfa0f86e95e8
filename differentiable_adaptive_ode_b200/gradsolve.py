"""Thin Python binding of the C ABI in include/gradsolve_b200.h (ctypes; argument marshalling only).

Every computation runs in libgradsolve_b200.so on the GPU; this module only turns torch tensors
into device pointers and the current CUDA stream into a cudaStream_t.  There is no fallback: if
the library is missing or does not load, every call raises.

The names follow the C entry points: gs_solve_forward, gs_solve_record, gs_replay_grad,
gs_record_info, gs_record_export, gs_record_import.  The method is the record-and-replay discrete
adjoint of "gradsolve: fast exact gradients for ODE ensembles on GPUs" (§3).
"""
import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgradsolve_b200.so")
CHECKED_LIB_PATH = os.path.join(PKG, "libgradsolve_b200_checked.so")
if os.environ.get("GRADSOLVE_B200_CHECKED") == "1":   # the bounds-checked build of the library
    LIB_PATH = CHECKED_LIB_PATH

GS_OK, GS_ERR_INVALID_ARG, GS_ERR_CUDA, GS_ERR_CAPACITY, GS_ERR_UNSUPPORTED, GS_ERR_TRAJ_FAILED = range(6)
GS_F64, GS_F32 = 0, 1
GS_TSIT5, GS_ROS34PW2, GS_VERN7, GS_ROSENBROCK23 = 0, 1, 2, 3
FIELDS = {"lotka_volterra": 0, "lorenz63": 1, "mlp": 2, "robertson": 3, "nfw_mn": 4, "linear3": 5,
          "log_halo": 6, "hires": 7}
# (d, m) of each field, as the library checks them
FIELD_DIMS = {"lotka_volterra": (2, 4), "lorenz63": (3, 3), "mlp": (4, 1348), "robertson": (3, 3),
              "nfw_mn": (6, 5), "linear3": (3, 9), "log_halo": (6, 2), "hires": (8, 12)}
METHODS = {"tsit5": GS_TSIT5, "ros34pw2": GS_ROS34PW2, "vern7": GS_VERN7,
           "rosenbrock23": GS_ROSENBROCK23}
STATUS_NAMES = {0: "GS_OK", 1: "GS_ERR_INVALID_ARG", 2: "GS_ERR_CUDA", 3: "GS_ERR_CAPACITY",
                4: "GS_ERR_UNSUPPORTED", 5: "GS_ERR_TRAJ_FAILED"}

# every entry point declared in include/gradsolve_b200.h
EXPORTS = ("gs_solve_forward", "gs_solve_forward_sens", "gs_solve_record", "gs_replay_grad",
           "gs_replay_forward", "gs_replay_grad_noalloc", "gs_replay_outputs",
           "gs_replay_grad_outputs", "gs_record_info", "gs_record_export", "gs_record_import",
           "gs_record_destroy", "gs_memory_trim", "gs_last_error", "gs_version",
           "gs_checked_violations")


class GsSystem(C.Structure):
    _fields_ = [("field", C.c_int32), ("method", C.c_int32), ("dtype", C.c_int32),
                ("d", C.c_int32), ("m", C.c_int32), ("theta_shared", C.c_int32)]


class GsOptions(C.Structure):
    _fields_ = [("max_attempts", C.c_int64), ("record_capacity_steps", C.c_int64),
                ("start_order", C.c_void_p)]


class GsRecordInfo(C.Structure):
    _fields_ = [("N", C.c_int64), ("total_steps", C.c_int64), ("max_steps", C.c_int32),
                ("chunk_steps", C.c_int32), ("entry_reals", C.c_int32), ("dtype", C.c_int32),
                ("nchunks", C.c_int64), ("pool_bytes", C.c_int64), ("nsteps", C.c_void_p),
                ("status", C.c_void_p), ("offsets", C.c_void_p), ("chunk_offsets", C.c_void_p),
                ("chunk_table", C.c_void_p), ("pool", C.c_void_p), ("solve_ms", C.c_double),
                ("order", C.c_void_p)]


class GradsolveError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("%s: %s" % (STATUS_NAMES.get(code, code), msg))
        self.code = code


_lib = None


def lib():
    """The loaded CUDA library (raises if it is missing: there is no CPU path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libgradsolve_b200.so is not built (run "
                               "python -m differentiable_adaptive_ode_b200.build)")
        L = C.CDLL(LIB_PATH)
        vp, i64, d = C.c_void_p, C.c_int64, C.c_double
        P = C.POINTER
        L.gs_solve_forward.argtypes = [P(GsSystem), P(GsOptions), i64, vp, vp, d, d, d, d, vp, vp,
                                       vp, vp, vp]
        L.gs_solve_forward_sens.argtypes = [P(GsSystem), P(GsOptions), i64, vp, vp, vp, d, d, d,
                                            d, vp, vp, vp, vp, vp, vp]
        L.gs_solve_record.argtypes = [P(GsSystem), P(GsOptions), i64, vp, vp, d, d, d, d,
                                      P(vp), vp, vp, vp]
        L.gs_replay_grad.argtypes = [vp, vp, vp, vp, vp, vp]
        L.gs_replay_forward.argtypes = [vp, vp, vp, vp, vp]
        L.gs_replay_grad_noalloc.argtypes = [vp, vp, vp, vp, vp, vp]
        pd = C.POINTER(C.c_double)
        L.gs_replay_outputs.argtypes = [vp, vp, vp, C.c_int32, pd, vp, vp]
        L.gs_replay_grad_outputs.argtypes = [vp, vp, C.c_int32, pd, vp, vp, vp, vp, vp]
        L.gs_record_info.argtypes = [vp, P(GsRecordInfo)]
        L.gs_checked_violations.argtypes = [P(C.c_int64)]
        L.gs_checked_violations.restype = C.c_int
        L.gs_record_export.argtypes = [vp, vp, vp, vp, vp, vp]
        L.gs_record_import.argtypes = [P(GsSystem), i64, vp, vp, vp, vp, P(vp), vp]
        L.gs_record_destroy.argtypes = [vp]
        L.gs_record_destroy.restype = None
        L.gs_memory_trim.argtypes = [i64]
        L.gs_memory_trim.restype = C.c_int
        L.gs_last_error.restype = C.c_char_p
        L.gs_version.restype = C.c_char_p
        for name in ("gs_solve_forward", "gs_solve_forward_sens", "gs_solve_record", "gs_replay_grad", "gs_replay_forward",
                     "gs_replay_grad_noalloc", "gs_replay_outputs", "gs_replay_grad_outputs",
                     "gs_record_info",
                     "gs_record_export", "gs_record_import"):
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def last_error():
    return lib().gs_last_error().decode()


def _check(code, allow=()):
    if code != GS_OK and code not in allow:
        raise GradsolveError(code, last_error())
    return code


def system(field, method=None, dtype="f64", theta_shared=False):
    d, m = FIELD_DIMS[field]
    if method is None:
        method = "ros34pw2" if field in ("robertson", "hires") else "tsit5"
    return GsSystem(FIELDS[field], METHODS[method], GS_F64 if dtype in ("f64", "float64") else GS_F32,
                    d, m, int(bool(theta_shared)))


def options(max_attempts=0, record_capacity_steps=0, start_order=None):
    """start_order: optional int32 device tensor [N], the order in which trajectories are started
    (scheduling only).  The tensor must stay alive while the call's work runs."""
    return GsOptions(max_attempts, record_capacity_steps,
                     None if start_order is None else _ptr(start_order).value)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device (got %s)" % t.device)
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def gs_solve_forward(sys, N, theta, y0, t0, t1, rtol, atol, y1, nsteps=None, nrejected=None,
                     status=None, opts=None, stream=None):
    """Forward-only ensemble solve; fills y1 [N, d] (and the optional int32 arrays)."""
    opts = opts or options()
    _check(lib().gs_solve_forward(C.byref(sys), C.byref(opts), N, _ptr(theta), _ptr(y0), t0, t1,
                                  rtol, atol, _ptr(y1), _ptr(nsteps), _ptr(nrejected),
                                  _ptr(status), _stream(stream)))


def gs_solve_forward_sens(sys, N, theta, y0, t0, t1, rtol, atol, y1, S1, S0=None, nsteps=None,
                          nrejected=None, status=None, opts=None, stream=None):
    """Forward solve with the sensitivities S = dy/dtheta [N, d, m] integrated alongside (step
    control on y alone); S0 [N, d, m] optional (zero start)."""
    opts = opts or options()
    _check(lib().gs_solve_forward_sens(C.byref(sys), C.byref(opts), N, _ptr(theta), _ptr(y0),
                                       _ptr(S0), t0, t1, rtol, atol, _ptr(y1), _ptr(S1),
                                       _ptr(nsteps), _ptr(nrejected), _ptr(status),
                                       _stream(stream)))


class Record:
    """Owner of a library record (gs_record*); freed with gs_record_destroy."""

    def __init__(self, handle=None):
        self.handle = C.c_void_p(handle)

    def info(self):
        return gs_record_info(self)

    def order(self):
        """The record's longest-first trajectory order as an int32 CUDA tensor that views the
        library-owned array (valid until the record is made again or freed), or None; usable as
        options(start_order=...) for later solves of the same ensemble."""
        import torch
        inf = self.info()
        if not inf.order or inf.N == 0:
            return None

        class _View:
            def __init__(self, ptr, n):
                self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i4",
                                                 "data": (ptr, False), "version": 3}

        return torch.as_tensor(_View(inf.order, int(inf.N)), device="cuda")

    def close(self):
        if self.handle and self.handle.value:
            lib().gs_record_destroy(self.handle)
            self.handle = C.c_void_p(None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gs_solve_record(sys, N, theta, y0, t0, t1, rtol, atol, y1, status=None, rec=None, opts=None,
                    stream=None, allow_failed=False):
    """Record pass: adaptive solve keeping (t_n, h_n, y_n) of accepted steps.  Reuses `rec`'s
    storage when given.  Returns the Record (and raises on GS_ERR_TRAJ_FAILED unless allowed)."""
    opts = opts or options()
    rec = rec if rec is not None else Record()
    code = lib().gs_solve_record(C.byref(sys), C.byref(opts), N, _ptr(theta), _ptr(y0), t0, t1,
                                 rtol, atol, C.byref(rec.handle), _ptr(y1), _ptr(status),
                                 _stream(stream))
    _check(code, allow=(GS_ERR_TRAJ_FAILED,) if allow_failed else ())
    return rec


def gs_replay_grad(rec, theta, dL_dy1, dL_dtheta=None, dL_dy0=None, stream=None):
    """Replay gradient over the recorded mesh: fills dL_dtheta ([N, m] or [m]) and/or dL_dy0."""
    _check(lib().gs_replay_grad(rec.handle, _ptr(theta), _ptr(dL_dy1), _ptr(dL_dtheta),
                                _ptr(dL_dy0), _stream(stream)))


def gs_replay_grad_noalloc(rec, theta, dL_dy1, dL_dtheta=None, dL_dy0=None, stream=None):
    """gs_replay_grad without any device allocation: for callers that may not allocate when they
    ask for a gradient (e.g. inside CUDA-graph capture); its scratch is a fixed 8 MiB array in the
    library, shared by all calls, so calls must not overlap on the GPU."""
    _check(lib().gs_replay_grad_noalloc(rec.handle, _ptr(theta), _ptr(dL_dy1), _ptr(dL_dtheta),
                                        _ptr(dL_dy0), _stream(stream)))


def gs_replay_forward(rec, theta, y0, y1=None, stream=None):
    """Forward replay over the recorded mesh at theta: refreshes the stored states, fills y1."""
    _check(lib().gs_replay_forward(rec.handle, _ptr(theta), _ptr(y0), _ptr(y1), _stream(stream)))


def _times(tau):
    arr = (C.c_double * len(tau))(*[float(t) for t in tau])
    return len(tau), arr


def gs_replay_outputs(rec, theta, y0, tau, y_out, stream=None):
    """States at the requested times tau (host sequence, ascending) into y_out [N, J, d]."""
    J, arr = _times(tau)
    _check(lib().gs_replay_outputs(rec.handle, _ptr(theta), _ptr(y0), J, arr, _ptr(y_out),
                                   _stream(stream)))


def gs_replay_grad_outputs(rec, theta, tau, dL_dyout, dL_dy1=None, dL_dtheta=None, dL_dy0=None,
                           stream=None):
    """Gradient of a loss on the outputs at requested times (dL_dyout [N, J, d]) and optionally
    on the final state (dL_dy1)."""
    J, arr = _times(tau)
    _check(lib().gs_replay_grad_outputs(rec.handle, _ptr(theta), J, arr, _ptr(dL_dyout),
                                        _ptr(dL_dy1), _ptr(dL_dtheta), _ptr(dL_dy0),
                                        _stream(stream)))


def gs_record_info(rec):
    info = GsRecordInfo()
    _check(lib().gs_record_info(rec.handle, C.byref(info)))
    return info


def gs_record_export(rec, T=None, H=None, Y=None, offsets=None, stream=None):
    _check(lib().gs_record_export(rec.handle, _ptr(T), _ptr(H), _ptr(Y), _ptr(offsets),
                                  _stream(stream)))


def gs_record_import(sys, N, nsteps, T, H, Y, stream=None):
    rec = Record()
    _check(lib().gs_record_import(C.byref(sys), N, _ptr(nsteps), _ptr(T), _ptr(H), _ptr(Y),
                                  C.byref(rec.handle), _stream(stream)))
    return rec


def checked_violations():
    """Out-of-range record accesses counted by the checked build since the last call."""
    v = C.c_int64(0)
    _check(lib().gs_checked_violations(C.byref(v)))
    return v.value


def gs_memory_trim(keep_bytes=0):
    """Hand the record storage the device's pool keeps beyond keep_bytes back to the device."""
    _check(lib().gs_memory_trim(int(keep_bytes)))


def version():
    return lib().gs_version().decode()
