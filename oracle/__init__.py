"""float64 CPU oracle for the selective scan (S6) forward, its backward and the recurrent step.

TEST INFRASTRUCTURE. Only tests/, the package smoke check and the benchmark's
CPU-baseline leg may import this package. It shares no code with the CUDA path.

The arithmetic lives in ``ssm_oracle.c`` (one sequential loop over time per
channel, in double); this module only marshals numpy arrays into it.
Storage dtypes: ``"f32"`` (numpy float32) or ``"bf16"`` (numpy uint16 holding
bfloat16 bit patterns). Results come back as float64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

DELTA_SOFTPLUS = 1
EXACT_ZOH = 2


def _open(path):
    lib = ctypes.CDLL(path)
    vp, i64, c_int, c_uint = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint
    lib.oracle_scan_f64.argtypes = [i64, i64, i64, i64, c_int, c_uint] + [vp] * 11 + [c_int]
    lib.oracle_scan_f64.restype = c_int
    lib.oracle_scan_conv_f64.argtypes = [i64, i64, i64, i64, c_int, c_uint] + [vp] * 14 + [c_int]
    lib.oracle_scan_conv_f64.restype = c_int
    lib.oracle_step_f64.argtypes = [i64, i64, i64, c_int, c_uint] + [vp] * 10 + [c_int]
    lib.oracle_step_f64.restype = c_int
    lib.oracle_step_conv_f64.argtypes = [i64, i64, i64, c_int, c_uint] + [vp] * 13 + [c_int]
    lib.oracle_step_conv_f64.restype = c_int
    lib.oracle_scan_bwd_f64.argtypes = [i64, i64, i64, i64, c_int, c_uint] + [vp] * 20
    lib.oracle_scan_bwd_f64.restype = c_int
    lib.oracle_scan_bwd_conv_f64.argtypes = [i64, i64, i64, i64, c_int, c_uint] + [vp] * 26
    lib.oracle_scan_bwd_conv_f64.restype = c_int
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _tok(a, dtype, shape, name):
    """Check a token-type array (x, dt, z, B, C) and return it contiguous."""
    want = np.float32 if dtype == "f32" else np.uint16
    a = np.ascontiguousarray(a)
    if a.dtype != want or a.shape != tuple(shape):
        raise ValueError(f"{name}: expected {want.__name__}{tuple(shape)}, got {a.dtype}{a.shape}")
    return a


def _f32(a, shape, name):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.float32)
    if a.shape != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {a.shape}")
    return a


def default_threads():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


class Oracle:
    """The oracle bound to one compiled library (the default build, or a test's variant)."""

    def __init__(self, path=None):
        self.path = path or _build.build()
        self.lib = _open(self.path)

    def scan(self, x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, dtype="f32",
             delta_softplus=True, exact_zoh=False, nthreads=None, conv_w=None, conv_b=None,
             conv_x0=None):
        return _scan(self.lib, x, dt, A, B, C, D, z, dt_bias, h0, dtype, delta_softplus,
                     exact_zoh, nthreads, conv_w, conv_b, conv_x0)

    def scan_bwd(self, x, dt, A, B, C, dy, D=None, z=None, dt_bias=None, h0=None, dh_last=None,
                 dtype="f32", delta_softplus=True, exact_zoh=False, conv_w=None, conv_b=None, conv_x0=None):
        return _scan_bwd(self.lib, x, dt, A, B, C, dy, D, z, dt_bias, h0, dh_last, dtype, delta_softplus,
                         exact_zoh, conv_w, conv_b, conv_x0)

    def step(self, x, dt, A, B, C, h, D=None, z=None, dt_bias=None, dtype="f32",
             delta_softplus=True, exact_zoh=False, nthreads=None, conv_w=None, conv_b=None,
             conv_state=None):
        return _step(self.lib, x, dt, A, B, C, h, D, z, dt_bias, dtype, delta_softplus,
                     exact_zoh, nthreads, conv_w, conv_b, conv_state)


_default = None


def default():
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def scan(*args, **kw):
    """Selective scan with the default oracle build; see ``_scan``."""
    return default().scan(*args, **kw)


def step(*args, **kw):
    """One decode step with the default oracle build; see ``_step``."""
    return default().step(*args, **kw)


def scan_bwd(*args, **kw):
    """Backward of the scan with the default oracle build; see ``_scan_bwd``."""
    return default().scan_bwd(*args, **kw)


def _scan(lib, x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, dtype="f32",
          delta_softplus=True, exact_zoh=False, nthreads=None, conv_w=None, conv_b=None,
          conv_x0=None):
    """Selective scan over a whole sequence.

    x, dt, z: [Bsz, L, Dm]; B, C: [Bsz, L, N]; A: [Dm, N]; D, dt_bias: [Dm];
    h0: [Bsz, Dm, N] (float32) or None for a zero initial state.
    conv_w: [Dm, 4] (float32) puts the block's causal convolution and SiLU in front of
    the SSM (its input becomes silu(conv_b + sum_k conv_w[:, k] x_{t-3+k})); conv_b: [Dm]
    or None; conv_x0: [Bsz, 3, Dm] tokens before t = 0 (x's storage type) or None (zeros).
    Returns (y [Bsz, L, Dm] float64, h_last [Bsz, Dm, N] float64).
    """
    Bsz, L, Dm = np.shape(x)
    N = np.shape(A)[1]
    x = _tok(x, dtype, (Bsz, L, Dm), "x")
    dt = _tok(dt, dtype, (Bsz, L, Dm), "dt")
    z = None if z is None else _tok(z, dtype, (Bsz, L, Dm), "z")
    B = _tok(B, dtype, (Bsz, L, N), "B")
    C = _tok(C, dtype, (Bsz, L, N), "C")
    A = _f32(A, (Dm, N), "A")
    D = _f32(D, (Dm,), "D")
    dt_bias = _f32(dt_bias, (Dm,), "dt_bias")
    h0 = _f32(h0, (Bsz, Dm, N), "h0")
    y = np.empty((Bsz, L, Dm), dtype=np.float64)
    h_last = np.empty((Bsz, Dm, N), dtype=np.float64)
    flags = (DELTA_SOFTPLUS if delta_softplus else 0) | (EXACT_ZOH if exact_zoh else 0)
    nt = default_threads() if nthreads is None else nthreads
    common = (Bsz, L, Dm, N, 0 if dtype == "f32" else 1, flags, _ptr(x), _ptr(dt), _ptr(z), _ptr(B),
              _ptr(C), _ptr(A), _ptr(D), _ptr(dt_bias), _ptr(h0))
    if conv_w is None:
        if conv_b is not None or conv_x0 is not None:
            raise ValueError("conv_b and conv_x0 need conv_w")
        rc = lib.oracle_scan_f64(*common, _ptr(y), _ptr(h_last), nt)
    else:
        conv_w = _f32(conv_w, (Dm, 4), "conv_w")
        conv_b = _f32(conv_b, (Dm,), "conv_b")
        conv_x0 = None if conv_x0 is None else _tok(conv_x0, dtype, (Bsz, 3, Dm), "conv_x0")
        rc = lib.oracle_scan_conv_f64(*common, _ptr(conv_w), _ptr(conv_b), _ptr(conv_x0), _ptr(y),
                                      _ptr(h_last), nt)
    if rc != 0:
        raise ValueError("oracle scan rejected its arguments")
    return y, h_last


def _step(lib, x, dt, A, B, C, h, D=None, z=None, dt_bias=None, dtype="f32",
          delta_softplus=True, exact_zoh=False, nthreads=None, conv_w=None, conv_b=None,
          conv_state=None):
    """One recurrent decode step. x, dt, z: [Bsz, Dm]; B, C: [Bsz, N];
    h: float64 [Bsz, Dm, N], updated in place. Returns y [Bsz, Dm] float64.
    conv_w [Dm, 4] (float32) puts the block's causal convolution and SiLU in front: the
    three previous tokens come from conv_state [Bsz, 3, Dm] (x's storage type, oldest
    first), which is then shifted in place to end with x; conv_b [Dm] or None."""
    Bsz, Dm = np.shape(x)
    N = np.shape(A)[1]
    x = _tok(x, dtype, (Bsz, Dm), "x")
    dt = _tok(dt, dtype, (Bsz, Dm), "dt")
    z = None if z is None else _tok(z, dtype, (Bsz, Dm), "z")
    B = _tok(B, dtype, (Bsz, N), "B")
    C = _tok(C, dtype, (Bsz, N), "C")
    A = _f32(A, (Dm, N), "A")
    D = _f32(D, (Dm,), "D")
    dt_bias = _f32(dt_bias, (Dm,), "dt_bias")
    if not (isinstance(h, np.ndarray) and h.dtype == np.float64 and h.shape == (Bsz, Dm, N)
            and h.flags.c_contiguous):
        raise ValueError("h must be a C-contiguous float64 array of shape [Bsz, Dm, N]")
    y = np.empty((Bsz, Dm), dtype=np.float64)
    flags = (DELTA_SOFTPLUS if delta_softplus else 0) | (EXACT_ZOH if exact_zoh else 0)
    nt = default_threads() if nthreads is None else nthreads
    common = (Bsz, Dm, N, 0 if dtype == "f32" else 1, flags, _ptr(x), _ptr(dt), _ptr(z), _ptr(B), _ptr(C),
              _ptr(A), _ptr(D), _ptr(dt_bias))
    if conv_w is None:
        if conv_b is not None or conv_state is not None:
            raise ValueError("conv_b and conv_state need conv_w")
        rc = lib.oracle_step_f64(*common, _ptr(h), _ptr(y), nt)
    else:
        want = np.float32 if dtype == "f32" else np.uint16
        if not (isinstance(conv_state, np.ndarray) and conv_state.dtype == want
                and conv_state.shape == (Bsz, 3, Dm) and conv_state.flags.c_contiguous):
            raise ValueError(f"conv_state must be a C-contiguous {want.__name__} array of shape [Bsz, 3, Dm]")
        conv_w = _f32(conv_w, (Dm, 4), "conv_w")
        conv_b = _f32(conv_b, (Dm,), "conv_b")
        rc = lib.oracle_step_conv_f64(*common, _ptr(conv_w), _ptr(conv_b), _ptr(conv_state), _ptr(h),
                                      _ptr(y), nt)
        if rc == 0:  # the window moves by one token (bookkeeping, no arithmetic)
            conv_state[:, :2] = conv_state[:, 1:].copy()
            conv_state[:, 2] = x
    if rc != 0:
        raise ValueError("oracle step rejected its arguments")
    return y


def _scan_bwd(lib, x, dt, A, B, C, dy, D=None, z=None, dt_bias=None, h0=None, dh_last=None, dtype="f32",
              delta_softplus=True, exact_zoh=False, conv_w=None, conv_b=None, conv_x0=None):
    """Gradients of the scan given dy = dL/dy ([Bsz, L, Dm], token storage type) and
    dh_last = dL/dh_L ([Bsz, Dm, N] float64 or None); exact_zoh and the short convolution
    (conv_w, conv_b, conv_x0) as for ``_scan``. Returns a dict of float64 arrays: dx, ddt,
    dz (None without z) [Bsz, L, Dm]; dB, dC [Bsz, L, N]; dA [Dm, N]; dD, ddt_bias [Dm];
    dh0 [Bsz, Dm, N]; with the convolution also dconv_w [Dm, 4], dconv_b [Dm] and
    dconv_x0 [Bsz, 3, Dm] (dx is then the gradient of the raw tokens before it)."""
    Bsz, L, Dm = np.shape(x)
    N = np.shape(A)[1]
    x = _tok(x, dtype, (Bsz, L, Dm), "x")
    dt = _tok(dt, dtype, (Bsz, L, Dm), "dt")
    z = None if z is None else _tok(z, dtype, (Bsz, L, Dm), "z")
    B = _tok(B, dtype, (Bsz, L, N), "B")
    C = _tok(C, dtype, (Bsz, L, N), "C")
    dy = _tok(dy, dtype, (Bsz, L, Dm), "dy")
    A = _f32(A, (Dm, N), "A")
    D = _f32(D, (Dm,), "D")
    dt_bias = _f32(dt_bias, (Dm,), "dt_bias")
    h0 = _f32(h0, (Bsz, Dm, N), "h0")
    if dh_last is not None:
        dh_last = np.ascontiguousarray(dh_last, dtype=np.float64)
        if dh_last.shape != (Bsz, Dm, N):
            raise ValueError("dh_last must have shape [Bsz, Dm, N]")
    out = dict(dx=np.empty((Bsz, L, Dm)), ddt=np.empty((Bsz, L, Dm)),
               dz=None if z is None else np.empty((Bsz, L, Dm)), dB=np.empty((Bsz, L, N)),
               dC=np.empty((Bsz, L, N)), dA=np.empty((Dm, N)), dD=np.empty(Dm), ddt_bias=np.empty(Dm),
               dh0=np.empty((Bsz, Dm, N)))
    if conv_w is None:
        if conv_b is not None or conv_x0 is not None:
            raise ValueError("conv_b and conv_x0 need conv_w")
    else:
        conv_w = _f32(conv_w, (Dm, 4), "conv_w")
        conv_b = _f32(conv_b, (Dm,), "conv_b")
        conv_x0 = None if conv_x0 is None else _tok(conv_x0, dtype, (Bsz, 3, Dm), "conv_x0")
        out.update(dconv_w=np.empty((Dm, 4)), dconv_b=np.empty(Dm), dconv_x0=np.empty((Bsz, 3, Dm)))
    flags = (DELTA_SOFTPLUS if delta_softplus else 0) | (EXACT_ZOH if exact_zoh else 0)
    rc = lib.oracle_scan_bwd_conv_f64(Bsz, L, Dm, N, 0 if dtype == "f32" else 1, flags,
                                      _ptr(x), _ptr(dt), _ptr(z), _ptr(B), _ptr(C), _ptr(A), _ptr(D), _ptr(dt_bias),
                                      _ptr(h0), _ptr(conv_w), _ptr(conv_b), _ptr(conv_x0), _ptr(dy), _ptr(dh_last),
                                      _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dz"]), _ptr(out["dB"]),
                                      _ptr(out["dC"]), _ptr(out["dA"]), _ptr(out["dD"]), _ptr(out["ddt_bias"]),
                                      _ptr(out["dh0"]), _ptr(out.get("dconv_w")), _ptr(out.get("dconv_b")),
                                      _ptr(out.get("dconv_x0")))
    if rc != 0:
        raise ValueError("oracle_scan_bwd_conv_f64 rejected its arguments")
    return out
