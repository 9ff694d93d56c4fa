"""B200-native selective state space (S6) scan: Python binding of libssmscan.so.

Every step of the computation runs in the library's CUDA kernels; this module
only checks tensors and passes their device pointers and the current CUDA stream
through the C ABI (include/ssm_scan.h). PyTorch provides device memory and
streams. There is no CPU fallback: without the built library, or without a CUDA
device, the calls raise.

    y = scan_fwd(x, dt, A, B, C, D, z, dt_bias)              # [B, L, D]
    y, h_last = scan_fwd(..., return_last_state=True)         # h_last [B, D, N] fp32
    y = step(x_t, dt_t, A, B_t, C_t, h, D, z_t, dt_bias)     # h [B, D, N] updated in place
    y = scan_fwd_host(x, dt, A, B, C, D, z, dt_bias)         # x, dt, z, B, C, y in host memory
"""
import ctypes

import torch

from . import _native
from ._native import SSM_A_GENERAL, SSM_DELTA_SOFTPLUS, SSM_EXACT_ZOH

__all__ = ["scan_fwd", "scan_fwd_host", "scan_bwd", "selective_scan", "ssd_fwd", "step", "workspace_size",
           "workspace_status", "ScanWorkspace"]

_TOKEN_DTYPES = {torch.float32: _native.SSM_F32, torch.bfloat16: _native.SSM_BF16}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _resolve_stream(stream, dev):
    """The stream a call on `dev`'s tensors is launched on: the caller's (which must
    belong to `dev`), else `dev`'s current stream. The library plans and launches on
    the current CUDA device, so every call below also runs with `dev` made current."""
    if stream is None:
        return torch.cuda.current_stream(dev)
    if torch.device(stream.device) != torch.device(dev):
        raise ValueError(f"stream belongs to {stream.device}, the tensors to {dev}")
    return stream


def _handle(s):
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device != device or t.device.type != "cuda":
        raise ValueError(f"{name}: must be on {device} (a CUDA device)")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _flags(delta_softplus, general_A, exact_zoh=False, seq_parallel=None):
    return ((SSM_DELTA_SOFTPLUS if delta_softplus else 0) | (SSM_A_GENERAL if general_A else 0)
            | (SSM_EXACT_ZOH if exact_zoh else 0)
            | {None: 0, True: _native.SSM_SEQ_PARALLEL, False: _native.SSM_SEQ_HANDOFF}[seq_parallel])


def _need_conv(conv_w, conv_b, conv_x0, Bsz, Dm, tok, dev):
    """Check the optional short-convolution arguments (taps [D, 4], bias [D], prefix [B, 3, D])."""
    if conv_w is None:
        if conv_b is not None or conv_x0 is not None:
            raise ValueError("conv_b and conv_x0 need conv_w")
        return
    _need(conv_w, "conv_w", (Dm, 4), torch.float32, dev)
    if conv_b is not None:
        _need(conv_b, "conv_b", (Dm,), torch.float32, dev)
    if conv_x0 is not None:
        _need(conv_x0, "conv_x0", (Bsz, 3, Dm), tok, dev)


def _scan_args(x, dt, A, B, C, D, z, dt_bias, h0, y, h_last, flags, conv_w=None, conv_b=None, conv_x0=None):
    a = _native.ScanArgs()
    a.batch, a.seqlen, a.dim = x.shape
    a.dstate = A.shape[1]
    a.dtype = _TOKEN_DTYPES[x.dtype]
    a.flags = flags
    a.x, a.dt, a.z, a.Bm, a.Cm = (_ptr(t) for t in (x, dt, z, B, C))
    a.A, a.Dskip, a.dt_bias, a.h0 = (_ptr(t) for t in (A, D, dt_bias, h0))
    a.y, a.h_last = _ptr(y), _ptr(h_last)
    a.conv_w, a.conv_b, a.conv_x0 = (_ptr(t) for t in (conv_w, conv_b, conv_x0))
    return a


def workspace_size(batch, seqlen, dim, dstate, dtype=torch.bfloat16):
    """Bytes of device workspace a scan of these shapes needs."""
    a = _native.ScanArgs()
    a.batch, a.seqlen, a.dim, a.dstate = batch, seqlen, dim, dstate
    a.dtype = _TOKEN_DTYPES[dtype]
    return int(_native.lib().ssm_scan_workspace_size(ctypes.byref(a)))


class ScanWorkspace:
    """A reusable device workspace (grown on demand) for one stream's scans."""

    def __init__(self, device=None):
        self.device = torch.device(device) if device is not None else None
        self.buf = None

    def get(self, nbytes, device):
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


_default_ws = {}


def scan_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, *, delta_softplus=True,
             general_A=False, exact_zoh=False, return_last_state=False, out=None, h_last=None, workspace=None,
             stream=None, conv_w=None, conv_b=None, conv_x0=None, seq_parallel=None):
    """Selective scan forward over whole sequences (see include/ssm_scan.h, ssm_scan_fwd).

    x, dt, z: [B, L, D] float32 or bfloat16; B, C: [B, L, N] same dtype; A: [D, N]
    float32; D, dt_bias: [D] float32; h0: [B, D, N] float32. Returns y (same dtype
    as x) and, with return_last_state, the final state [B, D, N] float32. exact_zoh:
    Bbar = (exp(Delta A) - 1) / A B instead of Delta B. conv_w [D, 4] float32 (with
    conv_b [D] and conv_x0 [B, 3, D], the tokens before t = 0, both optional) runs the
    block's causal convolution and SiLU on x inside the scan kernel. seq_parallel: None
    lets the library choose between the hand-off and the sequence-parallel evaluation,
    True forces the latter, False the former.
    """
    dev = x.device
    if x.dtype not in _TOKEN_DTYPES:
        raise TypeError(f"x: dtype must be float32 or bfloat16, got {x.dtype}")
    if x.dim() != 3 or A.dim() != 2:
        raise ValueError("x must be [B, L, D] and A [D, N]")
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    tok = x.dtype
    _need(x, "x", (Bsz, L, Dm), tok, dev)
    _need(dt, "dt", (Bsz, L, Dm), tok, dev)
    if z is not None:
        _need(z, "z", (Bsz, L, Dm), tok, dev)
    _need(B, "B", (Bsz, L, N), tok, dev)
    _need(C, "C", (Bsz, L, N), tok, dev)
    _need(A, "A", (Dm, N), torch.float32, dev)
    if D is not None:
        _need(D, "D", (Dm,), torch.float32, dev)
    if dt_bias is not None:
        _need(dt_bias, "dt_bias", (Dm,), torch.float32, dev)
    if h0 is not None:
        _need(h0, "h0", (Bsz, Dm, N), torch.float32, dev)
    y = torch.empty_like(x) if out is None else out
    _need(y, "out", (Bsz, L, Dm), tok, dev)
    if return_last_state and h_last is None:
        h_last = torch.empty((Bsz, Dm, N), dtype=torch.float32, device=dev)
    if h_last is not None:
        _need(h_last, "h_last", (Bsz, Dm, N), torch.float32, dev)
    _need_conv(conv_w, conv_b, conv_x0, Bsz, Dm, tok, dev)
    args = _scan_args(x, dt, A, B, C, D, z, dt_bias, h0, y, h_last,
                      _flags(delta_softplus, general_A, exact_zoh, seq_parallel), conv_w, conv_b, conv_x0)
    s = _resolve_stream(stream, dev)
    nbytes = int(_native.lib().ssm_scan_workspace_size(ctypes.byref(args)))
    if workspace is None:
        workspace = _default_ws.setdefault((dev, s.cuda_stream), ScanWorkspace())
    ws = workspace.get(nbytes, dev) if isinstance(workspace, ScanWorkspace) else workspace
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError(f"workspace too small: {ws.numel() * ws.element_size()} < {nbytes} bytes")
    args.workspace = ctypes.c_void_p(ws.data_ptr())
    args.workspace_bytes = ws.numel() * ws.element_size()
    with torch.cuda.device(dev):
        _native.check(_native.lib().ssm_scan_fwd(ctypes.byref(args), _handle(s)), "ssm_scan_fwd")
    return (y, h_last) if return_last_state else y


def _need_host(t, name, shape, dtype):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device.type != "cpu" or not t.is_contiguous():
        raise ValueError(f"{name}: must be a contiguous host tensor (page-locked for overlapped copies)")


_default_staging = {}


def scan_fwd_host(x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, *, chunk_len=16384,
                  delta_softplus=True, general_A=False, exact_zoh=False, return_last_state=False, out=None,
                  h_last=None, workspace=None, staging=None, stream=None, conv_w=None, conv_b=None,
                  conv_x0=None):
    """Selective scan over host-resident tokens (see include/ssm_scan.h, ssm_scan_fwd_host).

    x, dt, z: [B, L, D] and B, C: [B, L, N] host tensors (page-locked memory lets the
    copies overlap the scan); the result y is a host tensor too (`out`, or a new
    page-locked one). A, D, dt_bias, h0, h_last and the optional short convolution's
    conv_w, conv_b, conv_x0 live on the GPU (A's device). The call is asynchronous on
    `stream`: synchronise it before reading y.
    """
    dev = A.device
    if x.dtype not in _TOKEN_DTYPES:
        raise TypeError(f"x: dtype must be float32 or bfloat16, got {x.dtype}")
    if x.dim() != 3 or A.dim() != 2:
        raise ValueError("x must be [B, L, D] and A [D, N]")
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    tok = x.dtype
    _need_host(x, "x", (Bsz, L, Dm), tok)
    _need_host(dt, "dt", (Bsz, L, Dm), tok)
    if z is not None:
        _need_host(z, "z", (Bsz, L, Dm), tok)
    _need_host(B, "B", (Bsz, L, N), tok)
    _need_host(C, "C", (Bsz, L, N), tok)
    _need(A, "A", (Dm, N), torch.float32, dev)
    if D is not None:
        _need(D, "D", (Dm,), torch.float32, dev)
    if dt_bias is not None:
        _need(dt_bias, "dt_bias", (Dm,), torch.float32, dev)
    if h0 is not None:
        _need(h0, "h0", (Bsz, Dm, N), torch.float32, dev)
    y = torch.empty(x.shape, dtype=tok, pin_memory=True) if out is None else out
    _need_host(y, "out", (Bsz, L, Dm), tok)
    if return_last_state and h_last is None:
        h_last = torch.empty((Bsz, Dm, N), dtype=torch.float32, device=dev)
    if h_last is not None:
        _need(h_last, "h_last", (Bsz, Dm, N), torch.float32, dev)
    _need_conv(conv_w, conv_b, conv_x0, Bsz, Dm, tok, dev)
    args = _scan_args(x, dt, A, B, C, D, z, dt_bias, h0, y, h_last, _flags(delta_softplus, general_A, exact_zoh),
                      conv_w, conv_b, conv_x0)
    lib = _native.lib()
    s = _resolve_stream(stream, dev)
    key = (dev, s.cuda_stream)
    nbytes = int(lib.ssm_scan_workspace_size(ctypes.byref(args)))
    if workspace is None:
        workspace = _default_ws.setdefault(key, ScanWorkspace())
    ws = workspace.get(nbytes, dev) if isinstance(workspace, ScanWorkspace) else workspace
    args.workspace = ctypes.c_void_p(ws.data_ptr())
    args.workspace_bytes = ws.numel() * ws.element_size()
    sbytes = int(lib.ssm_scan_host_staging_size(ctypes.byref(args), int(chunk_len)))
    if staging is None:
        staging = _default_staging.setdefault(key, ScanWorkspace())
    st = staging.get(sbytes, dev) if isinstance(staging, ScanWorkspace) else staging
    with torch.cuda.device(dev):
        _native.check(lib.ssm_scan_fwd_host(ctypes.byref(args), int(chunk_len), ctypes.c_void_p(st.data_ptr()),
                                            st.numel() * st.element_size(), _handle(s)), "ssm_scan_fwd_host")
    return (y, h_last) if return_last_state else y


def scan_bwd(x, dt, A, B, C, dy, D=None, z=None, dt_bias=None, h0=None, dh_last=None, *, delta_softplus=True,
             exact_zoh=False, conv_w=None, conv_b=None, conv_x0=None, workspace=None, stream=None):
    """Backward of scan_fwd (see include/ssm_scan.h, ssm_scan_bwd): gradients given
    dy = dL/dy [B, L, D] (dtype of x) and optionally dh_last = dL/dh_L [B, D, N] float32.
    exact_zoh and the short convolution (conv_w, conv_b, conv_x0) as in the forward call.

    Returns a dict: dx, ddt, dz (None without z) in x's dtype [B, L, D]; dB, dC float32
    [B, L, N]; dA float32 [D, N]; dD, ddt_bias float32 [D]; dh0 float32 [B, D, N]; with
    the convolution also dconv_w float32 [D, 4], dconv_b float32 [D] and dconv_x0 [B, 3, D]
    in x's dtype (None without conv_x0), dx then being the gradient of the raw tokens.
    """
    dev = x.device
    if x.dtype not in _TOKEN_DTYPES:
        raise TypeError(f"x: dtype must be float32 or bfloat16, got {x.dtype}")
    if x.dim() != 3 or A.dim() != 2:
        raise ValueError("x must be [B, L, D] and A [D, N]")
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    tok = x.dtype
    for t, name, shape in ((x, "x", (Bsz, L, Dm)), (dt, "dt", (Bsz, L, Dm)), (dy, "dy", (Bsz, L, Dm)),
                           (B, "B", (Bsz, L, N)), (C, "C", (Bsz, L, N))):
        _need(t, name, shape, tok, dev)
    if z is not None:
        _need(z, "z", (Bsz, L, Dm), tok, dev)
    _need(A, "A", (Dm, N), torch.float32, dev)
    for t, name, shape in ((D, "D", (Dm,)), (dt_bias, "dt_bias", (Dm,)), (h0, "h0", (Bsz, Dm, N)),
                           (dh_last, "dh_last", (Bsz, Dm, N))):
        if t is not None:
            _need(t, name, shape, torch.float32, dev)
    _need_conv(conv_w, conv_b, conv_x0, Bsz, Dm, tok, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = dict(dx=torch.empty_like(x), ddt=torch.empty_like(x), dz=None if z is None else torch.empty_like(x),
               dB=torch.empty((Bsz, L, N), **f32), dC=torch.empty((Bsz, L, N), **f32),
               dA=torch.empty((Dm, N), **f32), dD=torch.empty((Dm,), **f32),
               ddt_bias=torch.empty((Dm,), **f32), dh0=torch.empty((Bsz, Dm, N), **f32))
    a = _native.ScanBwdArgs()
    a.batch, a.seqlen, a.dim, a.dstate = Bsz, L, Dm, N
    a.dtype = _TOKEN_DTYPES[tok]
    a.flags = _flags(delta_softplus, False, exact_zoh)
    if conv_w is not None:
        out.update(dconv_w=torch.empty((Dm, 4), **f32), dconv_b=torch.empty((Dm,), **f32),
                   dconv_x0=None if conv_x0 is None else torch.empty((Bsz, 3, Dm), dtype=tok, device=dev))
        a.conv_w, a.conv_b, a.conv_x0 = _ptr(conv_w), _ptr(conv_b), _ptr(conv_x0)
        a.dconv_w, a.dconv_b, a.dconv_x0 = _ptr(out["dconv_w"]), _ptr(out["dconv_b"]), _ptr(out["dconv_x0"])
    a.x, a.dt, a.z, a.Bm, a.Cm = (_ptr(t) for t in (x, dt, z, B, C))
    a.A, a.Dskip, a.dt_bias, a.h0 = (_ptr(t) for t in (A, D, dt_bias, h0))
    a.dy, a.dh_last = _ptr(dy), _ptr(dh_last)
    a.dx, a.ddt, a.dz = _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dz"])
    a.dB, a.dC, a.dA, a.dD, a.ddt_bias, a.dh0 = (_ptr(out[k]) for k in ("dB", "dC", "dA", "dD", "ddt_bias", "dh0"))
    lib = _native.lib()
    nbytes = int(lib.ssm_scan_bwd_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = ScanWorkspace()
    ws = workspace.get(nbytes, dev) if isinstance(workspace, ScanWorkspace) else workspace
    a.workspace = ctypes.c_void_p(ws.data_ptr())
    a.workspace_bytes = ws.numel() * ws.element_size()
    s = _resolve_stream(stream, dev)
    with torch.cuda.device(dev):
        _native.check(lib.ssm_scan_bwd(ctypes.byref(a), _handle(s)), "ssm_scan_bwd")
    return out


def workspace_status(workspace, stream=None):
    """Synchronise and return the device status code of the last scan on this workspace."""
    ws = workspace.buf if isinstance(workspace, ScanWorkspace) else workspace
    s = _resolve_stream(stream, ws.device)
    with torch.cuda.device(ws.device):
        return int(_native.lib().ssm_workspace_status(ctypes.c_void_p(ws.data_ptr()), _handle(s)))


def step(x, dt, A, B, C, h, D=None, z=None, dt_bias=None, *, delta_softplus=True, general_A=False,
         exact_zoh=False, out=None, stream=None, conv_w=None, conv_b=None, conv_state=None):
    """One recurrent decode step (see include/ssm_scan.h, ssm_step); h is updated in place.

    x, dt, z: [B, D]; B, C: [B, N]; A: [D, N]; h: [B, D, N] float32. Returns y [B, D].
    conv_w [D, 4] float32 with conv_state [B, 3, D] (x's dtype: the three previous
    tokens, oldest first, moved on by one token in place) and optional conv_b [D]: the
    block's short convolution and SiLU in front (ssm_step_conv).
    """
    dev = x.device
    if x.dtype not in _TOKEN_DTYPES:
        raise TypeError(f"x: dtype must be float32 or bfloat16, got {x.dtype}")
    Bsz, Dm = x.shape
    N = A.shape[1]
    tok = x.dtype
    _need(x, "x", (Bsz, Dm), tok, dev)
    _need(dt, "dt", (Bsz, Dm), tok, dev)
    if z is not None:
        _need(z, "z", (Bsz, Dm), tok, dev)
    _need(B, "B", (Bsz, N), tok, dev)
    _need(C, "C", (Bsz, N), tok, dev)
    _need(A, "A", (Dm, N), torch.float32, dev)
    _need(h, "h", (Bsz, Dm, N), torch.float32, dev)
    if D is not None:
        _need(D, "D", (Dm,), torch.float32, dev)
    if dt_bias is not None:
        _need(dt_bias, "dt_bias", (Dm,), torch.float32, dev)
    y = torch.empty_like(x) if out is None else out
    _need(y, "out", (Bsz, Dm), tok, dev)
    flags = _flags(delta_softplus, general_A, exact_zoh)
    common = (Bsz, Dm, N, _TOKEN_DTYPES[tok], flags, _ptr(x), _ptr(dt), _ptr(z), _ptr(B), _ptr(C), _ptr(A),
              _ptr(D), _ptr(dt_bias))
    if conv_w is None:
        if conv_b is not None or conv_state is not None:
            raise ValueError("conv_b and conv_state need conv_w")
        with torch.cuda.device(dev):
            rc = _native.lib().ssm_step(*common, _ptr(h), _ptr(y), _handle(_resolve_stream(stream, dev)))
        _native.check(rc, "ssm_step")
        return y
    _need(conv_w, "conv_w", (Dm, 4), torch.float32, dev)
    if conv_b is not None:
        _need(conv_b, "conv_b", (Dm,), torch.float32, dev)
    if conv_state is None:
        raise ValueError("conv_state [B, 3, D] is required with conv_w")
    _need(conv_state, "conv_state", (Bsz, 3, Dm), tok, dev)
    with torch.cuda.device(dev):
        rc = _native.lib().ssm_step_conv(*common, _ptr(conv_w), _ptr(conv_b), _ptr(conv_state), _ptr(h), _ptr(y),
                                         _handle(_resolve_stream(stream, dev)))
    _native.check(rc, "ssm_step_conv")
    return y


def ssd_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, *, delta_softplus=True,
            return_last_state=False, out=None, h_last=None, workspace=None, stream=None, _test_flags=0):
    """The chunked (Mamba-2) form on the tensor cores (see include/ssm_scan.h, ssm_ssd_fwd).

    x, z: [B, L, H, P] bfloat16 (P = 64); dt: [B, L, H] bfloat16 (one step size per head);
    B, C: [B, L, N] bfloat16 (N = 128); A, D, dt_bias: [H] float32 (one scalar A per head);
    h0: [B, H, P, N] float32. Returns y [B, L, H, P] and, with return_last_state, the final
    state [B, H, P, N] float32. _test_flags: test hooks of the C ABI (SSM_TEST_DROP_HANDOFF).
    """
    dev = x.device
    if x.dim() != 4:
        raise ValueError("x must be [B, L, H, P]")
    Bsz, L, H, Pd = x.shape
    N = B.shape[-1]
    tok = x.dtype
    if tok not in _TOKEN_DTYPES:
        raise TypeError(f"x: dtype must be float32 or bfloat16, got {tok}")
    _need(x, "x", (Bsz, L, H, Pd), tok, dev)
    _need(dt, "dt", (Bsz, L, H), tok, dev)
    if z is not None:
        _need(z, "z", (Bsz, L, H, Pd), tok, dev)
    _need(B, "B", (Bsz, L, N), tok, dev)
    _need(C, "C", (Bsz, L, N), tok, dev)
    _need(A, "A", (H,), torch.float32, dev)
    for t, name in ((D, "D"), (dt_bias, "dt_bias")):
        if t is not None:
            _need(t, name, (H,), torch.float32, dev)
    if h0 is not None:
        _need(h0, "h0", (Bsz, H, Pd, N), torch.float32, dev)
    y = torch.empty_like(x) if out is None else out
    _need(y, "out", (Bsz, L, H, Pd), tok, dev)
    if return_last_state and h_last is None:
        h_last = torch.empty((Bsz, H, Pd, N), dtype=torch.float32, device=dev)
    if h_last is not None:
        _need(h_last, "h_last", (Bsz, H, Pd, N), torch.float32, dev)
    a = _native.SsdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate = Bsz, L, H, Pd, N
    a.dtype = _TOKEN_DTYPES[tok]
    a.flags = (SSM_DELTA_SOFTPLUS if delta_softplus else 0) | int(_test_flags)
    a.x, a.dt, a.z, a.Bm, a.Cm = (_ptr(t) for t in (x, dt, z, B, C))
    a.A, a.Dskip, a.dt_bias, a.h0 = (_ptr(t) for t in (A, D, dt_bias, h0))
    a.y, a.h_last = _ptr(y), _ptr(h_last)
    lib = _native.lib()
    s = _resolve_stream(stream, dev)
    nbytes = int(lib.ssm_ssd_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = _default_ws.setdefault((dev, s.cuda_stream, "ssd"), ScanWorkspace())
    ws = workspace.get(max(nbytes, 256), dev) if isinstance(workspace, ScanWorkspace) else workspace
    a.workspace = ctypes.c_void_p(ws.data_ptr())
    a.workspace_bytes = ws.numel() * ws.element_size()
    with torch.cuda.device(dev):
        _native.check(lib.ssm_ssd_fwd(ctypes.byref(a), _handle(s)), "ssm_ssd_fwd")
    return (y, h_last) if return_last_state else y


class _SelectiveScan(torch.autograd.Function):
    """scan_fwd as an autograd function: the forward keeps its inputs (the states are not
    kept: scan_bwd recomputes them) and the backward is scan_bwd."""

    @staticmethod
    def forward(ctx, x, dt, A, B, C, D, z, dt_bias, h0, conv_w, conv_b, conv_x0, delta_softplus, exact_zoh):
        conv = {} if conv_w is None else dict(conv_w=conv_w, conv_b=conv_b, conv_x0=conv_x0)
        y, h_last = scan_fwd(x, dt, A, B, C, D, z, dt_bias, h0, delta_softplus=delta_softplus, exact_zoh=exact_zoh,
                             return_last_state=True, **conv)
        ctx.save_for_backward(x, dt, A, B, C, D, z, dt_bias, h0, conv_w, conv_b, conv_x0)
        ctx.flags = (delta_softplus, exact_zoh)
        return y, h_last

    @staticmethod
    def backward(ctx, dy, dh_last):
        x, dt, A, B, C, D, z, dt_bias, h0, conv_w, conv_b, conv_x0 = ctx.saved_tensors
        delta_softplus, exact_zoh = ctx.flags
        conv = {} if conv_w is None else dict(conv_w=conv_w, conv_b=conv_b, conv_x0=conv_x0)
        dy = torch.zeros_like(x) if dy is None else dy.to(x.dtype).contiguous()
        dh_last = None if dh_last is None else dh_last.float().contiguous()
        g = scan_bwd(x, dt, A, B, C, dy, D, z, dt_bias, h0, dh_last, delta_softplus=delta_softplus,
                     exact_zoh=exact_zoh, **conv)
        cg = (g.get("dconv_w"), g.get("dconv_b") if conv_b is not None else None, g.get("dconv_x0")) if conv_w is not None \
            else (None, None, None)
        return (g["dx"], g["ddt"], g["dA"], g["dB"].to(B.dtype), g["dC"].to(C.dtype),
                g["dD"] if D is not None else None, g["dz"], g["ddt_bias"] if dt_bias is not None else None,
                g["dh0"] if h0 is not None else None, *cg, None, None)


def selective_scan(x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, *, delta_softplus=True, exact_zoh=False,
                   conv_w=None, conv_b=None, conv_x0=None, return_last_state=False):
    """The scan with its backward attached for torch.autograd: y (and the final state) from
    scan_fwd; gradients for every tensor input from scan_bwd (dB and dC in B's and C's
    dtype). Device tensors as for scan_fwd."""
    y, h_last = _SelectiveScan.apply(x, dt, A, B, C, D, z, dt_bias, h0, conv_w, conv_b, conv_x0, delta_softplus,
                                     exact_zoh)
    return (y, h_last) if return_last_state else y
