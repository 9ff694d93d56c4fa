"""Helpers shared by the GPU parity tests: oracle runs on the same bytes, error metrics."""
import numpy as np
import torch

import oracle
from selective_state_space_47_b200 import synth


def storage(t):
    return synth.to_numpy_storage(t)


def dtype_name(t):
    return "bf16" if t.dtype == torch.bfloat16 else "f32"


def f32np(t):
    return None if t is None else t.detach().cpu().float().numpy()


def oracle_scan(inp, delta_softplus=True, sel=None, exact_zoh=False, conv=None):
    """Run the float64 oracle on exactly the tensors the GPU saw (optionally a channel subset).
    conv: the short convolution's conv_w / conv_b / conv_x0 tensors (no channel subset)."""
    def tok(name):
        t = inp[name]
        if t is None:
            return None
        if sel is not None:
            t = t[:, :, sel]
        return storage(t.contiguous())
    def par(name, dim=0):
        t = inp[name]
        if t is None:
            return None
        if sel is not None:
            t = t.index_select(dim, sel.to(t.device))
        return f32np(t)
    h0 = inp.get("h0")
    if h0 is not None and sel is not None:
        h0 = h0[:, sel]
    kw = {}
    if conv is not None:
        assert sel is None
        kw = dict(conv_w=f32np(conv["conv_w"]), conv_b=f32np(conv.get("conv_b")),
                  conv_x0=storage(conv.get("conv_x0")))
    return oracle.scan(tok("x"), tok("dt"), par("A"), storage(inp["B"]), storage(inp["C"]),
                       D=par("D"), z=tok("z"), dt_bias=par("dt_bias"), h0=f32np(h0),
                       dtype=dtype_name(inp["x"]), delta_softplus=delta_softplus, exact_zoh=exact_zoh, **kw)


def rowwise_rel(got, ref, axis):
    """max over rows of  max|got - ref| / max|ref|  along `axis` (the row direction)."""
    got = np.asarray(got, dtype=np.float64)
    num = np.abs(got - ref).max(axis=axis)
    den = np.abs(ref).max(axis=axis)
    return float((num / np.maximum(den, 1e-30)).max())


def y_err(y_gpu, y_ref):
    """Per (b, d) row over t: the tolerance metric of the scan."""
    return rowwise_rel(y_gpu.detach().float().cpu().numpy(), y_ref, axis=1)


def h_err(h_gpu, h_ref):
    """Per (b, d) row over n."""
    return rowwise_rel(h_gpu.detach().cpu().numpy(), h_ref, axis=2)


TOL = {"f32": 1e-4, "bf16": 1e-2}
