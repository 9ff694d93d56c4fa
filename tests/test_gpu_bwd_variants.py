"""GPU parity of the backward scan for the two forward variants, against the float64
oracle's backward (itself pinned to central differences of the forward oracle):

- the exact zero-order hold (Bbar = (exp(Delta A) - 1) / A B, SSM_EXACT_ZOH), with A
  entries small enough that Delta A falls on the series side of the input weight and of
  its derivative in A;
- the short causal convolution and SiLU in front of the SSM (conv_w, conv_b, conv_x0):
  dx is then the gradient of the raw tokens, and the taps, bias and prefix tokens get
  their own gradients.

Gradients are compared row by row as in the default backward's tests (dconv_w per
channel over its four taps, dconv_x0 per (b, d) over its three tokens, dconv_b against
its largest entry). Tolerances: float32 1e-4; bfloat16 tokens 1e-2. With the convolution
and bfloat16 tokens the SSM input u = silu(conv(x)) is held in bfloat16 between the
kernels, a relative rounding of up to 2^-9 in every term that u enters, so there the
float32 reductions are held to 1e-2 as well.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available
from tests.gpu_util import dtype_name, rowwise_rel, storage
from tests.test_gpu_bwd import _check, _rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


def _np(t):
    return None if t is None else t.detach().cpu().float().numpy()


def _oracle(inp, dy, dh_last, zoh, conv):
    tok = lambda t: None if t is None else storage(t.contiguous().cpu())
    kw = {}
    if conv is not None:
        kw = dict(conv_w=_np(conv["conv_w"]), conv_b=_np(conv.get("conv_b")), conv_x0=tok(conv.get("conv_x0")))
    return oracle.scan_bwd(tok(inp["x"]), tok(inp["dt"]), _np(inp["A"]), tok(inp["B"]), tok(inp["C"]), tok(dy),
                           D=_np(inp["D"]), z=tok(inp["z"]), dt_bias=_np(inp["dt_bias"]), h0=_np(inp.get("h0")),
                           dh_last=None if dh_last is None else _np(dh_last).astype(np.float64),
                           dtype=dtype_name(inp["x"]), exact_zoh=zoh, **kw)


def _run(ssm, case, zoh, conv_on, bias=True, prefix=True, seed=81):
    Bsz, L, Dm, N, dtype, gate, h0, dhl = case
    inp = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=seed, gate=gate, h0=h0)
    gen = torch.Generator().manual_seed(seed + 1)
    A = -torch.rand((Dm, N), generator=gen) * 3.0 - 0.05
    if zoh:  # some states with |Delta A| below the series thresholds (1/16 and 1/2), one A = 0
        A[:, 0] = -1e-3
        A[:, 1] = -0.2
        A[0, 2] = 0.0
    inp["A"] = A
    conv = synth.conv_params(Dm, Bsz, dtype, seed=seed + 2, bias=bias, prefix=prefix) if conv_on else None
    dy = torch.randn((Bsz, L, Dm), generator=gen).to(dtype)
    dh_last = torch.randn((Bsz, Dm, N), generator=gen) if dhl else None
    ref = _oracle(inp, dy, dh_last, zoh, conv)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    cv = {} if conv is None else {k: (v.cuda() if v is not None else None) for k, v in conv.items()}
    g = ssm.scan_bwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dy.cuda(), dev["D"], dev["z"],
                     dev["dt_bias"], dev.get("h0"), None if dh_last is None else dh_last.cuda(), exact_zoh=zoh,
                     **cv)
    torch.cuda.synchronize()
    return g, ref


ZOH_CASES = [
    # (batch, seqlen, dim, dstate, dtype, gate, h0, dh_last)
    (1, 300, 64, 16, torch.float32, True, True, True),
    (2, 129, 40, 5, torch.float32, True, False, False),   # lanes past D; N = 5
    (2, 1000, 256, 16, torch.bfloat16, True, True, True),
    (3, 1, 32, 16, torch.float32, True, True, True),      # L = 1
]


@pytest.mark.parametrize("case", ZOH_CASES, ids=lambda c: f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{str(c[4])[6:]}")
def test_bwd_exact_zoh_matches_oracle(ssm, case):
    g, ref = _run(ssm, case, zoh=True, conv_on=False)
    print(f"\nbwd exact ZOH {case[:5]}: ", end="")
    f32 = case[4] == torch.float32
    _check(g, ref, 1e-4 if f32 else 1e-2, 1e-4)


CONV_CASES = [
    # (case, bias, prefix, exact_zoh)
    ((1, 300, 64, 16, torch.float32, True, True, True), True, True, False),
    ((2, 1000, 96, 16, torch.bfloat16, True, True, False), True, True, False),
    ((2, 700, 64, 16, torch.float32, False, False, True), False, False, False),  # no bias, no prefix
    ((1, 2, 32, 16, torch.float32, True, False, True), True, True, False),       # L < 3: prefix and tokens mix
    ((1, 517, 64, 16, torch.float32, True, True, True), True, True, True),       # with the exact hold
    ((2, 2100, 40, 7, torch.float32, True, True, False), True, True, False),     # several runs; lanes past D
]


@pytest.mark.parametrize("case,bias,prefix,zoh", CONV_CASES,
                         ids=lambda c: "" if not isinstance(c, tuple) else f"B{c[0]}L{c[1]}D{c[2]}{str(c[4])[6:]}")
def test_bwd_conv_matches_oracle(ssm, case, bias, prefix, zoh):
    g, ref = _run(ssm, case, zoh=zoh, conv_on=True, bias=bias, prefix=prefix, seed=91)
    f32 = case[4] == torch.float32
    tol = 1e-4 if f32 else 1e-2
    print(f"\nbwd conv {case[:5]} bias={bias} prefix={prefix} zoh={zoh}: ", end="")
    _check(g, ref, tol, tol)
    e = {"dconv_w": rowwise_rel(g["dconv_w"].cpu().numpy(), ref["dconv_w"], axis=1),
         "dconv_b": _rel(g["dconv_b"].cpu().numpy(), ref["dconv_b"])}
    if prefix:
        e["dconv_x0"] = rowwise_rel(g["dconv_x0"].float().cpu().numpy(), ref["dconv_x0"], axis=1)
    else:
        assert g["dconv_x0"] is None
    print("  ".join(f"{k} {v:.1e}" for k, v in e.items()))
    for k, v in e.items():
        assert v <= tol, f"{k}: {v:.3e}"
