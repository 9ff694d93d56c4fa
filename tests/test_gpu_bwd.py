"""GPU parity of the backward scan (ssm_scan_bwd) against the float64 oracle's backward,
which is itself pinned to central differences of the forward oracle.

Per-(t, channel) gradients (dx, ddt, dz) are compared row by row over t per (b, d), like
y; the reduced ones row by row too, so that a wrong small row cannot hide under a large
one: dB and dC per (b, t) over n, dA per channel over n, dh0 per (b, d) over n; dD and
ddt_bias ([D] vectors) against their largest entry. Tolerances: float32 1e-4 everywhere;
bfloat16 tokens 1e-2 for the [B, L, D] gradients (stored in bfloat16) and 1e-4 for the
float32 reductions.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available
from tests.gpu_util import dtype_name, rowwise_rel, storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


def _rel(got, ref):
    got = np.asarray(got, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))


def _oracle_bwd(inp, dy, dh_last, softplus=True, sel=None):
    def tok(t):
        if t is None:
            return None
        return storage((t[:, :, sel] if sel is not None else t).contiguous().cpu())
    def par(t, dim=0):
        if t is None:
            return None
        t = t.cpu()
        return (t.index_select(dim, sel) if sel is not None else t).float().numpy()
    dhl = None if dh_last is None else par(dh_last, 1).astype(np.float64)
    return oracle.scan_bwd(tok(inp["x"]), tok(inp["dt"]), par(inp["A"]), storage(inp["B"].cpu()),
                           storage(inp["C"].cpu()), tok(dy), D=par(inp["D"]), z=tok(inp["z"]),
                           dt_bias=par(inp["dt_bias"]), h0=par(inp.get("h0"), 1), dh_last=dhl,
                           dtype=dtype_name(inp["x"]), delta_softplus=softplus)


def _check(g, ref, tok_tol, red_tol, sel=None, check_bc=True):
    errs = {}
    for k in ("dx", "ddt", "dz"):
        if ref[k] is None:
            assert g[k] is None
            continue
        got = g[k] if sel is None else g[k][:, :, sel.to(g[k].device)]
        errs[k] = rowwise_rel(got.float().cpu().numpy(), ref[k], axis=1)
    red = ["dA", "dD", "ddt_bias", "dh0"] + (["dB", "dC"] if check_bc else [])
    for k in red:
        got = g[k]
        if sel is not None and k not in ("dB", "dC"):
            got = got.index_select(0 if k in ("dA", "dD", "ddt_bias") else 1, sel.to(got.device))
        got = got.cpu().numpy()
        if k in ("dD", "ddt_bias"):
            errs[k] = _rel(got, ref[k])
        else:  # rows over the state index n: dA [D, N], dB / dC [B, L, N], dh0 [B, D, N]
            errs[k] = rowwise_rel(got, ref[k], axis=got.ndim - 1)
    print("  ".join(f"{k} {v:.1e}" for k, v in errs.items()))
    for k, v in errs.items():
        assert v <= (tok_tol if k in ("dx", "ddt", "dz") else red_tol), f"{k}: {v:.3e}"


BWD_CASES = [
    # (batch, seqlen, dim, dstate, dtype, gate, h0, dh_last, softplus, random_A)
    (1, 300, 64, 16, torch.float32, True, True, True, True, False),     # ragged last chunk
    (2, 129, 40, 5, torch.float32, True, False, False, True, True),     # lanes past D; N = 5 (B, C by elements)
    (2, 1000, 256, 16, torch.bfloat16, True, True, True, True, False),
    (1, 77, 32, 8, torch.bfloat16, False, False, True, False, True),    # no gate, no softplus; N = 8
    (3, 1, 32, 16, torch.float32, True, True, True, True, False),       # L = 1
    (1, 16, 32, 16, torch.float32, True, False, False, True, False),    # exactly one half chunk
]


@pytest.mark.parametrize("case", BWD_CASES)
def test_bwd_matches_oracle(ssm, case):
    Bsz, L, Dm, N, dtype, gate, h0, dhl, softplus, random_A = case
    inp = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=71, gate=gate, h0=h0)
    if random_A:
        gen = torch.Generator().manual_seed(72)
        inp["A"] = -torch.rand((Dm, N), generator=gen) * 3.0 - 0.05
    if not softplus:  # Delta = dt + bias itself: keep it positive (Abar <= 1), as softplus would
        inp["dt"] = (inp["dt"].float().abs() * 0.2).to(dtype)
        inp["dt_bias"] = torch.full((Dm,), 0.05)
    gen = torch.Generator().manual_seed(73)
    dy = torch.randn((Bsz, L, Dm), generator=gen).to(dtype)
    dh_last = torch.randn((Bsz, Dm, N), generator=gen) if dhl else None
    ref = _oracle_bwd(inp, dy, dh_last, softplus)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    g = ssm.scan_bwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dy.cuda(), dev["D"], dev["z"],
                     dev["dt_bias"], dev.get("h0"), None if dh_last is None else dh_last.cuda(),
                     delta_softplus=softplus)
    torch.cuda.synchronize()
    print(f"\nbwd case {case[:5]}: ", end="")
    _check(g, ref, 1e-4 if dtype == torch.float32 else 1e-2, 1e-4)


def test_bwd_empty_sequence(ssm):
    """L = 0: dh0 = dh_last, every reduced gradient zero."""
    Bsz, Dm, N = 2, 64, 16
    x = torch.empty((Bsz, 0, Dm), device="cuda")
    bc = torch.empty((Bsz, 0, N), device="cuda")
    A = -torch.ones((Dm, N), device="cuda")
    dhl = torch.randn((Bsz, Dm, N), device="cuda")
    g = ssm.scan_bwd(x, x, A, bc, bc, x, dh_last=dhl)
    torch.cuda.synchronize()
    assert torch.equal(g["dh0"], dhl)
    assert not g["dA"].any() and not g["dD"].any() and not g["ddt_bias"].any()


def test_bwd_long_context_sampled(ssm):
    """B=1, L=262144, D=5120 at full size; the oracle runs on 34 channels spread over D, at
    a lane that moves with the channel group (all 262,144 steps): dx, ddt, dz, dA, dD,
    ddt_bias and dh0 of those channels (dB, dC sum over all channels: the next test checks
    them against an oracle over every channel)."""
    inp = synth.workload_inputs("long_context", device="cuda", h0=True)
    gen = torch.Generator(device="cuda").manual_seed(74)
    dy = torch.randn(inp["x"].shape, generator=gen, device="cuda").to(inp["x"].dtype)
    g = ssm.scan_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"], inp["z"], inp["dt_bias"],
                     inp["h0"])
    torch.cuda.synchronize()
    groups = torch.arange(0, 160, 5)
    sel = torch.unique(torch.cat([groups * 32 + (groups * 11) % 32, torch.tensor([0, 5119])]))
    ref = _oracle_bwd(inp, dy, None, sel=sel)
    print(f"\nbwd long_context ({len(sel)} channels, all steps): ", end="")
    _check(g, ref, 1e-2, 1e-4, sel=sel, check_bc=False)


def test_bwd_long_context_width_all_channels(ssm):
    """The long-context width (B=1, D=5120, N=16, bf16, with h0 and dL/dh_L) on a sequence
    shortened to L=2048, so that the oracle runs over every channel: dB and dC, which sum
    the contributions of all 5120 channels, compared for every (b, t) row, and every other
    gradient in full."""
    w = synth.WORKLOADS["long_context"]
    inp = synth.scan_inputs(w.batch, 2048, w.dim, w.dstate, w.dtype, seed=75, h0=True)
    gen = torch.Generator().manual_seed(76)
    dy = torch.randn(inp["x"].shape, generator=gen).to(w.dtype)
    dh_last = torch.randn((w.batch, w.dim, w.dstate), generator=gen)
    ref = _oracle_bwd(inp, dy, dh_last)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    g = ssm.scan_bwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dy.cuda(), dev["D"], dev["z"],
                     dev["dt_bias"], dev["h0"], dh_last.cuda())
    torch.cuda.synchronize()
    print("\nbwd long_context width, L=2048, all channels: ", end="")
    _check(g, ref, 1e-2, 1e-4)
