"""GPU check of selective_scan, the autograd wrapper over ssm_scan_fwd / ssm_scan_bwd: the
gradients torch.autograd delivers for L = sum(dy * y) + sum(dh_last * h_L) equal the
float64 oracle's backward for that dy and dh_last, for every input (with the short
convolution, its taps, bias and prefix tokens too), compared per row as in the backward's
own tests (float32 1e-4)."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available
from tests.gpu_util import rowwise_rel, storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


def _np(t):
    return None if t is None else t.detach().cpu().float().numpy()


@pytest.mark.parametrize("conv,zoh", [(False, False), (True, False), (False, True)], ids=["plain", "conv", "zoh"])
def test_autograd_matches_oracle(ssm, conv, zoh):
    Bsz, L, Dm, N = 2, 333, 64, 16
    cpu = synth.scan_inputs(Bsz, L, Dm, N, torch.float32, seed=3001, h0=True)
    gen = torch.Generator().manual_seed(3002)
    cpu["A"] = -torch.rand((Dm, N), generator=gen) * 3.0 - 0.05
    cv = synth.conv_params(Dm, Bsz, torch.float32, seed=3003) if conv else {}
    dy = torch.randn((Bsz, L, Dm), generator=gen)
    dhl = torch.randn((Bsz, Dm, N), generator=gen)
    names = ["x", "dt", "A", "B", "C", "D", "z", "dt_bias", "h0"]
    leaf = {k: cpu[k].cuda().requires_grad_(True) for k in names}
    cleaf = {k: v.cuda().requires_grad_(True) for k, v in cv.items()}
    y, h = ssm.selective_scan(*[leaf[k] for k in names], exact_zoh=zoh, return_last_state=True, **cleaf)
    loss = (y * dy.cuda()).sum() + (h * dhl.cuda()).sum()
    loss.backward()
    torch.cuda.synchronize()
    kw = {}
    if conv:
        kw = dict(conv_w=_np(cv["conv_w"]), conv_b=_np(cv["conv_b"]), conv_x0=storage(cv["conv_x0"]))
    ref = oracle.scan_bwd(*(storage(cpu[k]) if k in ("x", "dt", "B", "C") else _np(cpu[k]) for k in ("x", "dt", "A", "B", "C")),
                          storage(dy), D=_np(cpu["D"]), z=storage(cpu["z"]), dt_bias=_np(cpu["dt_bias"]),
                          h0=_np(cpu["h0"]), dh_last=dhl.double().numpy(), exact_zoh=zoh, **kw)
    pairs = {"x": ("dx", 1), "dt": ("ddt", 1), "z": ("dz", 1), "B": ("dB", 2), "C": ("dC", 2), "A": ("dA", 1),
             "h0": ("dh0", 2)}
    errs = {}
    for k, (r, axis) in pairs.items():
        errs[r] = rowwise_rel(leaf[k].grad.cpu().numpy(), ref[r], axis=axis)
    for k, r in (("D", "dD"), ("dt_bias", "ddt_bias")):
        g = leaf[k].grad.cpu().numpy()
        errs[r] = float(np.abs(g - ref[r]).max() / np.abs(ref[r]).max())
    if conv:
        errs["dconv_w"] = rowwise_rel(cleaf["conv_w"].grad.cpu().numpy(), ref["dconv_w"], axis=1)
        errs["dconv_b"] = float(np.abs(cleaf["conv_b"].grad.cpu().numpy() - ref["dconv_b"]).max()
                                / np.abs(ref["dconv_b"]).max())
        errs["dconv_x0"] = rowwise_rel(cleaf["conv_x0"].grad.cpu().numpy(), ref["dconv_x0"], axis=1)
    print(f"\nautograd conv={conv} zoh={zoh}: " + "  ".join(f"{k} {v:.1e}" for k, v in errs.items()))
    for k, v in errs.items():
        assert v <= 1e-4, f"{k}: {v:.3e}"
