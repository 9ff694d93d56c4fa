"""GPU parity of ssm_step (one-token recurrent decode) against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available
from tests.gpu_util import dtype_name, f32np, rowwise_rel, storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


def _oracle_steps(inp, steps, bsel=None, dsel=None):
    """Oracle over `steps` chained steps on a (batch, channel) sub-grid; returns ys, h."""
    def sub(t):
        if t is None:
            return None
        if bsel is not None:
            t = t[:, bsel]
        if dsel is not None:
            t = t[:, :, dsel] if t.dim() == 3 else t[:, dsel]
        return t
    h = inp["h"]
    if bsel is not None:
        h = h[bsel]
    if dsel is not None:
        h = h[:, dsel]
    h = h.double().numpy().copy()
    A = inp["A"] if dsel is None else inp["A"][dsel]
    Dk = inp["D"] if dsel is None else inp["D"][dsel]
    bias = inp["dt_bias"] if dsel is None else inp["dt_bias"][dsel]
    x, dt, z = sub(inp["x"]), sub(inp["dt"]), sub(inp["z"])
    Bm = inp["B"] if bsel is None else inp["B"][:, bsel]
    Cm = inp["C"] if bsel is None else inp["C"][:, bsel]
    dn = dtype_name(inp["x"])
    ys = []
    for s in range(steps):
        ys.append(oracle.step(storage(x[s].contiguous()), storage(dt[s].contiguous()), f32np(A),
                              storage(Bm[s].contiguous()), storage(Cm[s].contiguous()), h,
                              D=f32np(Dk), z=None if z is None else storage(z[s].contiguous()),
                              dt_bias=f32np(bias), dtype=dn, nthreads=1))
    return np.stack(ys), h


@pytest.mark.parametrize("shape", [(3, 16, 16, torch.float32), (4, 40, 16, torch.bfloat16),
                                   (2, 24, 5, torch.float32), (1, 8, 1, torch.bfloat16)],
                         ids=lambda s: f"B{s[0]}D{s[1]}N{s[2]}")
def test_step_parity(ssm, shape):
    Bsz, Dm, N, dt_ = shape
    steps = 12
    inp = synth.step_inputs(Bsz, Dm, N, steps, dt_, seed=300 + Dm)
    ys_ref, h_ref = _oracle_steps(inp, steps)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    h = dev["h"].clone()
    ys = [ssm.step(dev["x"][s], dev["dt"][s], dev["A"], dev["B"][s], dev["C"][s], h, dev["D"],
                   dev["z"][s], dev["dt_bias"]) for s in range(steps)]
    torch.cuda.synchronize()
    tol = 1e-4 if dt_ == torch.float32 else 1e-2
    ys = torch.stack(ys).float().cpu().numpy()
    assert rowwise_rel(ys, ys_ref, axis=2) <= tol
    assert rowwise_rel(h.cpu().numpy(), h_ref, axis=2) <= tol


def test_step_equals_scan(ssm):
    """L chained steps on the GPU equal one GPU scan of length L (both float32)."""
    Bsz, Dm, N, L = 2, 64, 16, 40
    inp = synth.scan_inputs(Bsz, L, Dm, N, torch.float32, seed=31, h0=True)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, hL = ssm.scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                         dev["dt_bias"], dev["h0"], return_last_state=True)
    h = dev["h0"].clone()
    ys = [ssm.step(dev["x"][:, t].contiguous(), dev["dt"][:, t].contiguous(), dev["A"],
                   dev["B"][:, t].contiguous(), dev["C"][:, t].contiguous(), h, dev["D"],
                   dev["z"][:, t].contiguous(), dev["dt_bias"]) for t in range(L)]
    torch.cuda.synchronize()
    ys = torch.stack(ys, 1)
    assert torch.allclose(ys, y, rtol=1e-5, atol=1e-5 * y.abs().max().item())
    assert torch.allclose(h, hL, rtol=1e-5, atol=1e-5)


def test_decode_workload_sampled(ssm):
    """B=256, D=5120, N=16, 1000 chained steps on the GPU; the oracle follows 64 sequences x
    64 channels (spread over both dimensions, ends included) through all 1000 steps."""
    w = synth.WORKLOADS["decode"]
    inp = synth.step_inputs(w.batch, w.dim, w.dstate, w.steps, w.dtype, seed=synth.SEEDS["decode"])
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    h = dev["h"].clone()
    out = torch.empty((w.steps, w.batch, w.dim), dtype=w.dtype, device="cuda")
    for s in range(w.steps):
        ssm.step(dev["x"][s], dev["dt"][s], dev["A"], dev["B"][s], dev["C"][s], h, dev["D"],
                 dev["z"][s], dev["dt_bias"], out=out[s])
    torch.cuda.synchronize()
    bsel = torch.unique(torch.cat([torch.linspace(0, 255, 62).round().long(), torch.tensor([1, 254])]))
    dsel = torch.unique(torch.cat([torch.linspace(0, 5112, 66).round().long() + (torch.arange(66) % 7),
                                   torch.tensor([0, 5119])]))
    ys_ref, h_ref = _oracle_steps(inp, w.steps, bsel, dsel)
    ys = out[:, bsel.cuda()][:, :, dsel.cuda()].float().cpu().numpy()
    hs = h[bsel.cuda()][:, dsel.cuda()].cpu().numpy()
    e_y, e_h = rowwise_rel(ys, ys_ref, axis=2), rowwise_rel(hs, h_ref, axis=2)
    print(f"\ndecode ({len(bsel)} x {len(dsel)} pairs, 1000 steps): max rel err y {e_y:.3e}, h {e_h:.3e}")
    assert e_y <= 1e-2
    assert e_h <= 1e-2
