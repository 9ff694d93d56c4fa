"""GPU parity of the exact zero-order hold (flag SSM_EXACT_ZOH): Bbar = (exp(Delta A) - 1) / A B.

Against the float64 oracle's exact-ZOH mode for the scan and the decode step, and, for
N = 1 and A = -1, against the gated RNN of the Mamba summary's Theorem 1 written out
directly: h_t = (1 - g_t) h_{t-1} + g_t x_t with g_t = sigmoid(dt_t + bias).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available
from tests.gpu_util import TOL, dtype_name, h_err, oracle_scan, rowwise_rel, y_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


ZOH_CASES = [
    # (batch, seqlen, dim, dstate, dtype, gate, h0, random_A)
    (1, 300, 64, 16, torch.float32, True, True, False),     # arithmetic rows of A
    (2, 2000, 256, 16, torch.bfloat16, True, False, False),
    (1, 257, 32, 16, torch.float32, False, True, True),     # general A
    (2, 129, 40, 5, torch.float32, True, False, True),      # N = 5: B, C rows not 16-byte multiples
]


@pytest.mark.parametrize("case", ZOH_CASES)
def test_exact_zoh_scan_matches_oracle(ssm, case):
    Bsz, L, Dm, N, dtype, gate, h0, random_A = case
    inp = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=41, gate=gate, h0=h0)
    if random_A:
        g = torch.Generator().manual_seed(42)
        inp["A"] = -torch.rand((Dm, N), generator=g) * 4.0 - 0.05
    y_ref, h_ref = oracle_scan(inp, exact_zoh=True)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, h = ssm.scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"], dev["dt_bias"],
                        dev.get("h0"), exact_zoh=True, return_last_state=True)
    torch.cuda.synchronize()
    tol = TOL[dtype_name(inp["x"])]
    assert y_err(y, y_ref) <= tol
    assert h_err(h, h_ref) <= tol


def test_theorem1_gated_rnn_on_gpu(ssm):
    """N = 1, A = -1, B = C = 1, D = 0, no gate: with the exact ZOH the scan is the gated
    RNN h_t = (1 - g_t) h_{t-1} + g_t x_t, g_t = sigmoid(dt_t + bias) (Theorem 1)."""
    Bsz, L, Dm = 2, 777, 32
    g = torch.Generator().manual_seed(43)
    x = torch.randn((Bsz, L, Dm), generator=g)
    dt = torch.randn((Bsz, L, Dm), generator=g) * 2.0
    bias = torch.randn((Dm,), generator=g)
    h0 = torch.randn((Bsz, Dm, 1), generator=g)
    ones = torch.ones((Bsz, L, 1))
    A = -torch.ones((Dm, 1))
    # the gated RNN in float64, written out directly
    gate = 1.0 / (1.0 + np.exp(-(dt.double().numpy() + bias.double().numpy())))
    h = h0[:, :, 0].double().numpy().copy()
    ys = np.empty((Bsz, L, Dm))
    xs = x.double().numpy()
    for t in range(L):
        h = (1.0 - gate[:, t]) * h + gate[:, t] * xs[:, t]
        ys[:, t] = h
    c = lambda t: t.cuda()
    y, hl = ssm.scan_fwd(c(x), c(dt), c(A), c(ones), c(ones), None, None, c(bias), c(h0), exact_zoh=True,
                         return_last_state=True)
    torch.cuda.synchronize()
    assert rowwise_rel(y.cpu().numpy(), ys, axis=1) <= 1e-4
    assert np.abs(hl[:, :, 0].cpu().numpy() - h).max() <= 1e-4 * max(1.0, np.abs(h).max())


@pytest.mark.parametrize("N", [16, 5])
def test_exact_zoh_step_matches_oracle(ssm, N):
    """Decode steps with the exact ZOH: two-threads-per-channel kernel (N = 16) and the
    one-thread-per-channel kernel (N = 5), 20 chained steps."""
    Bsz, Dm, steps = 4, 96, 20
    inp = synth.step_inputs(Bsz, Dm, N, steps, torch.bfloat16, seed=44)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    h = dev["h"].clone()
    hr = inp["h"].double().numpy().copy()
    st = synth.to_numpy_storage
    worst = 0.0
    for s in range(steps):
        y = ssm.step(dev["x"][s], dev["dt"][s], dev["A"], dev["B"][s], dev["C"][s], h, dev["D"], dev["z"][s],
                     dev["dt_bias"], exact_zoh=True)
        yr = oracle.step(st(inp["x"][s]), st(inp["dt"][s]), inp["A"].numpy(), st(inp["B"][s]), st(inp["C"][s]),
                         hr, D=inp["D"].numpy(), z=st(inp["z"][s]), dt_bias=inp["dt_bias"].numpy(), dtype="bf16",
                         exact_zoh=True)
        worst = max(worst, rowwise_rel(y.float().cpu().numpy(), yr, axis=1))
    torch.cuda.synchronize()
    assert worst <= 1e-2
    assert rowwise_rel(h.cpu().numpy(), hr, axis=2) <= 1e-2
