"""GPU parity of the chunked tensor-core form (ssm_ssd_fwd) against the float64 oracle.

The oracle is the sequential scan of the model with one scalar A per head: every head's
step size, A, D and dt_bias repeated over its P channels (the restriction under which the
oracle's scan equals its semiseparable matrix form, pinned on the CPU by
pin_ssd_semiseparable_form). Tolerance: bfloat16 tokens 1e-2, per (b, channel) row of y
over t and per (b, channel) row of the final state over n, as for the scan.
"""
import numpy as np
import pytest
import torch

from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available
from tests.gpu_util import rowwise_rel
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


def oracle_ssd(inp, delta_softplus=True):
    """The float64 oracle scan on the channel expansion of the per-head inputs."""
    Bsz, L, H, P = inp["x"].shape
    N = inp["B"].shape[-1]
    st = synth.to_numpy_storage
    x = st(inp["x"].reshape(Bsz, L, H * P).contiguous())
    dt = st(inp["dt"].repeat_interleave(P, dim=2).contiguous())
    z = None if inp["z"] is None else st(inp["z"].reshape(Bsz, L, H * P).contiguous())
    A = inp["A"].repeat_interleave(P)[:, None].repeat(1, N).numpy()
    D = inp["D"].repeat_interleave(P).numpy()
    bias = inp["dt_bias"].repeat_interleave(P).numpy()
    h0 = None if inp["h0"] is None else inp["h0"].reshape(Bsz, H * P, N).numpy()
    y, h = oracle.scan(x, dt, A, st(inp["B"]), st(inp["C"]), D=D, z=z, dt_bias=bias, h0=h0, dtype="bf16",
                       delta_softplus=delta_softplus)
    return y.reshape(Bsz, L, H, P), h.reshape(Bsz, H, P, N)


SSD_CASES = [
    # (batch, seqlen, nheads, gate, h0, softplus)
    (1, 128, 1, True, False, True),      # one whole chunk
    (2, 300, 3, True, True, True),       # ragged last chunk, h0
    (1, 1, 2, True, True, True),         # L = 1
    (1, 4097, 2, True, True, True),      # three segments of 16 chunks, handed over between blocks
    (2, 777, 5, False, False, False),    # no gate, no softplus
]


@pytest.mark.parametrize("case", SSD_CASES, ids=lambda c: f"B{c[0]}L{c[1]}H{c[2]}")
def test_ssd_matches_oracle(ssm, case):
    Bsz, L, H, gate, h0, softplus = case
    inp = synth.ssd_inputs(Bsz, L, H, seed=90 + L, gate=gate, h0=h0)
    if not softplus:  # Delta = dt + bias itself: keep it positive, as softplus would
        inp["dt"] = (inp["dt"].float().abs() * 0.05).to(torch.bfloat16)
        inp["dt_bias"] = torch.full((H,), 0.01)
    y_ref, h_ref = oracle_ssd(inp, softplus)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, h = ssm.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"], dev["dt_bias"],
                       dev["h0"], delta_softplus=softplus, return_last_state=True)
    torch.cuda.synchronize()
    yg = y.float().cpu().numpy().reshape(Bsz, L, H * 64)
    e_y = rowwise_rel(yg, y_ref.reshape(Bsz, L, H * 64), axis=1)
    e_h = rowwise_rel(h.cpu().numpy(), h_ref, axis=3)
    print(f"\nssd {case}: max rel err y {e_y:.3e}, h_L {e_h:.3e}")
    assert e_y <= 1e-2 and e_h <= 1e-2


def test_ssd_layer_sampled(ssm):
    """The benchmark's SSD workload (B=2, L=16384, H=80, P=64, N=128) at full size; the
    oracle follows 4 heads of each sequence (all 64 channels each, every step)."""
    w = synth.WORKLOADS["ssd_layer"]
    inp = synth.ssd_inputs(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, seed=synth.SEEDS["ssd_layer"])
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, h = ssm.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"], dev["dt_bias"],
                       return_last_state=True)
    torch.cuda.synchronize()
    heads = torch.tensor([0, 17, 41, 79])
    sub = dict(x=inp["x"][:, :, heads], dt=inp["dt"][:, :, heads], z=inp["z"][:, :, heads], B=inp["B"], C=inp["C"],
               A=inp["A"][heads], D=inp["D"][heads], dt_bias=inp["dt_bias"][heads], h0=None)
    y_ref, h_ref = oracle_ssd(sub)
    yg = y[:, :, heads.cuda()].float().cpu().numpy()
    e_y = rowwise_rel(yg.reshape(w.batch, w.seqlen, -1), y_ref.reshape(w.batch, w.seqlen, -1), axis=1)
    e_h = rowwise_rel(h[:, heads.cuda()].cpu().numpy(), h_ref, axis=3)
    print(f"\nssd_layer (4 heads x 2 sequences, all steps): max rel err y {e_y:.3e}, h_L {e_h:.3e}")
    assert e_y <= 1e-2 and e_h <= 1e-2


def test_ssd_rejects_unsupported(ssm):
    inp = synth.ssd_inputs(1, 64, 1, headdim=32, seed=99)  # P = 32: not the supported head shape
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    with pytest.raises(RuntimeError):
        ssm.ssd_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"], dev["dt_bias"])


def test_ssd_handoff_timeout_is_reported(ssm):
    """A dropped state hand-off between time segments (host-requested test hook) makes the
    successor's bounded wait run out: the call reports SSM_ERR_TIMEOUT, and the next call
    on the same workspace is correct again (the GPU stays usable)."""
    from selective_state_space_47_b200 import _native
    inp = synth.ssd_inputs(1, 4097, 2, seed=4097 + 90, gate=True, h0=False)  # three segments per head
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    args = [dev[k] for k in ("x", "dt", "A", "B", "C", "D", "z", "dt_bias")]
    ws = ssm.ScanWorkspace()
    ssm.ssd_fwd(*args, workspace=ws, _test_flags=_native.SSM_TEST_DROP_HANDOFF)
    assert ssm.workspace_status(ws) == _native.SSM_ERR_TIMEOUT
    y = ssm.ssd_fwd(*args, workspace=ws)
    assert ssm.workspace_status(ws) == _native.SSM_OK
    y_ref, _ = oracle_ssd(inp)
    err = rowwise_rel(y.float().cpu().numpy().reshape(1, 4097, 2 * 64), y_ref.reshape(1, 4097, 2 * 64), axis=1)
    assert err <= 1e-2, err
