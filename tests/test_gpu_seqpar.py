"""GPU parity of the sequence-parallel evaluation of ssm_scan_fwd (SSM_SEQ_PARALLEL):
a local pass runs every time segment of a channel group from a zero state, a combine
kernel composes the segments' affine maps h -> a h + l along the sequence, and a main
pass runs every segment from its combined start state.

Against the float64 oracle on the same bytes (tolerances as for the scan), with one-tile
segments (test hook SSM_TEST_SHORT_SEGMENTS: every 32-step boundary is a combined carry)
and with the planner's segments; the general and the structured exponential paths, the
exact zero-order hold and the fused short convolution (whose three-token window reaches
across every segment boundary). The hand-off evaluation of the same call is compared
too: both are float32 evaluations of one recurrence and must agree within tolerance.
"""
import ctypes

import numpy as np
import pytest
import torch

from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available
from tests.gpu_util import TOL, dtype_name, h_err, oracle_scan, y_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


def _cuda(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _call(ssm, inp, flags, conv=None):
    """ssm_scan_fwd through the C ABI with explicit flags; returns y, h_last, status."""
    from selective_state_space_47_b200 import _native
    conv = conv or {}
    Bsz, L, Dm = inp["x"].shape
    N = inp["A"].shape[1]
    y = torch.full_like(inp["x"], float("nan"))
    h = torch.full((Bsz, Dm, N), float("nan"), dtype=torch.float32, device="cuda")
    a = ssm._scan_args(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], inp["dt_bias"],
                       inp.get("h0"), y, h, flags, conv.get("conv_w"), conv.get("conv_b"), conv.get("conv_x0"))
    ws = ssm.ScanWorkspace()
    buf = ws.get(_native.lib().ssm_scan_workspace_size(ctypes.byref(a)), y.device)
    a.workspace, a.workspace_bytes = ctypes.c_void_p(buf.data_ptr()), buf.numel()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert _native.lib().ssm_scan_fwd(ctypes.byref(a), stream) == _native.SSM_OK
    return y, h, ssm.workspace_status(ws)


CASES = [
    # (batch, seqlen, dim, dstate, dtype, one-tile segments, h0)
    (1, 4097, 64, 16, torch.float32, True, True),     # 129 segments per group, ragged last tile
    (1, 4097, 64, 16, torch.bfloat16, True, False),
    (2, 5000, 96, 16, torch.bfloat16, False, True),   # the planner's segments, six groups
    (1, 20000, 40, 7, torch.float32, False, True),    # lanes past D, odd dstate, long segments
    (3, 2100, 32, 1, torch.float32, True, False),     # dstate 1, 66 segments x 3 groups
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{str(c[4])[6:]}"
                         f"{'short' if c[5] else ''}")
@pytest.mark.parametrize("general", [False, True], ids=["auto", "generalA"])
def test_seq_parallel_matches_oracle(ssm, case, general):
    from selective_state_space_47_b200 import _native
    Bsz, L, Dm, N, dtype, short, h0 = case
    cpu = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=2000 + L + Dm, h0=h0)
    inp = _cuda(cpu)
    base = _native.SSM_DELTA_SOFTPLUS | (_native.SSM_A_GENERAL if general else 0)
    hook = _native.SSM_TEST_SHORT_SEGMENTS if short else 0
    y, h, st = _call(ssm, inp, base | _native.SSM_SEQ_PARALLEL | hook)
    assert st == _native.SSM_OK
    y_ref, h_ref = oracle_scan(cpu)
    tol = TOL[dtype_name(cpu["x"])]
    # The state's error per (b, d) row over n; with N = 1 a row is a single state, which can
    # be a near-cancelled sum, so there it is taken relative to the largest state instead.
    herr = h_err if N > 1 else (lambda g, r: float(np.abs(g.cpu().double().numpy() - r).max() / np.abs(r).max()))
    ey, eh = y_err(y, y_ref), herr(h, h_ref)
    y_ho, h_ho, st_ho = _call(ssm, inp, base | _native.SSM_SEQ_HANDOFF | hook)
    assert st_ho == _native.SSM_OK
    eh_ho = herr(h_ho, h_ref)
    # the two evaluations against each other, relative to the largest state
    d = float((h - h_ho).abs().max() / h_ho.abs().max())
    print(f"\nseq-parallel {case} general={general}: y {ey:.3e}, h_L {eh:.3e} (hand-off {eh_ho:.3e}); "
          f"max |h_L - hand-off| / max |h_L| {d:.3e}")
    assert ey <= tol and eh <= tol
    assert eh <= 1e-4  # the float32 state regression bound of the scan tests
    assert d <= 1e-5
    assert y_err(y, y_ho.float().cpu().double().numpy()) <= tol


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("zoh,conv", [(True, False), (False, True), (True, True)], ids=["zoh", "conv", "zoh+conv"])
def test_seq_parallel_zoh_and_conv(ssm, zoh, conv, dtype):
    from selective_state_space_47_b200 import _native
    Bsz, L, Dm, N = 2, 3001, 64, 16
    cpu = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=2101, h0=True)
    g = torch.Generator().manual_seed(2102)
    cpu["A"] = -torch.rand((Dm, N), generator=g) * 4.0 - 0.05  # general A
    cv = synth.conv_params(Dm, Bsz, dtype, seed=2103) if conv else None
    flags = (_native.SSM_DELTA_SOFTPLUS | _native.SSM_SEQ_PARALLEL | _native.SSM_TEST_SHORT_SEGMENTS
             | (_native.SSM_EXACT_ZOH if zoh else 0))
    y, h, st = _call(ssm, _cuda(cpu), flags, _cuda(cv) if cv else None)
    assert st == _native.SSM_OK
    y_ref, h_ref = oracle_scan(cpu, exact_zoh=zoh, conv=cv)
    ey, eh = y_err(y, y_ref), h_err(h, h_ref)
    print(f"\nseq-parallel zoh={zoh} conv={conv} {dtype}: y {ey:.3e}, h_L {eh:.3e}")
    tol = TOL[dtype_name(cpu["x"])]
    assert ey <= tol and eh <= tol
    assert eh <= 1e-4


def test_seq_parallel_chosen_for_few_groups(ssm):
    """One channel group over a long sequence: the library's own choice (no flag) is the
    sequence-parallel evaluation, which is correct and gives the same bits as the forced one."""
    from selective_state_space_47_b200 import _native
    cpu = synth.scan_inputs(1, 40000, 32, 16, torch.bfloat16, seed=2104, h0=True)
    inp = _cuda(cpu)
    y_auto, h_auto, _ = _call(ssm, inp, _native.SSM_DELTA_SOFTPLUS)
    y_sp, h_sp, _ = _call(ssm, inp, _native.SSM_DELTA_SOFTPLUS | _native.SSM_SEQ_PARALLEL)
    torch.cuda.synchronize()
    assert torch.equal(y_auto, y_sp) and torch.equal(h_auto, h_sp)
    y_ref, h_ref = oracle_scan(cpu)
    assert y_err(y_auto, y_ref) <= TOL["bf16"] and h_err(h_auto, h_ref) <= 1e-4


def test_seq_parallel_flags_conflict(ssm):
    from selective_state_space_47_b200 import _native
    inp = _cuda(synth.scan_inputs(1, 64, 32, 16, torch.bfloat16, seed=2105))
    a = ssm._scan_args(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], inp["dt_bias"],
                       None, torch.empty_like(inp["x"]), None,
                       _native.SSM_SEQ_PARALLEL | _native.SSM_SEQ_HANDOFF)
    buf = torch.empty(_native.lib().ssm_scan_workspace_size(ctypes.byref(a)), dtype=torch.uint8, device="cuda")
    a.workspace, a.workspace_bytes = ctypes.c_void_p(buf.data_ptr()), buf.numel()
    assert _native.lib().ssm_scan_fwd(ctypes.byref(a), None) == _native.SSM_ERR_INVALID


def test_host_path_chunks_take_the_sequence_parallel_evaluation(ssm):
    """The host-resident path on one channel group: each 4096-step chunk is long enough
    for the sequence-parallel evaluation, and the chunks hand their states on through
    h0 / h_last; the result matches the oracle."""
    cpu = synth.scan_inputs(1, 12000, 32, 16, torch.bfloat16, seed=2106, h0=True)
    host = {k: cpu[k].pin_memory() for k in ("x", "dt", "z", "B", "C")}
    dev = {k: cpu[k].cuda() for k in ("A", "D", "dt_bias", "h0")}
    y, h = ssm.scan_fwd_host(host["x"], host["dt"], dev["A"], host["B"], host["C"], dev["D"], host["z"],
                             dev["dt_bias"], dev["h0"], chunk_len=4096, return_last_state=True)
    torch.cuda.synchronize()
    y_ref, h_ref = oracle_scan(cpu)
    ey, eh = y_err(y, y_ref), h_err(h, h_ref)
    print(f"\nhost path, 4096-step chunks, one group: y {ey:.3e}, h_L {eh:.3e}")
    assert ey <= TOL["bf16"] and eh <= 1e-4


def test_long_narrow_sampled(ssm):
    """long_narrow (B=1, L=262144, D=1024: the benchmark's sequence-parallel leg) at full size
    in that leg's launch configuration (general exponentials, the planner's segments); the
    oracle follows one channel in every one of the 32 groups (at a lane that moves with the
    group) plus the last channel, over all 262144 steps, so every group's chain of combined
    carries is compared at full length."""
    w = synth.WORKLOADS["long_narrow"]
    inp = synth.scan_inputs(w.batch, w.seqlen, w.dim, w.dstate, w.dtype, seed=synth.SEEDS["long_narrow"],
                            device="cuda", gate=w.gate)
    y, h = ssm.scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], inp["dt_bias"],
                        return_last_state=True, general_A=True, seq_parallel=True)
    torch.cuda.synchronize()
    groups = torch.arange(w.dim // 32)
    sel = torch.unique(torch.cat([groups * 32 + (groups * 7) % 32, torch.tensor([w.dim - 1])]))
    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y_ref, h_ref = oracle_scan(cpu, sel=sel)
    e_y, e_h = y_err(y[:, :, sel.cuda()], y_ref), h_err(h[:, sel.cuda()], h_ref)
    print(f"\nlong_narrow ({len(sel)} channels, all steps, sequence-parallel): y {e_y:.3e}, h_L {e_h:.3e}")
    assert e_y <= TOL["bf16"] and e_h <= 1e-4
