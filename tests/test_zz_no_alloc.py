"""The allocation-free scan entry point, ssm_scan_fwd_noalloc, through the C ABI.

It serves callers that must not allocate device memory (a runtime whose pool owns
all GPU memory, or a real-time loop that cannot take cudaMalloc's synchronisation):
its scratch is a fixed array inside the library, shared by every call. Here its output
is compared with the float64 oracle on the same bytes and with ssm_scan_fwd (caller-
provided workspace). Consecutive calls with the same shape and different inputs show
that no call sees its predecessor's leftovers in the shared array (flags or carried
states of the same channel groups), and the array's status word is read back through
ssm_noalloc_status. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from selective_state_space_47_b200 import _native, synth
from tests.conftest import cuda_available
from tests.gpu_util import TOL, h_err, oracle_scan, y_err

pytestmark = pytest.mark.gpu


def _args(inp, y, h_last, flags=_native.SSM_DELTA_SOFTPLUS):
    import selective_state_space_47_b200 as ssm
    return ssm._scan_args(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                          inp["dt_bias"], inp.get("h0"), y, h_last, flags)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_oracle_and_workspace_entry_point():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as ssm
    lib = _native.lib()
    # Calls in a row: the first two share shape and group count (the same flags and carry
    # slots of the shared array) with different inputs; the third changes type and shape.
    shapes = [(2, 3000, 256, 16, torch.bfloat16, 501, True), (2, 3000, 256, 16, torch.bfloat16, 503, False),
              (1, 1500, 512, 16, torch.float32, 502, False)]
    for Bsz, L, Dm, N, dt_, seed, h0 in shapes:
        cpu = synth.scan_inputs(Bsz, L, Dm, N, dt_, seed=seed, h0=h0)
        inp = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in cpu.items()}
        y = torch.full_like(inp["x"], float("nan"))
        h = torch.full((Bsz, Dm, N), float("nan"), dtype=torch.float32, device="cuda")
        a = _args(inp, y, h)
        assert lib.ssm_scan_fwd_noalloc(ctypes.byref(a), _stream()) == _native.SSM_OK
        assert lib.ssm_noalloc_status(_stream()) == _native.SSM_OK
        tol = TOL["bf16" if dt_ == torch.bfloat16 else "f32"]
        y_ref, h_ref = oracle_scan(cpu)
        ey, eh = y_err(y, y_ref), h_err(h, h_ref)
        print(f"noalloc B={Bsz} L={L} D={Dm} {dt_}: y {ey:.2e}, h_L {eh:.2e}")
        assert ey <= tol and eh <= tol
        # the same bytes through the workspace entry point
        y_ws, h_ws = ssm.scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], inp["dt_bias"], inp["h0"], return_last_state=True)
        torch.cuda.synchronize()
        assert y_err(y, y_ws.float().cpu().double().numpy()) <= tol
        assert h_err(h, h_ws.cpu().double().numpy()) <= tol


def test_noalloc_status_reports_a_dropped_handoff():
    """The bounded device wait of the no-alloc path reports through its status word: a
    dropped state hand-off (host-requested test hook) gives SSM_ERR_TIMEOUT, and the next
    normal call is correct and reports SSM_OK."""
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    lib = _native.lib()
    cpu = synth.scan_inputs(1, 4096, 64, 16, torch.bfloat16, seed=14)
    inp = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in cpu.items()}
    y = torch.empty_like(inp["x"])
    a = _args(inp, y, None, _native.SSM_DELTA_SOFTPLUS | _native.SSM_TEST_DROP_HANDOFF)
    assert lib.ssm_scan_fwd_noalloc(ctypes.byref(a), _stream()) == _native.SSM_OK
    assert lib.ssm_noalloc_status(_stream()) == _native.SSM_ERR_TIMEOUT
    a = _args(inp, y, None)
    assert lib.ssm_scan_fwd_noalloc(ctypes.byref(a), _stream()) == _native.SSM_OK
    assert lib.ssm_noalloc_status(_stream()) == _native.SSM_OK
    y_ref, _ = oracle_scan(cpu)
    assert y_err(y, y_ref) <= TOL["bf16"]


def test_noalloc_rejects_oversized_shapes():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    lib = _native.lib()
    Bsz, L, Dm, N = 8, 16, 8192, 16   # 65,536 channels: beyond the fixed scratch
    bf = dict(dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((Bsz, L, Dm), **bf)
    bc = torch.zeros((Bsz, L, N), **bf)
    A = torch.full((Dm, N), -1.0, device="cuda")
    inp = dict(x=x, dt=x, z=None, B=bc, C=bc, A=A, D=None, dt_bias=None)
    a = _args(inp, torch.empty_like(x), None)
    assert lib.ssm_scan_fwd_noalloc(ctypes.byref(a), _stream()) == _native.SSM_ERR_UNSUPPORTED
    assert lib.ssm_scan_fwd_noalloc(None, None) == _native.SSM_ERR_INVALID
