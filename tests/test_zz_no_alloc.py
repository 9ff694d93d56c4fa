"""The allocation-free scan entry point, ssm_scan_fwd_noalloc, through the C ABI.

It serves callers that must not allocate device memory (a runtime whose pool owns
all GPU memory, or a real-time loop that cannot take cudaMalloc's synchronisation):
its scratch is a fixed array inside the library. Here its output is compared with
that of ssm_scan_fwd (caller-provided workspace) on two calls in a row, which also
shows that the second call does not see the first call's leftovers in the shared
array. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from selective_state_space_47_b200 import _native, synth
from tests.conftest import cuda_available
from tests.gpu_util import TOL, h_err, rowwise_rel

pytestmark = pytest.mark.gpu


def _args(inp, y, h_last):
    import selective_state_space_47_b200 as ssm
    return ssm._scan_args(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                          inp["dt_bias"], inp.get("h0"), y, h_last, _native.SSM_DELTA_SOFTPLUS)


def test_noalloc_matches_workspace_entry_point():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as ssm
    lib = _native.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    shapes = [(2, 3000, 256, 16, torch.bfloat16, 501, True), (1, 1500, 512, 16, torch.float32, 502, False)]
    for Bsz, L, Dm, N, dt_, seed, h0 in shapes:   # two calls in a row
        cpu = synth.scan_inputs(Bsz, L, Dm, N, dt_, seed=seed, h0=h0)
        inp = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in cpu.items()}
        y_ref, h_ref = ssm.scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    inp["z"], inp["dt_bias"], inp["h0"], return_last_state=True)
        y = torch.full_like(y_ref, float("nan"))
        h = torch.full_like(h_ref, float("nan"))
        a = _args(inp, y, h)
        assert lib.ssm_scan_fwd_noalloc(ctypes.byref(a), stream) == _native.SSM_OK
        torch.cuda.synchronize()
        tol = TOL["bf16" if dt_ == torch.bfloat16 else "f32"]
        ref = y_ref.float().cpu().double().numpy()
        assert rowwise_rel(y.float().cpu().numpy(), ref, axis=1) <= tol
        assert h_err(h, h_ref.cpu().double().numpy()) <= tol


def test_noalloc_rejects_oversized_shapes():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    lib = _native.lib()
    a = _native.ScanArgs()
    a.batch, a.seqlen, a.dim, a.dstate = 8, 16, 8192, 16   # 65,536 channels: beyond the fixed scratch
    a.dtype = _native.SSM_BF16
    assert lib.ssm_scan_fwd_noalloc(ctypes.byref(a), None) == _native.SSM_ERR_UNSUPPORTED
    assert lib.ssm_scan_fwd_noalloc(None, None) == _native.SSM_ERR_INVALID
