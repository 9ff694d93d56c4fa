"""GPU checks of ssm_scan_fwd_host (tokens in host memory, chunked, copies overlapped):
its result must equal ssm_scan_fwd over the whole sequence bit for bit, because the
state passes from chunk to chunk exactly through h0/h_last."""
import pytest
import torch

from selective_state_space_47_b200 import synth
from tests.conftest import cuda_available

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssm():
    if not cuda_available():
        pytest.skip("needs a CUDA device")
    import selective_state_space_47_b200 as m
    return m


HOST_CASES = [
    # (batch, seqlen, dim, dstate, dtype, gate, h0, chunk_len)
    (2, 5000, 256, 16, torch.bfloat16, True, True, 1024),   # five chunks, the last one ragged
    (1, 700, 64, 5, torch.float32, False, False, 256),      # B, C rows not 16-byte multiples
    (3, 100, 32, 16, torch.bfloat16, True, False, 1000),    # one chunk longer than the sequence
    (2, 96, 64, 16, torch.bfloat16, True, True, 32),        # many short chunks
]


@pytest.mark.parametrize("case", HOST_CASES)
def test_host_scan_equals_device_scan(ssm, case):
    Bsz, L, Dm, N, dtype, gate, h0, chunk = case
    cpu = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=31, gate=gate, h0=h0)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in cpu.items()}
    y_dev, h_dev = ssm.scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                dev["dt_bias"], dev.get("h0"), return_last_state=True, seq_parallel=False)
    host = {k: cpu[k].pin_memory() for k in ("x", "dt", "B", "C")}
    z = cpu["z"].pin_memory() if gate else None
    y_host, h_host = ssm.scan_fwd_host(host["x"], host["dt"], dev["A"], host["B"], host["C"], dev["D"], z,
                                       dev["dt_bias"], dev.get("h0"), chunk_len=chunk, return_last_state=True)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())
    assert torch.equal(h_host, h_dev)


def test_host_scan_rejects_device_tokens(ssm):
    cpu = synth.scan_inputs(1, 64, 32, 16, torch.bfloat16, seed=32)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in cpu.items()}
    with pytest.raises(ValueError):
        ssm.scan_fwd_host(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"], dev["dt_bias"])
