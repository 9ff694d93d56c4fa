"""GPU parity of the scan with the block's short causal convolution and SiLU fused in
front of it (conv_w / conv_b / conv_x0): u_t = silu(conv_b + sum_k conv_w[:, k] x_{t-3+k}).

Against the float64 oracle's convolution front end (itself pinned to numpy's
cross-correlation); then properties that need no oracle: a sequence split in two calls
(the second given the first's final state and last three tokens) equals one call bit
for bit, and the host-resident path equals the device path bit for bit, also with
chunks shorter than the convolution's reach.
"""
import pytest
import torch

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


def _cuda(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


CONV_CASES = [
    # (batch, seqlen, dim, dstate, dtype, gate, h0, bias, prefix, exact_zoh, random_A)
    (1, 300, 64, 16, torch.float32, True, True, True, True, False, False),       # ragged last tile
    (2, 2000, 256, 16, torch.bfloat16, True, False, True, True, False, False),
    (1, 8209, 64, 16, torch.bfloat16, True, True, True, False, False, False),     # several time segments
    (2, 129, 40, 5, torch.float32, True, False, False, True, False, True),        # lanes past D; N = 5
    (1, 257, 32, 16, torch.float32, False, True, True, True, True, True),         # exact ZOH, general A
    (3, 2, 32, 16, torch.bfloat16, True, False, True, True, False, False),        # L < 3: prefix and tokens mix
    (2, 1, 64, 16, torch.float32, True, True, True, True, False, False),          # L = 1
]


@pytest.mark.parametrize("case", CONV_CASES)
def test_conv_scan_matches_oracle(ssm, case):
    Bsz, L, Dm, N, dtype, gate, h0, bias, prefix, zoh, random_A = case
    inp = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=51, gate=gate, h0=h0)
    if random_A:
        g = torch.Generator().manual_seed(52)
        inp["A"] = -torch.rand((Dm, N), generator=g) * 4.0 - 0.05
    conv = synth.conv_params(Dm, Bsz, dtype, seed=53, bias=bias, prefix=prefix)
    y_ref, h_ref = oracle_scan(inp, exact_zoh=zoh, conv=conv)
    dev, cv = _cuda(inp), _cuda(conv)
    y, h = ssm.scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"], dev["dt_bias"],
                        dev.get("h0"), exact_zoh=zoh, return_last_state=True, **cv)
    torch.cuda.synchronize()
    tol = TOL[dtype_name(inp["x"])]
    ey, eh = y_err(y, y_ref), h_err(h, h_ref)
    print(f"conv case {case[:5]}: y {ey:.2e}  h {eh:.2e}")
    assert ey <= tol
    assert eh <= tol


@pytest.mark.parametrize("dtype,L,split", [(torch.bfloat16, 5000, 2077), (torch.float32, 700, 1),
                                           (torch.bfloat16, 300, 2)])
def test_split_sequence_equals_one_call(ssm, dtype, L, split):
    """[0, L) in one call == [0, split) then [split, L) from (h_last, last three tokens)."""
    Bsz, Dm, N = 2, 96, 16
    inp = _cuda(synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=54, gate=True, h0=True))
    conv = _cuda(synth.conv_params(Dm, Bsz, dtype, seed=55))
    args = lambda s: [inp[k][:, s].contiguous() for k in ("x", "dt", "B", "C")]
    y, h = ssm.scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], inp["dt_bias"],
                        inp["h0"], return_last_state=True, seq_parallel=False, **conv)
    a, b = slice(0, split), slice(split, L)
    xa, dta, Ba, Ca = args(a)
    xb, dtb, Bb, Cb = args(b)
    ya, ha = ssm.scan_fwd(xa, dta, inp["A"], Ba, Ca, inp["D"], inp["z"][:, a].contiguous(), inp["dt_bias"],
                          inp["h0"], return_last_state=True, seq_parallel=False, **conv)
    # the second call's prefix: the three tokens before `split` (from the first prefix if split < 3)
    x0 = torch.cat([conv["conv_x0"], xa], dim=1)[:, -3:].contiguous()
    yb, hb = ssm.scan_fwd(xb, dtb, inp["A"], Bb, Cb, inp["D"], inp["z"][:, b].contiguous(), inp["dt_bias"], ha,
                          return_last_state=True, conv_w=conv["conv_w"], conv_b=conv["conv_b"], conv_x0=x0,
                          seq_parallel=False)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([ya, yb], dim=1), y)
    assert torch.equal(hb, h)


@pytest.mark.parametrize("chunk", [1000, 2])
def test_host_path_with_conv_equals_device_path(ssm, chunk):
    Bsz, L, Dm, N = 2, 2500, 64, 16
    dtype = torch.bfloat16
    host = synth.scan_inputs(Bsz, L, Dm, N, dtype, seed=56, gate=True, h0=True)
    conv = _cuda(synth.conv_params(Dm, Bsz, dtype, seed=57))
    dev = _cuda(host)
    y_dev, h_dev = ssm.scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                dev["dt_bias"], dev["h0"], return_last_state=True, seq_parallel=False, **conv)
    pin = {k: (v.pin_memory() if k in ("x", "dt", "z", "B", "C") else v) for k, v in host.items()}
    y_host, h_host = ssm.scan_fwd_host(pin["x"], pin["dt"], dev["A"], pin["B"], pin["C"], dev["D"], pin["z"],
                                       dev["dt_bias"], dev["h0"], chunk_len=chunk, return_last_state=True, **conv)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())
    assert torch.equal(h_host, h_dev)


@pytest.mark.parametrize("N", [16, 5])
def test_conv_step_matches_oracle(ssm, N):
    """Decode behind the short convolution: 20 chained steps of ssm_step_conv (two threads
    per channel for N = 16, one for N = 5) against the oracle's step; the window ends as
    the last three tokens, bit for bit."""
    import oracle
    Bsz, Dm, steps = 4, 96, 20
    inp = synth.step_inputs(Bsz, Dm, N, steps, torch.bfloat16, seed=58)
    conv = synth.conv_params(Dm, Bsz, torch.bfloat16, seed=59)
    dev, cv = _cuda(inp), _cuda(conv)
    h = dev["h"].clone()
    hr = inp["h"].double().numpy().copy()
    win = cv["conv_x0"].clone()
    st = synth.to_numpy_storage
    win_r = st(conv["conv_x0"]).copy()
    worst = 0.0
    for s in range(steps):
        y = ssm.step(dev["x"][s], dev["dt"][s], dev["A"], dev["B"][s], dev["C"][s], h, dev["D"], dev["z"][s],
                     dev["dt_bias"], conv_w=cv["conv_w"], conv_b=cv["conv_b"], conv_state=win)
        yr = oracle.step(st(inp["x"][s]), st(inp["dt"][s]), inp["A"].numpy(), st(inp["B"][s]), st(inp["C"][s]),
                         hr, D=inp["D"].numpy(), z=st(inp["z"][s]), dt_bias=inp["dt_bias"].numpy(), dtype="bf16",
                         conv_w=conv["conv_w"].numpy(), conv_b=conv["conv_b"].numpy(), conv_state=win_r)
        worst = max(worst, rowwise_rel(y.float().cpu().numpy(), yr, axis=1))
    torch.cuda.synchronize()
    print(f"conv step N={N}: y {worst:.2e}")
    assert worst <= 1e-2
    assert rowwise_rel(h.cpu().numpy(), hr, axis=2) <= 1e-2
    assert torch.equal(win.cpu(), inp["x"][steps - 3:].permute(1, 0, 2))


def test_prefill_then_conv_step_continues_the_sequence(ssm):
    """A scan with the convolution over L tokens, then one ssm_step_conv from its final
    state and last three tokens, gives the oracle's y at t = L of the L + 1 token scan."""
    Bsz, L, Dm, N = 2, 77, 64, 16
    inp = synth.scan_inputs(Bsz, L + 1, Dm, N, torch.float32, seed=60, gate=True, h0=True)
    conv = synth.conv_params(Dm, Bsz, torch.float32, seed=61)
    y_ref, _ = oracle_scan(inp, conv=conv)
    dev, cv = _cuda(inp), _cuda(conv)
    pre = {k: dev[k][:, :L].contiguous() for k in ("x", "dt", "z", "B", "C")}
    _, hL = ssm.scan_fwd(pre["x"], pre["dt"], dev["A"], pre["B"], pre["C"], dev["D"], pre["z"], dev["dt_bias"],
                         dev["h0"], return_last_state=True, **cv)
    win = dev["x"][:, L - 3:L].contiguous()
    y = ssm.step(dev["x"][:, L].contiguous(), dev["dt"][:, L].contiguous(), dev["A"], dev["B"][:, L].contiguous(),
                 dev["C"][:, L].contiguous(), hL, dev["D"], dev["z"][:, L].contiguous(), dev["dt_bias"],
                 conv_w=cv["conv_w"], conv_b=cv["conv_b"], conv_state=win)
    torch.cuda.synchronize()
    assert rowwise_rel(y.cpu().numpy(), y_ref[:, L], axis=1) <= 1e-4
