"""CPU checks of the C ABI: the library loads, exports what the header declares, and
rejects bad arguments on the host before any CUDA call. No compute runs here."""
import ctypes
import os
import re
import subprocess

import pytest

from selective_state_space_47_b200 import _native
from selective_state_space_47_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_scan.h")


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return _native.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(ssm_\w+)\s*\(", text, flags=re.M))


def test_header_and_exports_agree(lib):
    declared = _declared_functions()
    assert declared == set(_native.EXPORTS)
    out = subprocess.check_output(["nm", "-D", "--defined-only", _native.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (ssm_\w+)$", out, flags=re.M))
    assert declared <= exported, f"missing exports: {declared - exported}"
    for name in declared:
        assert hasattr(lib, name)


@pytest.mark.parametrize("cname,pyname", [("ssm_scan_args", "ScanArgs"), ("ssm_scan_bwd_args", "ScanBwdArgs"),
                                          ("ssm_ssd_args", "SsdArgs")])
def test_args_struct_layout_matches_binding(tmp_path, cname, pyname):
    """The ctypes mirrors of the argument structs have the C compiler's field offsets and size."""
    cls = getattr(_native, pyname)
    names = [f[0] for f in cls._fields_]
    src = tmp_path / "layout.c"
    body = "".join(f'printf("%zu\\n", offsetof({cname}, {n}));' for n in names)
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "ssm_scan.h"\n'
                   f'int main(void){{ {body} printf("%zu\\n", sizeof({cname})); return 0; }}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = [int(v) for v in subprocess.check_output([str(exe)]).decode().split()]
    want = [getattr(cls, n).offset for n in names] + [ctypes.sizeof(cls)]
    assert got == want


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "ssm_scan.h"\nint main(void){ ssm_scan_args a = {0}; (void)a;'
                   ' return (int)ssm_scan_workspace_size(&a) * 0; }\n')
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only",
                           "-I", os.path.join(ROOT, "include"), str(src)])


def test_status_strings(lib):
    for code in range(5):
        assert _native.status_string(code).startswith("SSM_")
    assert "unknown" in _native.status_string(99)


def _args(**kw):
    a = _native.ScanArgs()
    a.batch, a.seqlen, a.dim, a.dstate = 2, 64, 32, 16
    a.dtype = _native.SSM_BF16
    a.flags = _native.SSM_DELTA_SOFTPLUS
    fake = 1 << 20  # host-side stand-ins: never dereferenced, the calls must fail first
    for name in ("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias", "h0", "y", "h_last"):
        setattr(a, name, fake)
        fake += 1 << 16
    a.workspace = fake
    a.workspace_bytes = lib_ws(a)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def lib_ws(a):
    return _native.lib().ssm_scan_workspace_size(ctypes.byref(a))


def test_workspace_size(lib):
    a = _args()
    a.batch, a.seqlen, a.dim = 1, 262144, 5120
    n = lib_ws(a)
    # per-group flags (rounded) plus one float32 state of 16 per channel: the hand-over part
    handover = 256 * ((256 + 4 * (5120 // 16) + 255) // 256) + 5120 * 16 * 4
    assert handover < 400_000
    # then, 256-aligned, the sequence-parallel area: 1024 items x (two [4][32] float4 states
    # + [4][32] float sums)
    assert n == 256 * ((handover + 255) // 256) + 1024 * (2 * 4 * 32 * 16 + 4 * 32 * 4)
    a.batch = -1
    assert lib_ws(a) == 0
    assert lib.ssm_scan_workspace_size(None) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(dstate=17), _native.SSM_ERR_UNSUPPORTED),
    (dict(dstate=0), _native.SSM_ERR_INVALID),
    (dict(dim=12), _native.SSM_ERR_UNSUPPORTED),          # bf16 needs dim % 8 == 0
    (dict(dtype=7), _native.SSM_ERR_INVALID),
    (dict(flags=0x40), _native.SSM_ERR_INVALID),
    (dict(flags=_native.SSM_SEQ_PARALLEL | _native.SSM_SEQ_HANDOFF), _native.SSM_ERR_INVALID),
    (dict(seqlen=-1), _native.SSM_ERR_INVALID),
    (dict(x=None), _native.SSM_ERR_INVALID),
    (dict(Bm=None), _native.SSM_ERR_INVALID),
    (dict(y=None), _native.SSM_ERR_INVALID),
    (dict(A=None), _native.SSM_ERR_INVALID),
    (dict(x=(1 << 20) + 4), _native.SSM_ERR_UNSUPPORTED),  # misaligned
    (dict(y=(1 << 20) + 8), _native.SSM_ERR_UNSUPPORTED),
    (dict(h_last=(1 << 20) + 2), _native.SSM_ERR_UNSUPPORTED),
    (dict(Bm=(1 << 20) + 1), _native.SSM_ERR_UNSUPPORTED),
    (dict(workspace=(1 << 20) + 8), _native.SSM_ERR_UNSUPPORTED),
    (dict(workspace=None), _native.SSM_ERR_INVALID),
    (dict(workspace_bytes=100), _native.SSM_ERR_INVALID),
    (dict(conv_b=1 << 30), _native.SSM_ERR_INVALID),                         # bias without taps
    (dict(conv_x0=1 << 30), _native.SSM_ERR_INVALID),                        # prefix without taps
    (dict(conv_w=(1 << 30) + 4), _native.SSM_ERR_UNSUPPORTED),               # taps: one float4 per channel
    (dict(conv_w=1 << 30, conv_x0=(1 << 30) + 1), _native.SSM_ERR_UNSUPPORTED),  # bf16 prefix on 2 bytes
    (dict(conv_w=1 << 30, conv_b=(1 << 30) + 2), _native.SSM_ERR_UNSUPPORTED),
])
def test_scan_rejects_on_host(lib, bad, code):
    a = _args(**bad)
    assert lib.ssm_scan_fwd(ctypes.byref(a), None) == code
    assert lib.ssm_scan_fwd(None, None) == _native.SSM_ERR_INVALID


def test_scan_empty_batch_is_a_no_op(lib):
    a = _args(batch=0)
    assert lib.ssm_scan_fwd(ctypes.byref(a), None) == _native.SSM_OK


def test_step_rejects_on_host(lib):
    f = 1 << 20
    ptrs = [f + (i << 16) for i in range(10)]
    call = lambda *a: lib.ssm_step(*a)
    assert call(2, 32, 17, 1, 1, *ptrs, None) == _native.SSM_ERR_UNSUPPORTED
    assert call(2, 32, 16, 3, 1, *ptrs, None) == _native.SSM_ERR_INVALID
    assert call(-1, 32, 16, 1, 1, *ptrs, None) == _native.SSM_ERR_INVALID
    bad = list(ptrs)
    bad[0] = None
    assert call(2, 32, 16, 1, 1, *bad, None) == _native.SSM_ERR_INVALID
    bad = list(ptrs)
    bad[8] = f + 4                      # h must start on 16 bytes when dstate == 16
    assert call(2, 32, 16, 1, 1, *bad, None) == _native.SSM_ERR_UNSUPPORTED
    bad[8] = f + 2                      # and on 4 bytes otherwise
    assert call(2, 32, 5, 1, 1, *bad, None) == _native.SSM_ERR_UNSUPPORTED
    bad = list(ptrs)
    bad[0] = f + 1                      # bf16 token pointer not on its element size
    assert call(2, 32, 16, 1, 1, *bad, None) == _native.SSM_ERR_UNSUPPORTED
    assert call(0, 32, 16, 1, 1, *ptrs, None) == _native.SSM_OK


def test_step_conv_rejects_on_host(lib):
    """ssm_step_conv: the taps and the window are required; alignment as documented."""
    f = 1 << 20
    p = [f + (i << 16) for i in range(15)]
    # x dt z Bm Cm A Dskip dt_bias conv_w conv_b conv_state h y
    args = lambda **kw: [kw.get(k, v) for k, v in zip(
        ("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias", "conv_w", "conv_b", "conv_state", "h", "y"), p)]
    call = lambda *a: lib.ssm_step_conv(2, 32, 16, 1, 1, *a, None)
    assert call(*args(conv_w=None)) == _native.SSM_ERR_INVALID
    assert call(*args(conv_state=None)) == _native.SSM_ERR_INVALID
    assert call(*args(conv_w=f + 4)) == _native.SSM_ERR_UNSUPPORTED      # taps on 16 bytes
    assert call(*args(conv_b=f + 2)) == _native.SSM_ERR_UNSUPPORTED      # bias on 4 bytes
    assert call(*args(conv_state=f + 1)) == _native.SSM_ERR_UNSUPPORTED  # bf16 window on 2 bytes
    assert lib.ssm_step_conv(2, 32, 17, 1, 1, *args(), None) == _native.SSM_ERR_UNSUPPORTED
    assert lib.ssm_step_conv(0, 32, 16, 1, 1, *args(), None) == _native.SSM_OK


def test_python_binding_refuses_cpu_tensors():
    import torch
    import selective_state_space_47_b200 as ssm
    x = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        ssm.scan_fwd(x, x, torch.zeros(8, 16), torch.zeros(1, 4, 16), torch.zeros(1, 4, 16))


def test_python_binding_checks_chunked_form_arguments():
    """ssd_fwd refuses host tensors and wrong shapes before any CUDA call."""
    import torch
    import selective_state_space_47_b200 as ssm
    Bsz, L, H = 1, 4, 2
    x = torch.zeros(Bsz, L, H, 64, dtype=torch.bfloat16)
    dt = torch.zeros(Bsz, L, H, dtype=torch.bfloat16)
    Bm = torch.zeros(Bsz, L, 128, dtype=torch.bfloat16)
    A = torch.zeros(H)
    with pytest.raises(ValueError):  # host tensors
        ssm.ssd_fwd(x, dt, A, Bm, Bm)
    with pytest.raises(ValueError):  # x must be [B, L, H, P]
        ssm.ssd_fwd(x[0], dt, A, Bm, Bm)
    with pytest.raises(ValueError):  # dt per head, not per channel
        ssm.ssd_fwd(x, torch.zeros(Bsz, L, H * 64, dtype=torch.bfloat16), A, Bm, Bm)


def test_host_scan_staging_size_and_argument_checks(lib):
    """ssm_scan_fwd_host: staging size arithmetic and the checks made before any CUDA call."""
    a = _args()
    a.batch, a.seqlen, a.dim, a.dstate = 3, 1000, 64, 16
    up = lambda v: (v + 255) // 256 * 256
    Lc = 256
    tok, bc = up(3 * Lc * 64 * 2), up(3 * Lc * 16 * 2)
    carry = up(3 * 64 * 16 * 4)
    assert lib.ssm_scan_host_staging_size(ctypes.byref(a), Lc) == 2 * (4 * tok + 2 * bc) + 2 * carry
    # chunks longer than the sequence are sized for the sequence
    assert lib.ssm_scan_host_staging_size(ctypes.byref(a), 10**6) == lib.ssm_scan_host_staging_size(
        ctypes.byref(a), 1000)
    assert lib.ssm_scan_host_staging_size(ctypes.byref(a), 0) == 0
    need = lib.ssm_scan_host_staging_size(ctypes.byref(a), Lc)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: every case below fails first
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), 0, fake, need, None) == _native.SSM_ERR_INVALID
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), Lc, None, need, None) == _native.SSM_ERR_INVALID
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), Lc, ctypes.c_void_p((1 << 20) + 16), need, None) == \
        _native.SSM_ERR_UNSUPPORTED
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), Lc, fake, need - 1, None) == _native.SSM_ERR_INVALID
    # with the short convolution each buffer also holds the three tokens before its chunk
    a.conv_w = 1 << 30
    assert lib.ssm_scan_host_staging_size(ctypes.byref(a), Lc) == 2 * (4 * tok + 2 * bc + up(3 * 3 * 64 * 2)) + \
        2 * carry


def _bwd_args(**kw):
    a = _native.ScanBwdArgs()
    a.batch, a.seqlen, a.dim, a.dstate = 2, 100, 64, 16
    a.dtype = _native.SSM_BF16
    a.flags = _native.SSM_DELTA_SOFTPLUS
    fake = 1 << 20  # host-side stand-ins: never dereferenced, the calls must fail first
    for name in ("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias", "h0", "dy", "dh_last", "dx", "ddt", "dz",
                 "dB", "dC", "dA", "dD", "ddt_bias", "dh0"):
        setattr(a, name, fake)
        fake += 1 << 16
    a.workspace = fake
    a.workspace_bytes = 1 << 40
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_bwd_workspace_size(lib):
    """Checkpoints: one float4 per (group, 32-step chunk, warp, lane) and one float per
    (group, chunk, lane); per (group, segment) item four float4 per (warp, lane) and one
    float per lane. Segments: whole chunks, about 1800 items in all."""
    a = _bwd_args()
    a.batch, a.seqlen, a.dim = 3, 1000, 100             # 12 groups, 32 chunks: one chunk per segment
    G, nch, K = 12, 32, 32
    assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(a)) == \
        G * nch * 2048 + 4 * G * K * 2048 + G * K * 128 + G * nch * 128
    a.batch, a.seqlen, a.dim = 1, 262144, 5120           # 160 groups, 8192 chunks: 729 per segment
    G, nch, K = 160, 8192, 12
    assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(a)) == \
        G * nch * 2048 + 4 * G * K * 2048 + G * K * 128 + G * nch * 128
    # with the short convolution: u (bf16) and dL/du (float32) after it, each on 256 bytes
    base = G * nch * 2048 + 4 * G * K * 2048 + G * K * 128 + G * nch * 128
    a.conv_w = 1 << 32
    r256 = lambda v: (v + 255) // 256 * 256
    n_tok = 262144 * 5120
    assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(a)) == r256(r256(base) + 2 * n_tok) + 4 * n_tok
    a.conv_w = None
    a.seqlen = -1
    assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(a)) == 0
    assert lib.ssm_scan_bwd_workspace_size(None) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(flags=0x40), _native.SSM_ERR_INVALID),
    (dict(conv_b=4294967296), _native.SSM_ERR_INVALID),                            # convolution bias without taps
    (dict(dconv_w=4294967296), _native.SSM_ERR_INVALID),                           # its gradient without taps
    (dict(conv_w=4294967296, dconv_b=4294967552), _native.SSM_ERR_INVALID),          # taps without dconv_w
    (dict(conv_w=4294967296, dconv_w=4294967552), _native.SSM_ERR_INVALID),          # taps without dconv_b
    (dict(conv_w=4294967296, dconv_w=4294967552, dconv_b=4294967808, conv_x0=4294968064),
     _native.SSM_ERR_INVALID),                                              # prefix without its gradient
    (dict(conv_w=4294967300, dconv_w=4294967552, dconv_b=4294967808), _native.SSM_ERR_UNSUPPORTED),  # taps: float4
    (dict(conv_w=4294967296, dconv_w=4294967552, dconv_b=4294967808, conv_x0=4294968065, dconv_x0=4294968320),
     _native.SSM_ERR_UNSUPPORTED),                                          # bf16 prefix on 2 bytes
    (dict(flags=_native.SSM_SEQ_PARALLEL | _native.SSM_SEQ_HANDOFF), _native.SSM_ERR_INVALID),
    (dict(dstate=17), _native.SSM_ERR_UNSUPPORTED),
    (dict(dim=12), _native.SSM_ERR_UNSUPPORTED),
    (dict(dz=None), _native.SSM_ERR_INVALID),              # z given without dz
    (dict(z=None), _native.SSM_ERR_INVALID),               # dz given without z
    (dict(dy=None), _native.SSM_ERR_INVALID),
    (dict(dB=None), _native.SSM_ERR_INVALID),
    (dict(dA=None), _native.SSM_ERR_INVALID),
    (dict(dy=(1 << 20) + 8), _native.SSM_ERR_UNSUPPORTED),  # copied 16 bytes at a time
    (dict(dx=(1 << 20) + 1), _native.SSM_ERR_UNSUPPORTED),
    (dict(dA=(1 << 20) + 2), _native.SSM_ERR_UNSUPPORTED),
    (dict(workspace=None), _native.SSM_ERR_INVALID),
    (dict(workspace_bytes=64), _native.SSM_ERR_INVALID),
])
def test_bwd_rejects_on_host(lib, bad, code):
    a = _bwd_args(**bad)
    assert lib.ssm_scan_bwd(ctypes.byref(a), None) == code
    assert lib.ssm_scan_bwd(None, None) == _native.SSM_ERR_INVALID
    assert lib.ssm_scan_bwd(ctypes.byref(_bwd_args(batch=0)), None) == _native.SSM_OK


def _ssd_args(**kw):
    a = _native.SsdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate = 2, 300, 3, 64, 128
    a.dtype = _native.SSM_BF16
    a.flags = _native.SSM_DELTA_SOFTPLUS
    fake = 1 << 20  # host-side stand-ins: never dereferenced, the calls must fail first
    for name in ("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias", "h0", "y", "h_last"):
        setattr(a, name, fake)
        fake += 1 << 16
    a.workspace = fake
    a.workspace_bytes = 1 << 40
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_ssd_workspace_size(lib):
    """The chunked form's workspace: a 256-byte header (item counter, status word) and a
    32-bit flag per (sequence, head), rounded up to 256 bytes, then the float32 state handed
    between time segments, N x P floats per (sequence, head)."""
    a = _ssd_args()
    bh = 2 * 3
    head = (256 + bh * 4 + 255) // 256 * 256
    assert lib.ssm_ssd_workspace_size(ctypes.byref(a)) == head + bh * 128 * 64 * 4
    assert lib.ssm_ssd_workspace_size(ctypes.byref(_ssd_args(batch=-1))) == 0
    assert lib.ssm_ssd_workspace_size(None) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(flags=_native.SSM_DELTA_SOFTPLUS | _native.SSM_EXACT_ZOH), _native.SSM_ERR_INVALID),      # the scan's flags only
    (dict(flags=_native.SSM_DELTA_SOFTPLUS | _native.SSM_SEQ_PARALLEL), _native.SSM_ERR_INVALID),
    (dict(headdim=32), _native.SSM_ERR_UNSUPPORTED),       # the Mamba-2 head shape only
    (dict(dstate=64), _native.SSM_ERR_UNSUPPORTED),
    (dict(dtype=_native.SSM_F32), _native.SSM_ERR_UNSUPPORTED),
    (dict(seqlen=-1), _native.SSM_ERR_INVALID),
    (dict(x=None), _native.SSM_ERR_INVALID),
    (dict(A=None), _native.SSM_ERR_INVALID),
    (dict(y=None), _native.SSM_ERR_INVALID),
    (dict(y=(1 << 20) + 8), _native.SSM_ERR_UNSUPPORTED),  # tiles move 16 bytes at a time
    (dict(A=(1 << 20) + 2), _native.SSM_ERR_UNSUPPORTED),
    (dict(dt=(1 << 20) + 1), _native.SSM_ERR_UNSUPPORTED),
    (dict(workspace=None), _native.SSM_ERR_INVALID),
    (dict(workspace_bytes=64), _native.SSM_ERR_INVALID),
])
def test_ssd_rejects_on_host(lib, bad, code):
    assert lib.ssm_ssd_fwd(ctypes.byref(_ssd_args(**bad)), None) == code


def test_ssd_accepts_its_test_hook_and_empty_shapes(lib):
    """The dropped-hand-off hook passes validation; an empty batch or no heads is a no-op
    that returns before any CUDA call."""
    hook = _native.SSM_DELTA_SOFTPLUS | _native.SSM_TEST_DROP_HANDOFF
    assert lib.ssm_ssd_fwd(ctypes.byref(_ssd_args(batch=0, flags=hook)), None) == _native.SSM_OK
    assert lib.ssm_ssd_fwd(ctypes.byref(_ssd_args(nheads=0)), None) == _native.SSM_OK
    assert lib.ssm_ssd_fwd(None, None) == _native.SSM_ERR_INVALID
