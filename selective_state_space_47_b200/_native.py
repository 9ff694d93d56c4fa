"""ctypes view of the C ABI declared in include/ssm_scan.h (argument marshalling only)."""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libssmscan.so")

SSM_OK, SSM_ERR_INVALID, SSM_ERR_UNSUPPORTED, SSM_ERR_CUDA, SSM_ERR_TIMEOUT = range(5)
SSM_F32, SSM_BF16 = 0, 1
SSM_DELTA_SOFTPLUS = 1
SSM_A_GENERAL = 2
SSM_EXACT_ZOH = 4
SSM_SEQ_PARALLEL = 8
SSM_SEQ_HANDOFF = 16
SSM_TEST_SHORT_SEGMENTS = 0x40000000
SSM_TEST_DROP_HANDOFF = 0x80000000

# Every symbol the header declares (checked by the CPU test suite).
EXPORTS = ("ssm_scan_workspace_size", "ssm_scan_fwd", "ssm_step", "ssm_step_conv", "ssm_workspace_status",
           "ssm_status_string", "ssm_scan_fwd_noalloc", "ssm_noalloc_status", "ssm_scan_host_staging_size",
           "ssm_scan_fwd_host", "ssm_scan_bwd_workspace_size", "ssm_scan_bwd", "ssm_ssd_workspace_size",
           "ssm_ssd_fwd")


class ScanArgs(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
        ("dstate", ctypes.c_int64), ("dtype", ctypes.c_int), ("flags", ctypes.c_uint32),
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("z", ctypes.c_void_p),
        ("Bm", ctypes.c_void_p), ("Cm", ctypes.c_void_p), ("A", ctypes.c_void_p),
        ("Dskip", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("h0", ctypes.c_void_p),
        ("y", ctypes.c_void_p), ("h_last", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p), ("conv_x0", ctypes.c_void_p),
    ]


class ScanBwdArgs(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
        ("dstate", ctypes.c_int64), ("dtype", ctypes.c_int), ("flags", ctypes.c_uint32),
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("z", ctypes.c_void_p),
        ("Bm", ctypes.c_void_p), ("Cm", ctypes.c_void_p), ("A", ctypes.c_void_p),
        ("Dskip", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("h0", ctypes.c_void_p),
        ("dy", ctypes.c_void_p), ("dh_last", ctypes.c_void_p), ("dx", ctypes.c_void_p),
        ("ddt", ctypes.c_void_p), ("dz", ctypes.c_void_p), ("dB", ctypes.c_void_p), ("dC", ctypes.c_void_p),
        ("dA", ctypes.c_void_p), ("dD", ctypes.c_void_p), ("ddt_bias", ctypes.c_void_p), ("dh0", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p), ("conv_x0", ctypes.c_void_p),
        ("dconv_w", ctypes.c_void_p), ("dconv_b", ctypes.c_void_p), ("dconv_x0", ctypes.c_void_p),
    ]


class SsdArgs(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
        ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("dtype", ctypes.c_int),
        ("flags", ctypes.c_uint32), ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("z", ctypes.c_void_p),
        ("Bm", ctypes.c_void_p), ("Cm", ctypes.c_void_p), ("A", ctypes.c_void_p), ("Dskip", ctypes.c_void_p),
        ("dt_bias", ctypes.c_void_p), ("h0", ctypes.c_void_p), ("y", ctypes.c_void_p),
        ("h_last", ctypes.c_void_p), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


_lib = None


def lib():
    """Load libssmscan.so. There is no fallback: a missing library is an error."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m selective_state_space_47_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        L.ssm_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs)]
        L.ssm_scan_workspace_size.restype = ctypes.c_size_t
        L.ssm_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), vp]
        L.ssm_scan_fwd.restype = ctypes.c_int
        L.ssm_scan_fwd_noalloc.argtypes = [ctypes.POINTER(ScanArgs), vp]
        L.ssm_scan_fwd_noalloc.restype = ctypes.c_int
        L.ssm_ssd_workspace_size.argtypes = [ctypes.POINTER(SsdArgs)]
        L.ssm_ssd_workspace_size.restype = ctypes.c_size_t
        L.ssm_ssd_fwd.argtypes = [ctypes.POINTER(SsdArgs), vp]
        L.ssm_ssd_fwd.restype = ctypes.c_int
        L.ssm_noalloc_status.argtypes = [vp]
        L.ssm_noalloc_status.restype = ctypes.c_int
        L.ssm_scan_host_staging_size.argtypes = [ctypes.POINTER(ScanArgs), i64]
        L.ssm_scan_host_staging_size.restype = ctypes.c_size_t
        L.ssm_scan_fwd_host.argtypes = [ctypes.POINTER(ScanArgs), i64, vp, ctypes.c_size_t, vp]
        L.ssm_scan_fwd_host.restype = ctypes.c_int
        L.ssm_step.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_uint32] + [vp] * 10 + [vp]
        L.ssm_step.restype = ctypes.c_int
        L.ssm_step_conv.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_uint32] + [vp] * 13 + [vp]
        L.ssm_step_conv.restype = ctypes.c_int
        L.ssm_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(ScanBwdArgs)]
        L.ssm_scan_bwd_workspace_size.restype = ctypes.c_size_t
        L.ssm_scan_bwd.argtypes = [ctypes.POINTER(ScanBwdArgs), vp]
        L.ssm_scan_bwd.restype = ctypes.c_int
        L.ssm_workspace_status.argtypes = [vp, vp]
        L.ssm_workspace_status.restype = ctypes.c_int
        L.ssm_status_string.argtypes = [ctypes.c_int]
        L.ssm_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(code):
    return lib().ssm_status_string(int(code)).decode()


def check(code, what):
    if code != SSM_OK:
        raise RuntimeError(f"{what}: {status_string(code)}")
