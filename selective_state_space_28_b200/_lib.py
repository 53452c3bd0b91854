"""ctypes view of libssm.so (include/ssm.h).  Argument marshalling only.

The library is loaded from this package directory.  If it is missing the
import of the binding raises: there is no fallback of any kind.
"""
import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssm.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "ssm.h")

SSM_F32, SSM_BF16 = 0, 1
SSM_DT_SOFTPLUS, SSM_RMSNORM_BC, SSM_RMSNORM_DT = 1, 2, 4
SSM_STEP_MAMBA1, SSM_STEP_MAMBA2 = 1, 2

STATUS = {0: "SSM_OK", 1: "SSM_ERR_NULL", 2: "SSM_ERR_SHAPE", 3: "SSM_ERR_DTYPE",
          4: "SSM_ERR_ALIGN", 5: "SSM_ERR_UNSUPPORTED", 6: "SSM_ERR_WORKSPACE",
          7: "SSM_ERR_CUDA", 8: "SSM_ERR_TIMEOUT"}

SSM_CONV_SILU = 1

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


class ScanArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("channels", _i64), ("state", _i64),
                ("groups", _i64), ("io", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("rms_eps", ctypes.c_float),
                ("x", _vp), ("dt", _vp), ("z", _vp), ("B", _vp), ("C", _vp),
                ("A", _vp), ("D", _vp), ("dt_bias", _vp), ("h0", _vp),
                ("y", _vp), ("h_last", _vp), ("states", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class SsdArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("heads", _i64), ("head_dim", _i64),
                ("state", _i64), ("groups", _i64), ("chunk", _i64),
                ("io", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("x", _vp), ("z", _vp), ("dt", _vp), ("B", _vp), ("C", _vp),
                ("A", _vp), ("D", _vp), ("dt_bias", _vp), ("h0", _vp),
                ("y", _vp), ("h_last", _vp), ("states", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class SsdConvArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("heads", _i64), ("head_dim", _i64),
                ("state", _i64), ("groups", _i64), ("chunk", _i64),
                ("io", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("xBC", _vp), ("conv_w", _vp), ("conv_bias", _vp), ("conv_state_in", _vp),
                ("conv_state_out", _vp), ("z", _vp), ("dt", _vp),
                ("A", _vp), ("D", _vp), ("dt_bias", _vp), ("h0", _vp),
                ("y", _vp), ("h_last", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class StepArgs(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("io", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("rms_eps", ctypes.c_float),
                ("batch", _i64), ("units", _i64), ("head_dim", _i64), ("state", _i64),
                ("groups", _i64),
                ("x", _vp), ("dt", _vp), ("z", _vp), ("B", _vp), ("C", _vp),
                ("A", _vp), ("D", _vp), ("dt_bias", _vp),
                ("state_io", _vp), ("y", _vp)]


class ConvArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("channels", _i64), ("width", _i64),
                ("io", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("x", _vp), ("w", _vp), ("bias", _vp), ("state_in", _vp),
                ("u", _vp), ("state_out", _vp)]


class GatedNormArgs(ctypes.Structure):
    _fields_ = [("rows", _i64), ("width", _i64), ("io", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("eps", ctypes.c_float),
                ("y", _vp), ("z", _vp), ("weight", _vp), ("out", _vp)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("heads", _i64), ("state", _i64),
                ("groups", _i64), ("io", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("dt", _vp), ("B", _vp), ("C", _vp), ("A", _vp), ("dt_bias", _vp),
                ("alpha", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


def header_functions(path=HEADER):
    """Names of the functions include/ssm.h declares."""
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(\w+)\s*\([^;{]*\)\s*;", text, re.M)))


_lib = None


def lib():
    """The loaded libssm.so, with argument types set.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                "libssm.so is not built (%s); run `python -m selective_state_space_28_b200.build`"
                % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        L.ssm_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), _vp]
        L.ssm_scan_workspace.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ctypes.c_size_t)]
        L.ssd_chunk_scan_fwd.argtypes = [ctypes.POINTER(SsdArgs), _vp]
        L.ssd_chunk_scan_workspace.argtypes = [ctypes.POINTER(SsdArgs),
                                               ctypes.POINTER(ctypes.c_size_t)]
        L.ssd_conv_chunk_scan_fwd.argtypes = [ctypes.POINTER(SsdConvArgs), _vp]
        L.ssd_conv_chunk_scan_workspace.argtypes = [ctypes.POINTER(SsdConvArgs),
                                                    ctypes.POINTER(ctypes.c_size_t)]
        L.ssm_scan_step.argtypes = [ctypes.POINTER(StepArgs), _vp]
        L.ssm_conv1d_fwd.argtypes = [ctypes.POINTER(ConvArgs), _vp]
        L.ssm_gated_rmsnorm_fwd.argtypes = [ctypes.POINTER(GatedNormArgs), _vp]
        L.ssm_scan_fwd_write.argtypes = [ctypes.POINTER(ScanArgs), _i64, _vp, _vp]
        L.ssd_attention_fwd.argtypes = [ctypes.POINTER(AttnArgs), _vp]
        L.ssd_attention_workspace.argtypes = [ctypes.POINTER(AttnArgs),
                                              ctypes.POINTER(ctypes.c_size_t)]
        L.ssm_scan_fwd_static.argtypes = [ctypes.POINTER(ScanArgs), _vp]
        L.ssm_workspace_status.argtypes = [_vp, _vp]
        L.ssm_scan_fwd_host.argtypes = [ctypes.POINTER(ScanArgs), _vp]
        L.ssm_scan_host_workspace.argtypes = [ctypes.POINTER(ScanArgs),
                                              ctypes.POINTER(ctypes.c_size_t)]
        for fn in (L.ssm_scan_fwd_static, L.ssm_workspace_status, L.ssm_scan_fwd_host,
                   L.ssm_scan_host_workspace,
                   L.ssm_scan_fwd, L.ssm_scan_workspace, L.ssd_chunk_scan_fwd,
                   L.ssd_chunk_scan_workspace, L.ssd_conv_chunk_scan_fwd,
                   L.ssd_conv_chunk_scan_workspace, L.ssm_scan_step, L.ssm_conv1d_fwd,
                   L.ssm_gated_rmsnorm_fwd, L.ssm_scan_fwd_write, L.ssd_attention_fwd,
                   L.ssd_attention_workspace):
            fn.restype = ctypes.c_int
        L.ssm_status_string.argtypes = [ctypes.c_int]
        L.ssm_status_string.restype = ctypes.c_char_p
        L.ssm_abi_version.argtypes = []
        L.ssm_abi_version.restype = ctypes.c_int
        _lib = L
    return _lib


class SsmError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = lib().ssm_status_string(status).decode()
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), msg))


def check(status, where):
    if status != 0:
        raise SsmError(status, where)
