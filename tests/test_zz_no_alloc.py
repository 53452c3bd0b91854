"""The allocation-free Mamba-1 scan entry point, ssm_scan_fwd_static.

It serves callers that cannot allocate device memory where they run the scan
(an engine callback limited to memory reserved up front, a latency-bound
decode loop that must not meet an allocator, a process whose device memory
is reserved elsewhere): with the step-input RMS norm on, ssm_scan_fwd needs a
caller workspace, while this entry point uses a fixed array in the library's
own device memory.  The test calls it through the C ABI with only inputs and
outputs, twice in a row on different inputs (the array keeps the first
call's contents), and compares each result with ssm_scan_fwd's.
"""
import ctypes

import pytest
import torch

from selective_state_space_28_b200 import _lib as L
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise

pytestmark = pytest.mark.gpu

FLAGS = I.SOFTPLUS | I.RMS_BC | I.RMS_DT


def _static_fn():
    fn = L.lib().ssm_scan_fwd_static
    fn.argtypes = [ctypes.POINTER(L.ScanArgs), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _args(d, y, h_last, **kw):
    b, Lq, C = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    a = dict(batch=b, seqlen=Lq, channels=C, state=N, groups=G, io=L.SSM_BF16, flags=FLAGS,
             rms_eps=1e-6, x=d["x"].data_ptr(), dt=d["dt"].data_ptr(), z=d["z"].data_ptr(),
             B=d["B"].data_ptr(), C=d["C"].data_ptr(), A=d["A"].data_ptr(),
             D=d["D"].data_ptr(), dt_bias=d["dt_bias"].data_ptr(), h0=None,
             y=y.data_ptr(), h_last=h_last.data_ptr(), states=None)
    a.update(kw)
    return L.ScanArgs(**a)


def test_static_entry_rejects_problems_beyond_its_scratch():
    fn = _static_fn()
    big = L.ScanArgs(batch=2, seqlen=200000, channels=64, state=16, groups=1, io=L.SSM_BF16,
                     flags=FLAGS, rms_eps=1e-6)
    assert fn(ctypes.byref(big), None) == 6  # SSM_ERR_WORKSPACE, nothing launched


def test_static_entry_matches_workspace_entry(cuda_ok):
    from selective_state_space_28_b200 import ops
    fn = _static_fn()
    stream = torch.cuda.current_stream().cuda_stream
    for seed in (31, 32):
        d = I.m1_inputs(3, 300, 256, 16, io="bf16", gate=True, seed=seed)
        dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
        y_ref, h_ref, _ = ops.ssm_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"],
                                           D=dv["D"], z=dv["z"], dt_bias=dv["dt_bias"],
                                           flags=FLAGS, rms_eps=1e-6)
        y = torch.empty_like(dv["x"])
        h_last = torch.empty_like(h_ref)
        status = fn(ctypes.byref(_args(dv, y, h_last)), stream)
        assert status == 0, L.lib().ssm_status_string(status)
        torch.cuda.synchronize()
        assert_close_normwise(y, y_ref.double().cpu().numpy(), REL[torch.bfloat16], "y")
        assert_close_normwise(h_last, h_ref.double().cpu().numpy(), REL[torch.bfloat16],
                              "h_last")
