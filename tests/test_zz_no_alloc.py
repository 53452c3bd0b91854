"""The allocation-free Mamba-1 scan entry point, ssm_scan_fwd_static.

It serves callers that cannot allocate device memory where they run the scan
(an engine callback limited to memory reserved up front, a latency-bound
decode loop that must not meet an allocator, a process whose device memory
is reserved elsewhere): ssm_scan_fwd needs a caller workspace (a status word,
the step-input RMS factors, segment states), while this entry point uses a
fixed array in the library's own device memory and never cuts the sequence.

The tests call it through the C ABI with only inputs and outputs:
* twice in a row on different inputs (the array keeps the first call's
  contents), each result bit for bit equal to ssm_scan_fwd's on a shape that
  ssm_scan_fwd does not cut either (the same kernel on the same inputs), and
  the first also against the float64 oracle;
* a smaller problem after a larger one (stale factors beyond the new rows
  are never read), again bit for bit;
* a problem that fills the scratch exactly (batch * seqlen = 262144) against
  the oracle, and one row more refused before anything is launched;
* its status word, read through ssm_workspace_status(NULL, stream), is clear.
"""
import ctypes

import pytest
import torch

import oracle
from selective_state_space_28_b200 import _lib as L
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise

pytestmark = pytest.mark.gpu

FLAGS = I.SOFTPLUS | I.RMS_BC | I.RMS_DT
CAPACITY = 1 << 18  # batch * seqlen RMS factors the static scratch holds


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


def _static(dv):
    """One ssm_scan_fwd_static call; returns (y, h_last) after the stream ends."""
    b, Lq, C = dv["x"].shape
    N = dv["B"].shape[3]
    y = torch.empty_like(dv["x"])
    h_last = torch.empty((b, C, N), dtype=torch.float32, device=dv["x"].device)
    stream = torch.cuda.current_stream().cuda_stream
    status = L.lib().ssm_scan_fwd_static(ctypes.byref(_args(dv, y, h_last)), stream)
    assert status == 0, L.lib().ssm_status_string(status)
    assert L.lib().ssm_workspace_status(None, stream) == 0  # no wait ran out
    return y, h_last


def _with_workspace(dv):
    from selective_state_space_28_b200 import ops
    y, h, _ = ops.ssm_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], D=dv["D"],
                               z=dv["z"], dt_bias=dv["dt_bias"], flags=FLAGS, rms_eps=1e-6,
                               check=True)
    return y, h


def _not_cut(dv):
    """ssm_scan_fwd runs this shape as one pass (workspace = status word and
    the step-norm factors only), so both entry points run the same launch."""
    b, Lq, C = dv["x"].shape
    a = L.ScanArgs(batch=b, seqlen=Lq, channels=C, state=dv["B"].shape[3], groups=1,
                   io=L.SSM_BF16, flags=FLAGS, rms_eps=1e-6)
    n = ctypes.c_size_t(0)
    L.check(L.lib().ssm_scan_workspace(ctypes.byref(a), ctypes.byref(n)), "ws")
    return n.value == 256 + ((b * Lq * 4 + 255) // 256) * 256


def _inputs(b, Lq, C, seed):
    d = I.m1_inputs(b, Lq, C, 16, io="bf16", gate=True, seed=seed)
    return d, {k: (v.cuda() if v is not None else None) for k, v in d.items()}


def test_static_entry_rejects_problems_beyond_its_scratch():
    fn = L.lib().ssm_scan_fwd_static
    big = L.ScanArgs(batch=2, seqlen=CAPACITY // 2 + 1, channels=64, state=16, groups=1,
                     io=L.SSM_BF16, flags=FLAGS, rms_eps=1e-6, x=16, dt=16, B=16, C=16, A=16,
                     y=16)
    assert fn(ctypes.byref(big), None) == 6  # SSM_ERR_WORKSPACE, nothing launched


def test_static_entry_matches_workspace_entry_bitwise(cuda_ok):
    first = None
    for seed in (31, 32):
        d, dv = _inputs(4, 300, 1536, seed)
        assert _not_cut(dv)
        y, h = _static(dv)
        y_ref, h_ref = _with_workspace(dv)
        assert torch.equal(y, y_ref) and torch.equal(h, h_ref)
        if first is None:
            first = (d, y, h)
    d, y, h = first  # the first call, against the oracle
    ry, rh, _ = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                               dt_bias=d["dt_bias"], flags=FLAGS, rms_eps=1e-6)
    assert_close_normwise(y, ry, REL[torch.bfloat16], "y")
    assert_close_normwise(h, rh, REL[torch.bfloat16], "h_last")


def test_static_entry_smaller_problem_after_a_larger_one(cuda_ok):
    _, dv = _inputs(8, 1000, 1536, 33)
    _static(dv)  # fills 8000 factors
    d, dv = _inputs(1, 100, 1536, 34)
    assert _not_cut(dv)
    y, h = _static(dv)
    y_ref, h_ref = _with_workspace(dv)
    assert torch.equal(y, y_ref) and torch.equal(h, h_ref)


def test_static_entry_at_its_capacity(cuda_ok):
    """batch * seqlen = 262144 uses every factor of the scratch."""
    d, dv = _inputs(2, CAPACITY // 2, 8, 35)
    y, h = _static(dv)
    ry, rh, _ = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                               dt_bias=d["dt_bias"], flags=FLAGS, rms_eps=1e-6)
    assert_close_normwise(y, ry, REL[torch.bfloat16], "y")
    assert_close_normwise(h, rh, REL[torch.bfloat16], "h_last")
