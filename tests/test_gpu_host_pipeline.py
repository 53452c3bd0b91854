"""GPU parity of ssm_scan_fwd_host (host buffers in and out, the copies in
both directions overlapped with the scans over batch-row chunks): bitwise
equal to ssm_scan_fwd on device copies of the same inputs, and close to the
float64 oracle."""
import pytest
import torch

import oracle
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise

pytestmark = pytest.mark.gpu


def _ops():
    from selective_state_space_28_b200 import ops
    return ops


def _call(d, h0, pinned=None, flags=I.SOFTPLUS, eps=1e-6, want_states=False):
    """ssm_scan_fwd on host tensors (pinned or pageable) when pinned is not
    None, else on device copies (results brought back)."""
    t = dict(d, h0=h0)
    if pinned is None:
        t = {k: (v.cuda() if v is not None else None) for k, v in t.items()}
    elif pinned:
        t = {k: (v.pin_memory() if v is not None else None) for k, v in t.items()}
    y, h, st = _ops().ssm_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], D=t["D"],
                                   z=t["z"], dt_bias=t["dt_bias"], h0=t["h0"], flags=flags,
                                   rms_eps=eps, want_states=want_states)
    if pinned is None:
        torch.cuda.synchronize()
        return y.cpu(), h.cpu(), (st.cpu() if st is not None else None)
    assert y.device.type == "cpu" and h.device.type == "cpu"
    if y.numel():
        assert y.is_pinned() == pinned and h.is_pinned() == pinned
    return y, h, st


@pytest.mark.parametrize("b", [1, 2, 3, 8, 17])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_equals_device_bitwise(cuda_ok, b, pinned):
    # 1 row: one chunk (cut along the sequence like the device call); 2, 3,
    # 8 rows: one row a chunk; 17 rows: six chunks of three rows, the last
    # of two, so both slots are reused
    d = I.m1_inputs(b, 300, 96, 16, io="bf16", seed=40 + b)
    h0 = torch.randn(b, 96, 16, generator=torch.Generator().manual_seed(b)) * 0.5
    y, h, _ = _call(d, h0, pinned=pinned)
    yd, hd, _ = _call(d, h0)
    assert torch.equal(y, yd)
    assert torch.equal(h, hd)


@pytest.mark.parametrize("io,flags,gate,states", [
    ("f32", I.SOFTPLUS, False, True),
    ("bf16", I.SOFTPLUS | I.RMS_BC | I.RMS_DT, True, False),
    ("bf16", 0, True, True),
])
def test_host_options_and_oracle(cuda_ok, io, flags, gate, states):
    d = I.m1_inputs(5, 200, 64, 16, io=io, gate=gate, seed=7)
    if flags == 0:  # a positive step without softplus, and no bias
        d["dt"] = (d["dt"].float().abs() * 0.1).to(d["dt"].dtype)
        d["dt_bias"] = None
    y, h, st = _call(d, None, pinned=True, flags=flags, want_states=states)
    yd, hd, std = _call(d, None, flags=flags, want_states=states)
    assert torch.equal(y, yd) and torch.equal(h, hd)
    if states:
        assert torch.equal(st, std)
    ref = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                         dt_bias=d["dt_bias"], flags=flags, rms_eps=1e-6)
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    assert_close_normwise(y, ref[0], rel, "y")
    assert_close_normwise(h, ref[1], rel, "h_last")


@pytest.mark.parametrize("b,L,C,N,G", [(4, 100, 64, 16, 2), (3, 50, 36, 16, 1)])
def test_host_groups_and_generic_kernel(cuda_ok, b, L, C, N, G):
    # two groups (B, C rows [b, L, G, N] cut by batch row); 36 bf16 channels
    # are not whole 16-byte rows, so the chunks run the generic kernel
    d = I.m1_inputs(b, L, C, N, groups=G, io="bf16", seed=C + G)
    y, h, _ = _call(d, None, pinned=True)
    yd, hd, _ = _call(d, None)
    assert torch.equal(y, yd) and torch.equal(h, hd)


def test_host_h_last_into_h0(cuda_ok):
    # h_last may be h0's (host) buffer: every chunk's h0 rows are uploaded
    # before its h_last rows come back
    d = I.m1_inputs(5, 120, 64, 16, io="bf16", seed=31)
    h0 = torch.randn(5, 64, 16, generator=torch.Generator().manual_seed(31))
    _, h_ref, _ = _call(d, h0, pinned=True)
    t = {k: (v.pin_memory() if v is not None else None) for k, v in dict(d, h0=h0.clone()).items()}
    y, h, _ = _ops().ssm_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                                  dt_bias=t["dt_bias"], h0=t["h0"], h_last=t["h0"])
    assert torch.equal(h, h_ref) and torch.equal(t["h0"], h_ref)


def test_host_empty_sequence_passes_the_state(cuda_ok):
    d = I.m1_inputs(3, 0, 64, 16, io="bf16", seed=9)
    h0 = torch.randn(3, 64, 16)
    _, h, _ = _call(d, h0, pinned=True)
    assert torch.equal(h, h0)
    _, h, _ = _call(d, None, pinned=True)
    assert torch.count_nonzero(h) == 0


def test_host_calls_back_to_back(cuda_ok):
    # successive calls reuse the library's copy streams and events; each
    # call's results are its own
    outs = []
    for seed in range(3):
        d = I.m1_inputs(4, 128, 64, 16, io="bf16", seed=100 + seed)
        outs.append((d, _call(d, None, pinned=True)))
    for d, (y, h, _) in outs:
        yd, hd, _ = _call(d, None)
        assert torch.equal(y, yd) and torch.equal(h, hd)
