"""GPU parity of the Mamba-1 scan with the state written at one token
(ssm_scan_fwd_write, through the C ABI) against the float64 oracle."""
import pytest
import torch

import oracle
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise

pytestmark = pytest.mark.gpu


def _ops():
    from selective_state_space_28_b200 import ops
    return ops


def _dev(d):
    return {k: (v.cuda() if v is not None else None) for k, v in d.items()}


def _args(d):
    return (d["x"], d["dt"], d["A"], d["B"], d["C"])


def _kw(d):
    return dict(D=d["D"], z=d["z"], dt_bias=d["dt_bias"], h0=d["h0"])


@pytest.mark.parametrize("t", [0, 31, 32, 70, 99])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_state_write_matches_oracle(cuda_ok, t, io):
    d = I.m1_inputs(2, 100, 64, 16, io=io, seed=t, h0=True)
    s = torch.randn((2, 64, 16), generator=torch.Generator().manual_seed(t)) * 0.5
    y, h, _ = _ops().ssm_scan_fwd_write(*_args(_dev(d)), **_kw(_dev(d)), t=t, state=s.cuda())
    yr, hr, _ = oracle.m1_scan_write(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                                     dt_bias=d["dt_bias"], h0=d["h0"], t=t, state=s)
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    assert_close_normwise(y.float().cpu(), yr, rel, "y")
    assert_close_normwise(h.cpu(), hr, rel, "h_last")


def test_state_write_with_norms_and_states(cuda_ok):
    d = I.m1_inputs(2, 50, 32, 16, io="f32", seed=3, h0=True)
    s = torch.zeros((2, 32, 16))
    flags = I.SOFTPLUS | I.RMS_BC | I.RMS_DT
    y, h, st = _ops().ssm_scan_fwd_write(*_args(_dev(d)), **_kw(_dev(d)), t=20, state=s.cuda(),
                                         flags=flags, want_states=True)
    yr, hr, sr = oracle.m1_scan_write(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"],
                                      z=d["z"], dt_bias=d["dt_bias"], h0=d["h0"], t=20,
                                      state=s, flags=flags, want_states=True)
    assert_close_normwise(y.cpu(), yr, REL[torch.float32], "y")
    assert_close_normwise(st.cpu(), sr, REL[torch.float32], "states")
    assert torch.count_nonzero(st[:, 20]) == 0


def test_state_write_of_the_scans_own_state_is_the_scan(cuda_ok):
    # writing back the state the scan itself had at t reproduces the plain
    # scan bit for bit: the state at t comes from a scan of tokens 0..t on the
    # same kernel, and the write form does the same arithmetic per token
    d = _dev(I.m1_inputs(2, 150, 64, 16, io="bf16", seed=4, h0=True))
    ops = _ops()
    y, h, _ = ops.ssm_scan_fwd(*_args(d), **_kw(d))
    t = 70
    head = {k: (v[:, :t + 1].contiguous() if k in ("x", "dt", "z", "B", "C") else v)
            for k, v in d.items()}
    _, h_t, _ = ops.ssm_scan_fwd(*_args(head), **_kw(head))
    y2, h2, _ = ops.ssm_scan_fwd_write(*_args(d), **_kw(d), t=t, state=h_t)
    assert torch.equal(y2, y) and torch.equal(h2, h)


@pytest.mark.parametrize("t", [0, 37, 149])
def test_state_write_with_h_last_aliasing_h0_or_the_state(cuda_ok, t):
    # h_last may be h0's buffer (the ABI allows it) or the written state's:
    # the write then runs the tokens after t as a launch of its own, after
    # the parts that read h0 and the written state; the results equal the
    # call with separate buffers, bit for bit
    d = _dev(I.m1_inputs(3, 150, 96, 16, io="bf16", seed=20 + t, h0=True))
    ops = _ops()
    state = torch.randn(3, 96, 16, device="cuda", generator=torch.Generator("cuda").manual_seed(t))
    y, h, _ = ops.ssm_scan_fwd_write(*_args(d), **_kw(d), t=t, state=state)
    h0 = d["h0"].clone()
    y1, h1, _ = ops.ssm_scan_fwd_write(*_args(d), **dict(_kw(d), h0=h0), t=t, state=state,
                                       h_last=h0)
    assert torch.equal(y1, y) and torch.equal(h1, h) and torch.equal(h0, h)
    st = state.clone()
    y2, h2, _ = ops.ssm_scan_fwd_write(*_args(d), **_kw(d), t=t, state=st, h_last=st)
    assert torch.equal(y2, y) and torch.equal(h2, h) and torch.equal(st, h)


def test_state_write_per_token_kernel_with_states(cuda_ok):
    # with per-token states the per-token kernel carries the write; its
    # states at t are the written state and later ones continue from it
    d = _dev(I.m1_inputs(1, 80, 32, 16, io="f32", seed=6, h0=True))
    s = torch.randn((1, 32, 16), device="cuda")
    y, h, st = _ops().ssm_scan_fwd_write(*_args(d), **_kw(d), t=33, state=s, want_states=True)
    assert torch.equal(st[:, 33], s)
    assert torch.equal(st[:, -1], h)


def test_state_write_130m_full_size_sampled(cuda_ok):
    """The state write at full Mamba-130m size (b8 L2048 C1536 N16, bf16), at
    token 1024, in the launch configuration the benchmark times; the oracle
    checks a sample of channels of two batch rows (channels are independent)."""
    w = I.WORKLOADS["m1_130m_b8_l2048_c1536_n16_bf16"]
    d = I.workload_inputs(w)
    s = torch.randn((w.batch, w.channels, w.state),
                    generator=torch.Generator().manual_seed(1024)) * 0.5
    dd = _dev(d)
    y, h, _ = _ops().ssm_scan_fwd_write(*_args(dd), D=dd["D"], z=dd["z"],
                                        dt_bias=dd["dt_bias"], t=1024, state=s.cuda())
    rows, cols = [0, 7], list(range(0, 64)) + list(range(1472, 1536))
    sel = torch.tensor(cols)
    sub = {k: d[k][rows][:, :, sel] for k in ("x", "dt", "z")}
    yr, hr, _ = oracle.m1_scan_write(sub["x"], sub["dt"], d["B"][rows], d["C"][rows],
                                     d["A"][sel], d["D"][sel], z=sub["z"],
                                     dt_bias=d["dt_bias"][sel], t=1024,
                                     state=s[rows][:, sel])
    assert_close_normwise(y[rows][:, :, sel.cuda()].float().cpu(), yr, REL[torch.bfloat16], "y")
    assert_close_normwise(h[rows][:, sel.cuda()].cpu(), hr, REL[torch.bfloat16], "h_last")


def test_state_write_rejects_bad_token(cuda_ok):
    d = _dev(I.m1_inputs(1, 10, 32, 16, io="f32", seed=5))
    ops = _ops()
    from selective_state_space_28_b200._lib import SsmError
    for t in (-1, 10):
        with pytest.raises(SsmError):
            ops.ssm_scan_fwd_write(*_args(d), **_kw(d), t=t,
                                   state=torch.zeros((1, 32, 16), device="cuda"))
