"""GPU parity of the decode step (ssm_scan_step, through the C ABI) against
the float64 oracle: the state is updated first, then y is read from it."""
import numpy as np
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


def _step(dv, flags=I.SOFTPLUS, eps=1e-6):
    y = _ops().ssm_scan_step(dv["state"], dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"],
                             D=dv["D"], z=dv["z"], dt_bias=dv["dt_bias"], flags=flags,
                             rms_eps=eps)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("N,P,G", [(128, 64, 1), (16, 64, 1), (64, 32, 2), (128, 128, 1),
                                   (8, 4, 1)])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_m2_step(cuda_ok, N, P, G, io):
    d = I.m2_step_inputs(3, 4, P, N, groups=G, io=io, gate=True, seed=N + P)
    ref_state, ref_y = oracle.m2_step(d["state"], d["x"], d["dt"], d["B"], d["C"], d["A"],
                                      d["D"], z=d["z"], dt_bias=d["dt_bias"])
    dv = _dev(d)
    y = _step(dv)
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    assert_close_normwise(dv["state"], ref_state, rel, "state")
    assert_close_normwise(y, ref_y, rel, "y")


@pytest.mark.parametrize("N", [4, 8, 16, 32, 64])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_m1_step(cuda_ok, N, io):
    d = I.m1_step_inputs(5, 72, N, io=io, gate=True, seed=N)
    ref_state, ref_y = oracle.m1_step(d["state"], d["x"], d["dt"], d["B"], d["C"], d["A"],
                                      d["D"], z=d["z"], dt_bias=d["dt_bias"])
    dv = _dev(d)
    y = _step(dv)
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    assert_close_normwise(dv["state"], ref_state, rel, "state")
    assert_close_normwise(y, ref_y, rel, "y")


def test_m1_step_rms_bc(cuda_ok):
    d = I.m1_step_inputs(4, 64, 16, io="bf16", seed=3)
    f = I.SOFTPLUS | I.RMS_BC
    ref_state, ref_y = oracle.m1_step(d["state"], d["x"], d["dt"], d["B"], d["C"], d["A"],
                                      d["D"], z=d["z"], dt_bias=d["dt_bias"], flags=f)
    dv = _dev(d)
    y = _step(dv, flags=f)
    assert_close_normwise(dv["state"], ref_state, REL[torch.bfloat16], "state")
    assert_close_normwise(y, ref_y, REL[torch.bfloat16], "y")


def test_steps_chain_like_a_scan(cuda_ok):
    """Four decode steps, each handing its state to the next, equal a 4-token
    scan from the same state (the cache hand-off of "Mamba", "The state")."""
    ops = _ops()
    d = I.m1_inputs(2, 4, 64, 16, io="f32", seed=21, h0=True)
    dv = _dev(d)
    y_scan, h_scan, _ = ops.ssm_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"],
                                         D=dv["D"], z=dv["z"], dt_bias=dv["dt_bias"],
                                         h0=dv["h0"])
    st = dv["h0"].clone()
    ys = []
    for t in range(4):
        ys.append(ops.ssm_scan_step(st, dv["x"][:, t].contiguous(), dv["dt"][:, t].contiguous(),
                                    dv["A"], dv["B"][:, t].contiguous(),
                                    dv["C"][:, t].contiguous(), D=dv["D"],
                                    z=dv["z"][:, t].contiguous(), dt_bias=dv["dt_bias"]))
    torch.cuda.synchronize()
    torch.testing.assert_close(torch.stack(ys, 1), y_scan, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(st, h_scan, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("io,N,P", [("f32", 128, 64), ("bf16", 128, 64), ("f32", 64, 32)])
def test_m2_step_is_one_token_ssd(cuda_ok, io, N, P):
    """The Mamba-2 step equals the SSD scan of one token from the same state.
    Bit for bit where both calls run the same float32 token-recurrence kernel
    (N=64, P=32); within tolerance where the step has its own kernel (N=128,
    P=64) or the SSD runs on the tensor cores (bf16)."""
    ops = _ops()
    d = I.ssd_inputs(2, 1, 4, P, N, io=io, seed=22, h0=True)
    dv = _dev(d)
    y_scan, h_scan, _ = ops.ssd_chunk_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"],
                                               D=dv["D"], dt_bias=dv["dt_bias"], h0=dv["h0"])
    st = dv["h0"].clone()
    y = ops.ssm_scan_step(st, dv["x"][:, 0].contiguous(), dv["dt"][:, 0].contiguous(),
                          dv["A"], dv["B"][:, 0].contiguous(), dv["C"][:, 0].contiguous(),
                          D=dv["D"], dt_bias=dv["dt_bias"])
    torch.cuda.synchronize()
    if (N, P) == (64, 32):
        assert torch.equal(st, h_scan)
        assert torch.equal(y, y_scan[:, 0])
    else:
        rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
        assert_close_normwise(st, h_scan.cpu().double().numpy(), rel, "state")
        assert_close_normwise(y, y_scan[:, 0].cpu().double().numpy(), rel, "y")


def test_zero_step_leaves_state_bitwise(cuda_ok):
    d = I.m2_step_inputs(2, 3, 64, 128, io="bf16", seed=23)
    d["dt"][:] = -float("inf")
    dv = _dev(d)
    before = dv["state"].clone()
    _step(dv)
    assert torch.equal(dv["state"], before)


def test_2p7b_layer_full_size_sampled(cuda_ok):
    """One layer of the Mamba-2 2.7B decode stack at full size (b256 x 80 heads
    x N128 x P64), checked on sampled (batch, head) units; and one Mamba-130m
    layer (b256 x 1536 x 16) in full."""
    d = I.m2_step_inputs(256, 80, 64, 128, io="bf16", seed=4)
    dv = _dev(d)
    y = _step(dv)
    bs, hs = [0, 77, 255], [0, 41, 79]
    sub = dict(d)
    for k in ("state", "x", "z", "dt"):
        if d[k] is not None:
            sub[k] = d[k][bs][:, hs]
    sub["B"], sub["C"] = d["B"][bs], d["C"][bs]
    for k in ("A", "D", "dt_bias"):
        sub[k] = d[k][hs]
    ref_state, ref_y = oracle.m2_step(sub["state"], sub["x"], sub["dt"], sub["B"], sub["C"],
                                      sub["A"], sub["D"], z=sub["z"], dt_bias=sub["dt_bias"])
    got_state = dv["state"][bs][:, hs]
    assert_close_normwise(got_state, ref_state, REL[torch.bfloat16], "state")
    assert_close_normwise(y[bs][:, hs], ref_y, REL[torch.bfloat16], "y")
    e = I.m1_step_inputs(256, 1536, 16, io="bf16", seed=5)
    ref_state, ref_y = oracle.m1_step(e["state"], e["x"], e["dt"], e["B"], e["C"], e["A"],
                                      e["D"], z=e["z"], dt_bias=e["dt_bias"])
    ev = _dev(e)
    y1 = _step(ev)
    assert_close_normwise(ev["state"], ref_state, REL[torch.bfloat16], "m1 state")
    assert_close_normwise(y1, ref_y, REL[torch.bfloat16], "m1 y")


def test_host_state_round_trip(cuda_ok):
    d = I.m2_step_inputs(2, 3, 64, 16, io="bf16", seed=24)
    ref_state, ref_y = oracle.m2_step(d["state"], d["x"], d["dt"], d["B"], d["C"], d["A"],
                                      d["D"], dt_bias=d["dt_bias"])
    st = d["state"].clone()
    y = _ops().ssm_scan_step(st, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                             dt_bias=d["dt_bias"])
    assert y.device.type == "cpu"
    assert_close_normwise(st, ref_state, REL[torch.bfloat16], "state")
    assert_close_normwise(y, ref_y, REL[torch.bfloat16], "y")
