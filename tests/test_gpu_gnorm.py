"""GPU parity of the Mamba-2 mixer's gated norm (ssm_gated_rmsnorm_fwd,
through the C ABI) against the float64 oracle."""
import pytest
import torch

import oracle
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise

pytestmark = pytest.mark.gpu


def _ops():
    from selective_state_space_28_b200 import ops
    return ops


@pytest.mark.parametrize("width", [64, 1536, 3072, 4000, 5120, 8192, 8200, 12, 1000, 1002])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_gnorm_shapes(cuda_ok, width, io):
    # Rows of whole 16-byte vectors (8 bf16 / 4 float32 values) up to 2048
    # values a vector slot (bf16) or 1024 (f32) per thread, four slots at
    # most, keep the row in registers: bf16 64..1536 one slot, 3072 and 4000
    # two, 5120 three (the last one partial), 8192 four; f32 1536 two, 3072
    # three, 4000 four.  Wider vector rows (bf16 8200, f32 5120..8200) keep
    # it in shared memory; 1002 and bf16 12 are not whole vectors and take
    # the per-element form.
    d = I.gnorm_inputs(2, 17, width, io=io, seed=width)
    out = _ops().ssm_gated_rmsnorm_fwd(d["y"].cuda(), d["z"].cuda(), d["weight"].cuda(), 1e-5)
    ref = oracle.gated_rmsnorm(d["y"], d["z"], d["weight"], 1e-5)
    assert_close_normwise(out.float().cpu(), torch.tensor(ref),
                          REL[torch.float32 if io == "f32" else torch.bfloat16], "out")


@pytest.mark.parametrize("gate,weight", [(False, False), (True, False), (False, True)])
def test_gnorm_options(cuda_ok, gate, weight):
    d = I.gnorm_inputs(3, 5, 256, io="f32", seed=3, gate=gate, weight=weight)
    dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    out = _ops().ssm_gated_rmsnorm_fwd(dv["y"], dv["z"], dv["weight"], 1e-3)
    ref = oracle.gated_rmsnorm(d["y"], d["z"], d["weight"], 1e-3)
    assert_close_normwise(out.cpu(), torch.tensor(ref), REL[torch.float32], "out")


def test_gnorm_in_place_and_rows_independent(cuda_ok):
    d = I.gnorm_inputs(4, 33, 640, io="bf16", seed=5)
    y, z, wt = d["y"].cuda(), d["z"].cuda(), d["weight"].cuda()
    ops = _ops()
    ref = ops.ssm_gated_rmsnorm_fwd(y, z, wt)
    yy = y.clone()
    ops.ssm_gated_rmsnorm_fwd(yy, z, wt, out=yy)
    assert torch.equal(yy, ref)
    # a row's result depends on that row only
    part = ops.ssm_gated_rmsnorm_fwd(y[1:3, 4:9].contiguous(), z[1:3, 4:9].contiguous(), wt)
    assert torch.equal(part, ref[1:3, 4:9])


def test_gnorm_zero_rows_and_zero_input(cuda_ok):
    ops = _ops()
    y = torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda")
    assert ops.ssm_gated_rmsnorm_fwd(y).shape == (0, 128)
    # an all-zero row stays zero (eps keeps the scale finite)
    y = torch.zeros((2, 128), dtype=torch.float32, device="cuda")
    out = ops.ssm_gated_rmsnorm_fwd(y, torch.randn_like(y), eps=1e-5)
    assert torch.count_nonzero(out) == 0


def test_gnorm_full_size_sampled(cuda_ok):
    """The Mamba-2 2.7B gated norm at full size (b4 L4096, width 5120), in the
    launch bench.py times; rows are independent, so the oracle on a sample of
    rows checks them exactly."""
    w = I.WORKLOADS["gnorm_2p7b_b4_l4096_w5120_bf16"]
    d = I.workload_inputs(w, device="cuda")
    out = _ops().ssm_gated_rmsnorm_fwd(d["y"], d["z"], d["weight"], w.rms_eps)
    torch.cuda.synchronize()
    rows = [(0, 0), (0, 4095), (1, 1234), (2, 2047), (3, 4095)]
    for b, t in rows:
        ref = oracle.gated_rmsnorm(d["y"][b, t].cpu(), d["z"][b, t].cpu(), d["weight"].cpu(),
                                   w.rms_eps)
        assert_close_normwise(out[b, t].float().cpu(), torch.tensor(ref), REL[torch.bfloat16],
                              "out[%d,%d]" % (b, t))
