"""GPU parity of the SSD map's hidden attention (ssd_attention_fwd, through
the C ABI) against the float64 oracle."""
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


def _run(d, flags=1):
    dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    al = _ops().ssd_attention_fwd(dv["dt"], dv["A"], dv["B"], dv["C"], dv["dt_bias"], flags=flags)
    torch.cuda.synchronize()
    return al.cpu()


@pytest.mark.parametrize("L", [1, 37, 128, 200, 300])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_attention_shapes(cuda_ok, L, io):
    # several tiles, ragged tails, the diagonal-block and factorised parts;
    # the output is float32 from float32 arithmetic for either input type
    d = I.ssd_inputs(2, L, 4, 16, 64, io=io, seed=L)
    al = _run(d)
    ref = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"])
    assert_close_normwise(al, ref, REL[torch.float32], "alpha")
    # causal: exactly zero above the diagonal
    assert torch.count_nonzero(torch.triu(al, 1)) == 0


@pytest.mark.parametrize("N,G,H", [(16, 1, 3), (128, 2, 8), (100, 4, 12)])
def test_attention_groups_and_states(cuda_ok, N, G, H):
    d = I.ssd_inputs(1, 150, H, 16, N, groups=G, io="bf16", seed=N + G)
    al = _run(d)
    ref = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"])
    assert_close_normwise(al, ref, REL[torch.float32], "alpha")


@pytest.mark.parametrize("L,G", [(1, 1), (129, 1), (300, 2)])
def test_attention_tensor_core_tiles(cuda_ok, L, G):
    # bf16 inputs with state 128 take the tensor-core C . B^T: one tile, a
    # ragged second tile (rows past the end arrive as zeros), two groups
    d = I.ssd_inputs(1, L, 4, 16, 128, groups=G, io="bf16", seed=L + G)
    al = _run(d)
    ref = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"])
    assert_close_normwise(al, ref, REL[torch.float32], "alpha")
    assert torch.count_nonzero(torch.triu(al, 1)) == 0


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_attention_long_batched(cuda_ok, io):
    # more than one 1024-token round of the running sums (the second one
    # ragged), two batch rows and two groups: bf16 with state 128 runs the
    # C . B^T tiles and the running sums in one launch, f32 the two passes
    d = I.ssd_inputs(2, 1100, 4, 16, 128, groups=2, io=io, seed=77)
    al = _run(d)
    ref = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"])
    assert_close_normwise(al, ref, REL[torch.float32], "alpha")
    assert torch.count_nonzero(torch.triu(al, 1)) == 0


def test_attention_without_softplus(cuda_ok):
    d = I.ssd_inputs(1, 90, 2, 16, 32, io="f32", seed=3)
    d["dt"] = d["dt"].abs() * 0.1   # a positive step without softplus, and no bias
    d["dt_bias"] = None             # (the inverse-softplus bias would make it negative)
    al = _run(d, flags=0)
    ref = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"], flags=0)
    assert_close_normwise(al, ref, REL[torch.float32], "alpha")


def test_attention_rebuilds_the_ssd_output(cuda_ok):
    # the page's check: alpha x + D x is the scan's y (zero initial state)
    d = I.ssd_inputs(1, 256, 4, 64, 128, io="bf16", seed=5)
    dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    ops = _ops()
    al = ops.ssd_attention_fwd(dv["dt"], dv["A"], dv["B"], dv["C"], dv["dt_bias"])
    y, _, _ = ops.ssd_chunk_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], D=dv["D"],
                                     dt_bias=dv["dt_bias"])
    x = dv["x"].float()
    y_att = torch.einsum("bhts,bshp->bthp", al, x) + dv["D"][None, None, :, None] * x
    assert_close_normwise(y_att.cpu(), y.float().cpu().numpy(), REL[torch.bfloat16], "y")


def test_attention_full_size_sampled(cuda_ok):
    """The 2.7B hidden attention at full size (b1 L1024 H80 N128), in the
    launch bench.py times; heads are independent, so the oracle on two heads
    checks those matrices entirely."""
    w = I.WORKLOADS["attn_2p7b_b1_l1024_h80_n128_bf16"]
    d = I.workload_inputs(w, device="cuda")
    al = _ops().ssd_attention_fwd(d["dt"], d["A"], d["B"], d["C"], d["dt_bias"])
    torch.cuda.synchronize()
    for h in (0, 79):
        ref = oracle.m2_attention(d["dt"][:, :, h:h + 1].cpu(), d["B"].cpu(), d["C"].cpu(),
                                  d["A"][h:h + 1].cpu(), d["dt_bias"][h:h + 1].cpu())
        assert_close_normwise(al[:, h:h + 1].cpu(), ref, REL[torch.float32], "alpha[h=%d]" % h)
