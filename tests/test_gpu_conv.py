"""GPU parity of the mixers' causal convolution (ssm_conv1d_fwd, through the
C ABI) against the float64 oracle."""
import pytest
import torch

import oracle
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise

pytestmark = pytest.mark.gpu


def _ops():
    from selective_state_space_28_b200 import ops
    return ops


def _run(d, silu=True, with_bias=True, with_state=True):
    dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    u, st = _ops().ssm_conv1d_fwd(dv["x"], dv["w"], dv["bias"] if with_bias else None,
                                  dv["state"] if with_state else None, silu=silu)
    torch.cuda.synchronize()
    return u.cpu(), st.cpu()


def _ref(d, silu=True, with_bias=True, with_state=True):
    return oracle.conv1d(d["x"], d["w"], d["bias"] if with_bias else None,
                         d["state"] if with_state else None, act=silu)


@pytest.mark.parametrize("L", [1, 3, 37, 128, 129, 300])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_shapes(cuda_ok, L, io):
    # several 128-token runs (halo across runs), a ragged tail, a state
    d = I.conv_inputs(3, L, 64, 4, io=io, seed=L, state=True)
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    (u, st), (ur, sr) = _run(d), _ref(d)
    assert_close_normwise(u.float(), torch.tensor(ur), rel, "u")
    # the state is the inputs themselves: exact
    assert torch.equal(st.double(), torch.tensor(sr))


@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("C", [64, 36])
def test_conv_bf16_vector_widths(cuda_ok, W, C):
    # bf16 rows of whole 16-byte vectors take eight channels a thread (64),
    # rows of 8-byte vectors four (36), for every kernel width; runs cross
    # the fitted run length (300 tokens)
    d = I.conv_inputs(2, 300, C, W, io="bf16", seed=7 * W + C, state=True)
    (u, st), (ur, sr) = _run(d, True, True, True), _ref(d, True, True, True)
    assert_close_normwise(u, torch.tensor(ur), REL[torch.bfloat16], "u")
    if W > 1:
        assert torch.equal(st.double(), torch.tensor(sr))


@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("silu,with_bias,with_state", [(True, True, True), (False, False, False),
                                                       (True, False, True), (False, True, False)])
def test_conv_widths_and_options(cuda_ok, W, silu, with_bias, with_state):
    d = I.conv_inputs(2, 45, 24, W, io="f32", seed=10 * W, state=True)
    (u, st), (ur, sr) = _run(d, silu, with_bias, with_state), _ref(d, silu, with_bias, with_state)
    assert_close_normwise(u, torch.tensor(ur), REL[torch.float32], "u")
    if W > 1:
        assert torch.equal(st.double(), torch.tensor(sr))


@pytest.mark.parametrize("C", [1, 13, 100])
def test_conv_ragged_channel_counts(cuda_ok, C):
    # channel counts that are not a multiple of the 16-byte vector take the
    # per-channel form
    d = I.conv_inputs(2, 70, C, 4, io="bf16", seed=C, state=True)
    (u, st), (ur, sr) = _run(d), _ref(d)
    assert_close_normwise(u.float(), torch.tensor(ur), REL[torch.bfloat16], "u")
    assert torch.equal(st.double(), torch.tensor(sr))


def test_conv_split_and_carry_bitwise(cuda_ok):
    d = I.conv_inputs(2, 300, 40, 4, io="bf16", seed=7, state=True)
    ops = _ops()
    x, w, bias, st0 = (d[k].cuda() for k in ("x", "w", "bias", "state"))
    u, st = ops.ssm_conv1d_fwd(x, w, bias, st0)
    for cut in (1, 2, 100, 257):
        u1, s1 = ops.ssm_conv1d_fwd(x[:, :cut].contiguous(), w, bias, st0)
        u2, s2 = ops.ssm_conv1d_fwd(x[:, cut:].contiguous(), w, bias, s1)
        assert torch.equal(torch.cat([u1, u2], dim=1), u)
        assert torch.equal(s2, st)


def test_conv_decode_in_place_equals_prompt(cuda_ok):
    # one token at a time, state updated in place, equals the whole prompt
    d = I.conv_inputs(4, 20, 48, 4, io="bf16", seed=8, state=True)
    ops = _ops()
    x, w, bias, st0 = (d[k].cuda() for k in ("x", "w", "bias", "state"))
    u, st = ops.ssm_conv1d_fwd(x, w, bias, st0)
    state = st0.clone()
    for t in range(20):
        ut, _ = ops.ssm_conv1d_fwd(x[:, t:t + 1].contiguous(), w, bias, state, in_place=True)
        assert torch.equal(ut[:, 0], u[:, t])
    assert torch.equal(state, st)


def test_conv_in_place_long_prompt(cuda_ok):
    # in place over more than one 128-token run: one run per thread
    d = I.conv_inputs(2, 333, 32, 4, io="f32", seed=9, state=True)
    ops = _ops()
    x, w, bias, st0 = (d[k].cuda() for k in ("x", "w", "bias", "state"))
    u_ref, st_ref = ops.ssm_conv1d_fwd(x, w, bias, st0)
    state = st0.clone()
    u, _ = ops.ssm_conv1d_fwd(x, w, bias, state, in_place=True)
    assert torch.equal(u, u_ref)
    assert torch.equal(state, st_ref)


def test_conv_empty_sequence_passes_state(cuda_ok):
    d = I.conv_inputs(2, 0, 16, 4, io="bf16", seed=11, state=True)
    (u, st), (_, sr) = _run(d), _ref(d)
    assert u.shape == (2, 0, 16)
    assert torch.equal(st.double(), torch.tensor(sr))
    d2 = I.conv_inputs(2, 0, 16, 4, io="bf16", seed=11, state=False)
    _, st2 = _run(d2, with_state=False)
    assert torch.count_nonzero(st2) == 0


def test_conv_full_size_sampled(cuda_ok):
    """The Mamba-2 2.7B conv workload at full size, in the launch bench.py
    times; the convolution is per channel, so the oracle on a sample of
    channels (over every batch row and token) checks those outputs exactly."""
    w = I.WORKLOADS["conv_2p7b_b4_l4096_c5376_bf16"]
    d = I.workload_inputs(w, device="cuda")
    u, st = _ops().ssm_conv1d_fwd(d["x"], d["w"], d["bias"], d["state"])
    torch.cuda.synchronize()
    cs = torch.tensor([0, 1, 7, 8, 2047, 2560, 5119, 5120, 5247, 5375])
    sub = {"x": d["x"][:, :, cs].cpu(), "w": d["w"][cs].cpu(), "bias": d["bias"][cs].cpu(),
           "state": d["state"][:, cs].cpu()}
    ur, sr = oracle.conv1d(sub["x"], sub["w"], sub["bias"], sub["state"], act=True)
    assert_close_normwise(u[:, :, cs].float().cpu(), torch.tensor(ur), REL[torch.bfloat16], "u")
    assert torch.equal(st[:, cs].double().cpu(), torch.tensor(sr))
