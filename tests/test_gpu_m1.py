"""GPU parity of the Mamba-1 scan (ssm_scan_fwd, through the C ABI) against
the float64 oracle, plus the bitwise invariants the pages state."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise, to_np

pytestmark = pytest.mark.gpu


def _ops():
    from selective_state_space_28_b200 import ops
    return ops


def _run(d, flags=I.SOFTPLUS, eps=1e-6, want_states=False, h0=None):
    dev = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    h0 = dev["h0"] if h0 is None else h0
    y, h_last, states = _ops().ssm_scan_fwd(
        dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
        dt_bias=dev["dt_bias"], h0=h0, flags=flags, rms_eps=eps, want_states=want_states)
    torch.cuda.synchronize()
    return y, h_last, states


def _oracle(d, flags=I.SOFTPLUS, eps=1e-6, want_states=False):
    return oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                          dt_bias=d["dt_bias"], h0=d["h0"], flags=flags, rms_eps=eps,
                          want_states=want_states)


def _check(d, got, ref, rel, states=False):
    assert_close_normwise(got[0], ref[0], rel, "y")
    assert_close_normwise(got[1], ref[1], rel, "h_last")
    if states:
        assert_close_normwise(got[2], ref[2], rel, "states")


def test_toy_fp32_with_states(cuda_ok):
    w = I.WORKLOADS["m1_toy_b1_l64_c32_n4_f32"]
    d = I.workload_inputs(w)
    got = _run(d, want_states=True)
    ref = _oracle(d, want_states=True)
    _check(d, got, ref, REL[torch.float32], states=True)
    # states[:, -1] == state_output, bit for bit ("Mamba-2", "The state")
    assert torch.equal(got[2][:, -1], got[1])


@pytest.mark.parametrize("N", [4, 8, 16, 32, 64])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_ragged_shapes(cuda_ok, N, io):
    # L spans several 32-token stages and a ragged tail; C a ragged channel tile
    d = I.m1_inputs(2, 77, 40, N, io=io, gate=True, seed=100 + N, h0=True)
    got = _run(d, want_states=True)
    ref = _oracle(d, want_states=True)
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    _check(d, got, ref, rel, states=True)
    assert torch.equal(got[2][:, -1], got[1])


@pytest.mark.parametrize("gate", [True, False])
def test_no_gate_no_bias_no_D(cuda_ok, gate):
    d = I.m1_inputs(3, 45, 64, 16, io="bf16", gate=gate, seed=7)
    d["D"] = None
    d["dt_bias"] = None
    _check(d, _run(d), _oracle(d), REL[torch.bfloat16])


def test_groups(cuda_ok):
    d = I.m1_inputs(2, 40, 128, 16, groups=4, io="f32", seed=8, h0=True)
    _check(d, _run(d), _oracle(d), REL[torch.float32])


def test_softplus_off(cuda_ok):
    d = I.m1_inputs(2, 33, 32, 8, io="f32", seed=9, h0=True)
    d["dt"] = d["dt"].abs() * 0.1
    d["dt_bias"] = None
    _check(d, _run(d, flags=0), _oracle(d, flags=0), REL[torch.float32])


@pytest.mark.parametrize("flags", [I.SOFTPLUS | I.RMS_BC, I.SOFTPLUS | I.RMS_DT,
                                   I.SOFTPLUS | I.RMS_BC | I.RMS_DT])
def test_rms_norms(cuda_ok, flags):
    d = I.m1_inputs(2, 70, 96, 16, io="bf16", seed=10, h0=True)
    _check(d, _run(d, flags=flags), _oracle(d, flags=flags), REL[torch.bfloat16])


@pytest.mark.parametrize("io,C", [("bf16", 200), ("bf16", 8200), ("bf16", 100), ("f32", 1032),
                                  ("f32", 1030)])
def test_step_norm_widths(cuda_ok, io, C):
    # the step-norm pre-pass: rows of whole 16-byte vectors (bf16 200: a
    # partial round of lanes; 8200: four-vector rounds and a remainder; f32
    # 1032) read by vector, others (bf16 100, f32 1030) value by value
    d = I.m1_inputs(2, 9, C, 16, io=io, seed=C, h0=True)
    flags = I.SOFTPLUS | I.RMS_DT
    _check(d, _run(d, flags=flags), _oracle(d, flags=flags),
           REL[torch.bfloat16 if io == "bf16" else torch.float32])


def test_zero_step_skips_token_bitwise(cuda_ok):
    """dt_raw = -inf -> softplus step exactly 0 -> states[:, 3] == states[:, 2]."""
    d = I.m1_inputs(2, 20, 64, 16, io="f32", seed=11, h0=True)
    d["dt"][:, 3] = -float("inf")
    _, _, s = _run(d, want_states=True)
    assert torch.equal(s[:, 3], s[:, 2])


def test_split_and_carry_bitwise(cuda_ok):
    """state_output fed back as state_input continues the scan exactly."""
    d = I.m1_inputs(2, 96, 64, 16, io="bf16", seed=12, h0=True)
    y, h, _ = _run(d)
    k = 37
    first = {n: (v[:, :k].contiguous() if v is not None and v.dim() == 3 and n != "h0"
                 else v) for n, v in d.items()}
    first["B"], first["C"] = d["B"][:, :k].contiguous(), d["C"][:, :k].contiguous()
    rest = {n: (v[:, k:].contiguous() if v is not None and v.dim() == 3 and n != "h0"
                else v) for n, v in d.items()}
    rest["B"], rest["C"] = d["B"][:, k:].contiguous(), d["C"][:, k:].contiguous()
    y1, h1, _ = _run(first)
    y2, h2, _ = _run(rest, h0=h1)
    assert torch.equal(torch.cat([y1, y2], 1), y)
    assert torch.equal(h2, h)


def test_edge_lengths(cuda_ok):
    ops = _ops()
    d = I.m1_inputs(2, 1, 32, 16, io="bf16", seed=13, h0=True)
    _check(d, _run(d), _oracle(d), REL[torch.bfloat16])
    # seqlen 0: nothing to scan; h_last is h0 (or zeros without h0)
    e = I.m1_inputs(2, 0, 32, 16, io="bf16", seed=14, h0=True)
    dev = {k: (v.cuda() if v is not None else None) for k, v in e.items()}
    y, h, _ = ops.ssm_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"],
                               h0=dev["h0"])
    assert y.numel() == 0 and torch.equal(h, dev["h0"])
    y, h, _ = ops.ssm_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"])
    assert torch.count_nonzero(h) == 0
    # h_last may alias h0 (in-place state hand-off)
    f = I.m1_inputs(1, 50, 32, 16, io="f32", seed=15, h0=True)
    ref = _oracle(f)
    dev = {k: (v.cuda() if v is not None else None) for k, v in f.items()}
    h_io = dev["h0"].clone()
    ops.ssm_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                     z=dev["z"], dt_bias=dev["dt_bias"], h0=h_io, h_last=h_io)
    assert_close_normwise(h_io, ref[1], REL[torch.float32], "h_last aliasing h0")


def test_extreme_rates(cuda_ok):
    """A from -36316 to -4e-4 and large/small steps stay finite and match."""
    d = I.m1_inputs(1, 64, 32, 16, io="f32", seed=16, h0=True)
    d["A"][0] = -36316.0
    d["A"][1] = -4e-4
    d["dt"][0, ::5] = 25.0
    d["dt"][0, 1::5] = -25.0
    got, ref = _run(d), _oracle(d)
    _check(d, got, ref, REL[torch.float32])


def test_130m_full_size_sampled(cuda_ok):
    """Mamba-130m-shaped scan at full size (b8 L2048 C1536 N16, bf16), in the
    launch configuration the benchmark times; the oracle checks a sample of
    channels of two batch rows (channels are independent)."""
    w = I.WORKLOADS["m1_130m_b8_l2048_c1536_n16_bf16"]
    d = I.workload_inputs(w)
    y, h, _ = _run(d)
    rows, cols = [0, 7], list(range(0, 64)) + list(range(1472, 1536))
    sub = {k: v for k, v in d.items()}
    sel = torch.tensor(cols)
    for k in ("x", "dt", "z"):
        sub[k] = d[k][rows][:, :, sel]
    sub["B"], sub["C"] = d["B"][rows], d["C"][rows]
    sub["A"], sub["D"], sub["dt_bias"] = d["A"][sel], d["D"][sel], d["dt_bias"][sel]
    ref = _oracle(sub)
    assert_close_normwise(y[rows][:, :, sel.cuda()], ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(h[rows][:, sel.cuda()], ref[1], REL[torch.bfloat16], "h_last")


@pytest.mark.slow
def test_falcon_width_full_size_one_row(cuda_ok):
    """Falcon-Mamba width with all three norms (b4 L8192 C8192 N16, bf16):
    the oracle recomputes batch row 0 in full (the step norm spans all
    channels of a token)."""
    w = I.WORKLOADS["m1_falcon_rms_b4_l8192_c8192_n16_bf16"]
    d = I.workload_inputs(w)
    y, h, _ = _run(d, flags=w.flags, eps=w.rms_eps)
    sub = {k: (v[:1] if (v is not None and k in ("x", "dt", "z", "B", "C")) else v)
           for k, v in d.items()}
    ref = _oracle(sub, flags=w.flags, eps=w.rms_eps)
    assert_close_normwise(y[:1], ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(h[:1], ref[1], REL[torch.bfloat16], "h_last")


def test_host_buffers_round_trip(cuda_ok):
    """Host (pinned) tensors in, host tensors out: the end-to-end API path."""
    d = I.m1_inputs(2, 40, 64, 16, io="bf16", seed=17)
    pinned = {k: (v.pin_memory() if v is not None else None) for k, v in d.items()}
    y, h, _ = _ops().ssm_scan_fwd(pinned["x"], pinned["dt"], pinned["A"], pinned["B"],
                                  pinned["C"], D=pinned["D"], z=pinned["z"],
                                  dt_bias=pinned["dt_bias"])
    assert y.device.type == "cpu" and h.device.type == "cpu"
    ref = _oracle(d)
    assert_close_normwise(y, ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(h, ref[1], REL[torch.bfloat16], "h_last")


# ------------------------------------------------------ sequence segments
# When batch x channels leaves the SMs short of warps the pipelined kernel
# cuts the sequence into segments: segments from their own start, a carry
# (an associative scan over (decay product, end state) pairs), and a rescan
# from the carried states.  The shapes below are cut on a 148-SM B200 (the
# workspace size says so); the results must match the oracle like the whole
# sequence does.

def _workspace_bytes(d, flags=I.SOFTPLUS):
    import ctypes
    from selective_state_space_28_b200 import _lib as L
    b, Lq, C = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    io = L.SSM_BF16 if d["x"].dtype == torch.bfloat16 else L.SSM_F32
    a = L.ScanArgs(batch=b, seqlen=Lq, channels=C, state=N, groups=G, io=io, flags=flags,
                   rms_eps=1e-6)
    n = ctypes.c_size_t(0)
    L.check(L.lib().ssm_scan_workspace(ctypes.byref(a), ctypes.byref(n)), "ws")
    return n.value


@pytest.mark.parametrize("b,L,C,N,io,h0", [
    (1, 2048, 1536, 16, "bf16", True),    # 8 segments of 256 tokens
    (1, 1000, 1536, 16, "bf16", False),   # ragged last segment, zero start state
    (2, 4096, 256, 8, "f32", True),       # state 8, float32 I/O
    (1, 3000, 512, 32, "bf16", True),     # state 32
])
def test_sequence_segments_match_the_oracle(cuda_ok, b, L, C, N, io, h0):
    d = I.m1_inputs(b, L, C, N, io=io, gate=True, seed=200 + L + N, h0=h0)
    assert _workspace_bytes(d) > 256, "shape not cut into segments"
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    _check(d, _run(d), _oracle(d), rel)


def test_sequence_segments_with_norms_and_extreme_rates(cuda_ok):
    """Cut sequence with all three norms, A at the pages' extremes and steps
    driven to +-25: the decay products the carry multiplies by span 0 to 1."""
    flags = I.SOFTPLUS | I.RMS_BC | I.RMS_DT
    d = I.m1_inputs(1, 2048, 512, 16, io="bf16", gate=True, seed=210, h0=True)
    d["A"][0] = -36316.0
    d["A"][1] = -4e-4
    d["A"][2, :8] = -4e-4
    d["dt"][0, ::97] = 25.0
    d["dt"][0, 5::13] = -25.0
    assert _workspace_bytes(d, flags) > 256 + 256 + 2048 * 4
    _check(d, _run(d, flags=flags), _oracle(d, flags=flags), REL[torch.bfloat16])


def test_sequence_segments_zero_steps_on_segment_edges(cuda_ok):
    """dt_raw = -inf (a zero step) on the first and last tokens of segments
    and in a run across a segment boundary."""
    d = I.m1_inputs(1, 2048, 1536, 16, io="bf16", gate=True, seed=212, h0=True)
    assert _workspace_bytes(d) > 256
    for t in (0, 255, 256, 257, 511, 512, 1023, 2047):
        d["dt"][0, t] = -float("inf")
    d["dt"][0, 700:800, :100] = -float("inf")
    _check(d, _run(d), _oracle(d), REL[torch.bfloat16])


def test_sequence_segments_h_last_may_alias_h0(cuda_ok):
    """The rescan reads the carried states, never h0, so h_last may be h0
    itself even when the call runs as three launches."""
    d = I.m1_inputs(1, 2048, 1536, 16, io="bf16", gate=True, seed=211, h0=True)
    assert _workspace_bytes(d) > 256
    ref = _oracle(d)
    dev = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    h_io = dev["h0"].clone()
    y, h, _ = _ops().ssm_scan_fwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"],
                                  D=dev["D"], z=dev["z"], dt_bias=dev["dt_bias"], h0=h_io,
                                  h_last=h_io)
    torch.cuda.synchronize()
    assert_close_normwise(y, ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(h_io, ref[1], REL[torch.bfloat16], "h_last aliasing h0")


def test_generic_kernel_shapes(cuda_ok):
    """Shapes the pipelined kernel cannot tile (bf16 rows that are not
    16-byte multiples, state 64) run the generic kernel and still match."""
    for b, L, C, N, io in ((2, 50, 36, 16, "bf16"), (1, 70, 64, 64, "f32"),
                           (2, 40, 24, 4, "bf16")):
        d = I.m1_inputs(b, L, C, N, io=io, gate=True, seed=220 + C, h0=True)
        rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
        _check(d, _run(d), _oracle(d), rel)
