"""GPU parity of the Mamba-2 SSD scan (ssd_chunk_scan_fwd, through the C ABI)
against the float64 oracle's token loop."""
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


def _run(d, chunk=256, want_states=False, h0="from_d"):
    dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    out = _ops().ssd_chunk_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], D=dv["D"],
                                    z=dv["z"], dt_bias=dv["dt_bias"],
                                    h0=dv["h0"] if h0 == "from_d" else h0, chunk=chunk,
                                    want_states=want_states)
    torch.cuda.synchronize()
    return out


def _oracle(d, want_states=False):
    return oracle.m2_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                          dt_bias=d["dt_bias"], h0=d["h0"], want_states=want_states)


@pytest.mark.parametrize("L", [1, 63, 256, 600])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_ssd_shapes(cuda_ok, L, io):
    d = I.ssd_inputs(2, L, 3, 64, 128, io=io, gate=True, seed=L, h0=True)
    got, ref = _run(d), _oracle(d)
    rel = REL[torch.float32 if io == "f32" else torch.bfloat16]
    assert_close_normwise(got[0], ref[0], rel, "y")
    assert_close_normwise(got[1], ref[1], rel, "h_last")


@pytest.mark.parametrize("N,P,G,H", [(16, 32, 1, 4), (64, 64, 2, 4), (128, 64, 4, 8)])
def test_ssd_groups_and_sizes(cuda_ok, N, P, G, H):
    d = I.ssd_inputs(2, 300, H, P, N, groups=G, io="bf16", seed=N + G, h0=True)
    got, ref = _run(d), _oracle(d)
    assert_close_normwise(got[0], ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(got[1], ref[1], REL[torch.bfloat16], "h_last")


def test_ssd_states_and_last_state(cuda_ok):
    d = I.ssd_inputs(1, 40, 2, 64, 128, io="f32", seed=5, h0=True)
    got, ref = _run(d, want_states=True), _oracle(d, want_states=True)
    assert_close_normwise(got[2], ref[2], REL[torch.float32], "states")
    assert torch.equal(got[2][:, -1], got[1])


def test_ssd_zero_step_within_tolerance(cuda_ok):
    """A zero step leaves the state unchanged; for the chunked path the pages'
    bit-for-bit claim is from a per-token loop, so it is held to tolerance."""
    d = I.ssd_inputs(1, 300, 2, 64, 128, io="f32", seed=6, h0=True)
    d["dt"][:, 3] = -float("inf")
    got = _run(d, want_states=True)
    s = got[2]
    diff = (s[:, 3] - s[:, 2]).abs().max().item()
    assert diff <= 1e-5 * s[:, 2].abs().max().item()


def test_ssd_chunk_size_does_not_change_result(cuda_ok):
    d = I.ssd_inputs(2, 512, 4, 64, 128, io="bf16", seed=7, h0=True)
    a = _run(d, chunk=256)
    b = _run(d, chunk=128)
    ref = _oracle(d)
    for got in (a, b):
        assert_close_normwise(got[0], ref[0], REL[torch.bfloat16], "y")
        assert_close_normwise(got[1], ref[1], REL[torch.bfloat16], "h_last")


def test_ssd_split_and_carry(cuda_ok):
    d = I.ssd_inputs(1, 520, 2, 64, 128, io="f32", seed=8, h0=True)
    full = _run(d)
    k = 300
    first = {n: (v[:, :k].contiguous() if v is not None and n in ("x", "dt", "z", "B", "C")
                 else v) for n, v in d.items()}
    rest = {n: (v[:, k:].contiguous() if v is not None and n in ("x", "dt", "z", "B", "C")
                else v) for n, v in d.items()}
    a = _run(first)
    b = _run(rest, h0=a[1])
    torch.testing.assert_close(torch.cat([a[0], b[0]], 1), full[0], rtol=1e-4, atol=1e-4)
    torch.testing.assert_close(b[1], full[1], rtol=1e-4, atol=1e-4)


def test_2p7b_full_size_sampled(cuda_ok):
    """Mamba-2 2.7B-shaped SSD at full size (b4 L4096 H80 P64 N128 chunk 256,
    bf16), in the benchmark's launch configuration; the oracle checks four
    heads of two batch rows (heads are independent given B and C)."""
    w = I.WORKLOADS["ssd_2p7b_b4_l4096_h80_p64_n128_bf16"]
    d = I.workload_inputs(w)
    y, h, _ = _run(d, chunk=w.chunk)
    for _ in range(2):  # the same bits on every run (the roles' hand-offs leave no race)
        y2, h2, _ = _run(d, chunk=w.chunk)
        assert torch.equal(y2, y) and torch.equal(h2, h)
    rows, hs = [0, 3], [0, 40, 60, 79]  # (3, 60) and (3, 79) are in the cut last wave
    sub = dict(d)
    sub["x"] = d["x"][rows][:, :, hs]
    sub["dt"] = d["dt"][rows][:, :, hs]
    sub["B"], sub["C"] = d["B"][rows], d["C"][rows]
    for k in ("A", "D", "dt_bias"):
        sub[k] = d[k][hs]
    ref = _oracle(sub)
    hsel = torch.tensor(hs).cuda()
    assert_close_normwise(y[rows][:, :, hsel], ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(h[rows][:, hsel], ref[1], REL[torch.bfloat16], "h_last")


@pytest.mark.parametrize("b,H,L,h0,gate", [
    (1, 4, 4096, True, True),      # every unit cut into 8 segments
    (2, 3, 1700, False, False),    # ragged last tile, zero start state, 3 segments
    (1, 150, 1536, True, False),   # 148 whole units and a 2-unit tail in 3 segments
])
def test_ssd_sequence_segments(cuda_ok, b, H, L, h0, gate):
    """Units of a partial last wave run as sequence segments, the state
    carried from segment to segment (shapes chosen so that 148 SMs cut them)."""
    d = I.ssd_inputs(b, L, H, 64, 128, io="bf16", gate=gate, seed=L + H, h0=h0)
    got, ref = _run(d), _oracle(d)
    assert_close_normwise(got[0], ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(got[1], ref[1], REL[torch.bfloat16], "h_last")


def test_ssd_segments_in_place_state_and_groups(cuda_ok):
    """A cut call with h_last aliasing h0 (the ABI allows it: the first pass
    reads the start states before any segment writes an end state) and two
    B/C groups."""
    d = I.ssd_inputs(1, 2048, 8, 64, 128, groups=2, io="bf16", gate=True, seed=33, h0=True)
    ref = _oracle(d)
    dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    state = dv["h0"].clone()
    y, h, _ = _ops().ssd_chunk_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], D=dv["D"],
                                        z=dv["z"], dt_bias=dv["dt_bias"], h0=state, h_last=state)
    torch.cuda.synchronize()
    assert h.data_ptr() == state.data_ptr()
    assert_close_normwise(y, ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(state, ref[1], REL[torch.bfloat16], "h_last")


def test_ssd_segments_match_whole_units(cuda_ok):
    """The same heads computed in a cut last wave and in whole waves agree
    to rounding (h_last, y)."""
    d = I.ssd_inputs(1, 2048, 150, 64, 128, io="bf16", seed=21, h0=True)
    full = _run(d)                                   # heads 148, 149 cut
    sub = dict(d)
    for k in ("x", "dt"):
        sub[k] = d[k][:, :, 2:].contiguous()
    for k in ("A", "D", "dt_bias"):
        sub[k] = d[k][2:].contiguous()
    sub["h0"] = d["h0"][:, 2:].contiguous()
    part = _run(sub)                                 # 148 heads: whole units
    assert_close_normwise(full[1][:, -2:], part[1][:, -2:].cpu(), REL[torch.bfloat16], "h_last")
    assert_close_normwise(full[0][:, :, -2:], part[0][:, :, -2:].float().cpu(),
                          REL[torch.bfloat16], "y")


def test_ssd_status_word_clear(cuda_ok):
    """The tensor-core path reports bounded-wait timeouts in the first word of
    its workspace; a normal call leaves it zero."""
    ops = _ops()
    d = I.ssd_inputs(2, 300, 3, 64, 128, io="bf16", seed=9, h0=True)
    dv = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    n = ops.ssd_workspace_bytes(batch=2, seqlen=300, heads=3, head_dim=64, state=128, groups=1,
                                chunk=256, io=1, flags=1)
    ws = torch.full((n,), 7, dtype=torch.uint8, device="cuda")
    ops.ssd_chunk_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], D=dv["D"],
                           dt_bias=dv["dt_bias"], h0=dv["h0"], workspace=ws)
    torch.cuda.synchronize()
    assert ws[:4].view(torch.int32).item() == 0


# ------------------------------------------------ the tensor-core path's edges
# The shapes below (bf16 I/O, state 128, head_dim 64, no per-token states) run
# the tcgen05 kernel; each test first checks, through the workspace size, that
# the call takes that path.  Values from the "Mamba-2" page: a zero step skips
# a token exactly ("A zero step skips a token exactly"), and the checkpoints'
# A_h span -exp(A_log) from about -36316 to -4e-4 ("The mixer's values").

def _assert_tensor_core_path(d):
    import ctypes
    from selective_state_space_28_b200 import _lib as L
    b, Lq, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    a = L.SsdArgs(batch=b, seqlen=Lq, heads=H, head_dim=P, state=N, groups=G, chunk=256,
                  io=L.SSM_BF16, flags=L.SSM_DT_SOFTPLUS)
    n = ctypes.c_size_t(0)
    L.check(L.lib().ssd_chunk_scan_workspace(ctypes.byref(a), ctypes.byref(n)), "ws")
    assert n.value > 0, "not the tensor-core path"


def _check(d, what=""):
    _assert_tensor_core_path(d)
    got, ref = _run(d), _oracle(d)
    assert_close_normwise(got[0], ref[0], REL[torch.bfloat16], what + " y")
    assert_close_normwise(got[1], ref[1], REL[torch.bfloat16], what + " h_last")
    return got, ref


@pytest.mark.parametrize("gate", [False, True])
def test_ssd_tc_zero_steps_at_tile_edges(cuda_ok, gate):
    """dt_raw = -inf gives a zero step: the token adds nothing and decays
    nothing.  Zero steps at the first token, on both sides of 128-token tile
    and 256-token chunk boundaries, in runs, and at the last token."""
    d = I.ssd_inputs(2, 600, 4, 64, 128, io="bf16", gate=gate, seed=41, h0=True)
    for t in (0, 1, 127, 128, 129, 255, 256, 300, 301, 302, 383, 384, 599):
        d["dt"][:, t] = -float("inf")
    d["dt"][1, 400:520, 2] = -float("inf")  # a whole tile of one head skipped
    _check(d, "zero steps")


def test_ssd_tc_all_zero_steps_keep_the_state(cuda_ok):
    """Every step zero: y = C_t . h0 + D x_t and h_last = h0 (to rounding of
    the bf16 operands the tensor cores read)."""
    d = I.ssd_inputs(1, 300, 3, 64, 128, io="bf16", seed=42, h0=True)
    d["dt"][:] = -float("inf")
    got, ref = _check(d, "all zero")
    np.testing.assert_array_equal(ref[1], d["h0"].double().numpy())


@pytest.mark.parametrize("L", [300, 1536])
def test_ssd_tc_extreme_rates(cuda_ok, L):
    """Per-head A_h at the pages' extremes (-36316 and -4e-4) beside ordinary
    ones, and steps driven to +-25 on scattered tokens: a state wiped out in
    one token, a state that barely decays over the whole prompt, and tokens
    that add almost nothing."""
    d = I.ssd_inputs(1, L, 6, 64, 128, io="bf16", gate=True, seed=43 + L, h0=True)
    d["A"] = torch.tensor([-36316.0, -4e-4, -1.0, -16.0, -36316.0, -4e-4])
    g = torch.Generator().manual_seed(L)
    pick = torch.rand(d["dt"].shape, generator=g)
    d["dt"][pick < 0.05] = 25.0
    d["dt"][pick > 0.95] = -25.0
    _check(d, "extreme rates")


def test_ssd_tc_split_and_carry_through_h0(cuda_ok):
    """A prompt cut at a token that is not a tile boundary and continued
    from h_last through h0 agrees with the whole prompt and the oracle."""
    d = I.ssd_inputs(2, 700, 4, 64, 128, io="bf16", gate=True, seed=44, h0=True)
    _assert_tensor_core_path(d)
    k = 333
    cut = ("x", "dt", "z", "B", "C")
    first = {n: (v[:, :k].contiguous() if v is not None and n in cut else v)
             for n, v in d.items()}
    rest = {n: (v[:, k:].contiguous() if v is not None and n in cut else v)
            for n, v in d.items()}
    a = _run(first)
    b = _run(rest, h0=a[1])
    ref = _oracle(d)
    assert_close_normwise(torch.cat([a[0], b[0]], 1), ref[0], REL[torch.bfloat16], "y")
    assert_close_normwise(b[1], ref[1], REL[torch.bfloat16], "h_last")


def test_ssd_tc_cut_wave_with_extreme_values(cuda_ok):
    """A shape whose last wave is cut into sequence segments (one batch row,
    four heads, 4096 tokens), with zero steps on segment boundaries and the
    extreme A_h: the carried state and the decay products stay exact enough."""
    d = I.ssd_inputs(1, 4096, 4, 64, 128, io="bf16", gate=False, seed=45, h0=True)
    d["A"] = torch.tensor([-36316.0, -4e-4, -2.0, -4e-4])
    for t in range(0, 4096, 512):
        d["dt"][:, t] = -float("inf")
    d["dt"][0, 1000:1100, 1] = 25.0
    _check(d, "cut wave")
