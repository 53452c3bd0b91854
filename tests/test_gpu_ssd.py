"""GPU parity of the Mamba-2 SSD scan (ssd_chunk_scan_fwd, through the C ABI)
against the float64 oracle's token loop."""
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
    bf16), in the benchmark's launch configuration; the oracle checks three
    heads of two batch rows (heads are independent given B and C)."""
    w = I.WORKLOADS["ssd_2p7b_b4_l4096_h80_p64_n128_bf16"]
    d = I.workload_inputs(w)
    y, h, _ = _run(d, chunk=w.chunk)
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
    ws = torch.full((256,), 7, dtype=torch.uint8, device="cuda")
    ops.ssd_chunk_scan_fwd(dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], D=dv["D"],
                           dt_bias=dv["dt_bias"], h0=dv["h0"], workspace=ws)
    torch.cuda.synchronize()
    assert ws[:4].view(torch.int32).item() == 0
