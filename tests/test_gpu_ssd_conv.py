"""GPU parity of the fused Mamba-2 prologue + SSD (ssd_conv_chunk_scan_fwd,
through the C ABI): the causal convolution of xBC, then silu, split into x,
B and C, then the SSD ("Mamba-2", the module tree and "The mixer's values").

Checked three ways: against the float64 oracle (oracle.conv1d, then
oracle.m2_scan) at the bf16 tolerance; bit for bit against the unfused pair
ssm_conv1d_fwd then ssd_chunk_scan_fwd (the same convolution order and the
same SSD kernel, so the same bits); and the conv state out against the last
three inputs, exactly."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_28_b200 import inputs as I
from tests.parity import REL, assert_close_normwise

pytestmark = pytest.mark.gpu

P, N = 64, 128


def _ops():
    from selective_state_space_28_b200 import ops
    return ops


def _inputs(b, L, H, G=1, seed=0, state_in=True, h0=True, gate=True, bias=True):
    d = I.ssd_conv_inputs(b, L, H, P, N, groups=G, io="bf16", gate=gate, seed=seed, h0=h0,
                          state_in=state_in, bias=bias)
    return dict(xbc=d["xBC"], w=d["conv_w"], cb=d["conv_bias"], cs=d["conv_state"],
                dt=d["dt"], z=d["z"], A=d["A"], D=d["D"], dt_bias=d["dt_bias"], h0=d["h0"],
                H=H, G=G)


def _cuda(t):
    return t.cuda() if t is not None else None


def _fused(d, **kw):
    out = _ops().ssd_conv_chunk_scan_fwd(
        _cuda(d["xbc"]), _cuda(d["w"]), _cuda(d["dt"]), _cuda(d["A"]), heads=d["H"], state=N,
        groups=d["G"], conv_bias=_cuda(d["cb"]), conv_state_in=_cuda(d["cs"]),
        want_conv_state=True, D=_cuda(d["D"]), z=_cuda(d["z"]), dt_bias=_cuda(d["dt_bias"]),
        h0=_cuda(d["h0"]), check=True, **kw)
    torch.cuda.synchronize()
    return out


def _split(u, H, G):
    b, L, _ = u.shape
    x = u[..., :H * P].reshape(b, L, H, P)
    B = u[..., H * P:H * P + G * N].reshape(b, L, G, N)
    C = u[..., H * P + G * N:].reshape(b, L, G, N)
    return x, B, C


def _unfused(d):
    ops = _ops()
    u, so = ops.ssm_conv1d_fwd(_cuda(d["xbc"]), _cuda(d["w"]), bias=_cuda(d["cb"]),
                               state=_cuda(d["cs"]))
    x, B, C = (t.contiguous() for t in _split(u, d["H"], d["G"]))
    y, h, _ = ops.ssd_chunk_scan_fwd(x, _cuda(d["dt"]), _cuda(d["A"]), B, C, D=_cuda(d["D"]),
                                     z=_cuda(d["z"]), dt_bias=_cuda(d["dt_bias"]),
                                     h0=_cuda(d["h0"]), check=True)
    torch.cuda.synchronize()
    return y, h, so


def _oracle(d, heads=None):
    """float64: the convolution, then the scan (optionally on some heads)."""
    u, so = oracle.conv1d(d["xbc"], d["w"], d["cb"], d["cs"], act=True)
    x, B, C = _split(torch.from_numpy(u), d["H"], d["G"])
    hs = list(range(d["H"])) if heads is None else heads
    gsel = [h // (d["H"] // d["G"]) for h in hs]
    if heads is not None:  # one group per selected head, in order
        B, C = B[:, :, gsel], C[:, :, gsel]
    h0 = d["h0"][:, hs] if d["h0"] is not None else None
    z = d["z"][:, :, hs] if d["z"] is not None else None
    y, h, _ = oracle.m2_scan(x[:, :, hs], d["dt"][:, :, hs], B, C, d["A"][hs], d["D"][hs],
                             z=z, dt_bias=d["dt_bias"][hs], h0=h0)
    return y, h, so


@pytest.mark.parametrize("b,L,H,G,state_in,h0,gate,bias", [
    (2, 600, 3, 1, True, True, True, True),      # ragged last tile, conv state in, h0
    (1, 256, 4, 2, False, False, False, False),  # two groups, sequence start, no gate/bias
    (2, 2, 2, 1, True, True, True, True),        # shorter than the conv window
    (1, 129, 2, 1, True, False, True, True),     # one token into a second tile
])
def test_fused_matches_oracle_and_unfused(cuda_ok, b, L, H, G, state_in, h0, gate, bias):
    d = _inputs(b, L, H, G, seed=L + H, state_in=state_in, h0=h0, gate=gate, bias=bias)
    y, h, so = _fused(d)
    ry, rh, rso = _oracle(d)
    assert_close_normwise(y, ry, REL[torch.bfloat16], "y")
    assert_close_normwise(h, rh, REL[torch.bfloat16], "h_last")
    np.testing.assert_array_equal(so.cpu().numpy(), rso.astype(np.float32))
    uy, uh, uso = _unfused(d)
    assert torch.equal(y, uy) and torch.equal(h, uh) and torch.equal(so, uso)


@pytest.mark.parametrize("b,H,L", [
    (1, 4, 4096),    # every unit cut into 8 segments: halos of later segments from xBC
    (1, 150, 1536),  # 148 whole units and a 2-unit tail in 3 segments
])
def test_fused_sequence_segments(cuda_ok, b, H, L):
    d = _inputs(b, L, H, seed=H + L)
    y, h, so = _fused(d)
    uy, uh, uso = _unfused(d)
    assert torch.equal(y, uy) and torch.equal(h, uh) and torch.equal(so, uso)
    heads = [0, H - 1]
    ry, rh, _ = _oracle(d, heads)
    hsel = torch.tensor(heads).cuda()
    assert_close_normwise(y[:, :, hsel], ry, REL[torch.bfloat16], "y")
    assert_close_normwise(h[:, hsel], rh, REL[torch.bfloat16], "h_last")


def test_fused_split_and_carry(cuda_ok):
    """A prompt cut in two, the conv state and the SSD state handed on, gives
    the whole prompt's outputs (within tolerance: the tiles fall elsewhere)."""
    d = _inputs(1, 700, 3, seed=21, state_in=False, h0=False)
    y, h, so = _fused(d)
    first = dict(d, xbc=d["xbc"][:, :300], dt=d["dt"][:, :300], z=d["z"][:, :300])
    y1, h1, so1 = _fused(first)
    second = dict(d, xbc=d["xbc"][:, 300:], dt=d["dt"][:, 300:], z=d["z"][:, 300:],
                  cs=so1.cpu(), h0=h1.cpu())
    y2, h2, so2 = _fused(second)
    assert torch.equal(so2, so)
    assert_close_normwise(torch.cat([y1, y2], 1), y.double().cpu().numpy(), REL[torch.bfloat16],
                          "y")
    assert_close_normwise(h2, h.double().cpu().numpy(), REL[torch.bfloat16], "h_last")


def test_fused_2p7b_full_size_sampled(cuda_ok):
    """The Mamba-2 2.7B mixer at full size (b4 L4096, 80 heads, xBC of 5376
    channels, a carried conv state), in the benchmark's launch configuration:
    bit for bit against the unfused pair, and against the oracle on two heads
    of one row."""
    w = I.WORKLOADS["ssd_conv_2p7b_b4_l4096_h80_p64_n128_bf16"]
    d = _inputs(w.batch, w.seqlen, w.heads, seed=w.seed, state_in=True, h0=False, gate=False)
    y, h, so = _fused(d)
    uy, uh, uso = _unfused(d)
    assert torch.equal(y, uy) and torch.equal(h, uh) and torch.equal(so, uso)
    for _ in range(2):  # the same bits on every run (the roles' hand-offs leave no race)
        y2, h2, _ = _fused(d)
        assert torch.equal(y2, y) and torch.equal(h2, h)
    row = dict(d, xbc=d["xbc"][3:], dt=d["dt"][3:], cs=d["cs"][3:], z=None)
    heads = [5, 79]  # (3, 79) is in the cut last wave
    ry, rh, _ = _oracle(row, heads)
    hsel = torch.tensor(heads).cuda()
    assert_close_normwise(y[3:][:, :, hsel], ry, REL[torch.bfloat16], "y")
    assert_close_normwise(h[3:][:, hsel], rh, REL[torch.bfloat16], "h_last")
