"""Host-only checks of the C ABI: the library loads, exports every function
include/ssm.h declares, and rejects bad arguments with the documented status
before launching anything.  No call here reaches a kernel, so these run
without a GPU; fake device addresses are never dereferenced."""
import ctypes
import subprocess

import pytest

from selective_state_space_28_b200 import _lib as L
from selective_state_space_28_b200 import build as B

OK, NULL, SHAPE, DTYPE, ALIGN, UNSUP, WS = 0, 1, 2, 3, 4, 5, 6
P = 0x7f0000001000  # a 16-byte-aligned fake device address


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def test_exports_every_declared_symbol(lib):
    names = L.header_functions()
    assert {"ssm_scan_fwd", "ssm_scan_workspace", "ssd_chunk_scan_fwd",
            "ssd_chunk_scan_workspace", "ssm_scan_step", "ssm_status_string",
            "ssm_abi_version", "ssm_conv1d_fwd", "ssm_scan_fwd_static",
            "ssm_gated_rmsnorm_fwd", "ssm_scan_fwd_write", "ssd_attention_fwd",
            "ssd_attention_workspace", "ssm_workspace_status", "ssd_conv_chunk_scan_fwd",
            "ssd_conv_chunk_scan_workspace"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert getattr(lib, n) is not None


def test_no_runtime_symbols_leak(lib):
    """The static CUDA runtime stays private to the library."""
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    assert not [l for l in out.splitlines() if " cuda" in l and " T " in l]


def test_version_and_strings(lib):
    assert lib.ssm_abi_version() == 4
    for s in range(9):
        assert lib.ssm_status_string(s)
    assert lib.ssm_status_string(99) == b"unknown status"


def _scan(**kw):
    d = dict(batch=2, seqlen=8, channels=64, state=16, groups=1, io=1, flags=1,
             rms_eps=1e-6, x=P, dt=P, z=None, B=P, C=P, A=P, D=None, dt_bias=None,
             h0=None, y=P, h_last=None, states=None)
    d.update(kw)
    return L.ScanArgs(**d)


def _call_scan(lib, a):
    return lib.ssm_scan_fwd(ctypes.byref(a), None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), NULL), (dict(dt=None), NULL), (dict(B=None), NULL), (dict(A=None), NULL),
    (dict(y=None), NULL), (dict(io=7), DTYPE), (dict(channels=0), SHAPE),
    (dict(state=0), SHAPE), (dict(batch=-1), SHAPE), (dict(groups=3), SHAPE),
    (dict(groups=0), SHAPE), (dict(x=P + 2), ALIGN), (dict(h_last=P + 8), ALIGN),
    (dict(state=12), UNSUP), (dict(state=128), UNSUP), (dict(flags=8), UNSUP),
    (dict(groups=2, channels=48), UNSUP), (dict(batch=70000), UNSUP),
    (dict(flags=5), WS), (dict(flags=3, rms_eps=-1.0), SHAPE),
])
def test_scan_rejects(lib, kw, status):
    assert _call_scan(lib, _scan(**kw)) == status


def test_scan_null_args(lib):
    assert lib.ssm_scan_fwd(None, None) == NULL
    n = ctypes.c_size_t(0)
    assert lib.ssm_scan_workspace(None, ctypes.byref(n)) == NULL
    assert lib.ssm_scan_workspace(ctypes.byref(_scan()), None) == NULL


def test_scan_workspace_sizes(lib):
    """256 bytes of status word, then the dt-norm factors (rounded up to 256
    bytes) with SSM_RMSNORM_DT; a workspace one byte short is refused before
    anything is launched."""
    n = ctypes.c_size_t(123)
    assert lib.ssm_scan_workspace(ctypes.byref(_scan()), ctypes.byref(n)) == OK
    assert n.value == 256
    assert lib.ssm_scan_workspace(ctypes.byref(_scan(flags=5)), ctypes.byref(n)) == OK
    assert n.value == 256 + 256  # 2 x 8 factors, rounded up
    assert _call_scan(lib, _scan(flags=5, workspace=P, workspace_bytes=511)) == WS
    assert _call_scan(lib, _scan(workspace=None, workspace_bytes=0)) == WS


def _scan_ws(lib, **kw):
    n = ctypes.c_size_t(0)
    assert lib.ssm_scan_workspace(ctypes.byref(_scan(**kw)), ctypes.byref(n)) == OK
    return n.value


def test_scan_sequence_cut_rule(lib):
    """The pipelined Mamba-1 kernel cuts the sequence into segments only when
    batch x channels leaves the SMs short of warps, and then asks for the
    segments' states in the workspace (sizes for a 148-SM device, which is
    what the query assumes without one)."""
    big = dict(channels=1536, state=16, seqlen=2048)
    assert _scan_ws(lib, batch=8, **big) == 256                  # 1536 warps: whole sequence
    b1 = _scan_ws(lib, batch=1, **big)                           # 192-384 warps: cut
    bcn, bc = 1536 * 16 * 4, 1536 * 4
    # S segments: S - 1 end states, S - 1 step sums, S entering states
    cuts = [S for S in range(2, 33) if b1 == 256 + (S - 1) * bcn + (S - 1) * bc + S * bcn]
    assert len(cuts) == 1 and 2048 // cuts[0] >= 128, b1
    assert _scan_ws(lib, batch=1, channels=1536, state=16, seqlen=64) == 256  # too short
    # per-token states are never cut
    assert _scan_ws(lib, batch=1, states=P, **big) == 256
    # the generic kernel's shapes (state 64) are never cut
    assert _scan_ws(lib, batch=1, channels=1536, state=64, seqlen=2048) == 256


def test_static_entry_checks_before_touching_the_device(lib):
    """ssm_scan_fwd_static runs every host-side check first: on a host with no
    GPU a bad call returns its own status, not SSM_ERR_CUDA."""
    fn = lib.ssm_scan_fwd_static
    assert fn(None, None) == NULL
    assert fn(ctypes.byref(_scan(x=None)), None) == NULL
    assert fn(ctypes.byref(_scan(x=P + 2)), None) == ALIGN
    assert fn(ctypes.byref(_scan(state=12)), None) == UNSUP
    assert fn(ctypes.byref(_scan(io=7)), None) == DTYPE
    # beyond its scratch: batch * seqlen > 262144 with the step norm
    assert fn(ctypes.byref(_scan(flags=5, batch=2, seqlen=131073)), None) == WS
    # batch 0: nothing to do
    assert fn(ctypes.byref(_scan(batch=0, x=None, dt=None, B=None, C=None, A=None,
                                 y=None)), None) == OK


def test_host_entry_checks_before_touching_the_device(lib):
    """ssm_scan_fwd_host runs ssm_scan_fwd's checks, then the workspace
    check, before anything is enqueued: on a host with no GPU a bad call
    returns its own status."""
    fn = lib.ssm_scan_fwd_host
    assert fn(None, None) == NULL
    assert fn(ctypes.byref(_scan(x=None)), None) == NULL
    assert fn(ctypes.byref(_scan(x=P + 2)), None) == ALIGN
    assert fn(ctypes.byref(_scan(state=12)), None) == UNSUP
    assert fn(ctypes.byref(_scan(io=7)), None) == DTYPE
    assert fn(ctypes.byref(_scan(workspace=P, workspace_bytes=255)), None) == WS
    assert fn(ctypes.byref(_scan(batch=0, x=None, dt=None, B=None, C=None, A=None,
                                 y=None)), None) == OK


def _host_ws(lib, **kw):
    n = ctypes.c_size_t(0)
    assert lib.ssm_scan_host_workspace(ctypes.byref(_scan(**kw)), ctypes.byref(n)) == OK
    return n.value


def test_host_workspace_layout(lib):
    """The host entry's device workspace: the scans' own workspace, the
    per-channel constants, then one chunk's copies of the inputs and results
    per slot (two slots when the batch is cut into chunks), each piece
    rounded up to 256 bytes.  The headline shape (b8 L2048 C1536 N16 bf16,
    gate and h_last) runs 8 one-row chunks, never cut along the sequence."""
    big = dict(batch=8, seqlen=2048, channels=1536, state=16, z=P, h_last=P)
    seq = 2048 * 1536 * 2          # x, dt, z or y of one row
    bc = 2048 * 16 * 2             # B or C of one row
    state = 1536 * 16 * 4          # h_last of one row
    slot = 4 * seq + 2 * bc + state
    assert _host_ws(lib, **big) == 256 + 1536 * 16 * 4 + 2 * slot
    # D and dt_bias add one 256-byte-rounded channel vector each
    assert _host_ws(lib, D=P, dt_bias=P, **big) == 256 + 1536 * 16 * 4 + 2 * 6144 + 2 * slot
    # 17 rows: 6 chunks of up to 3 rows
    r17 = dict(big, batch=17)
    assert _host_ws(lib, **r17) == 256 + 1536 * 16 * 4 + 2 * 3 * slot
    # one row: one chunk, one slot, and the scan's workspace holds the
    # segments of the sequence cut (the same size ssm_scan_workspace asks)
    one = dict(big, batch=1)
    n = ctypes.c_size_t(0)
    assert lib.ssm_scan_workspace(ctypes.byref(_scan(**one)), ctypes.byref(n)) == OK
    cut_ws = (n.value + 255) // 256 * 256
    assert cut_ws > 256
    assert _host_ws(lib, **one) == cut_ws + 1536 * 16 * 4 + slot


def test_workspace_status_needs_a_stream_copy(lib):
    assert lib.ssm_workspace_status(None, None) in (OK, 7)  # 7: no device here


def test_scan_empty_batch_is_a_no_op(lib):
    # batch 0: nothing to do, nothing launched, even with NULL tensors
    assert _call_scan(lib, _scan(batch=0, x=None, dt=None, B=None, C=None, A=None,
                                 y=None)) == OK


def _ssd(**kw):
    d = dict(batch=1, seqlen=64, heads=4, head_dim=64, state=128, groups=1, chunk=256,
             io=1, flags=1, x=P, z=None, dt=P, B=P, C=P, A=P, D=None, dt_bias=None,
             h0=None, y=P, h_last=None, states=None)
    d.update(kw)
    return L.SsdArgs(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), NULL), (dict(C=None), NULL), (dict(io=2), DTYPE), (dict(heads=0), SHAPE),
    (dict(groups=3), SHAPE), (dict(chunk=0), SHAPE), (dict(head_dim=6), UNSUP),
    (dict(flags=2), UNSUP), (dict(B=P + 4), ALIGN), (dict(batch=70000), UNSUP),
])
def test_ssd_rejects(lib, kw, status):
    assert lib.ssd_chunk_scan_fwd(ctypes.byref(_ssd(**kw)), None) == status


def _step(**kw):
    d = dict(kind=2, io=1, flags=1, rms_eps=1e-6, batch=4, units=8, head_dim=64, state=128,
             groups=1, x=P, dt=P, z=None, B=P, C=P, A=P, D=None, dt_bias=None, state_io=P,
             y=P)
    d.update(kw)
    return L.StepArgs(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(state_io=None), NULL), (dict(y=None), NULL), (dict(kind=3), UNSUP),
    (dict(io=5), DTYPE), (dict(units=0), SHAPE), (dict(kind=1, head_dim=2), SHAPE),
    (dict(kind=1, head_dim=1, state=12), UNSUP), (dict(flags=4), UNSUP),
    (dict(kind=2, flags=2), UNSUP), (dict(x=P + 1), ALIGN), (dict(groups=3), SHAPE),
])
def test_step_rejects(lib, kw, status):
    assert lib.ssm_scan_step(ctypes.byref(_step(**kw)), None) == status


def test_step_empty_batch_is_a_no_op(lib):
    assert lib.ssm_scan_step(ctypes.byref(_step(batch=0, x=None, dt=None, B=None, C=None,
                                                A=None, state_io=None, y=None)), None) == OK


def test_workspace_queries_need_no_pointers(lib):
    n = ctypes.c_size_t(7)
    a = _scan(x=None, dt=None, B=None, C=None, A=None, y=None, flags=5)
    assert lib.ssm_scan_workspace(ctypes.byref(a), ctypes.byref(n)) == OK
    assert n.value == 256 + 256
    s = _ssd(x=None, dt=None, B=None, C=None, A=None, y=None)
    assert lib.ssd_chunk_scan_workspace(ctypes.byref(s), ctypes.byref(n)) == OK


@pytest.mark.parametrize("batch,heads,seqlen,segs", [
    (4, 80, 4096, (24, 6)),   # 320 units: a 24-unit last wave cut six ways
    (1, 4, 4096, (4, 8)),     # below one wave: 37 ways, capped at 32 tiles / 4
    (1, 150, 1536, (2, 3)),   # 148 whole units, a 2-unit tail cut three ways
    (2, 74, 4096, None),      # 148 units: whole waves, no cut
    (1, 60, 4096, None),      # 148 // 60 = 2 segments: not worth a cut
    (1, 4, 1300, None),       # 11 tiles: fewer than three 4-tile segments
    (1, 8, 128, None),        # one tile
])
def test_ssd_workspace_follows_the_wave_cut(lib, batch, heads, seqlen, segs):
    """With no device the SSD sizes its workspace for 148 SMs: the status word,
    then per tail segment an end state, a carried state and a decay (float32).
    A partial last wave of `tail` units is cut into min(148 // tail, tiles // 4)
    segments when that is three or more."""
    n = ctypes.c_size_t(0)
    s = _ssd(batch=batch, heads=heads, seqlen=seqlen, x=None, dt=None, B=None, C=None, A=None,
             y=None)
    assert lib.ssd_chunk_scan_workspace(ctypes.byref(s), ctypes.byref(n)) == OK
    extra = 0 if segs is None else segs[0] * segs[1] * (2 * 128 * 64 + 4) * 4
    assert n.value == 256 + extra


def _conv(**kw):
    d = dict(batch=2, seqlen=8, channels=64, width=4, io=1, flags=1, x=P, w=P + 0x10000,
             bias=None, state_in=None, u=P + 0x20000, state_out=None)
    d.update(kw)
    return L.ConvArgs(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(width=0), SHAPE), (dict(width=5), UNSUP), (dict(channels=0), SHAPE),
    (dict(batch=-1), SHAPE), (dict(seqlen=-1), SHAPE), (dict(io=7), DTYPE),
    (dict(flags=2), UNSUP), (dict(w=None), NULL), (dict(x=None), NULL), (dict(u=None), NULL),
    (dict(x=P + 4), ALIGN), (dict(state_in=P + 0x30004), ALIGN),
    # x and u overlap (the call's x is 2*8*64*2 bytes)
    (dict(u=P + 0x100), SHAPE),
    # partially overlapping states (equal pointers are the in-place form)
    (dict(state_in=P + 0x30000, state_out=P + 0x30010), SHAPE),
])
def test_conv_rejects(lib, kw, status):
    assert lib.ssm_conv1d_fwd(ctypes.byref(_conv(**kw)), None) == status


def test_conv_empty_batch_is_a_no_op(lib):
    # batch 0: nothing to read or write, no pointer is looked at
    assert lib.ssm_conv1d_fwd(ctypes.byref(_conv(batch=0, x=None, u=None)), None) == OK


def _gnorm(**kw):
    d = dict(rows=8, width=256, io=1, flags=0, eps=1e-5, y=P, z=None, weight=None,
             out=P + 0x10000)
    d.update(kw)
    return L.GatedNormArgs(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(width=0), SHAPE), (dict(rows=-1), SHAPE), (dict(eps=-1.0), SHAPE),
    (dict(eps=float("nan")), SHAPE), (dict(io=5), DTYPE), (dict(flags=1), UNSUP),
    (dict(width=49153, out=P + 0x10000000), UNSUP), (dict(y=None), NULL), (dict(out=None), NULL),
    (dict(y=P + 8), ALIGN), (dict(out=P + 0x100), SHAPE), (dict(z=P + 0x10000), SHAPE),
])
def test_gnorm_rejects(lib, kw, status):
    assert lib.ssm_gated_rmsnorm_fwd(ctypes.byref(_gnorm(**kw)), None) == status


def test_gnorm_empty_is_a_no_op(lib):
    assert lib.ssm_gated_rmsnorm_fwd(ctypes.byref(_gnorm(rows=0, y=None, out=None)), None) == OK


@pytest.mark.parametrize("t,state,status", [
    (-1, P + 0x40000, SHAPE), (8, P + 0x40000, SHAPE), (0, None, NULL), (0, P + 0x40004, ALIGN),
])
def test_scan_write_rejects(lib, t, state, status):
    assert lib.ssm_scan_fwd_write(ctypes.byref(_scan()), t, state, None) == status


def _attn(**kw):
    d = dict(batch=1, seqlen=16, heads=4, state=64, groups=1, io=1, flags=1, dt=P, B=P, C=P,
             A=P, dt_bias=None, alpha=P + 0x100000, workspace=P + 0x200000,
             workspace_bytes=1 << 20)
    d.update(kw)
    return L.AttnArgs(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(heads=0), SHAPE), (dict(groups=3), SHAPE), (dict(state=0), SHAPE),
    (dict(state=257), UNSUP), (dict(io=2), DTYPE), (dict(flags=2), UNSUP),
    (dict(alpha=None), NULL), (dict(dt=None), NULL), (dict(alpha=P + 0x100004), ALIGN),
    (dict(workspace=None), WS), (dict(workspace_bytes=16), WS),
])
def test_attention_rejects(lib, kw, status):
    assert lib.ssd_attention_fwd(ctypes.byref(_attn(**kw)), None) == status


def test_attention_workspace_size(lib):
    n = ctypes.c_size_t(0)
    assert lib.ssd_attention_workspace(ctypes.byref(_attn(batch=2, seqlen=100, heads=8,
                                                          dt=None, B=None)), ctypes.byref(n)) == OK
    # steps and float64 running sums per (batch, head, token), then one
    # 128 x 128 float32 C . B^T tile per (batch, group) for the single tile
    assert n.value == 2 * 8 * 100 * 12 + 2 * 1 * 128 * 128 * 4


def test_empty_calls_launch_nothing(lib):
    """An empty batch (or, where the state needs no pass-through, an empty
    sequence) returns OK before any device call: these run without a GPU."""
    a = _ssd(batch=0, io=0, x=None, dt=None, B=None, C=None, A=None, y=None)
    assert lib.ssd_chunk_scan_fwd(ctypes.byref(a), None) == OK
    # the tensor-core shapes too: no workspace is needed when there is no work
    a = _ssd(batch=0, x=None, dt=None, B=None, C=None, A=None, y=None)
    assert lib.ssd_chunk_scan_fwd(ctypes.byref(a), None) == OK
    a = _ssd(batch=1, x=P, workspace=None)
    assert lib.ssd_chunk_scan_fwd(ctypes.byref(a), None) == WS
    s = _scan(batch=0, x=None, dt=None, B=None, C=None, A=None, y=None)
    assert lib.ssm_scan_fwd_write(ctypes.byref(s), 0, ctypes.c_void_p(P), None) == OK
    for kw in (dict(batch=0), dict(seqlen=0)):
        t = _attn(dt=None, B=None, C=None, A=None, alpha=None, workspace=None,
                  workspace_bytes=0, **kw)
        assert lib.ssd_attention_fwd(ctypes.byref(t), None) == OK


def test_fused_conv_ssd_rejects_before_launch(lib):
    """ssd_conv_chunk_scan_fwd: host checks only (no device is touched)."""
    ctot = 4 * 64 + 2 * 128
    a = L.SsdConvArgs(batch=1, seqlen=8, heads=4, head_dim=64, state=128, groups=1, chunk=256,
                      io=L.SSM_BF16, flags=1, xBC=16, conv_w=16, dt=16, A=16, y=16,
                      conv_state_in=4096, conv_state_out=4096 + 16)
    n = ctypes.c_size_t(0)
    assert lib.ssd_conv_chunk_scan_workspace(ctypes.byref(a), ctypes.byref(n)) == 0
    # status word, then the convolved B and C (8 tokens x 256 channels bf16)
    assert n.value == 256 + 4096
    assert lib.ssd_conv_chunk_scan_fwd(ctypes.byref(a), None) == 2   # the states overlap
    a.conv_state_out = 4096 + ctot * 3 * 4
    assert lib.ssd_conv_chunk_scan_fwd(ctypes.byref(a), None) == 6   # no workspace
    a.xBC = None
    assert lib.ssd_conv_chunk_scan_fwd(ctypes.byref(a), None) == 1   # NULL xBC
    a.xBC = 24
    assert lib.ssd_conv_chunk_scan_fwd(ctypes.byref(a), None) == 4   # misaligned
    a.xBC = 16
    for field, value, code in (("state", 64, 5), ("head_dim", 32, 5), ("io", 0, 5),
                               ("io", 7, 3), ("groups", 3, 2), ("flags", 2, 5)):
        old = getattr(a, field)
        setattr(a, field, value)
        assert lib.ssd_conv_chunk_scan_fwd(ctypes.byref(a), None) == code, field
        setattr(a, field, old)
    a.batch = 0
    assert lib.ssd_conv_chunk_scan_fwd(ctypes.byref(a), None) == 0   # nothing to do
