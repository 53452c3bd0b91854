"""Python binding of libssm: the C-ABI calls, same names, torch tensors in.

Argument marshalling only: shapes are read off the tensors, outputs and the
workspace are allocated with torch (device memory), and the call is queued
on the current torch stream.  Every step of the scan runs in the library's
CUDA kernels; if ``libssm.so`` is missing these functions raise.

Host tensors are accepted too: they are copied to the GPU on the current
stream, the call runs there, the outputs are copied back into host tensors
(pinned when the inputs were pinned) and the stream is synchronised before
returning.  This is the end-to-end path a caller with host buffers uses; for
ssm_scan_fwd it is the library's own ssm_scan_fwd_host, which overlaps the
copies in both directions with each other and with the scan.
"""
import ctypes

import torch

from . import _lib as L

SOFTPLUS = L.SSM_DT_SOFTPLUS
RMS_BC = L.SSM_RMSNORM_BC
RMS_DT = L.SSM_RMSNORM_DT

_IO = {torch.float32: L.SSM_F32, torch.bfloat16: L.SSM_BF16}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream, device):
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return getattr(stream, "cuda_stream", stream)


class _Staging:
    """Moves host inputs to the device and device outputs back, on one stream."""

    def __init__(self, tensors):
        firsts = [t for t in tensors if t is not None]
        self.host = firsts[0].device.type == "cpu"
        self.pinned = self.host and firsts[0].is_pinned()
        self.device = torch.device("cuda", torch.cuda.current_device()) if self.host \
            else firsts[0].device

    def dev(self, t):
        if t is None:
            return None
        if self.host:
            return t.contiguous().to(self.device, non_blocking=self.pinned)
        return t.contiguous()

    def back(self, outs):
        if not self.host:
            return outs
        res = []
        for t in outs:
            if t is None:
                res.append(None)
                continue
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=self.pinned)
            h.copy_(t, non_blocking=self.pinned)
            res.append(h)
        torch.cuda.current_stream(self.device).synchronize()
        return tuple(res)


def _io_of(x):
    if x.dtype not in _IO:
        raise TypeError("io dtype must be float32 or bfloat16, got %s" % x.dtype)
    return _IO[x.dtype]


_CHECK_ALL = False


def check_every_call(on=True):
    """Make every scan call synchronise and check its status word (as if
    check=True were passed), e.g. for a test session."""
    global _CHECK_ALL
    _CHECK_ALL = bool(on)


def _check_status(ws, stream, where):
    """Synchronise ``stream`` and raise SsmError(SSM_ERR_TIMEOUT) if the call
    that used workspace ``ws`` recorded an expired device wait."""
    L.check(L.lib().ssm_workspace_status(ws.data_ptr(), stream), where)


def _workspace(nbytes, workspace, device):
    if workspace is None or workspace.numel() * workspace.element_size() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace


def ssm_scan_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, *,
                 flags=SOFTPLUS, rms_eps=1e-6, want_states=False, y=None, h_last=None,
                 workspace=None, check=False, stream=None, _write=None):
    """Mamba-1 selective scan (include/ssm.h, ssm_scan_fwd).

    x, dt, z: [b, L, C]; B, C: [b, L, G, N]; A: [C, N] f32; D, dt_bias: [C] f32;
    h0: [b, C, N] f32.  Returns (y [b, L, C], h_last [b, C, N] f32,
    states [b, L, C, N] f32 or None).  With check=True (always for host
    tensors) the stream is synchronised and an expired device wait raises."""
    sg = _Staging([x, dt, A, B, C, D, z, dt_bias, h0])
    if sg.host and _write is None:
        return _scan_host(x, dt, A, B, C, D, z, dt_bias, h0, flags, rms_eps, want_states,
                          y, h_last, workspace, sg, stream)
    x, dt, A, B, C, D, z, dt_bias, h0 = map(sg.dev, (x, dt, A, B, C, D, z, dt_bias, h0))
    if _write is not None:
        _write = (_write[0], sg.dev(_write[1]))
    b, Lq, Cn = x.shape
    G, N = B.shape[2], B.shape[3]
    if y is None:
        y = torch.empty_like(x)
    if h_last is None:
        h_last = torch.empty((b, Cn, N), dtype=torch.float32, device=x.device)
    states = (torch.empty((b, Lq, Cn, N), dtype=torch.float32, device=x.device)
              if want_states else None)
    a = L.ScanArgs(batch=b, seqlen=Lq, channels=Cn, state=N, groups=G, io=_io_of(x),
                   flags=flags, rms_eps=rms_eps, x=_ptr(x), dt=_ptr(dt), z=_ptr(z),
                   B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D), dt_bias=_ptr(dt_bias),
                   h0=_ptr(h0), y=_ptr(y), h_last=_ptr(h_last), states=_ptr(states))
    lib = L.lib()
    nbytes = ctypes.c_size_t(0)
    L.check(lib.ssm_scan_workspace(ctypes.byref(a), ctypes.byref(nbytes)), "ssm_scan_workspace")
    ws = _workspace(nbytes.value, workspace, x.device)
    a.workspace, a.workspace_bytes = ws.data_ptr(), nbytes.value
    st = _stream(stream, x.device)
    if _write is None:
        L.check(lib.ssm_scan_fwd(ctypes.byref(a), st), "ssm_scan_fwd")
    else:
        L.check(lib.ssm_scan_fwd_write(ctypes.byref(a), int(_write[0]), _ptr(_write[1]), st),
                "ssm_scan_fwd_write")
    if check or sg.host or _CHECK_ALL:
        _check_status(ws, st, "ssm_scan_fwd")
    return sg.back((y, h_last, states))


def _scan_host(x, dt, A, B, C, D, z, dt_bias, h0, flags, rms_eps, want_states, y, h_last,
               workspace, sg, stream):
    """ssm_scan_fwd on host tensors through ssm_scan_fwd_host: outputs are host
    tensors (the given ones, else new ones, pinned when the inputs are), the
    workspace device memory; the stream is synchronised and the status word
    checked before returning."""
    x, dt, A, B, C, D, z, dt_bias, h0 = (None if t is None else t.contiguous()
                                         for t in (x, dt, A, B, C, D, z, dt_bias, h0))
    b, Lq, Cn = x.shape
    G, N = B.shape[2], B.shape[3]
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, pin_memory=sg.pinned)
    if h_last is None:
        h_last = torch.empty((b, Cn, N), dtype=torch.float32, pin_memory=sg.pinned)
    states = (torch.empty((b, Lq, Cn, N), dtype=torch.float32, pin_memory=sg.pinned)
              if want_states else None)
    a = L.ScanArgs(batch=b, seqlen=Lq, channels=Cn, state=N, groups=G, io=_io_of(x),
                   flags=flags, rms_eps=rms_eps, x=_ptr(x), dt=_ptr(dt), z=_ptr(z),
                   B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D), dt_bias=_ptr(dt_bias),
                   h0=_ptr(h0), y=_ptr(y), h_last=_ptr(h_last), states=_ptr(states))
    lib = L.lib()
    nbytes = ctypes.c_size_t(0)
    L.check(lib.ssm_scan_host_workspace(ctypes.byref(a), ctypes.byref(nbytes)),
            "ssm_scan_host_workspace")
    ws = _workspace(nbytes.value, workspace, sg.device)
    a.workspace, a.workspace_bytes = ws.data_ptr(), nbytes.value
    st = _stream(stream, sg.device)
    L.check(lib.ssm_scan_fwd_host(ctypes.byref(a), st), "ssm_scan_fwd_host")
    _check_status(ws, st, "ssm_scan_fwd_host")
    return y, h_last, states


def ssm_scan_fwd_write(x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, *, t, state,
                       flags=SOFTPLUS, rms_eps=1e-6, want_states=False, y=None, h_last=None,
                       check=False, stream=None):
    """Mamba-1 scan with the state written at token t (include/ssm.h,
    ssm_scan_fwd_write): h_t is replaced by ``state`` [b, C, N] float32, y_t
    reads it and tokens t+1.. continue from it.  Arguments and results as
    ssm_scan_fwd."""
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    return ssm_scan_fwd(x, dt, A, B, C, D, z, dt_bias, h0, flags=flags, rms_eps=rms_eps,
                        want_states=want_states, y=y, h_last=h_last, check=check,
                        stream=stream, _write=(t, state))


def ssd_workspace_bytes(**shape):
    a = L.SsdArgs(**shape)
    n = ctypes.c_size_t(0)
    L.check(L.lib().ssd_chunk_scan_workspace(ctypes.byref(a), ctypes.byref(n)),
            "ssd_chunk_scan_workspace")
    return n.value


def ssd_conv_workspace_bytes(**shape):
    a = L.SsdConvArgs(**shape)
    n = ctypes.c_size_t(0)
    L.check(L.lib().ssd_conv_chunk_scan_workspace(ctypes.byref(a), ctypes.byref(n)),
            "ssd_conv_chunk_scan_workspace")
    return n.value


def ssd_chunk_scan_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, h0=None, *,
                       chunk=256, flags=SOFTPLUS, want_states=False, y=None, h_last=None,
                       workspace=None, check=False, stream=None):
    """Mamba-2 SSD scan (include/ssm.h, ssd_chunk_scan_fwd).

    x, z: [b, L, H, P]; dt: [b, L, H]; B, C: [b, L, G, N]; A, D, dt_bias: [H] f32;
    h0: [b, H, N, P] f32.  Returns (y, h_last [b, H, N, P], states or None).
    With check=True (always for host tensors) the stream is synchronised and
    an expired device wait raises."""
    sg = _Staging([x, dt, A, B, C, D, z, dt_bias, h0])
    x, dt, A, B, C, D, z, dt_bias, h0 = map(sg.dev, (x, dt, A, B, C, D, z, dt_bias, h0))
    b, Lq, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if y is None:
        y = torch.empty_like(x)
    if h_last is None:
        h_last = torch.empty((b, H, N, P), dtype=torch.float32, device=x.device)
    states = (torch.empty((b, Lq, H, N, P), dtype=torch.float32, device=x.device)
              if want_states else None)
    a = L.SsdArgs(batch=b, seqlen=Lq, heads=H, head_dim=P, state=N, groups=G, chunk=chunk,
                  io=_io_of(x), flags=flags, x=_ptr(x), z=_ptr(z), dt=_ptr(dt), B=_ptr(B),
                  C=_ptr(C), A=_ptr(A), D=_ptr(D), dt_bias=_ptr(dt_bias), h0=_ptr(h0),
                  y=_ptr(y), h_last=_ptr(h_last), states=_ptr(states))
    lib = L.lib()
    nbytes = ctypes.c_size_t(0)
    L.check(lib.ssd_chunk_scan_workspace(ctypes.byref(a), ctypes.byref(nbytes)),
            "ssd_chunk_scan_workspace")
    if nbytes.value:
        workspace = _workspace(nbytes.value, workspace, x.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), nbytes.value
    st = _stream(stream, x.device)
    L.check(lib.ssd_chunk_scan_fwd(ctypes.byref(a), st), "ssd_chunk_scan_fwd")
    if nbytes.value and (check or sg.host or _CHECK_ALL):
        _check_status(workspace, st, "ssd_chunk_scan_fwd")
    return sg.back((y, h_last, states))


def ssd_conv_chunk_scan_fwd(xBC, conv_w, dt, A, *, heads, state, groups=1, conv_bias=None,
                            conv_state_in=None, want_conv_state=False, D=None, z=None,
                            dt_bias=None, h0=None, chunk=256, flags=SOFTPLUS, y=None,
                            h_last=None, conv_state_out=None, workspace=None, check=False,
                            stream=None):
    """The Mamba-2 mixer's causal convolution fused in front of the SSD scan
    (include/ssm.h, ssd_conv_chunk_scan_fwd).

    xBC: [b, L, heads*64 + 2*groups*state] bf16, before the convolution;
    conv_w: [channels, 4] f32; conv_bias: [channels]; conv_state_in:
    [b, channels, 3] f32; dt: [b, L, H]; z: [b, L, H, 64]; A, D, dt_bias: [H];
    h0: [b, H, N, 64].  Returns (y, h_last, conv_state_out or None)."""
    sg = _Staging([xBC, conv_w, dt, A, conv_bias, conv_state_in, D, z, dt_bias, h0])
    xBC, conv_w, dt, A, conv_bias, conv_state_in, D, z, dt_bias, h0 = map(
        sg.dev, (xBC, conv_w, dt, A, conv_bias, conv_state_in, D, z, dt_bias, h0))
    b, Lq, ctot = xBC.shape
    P = (ctot - 2 * groups * state) // heads
    if y is None:
        y = torch.empty((b, Lq, heads, P), dtype=xBC.dtype, device=xBC.device)
    if h_last is None:
        h_last = torch.empty((b, heads, state, P), dtype=torch.float32, device=xBC.device)
    if conv_state_out is None and want_conv_state:
        conv_state_out = torch.empty((b, ctot, 3), dtype=torch.float32, device=xBC.device)
    a = L.SsdConvArgs(batch=b, seqlen=Lq, heads=heads, head_dim=P, state=state, groups=groups,
                      chunk=chunk, io=_io_of(xBC), flags=flags, xBC=_ptr(xBC),
                      conv_w=_ptr(conv_w), conv_bias=_ptr(conv_bias),
                      conv_state_in=_ptr(conv_state_in), conv_state_out=_ptr(conv_state_out),
                      z=_ptr(z), dt=_ptr(dt), A=_ptr(A), D=_ptr(D), dt_bias=_ptr(dt_bias),
                      h0=_ptr(h0), y=_ptr(y), h_last=_ptr(h_last))
    lib = L.lib()
    nbytes = ctypes.c_size_t(0)
    L.check(lib.ssd_conv_chunk_scan_workspace(ctypes.byref(a), ctypes.byref(nbytes)),
            "ssd_conv_chunk_scan_workspace")
    workspace = _workspace(nbytes.value, workspace, xBC.device)
    a.workspace, a.workspace_bytes = workspace.data_ptr(), nbytes.value
    st = _stream(stream, xBC.device)
    L.check(lib.ssd_conv_chunk_scan_fwd(ctypes.byref(a), st), "ssd_conv_chunk_scan_fwd")
    if Lq and (check or sg.host or _CHECK_ALL):
        _check_status(workspace, st, "ssd_conv_chunk_scan_fwd")
    return sg.back((y, h_last, conv_state_out))


def ssm_scan_step(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, *, flags=SOFTPLUS,
                  rms_eps=1e-6, y=None, stream=None):
    """One decode token (include/ssm.h, ssm_scan_step); ``state`` is updated in place.

    Mamba-1: state [b, C, N], x/dt/z [b, C], B/C [b, G, N], A [C, N].
    Mamba-2: state [b, H, N, P], x/z [b, H, P], dt [b, H], B/C [b, G, N], A [H].
    Returns y (and, for host tensors, the updated state copied back)."""
    if state.dim() == 3:
        kind, (b, U, N), P = L.SSM_STEP_MAMBA1, state.shape, 1
    elif state.dim() == 4:
        kind, (b, U, N, P) = L.SSM_STEP_MAMBA2, state.shape
    else:
        raise ValueError("state must be [b, C, N] or [b, H, N, P]")
    sg = _Staging([state, x, dt, A, B, C, D, z, dt_bias])
    host_state = state
    state = state if not sg.host else state.contiguous().to(sg.device, non_blocking=sg.pinned)
    if not state.is_contiguous():
        raise ValueError("state must be contiguous (it is updated in place)")
    x, dt, A, B, C, D, z, dt_bias = map(sg.dev, (x, dt, A, B, C, D, z, dt_bias))
    G = B.shape[1]
    if y is None:
        y = torch.empty_like(x)
    a = L.StepArgs(kind=kind, io=_io_of(x), flags=flags, rms_eps=rms_eps, batch=b, units=U,
                   head_dim=P, state=N, groups=G, x=_ptr(x), dt=_ptr(dt), z=_ptr(z),
                   B=_ptr(B), C=_ptr(C), A=_ptr(A), D=_ptr(D), dt_bias=_ptr(dt_bias),
                   state_io=_ptr(state), y=_ptr(y))
    L.check(L.lib().ssm_scan_step(ctypes.byref(a), _stream(stream, x.device)), "ssm_scan_step")
    if sg.host:
        y_h, st_h = sg.back((y, state))
        host_state.copy_(st_h)
        return y_h
    return y


def ssm_conv1d_fwd(x, w, bias=None, state=None, *, silu=True, u=None, state_out=None,
                   in_place=False, stream=None):
    """The mixers' causal depthwise convolution, then silu (include/ssm.h,
    ssm_conv1d_fwd).

    x: [b, L, C] (float32 or bfloat16); w: [C, W] float32 (W <= 4); bias: [C]
    float32; state: [b, C, W - 1] float32, the inputs before the sequence
    (oldest first) or None for a sequence start.  Returns (u, state_out):
    u [b, L, C] in x's dtype and the last W - 1 inputs.  With in_place=True
    the state tensor itself is updated (the decode form, one token)."""
    sg = _Staging([x, w, bias, state])
    host_state = state
    x, w, bias = map(sg.dev, (x, w, bias))
    if state is not None:
        state = sg.dev(state)
    b, Lq, C = x.shape
    W = w.shape[1]
    if u is None:
        u = torch.empty_like(x)
    if in_place:
        if state is None:
            raise ValueError("in_place needs a state tensor")
        state_out = state
    elif state_out is None:
        state_out = torch.empty((b, C, max(W - 1, 0)), dtype=torch.float32, device=x.device)
    a = L.ConvArgs(batch=b, seqlen=Lq, channels=C, width=W, io=_io_of(x),
                   flags=L.SSM_CONV_SILU if silu else 0, x=_ptr(x), w=_ptr(w),
                   bias=_ptr(bias), state_in=_ptr(state), u=_ptr(u),
                   state_out=_ptr(state_out) if W > 1 else None)
    L.check(L.lib().ssm_conv1d_fwd(ctypes.byref(a), _stream(stream, x.device)),
            "ssm_conv1d_fwd")
    if sg.host:
        u_h, so_h = sg.back((u, state_out))
        if in_place:
            host_state.copy_(so_h)
        return u_h, so_h
    return u, state_out


def ssm_gated_rmsnorm_fwd(y, z=None, weight=None, eps=1e-5, *, out=None, stream=None):
    """The Mamba-2 mixer's gated norm (include/ssm.h, ssm_gated_rmsnorm_fwd):
    y * silu(z), RMS-normalised over the last axis (the mixer's whole width,
    heads x head_dim), times weight.  y, z: [..., width] (float32 or
    bfloat16); weight: [width] float32.  out may be y (in place)."""
    sg = _Staging([y, z, weight])
    y, z, weight = map(sg.dev, (y, z, weight))
    width = y.shape[-1]
    rows = y.numel() // width if width else 0
    if out is None:
        out = torch.empty_like(y)
    a = L.GatedNormArgs(rows=rows, width=width, io=_io_of(y), flags=0, eps=eps, y=_ptr(y),
                        z=_ptr(z), weight=_ptr(weight), out=_ptr(out))
    L.check(L.lib().ssm_gated_rmsnorm_fwd(ctypes.byref(a), _stream(stream, y.device)),
            "ssm_gated_rmsnorm_fwd")
    if sg.host:
        return sg.back((out,))[0]
    return out


def ssd_attention_fwd(dt, A, B, C, dt_bias=None, *, flags=SOFTPLUS, alpha=None,
                      workspace=None, stream=None):
    """The hidden attention of the SSD map (include/ssm.h, ssd_attention_fwd):
    alpha [b, H, L, L] float32 (query t, key s), causal, with
    y_t = sum_s alpha[t, s] x_s + D x_t from a zero state.
    dt [b, L, H] and B, C [b, L, G, N] (float32 or bfloat16); A, dt_bias [H]."""
    sg = _Staging([dt, A, B, C, dt_bias])
    dt, A, B, C, dt_bias = map(sg.dev, (dt, A, B, C, dt_bias))
    b, Lq, H = dt.shape
    G, N = B.shape[2], B.shape[3]
    if alpha is None:
        alpha = torch.empty((b, H, Lq, Lq), dtype=torch.float32, device=dt.device)
    a = L.AttnArgs(batch=b, seqlen=Lq, heads=H, state=N, groups=G, io=_io_of(dt), flags=flags,
                   dt=_ptr(dt), B=_ptr(B), C=_ptr(C), A=_ptr(A), dt_bias=_ptr(dt_bias),
                   alpha=_ptr(alpha))
    lib = L.lib()
    nbytes = ctypes.c_size_t(0)
    L.check(lib.ssd_attention_workspace(ctypes.byref(a), ctypes.byref(nbytes)),
            "ssd_attention_workspace")
    if nbytes.value:
        if workspace is None or workspace.numel() * workspace.element_size() < nbytes.value:
            workspace = torch.empty(nbytes.value, dtype=torch.uint8, device=dt.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), nbytes.value
    L.check(lib.ssd_attention_fwd(ctypes.byref(a), _stream(stream, dt.device)),
            "ssd_attention_fwd")
    if sg.host:
        return sg.back((alpha,))[0]
    return alpha
