"""Float64 CPU oracle for the selective state-space scan.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The
product path (``selective_state_space_28_b200``) never imports it, and the two
share no code: the oracle is plain C (``ssm_oracle.c``) in float64, written as
the pages' token loop, loaded here with ctypes.

Every function takes numpy arrays (any float dtype; they are widened to
float64) and returns float64 numpy arrays.  Sources, per function, are in
``ssm_oracle.h`` / ``ssm_oracle.c``:

* ``m1_scan``    -- "Mamba" (nnterp guide): the per-channel recurrence, the
  values table; "Falcon-Mamba": the weightless norms on B, C and the step.
* ``m2_scan``    -- "Mamba-2" (nnterp encyclopedia): one scalar decay per head
  and token, an N x P state per head, key side first.
* ``m1_step`` / ``m2_step`` -- the decode step: update the state, then read.
* ``m1_quadratic`` / ``m2_quadratic`` -- "Mamba-2", "The hidden attention":
  the O(L^2) masked form, evaluated by brute force.
"""
import ctypes
import os

import numpy as np

from . import build as _build

SOFTPLUS = 1
RMS_BC = 2
RMS_DT = 4

_lib = None
_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        for name, argtypes in {
            "orc_m1_scan": [_I64] * 5 + [ctypes.c_uint32, ctypes.c_double] + [_D] * 12 + [ctypes.c_int],
            "orc_m2_scan": [_I64] * 6 + [ctypes.c_uint32] + [_D] * 12 + [ctypes.c_int],
            "orc_m1_scan_write": [_I64] * 5 + [ctypes.c_uint32, ctypes.c_double] + [_D] * 9
                                 + [_I64, _D] + [_D] * 3 + [ctypes.c_int],
            "orc_m1_step": [_I64] * 4 + [ctypes.c_uint32, ctypes.c_double] + [_D] * 10,
            "orc_m2_step": [_I64] * 5 + [ctypes.c_uint32] + [_D] * 10,
            "orc_m2_quadratic": [_I64] * 6 + [_D] * 9,
            "orc_m1_quadratic": [_I64] * 5 + [_D] * 9,
            "orc_conv1d": [_I64] * 4 + [_D] * 4 + [ctypes.c_int] + [_D] * 2,
            "orc_gated_rmsnorm": [_I64] * 2 + [ctypes.c_double] + [_D] * 4,
            "orc_m2_attention": [_I64] * 5 + [ctypes.c_uint32] + [_D] * 6,
        }.items():
            fn = getattr(lib, name)
            fn.argtypes = argtypes
            fn.restype = ctypes.c_int
        lib.orc_softplus.argtypes = [ctypes.c_double]
        lib.orc_softplus.restype = ctypes.c_double
        lib.orc_silu.argtypes = [ctypes.c_double]
        lib.orc_silu.restype = ctypes.c_double
        lib.orc_rms_rows.argtypes = [_I64, _I64, ctypes.c_double, _D, _D]
        lib.orc_rms_rows.restype = None
        _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # a torch tensor: widen on the host
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(_D) if a is not None else None


def default_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def m1_scan(x, dt, B, C, A, D=None, z=None, dt_bias=None, h0=None, *,
            flags=SOFTPLUS, rms_eps=1e-6, want_states=False, nthreads=None):
    """Mamba-1 scan.  x, dt, z: [b, L, C]; B, C: [b, L, G, N]; A: [C, N].

    Returns (y [b,L,C], h_last [b,C,N], states [b,L,C,N] or None)."""
    x, dt, z, B, C, A, D, dt_bias, h0 = map(_f64, (x, dt, z, B, C, A, D, dt_bias, h0))
    b, L, Cn = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.empty_like(x)
    h_last = np.empty((b, Cn, N))
    states = np.empty((b, L, Cn, N)) if want_states else None
    rc = _load().orc_m1_scan(b, L, Cn, N, G, flags, rms_eps, _p(x), _p(dt), _p(z),
                             _p(B), _p(C), _p(A), _p(D), _p(dt_bias), _p(h0),
                             _p(y), _p(h_last), _p(states),
                             nthreads or default_threads())
    if rc:
        raise ValueError("orc_m1_scan failed: %d" % rc)
    return y, h_last, states


def m1_scan_write(x, dt, B, C, A, D=None, z=None, dt_bias=None, h0=None, *, t, state,
                  flags=SOFTPLUS, rms_eps=1e-6, want_states=False, nthreads=None):
    """Mamba-1 scan with the state written at token t ("Mamba", nnterp guide,
    "The state"): after token t's update the state is replaced by ``state``
    [b, C, N]; y_t reads it and tokens t+1.. continue from it.
    Returns (y, h_last, states or None) as m1_scan."""
    x, dt, z, B, C, A, D, dt_bias, h0, state = map(
        _f64, (x, dt, z, B, C, A, D, dt_bias, h0, state))
    b, L, Cn = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.empty_like(x)
    h_last = np.empty((b, Cn, N))
    states = np.empty((b, L, Cn, N)) if want_states else None
    rc = _load().orc_m1_scan_write(b, L, Cn, N, G, flags, rms_eps, _p(x), _p(dt), _p(z),
                                   _p(B), _p(C), _p(A), _p(D), _p(dt_bias), _p(h0),
                                   int(t), _p(state), _p(y), _p(h_last), _p(states),
                                   nthreads or default_threads())
    if rc:
        raise ValueError("orc_m1_scan_write failed: %d" % rc)
    return y, h_last, states


def m2_scan(x, dt, B, C, A, D=None, z=None, dt_bias=None, h0=None, *,
            flags=SOFTPLUS, want_states=False, nthreads=None):
    """Mamba-2 scan.  x, z: [b, L, H, P]; dt: [b, L, H]; B, C: [b, L, G, N].

    Returns (y [b,L,H,P], h_last [b,H,N,P], states [b,L,H,N,P] or None)."""
    x, dt, z, B, C, A, D, dt_bias, h0 = map(_f64, (x, dt, z, B, C, A, D, dt_bias, h0))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.empty_like(x)
    h_last = np.empty((b, H, N, P))
    states = np.empty((b, L, H, N, P)) if want_states else None
    rc = _load().orc_m2_scan(b, L, H, P, N, G, flags, _p(x), _p(dt), _p(z), _p(B),
                             _p(C), _p(A), _p(D), _p(dt_bias), _p(h0), _p(y),
                             _p(h_last), _p(states), nthreads or default_threads())
    if rc:
        raise ValueError("orc_m2_scan failed: %d" % rc)
    return y, h_last, states


def m1_step(state, x, dt, B, C, A, D=None, z=None, dt_bias=None, *,
            flags=SOFTPLUS, rms_eps=1e-6):
    """One Mamba-1 decode token.  state: [b, C, N]; x, dt, z: [b, C];
    B, C: [b, G, N].  Returns (new_state, y)."""
    st = _f64(state).copy()
    x, dt, z, B, C, A, D, dt_bias = map(_f64, (x, dt, z, B, C, A, D, dt_bias))
    b, Cn = x.shape
    G, N = B.shape[1], B.shape[2]
    y = np.empty_like(x)
    rc = _load().orc_m1_step(b, Cn, N, G, flags, rms_eps, _p(x), _p(dt), _p(z), _p(B),
                             _p(C), _p(A), _p(D), _p(dt_bias), _p(st), _p(y))
    if rc:
        raise ValueError("orc_m1_step failed: %d" % rc)
    return st, y


def m2_step(state, x, dt, B, C, A, D=None, z=None, dt_bias=None, *, flags=SOFTPLUS):
    """One Mamba-2 decode token.  state: [b, H, N, P]; x, z: [b, H, P];
    dt: [b, H]; B, C: [b, G, N].  Returns (new_state, y)."""
    st = _f64(state).copy()
    x, dt, z, B, C, A, D, dt_bias = map(_f64, (x, dt, z, B, C, A, D, dt_bias))
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    y = np.empty_like(x)
    rc = _load().orc_m2_step(b, H, P, N, G, flags, _p(x), _p(dt), _p(z), _p(B),
                             _p(C), _p(A), _p(D), _p(dt_bias), _p(st), _p(y))
    if rc:
        raise ValueError("orc_m2_step failed: %d" % rc)
    return st, y


def m2_quadratic(x, betas, B, C, A, D=None, z=None, h0=None):
    """Brute-force hidden-attention form (Mamba-2 layout); betas = the step
    after bias and softplus, [b, L, H]."""
    x, betas, z, B, C, A, D, h0 = map(_f64, (x, betas, z, B, C, A, D, h0))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.empty_like(x)
    rc = _load().orc_m2_quadratic(b, L, H, P, N, G, _p(x), _p(betas), _p(z), _p(B),
                                  _p(C), _p(A), _p(D), _p(h0), _p(y))
    if rc:
        raise ValueError("orc_m2_quadratic failed: %d" % rc)
    return y


def m1_quadratic(x, betas, B, C, A, D=None, z=None, h0=None):
    """Brute-force hidden-attention form (Mamba-1 layout); betas: [b, L, C]."""
    x, betas, z, B, C, A, D, h0 = map(_f64, (x, betas, z, B, C, A, D, h0))
    b, L, Cn = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.empty_like(x)
    rc = _load().orc_m1_quadratic(b, L, Cn, N, G, _p(x), _p(betas), _p(z), _p(B),
                                  _p(C), _p(A), _p(D), _p(h0), _p(y))
    if rc:
        raise ValueError("orc_m1_quadratic failed: %d" % rc)
    return y


def conv1d(x, w, bias=None, state=None, act=True):
    """Causal depthwise convolution over tokens, then silu when act (the
    mixers' conv1d: module tree, kernel W, padding W - 1, groups = channels;
    "Mamba-2" "The mixer's values", "Mamba" tokentrails "Code").
    x [b, L, C]; w [C, W]; bias [C]; state [b, C, W - 1] (inputs before the
    sequence, oldest first) or None for zeros.  Returns (u [b, L, C],
    state_out [b, C, W - 1])."""
    x, w, bias, state = _f64(x), _f64(w), _f64(bias), _f64(state)
    b, L, C = x.shape
    W = w.shape[1]
    u = np.zeros((b, L, C))
    so = np.zeros((b, C, max(W - 1, 0)))
    rc = _load().orc_conv1d(b, L, C, W, _p(x), _p(w), _p(bias), _p(state), int(bool(act)),
                            _p(u), _p(so) if W > 1 else None)
    if rc:
        raise ValueError("orc_conv1d: bad arguments")
    return u, so


def gated_rmsnorm(y, z=None, weight=None, eps=1e-5):
    """The Mamba-2 mixer's gated norm over the last axis (the mixer's whole
    width): y * silu(z), then RMS-normalised, then times weight ("Mamba-2",
    "The mixer's values" and the paragraph on the block's norms).
    y, z: [..., width]; weight: [width].  Returns float64 of y's shape."""
    y, z, weight = _f64(y), _f64(z), _f64(weight)
    width = y.shape[-1]
    rows = int(np.prod(y.shape[:-1])) if y.ndim > 1 else 1
    out = np.zeros_like(y)
    rc = _load().orc_gated_rmsnorm(rows, width, float(eps), _p(y), _p(z), _p(weight), _p(out))
    if rc:
        raise ValueError("orc_gated_rmsnorm: bad arguments")
    return out


def m2_attention(dt, B, C, A, dt_bias=None, *, flags=SOFTPLUS, heads=None):
    """The hidden attention of the Mamba-2 map ("Mamba-2", "The hidden
    attention"): alpha [b, H, L, L] (query t, key s), causal, with
    y_t = sum_s alpha[t, s] x_s + D x_t from a zero state.
    dt [b, L, H]; B, C [b, L, G, N]; A, dt_bias [H]."""
    dt, B, C, A, dt_bias = map(_f64, (dt, B, C, A, dt_bias))
    b, L, H = dt.shape
    G, N = B.shape[2], B.shape[3]
    alpha = np.zeros((b, H, L, L))
    rc = _load().orc_m2_attention(b, L, H, N, G, flags, _p(dt), _p(B), _p(C), _p(A),
                                  _p(dt_bias), _p(alpha))
    if rc:
        raise ValueError("orc_m2_attention: bad arguments")
    return alpha


def softplus(v):
    lib = _load()
    return np.vectorize(lib.orc_softplus, otypes=[np.float64])(np.asarray(v, np.float64))


def silu(v):
    lib = _load()
    return np.vectorize(lib.orc_silu, otypes=[np.float64])(np.asarray(v, np.float64))


def rms_rows(v, eps):
    v = _f64(v)
    out = np.empty_like(v)
    n = v.shape[-1]
    _load().orc_rms_rows(v.size // n, n, eps, _p(v), _p(out))
    return out


# ------------------------------------------------------------------ the block
# "Falcon-Mamba" and "Mamba-2" (nnterp encyclopedia), "The block, in order":
# out = x + mixer(norm(x)), the add in float32 (residual_in_fp32); the mixer's
# output (attention_output) is in the load dtype and is all the block adds
# ("The contribution is the whole block").  The blocks below are wrappers for
# the oracle's residual-identity checks: seeded random weights, the oracle's
# own scan as the mixer's core, library matmuls for the projections.

def _round_to(a, load_dtype):
    """Round float64 values to the load dtype, returned as float32."""
    if load_dtype == "float32":
        return np.asarray(a, dtype=np.float32)
    if load_dtype == "bfloat16":
        import torch
        return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()
    raise ValueError("load dtype %r" % load_dtype)


def _rmsnorm_gain(h, w, eps):
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps) * w


def falcon_mamba_block(h, W, *, rms_eps=1e-6, norm_eps=1e-5, load_dtype="float32"):
    """One Falcon-Mamba block ("Falcon-Mamba", "The block, in order" and
    "Where the norms sit"): norm, in_proj to (u, z), silu(conv1d(u)), x_proj to
    the low-rank step and B, C, the three weightless RMS norms, dt_proj, the
    scan with D*u and the silu(z) gate, out_proj; then the residual add.

    h: [b, L, d_model]; W: dict of weights (norm, in_proj, conv_w, conv_b,
    x_proj, dt_proj_w, dt_proj_b, A, D, out_proj).  Returns (layer_output
    float32, attention_output in the load dtype, widened to float32)."""
    h64 = _f64(h)
    R, N = W["dt_proj_w"].shape[1], W["A"].shape[1]
    hn = _rmsnorm_gain(h64, W["norm"], norm_eps)
    uz = hn @ W["in_proj"].T
    di = uz.shape[-1] // 2
    u, z = uz[..., :di], uz[..., di:]
    u, _ = conv1d(u, W["conv_w"], W["conv_b"], act=True)
    dbc = u @ W["x_proj"].T
    low = rms_rows(dbc[..., :R], rms_eps)
    Bn = rms_rows(dbc[..., R:R + N], rms_eps)
    Cn = rms_rows(dbc[..., R + N:], rms_eps)
    dt = low @ W["dt_proj_w"].T
    y, _, _ = m1_scan(u, dt, Bn[:, :, None, :], Cn[:, :, None, :], W["A"], W["D"], z=z,
                      dt_bias=W["dt_proj_b"])
    attn = _round_to(y @ W["out_proj"].T, load_dtype)
    out = np.asarray(h, dtype=np.float32) + attn       # the add, in float32
    return out, attn


def mamba2_block(h, W, *, heads, groups=1, norm_eps=1e-5, load_dtype="float32"):
    """One Mamba-2 block ("Mamba-2", "The block, in order"): norm, in_proj to
    (z, xBC, dt), silu(conv1d(xBC)) split into x, B, C, the SSD with D*x, the
    gated norm over the mixer's width, out_proj; then the residual add.

    h: [b, L, d_model]; W: dict (norm, in_proj, conv_w, conv_b, A, D,
    dt_bias, gnorm, out_proj).  Returns (layer_output float32,
    attention_output in the load dtype, widened to float32)."""
    h64 = _f64(h)
    b, L, _ = h64.shape
    di = W["out_proj"].shape[1]
    N = (W["conv_w"].shape[0] - di) // (2 * groups)
    hn = _rmsnorm_gain(h64, W["norm"], norm_eps)
    proj = hn @ W["in_proj"].T
    z, xbc, dt = proj[..., :di], proj[..., di:2 * di + 2 * groups * N], proj[..., -heads:]
    xbc, _ = conv1d(xbc, W["conv_w"], W["conv_b"], act=True)
    x = xbc[..., :di].reshape(b, L, heads, di // heads)
    Bm = xbc[..., di:di + groups * N].reshape(b, L, groups, N)
    Cm = xbc[..., di + groups * N:].reshape(b, L, groups, N)
    y, _, _ = m2_scan(x, dt, Bm, Cm, W["A"], W["D"], dt_bias=W["dt_bias"])
    g = gated_rmsnorm(y.reshape(b, L, di), z, W["gnorm"], eps=norm_eps)
    attn = _round_to(g @ W["out_proj"].T, load_dtype)
    out = np.asarray(h, dtype=np.float32) + attn       # the add, in float32
    return out, attn
