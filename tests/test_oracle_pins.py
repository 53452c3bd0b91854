"""Pins of the float64 oracle to facts that do not come from the oracle itself.

Each test fixes one part of the oracle against a closed form, a library
routine, a brute-force sum, an invariant the pages state, or a number the
pages print.  tests/test_oracle_mutants.py checks that plausible mistakes in
the oracle's source fail at least one of these pins.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng


def _m1_rand(b, L, C, N, G=1, seed=0, h0=True, z=True):
    r = rng(seed)
    d = dict(x=r.standard_normal((b, L, C)), dt=r.standard_normal((b, L, C)),
             B=r.standard_normal((b, L, G, N)), C=r.standard_normal((b, L, G, N)),
             A=-np.exp(r.uniform(-1, 1.5, (C, N))), D=r.standard_normal(C),
             dt_bias=r.uniform(-4, -1, C))
    d["z"] = r.standard_normal((b, L, C)) if z else None
    d["h0"] = r.standard_normal((b, C, N)) if h0 else None
    return d


def _m2_rand(b, L, H, P, N, G=1, seed=0, h0=True, z=True):
    r = rng(seed)
    d = dict(x=r.standard_normal((b, L, H, P)), dt=r.standard_normal((b, L, H)),
             B=r.standard_normal((b, L, G, N)), C=r.standard_normal((b, L, G, N)),
             A=-np.exp(r.uniform(0, 2.7, H)), D=r.standard_normal(H),
             dt_bias=r.uniform(-4, -1, H))
    d["z"] = r.standard_normal((b, L, H, P)) if z else None
    d["h0"] = r.standard_normal((b, H, N, P)) if h0 else None
    return d


# ------------------------------------------------------- elementwise pieces

def test_softplus_matches_library():
    v = np.concatenate([np.linspace(-60, 60, 2401), [-1e300, 0.0, 1e-12, -1e-12, 700.0]])
    got = oracle.softplus(v)
    ref = np.logaddexp(0.0, v)                      # numpy: log(exp(0) + exp(v))
    np.testing.assert_allclose(got, ref, rtol=1e-15, atol=0)
    ref_t = F.softplus(torch.tensor(v), beta=1.0, threshold=1e9).numpy()
    np.testing.assert_allclose(got[:-1], ref_t[:-1], rtol=1e-14, atol=1e-300)
    assert oracle.softplus(np.array([-np.inf]))[0] == 0.0   # a zero step stays zero


def test_silu_matches_library():
    v = np.linspace(-40, 40, 1601)
    np.testing.assert_allclose(oracle.silu(v), F.silu(torch.tensor(v)).numpy(),
                               rtol=1e-14, atol=1e-300)


def test_rms_matches_library():
    v = rng(1).standard_normal((37, 16)) * 3.0
    for eps in (1e-6, 1e-5, 0.5):
        ref = F.rms_norm(torch.tensor(v), (16,), eps=eps).numpy()
        np.testing.assert_allclose(oracle.rms_rows(v, eps), ref, rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------- closed forms

def test_m1_zero_decay_is_cumulative_sum():
    """A = 0: nothing decays, so h_t = sum_{s<=t} dt_s B_s x_s (a running sum)."""
    d = _m1_rand(2, 23, 5, 3, seed=2, h0=False, z=False)
    d["A"] = np.zeros_like(d["A"])
    y, h_last, states = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"],
                                       flags=0, want_states=True)
    w = d["dt"][..., None] * d["x"][..., None] * d["B"][:, :, 0, None, :]  # [b,L,C,N]
    h = np.cumsum(w, axis=1)
    np.testing.assert_allclose(states, h, rtol=1e-12, atol=1e-12)
    y_ref = np.einsum("bln,blcn->blc", d["C"][:, :, 0, :], h) + d["D"] * d["x"]
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h_last, h[:, -1], rtol=1e-12, atol=1e-12)


def test_m1_zero_step_is_skip_connection():
    """dt = 0: no write and no decay ("Mamba-2", a zero step skips a token
    exactly); y reduces to the gated skip D*x*silu(z) and the state is h0."""
    d = _m1_rand(2, 17, 6, 4, seed=3)
    zero = np.zeros_like(d["dt"])
    y, h_last, states = oracle.m1_scan(d["x"], zero, d["B"], d["C"], d["A"], d["D"],
                                       z=d["z"], h0=d["h0"], flags=0, want_states=True)
    assert np.array_equal(h_last, d["h0"])
    assert np.array_equal(states, np.broadcast_to(d["h0"][:, None], states.shape))
    ch0 = np.einsum("bln,bcn->blc", d["C"][:, :, 0, :], d["h0"])
    sig = 1.0 / (1.0 + np.exp(-d["z"]))
    np.testing.assert_allclose(y, (ch0 + d["D"] * d["x"]) * d["z"] * sig, rtol=1e-13, atol=1e-13)


def test_m1_single_state_geometric_series():
    """N = 1 with constant inputs: h_t = a^t h0 + beta (1 - a^t) / (1 - a)."""
    L, a_log, dt, Bv, Cv, xv, h0 = 40, -0.7, 0.3, 1.7, -0.4, 0.9, 2.5
    ones = np.ones((1, L, 1))
    y, h_last, states = oracle.m1_scan(xv * ones, dt * ones, Bv * ones[..., None],
                                       Cv * ones[..., None], np.array([[a_log]]),
                                       np.zeros(1), h0=np.array([[[h0]]]), flags=0,
                                       want_states=True)
    a, beta = math.exp(dt * a_log), dt * Bv * xv
    t = np.arange(1, L + 1)
    h = a ** t * h0 + beta * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(states[0, :, 0, 0], h, rtol=1e-13)
    np.testing.assert_allclose(y[0, :, 0], Cv * h, rtol=1e-13)


def test_m1_time_invariant_is_a_convolution():
    """Same step, B and C at every token (the S4 case of "Mamba", tokentrails,
    step 3): y = K * x with K_k = sum_n C_n exp(dt A_n)^k dt B_n, plus D x."""
    r = rng(5)
    L, N = 50, 4
    x = r.standard_normal((1, L, 1))
    dt, A = 0.21, -np.exp(r.uniform(-1, 1, (1, N)))
    Bv, Cv, D = r.standard_normal(N), r.standard_normal(N), 0.37
    y, _, _ = oracle.m1_scan(x, np.full((1, L, 1), dt), np.tile(Bv, (1, L, 1, 1)),
                             np.tile(Cv, (1, L, 1, 1)), A, np.array([D]), flags=0)
    k = np.arange(L)
    K = (Cv[None, :] * np.exp(dt * A[0])[None, :] ** k[:, None] * dt * Bv[None, :]).sum(1)
    y_ref = np.convolve(x[0, :, 0], K)[:L] + D * x[0, :, 0]
    np.testing.assert_allclose(y[0, :, 0], y_ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- brute force

@pytest.mark.parametrize("G", [1, 2])
def test_m2_scan_equals_hidden_attention(G):
    """"Mamba-2", "The hidden attention": the scan equals the causal masked
    form sum_s (C_t.B_s) exp(decays_{s+1..t}) betas_s x_s + D x_t (brute force)."""
    d = _m2_rand(2, 19, 4, 3, 5, G=G, seed=6)
    y, _, _ = oracle.m2_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                             dt_bias=d["dt_bias"], h0=d["h0"])
    betas = oracle.softplus(d["dt"] + d["dt_bias"])
    y_q = oracle.m2_quadratic(d["x"], betas, d["B"], d["C"], d["A"], d["D"], z=d["z"],
                              h0=d["h0"])
    np.testing.assert_allclose(y, y_q, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("G", [1, 3])
def test_m1_scan_equals_hidden_attention(G):
    d = _m1_rand(2, 14, 6, 4, G=G, seed=7)
    y, _, _ = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                             dt_bias=d["dt_bias"], h0=d["h0"])
    betas = oracle.softplus(d["dt"] + d["dt_bias"])
    y_q = oracle.m1_quadratic(d["x"], betas, d["B"], d["C"], d["A"], d["D"], z=d["z"],
                              h0=d["h0"])
    np.testing.assert_allclose(y, y_q, rtol=1e-11, atol=1e-11)


def test_hidden_attention_by_running_products():
    """The masked form rebuilt another way: per head, the transfer matrix
    T[t, s] = prod_{s<r<=t} exp(betas_r A_h) built one row at a time from
    the row above (T[t, :t] = a_t T[t-1, :t], T[t, t] = 1), then
    y = ((C B^T) * T * betas) x + D x as numpy matrix products.  It agrees
    with the brute-force sum, which sums exponents instead of multiplying
    factors."""
    H, Lq, P, N = 3, 12, 4, 6
    d = _m2_rand(1, Lq, H, P, N, G=1, seed=8, h0=False, z=False)
    betas = oracle.softplus(d["dt"] + d["dt_bias"])[0]            # [L, H]
    y_t = np.zeros((Lq, H, P))
    for h in range(H):
        a = np.exp(betas[:, h] * d["A"][h])
        T = np.zeros((Lq, Lq))
        for t in range(Lq):
            if t:
                T[t, :t] = a[t] * T[t - 1, :t]
            T[t, t] = 1.0
        cb = d["C"][0, :, 0, :] @ d["B"][0, :, 0, :].T               # [t, s]
        M = cb * T * betas[None, :, h]
        y_t[:, h, :] = M @ d["x"][0, :, h, :] + d["D"][h] * d["x"][0, :, h, :]
    y_q = oracle.m2_quadratic(d["x"], betas[None], d["B"], d["C"], d["A"], d["D"])
    np.testing.assert_allclose(y_q[0], y_t, rtol=1e-11, atol=1e-11)


# ------------------------------------------------------------------ invariants

def test_split_and_carry_equals_full_scan():
    """Carrying state_output into the next call's state_input continues the
    scan exactly ("Mamba-2", "The state"; "Mamba", decode hand-off)."""
    d = _m1_rand(2, 31, 5, 4, seed=9)
    full = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                          dt_bias=d["dt_bias"], h0=d["h0"], want_states=True)
    for k in (1, 13, 30):
        sl = lambda a, s: None if a is None else a[:, s]
        a = oracle.m1_scan(*(sl(d[n], slice(0, k)) for n in ("x", "dt", "B", "C")),
                           d["A"], d["D"], z=sl(d["z"], slice(0, k)), dt_bias=d["dt_bias"],
                           h0=d["h0"])
        b = oracle.m1_scan(*(sl(d[n], slice(k, None)) for n in ("x", "dt", "B", "C")),
                           d["A"], d["D"], z=sl(d["z"], slice(k, None)),
                           dt_bias=d["dt_bias"], h0=a[1])
        assert np.array_equal(np.concatenate([a[0], b[0]], 1), full[0])
        assert np.array_equal(b[1], full[1])
    d2 = _m2_rand(1, 20, 2, 3, 4, seed=10)
    f2 = oracle.m2_scan(d2["x"], d2["dt"], d2["B"], d2["C"], d2["A"], d2["D"], z=d2["z"],
                        dt_bias=d2["dt_bias"], h0=d2["h0"])
    a = oracle.m2_scan(d2["x"][:, :7], d2["dt"][:, :7], d2["B"][:, :7], d2["C"][:, :7],
                       d2["A"], d2["D"], z=d2["z"][:, :7], dt_bias=d2["dt_bias"], h0=d2["h0"])
    b = oracle.m2_scan(d2["x"][:, 7:], d2["dt"][:, 7:], d2["B"][:, 7:], d2["C"][:, 7:],
                       d2["A"], d2["D"], z=d2["z"][:, 7:], dt_bias=d2["dt_bias"], h0=a[1])
    assert np.array_equal(np.concatenate([a[0], b[0]], 1), f2[0])
    assert np.array_equal(b[1], f2[1])


def test_last_state_equals_state_output():
    """states[:, -1] == state_output, bit for bit ("Mamba-2", "The state")."""
    d = _m1_rand(2, 9, 3, 4, seed=11)
    _, h_last, states = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"],
                                       dt_bias=d["dt_bias"], h0=d["h0"], want_states=True)
    assert np.array_equal(states[:, -1], h_last)
    d2 = _m2_rand(2, 9, 2, 3, 4, seed=12)
    _, h2, s2 = oracle.m2_scan(d2["x"], d2["dt"], d2["B"], d2["C"], d2["A"], d2["D"],
                               dt_bias=d2["dt_bias"], h0=d2["h0"], want_states=True)
    assert np.array_equal(s2[:, -1], h2)


def test_zero_step_token_keeps_state_bitwise():
    """A zero step at token 3 leaves states[:, 3] == states[:, 2] exactly
    ("Mamba-2", "A zero step skips a token exactly"); dt_raw = -inf gives a
    softplus step of exactly 0."""
    d = _m2_rand(1, 8, 3, 4, 5, seed=13)
    d["dt"][:, 3] = -np.inf
    _, _, s = oracle.m2_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"],
                             dt_bias=d["dt_bias"], h0=d["h0"], want_states=True)
    assert np.array_equal(s[:, 3], s[:, 2])
    m = _m1_rand(1, 8, 3, 4, seed=14)
    m["dt"][:, 3] = -np.inf
    _, _, s1 = oracle.m1_scan(m["x"], m["dt"], m["B"], m["C"], m["A"], m["D"],
                              dt_bias=m["dt_bias"], h0=m["h0"], want_states=True)
    assert np.array_equal(s1[:, 3], s1[:, 2])


def test_mamba2_is_mamba1_with_shared_decay():
    """A Mamba-2 head of P channels is P Mamba-1 channels whose A[c, :] are
    all A_h and whose step is the head's: the two recurrences coincide."""
    H, P, N = 3, 4, 5
    d = _m2_rand(2, 11, H, P, N, seed=15)
    y2, h2, _ = oracle.m2_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                               dt_bias=d["dt_bias"], h0=d["h0"])
    b, L = 2, 11
    rep = lambda v: np.repeat(v, P, axis=-1)
    y1, h1, _ = oracle.m1_scan(d["x"].reshape(b, L, H * P), rep(d["dt"]), d["B"], d["C"],
                               np.repeat(d["A"], P)[:, None] * np.ones((1, N)),
                               rep(d["D"]), z=d["z"].reshape(b, L, H * P),
                               dt_bias=rep(d["dt_bias"]),
                               h0=d["h0"].transpose(0, 1, 3, 2).reshape(b, H * P, N))
    np.testing.assert_allclose(y1.reshape(y2.shape), y2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h1.reshape(b, H, P, N).transpose(0, 1, 3, 2), h2,
                               rtol=1e-12, atol=1e-12)


def test_step_is_scan_of_one_token():
    """The decode step equals the scan of one token from the cached state, with
    y read after the update ("Mamba", "Read order on a decode step")."""
    d = _m1_rand(3, 1, 7, 4, G=1, seed=16)
    y, h_last, _ = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"],
                                  z=d["z"], dt_bias=d["dt_bias"], h0=d["h0"])
    st, ys = oracle.m1_step(d["h0"], d["x"][:, 0], d["dt"][:, 0], d["B"][:, 0], d["C"][:, 0],
                            d["A"], d["D"], z=d["z"][:, 0], dt_bias=d["dt_bias"])
    assert np.array_equal(st, h_last) and np.array_equal(ys, y[:, 0])
    e = _m2_rand(2, 1, 3, 4, 5, seed=17)
    y2, h2, _ = oracle.m2_scan(e["x"], e["dt"], e["B"], e["C"], e["A"], e["D"], z=e["z"],
                               dt_bias=e["dt_bias"], h0=e["h0"])
    st2, ys2 = oracle.m2_step(e["h0"], e["x"][:, 0], e["dt"][:, 0], e["B"][:, 0],
                              e["C"][:, 0], e["A"], e["D"], z=e["z"][:, 0],
                              dt_bias=e["dt_bias"])
    assert np.array_equal(st2, h2) and np.array_equal(ys2, y2[:, 0])


def test_norm_flags_act_on_the_stated_axes():
    """"Falcon-Mamba", "Where the norms sit": B and C are RMS-normed over the
    state axis, the step input over its last axis (the channels), before the
    bias and softplus.  Pre-norming with torch's rms_norm gives the same scan."""
    d = _m1_rand(2, 10, 6, 4, seed=18)
    eps = 1e-6
    y, h, _ = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                             dt_bias=d["dt_bias"], h0=d["h0"],
                             flags=oracle.SOFTPLUS | oracle.RMS_BC | oracle.RMS_DT,
                             rms_eps=eps)
    rn = lambda v, n: F.rms_norm(torch.tensor(v), (n,), eps=eps).numpy()
    y2, h2, _ = oracle.m1_scan(d["x"], rn(d["dt"], 6), rn(d["B"], 4), rn(d["C"], 4),
                               d["A"], d["D"], z=d["z"], dt_bias=d["dt_bias"], h0=d["h0"],
                               flags=oracle.SOFTPLUS)
    np.testing.assert_allclose(y, y2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h, h2, rtol=1e-13, atol=1e-13)
    st, ys = oracle.m1_step(d["h0"], d["x"][:, 0], d["dt"][:, 0], d["B"][:, 0], d["C"][:, 0],
                            d["A"], d["D"], z=d["z"][:, 0], dt_bias=d["dt_bias"],
                            flags=oracle.SOFTPLUS | oracle.RMS_BC | oracle.RMS_DT,
                            rms_eps=eps)
    y1, h1, _ = oracle.m1_scan(d["x"][:, :1], d["dt"][:, :1], d["B"][:, :1], d["C"][:, :1],
                               d["A"], d["D"], z=d["z"][:, :1], dt_bias=d["dt_bias"],
                               h0=d["h0"],
                               flags=oracle.SOFTPLUS | oracle.RMS_BC | oracle.RMS_DT,
                               rms_eps=eps)
    np.testing.assert_allclose(st, h1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(ys, y1[:, 0], rtol=1e-13, atol=1e-13)


def test_extreme_rates_stay_finite():
    """The pages quote A down to -36316 and up to -4e-4 ("Mamba-2", "The
    mixer's values"); large steps then drive the decay to 0, tiny ones to 1."""
    d = _m1_rand(1, 30, 4, 4, seed=19)
    d["A"][0] = -36316.0
    d["A"][1] = -4e-4
    d["dt"][0, ::3] = 30.0
    d["dt"][0, 1::3] = -30.0
    y, h, _ = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                             dt_bias=d["dt_bias"], h0=d["h0"])
    assert np.isfinite(y).all() and np.isfinite(h).all()
    # channel 0 forgets everything on a step of ~30: its state is the last write
    betas = oracle.softplus(d["dt"][0, -1, 0] + d["dt_bias"][0])
    np.testing.assert_allclose(h[0, 0], betas * d["B"][0, -1, 0] * d["x"][0, -1, 0],
                               rtol=1e-12, atol=1e-300)


# ------------------------------------------------------ printed page values

def _golden():
    with open(os.path.join(GOLDEN, "page_shapes.json")) as f:
        return json.load(f)


def test_page_shapes():
    """The oracle's outputs carry the layouts the pages print for a 10-token
    prompt on mamba-130m and for mamba2-130m's state."""
    g = _golden()
    t = g["mamba1_trace"]
    d = _m1_rand(t["batch"], t["seqlen"], t["channels"], t["state"], seed=20)
    y, h, s = oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                             dt_bias=d["dt_bias"], want_states=True)
    assert list(d["B"].shape) == t["B"] and list(d["C"].shape) == t["C"]
    assert list(d["x"].shape) == t["x"] and list(d["dt"].shape) == t["dt"]
    assert list(y.shape) == t["y"] and list(h.shape) == t["state_output"]
    assert list(s.shape) == g["mamba1_states"]["states"]
    st, ys = oracle.m1_step(h, d["x"][:, 0], d["dt"][:, 0], d["B"][:, 0], d["C"][:, 0],
                            d["A"], d["D"], z=d["z"][:, 0], dt_bias=d["dt_bias"])
    assert list(st.shape) == g["mamba1_decode"]["state_input"]
    assert list(ys[:, None].shape) == g["mamba1_decode"]["y"]
    m = g["mamba2_130m"]
    e = _m2_rand(1, 3, m["heads"], m["head_dim"], m["state"], seed=21)
    _, h2, _ = oracle.m2_scan(e["x"], e["dt"], e["B"], e["C"], e["A"], e["D"])
    assert list(h2.shape[1:]) == m["state_output_tail"]


def test_page_state_sizes():
    """The state the scan hands on has the size the pages print: 1.3 MiB for
    Mamba-130m (crossing GPT-2's 36 KiB/token cache near 38 tokens) and 82 MiB
    for Mamba-2 2.7B, both in bf16 and counting the width-4 convolution's
    three carried tokens."""
    g = _golden()
    m = g["mamba130m_memory"]
    ssm = m["layers"] * m["channels"] * m["state"] * m["bytes_per_value"]
    conv = m["layers"] * m["channels"] * (m["conv_width"] - 1) * m["bytes_per_value"]
    mib = (ssm + conv) / 2 ** 20
    assert round(mib, 1) == m["state_mib_printed"]
    kv = m["gpt2_layers"] * 2 * m["gpt2_d_model"] * m["bytes_per_value"]
    assert kv / 1024 == m["gpt2_kib_per_token"]
    assert round((ssm + conv) / kv) == m["crossover_tokens"]
    q = g["mamba2_2p7b_memory"]
    d_inner = q["expand"] * q["d_model"]
    assert d_inner == q["heads"] * q["head_dim"]
    ssm2 = q["layers"] * q["heads"] * q["state"] * q["head_dim"] * q["bytes_per_value"]
    conv2 = q["layers"] * (d_inner + 2 * q["groups"] * q["state"]) * (q["conv_width"] - 1) \
        * q["bytes_per_value"]
    assert round((ssm2 + conv2) / 2 ** 20) == q["state_mib_printed"]


# ---------------------------------------------------------------- conv1d
# The mixers' causal depthwise convolution ("Mamba-2" module tree: Conv1d,
# kernel 4, padding 3, groups = channels; "The mixer's values" and "Mamba"
# tokentrails "Code": silu(conv1d(.)), causal, width 4).

def test_conv1d_matches_library_convolution():
    # Per channel, a causal convolution is the first L terms of the full
    # convolution with the kernel reversed (weight k multiplies the input
    # W - 1 - k tokens back): numpy's convolve is an independent routine.
    r = rng(40)
    x, w, bias = r.standard_normal((2, 37, 6)), r.standard_normal((6, 4)), r.standard_normal(6)
    u, _ = oracle.conv1d(x, w, bias, act=False)
    for b in range(2):
        for c in range(6):
            ref = np.convolve(x[b, :, c], w[c, ::-1])[:37] + bias[c]
            np.testing.assert_allclose(u[b, :, c], ref, rtol=0, atol=1e-12)


def test_conv1d_matches_torch_module_layout():
    # The module tree's layer itself: Conv1d(C, C, 4, padding=3, groups=C) on
    # [b, C, L], output cut to the first L positions.
    r = rng(41)
    x, w, bias = r.standard_normal((2, 19, 5)), r.standard_normal((5, 4)), r.standard_normal(5)
    u, _ = oracle.conv1d(x, w, bias, act=True)
    xt = torch.tensor(x).transpose(1, 2)
    ref = F.conv1d(xt, torch.tensor(w).unsqueeze(1), torch.tensor(bias), padding=3, groups=5)
    ref = F.silu(ref[..., :19]).transpose(1, 2).numpy()
    np.testing.assert_allclose(u, ref, rtol=0, atol=1e-12)


def test_conv1d_impulse_response_orientation():
    # One nonzero input at t0: the output at t0 + j is the weight that
    # multiplies an input j tokens back, w[W - 1 - j]; nothing before t0.
    w = np.array([[0.1, 0.2, 0.3, 0.4]])
    x = np.zeros((1, 12, 1))
    x[0, 5, 0] = 1.0
    u, _ = oracle.conv1d(x, w, act=False)
    assert np.all(u[0, :5, 0] == 0.0)
    assert list(u[0, 5:9, 0]) == [0.4, 0.3, 0.2, 0.1]
    assert np.all(u[0, 9:, 0] == 0.0)


def test_conv1d_constant_input_from_a_cold_start():
    # Constant input c with no history: the first W - 1 outputs see only the
    # tokens since the start (partial sums of the newest weights), the rest
    # the full sum.
    w = np.array([[1.0, 2.0, 4.0, 8.0]])
    x = np.full((1, 6, 1), 3.0)
    u, st = oracle.conv1d(x, w, bias=np.array([0.5]), act=False)
    assert list(u[0, :, 0]) == [0.5 + 24.0, 0.5 + 36.0, 0.5 + 42.0, 0.5 + 45.0, 45.5, 45.5]
    assert list(st[0, 0]) == [3.0, 3.0, 3.0]


def test_conv1d_split_and_carry_equals_full():
    # The conv state carries the last W - 1 inputs: a sequence cut anywhere
    # (also before W - 1 tokens) gives the same outputs, bit for bit.
    r = rng(42)
    x, w, bias = r.standard_normal((2, 23, 7)), r.standard_normal((7, 4)), r.standard_normal(7)
    st0 = r.standard_normal((2, 7, 3))
    u, st = oracle.conv1d(x, w, bias, state=st0)
    for cut in (1, 2, 3, 10, 22):
        u1, s1 = oracle.conv1d(x[:, :cut], w, bias, state=st0)
        u2, s2 = oracle.conv1d(x[:, cut:], w, bias, state=s1)
        assert np.array_equal(np.concatenate([u1, u2], axis=1), u)
        assert np.array_equal(s2, st)


def test_conv1d_state_is_the_history():
    # Running one token at a time from a state equals running the whole
    # sequence: the decode form of the same convolution.
    r = rng(43)
    x, w = r.standard_normal((1, 9, 3)), r.standard_normal((3, 4))
    st = r.standard_normal((1, 3, 3))
    u_full, st_full = oracle.conv1d(x, w, state=st)
    s = st
    for t in range(9):
        u1, s = oracle.conv1d(x[:, t:t + 1], w, state=s)
        assert np.array_equal(u1[:, 0], u_full[:, t])
    assert np.array_equal(s, st_full)
    # and the state is literally the last three inputs
    assert np.array_equal(st_full[0], x[0, -3:].T)


def test_conv1d_width_one_is_elementwise():
    r = rng(44)
    x, w, bias = r.standard_normal((2, 5, 4)), r.standard_normal((4, 1)), r.standard_normal(4)
    u, st = oracle.conv1d(x, w, bias, act=True)
    v = x * w[:, 0] + bias
    np.testing.assert_allclose(u, v / (1 + np.exp(-v)), rtol=1e-15, atol=0)
    assert st.shape == (2, 4, 0)


# ------------------------------------------------------------ gated norm
# "Mamba-2": out_proj(norm(y * silu(z))); the gated norm multiplies y by
# silu(z), then normalizes over the mixer's whole width, whatever n_groups is.

def test_gated_norm_matches_library():
    r = rng(50)
    y, z, wt = r.standard_normal((3, 5, 96)), r.standard_normal((3, 5, 96)), r.standard_normal(96)
    out = oracle.gated_rmsnorm(y, z, wt, eps=1e-5)
    g = torch.tensor(y) * F.silu(torch.tensor(z))
    ref = F.rms_norm(g, (96,), torch.tensor(wt), eps=1e-5).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_gated_norm_spans_the_whole_width():
    # Normalizing per group (here per half of the width) gives a different
    # answer: the norm's statistic is the whole row's.
    r = rng(51)
    y = r.standard_normal((4, 64))
    y[:, 32:] *= 10.0
    out = oracle.gated_rmsnorm(y, eps=0.0)
    np.testing.assert_allclose(np.mean(out ** 2, axis=-1), 1.0, rtol=1e-12)
    halves = np.concatenate([oracle.gated_rmsnorm(y[:, :32], eps=0.0),
                             oracle.gated_rmsnorm(y[:, 32:], eps=0.0)], axis=-1)
    assert np.max(np.abs(halves - out)) > 0.1


def test_gated_norm_gate_before_norm_and_scale_invariance():
    r = rng(52)
    y, z = r.standard_normal((2, 40)), r.standard_normal((2, 40))
    out = oracle.gated_rmsnorm(y, z, eps=0.0)
    # the gate acts before the norm: out is g / rms(g), g = y * silu(z)
    g = y * z / (1 + np.exp(-z))
    np.testing.assert_allclose(out, g / np.sqrt(np.mean(g ** 2, axis=-1, keepdims=True)),
                               rtol=1e-13)
    # and without eps the result does not depend on the scale of y
    np.testing.assert_allclose(oracle.gated_rmsnorm(7.5 * y, z, eps=0.0), out, rtol=1e-13)
    # no gate: a plain RMS norm
    np.testing.assert_allclose(oracle.gated_rmsnorm(y, None, eps=1e-3),
                               y / np.sqrt(np.mean(y ** 2, axis=-1, keepdims=True) + 1e-3),
                               rtol=1e-13)


# ------------------------------------------------------- state write at t
# "Mamba" (nnterp guide), "The state": writing the state at token t replaces
# h_t; y_t reads the written state and later tokens continue from it.

def test_state_write_of_the_same_state_changes_nothing():
    d = _m1_rand(2, 11, 6, 4, seed=60)
    y, h, st = oracle.m1_scan(**d, want_states=True)
    for t in (0, 4, 10):
        y2, h2, st2 = oracle.m1_scan_write(**d, t=t, state=st[:, t], want_states=True)
        assert np.array_equal(y2, y) and np.array_equal(h2, h) and np.array_equal(st2, st)


def test_state_write_zero_restarts_the_scan():
    # writing zeros at t: y_t = D x_t (gated) exactly, and the tokens after t
    # are a fresh scan from a zero state, bit for bit
    d = _m1_rand(2, 12, 5, 3, seed=61)
    t = 5
    y, h, st = oracle.m1_scan_write(**d, t=t, state=np.zeros((2, 5, 3)), want_states=True)
    z = d["z"][:, t]
    np.testing.assert_array_equal(y[:, t], d["D"] * d["x"][:, t] * (z / (1 + np.exp(-z))))
    assert np.all(st[:, t] == 0.0)
    tail = {k: (v[:, t + 1:] if k in ("x", "dt", "z", "B", "C") else v) for k, v in d.items()}
    tail["h0"] = None
    y_t, h_t, _ = oracle.m1_scan(**tail)
    assert np.array_equal(y[:, t + 1:], y_t) and np.array_equal(h, h_t)
    # and the tokens before t are untouched
    y_full, _, _ = oracle.m1_scan(**d)
    assert np.array_equal(y[:, :t], y_full[:, :t])


def test_state_write_at_the_last_token_is_the_last_state():
    d = _m1_rand(1, 7, 4, 2, seed=62)
    s = rng(63).standard_normal((1, 4, 2))
    y, h, _ = oracle.m1_scan_write(**d, t=6, state=s)
    assert np.array_equal(h, s)
    # y_6 = C_6 . s + D x_6, gated
    c6, x6, z6 = d["C"][0, 6, 0], d["x"][0, 6], d["z"][0, 6]
    ref = (s[0] @ c6 + d["D"] * x6) * (z6 / (1 + np.exp(-z6)))
    np.testing.assert_allclose(y[0, 6], ref, rtol=1e-14)


# ------------------------------------------------------ hidden attention
# "Mamba-2", "The hidden attention": alpha[t, s] = (C_t . B_s) *
# exp(decays_{s+1} + ... + decays_t) * betas_s, causal, one [seq, seq]
# matrix per head; y_t = sum_s alpha[t, s] x_s + D x_t.

def test_attention_rebuilds_the_scan(G=1):
    d = _m2_rand(2, 23, 4, 3, 5, G=G, seed=70, h0=False, z=False)
    al = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"])
    y, _, _ = oracle.m2_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"],
                             dt_bias=d["dt_bias"])
    y_att = np.einsum("bhts,bshp->bthp", al, d["x"]) + d["D"][None, None, :, None] * d["x"]
    np.testing.assert_allclose(y_att, y, rtol=1e-10, atol=1e-12)


def test_attention_columns_are_impulse_responses():
    """Column s of a head's attention matrix is that head's response to a
    unit input at token s: the oracle scan with one value channel, x = 1 at
    token s and 0 elsewhere, zero start state and no skip term, returns
    y_t = alpha[t, s] for every t."""
    b, Lq, H, N, G = 1, 11, 4, 5, 2
    d = _m2_rand(b, Lq, H, 1, N, G=G, seed=71, h0=False, z=False)
    al = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"])
    for s in range(Lq):
        x = np.zeros((b, Lq, H, 1))
        x[:, s] = 1.0
        y, _, _ = oracle.m2_scan(x, d["dt"], d["B"], d["C"], d["A"], np.zeros(H),
                                 dt_bias=d["dt_bias"])
        np.testing.assert_allclose(al[0, :, :, s], y[0, :, :, 0].T, rtol=1e-12, atol=1e-15)


def test_attention_is_causal_with_a_plain_diagonal():
    d = _m2_rand(1, 9, 2, 2, 3, G=2, seed=72, h0=False, z=False)
    al = oracle.m2_attention(d["dt"], d["B"], d["C"], d["A"], d["dt_bias"])
    assert np.all(np.triu(al[0, 0], 1) == 0.0) and np.all(np.triu(al[0, 1], 1) == 0.0)
    # no decay between a token and itself: alpha[t, t] = (C_t . B_t) betas_t
    beta = np.logaddexp(0.0, d["dt"][0] + d["dt_bias"])
    for h in range(2):
        for t in range(9):
            cb = d["C"][0, t, h] @ d["B"][0, t, h]
            assert al[0, h, t, t] == pytest.approx(cb * beta[t, h], rel=1e-13, abs=0)


def test_attention_without_decay_is_masked_cb():
    d = _m2_rand(1, 8, 2, 2, 4, G=1, seed=73, h0=False, z=False)
    al = oracle.m2_attention(d["dt"], d["B"], d["C"], np.zeros(2), d["dt_bias"], flags=0)
    beta = d["dt"][0] + d["dt_bias"]                                   # no softplus
    cb = d["C"][0, :, 0] @ d["B"][0, :, 0].T
    for h in range(2):
        np.testing.assert_allclose(al[0, h], np.tril(cb * beta[None, :, h]), rtol=1e-14)


# ------------------------------------------------------------------ the block
# "Falcon-Mamba" / "Mamba-2" (nnterp encyclopedia), "The block, in order" and
# "The contribution is the whole block": out = x + mixer(norm(x)), the add in
# float32, the mixer's output in the load dtype.

def _falcon_weights(seed, dm=8, di=16, N=4, R=3):
    r = rng(seed)
    return dict(norm=1 + 0.1 * r.standard_normal(dm),
                in_proj=r.standard_normal((2 * di, dm)) / 3,
                conv_w=r.uniform(-0.5, 0.5, (di, 4)), conv_b=r.uniform(-0.5, 0.5, di),
                x_proj=r.standard_normal((R + 2 * N, di)) / 4,
                dt_proj_w=r.standard_normal((di, R)) / 2, dt_proj_b=r.uniform(-4, -1, di),
                A=-np.exp(r.uniform(-1, 1.5, (di, N))), D=r.standard_normal(di),
                out_proj=r.standard_normal((dm, di)) / 4)


def _mamba2_weights(seed, dm=8, H=4, P=4, N=4, G=2):
    r = rng(seed)
    di = H * P
    conv = di + 2 * G * N
    return dict(norm=1 + 0.1 * r.standard_normal(dm),
                in_proj=r.standard_normal((di + conv + H, dm)) / 3,
                conv_w=r.uniform(-0.5, 0.5, (conv, 4)), conv_b=r.uniform(-0.5, 0.5, conv),
                A=-np.exp(r.uniform(0, 2.7, H)), D=r.standard_normal(H),
                dt_bias=r.uniform(-4, -1, H), gnorm=1 + 0.1 * r.standard_normal(di),
                out_proj=r.standard_normal((dm, di)) / 4)


def _block(kind, h, W, **kw):
    if kind == "falcon":
        return oracle.falcon_mamba_block(h, W, **kw)
    return oracle.mamba2_block(h, W, heads=4, groups=2, **kw)


@pytest.mark.parametrize("kind", ["falcon", "mamba2"])
@pytest.mark.parametrize("load", ["float32", "bfloat16"])
def test_block_output_is_input_plus_mixer_output_in_float32(kind, load):
    """layer_input + attention_output == layer_output, bit for bit, with the
    add done in float32 on the mixer output rounded to the load dtype."""
    W = _falcon_weights(80) if kind == "falcon" else _mamba2_weights(81)
    h = rng(82).standard_normal((2, 9, 8)) * 3
    out, attn = _block(kind, h, W, load_dtype=load)
    assert out.dtype == np.float32
    direct = np.add(h.astype(np.float32), attn.astype(np.float32), dtype=np.float32)
    np.testing.assert_array_equal(out, direct)
    if load == "bfloat16":  # attention_output really is in the load dtype
        bits = attn.astype(np.float32).view(np.uint32)
        assert np.all(bits & 0xFFFF == 0)


@pytest.mark.parametrize("kind", ["falcon", "mamba2"])
def test_block_without_the_mixer_output_is_the_identity(kind):
    """Ablating attention_output (out_proj = 0) ablates the block: the stream
    passes through unchanged."""
    W = _falcon_weights(83) if kind == "falcon" else _mamba2_weights(84)
    W["out_proj"] = np.zeros_like(W["out_proj"])
    h = rng(85).standard_normal((1, 7, 8))
    out, attn = _block(kind, h, W)
    assert not attn.any()
    np.testing.assert_array_equal(out, h.astype(np.float32))


@pytest.mark.parametrize("kind", ["falcon", "mamba2"])
def test_block_contribution_reads_only_the_normed_input(kind):
    """The mixer sees norm(x), so scaling the stream by c > 0 leaves the
    mixer's output unchanged (the norm's eps taken to ~0) while the output
    moves by exactly the residual: out(c x) - c x == out(x) - x."""
    W = _falcon_weights(86) if kind == "falcon" else _mamba2_weights(87)
    h = rng(88).standard_normal((1, 10, 8))
    _, a1 = _block(kind, h, W, norm_eps=1e-300)
    _, a3 = _block(kind, 3.0 * h, W, norm_eps=1e-300)
    np.testing.assert_allclose(a3, a1, rtol=1e-6, atol=1e-7)
