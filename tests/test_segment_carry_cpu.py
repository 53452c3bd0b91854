"""The identity the SSD's cut of a partial last wave rests on, pinned with the
oracle alone: the Mamba-2 state is linear in the start state with one scalar
decay per head and token ("Mamba-2", nnterp encyclopedia, "The state"), so a
segment run from zeros plus its decay products applied to the state that
entered it gives the run from that state -- for the end state and for every
output of the segment."""
import numpy as np

import oracle
from selective_state_space_28_b200 import inputs as I


def _softplus(v):
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def test_segment_from_zeros_plus_carried_decay_is_the_scan():
    b, L, H, P, N, cut = 2, 300, 3, 8, 16, 113
    d = I.ssd_inputs(b, L, H, P, N, io="f32", seed=7, h0=True)
    x, dt, B, C = d["x"], d["dt"], d["B"], d["C"]
    A, D, bias, h0 = d["A"], d["D"], d["dt_bias"], d["h0"]
    y_full, h_full, _ = oracle.m2_scan(x, dt, B, C, A, D, dt_bias=bias, h0=h0)
    # the state entering the second segment, and that segment from zeros
    _, h_mid, _ = oracle.m2_scan(x[:, :cut], dt[:, :cut], B[:, :cut], C[:, :cut], A, D,
                                 dt_bias=bias, h0=h0)
    y_loc, h_loc, _ = oracle.m2_scan(x[:, cut:], dt[:, cut:], B[:, cut:], C[:, cut:], A, D,
                                     dt_bias=bias)
    # per (batch, token, head): the step and the running log-decay from the cut
    step = _softplus(dt[:, cut:].double().numpy() + bias.double().numpy()[None, None, :])
    logdec = np.cumsum(step * A.double().numpy()[None, None, :], axis=1)     # [b, L2, H]
    # end state: from zeros + the segment's decay product times the entering state
    h_pred = h_loc + np.exp(logdec[:, -1])[:, :, None, None] * h_mid
    np.testing.assert_allclose(h_pred, h_full, rtol=1e-12, atol=1e-12)
    # every output: y_t reads h_t, whose carried part is exp(cum_t) h_mid
    Cn = C[:, cut:].double().numpy()                                         # [b, L2, G, N]
    g = np.arange(H) // (H // Cn.shape[2])
    carried = np.einsum("bthn,bhnp->bthp", Cn[:, :, g, :], h_mid)            # C_t . h_mid
    y_pred = y_loc + np.exp(logdec)[..., None] * carried
    np.testing.assert_allclose(y_pred, y_full[:, cut:], rtol=1e-11, atol=1e-11)


def test_segment_carry_chains_over_several_cuts():
    # the carry kernel's recursion: h_in[s+1] = h_end0[s] + decay[s] * h_in[s]
    b, L, H, P, N = 1, 240, 2, 4, 8
    cuts = [0, 50, 120, 181, 240]
    d = I.ssd_inputs(b, L, H, P, N, io="f32", seed=11, h0=True)
    x, dt, B, C = d["x"], d["dt"], d["B"], d["C"]
    A, D, bias, h0 = d["A"], d["D"], d["dt_bias"], d["h0"]
    _, h_full, _ = oracle.m2_scan(x, dt, B, C, A, D, dt_bias=bias, h0=h0)
    h_in = h0.double().numpy()
    for s0, s1 in zip(cuts[:-1], cuts[1:]):
        sl = slice(s0, s1)
        _, h_end0, _ = oracle.m2_scan(x[:, sl], dt[:, sl], B[:, sl], C[:, sl], A, D,
                                      dt_bias=bias)
        step = _softplus(dt[:, sl].double().numpy() + bias.double().numpy()[None, None, :])
        decay = np.exp((step * A.double().numpy()[None, None, :]).sum(axis=1))   # [b, H]
        h_in = h_end0 + decay[:, :, None, None] * h_in
    np.testing.assert_allclose(h_in, h_full, rtol=1e-12, atol=1e-12)
