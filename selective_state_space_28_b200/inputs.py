"""Seeded synthetic inputs for the scan workloads.

This module only draws numbers; it holds none of the scan's arithmetic.  The
same draws feed the CUDA library and the float64 oracle, so both read
identical values: every tensor is rounded to its I/O dtype here, on the host,
before anyone reads it.

Recipe (the pages print no dataset; these follow the shapes of the models
the pages describe):

* ``A = -exp(A_log)`` with ``A_log[c, n] = log(n + 1)`` for Mamba-1 (the
  S4D-real initialisation, "Mamba" tokentrails "Code": ``A = -exp(A_log)``),
  and ``A_h = -exp(U[log 1, log 16])`` per head for Mamba-2.
* ``dt_bias = softplus^-1(dt0)``, ``dt0 = exp(U[log 1e-3, log 0.1])`` per
  channel / head (1e-3 is the configs' ``time_step_min``).
* ``D = 1``; ``x, z, dt_raw, B, C ~ N(0, 1)``; decode states ``~ N(0, 0.1^2)``.
* Draw order: A, dt_bias, D, x, z, dt_raw, B, C, then the state.
* Convolution (the mixers' conv1d): ``x ~ N(0, 1)``; weight and bias
  ``U(-1/sqrt(W), 1/sqrt(W))``, the layer's default initialisation for a
  depthwise kernel of width W (fan-in W); conv state ``~ N(0, 1)`` (it holds
  past inputs).  Draw order: w, bias, x, state.  The Mamba-2 2.7B channel
  count is d_inner + 2 G N = 5120 + 256 (the module tree's Conv1d over xBC).
* Gated norm: ``y, z ~ N(0, 1)`` (the SSD's output and the gate), weight
  ``1 + 0.1 N(0, 1)`` (the norm's ones initialisation, perturbed so that the
  weight is exercised); eps 1e-5 (the Mamba-2 configs' layer-norm epsilon).
  Draw order: weight, y, z.
"""
import math
from dataclasses import dataclass, field
from typing import Optional

import torch

SOFTPLUS = 1
RMS_BC = 2
RMS_DT = 4


@dataclass(frozen=True)
class Workload:
    """One named scan workload.  ``kind`` is "m1", "ssd", "ssd_conv" (the SSD
    with the mixer's convolution in front), "decode", "conv", "gnorm" or
    "attn" (the SSD map's hidden attention; its inputs are the SSD's)."""
    name: str
    kind: str
    batch: int
    seqlen: int = 1
    channels: int = 0          # Mamba-1 inner width
    heads: int = 0             # Mamba-2 heads
    head_dim: int = 0
    state: int = 16
    groups: int = 1
    chunk: int = 256
    io: str = "bf16"
    gate: bool = True
    flags: int = SOFTPLUS
    rms_eps: float = 1e-6
    want_states: bool = False
    layers: int = 1            # decode stacks: one call per layer
    m1_layers: int = 0         # decode stacks: Mamba-1 layers after the Mamba-2 ones
    m1_channels: int = 0
    m1_state: int = 16
    seed: int = 0
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    # Mamba-1 toy scan, float32 I/O, with the per-token states.
    "m1_toy_b1_l64_c32_n4_f32": Workload(
        "m1_toy_b1_l64_c32_n4_f32", "m1", batch=1, seqlen=64, channels=32,
        state=4, io="f32", gate=True, want_states=True, seed=0),
    # One Mamba-130m-shaped mixer scan (inner width 1536, state 16).
    "m1_130m_b8_l2048_c1536_n16_bf16": Workload(
        "m1_130m_b8_l2048_c1536_n16_bf16", "m1", batch=8, seqlen=2048,
        channels=1536, state=16, io="bf16", gate=True, seed=1),
    # The same mixer scan for a single prompt (batch 1): too few (batch,
    # channel) chains to fill the SMs, so the scan cuts the sequence into
    # segments joined by the state carry.
    "m1_130m_b1_l2048_c1536_n16_bf16": Workload(
        "m1_130m_b1_l2048_c1536_n16_bf16", "m1", batch=1, seqlen=2048,
        channels=1536, state=16, io="bf16", gate=True, seed=8),
    # Falcon-Mamba-7B width (8192) with the weightless norms, long sequence.
    "m1_falcon_rms_b4_l8192_c8192_n16_bf16": Workload(
        "m1_falcon_rms_b4_l8192_c8192_n16_bf16", "m1", batch=4, seqlen=8192,
        channels=8192, state=16, io="bf16", gate=True,
        flags=SOFTPLUS | RMS_BC | RMS_DT, seed=2),
    # One prompt at the Falcon width (the profiling case of that kernel: its
    # inputs exceed L2 while a capture stays a few GB).
    "m1_falcon_rms_b1_l8192_c8192_n16_bf16": Workload(
        "m1_falcon_rms_b1_l8192_c8192_n16_bf16", "m1", batch=1, seqlen=8192,
        channels=8192, state=16, io="bf16", gate=True,
        flags=SOFTPLUS | RMS_BC | RMS_DT, seed=9),
    # Mamba-2 2.7B-shaped SSD chunk scan (80 heads x 64, state 128, chunk 256).
    "ssd_2p7b_b4_l4096_h80_p64_n128_bf16": Workload(
        "ssd_2p7b_b4_l4096_h80_p64_n128_bf16", "ssd", batch=4, seqlen=4096,
        heads=80, head_dim=64, state=128, chunk=256, io="bf16", gate=False,
        seed=3),
    # Decode across a Mamba-2 2.7B stack (64 layers) plus a Mamba-130m stack
    # (24 layers of 1536 x 16), batch 256, one token per layer.
    "decode_2p7b_stack_b256": Workload(
        "decode_2p7b_stack_b256", "decode", batch=256, heads=80, head_dim=64,
        state=128, io="bf16", gate=False, layers=64, m1_layers=24,
        m1_channels=1536, m1_state=16, seed=4),
    # One layer of each decode stack (a small case of the same kernels).
    "decode_2p7b_layer_b256": Workload(
        "decode_2p7b_layer_b256", "decode", batch=256, heads=80, head_dim=64,
        state=128, io="bf16", gate=False, layers=1, m1_layers=1,
        m1_channels=1536, m1_state=16, seed=4),
    # The Mamba-2 2.7B mixer's causal convolution over xBC (d_inner 5120 plus
    # B and C, 2 x 128) for the SSD workload's prompt, with a carried state.
    "conv_2p7b_b4_l4096_c5376_bf16": Workload(
        "conv_2p7b_b4_l4096_c5376_bf16", "conv", batch=4, seqlen=4096, channels=5376,
        io="bf16", seed=5, extra={"width": 4, "state": True}),
    # The SSD workload with the mixer's causal convolution fused in front:
    # xBC of 5120 + 2 x 128 channels before the convolution, a carried conv
    # state.
    "ssd_conv_2p7b_b4_l4096_h80_p64_n128_bf16": Workload(
        "ssd_conv_2p7b_b4_l4096_h80_p64_n128_bf16", "ssd_conv", batch=4, seqlen=4096,
        heads=80, head_dim=64, state=128, chunk=256, io="bf16", gate=False, seed=10,
        extra={"state": True}),
    # The Mamba-2 2.7B mixer's gated norm after the SSD workload: one row of
    # heads x head_dim = 5120 values per token.
    "gnorm_2p7b_b4_l4096_w5120_bf16": Workload(
        "gnorm_2p7b_b4_l4096_w5120_bf16", "gnorm", batch=4, seqlen=4096, channels=5120,
        io="bf16", gate=True, rms_eps=1e-5, seed=6),
    # The hidden attention of the Mamba-2 2.7B map for one 1024-token prompt:
    # 80 heads x 1024 x 1024 float32 (the interpretability workload).
    "attn_2p7b_b1_l1024_h80_n128_bf16": Workload(
        "attn_2p7b_b1_l1024_h80_n128_bf16", "attn", batch=1, seqlen=1024, heads=80,
        head_dim=64, state=128, io="bf16", gate=False, seed=7),
}


def _dtype(io):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[io]


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, dtype, device, std=1.0):
    t = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _dt_bias(n, g, device):
    # dt0 = exp(U[log 1e-3, log 1e-1]); bias = dt0 + log(-expm1(-dt0)) is the
    # inverse of softplus at dt0.
    u = torch.rand(n, generator=g, dtype=torch.float64, device=device)
    dt0 = torch.exp(u * (math.log(0.1) - math.log(1e-3)) + math.log(1e-3))
    return (dt0 + torch.log(-torch.expm1(-dt0))).to(torch.float32)


def m1_inputs(batch, seqlen, channels, state, groups=1, io="bf16", gate=True,
              seed=0, h0=False, device="cpu"):
    """Inputs of one Mamba-1 scan: dict of tensors on ``device``."""
    g = _gen(seed, device)
    dt_ = _dtype(io)
    A_log = torch.log(torch.arange(1, state + 1, dtype=torch.float32, device=device))
    A = (-torch.exp(A_log)).unsqueeze(0).expand(channels, state).contiguous()
    out = {"A": A, "dt_bias": _dt_bias(channels, g, device),
           "D": torch.ones(channels, dtype=torch.float32, device=device)}
    out["x"] = _randn((batch, seqlen, channels), g, dt_, device)
    out["z"] = _randn((batch, seqlen, channels), g, dt_, device) if gate else None
    out["dt"] = _randn((batch, seqlen, channels), g, dt_, device)
    out["B"] = _randn((batch, seqlen, groups, state), g, dt_, device)
    out["C"] = _randn((batch, seqlen, groups, state), g, dt_, device)
    out["h0"] = (_randn((batch, channels, state), g, torch.float32, device, 0.1)
                 if h0 else None)
    return out


def ssd_inputs(batch, seqlen, heads, head_dim, state, groups=1, io="bf16",
               gate=False, seed=0, h0=False, device="cpu"):
    """Inputs of one Mamba-2 SSD scan: dict of tensors on ``device``."""
    g = _gen(seed, device)
    dt_ = _dtype(io)
    u = torch.rand(heads, generator=g, dtype=torch.float64, device=device)
    A = (-torch.exp(u * math.log(16.0))).to(torch.float32)
    out = {"A": A, "dt_bias": _dt_bias(heads, g, device),
           "D": torch.ones(heads, dtype=torch.float32, device=device)}
    out["x"] = _randn((batch, seqlen, heads, head_dim), g, dt_, device)
    out["z"] = _randn((batch, seqlen, heads, head_dim), g, dt_, device) if gate else None
    out["dt"] = _randn((batch, seqlen, heads), g, dt_, device)
    out["B"] = _randn((batch, seqlen, groups, state), g, dt_, device)
    out["C"] = _randn((batch, seqlen, groups, state), g, dt_, device)
    out["h0"] = (_randn((batch, heads, state, head_dim), g, torch.float32, device, 0.1)
                 if h0 else None)
    return out


def m2_step_inputs(batch, heads, head_dim, state, groups=1, io="bf16", gate=False,
                   seed=0, device="cpu"):
    """One Mamba-2 decode token plus its cached state ~ N(0, 0.1^2)."""
    g = _gen(seed, device)
    dt_ = _dtype(io)
    u = torch.rand(heads, generator=g, dtype=torch.float64, device=device)
    A = (-torch.exp(u * math.log(16.0))).to(torch.float32)
    out = {"A": A, "dt_bias": _dt_bias(heads, g, device),
           "D": torch.ones(heads, dtype=torch.float32, device=device)}
    out["x"] = _randn((batch, heads, head_dim), g, dt_, device)
    out["z"] = _randn((batch, heads, head_dim), g, dt_, device) if gate else None
    out["dt"] = _randn((batch, heads), g, dt_, device)
    out["B"] = _randn((batch, groups, state), g, dt_, device)
    out["C"] = _randn((batch, groups, state), g, dt_, device)
    out["state"] = _randn((batch, heads, state, head_dim), g, torch.float32, device, 0.1)
    return out


def m1_step_inputs(batch, channels, state, groups=1, io="bf16", gate=True, seed=0,
                   device="cpu"):
    """One Mamba-1 decode token plus its cached state ~ N(0, 0.1^2)."""
    g = _gen(seed, device)
    dt_ = _dtype(io)
    A_log = torch.log(torch.arange(1, state + 1, dtype=torch.float32, device=device))
    A = (-torch.exp(A_log)).unsqueeze(0).expand(channels, state).contiguous()
    out = {"A": A, "dt_bias": _dt_bias(channels, g, device),
           "D": torch.ones(channels, dtype=torch.float32, device=device)}
    out["x"] = _randn((batch, channels), g, dt_, device)
    out["z"] = _randn((batch, channels), g, dt_, device) if gate else None
    out["dt"] = _randn((batch, channels), g, dt_, device)
    out["B"] = _randn((batch, groups, state), g, dt_, device)
    out["C"] = _randn((batch, groups, state), g, dt_, device)
    out["state"] = _randn((batch, channels, state), g, torch.float32, device, 0.1)
    return out


def conv_inputs(batch, seqlen, channels, width=4, io="bf16", seed=0, state=False,
                device="cpu"):
    """Inputs of one causal convolution: dict of tensors on ``device``."""
    g = _gen(seed, device)
    bound = 1.0 / math.sqrt(width)
    out = {"w": (torch.rand((channels, width), generator=g, dtype=torch.float32, device=device)
                 * 2 - 1) * bound,
           "bias": (torch.rand(channels, generator=g, dtype=torch.float32, device=device)
                    * 2 - 1) * bound}
    out["x"] = _randn((batch, seqlen, channels), g, _dtype(io), device)
    out["state"] = (_randn((batch, channels, width - 1), g, torch.float32, device)
                    if state else None)
    return out


def ssd_conv_inputs(batch, seqlen, heads, head_dim, state, groups=1, io="bf16", gate=False,
                    seed=0, h0=False, state_in=False, bias=True, device="cpu"):
    """Inputs of one Mamba-2 mixer prologue + SSD: the SSD's own inputs (dt,
    z, A, D, dt_bias, h0, drawn as ssd_inputs draws them) with x, B and C
    replaced by xBC [b, L, heads*head_dim + 2*groups*state] before the
    convolution, the width-4 kernel and bias (U(-1/2, 1/2): the Conv1d
    default bound for 4 taps) and, optionally, a conv state holding earlier
    inputs (values of the I/O type, as a previous call leaves them)."""
    out = ssd_inputs(batch, seqlen, heads, head_dim, state, groups, io, gate, seed, h0,
                     device)
    for k in ("x", "B", "C"):
        del out[k]
    g = _gen(seed + 7, device)
    ctot = heads * head_dim + 2 * groups * state
    out["xBC"] = _randn((batch, seqlen, ctot), g, _dtype(io), device)
    out["conv_w"] = torch.rand((ctot, 4), generator=g, dtype=torch.float32, device=device) - 0.5
    cb = torch.rand((ctot,), generator=g, dtype=torch.float32, device=device) - 0.5
    out["conv_bias"] = cb if bias else None
    out["conv_state"] = (_randn((batch, ctot, 3), g, _dtype(io), device).float()
                         if state_in else None)
    return out


def gnorm_inputs(batch, seqlen, width, io="bf16", seed=0, gate=True, weight=True,
                 device="cpu"):
    """Inputs of one gated norm: y, z [b, L, width], weight [width]."""
    g = _gen(seed, device)
    out = {"weight": (1.0 + 0.1 * torch.randn(width, generator=g, dtype=torch.float32,
                                              device=device)) if weight else None}
    out["y"] = _randn((batch, seqlen, width), g, _dtype(io), device)
    out["z"] = _randn((batch, seqlen, width), g, _dtype(io), device) if gate else None
    return out


def workload_inputs(w: Workload, device="cpu", seed: Optional[int] = None):
    """Inputs of a scan workload (Mamba-1 or SSD)."""
    s = w.seed if seed is None else seed
    if w.kind == "m1":
        return m1_inputs(w.batch, w.seqlen, w.channels, w.state, w.groups, w.io,
                         w.gate, s, device=device)
    if w.kind in ("ssd", "attn"):
        return ssd_inputs(w.batch, w.seqlen, w.heads, w.head_dim, w.state, w.groups,
                          w.io, w.gate, s, device=device)
    if w.kind == "gnorm":
        return gnorm_inputs(w.batch, w.seqlen, w.channels, w.io, s, gate=w.gate, device=device)
    if w.kind == "ssd_conv":
        return ssd_conv_inputs(w.batch, w.seqlen, w.heads, w.head_dim, w.state, w.groups,
                               w.io, w.gate, s, state_in=w.extra.get("state", False),
                               device=device)
    if w.kind == "conv":
        return conv_inputs(w.batch, w.seqlen, w.channels, w.extra.get("width", 4), w.io, s,
                           state=w.extra.get("state", False), device=device)
    raise ValueError("no scan inputs for kind %r" % w.kind)
