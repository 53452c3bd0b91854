#!/usr/bin/env python
"""Benchmark of the selective state-space scan on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  The headline workload is one Mamba-130m-shaped
mixer scan (ssm_scan_fwd: batch 8, seq 2048, 1536 channels, state 16, bf16
I/O, fp32 state, silu(z) gate); a step is one call over one batch.  ``value``
is algorithmic GB/s over all ranks (inputs read once, outputs written once),
timed with CUDA events over exactly K steps with inputs rotated over enough
buffer sets to exceed L2.  Beside it, under ``workloads``, the same
measurement for the Mamba-2 2.7B-shaped SSD chunk scan (tokens/s and tensor
FLOP rate), the 2.7B decode stack (64 + 24 layer steps, GB/s) and the
Falcon-width scan with its RMS norms (GB/s).

With N > 1 (launched by torchrun) every rank runs its own independent batch
(weak scaling, no collective on the data path); time is the max over ranks.

``--impl reference`` times the float64 CPU oracle on the host cores instead,
on bounded samples of the same workload (one batch row per step).
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE = "m1_130m_b8_l2048_c1536_n16_bf16"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true",
                    help="measure only the headline workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["m1", "m1_write", "m1_b1", "ssd", "ssd_conv", "decode",
                                       "decode_layer",
                                       "falcon", "falcon_b1", "conv", "gnorm", "attn"],
                    help="run just one workload's timed loop (for profiling); prints its timing")
    return ap.parse_args(argv)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


# ------------------------------------------------------------------ bytes/flops

def _esz(io):
    return 2 if io == "bf16" else 4


def m1_bytes(w):
    e = _esz(w.io)
    tc = w.batch * w.seqlen * w.channels
    n = (3 + (1 if w.gate else 0)) * tc * e            # x, dt, y (+ z)
    n += 2 * w.batch * w.seqlen * w.groups * w.state * e  # B, C
    n += w.channels * w.state * 4 + 2 * w.channels * 4    # A, D, dt_bias
    n += w.batch * w.channels * w.state * 4               # h_last
    return n


def m1_sfu_roofline(w, launch_ms, clocks):
    """The Mamba-1 scan's arithmetic floor on the special-function unit.
    Per (token, channel) it evaluates N decays exp(d A), the softplus (ex2,
    lg2) and, with a gate, one tanh; the unit's nominal rate is 16 results
    per clock per SM, 148 SMs, at the SM clock sampled under load."""
    ops = w.batch * w.seqlen * w.channels * (w.state + 2 + (1 if w.gate else 0))
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    peak = 148 * 16 * mhz * 1e6
    ach = ops / (launch_ms * 1e-3)
    return {"ops_per_launch": ops, "achieved_gops": round(ach / 1e9, 1),
            "peak_gops": round(peak / 1e9, 1), "frac": round(ach / peak, 4),
            "peak_source": "nominal 16/clk/SM x 148 SMs x sampled SM clock"}


def ssd_bytes(w):
    e = _esz(w.io)
    n = 2 * w.batch * w.seqlen * w.heads * w.head_dim * e  # x, y
    if w.gate:
        n += w.batch * w.seqlen * w.heads * w.head_dim * e
    n += w.batch * w.seqlen * w.heads * e                  # dt
    n += 2 * w.batch * w.seqlen * w.groups * w.state * e   # B, C
    n += w.batch * w.heads * w.state * w.head_dim * 4      # h_last
    n += 3 * w.heads * 4
    return n


def ssd_conv_bytes(w):
    """The fused mixer prologue + SSD: xBC read once (x, B, C before the
    convolution), dt (and z) read, y written, the float32 conv weights, bias
    and carried conv state (read and written), h_last, A, D, dt_bias."""
    e = _esz(w.io)
    ctot = w.heads * w.head_dim + 2 * w.groups * w.state
    n = w.batch * w.seqlen * ctot * e                      # xBC
    n += w.batch * w.seqlen * w.heads * w.head_dim * e     # y
    if w.gate:
        n += w.batch * w.seqlen * w.heads * w.head_dim * e
    n += w.batch * w.seqlen * w.heads * e                  # dt
    n += 5 * ctot * 4                                      # conv weights, bias
    if w.extra.get("state", False):
        n += 2 * w.batch * ctot * 3 * 4
    n += w.batch * w.heads * w.state * w.head_dim * 4      # h_last
    n += 3 * w.heads * 4
    return n


def ssd_flops(w):
    """Algorithmic FLOPs of the chunked form with chunk Q, causal half counted:
    C.B^T per (chunk, group) 2Q^2N; masked product per (chunk, head) Q(Q+1)P;
    chunk state and state-to-output 2QNP each."""
    Q = w.chunk
    nch = w.batch * ((w.seqlen + Q - 1) // Q)
    cb = nch * w.groups * 2 * Q * Q * w.state
    per_head = Q * (Q + 1) * w.head_dim + 2 * (2 * Q * w.state * w.head_dim)
    return cb + nch * w.heads * per_head


def conv_bytes(w):
    """x read and u written once in the I/O type, the float32 weights and
    bias, and the carried conv state read and written."""
    e = _esz(w.io)
    W = w.extra.get("width", 4)
    n = 2 * w.batch * w.seqlen * w.channels * e + (W + 1) * w.channels * 4
    if w.extra.get("state", False):
        n += 2 * w.batch * w.channels * (W - 1) * 4
    return n


def gnorm_bytes(w):
    """y and z read and out written once in the I/O type, and the weight."""
    e = _esz(w.io)
    rows = w.batch * w.seqlen
    return (3 if w.gate else 2) * rows * w.channels * e + w.channels * 4


def attn_bytes(w):
    """alpha [b, H, L, L] float32 written once (every entry), plus dt, B, C
    and the per-head parameters read."""
    e = _esz(w.io)
    return (4 * w.batch * w.heads * w.seqlen * w.seqlen + w.batch * w.seqlen * w.heads * e
            + 2 * w.batch * w.seqlen * w.groups * w.state * e + 2 * w.heads * 4)


def decode_bytes(w):
    e = _esz(w.io)
    m2 = 2 * w.batch * w.heads * w.state * w.head_dim * 4 \
        + 2 * w.batch * w.heads * w.head_dim * e + w.batch * w.heads * e \
        + 2 * w.batch * w.groups * w.state * e + 3 * w.heads * 4
    m1 = 2 * w.batch * w.m1_channels * w.m1_state * 4 + 4 * w.batch * w.m1_channels * e \
        + 2 * w.batch * w.groups * w.m1_state * e + (w.m1_state + 2) * w.m1_channels * 4
    return m2 * w.layers + m1 * w.m1_layers, m2, m1


# ------------------------------------------------------------------ clocks

class ClockSampler(threading.Thread):
    """Samples SM clock and throttle reasons with NVML every 50 ms."""

    def __init__(self, index):
        super().__init__(daemon=True)
        self.index = index
        self.samples = []
        self.stop_ev = threading.Event()
        self.ok = False
        self.max_mhz = None

    def run(self):
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            self.ok = True
            while not self.stop_ev.is_set():
                mhz = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                reasons = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                util = N.nvmlDeviceGetUtilizationRates(h).gpu
                self.samples.append((mhz, reasons, util))
                time.sleep(0.05)
        except Exception as exc:  # NVML missing: report no clocks
            self.err = repr(exc)

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": "nvml unavailable"}
        names = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                 0x100: "display_clock_setting"}
        loaded = [s for s in self.samples if s[2] > 0] or self.samples
        rs = set()
        for _, r, _ in loaded:
            for bit, n in names.items():
                if r & bit and n != "gpu_idle":
                    rs.add(n)
        return {"sm_mhz": statistics.median(s[0] for s in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(rs), "samples": len(loaded)}


# ------------------------------------------------------------------ helpers

def traffic_for(kernel_key):
    """dram read+write bytes per launch from the committed ncu summary, or None
    if the kernel's source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel_key)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != d["source_sha256"]:
            return None
    return d["bytes_per_launch"]


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v, device):
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def rank_seed(seed, rank):
    """Seed of one rank's batch: every rank scans its own independent batch of
    the same shape (weak scaling, nothing exchanged on the data path)."""
    return seed + 7919 * rank


def job_value(units_per_rank, world, ms_per_step):
    """Whole-job throughput: the units every rank processed in one step, over
    the slowest rank's step time (ms), per second."""
    return units_per_rank * world / (ms_per_step * 1e-3)


def timed(step, K, W, dist, device):
    """W untimed steps, then exactly K steps between two events, with a barrier
    and a device synchronize on both sides.  Returns max-over-ranks ms."""
    import torch
    for i in range(W):
        step(i)
    torch.cuda.synchronize(device)
    dist.barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(K):
        step(W + i)
    e.record()
    torch.cuda.synchronize(device)
    dist.barrier()
    return dist.max(s.elapsed_time(e), device)


def per_launch_ms(step, n, device):
    """Average device time of one step: n steps queued back to back between
    one event pair (the host enqueues faster than the GPU drains them)."""
    import torch
    step(0)
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(n):
        step(i)
    b.record()
    torch.cuda.synchronize(device)
    return a.elapsed_time(b) / n


def n_sets(bytes_per_set):
    return max(2, -(-3 * L2_BYTES // max(1, bytes_per_set)))


# ------------------------------------------------------------------ ours

def bench_m1(w, K, W, dist, device, pk, seed_base, write_at=None):
    """The Mamba-1 scan; with write_at = t, the same scan with the state
    written at token t (ssm_scan_fwd_write; the written state adds its bytes)."""
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    nb = m1_bytes(w) + (w.batch * w.channels * w.state * 4 if write_at is not None else 0)
    sets = []
    for r in range(n_sets(nb)):
        d = I.workload_inputs(w, device=device, seed=seed_base + 1000 * r)
        d["y"] = torch.empty_like(d["x"])
        d["h_last"] = torch.empty((w.batch, w.channels, w.state), device=device)
        if write_at is not None:
            d["s_write"] = torch.zeros((w.batch, w.channels, w.state), device=device)
        d["ws"] = torch.zeros(m1_workspace_bytes(w), dtype=torch.uint8, device=device)
        sets.append(d)

    def step(i):
        d = sets[i % len(sets)]
        if write_at is not None:
            ops.ssm_scan_fwd_write(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                                   dt_bias=d["dt_bias"], flags=w.flags, rms_eps=w.rms_eps,
                                   y=d["y"], h_last=d["h_last"], t=write_at,
                                   state=d["s_write"])
            return
        ops.ssm_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                         dt_bias=d["dt_bias"], flags=w.flags, rms_eps=w.rms_eps,
                         y=d["y"], h_last=d["h_last"], workspace=d["ws"])
    ms = timed(step, K, W, dist, device) / K
    launch_ms = per_launch_ms(step, max(10, K), device)
    ops._check_status(sets[0]["ws"], torch.cuda.current_stream(device).cuda_stream, "bench")
    nseg = m1_segments(w) if write_at is None else 1
    launches = (2 if (w.flags & I.RMS_DT) else 1) + (2 if nseg > 1 else 0)
    return {"ms_per_step": ms, "bytes": nb, "launch_ms": launch_ms, "sets": len(sets),
            "launches_per_step": launches, "segments": nseg}


def m1_workspace_bytes(w):
    """ssm_scan_workspace for the workload, on the current device."""
    import ctypes
    from selective_state_space_28_b200 import _lib as L
    a = L.ScanArgs(batch=w.batch, seqlen=w.seqlen, channels=w.channels, state=w.state,
                   groups=w.groups, io=L.SSM_BF16 if w.io == "bf16" else L.SSM_F32,
                   flags=w.flags, rms_eps=w.rms_eps)
    n = ctypes.c_size_t(0)
    L.check(L.lib().ssm_scan_workspace(ctypes.byref(a), ctypes.byref(n)), "ssm_scan_workspace")
    return n.value


def m1_segments(w):
    """Sequence segments the scan cuts the workload into: read back from the
    workspace size (status word, step-norm factors, then the segments'
    (S - 1) end states, (S - 1) step sums and S entering states)."""
    r256 = lambda v: (v + 255) // 256 * 256
    base = 256 + (r256(w.batch * w.seqlen * 4) if w.flags & 4 else 0)
    extra = m1_workspace_bytes(w) - base
    if extra <= 0:
        return 1
    bcn, bc = w.batch * w.channels * w.state * 4, w.batch * w.channels * 4
    for S in range(2, 65):
        if r256(bcn * (S - 1)) + r256(bc * (S - 1)) + r256(bcn * S) == extra:
            return S
    return -1


def bench_m1_static(w, K, W, dist, device, seed_base):
    """The same scan through ssm_scan_fwd_static, which never cuts the
    sequence: the uncut time beside a cut call's."""
    import ctypes
    import torch
    from selective_state_space_28_b200 import _lib as L
    from selective_state_space_28_b200 import inputs as I
    nb = m1_bytes(w)
    sets = []
    for r in range(n_sets(nb)):
        d = I.workload_inputs(w, device=device, seed=seed_base + 1000 * r)
        d["y"] = torch.empty_like(d["x"])
        d["h_last"] = torch.empty((w.batch, w.channels, w.state), device=device)
        sets.append(d)
    st = torch.cuda.current_stream(device).cuda_stream

    def step(i):
        d = sets[i % len(sets)]
        a = L.ScanArgs(batch=w.batch, seqlen=w.seqlen, channels=w.channels, state=w.state,
                       groups=w.groups, io=L.SSM_BF16 if w.io == "bf16" else L.SSM_F32,
                       flags=w.flags, rms_eps=w.rms_eps, x=d["x"].data_ptr(),
                       dt=d["dt"].data_ptr(), z=d["z"].data_ptr() if d["z"] is not None else None,
                       B=d["B"].data_ptr(), C=d["C"].data_ptr(), A=d["A"].data_ptr(),
                       D=d["D"].data_ptr(), dt_bias=d["dt_bias"].data_ptr(),
                       y=d["y"].data_ptr(), h_last=d["h_last"].data_ptr())
        L.check(L.lib().ssm_scan_fwd_static(ctypes.byref(a), st), "ssm_scan_fwd_static")
    ms = timed(step, K, W, dist, device) / K
    launch_ms = per_launch_ms(step, max(10, K), device)
    return {"ms_per_step": ms, "bytes": nb, "launch_ms": launch_ms}


def bench_conv(w, K, W, dist, device, pk, seed_base):
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    nb = conv_bytes(w)
    sets = []
    for r in range(n_sets(nb)):
        d = I.workload_inputs(w, device=device, seed=seed_base + 1000 * r)
        d["u"] = torch.empty_like(d["x"])
        d["state_out"] = torch.empty((w.batch, w.channels, w.extra.get("width", 4) - 1),
                                     device=device)
        sets.append(d)

    def step(i):
        d = sets[i % len(sets)]
        ops.ssm_conv1d_fwd(d["x"], d["w"], d["bias"], d["state"], silu=True, u=d["u"],
                           state_out=d["state_out"])
    ms = timed(step, K, W, dist, device) / K
    launch_ms = per_launch_ms(step, max(10, K), device)
    return {"ms_per_step": ms, "bytes": nb, "launch_ms": launch_ms, "sets": len(sets),
            "launches_per_step": 1}


def bench_gnorm(w, K, W, dist, device, pk, seed_base):
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    nb = gnorm_bytes(w)
    sets = []
    for r in range(n_sets(nb)):
        d = I.workload_inputs(w, device=device, seed=seed_base + 1000 * r)
        d["out"] = torch.empty_like(d["y"])
        sets.append(d)

    def step(i):
        d = sets[i % len(sets)]
        ops.ssm_gated_rmsnorm_fwd(d["y"], d["z"], d["weight"], w.rms_eps, out=d["out"])
    ms = timed(step, K, W, dist, device) / K
    launch_ms = per_launch_ms(step, max(10, K), device)
    return {"ms_per_step": ms, "bytes": nb, "launch_ms": launch_ms, "sets": len(sets),
            "launches_per_step": 1}


def bench_attn(w, K, W, dist, device, pk, seed_base):
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    nb = attn_bytes(w)
    sets = []
    for r in range(n_sets(nb)):
        d = I.workload_inputs(w, device=device, seed=seed_base + 1000 * r)
        d["alpha"] = torch.empty((w.batch, w.heads, w.seqlen, w.seqlen), device=device)
        sets.append(d)

    def step(i):
        d = sets[i % len(sets)]
        ops.ssd_attention_fwd(d["dt"], d["A"], d["B"], d["C"], d["dt_bias"], alpha=d["alpha"])
    ms = timed(step, K, W, dist, device) / K
    launch_ms = per_launch_ms(step, max(10, K), device)
    return {"ms_per_step": ms, "bytes": nb, "launch_ms": launch_ms, "sets": len(sets),
            "launches_per_step": 2}  # C . B^T with the pre-pass, the mask pass


def bench_ssd(w, K, W, dist, device, pk, seed_base):
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    nb = ssd_bytes(w)
    sets = []
    for r in range(n_sets(nb)):
        d = I.workload_inputs(w, device=device, seed=seed_base + 1000 * r)
        d["y"] = torch.empty_like(d["x"])
        d["h_last"] = torch.empty((w.batch, w.heads, w.state, w.head_dim), device=device)
        sets.append(d)
    ws = ops.ssd_workspace_bytes(batch=w.batch, seqlen=w.seqlen, heads=w.heads,
                                 head_dim=w.head_dim, state=w.state, groups=w.groups,
                                 chunk=w.chunk, io=1 if w.io == "bf16" else 0, flags=w.flags)
    wsb = torch.empty(max(ws, 1), dtype=torch.uint8, device=device)

    def step(i):
        d = sets[i % len(sets)]
        ops.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                               dt_bias=d["dt_bias"], chunk=w.chunk, flags=w.flags,
                               y=d["y"], h_last=d["h_last"], workspace=wsb)
    ms = timed(step, K, W, dist, device) / K
    launch_ms = per_launch_ms(step, max(5, K), device)
    # a workspace beyond the status word means the last wave is cut into
    # sequence segments: two SSD launches and the carry between them
    launches = 3 if ws > 256 else 1
    return {"ms_per_step": ms, "bytes": nb, "flops": ssd_flops(w), "launch_ms": launch_ms,
            "tokens": w.batch * w.seqlen, "sets": len(sets), "launches_per_step": launches}


def bench_ssd_conv(w, K, W, dist, device, pk, seed_base):
    """The SSD with the mixer's convolution fused in front
    (ssd_conv_chunk_scan_fwd): xBC before the convolution in, y out."""
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    nb = ssd_conv_bytes(w)
    ctot = w.heads * w.head_dim + 2 * w.groups * w.state
    sets = []
    for r in range(n_sets(nb)):
        d = I.workload_inputs(w, device=device, seed=seed_base + 1000 * r)
        d["y"] = torch.empty((w.batch, w.seqlen, w.heads, w.head_dim), dtype=d["xBC"].dtype,
                             device=device)
        d["h_last"] = torch.empty((w.batch, w.heads, w.state, w.head_dim), device=device)
        d["cs_out"] = torch.empty((w.batch, ctot, 3), device=device)
        sets.append(d)
    ws = ops.ssd_conv_workspace_bytes(batch=w.batch, seqlen=w.seqlen, heads=w.heads,
                                      head_dim=w.head_dim, state=w.state, groups=w.groups,
                                      chunk=w.chunk, io=1 if w.io == "bf16" else 0,
                                      flags=w.flags)
    wsb = torch.empty(max(ws, 1), dtype=torch.uint8, device=device)

    def step(i):
        d = sets[i % len(sets)]
        ops.ssd_conv_chunk_scan_fwd(d["xBC"], d["conv_w"], d["dt"], d["A"], heads=w.heads,
                                    state=w.state, groups=w.groups, conv_bias=d["conv_bias"],
                                    conv_state_in=d["conv_state"], D=d["D"], z=d["z"],
                                    dt_bias=d["dt_bias"], chunk=w.chunk, flags=w.flags,
                                    y=d["y"], h_last=d["h_last"], conv_state_out=d["cs_out"],
                                    workspace=wsb)
    ms = timed(step, K, W, dist, device) / K
    launch_ms = per_launch_ms(step, max(5, K), device)
    ops._check_status(wsb, torch.cuda.current_stream(device).cuda_stream, "bench")
    # the B/C pre-pass, then one SSD launch, or three when the last wave is cut
    split = ws - 256 - ((w.batch * w.seqlen * 2 * w.groups * w.state * 2 + 255) // 256 * 256)
    launches = 1 + (3 if split > 0 else 1)
    return {"ms_per_step": ms, "bytes": nb, "flops": ssd_flops(w), "launch_ms": launch_ms,
            "tokens": w.batch * w.seqlen, "sets": len(sets), "launches_per_step": launches}


def bench_decode(w, K, W, dist, device, pk, seed_base):
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    total, m2b, m1b = decode_bytes(w)
    m2_layers, m1_layers = [], []
    for l in range(w.layers):
        m2_layers.append(I.m2_step_inputs(w.batch, w.heads, w.head_dim, w.state, w.groups,
                                          w.io, w.gate, seed=seed_base + l, device=device))
        m2_layers[-1]["y"] = torch.empty_like(m2_layers[-1]["x"])
    for l in range(w.m1_layers):
        m1_layers.append(I.m1_step_inputs(w.batch, w.m1_channels, w.m1_state, w.groups,
                                          w.io, True, seed=seed_base + 500 + l, device=device))
        m1_layers[-1]["y"] = torch.empty_like(m1_layers[-1]["x"])

    def one(d):
        ops.ssm_scan_step(d["state"], d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                          z=d["z"], dt_bias=d["dt_bias"], y=d["y"])

    def step(i):
        for d in m2_layers:
            one(d)
        for d in m1_layers:
            one(d)
    ms = timed(step, K, W, dist, device) / K
    m2_ms = per_launch_ms(lambda i: one(m2_layers[i % len(m2_layers)]), 2 * len(m2_layers),
                          device)
    return {"ms_per_step": ms, "bytes": total, "launch_ms": m2_ms, "launch_bytes": m2b,
            "launches_per_step": w.layers + w.m1_layers}


def e2e_m1(w, device, n_steps=5):
    """The same metric through the public API with pinned HOST buffers: each
    step copies its inputs host->device, scans, and reads y and h_last back
    (ssm_scan_fwd_host: batch-row chunks, the two directions' copies
    overlapped with each other and with the scans)."""
    import torch
    from selective_state_space_28_b200 import inputs as I
    from selective_state_space_28_b200 import ops
    d = I.workload_inputs(w, device="cpu")
    d = {k: (v.pin_memory() if v is not None else None) for k, v in d.items()}
    h2d = sum(v.numel() * v.element_size() for v in d.values() if v is not None)
    d2h = d["x"].numel() * d["x"].element_size() + w.batch * w.channels * w.state * 4

    def step():
        y, h, _ = ops.ssm_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                                   z=d["z"], dt_bias=d["dt_bias"], flags=w.flags,
                                   rms_eps=w.rms_eps)
        return y, h
    step()
    torch.cuda.synchronize(device)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(n_steps):
        step()
    e.record()
    torch.cuda.synchronize(device)
    ms = s.elapsed_time(e) / n_steps
    return {"ms": ms, "h2d": h2d, "d2h": d2h}


# ------------------------------------------------------------------ CPU baselines

def _time_oracle(fn, threads, min_seconds):
    """Passes of fn(threads) until about min_seconds; returns (passes, seconds)."""
    passes, sec = 0, 0.0
    while sec < min_seconds and passes < 200:
        t0 = time.perf_counter()
        fn(threads)
        sec += time.perf_counter() - t0
        passes += 1
    return passes, sec


def _cpu_entry(unit_per_pass, unit, fn, sample, min_seconds):
    """The oracle on all the host cores this process may use, and on one."""
    import oracle
    threads = oracle.default_threads()
    fn(threads)  # page in, build
    n_all, s_all = _time_oracle(fn, threads, min_seconds)
    n_one, s_one = _time_oracle(fn, 1, min_seconds)
    try:
        hw = os.cpu_count()
    except Exception:  # pragma: no cover
        hw = None
    return {"value": unit_per_pass * n_all / s_all, "unit": unit, "cores": threads,
            "value_1core": unit_per_pass * n_one / s_one, "cores_hw": hw,
            "affinity_cores": threads, "kind": "oracle",
            "sample": "%s; %d pass(es) in %.1f s on %d cores, %d in %.1f s on 1 core"
                      % (sample, n_all, s_all, threads, n_one, s_one)}


def cpu_baseline_m1(w, min_seconds=4.0, rows=1, tokens=None):
    """The float64 oracle, as it stands, on a bounded sample of a Mamba-1
    workload: `rows` batch rows and the first `tokens` tokens (all channels,
    so that the step norm over the channels is the workload's)."""
    import oracle
    from selective_state_space_28_b200 import inputs as I
    L = tokens or w.seqlen
    d = I.m1_inputs(rows, L, w.channels, w.state, w.groups, w.io, w.gate, w.seed)
    ws = I.Workload(w.name, "m1", batch=rows, seqlen=L, channels=w.channels, state=w.state,
                    groups=w.groups, io=w.io, gate=w.gate, flags=w.flags)
    nb = m1_bytes(ws)

    def fn(threads):
        oracle.m1_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                       dt_bias=d["dt_bias"], flags=w.flags, rms_eps=w.rms_eps,
                       want_states=w.want_states, nthreads=threads)
    r = _cpu_entry(nb / 1e9, "GB/s", fn, "%d batch row(s) x %d tokens x %d channels x state %d "
                   "of %s, float64 C token loop" % (rows, L, w.channels, w.state, w.name),
                   min_seconds)
    return r


def cpu_baseline_ssd(w, min_seconds=4.0, heads=4):
    """The oracle's Mamba-2 token loop on one batch row and `heads` of the
    workload's heads (heads are independent given B and C); tokens/s scaled
    to the whole head count."""
    import oracle
    from selective_state_space_28_b200 import inputs as I
    d = I.ssd_inputs(1, w.seqlen, heads, w.head_dim, w.state, w.groups, w.io, w.gate, w.seed)

    def fn(threads):
        oracle.m2_scan(d["x"], d["dt"], d["B"], d["C"], d["A"], d["D"], z=d["z"],
                       dt_bias=d["dt_bias"], nthreads=threads)
    return _cpu_entry(w.seqlen * heads / w.heads, "tokens/s", fn,
                      "1 batch row x %d of %d heads x %d tokens of %s (tokens/s scaled by the "
                      "head fraction), float64 C token loop" % (heads, w.heads, w.seqlen, w.name),
                      min_seconds)


def cpu_baseline_decode(w, min_seconds=4.0, rows=16):
    """The oracle's decode step on `rows` batch rows of one Mamba-2 layer and
    one Mamba-1 layer (the stack runs layer by layer; every layer is the
    same shape), GB/s of state read-modify-write plus the token."""
    import oracle
    from selective_state_space_28_b200 import inputs as I
    e = I.m2_step_inputs(rows, w.heads, w.head_dim, w.state, w.groups, w.io, seed=w.seed)
    f = I.m1_step_inputs(rows, w.m1_channels, w.m1_state, 1, w.io, gate=True, seed=w.seed + 1)
    _, m2b, m1b = decode_bytes(w)
    nb = (m2b + m1b) * rows / w.batch

    def fn(threads):
        oracle.m2_step(e["state"], e["x"], e["dt"], e["B"], e["C"], e["A"], e["D"],
                       dt_bias=e["dt_bias"])
        oracle.m1_step(f["state"], f["x"], f["dt"], f["B"], f["C"], f["A"], f["D"], z=f["z"],
                       dt_bias=f["dt_bias"])
    return _cpu_entry(nb / 1e9, "GB/s", fn, "%d of %d batch rows of one Mamba-2 layer and one "
                      "Mamba-1 layer of %s, float64 C loop (single-threaded by construction)"
                      % (rows, w.batch, w.name), min_seconds)


def cpu_baselines(min_seconds=3.0):
    """Oracle timings for every configuration, keyed by workload name."""
    from selective_state_space_28_b200 import inputs as I
    W = I.WORKLOADS
    out = {}
    out["m1_toy_b1_l64_c32_n4_f32"] = cpu_baseline_m1(W["m1_toy_b1_l64_c32_n4_f32"], min_seconds)
    out[HEADLINE] = cpu_baseline_m1(W[HEADLINE], min_seconds, rows=1)
    wf = W["m1_falcon_rms_b4_l8192_c8192_n16_bf16"]
    out[wf.name] = cpu_baseline_m1(wf, min_seconds, rows=1, tokens=512)
    ws = W["ssd_2p7b_b4_l4096_h80_p64_n128_bf16"]
    out[ws.name] = cpu_baseline_ssd(ws, min_seconds)
    wd = W["decode_2p7b_stack_b256"]
    out[wd.name] = cpu_baseline_decode(wd, min_seconds)
    return out


def run_only(args):
    """One workload's warm-up and timed loop, nothing else (used under ncu)."""
    import torch
    from selective_state_space_28_b200 import build as B
    from selective_state_space_28_b200 import inputs as I
    B.build()
    dist = Dist()
    torch.cuda.set_device(dist.local)
    device = torch.device("cuda", dist.local)
    pk = peaks()
    name = {"m1": HEADLINE, "m1_write": HEADLINE, "m1_b1": "m1_130m_b1_l2048_c1536_n16_bf16",
            "falcon_b1": "m1_falcon_rms_b1_l8192_c8192_n16_bf16",
            "ssd": "ssd_2p7b_b4_l4096_h80_p64_n128_bf16",
            "ssd_conv": "ssd_conv_2p7b_b4_l4096_h80_p64_n128_bf16",
            "decode": "decode_2p7b_stack_b256", "decode_layer": "decode_2p7b_layer_b256",
            "falcon": "m1_falcon_rms_b4_l8192_c8192_n16_bf16",
            "conv": "conv_2p7b_b4_l4096_c5376_bf16",
            "gnorm": "gnorm_2p7b_b4_l4096_w5120_bf16",
            "attn": "attn_2p7b_b1_l1024_h80_n128_bf16"}[args.only]
    w = I.WORKLOADS[name]
    fn = {"m1": bench_m1, "m1_b1": bench_m1, "falcon_b1": bench_m1,
          "m1_write": lambda *a: bench_m1(*a, write_at=w.seqlen // 2),
          "falcon": bench_m1, "ssd": bench_ssd, "ssd_conv": bench_ssd_conv,
          "decode": bench_decode,
          "decode_layer": bench_decode, "conv": bench_conv, "gnorm": bench_gnorm,
          "attn": bench_attn}[args.only]
    r = fn(w, args.steps, args.warmup, dist, device, pk, w.seed)
    print(json.dumps({"only": name, "ms_per_step": r["ms_per_step"],
                      "launch_ms": r["launch_ms"]}), flush=True)


def run_ours(args):
    import torch
    from selective_state_space_28_b200 import build as B
    from selective_state_space_28_b200 import inputs as I
    B.build()
    dist = Dist()
    torch.cuda.set_device(dist.local)
    device = torch.device("cuda", dist.local)
    dist.init("nccl")
    pk = peaks()
    K, W = args.steps, args.warmup
    sampler = ClockSampler(dist.local)
    sampler.start()
    time.sleep(0.2)

    w = I.WORKLOADS[HEADLINE]
    r = bench_m1(w, K, W, dist, device, pk, seed_base=rank_seed(w.seed, dist.rank))
    sampler.stop_ev.set()
    sampler.join(timeout=2)
    clocks = sampler.summary()
    hbm = pk["hbm_gbs"]
    value = job_value(r["bytes"], dist.world, r["ms_per_step"]) / 1e9
    achieved = r["bytes"] / (r["launch_ms"] * 1e-3) / 1e9
    out = {
        "metric": "Mamba-1 selective scan algorithmic HBM throughput (GB/s); "
                  "SSD chunk-scan tokens/s under workloads",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": dist.world, "steps": K,
        "warmup": W, "ms_per_step": round(r["ms_per_step"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) inputs, S4D-real A, softplus^-1 dt_bias)",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen,
                   "channels": w.channels, "state": w.state, "groups": w.groups,
                   "io_dtype": w.io, "state_dtype": "f32", "gate": w.gate,
                   "sequence_segments": r["segments"],
                   "l2": "inputs rotated over %d buffer sets (%.0f MB each) > L2"
                         % (r["sets"], r["bytes"] / 1e6),
                   "parallelism": "dp%d (independent batches per GPU)" % dist.world},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": hbm,
                     "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "traffic": traffic_for("m1_scan_tma_130m"),
                     "peak_source": "%s hbm_gbs (copy)" % pk["_source"],
                     "kernel": "m1_scan_tma_kernel",
                     "sfu": m1_sfu_roofline(w, r["launch_ms"], clocks)},
        "clocks": clocks,
        "gpu_launches": r["launches_per_step"] * K,
    }
    if not args.no_e2e:
        e = e2e_m1(w, device)
        out["e2e"] = {"value": round(r["bytes"] / (e["ms"] * 1e-3) / 1e9, 3), "unit": "GB/s",
                      "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                      "ms_per_step": round(e["ms"], 3)}
    if not args.no_extra:
        wl = {}
        ws = I.WORKLOADS["ssd_2p7b_b4_l4096_h80_p64_n128_bf16"]
        Ke = max(3, min(K, 20))
        s = bench_ssd(ws, Ke, max(3, W), dist, device, pk, rank_seed(ws.seed, dist.rank))
        tf = s["flops"] / (s["launch_ms"] * 1e-3) / 1e12
        wl[ws.name] = {
            "value": round(job_value(s["tokens"], dist.world, s["ms_per_step"]), 1),
            "unit": "tokens/s", "ms_per_step": round(s["ms_per_step"], 4),
            "gpu_launches": s["launches_per_step"] * Ke,
            "gbs": round(s["bytes"] / (s["ms_per_step"] * 1e-3) / 1e9, 1),
            "roofline": {"bound": "tensor", "achieved": round(tf, 2),
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf / pk["bf16_tflops"], 4),
                         "traffic": traffic_for("ssd_2p7b"),
                         "flops_per_launch": s["flops"], "bytes_per_launch": s["bytes"],
                         "hbm_frac": round(s["bytes"] / (s["launch_ms"] * 1e-3) / 1e9 / hbm, 4)}}
        wd = I.WORKLOADS["decode_2p7b_stack_b256"]
        dd = bench_decode(wd, max(3, min(K, 5)), 3, dist, device, pk, rank_seed(wd.seed, dist.rank))
        ach = dd["launch_bytes"] / (dd["launch_ms"] * 1e-3) / 1e9
        wl[wd.name] = {
            "value": round(job_value(dd["bytes"], dist.world, dd["ms_per_step"]) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(dd["ms_per_step"], 4),
            "roofline": {"bound": "hbm", "achieved": round(ach, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4), "traffic": traffic_for("m2_step_2p7b"),
                         "kernel": "mamba-2 layer step"}}
        del dd
        torch.cuda.empty_cache()
        wf = I.WORKLOADS["m1_falcon_rms_b4_l8192_c8192_n16_bf16"]
        f = bench_m1(wf, max(3, min(K, 10)), 3, dist, device, pk, rank_seed(wf.seed, dist.rank))
        ach = f["bytes"] / (f["launch_ms"] * 1e-3) / 1e9
        # The step-norm statistic needs every channel of a token before the
        # scan's first channel block can use it: a pre-pass reads the whole
        # step input once more and writes one factor per token.
        pre = wf.batch * wf.seqlen * (wf.channels * _esz(wf.io) + 4)
        wl[wf.name] = {
            "value": round(job_value(f["bytes"], dist.world, f["ms_per_step"]) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(f["ms_per_step"], 4),
            "roofline": {"bound": "hbm", "achieved": round(ach, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4), "traffic": traffic_for("m1_scan_falcon"),
                         "kernel": "m1_scan_tma_kernel (+ dt_rms_kernel)",
                         "note": "achieved counts the scan's algorithmic bytes over the whole "
                                 "call's time; the pre-pass bytes are listed apart"},
            "prepass": {"kernel": "dt_rms_kernel", "bytes_per_call": pre,
                        "achieved_with_prepass_gbs":
                            round((f["bytes"] + pre) / (f["launch_ms"] * 1e-3) / 1e9, 2)}}
        wc = I.WORKLOADS["conv_2p7b_b4_l4096_c5376_bf16"]
        cv = bench_conv(wc, max(3, min(K, 20)), max(3, W), dist, device, pk,
                        rank_seed(wc.seed, dist.rank))
        ach = cv["bytes"] / (cv["launch_ms"] * 1e-3) / 1e9
        wl[wc.name] = {
            "value": round(job_value(cv["bytes"], dist.world, cv["ms_per_step"]) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(cv["ms_per_step"], 4),
            "roofline": {"bound": "hbm", "achieved": round(ach, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4), "traffic": traffic_for("conv_2p7b"),
                         "kernel": "conv1d_vec_kernel"}}
        # The SSD with the convolution fused in front, beside the unfused pair
        # (the convolution and the SSD lines above, same shapes, this run).
        wsc = I.WORKLOADS["ssd_conv_2p7b_b4_l4096_h80_p64_n128_bf16"]
        sc = bench_ssd_conv(wsc, Ke, max(3, W), dist, device, pk, rank_seed(wsc.seed, dist.rank))
        tf = sc["flops"] / (sc["launch_ms"] * 1e-3) / 1e12
        unfused = s["ms_per_step"] + cv["ms_per_step"]
        e = _esz(wsc.io)
        saved = 2 * wsc.batch * wsc.seqlen * wsc.heads * wsc.head_dim * e
        wl[wsc.name] = {
            "value": round(job_value(sc["tokens"], dist.world, sc["ms_per_step"]), 1),
            "unit": "tokens/s", "ms_per_step": round(sc["ms_per_step"], 4),
            "gpu_launches": sc["launches_per_step"] * Ke,
            "unfused_ms_per_step": round(unfused, 4),
            "speedup_vs_unfused": round(unfused / sc["ms_per_step"], 3),
            "bytes_saved_per_call": saved,
            "note": "unfused = the convolution line plus the SSD line; saved = the convolved "
                    "x written and read back (B and C still make one round trip)",
            "roofline": {"bound": "tensor", "achieved": round(tf, 2),
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf / pk["bf16_tflops"], 4),
                         "traffic": traffic_for("ssd_conv_2p7b"),
                         "flops_per_launch": sc["flops"], "bytes_per_launch": sc["bytes"],
                         "hbm_frac": round(sc["bytes"] / (sc["launch_ms"] * 1e-3) / 1e9 / hbm,
                                           4)}}
        w1 = I.WORKLOADS["m1_130m_b1_l2048_c1536_n16_bf16"]
        Kb = max(3, min(K, 20))
        cut = bench_m1(w1, Kb, max(3, W), dist, device, pk, rank_seed(w1.seed, dist.rank))
        whole = bench_m1_static(w1, Kb, max(3, W), dist, device, rank_seed(w1.seed, dist.rank))
        ach = cut["bytes"] / (cut["launch_ms"] * 1e-3) / 1e9
        wl[w1.name] = {
            "value": round(job_value(cut["bytes"], dist.world, cut["ms_per_step"]) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(cut["ms_per_step"], 4),
            "sequence_segments": cut["segments"],
            "uncut_ms_per_step": round(whole["ms_per_step"], 4),
            "speedup_from_segments": round(whole["ms_per_step"] / cut["ms_per_step"], 3),
            "roofline": {"bound": "hbm", "achieved": round(ach, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4),
                         "traffic": traffic_for("m1_scan_tma_130m_b1_segments"),
                         "kernel": "m1_scan_tma_kernel (state-only segments, carry, rescan)",
                         "note": "achieved and traffic are per call, its three launches together"}}
        sw = bench_m1(w, max(3, min(K, 10)), 3, dist, device, pk, rank_seed(w.seed, dist.rank),
                      write_at=w.seqlen // 2)
        ach = sw["bytes"] / (sw["launch_ms"] * 1e-3) / 1e9
        wl[w.name + "_state_write_t%d" % (w.seqlen // 2)] = {
            "value": round(job_value(sw["bytes"], dist.world, sw["ms_per_step"]) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(sw["ms_per_step"], 4),
            "roofline": {"bound": "hbm", "achieved": round(ach, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4),
                         "traffic": traffic_for("m1_scan_tma_130m_write"),
                         "kernel": "m1_scan_tma_kernel (write form)"}}
        wg = I.WORKLOADS["gnorm_2p7b_b4_l4096_w5120_bf16"]
        gn = bench_gnorm(wg, max(3, min(K, 20)), max(3, W), dist, device, pk,
                         rank_seed(wg.seed, dist.rank))
        ach = gn["bytes"] / (gn["launch_ms"] * 1e-3) / 1e9
        wl[wg.name] = {
            "value": round(job_value(gn["bytes"], dist.world, gn["ms_per_step"]) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(gn["ms_per_step"], 4),
            "roofline": {"bound": "hbm", "achieved": round(ach, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4), "traffic": traffic_for("gnorm_2p7b"),
                         "kernel": "gated_norm_kernel"}}
        wa = I.WORKLOADS["attn_2p7b_b1_l1024_h80_n128_bf16"]
        at = bench_attn(wa, max(3, min(K, 20)), max(3, W), dist, device, pk,
                        rank_seed(wa.seed, dist.rank))
        ach = at["bytes"] / (at["launch_ms"] * 1e-3) / 1e9
        wl[wa.name] = {
            "value": round(job_value(at["bytes"], dist.world, at["ms_per_step"]) / 1e9, 2),
            "unit": "GB/s", "ms_per_step": round(at["ms_per_step"], 4),
            "roofline": {"bound": "hbm", "achieved": round(ach, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4), "traffic": traffic_for("attn_2p7b"),
                         "kernel": "attn_mask_kernel (+ attn_prep_kernel, attn_cb_tc_kernel)"}}
        out["workloads"] = wl
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cb = cpu_baselines()
        out["cpu_baseline"] = cb.pop(HEADLINE)
        for name, entry in cb.items():
            out.setdefault("workloads", {}).setdefault(name, {})["cpu_baseline"] = entry
    dist.close()
    if dist.rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ reference

def run_reference(args):
    dist = Dist()
    if dist.rank != 0:
        return
    from selective_state_space_28_b200 import inputs as I
    import oracle
    w = I.WORKLOADS[HEADLINE]
    d = I.workload_inputs(w, device="cpu")
    threads = oracle.default_threads()
    rows = 1

    def step(i):
        r = i % w.batch
        sub = {k: (v[r:r + rows] if (v is not None and k in ("x", "dt", "z", "B", "C")) else v)
               for k, v in d.items()}
        oracle.m1_scan(sub["x"], sub["dt"], sub["B"], sub["C"], sub["A"], sub["D"], z=sub["z"],
                       dt_bias=sub["dt_bias"], flags=w.flags, rms_eps=w.rms_eps,
                       nthreads=threads)
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    sec = (time.perf_counter() - t0) / args.steps
    nb = m1_bytes(w) * rows / w.batch
    value = nb / sec / 1e9
    sample = ("one of %d batch rows of %s per step (all %d tokens x %d channels x state %d), "
              "float64 C token loop" % (w.batch, w.name, w.seqlen, w.channels, w.state))
    out = {"impl": "reference", "metric": "Mamba-1 selective scan algorithmic HBM throughput "
           "(GB/s); SSD chunk-scan tokens/s under workloads", "value": round(value, 4),
           "unit": "GB/s", "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen,
                      "channels": w.channels, "state": w.state, "io_dtype": w.io,
                      "sample_rows_per_step": rows},
           "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    elif a.only:
        run_only(a)
    else:
        run_ours(a)
