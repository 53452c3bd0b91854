"""Selective state-space scan for NVIDIA B200 (sm_100a).

The product is ``libssm.so``, a C-ABI CUDA library (``include/ssm.h``) with
six calls: ``ssm_scan_fwd`` (Mamba-1 selective scan), ``ssd_chunk_scan_fwd``
(Mamba-2 SSD chunk scan), ``ssm_scan_step`` (one decode token),
``ssm_conv1d_fwd`` (the mixers' causal convolution + silu) and
``ssm_gated_rmsnorm_fwd`` (the Mamba-2 mixer's gated norm) and
``ssd_attention_fwd`` (the SSD map's hidden attention matrix).  The
functions of the same names in ``selective_state_space_28_b200.ops`` are a
thin binding over it; PyTorch supplies device memory and streams only.

Import the binding lazily so that the input generators (``.inputs``) can be
used without a GPU.
"""

__all__ = ["ssm_scan_fwd", "ssm_scan_fwd_write", "ssd_chunk_scan_fwd", "ssm_scan_step", "ssm_conv1d_fwd",
           "ssm_gated_rmsnorm_fwd", "ssd_attention_fwd", "SOFTPLUS", "RMS_BC", "RMS_DT"]


def __getattr__(name):
    if name in __all__:
        from . import ops
        return getattr(ops, name)
    raise AttributeError(name)
