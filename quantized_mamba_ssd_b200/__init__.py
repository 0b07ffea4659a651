"""B200-native int8 Mamba-2 SSD chunk scan and decode state update.

The compute path is the C-ABI library ``libssd_i8.so`` (hand-written sm_100a CUDA, built by
``quantized_mamba_ssd_b200.build``); :mod:`quantized_mamba_ssd_b200.ssd_i8` marshals torch
tensors into its calls.  The library is loaded on first use, and a missing library is an
error: there is no fallback path.
"""
__all__ = ["ssd_i8", "workloads"]
