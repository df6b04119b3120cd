"""GDLA (Grouped Differential Latent Attention) forward core for NVIDIA B200.

Python binding of the C-ABI library ``libgdla.so`` (hand-written sm_100a CUDA
kernels). PyTorch supplies device memory and streams; the computation happens
only in the library. See ``include/gdla.h`` for the ABI.
"""
from .ops import (DC, DL, DQK, DR, DV, GROUP, GDLAError, attn_bwd, attn_bwd_workspace_bytes, attn_decode,
                  attn_decode_latent, attn_fwd, decode_latent_workspace_bytes, decode_workspace_bytes, device_error,
                  library, prologue, prologue_workspace_bytes)

__all__ = ["attn_fwd", "attn_bwd", "attn_bwd_workspace_bytes", "prologue", "prologue_workspace_bytes", "attn_decode", "attn_decode_latent", "decode_workspace_bytes",
           "decode_latent_workspace_bytes", "device_error", "library", "GDLAError", "GROUP", "DQK", "DV", "DC",
           "DR", "DL"]
