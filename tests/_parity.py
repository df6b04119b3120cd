"""Shared helpers for the GPU parity tests: run the CUDA path and the fp64
oracle on the same seeded inputs and compare element by element.

Tolerance (from the stated acceptance bar for this core): over all checked
elements, max |gpu - ref| <= 2e-2 and ||gpu - ref||_2 / ||ref||_2 <= 5e-3,
the bf16 GPU output widened exactly to double.
"""
import numpy as np
import torch

import differential_latent_attention_b200 as gdla
import gdla_inputs as gi
import oracle

MAX_ABS = 2e-2
REL_RMS = 5e-3


def metrics(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite GPU output"
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, ref, what=""):
    max_abs, rel = metrics(got, ref)
    assert max_abs <= MAX_ABS and rel <= REL_RMS, f"{what}: max_abs={max_abs:.3e} rel_rms={rel:.3e}"
    return max_abs, rel


def host_args(t):
    """Oracle arguments (bf16 bits / fp32 numpy) from prefill input tensors."""
    return [gi.bf16_bits(t["q_sig"]), gi.bf16_bits(t["q_noise"]), gi.bf16_bits(t["k"]), gi.bf16_bits(t["v"]),
            t["lam"].detach().cpu().numpy(), gi.bf16_bits(t["gate"])]


def gpu_prefill(t, seqlens, window, out=None):
    return gdla.attn_fwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], seqlens, window, out=out)


def check_prefill(seqlens, hkv, window, seed, rows=None, t=None, what=""):
    if t is None:
        t = gi.make_prefill_inputs(seqlens, hkv, seed, device="cuda")
    out = gpu_prefill(t, seqlens, window)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    ref = oracle.prefill(*host_args(t), seqlens, window, rows=rows)
    got = out.float().cpu().numpy() if rows is None else out[torch.as_tensor(rows, device=out.device)].float().cpu().numpy()
    return assert_close(got, ref, what or f"prefill seqlens={seqlens} hkv={hkv} window={window}")


def decode_host_args(d):
    return [gi.bf16_bits(d["q_sig"]), gi.bf16_bits(d["q_noise"]), gi.bf16_bits(d["k_cache"]),
            gi.bf16_bits(d["v_cache"]), d["cu_seqlens_k"].detach().cpu().numpy().astype(np.int64),
            d["lam"].detach().cpu().numpy(), gi.bf16_bits(d["gate"])]


def gpu_decode(d, max_len, window, out=None, workspace=None):
    return gdla.attn_decode(d["q_sig"], d["q_noise"], d["k_cache"], d["v_cache"], d["cu_seqlens_k"], max_len,
                            d["lam"], d["gate"], window, out=out, workspace=workspace)
