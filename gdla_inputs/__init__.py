"""Seeded synthetic inputs for the GDLA forward core.

This module is shared by the tests, the bench and the smoke check, and feeds
both the CUDA library and the fp64 oracle. It holds none of the method's
arithmetic: it only draws random tensors of the right shapes, dtypes and
layouts, and describes the workloads.

Distributions (the workload recipe): q_sig, q_noise, k, v and the gate logits
are N(0, 1) drawn in fp32 and rounded to nearest-even bf16 (for the latent-cache
decode likewise the absorbed queries and the cache rows [c | k_rope], and
W^UV ~ N(0, 1/512), so that an up-projected value row has unit scale); lambda is
U(0, 1) strictly inside the interval, (k + 0.5) / 2^24 for a uniform integer
k in [0, 2^24), stored as fp32 (exact); decode KV lengths are integers drawn
uniformly from [lo, hi] inclusive.

All draws come from one ``torch.Generator`` seeded per workload, on the device
the tensors are created on. The same seed on CPU and on CUDA gives different
values; a parity test draws once and hands the same tensors to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

GROUP = 4
DQK = 192
DV = 128
LAMBDA_BITS = 24


@dataclass(frozen=True)
class PrefillWorkload:
    """A packed varlen prefill problem: sequence lengths, KV heads, window, seed."""
    name: str
    seqlens: tuple
    num_kv_heads: int
    window: int
    seed: int

    @property
    def tokens(self) -> int:
        return int(sum(self.seqlens))

    def visible_pairs(self) -> int:
        """Number of visible (query, key) pairs per query head."""
        total = 0
        for length in self.seqlens:
            if self.window <= 0 or self.window >= length:
                total += length * (length + 1) // 2
            else:
                w = self.window
                total += w * (w + 1) // 2 + (length - w) * w
        return total


@dataclass(frozen=True)
class DecodeWorkload:
    """A varlen decode problem: one query per sequence over a packed KV cache."""
    name: str
    batch: int
    num_kv_heads: int
    window: int
    seed: int
    len_lo: int = 1024
    len_hi: int = 32768
    fixed_lengths: tuple = field(default=())

    def kv_lengths(self) -> np.ndarray:
        if self.fixed_lengths:
            return np.asarray(self.fixed_lengths, dtype=np.int64)
        g = torch.Generator(device="cpu").manual_seed(self.seed)
        return torch.randint(self.len_lo, self.len_hi + 1, (self.batch,), generator=g).numpy().astype(np.int64)


# The five workloads the library is measured and parity-checked on.
TINY = PrefillWorkload("tiny_T256_H1_full", (256,), 1, 0, 0)
PREFILL_FULL = PrefillWorkload("prefill_T4096_H16_full", (4096,), 16, 0, 1)
SWA = PrefillWorkload("swa128_B2_T32768_H16", (32768, 32768), 16, 128, 2)
HYBRID_LAYERS = tuple(
    PrefillWorkload(f"hybrid_T65536_H16_layer{l}_{'full' if l == 0 else 'w128'}", (65536,), 16,
                    0 if l == 0 else 128, 300 + l)
    for l in range(4)
)
DECODE_FULL = DecodeWorkload("decode_B64_H16_full", 64, 16, 0, 4)
DECODE_W128 = DecodeWorkload("decode_B64_H16_w128", 64, 16, 128, 4)
# The same decode batch over the compressed (latent) cache: one 576-wide row per token.
LATENT_FULL = DecodeWorkload("latent_decode_B64_H16_full", 64, 16, 0, 4)
LATENT_W128 = DecodeWorkload("latent_decode_B64_H16_w128", 64, 16, 128, 4)
DC, DR = 512, 64
DL = DC + DR


def _normal_bf16(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def _lambda(shape, gen, device):
    k = torch.randint(0, 1 << LAMBDA_BITS, shape, generator=gen, device=device, dtype=torch.int64)
    return ((k.to(torch.float64) + 0.5) / float(1 << LAMBDA_BITS)).to(torch.float32)


def make_prefill_inputs(seqlens, num_kv_heads, seed, device="cpu"):
    """Packed prefill inputs: dict of q_sig, q_noise, k, v (bf16), lam (fp32), gate (bf16)."""
    n = int(sum(int(s) for s in seqlens))
    hs = GROUP * num_kv_heads
    gen = torch.Generator(device=device).manual_seed(int(seed))
    return {
        "q_sig": _normal_bf16((n, hs, DQK), gen, device),
        "q_noise": _normal_bf16((n, num_kv_heads, DQK), gen, device),
        "k": _normal_bf16((n, num_kv_heads, DQK), gen, device),
        "v": _normal_bf16((n, num_kv_heads, DV), gen, device),
        "lam": _lambda((n, hs), gen, device),
        "gate": _normal_bf16((n, hs, DV), gen, device),
    }


def make_prefill_grad(seqlens, num_kv_heads, seed, device="cpu"):
    """Upstream gradient of the prefill output for the backward: dout [N, 4H, 128] bf16."""
    n = int(sum(int(s) for s in seqlens))
    gen = torch.Generator(device=device).manual_seed(int(seed) + 7919)
    return _normal_bf16((n, GROUP * num_kv_heads, DV), gen, device)


HIDDEN = 4096
Q_RANK = 1024


def make_prologue_inputs(seqlens, num_kv_heads, seed, device="cpu"):
    """Hidden states and projection weights for the prologue: x [N, 4096] bf16 (N(0,1));
    weights [out, in] bf16, N(0, 1/in) (unit-variance outputs): w_qa [1024, 4096],
    w_kva [576, 4096], w_qb [5H*192, 1024], w_uk / w_uv [H, 128, 512], w_lambda
    [4H, 4096], w_gate [4H*128, 4096]; RMSNorm weights gamma_q [1024], gamma_kv [512]
    fp32 (1 + N(0, 0.1^2))."""
    n = int(sum(int(s) for s in seqlens))
    hs = GROUP * num_kv_heads
    gen = torch.Generator(device=device).manual_seed(int(seed) + 104729)

    def w(shape, fan_in):
        return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
                / float(np.sqrt(fan_in))).to(torch.bfloat16)

    return {
        "x": _normal_bf16((n, HIDDEN), gen, device),
        "w_qa": w((Q_RANK, HIDDEN), HIDDEN),
        "w_kva": w((DC + DR, HIDDEN), HIDDEN),
        "gamma_q": 1.0 + 0.1 * torch.randn((Q_RANK,), generator=gen, device=device, dtype=torch.float32),
        "gamma_kv": 1.0 + 0.1 * torch.randn((DC,), generator=gen, device=device, dtype=torch.float32),
        "w_qb": w(((hs + num_kv_heads) * DQK, Q_RANK), Q_RANK),
        "w_uk": w((num_kv_heads, DV, DC), DC),
        "w_uv": w((num_kv_heads, DV, DC), DC),
        "w_lambda": w((hs, HIDDEN), HIDDEN),
        "w_gate": w((hs * DV, HIDDEN), HIDDEN),
    }


def make_decode_inputs(kv_lengths, num_kv_heads, seed, device="cpu"):
    """Decode inputs: one query per sequence plus the packed KV cache and cu_seqlens_k (int32)."""
    lengths = np.asarray(kv_lengths, dtype=np.int64)
    b = int(lengths.shape[0])
    nk = int(lengths.sum())
    hs = GROUP * num_kv_heads
    gen = torch.Generator(device=device).manual_seed(int(seed))
    cu = np.zeros(b + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    return {
        "q_sig": _normal_bf16((b, hs, DQK), gen, device),
        "q_noise": _normal_bf16((b, num_kv_heads, DQK), gen, device),
        "k_cache": _normal_bf16((nk, num_kv_heads, DQK), gen, device),
        "v_cache": _normal_bf16((nk, num_kv_heads, DV), gen, device),
        "lam": _lambda((b, hs), gen, device),
        "gate": _normal_bf16((b, hs, DV), gen, device),
        "cu_seqlens_k": torch.from_numpy(cu.astype(np.int32)).to(device),
    }


def make_latent_decode_inputs(kv_lengths, num_kv_heads, seed, device="cpu"):
    """Decode inputs over the latent cache: absorbed queries q_abs_sig [B, 4H, 576],
    q_abs_noise [B, H, 576], cache rows ckv [Nk, 576], w_uv [H, 128, 512] (bf16),
    lam [B, 4H] (fp32), gate [B, 4H, 128] (bf16) and cu_seqlens_k (int32)."""
    lengths = np.asarray(kv_lengths, dtype=np.int64)
    b = int(lengths.shape[0])
    nk = int(lengths.sum())
    hs = GROUP * num_kv_heads
    gen = torch.Generator(device=device).manual_seed(int(seed))
    cu = np.zeros(b + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    w_uv = (torch.randn((num_kv_heads, DV, DC), generator=gen, device=device, dtype=torch.float32)
            / float(np.sqrt(DC))).to(torch.bfloat16)
    return {
        "q_abs_sig": _normal_bf16((b, hs, DL), gen, device),
        "q_abs_noise": _normal_bf16((b, num_kv_heads, DL), gen, device),
        "ckv": _normal_bf16((nk, DL), gen, device),
        "w_uv": w_uv,
        "lam": _lambda((b, hs), gen, device),
        "gate": _normal_bf16((b, hs, DV), gen, device),
        "cu_seqlens_k": torch.from_numpy(cu.astype(np.int32)).to(device),
    }


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy uint16 view of a bf16 tensor's bit patterns (copies to host if needed)."""
    if t.dtype != torch.bfloat16:
        raise TypeError(f"expected bfloat16, got {t.dtype}")
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_from_bits(a: np.ndarray) -> torch.Tensor:
    """bf16 CPU tensor holding the given uint16 bit patterns."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def sample_rows(seqlens, per_seq, seed, must_include=(0, 1, 127, 128)):
    """Packed token indices of ``per_seq`` rows per sequence: the rows ``must_include``
    (clipped to the sequence), its last row, and uniform draws for the rest."""
    g = np.random.default_rng(seed)
    rows = []
    start = 0
    for length in seqlens:
        length = int(length)
        if length == 0:
            continue
        pick = {t for t in must_include if t < length} | {length - 1}
        if per_seq >= length:
            pick = set(range(length))
        else:
            rest = g.choice(length, size=min(length, per_seq), replace=False)
            for t in rest:
                if len(pick) >= per_seq:
                    break
                pick.add(int(t))
        rows.extend(start + t for t in sorted(pick))
        start += length
    return np.asarray(rows, dtype=np.int64)
