"""GPU parity of gdla_attn_decode_latent (through the C ABI) against the fp64
oracle of decode over the compressed KV cache (itself pinned to the expanded
decode oracle in test_oracle_latent.py)."""
import numpy as np
import pytest
import torch

import differential_latent_attention_b200 as gdla
import gdla_inputs as gi
import oracle
from _parity import assert_close

pytestmark = pytest.mark.gpu


def _host(d):
    return [gi.bf16_bits(d["q_abs_sig"]), gi.bf16_bits(d["q_abs_noise"]), gi.bf16_bits(d["ckv"]),
            d["cu_seqlens_k"].cpu().numpy().astype(np.int64), gi.bf16_bits(d["w_uv"]), d["lam"].cpu().numpy(),
            gi.bf16_bits(d["gate"])]


def _gpu(d, max_len, window, workspace=None):
    return gdla.attn_decode_latent(d["q_abs_sig"], d["q_abs_noise"], d["ckv"], d["cu_seqlens_k"], max_len,
                                   d["w_uv"], d["lam"], d["gate"], window, workspace=workspace)


def _check(lengths, hkv, window, seed, max_len=None):
    d = gi.make_latent_decode_inputs(lengths, hkv, seed, device="cuda")
    max_len = int(max(lengths)) if max_len is None else max_len
    out = _gpu(d, max_len, window)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    ref = oracle.decode_latent(*_host(d), window)
    return assert_close(out.float().cpu().numpy(), ref, f"latent decode lengths={lengths} window={window}")


EDGE_LENS = (1, 2, 47, 48, 49, 95, 96, 97, 2047, 2048, 2049, 4097, 5000)


@pytest.mark.parametrize("window", [0, 1, 48, 128, 3000])
def test_edge_lengths(window):
    """Stage edges (48 keys), split edges (2,048 keys) and windows."""
    _check(EDGE_LENS, 2, window, 80 + window)


@pytest.mark.parametrize("hkv", [1, 3, 5, 16])
def test_kv_head_counts(hkv):
    """1..16 KV heads: the noise rows start at 4H rounded up to 8 and the
    O^T product covers the used rows rounded up to 16."""
    _check((300, 2100, 7), hkv, 0, 81 + hkv)


@pytest.mark.parametrize("w", [gi.LATENT_FULL, gi.LATENT_W128], ids=lambda w: w.name)
def test_latent_decode_B64_H16(w):
    """The bench workload: 64 sequences, KV lengths U[1024, 32768], 16 KV heads."""
    lengths = w.kv_lengths()
    _check(tuple(int(x) for x in lengths), w.num_kv_heads, w.window, w.seed, max_len=32768)


def test_rescale_on_rising_scores():
    """Rotary keys whose magnitude grows along the sequence (1 + u/4 at position
    u; the 512 latent dims, which are also the values, keep unit scale): each
    48-key stage raises every head's running maximum by far more than 2^8, so
    O^T is rescaled on every stage of every split."""
    lengths = (3000, 700)
    d = gi.make_latent_decode_inputs(lengths, 2, 84, device="cuda")
    pos = torch.cat([torch.arange(n, device="cuda") for n in lengths]).float()
    ckv = d["ckv"].float()
    ckv[:, gi.DC:] *= 1.0 + pos[:, None] / 4.0
    d["ckv"] = ckv.to(torch.bfloat16)
    out = _gpu(d, 3000, 0)
    torch.cuda.synchronize()
    ref = oracle.decode_latent(*_host(d), 0)
    assert_close(out.float().cpu().numpy(), ref, "latent decode, rising scores")


def test_invalid_lengths_give_zero_output():
    lengths = (10, 20)
    d = gi.make_latent_decode_inputs(lengths, 1, 85, device="cuda")
    cu = d["cu_seqlens_k"].clone()
    cu[1] = cu[0]          # sequence 0 empty, sequence 1 then 30 rows long (> max_seqlen_k)
    d["cu_seqlens_k"] = cu
    out = _gpu(d, 20, 0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()) == 0


def test_deterministic_and_workspace_contents_do_not_matter():
    d = gi.make_latent_decode_inputs((3000, 5000, 17), 2, 86, device="cuda")
    need = gdla.decode_latent_workspace_bytes(3, 2, 5000, 0)
    ws = torch.full((need // 4,), float("nan"), dtype=torch.float32, device="cuda").view(torch.uint8)
    a = _gpu(d, 5000, 0).clone()
    b = _gpu(d, 5000, 0, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_window_one_closed_form():
    """Window 1: each query sees only its last cache row [c | k_rope], so every head of
    group j gives H = W^UV_j c and out = sigmoid(g) (1 - lambda) W^UV_j c (fp64)."""
    lengths = (1, 2, 49, 2049, 300)
    d = gi.make_latent_decode_inputs(lengths, 2, 62, device="cuda")
    out = _gpu(d, max(lengths), 1)
    torch.cuda.synchronize()
    last = d["cu_seqlens_k"][1:].long() - 1
    c = d["ckv"][last, :512].double().cpu()                                  # [B, 512]
    h = torch.einsum("jde,be->bjd", d["w_uv"].double().cpu(), c)              # [B, H, 128]
    h = h.repeat_interleave(4, dim=1)
    ref = torch.sigmoid(d["gate"].double().cpu()) * (1.0 - d["lam"].double().cpu())[..., None] * h
    assert_close(out.float().cpu().numpy(), ref.numpy(), "latent decode window 1")


@pytest.mark.parametrize("window", [0, 128])
def test_zero_query_gives_the_projected_mean(window):
    """Zero absorbed queries: every visible row scores 0, so each head of group j gives
    H = W^UV_j mean(c) over the visible rows and out = sigmoid(g) (1 - lambda) H (fp64)."""
    lengths = (1, 129, 2049, 5000, 64)
    d = gi.make_latent_decode_inputs(lengths, 2, 64 + window, device="cuda")
    d["q_abs_sig"] = torch.zeros_like(d["q_abs_sig"])
    d["q_abs_noise"] = torch.zeros_like(d["q_abs_noise"])
    out = _gpu(d, max(lengths), window)
    torch.cuda.synchronize()
    cu = d["cu_seqlens_k"].cpu().long()
    c = d["ckv"][:, :512].double().cpu()
    means = torch.stack([c[max(int(cu[b]), int(cu[b + 1]) - window) if window > 0 else int(cu[b]):int(cu[b + 1])]
                         .mean(0) for b in range(len(lengths))])                       # [B, 512]
    h = torch.einsum("jde,be->bjd", d["w_uv"].double().cpu(), means).repeat_interleave(4, dim=1)
    ref = torch.sigmoid(d["gate"].double().cpu()) * (1.0 - d["lam"].double().cpu())[..., None] * h
    assert_close(out.float().cpu().numpy(), ref.numpy(), f"latent decode zero queries, window {window}")


def test_group_permutation_equivariant_bitwise():
    """Permuting the KV groups (their queries, W^UV_j, lambda and gate) permutes the
    output groups bit for bit: every group's heads see the same cache rows."""
    lengths = (1, 300, 2049, 77)
    hkv, perm = 3, [2, 0, 1]
    d = gi.make_latent_decode_inputs(lengths, hkv, 65, device="cuda")
    a = _gpu(d, max(lengths), 0)

    def grp(x, per):
        b = x.shape[0]
        return x.reshape(b, hkv, per, *x.shape[2:])[:, perm].reshape(x.shape).contiguous()

    p = dict(d, q_abs_sig=grp(d["q_abs_sig"], 4), q_abs_noise=grp(d["q_abs_noise"], 1),
             w_uv=d["w_uv"][perm].contiguous(), lam=grp(d["lam"], 4), gate=grp(d["gate"], 4))
    b = _gpu(p, max(lengths), 0)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    assert torch.equal(grp(a, 4).view(torch.int16), b.view(torch.int16))
