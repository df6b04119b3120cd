"""GPU parity of gdla_attn_decode (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import differential_latent_attention_b200 as gdla
import gdla_inputs as gi
import oracle
from _parity import assert_close, decode_host_args, gpu_decode, gpu_prefill, host_args

pytestmark = pytest.mark.gpu

EDGE_LENS = (1, 2, 63, 64, 65, 127, 128, 129, 1023, 1024, 1025, 2047, 2048, 2049, 5000)


def _check(lengths, hkv, window, seed, max_len=None):
    d = gi.make_decode_inputs(lengths, hkv, seed, device="cuda")
    max_len = int(max(lengths)) if max_len is None else max_len
    out = gpu_decode(d, max_len, window)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    ref = oracle.decode(*decode_host_args(d), window)
    return assert_close(out.float().cpu().numpy(), ref, f"decode lengths={lengths} window={window}")


@pytest.mark.parametrize("window", [0, 1, 128, 129, 3000])
def test_edge_lengths(window):
    _check(EDGE_LENS, 2, window, 50 + window)


def test_split_boundaries():
    # max_seqlen_k 5000 -> 5 splits of 1024 keys; lengths at split edges +-1
    _check((1023, 1024, 1025, 2048, 2049, 4095, 4096, 4097, 5000), 1, 0, 51, max_len=5000)


def test_max_len_larger_than_needed():
    _check((700, 1300), 3, 0, 52, max_len=40000)


def test_decode_equals_last_prefill_row():
    lengths = (3, 700, 2500)
    t = gi.make_prefill_inputs(lengths, 2, 53, device="cuda")
    last = torch.as_tensor(np.cumsum(lengths) - 1, device="cuda")
    cu = torch.as_tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), device="cuda")
    pre = gpu_prefill(t, lengths, 0)
    d = {"q_sig": t["q_sig"][last].contiguous(), "q_noise": t["q_noise"][last].contiguous(),
         "k_cache": t["k"], "v_cache": t["v"], "cu_seqlens_k": cu, "lam": t["lam"][last].contiguous(),
         "gate": t["gate"][last].contiguous()}
    dec = gpu_decode(d, max(lengths), 0)
    torch.cuda.synchronize()
    assert_close(dec.float().cpu().numpy(), pre[last].double().cpu().numpy(), "decode vs prefill last row")


def test_invalid_lengths_give_zero_output():
    lengths = (10, 20)
    d = gi.make_decode_inputs(lengths, 1, 54, device="cuda")
    cu = d["cu_seqlens_k"].clone()
    cu[1] = cu[0]          # sequence 0 empty, sequence 1 then 30 rows long
    d["cu_seqlens_k"] = cu
    out = gpu_decode(d, 20, 0)        # 30 > max_seqlen_k for sequence 1 as well
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()) == 0


def test_deterministic():
    d = gi.make_decode_inputs((3000, 5000, 17), 2, 55, device="cuda")
    a = gpu_decode(d, 5000, 0).clone()
    b = gpu_decode(d, 5000, 0)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_single_split_persistent_uneven_items():
    """Short caches (one split): 700 sequences x 2 KV groups = 1,400 items, more
    than the resident persistent CTAs, with 1 to 32 key stages each, so each
    CTA's K/V stage ring runs on across items of different lengths."""
    rng = np.random.default_rng(57)
    lengths = tuple(int(x) for x in rng.integers(1, 1001, size=700))
    _check(lengths, 2, 0, 57, max_len=1000)
    _check(lengths, 2, 100, 58, max_len=1000)


@pytest.mark.parametrize("w", [gi.DECODE_FULL, gi.DECODE_W128], ids=lambda w: w.name)
def test_decode_B64_H16(w):
    lengths = w.kv_lengths()
    _check(tuple(int(x) for x in lengths), w.num_kv_heads, w.window, w.seed, max_len=32768)


@pytest.mark.parametrize("window", [0, 128])
def test_largest_kv_head_count(window):
    """GDLA_MAX_KV_HEADS = 64 KV heads."""
    _check((300, 2000, 1), 64, window, 56)


def test_64_splits_of_more_than_1024_keys():
    """max_seqlen_k = 81,920: the split plan reaches its cap of 64 splits, each of
    1,280 keys (more than the 1,024-key minimum), so the combine kernel merges a
    full 64-entry split row; lengths fill the last split fully, partly, or leave
    most splits empty."""
    from differential_latent_attention_b200 import ops
    assert ops.decode_workspace_bytes(4, 1, 81920, 0) == 4 * 1 * 64 * 5 * 130 * 4
    _check((81920, 70001, 5, 40000), 1, 0, 59, max_len=81920)


def _permute_groups(d, perm):
    """The same decode problem with its KV groups reordered by perm (query, lambda,
    gate and cache heads moved together)."""
    perm = torch.as_tensor(perm, device="cuda")
    sig = torch.stack([perm * 4 + i for i in range(4)], dim=1).reshape(-1)
    return {"q_sig": d["q_sig"][:, sig].contiguous(), "q_noise": d["q_noise"][:, perm].contiguous(),
            "k_cache": d["k_cache"][:, perm].contiguous(), "v_cache": d["v_cache"][:, perm].contiguous(),
            "cu_seqlens_k": d["cu_seqlens_k"], "lam": d["lam"][:, sig].contiguous(),
            "gate": d["gate"][:, sig].contiguous()}, sig


@pytest.mark.parametrize("window", [0, 128])
def test_group_permutation_equivariant_bitwise(window):
    """Reordering the KV groups (with their signal and noise heads) reorders the
    output the same way, bit for bit: groups are computed independently."""
    d = gi.make_decode_inputs((3000, 77, 1500), 3, 64, device="cuda")
    perm = [2, 0, 1]
    a = gpu_decode(d, 3000, window)
    dp, sig = _permute_groups(d, perm)
    b = gpu_decode(dp, 3000, window)
    torch.cuda.synchronize()
    assert torch.equal(a[:, sig].view(torch.int16), b.view(torch.int16))


def test_window_at_least_length_equals_full_bitwise():
    """A window no shorter than every sequence sees exactly the full context: the
    output is bit-identical to window 0 (both take the several-split path)."""
    d = gi.make_decode_inputs((2500, 3000, 17), 2, 65, device="cuda")
    a = gpu_decode(d, 3000, 0)
    b = gpu_decode(d, 3000, 3000)
    c = gpu_decode(d, 3000, 100000)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_window_one_closed_form():
    """Window 1: each query sees only its own (last) cache row, so out = sigmoid(g)
    (1 - lambda) v_last of its group: checked in fp64 against that closed form."""
    lengths = (1, 2, 64, 1025, 300)
    d = gi.make_decode_inputs(lengths, 2, 61, device="cuda")
    out = gpu_decode(d, max(lengths), 1)
    torch.cuda.synchronize()
    last = d["cu_seqlens_k"][1:].long() - 1
    v = d["v_cache"][last].double().cpu().repeat_interleave(4, dim=1)      # [B, 4H, 128]
    ref = torch.sigmoid(d["gate"].double().cpu()) * (1.0 - d["lam"].double().cpu())[..., None] * v
    assert_close(out.float().cpu().numpy(), ref.numpy(), "decode window 1")


@pytest.mark.parametrize("window", [0, 128])
def test_zero_query_gives_the_mean_of_the_visible_values(window):
    """Zero queries: every visible key scores 0, so out = sigmoid(g) (1 - lambda) times the
    mean of the visible value rows (fp64 closed form; one- and several-split plans)."""
    lengths = (1, 129, 1025, 5000, 64)
    d = gi.make_decode_inputs(lengths, 2, 63 + window, device="cuda")
    d["q_sig"] = torch.zeros_like(d["q_sig"])
    d["q_noise"] = torch.zeros_like(d["q_noise"])
    out = gpu_decode(d, max(lengths), window)
    torch.cuda.synchronize()
    cu = d["cu_seqlens_k"].cpu().long()
    v = d["v_cache"].double().cpu()
    means = torch.stack([v[max(int(cu[b]), int(cu[b + 1]) - window) if window > 0 else int(cu[b]):int(cu[b + 1])]
                         .mean(0) for b in range(len(lengths))])                       # [B, H, 128]
    ref = torch.sigmoid(d["gate"].double().cpu()) * (1.0 - d["lam"].double().cpu())[..., None] * \
        means.repeat_interleave(4, dim=1)
    assert_close(out.float().cpu().numpy(), ref.numpy(), f"decode zero queries, window {window}")
