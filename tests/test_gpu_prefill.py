"""GPU parity of gdla_attn_fwd (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import differential_latent_attention_b200 as gdla
import gdla_inputs as gi
import oracle
from _parity import assert_close, check_prefill, gpu_prefill, host_args

pytestmark = pytest.mark.gpu


def test_tiny_all_rows():
    w = gi.TINY
    check_prefill(w.seqlens, w.num_kv_heads, w.window, w.seed)


EDGE_SEQS = (1, 63, 64, 65, 127, 128, 129, 23, 24, 25, 0, 47, 48, 49, 300)


@pytest.mark.parametrize("window", [0, 1, 2, 24, 127, 128, 129, 4096])
def test_ragged_batch_all_rows(window):
    check_prefill(EDGE_SEQS, 2, window, 100 + max(window, 0))


@pytest.mark.parametrize("hkv", [1, 3, 5])
def test_kv_head_counts(hkv):
    check_prefill((200, 77), hkv, 0, 7)


def test_several_key_tiles_and_ragged_tail():
    # 1000 tokens: 8 key tiles of 128, a ragged last q-tile (1000 = 41*24 + 16)
    check_prefill((1000,), 2, 0, 8)
    check_prefill((1000,), 2, 128, 9)


def test_every_row_written_and_deterministic():
    seqlens = (5, 130, 1, 64)
    t = gi.make_prefill_inputs(seqlens, 2, 11, device="cuda")
    out = torch.full((sum(seqlens), 8, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    gpu_prefill(t, seqlens, 0, out=out)
    first = out.clone()
    gpu_prefill(t, seqlens, 0, out=out)
    torch.cuda.synchronize()
    assert torch.isfinite(first.float()).all()
    assert torch.equal(first.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("window", [0, 16])
def test_gate_and_out_only_16_byte_aligned(window):
    """gate/out at 16- but not 32-byte aligned addresses take the 16-byte access
    path of the epilogue; the result must be bit-identical to the aligned run."""
    seqlens = (70, 200, 3)
    t = gi.make_prefill_inputs(seqlens, 2, 18, device="cuda")
    ref = gpu_prefill(t, seqlens, window)
    n = sum(seqlens)
    gbuf = torch.empty(n * 8 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    obuf = torch.full((n * 8 * 128 + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    g16 = gbuf[8:].view(n, 8, 128)
    g16.copy_(t["gate"])
    o16 = obuf[8:].view(n, 8, 128)
    assert g16.data_ptr() % 32 == 16 and o16.data_ptr() % 32 == 16
    gdla.attn_fwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], g16, seqlens, window, out=o16)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    assert torch.equal(ref.view(torch.int16), o16.view(torch.int16))


def test_empty_batch_is_a_no_op():
    """Zero tokens: the call returns GDLA_OK without launching anything."""
    import ctypes
    lib = gdla.library()
    lens = np.zeros(2, dtype=np.int32)
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())
    assert lib.gdla_attn_fwd(p, p, p, p, p, p, p, 2, lens.ctypes.data_as(ctypes.c_void_p), 1, 0, None) == 0


@pytest.mark.parametrize("window", [0, 128, 1000])
def test_identical_paths_cancel_exactly(window):
    """Signal queries equal to their noise query and lambda = 1: the signal and
    noise rows of every MMA hold identical operands, so H_S and H_N agree bit for
    bit and D = 0 exactly in every configuration (a wrong noise/KV group pairing
    would leave O(1) outputs)."""
    seqlens = (150, 40)
    t = gi.make_prefill_inputs(seqlens, 2, 12, device="cuda")
    t["q_sig"] = t["q_noise"].repeat_interleave(4, dim=1).contiguous()
    t["lam"] = torch.ones_like(t["lam"])
    out = gpu_prefill(t, seqlens, window)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()).item() == 0


def test_lambda_zero_gate_open_is_gqa_attention():
    """lambda = 0, gate logit 40: the GPU output is plain causal GQA attention,
    checked against torch's SDPA (float64, CPU) rather than the oracle."""
    import torch.nn.functional as F
    seqlens = (300,)
    t = gi.make_prefill_inputs(seqlens, 2, 13, device="cuda")
    t["lam"] = torch.zeros_like(t["lam"])
    t["gate"] = torch.full_like(t["gate"], 40.0)
    out = gpu_prefill(t, seqlens, 0).float().cpu().numpy()
    q = t["q_sig"].double().cpu().permute(1, 0, 2)[None]
    k = t["k"].double().cpu().permute(1, 0, 2)[None]
    v = t["v"].double().cpu().permute(1, 0, 2)[None]
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)[0].permute(1, 0, 2).numpy()
    assert_close(out, ref, "lambda=0 vs SDPA")


def test_prefill_full_T4096_sampled_rows():
    """The bench's own workload and launch: T=4096, 16 KV groups, full causal."""
    w = gi.PREFILL_FULL
    rows = gi.sample_rows(w.seqlens, 512, seed=1, must_include=(0, 1, 23, 24, 127, 128, 4095))
    check_prefill(w.seqlens, w.num_kv_heads, w.window, w.seed, rows=rows)


def test_swa_B2_T32768_sampled_rows():
    w = gi.SWA
    rows = gi.sample_rows(w.seqlens, 512, seed=2, must_include=(0, 1, 126, 127, 128, 129))
    check_prefill(w.seqlens, w.num_kv_heads, w.window, w.seed, rows=rows)


@pytest.mark.slow
@pytest.mark.parametrize("layer", [0, 1, 2, 3])
def test_hybrid_T65536_layers_sampled_rows(layer):
    w = gi.HYBRID_LAYERS[layer]
    rows = gi.sample_rows(w.seqlens, 512, seed=40 + layer, must_include=(0, 1, 127, 128, 65535))
    check_prefill(w.seqlens, w.num_kv_heads, w.window, w.seed, rows=rows)


def test_no_device_error_recorded():
    assert gdla.device_error(clear=True) == 0


def test_more_sequences_than_one_launch_holds():
    """300 sequences (over the 256 a launch plan holds): the host splits the batch
    across launches; every row must still match."""
    rng = np.random.default_rng(5)
    seqlens = tuple(int(x) for x in rng.integers(0, 41, size=300))
    check_prefill(seqlens, 2, 0, 14)
    check_prefill(seqlens, 2, 16, 15)


def test_more_blocks_than_one_launch_holds():
    """200 sequences of 800 tokens: 6,800 token blocks (over the 6,144 a launch plan
    holds) in the full-causal configuration; sampled rows of every sequence."""
    seqlens = (800,) * 200
    rows = gi.sample_rows(seqlens, 3, seed=16, must_include=(0, 799))
    check_prefill(seqlens, 1, 0, 16, rows=rows)


@pytest.mark.parametrize("window", [0, 128])
def test_largest_kv_head_count(window):
    """GDLA_MAX_KV_HEADS = 64 KV heads (256 signal + 64 noise query heads)."""
    check_prefill((130, 31), 64, window, 20)


@pytest.mark.parametrize("window", [257, 300, 1000])
def test_windows_in_the_causal_configuration(window):
    """Windows over 256 run the one-tile configuration with window masks and key-tile
    skipping; the sequences are longer than the window, so both take effect."""
    check_prefill((1500, 700), 2, window, 21)


def _permute_prefill_groups(t, perm):
    perm = torch.as_tensor(perm, device="cuda")
    sig = torch.stack([perm * 4 + i for i in range(4)], dim=1).reshape(-1)
    return {"q_sig": t["q_sig"][:, sig].contiguous(), "q_noise": t["q_noise"][:, perm].contiguous(),
            "k": t["k"][:, perm].contiguous(), "v": t["v"][:, perm].contiguous(),
            "lam": t["lam"][:, sig].contiguous(), "gate": t["gate"][:, sig].contiguous()}, sig


@pytest.mark.parametrize("window", [0, 128, 1000])
def test_group_permutation_equivariant_bitwise(window):
    """Reordering the KV groups (with their signal and noise query heads, lambda
    and gate) reorders the output the same way, bit for bit."""
    seqlens = (1300, 77, 300)
    t = gi.make_prefill_inputs(seqlens, 3, 22, device="cuda")
    a = gpu_prefill(t, seqlens, window)
    tp, sig = _permute_prefill_groups(t, [1, 2, 0])
    b = gpu_prefill(tp, seqlens, window)
    torch.cuda.synchronize()
    assert torch.equal(a[:, sig].view(torch.int16), b.view(torch.int16))


def test_window_at_least_length_equals_full_bitwise():
    """Windows no shorter than the sequence see the full causal context: bit-identical
    outputs (one-tile configuration: window 4096 vs full causal; sliding
    configuration: windows 255 and 256 over sequences of at most 200 tokens)."""
    seqlens = (1000, 129, 1)
    t = gi.make_prefill_inputs(seqlens, 2, 23, device="cuda")
    a = gpu_prefill(t, seqlens, 0)
    b = gpu_prefill(t, seqlens, 4096)
    short = (200, 48, 1, 97)
    ts = gi.make_prefill_inputs(short, 2, 24, device="cuda")
    c = gpu_prefill(ts, short, 255)
    d = gpu_prefill(ts, short, 256)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(c.view(torch.int16), d.view(torch.int16))
    check_prefill(short, 2, 256, 24, t=ts)


def _closed_form(t, rows, v_rows):
    """sigma(g) (1 - lambda) v for the given output rows, each with its own value row
    per KV group (fp64, from the inputs as stored)."""
    g = t["gate"][rows].double().cpu()                               # [R, 4H, 128]
    lam = t["lam"][rows].double().cpu()                              # [R, 4H]
    v = v_rows.double().cpu().repeat_interleave(4, dim=1)            # [R, 4H, 128]
    return (torch.sigmoid(g) * (1.0 - lam)[..., None] * v).numpy()


@pytest.mark.parametrize("window", [1, 0])
def test_single_visible_key_closed_form(window):
    """A row that sees one key (every row at window 1; the first row of each sequence
    otherwise) has H_S = H_N = v_t, so out = sigmoid(g) (1 - lambda) v_t: the GPU output
    against that closed form in fp64, not against the oracle."""
    seqlens = (37, 1, 130, 24, 25)
    t = gi.make_prefill_inputs(seqlens, 2, 31 + window, device="cuda")
    out = gpu_prefill(t, seqlens, window)
    torch.cuda.synchronize()
    starts = np.concatenate([[0], np.cumsum(seqlens)[:-1]])
    rows = torch.arange(sum(seqlens)) if window == 1 else torch.as_tensor(starts)
    ref = _closed_form(t, rows, t["v"][rows])
    assert_close(out[rows.cuda()].float().cpu().numpy(), ref, f"one visible key, window {window}")


@pytest.mark.parametrize("window", [0, 128])
def test_identical_value_rows_closed_form(window):
    """All value rows of a group equal (v_u = c_j): the softmax weights sum to one, so
    out = sigmoid(g) (1 - lambda) c_j for every row, whatever the scores."""
    seqlens = (300, 61)
    t = gi.make_prefill_inputs(seqlens, 2, 33 + window, device="cuda")
    t["v"] = t["v"][:1].expand_as(t["v"]).contiguous()
    out = gpu_prefill(t, seqlens, window)
    torch.cuda.synchronize()
    rows = torch.arange(sum(seqlens))
    ref = _closed_form(t, rows, t["v"])
    assert_close(out.float().cpu().numpy(), ref, f"identical value rows, window {window}")


def test_saturated_gate_gives_the_ungated_difference():
    """Gate logits 40 and 60 both give sigmoid = 1 to fp32 resolution: the outputs are
    bit-identical, and equal to the oracle's D = H_S - lambda H_N."""
    seqlens = (200, 33)
    t = gi.make_prefill_inputs(seqlens, 2, 35, device="cuda")
    t["gate"] = torch.full_like(t["gate"], 40.0)
    a = gpu_prefill(t, seqlens, 0)
    t60 = dict(t, gate=torch.full_like(t["gate"], 60.0))
    b = gpu_prefill(t60, seqlens, 0)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    ref = oracle.prefill(*host_args(t), seqlens, 0)
    assert_close(a.float().cpu().numpy(), ref, "gate logit 40")


@pytest.mark.parametrize("window", [0, 128])
def test_zero_queries_give_the_running_mean(window):
    """All queries zero: every visible key scores 0, so each head's H is the plain mean of
    the visible value rows and out = sigmoid(g) (1 - lambda) mean(v) (fp64 closed form,
    over sequences spanning several key tiles)."""
    seqlens = (300, 61)
    t = gi.make_prefill_inputs(seqlens, 2, 37 + window, device="cuda")
    t["q_sig"] = torch.zeros_like(t["q_sig"])
    t["q_noise"] = torch.zeros_like(t["q_noise"])
    out = gpu_prefill(t, seqlens, window)
    torch.cuda.synchronize()
    v = t["v"].double().cpu()
    means = []
    s0 = 0
    for n in seqlens:
        c = torch.cumsum(v[s0:s0 + n], 0)
        for i in range(n):
            lo = 0 if window <= 0 else max(0, i - window + 1)
            tot = c[i] - (c[lo - 1] if lo > 0 else 0)
            means.append(tot / (i - lo + 1))
        s0 += n
    ref = _closed_form(t, torch.arange(sum(seqlens)), torch.stack(means))
    assert_close(out.float().cpu().numpy(), ref, f"zero queries, window {window}")
