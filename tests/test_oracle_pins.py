"""Pins of the fp64 oracle to facts other than itself (CPU only).

The pages print no worked example, so every pin here is a closed form, an
invariant of the method, a special case that reduces to a library routine
(torch's CPU scaled_dot_product_attention in float64), or brute force on tiny
inputs. Together they are chosen so that a plausible slip in the oracle (a
dropped term, a wrong sign, head or group index, a transposed operand, a wrong
scale or window edge) fails at least one of them; ``test_oracle_mutants.py``
plants such slips in a copy of the oracle and checks that they are caught.

Formulas followed (aitrends.kr/articles/94908, GDLA paragraphs):
D_t = H_S,t - lambda_t * Repeat_g(H_N,t), then the element-wise sigmoid gate;
g = 4, shared KV head per group, lambda in (0, 1).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gdla_inputs as gi
import oracle

G, DQK, DV = 4, 192, 128


def _np_inputs(seqlens, hkv, seed):
    t = gi.make_prefill_inputs(seqlens, hkv, seed, device="cpu")
    return {
        "q_sig": gi.bf16_bits(t["q_sig"]), "q_noise": gi.bf16_bits(t["q_noise"]),
        "k": gi.bf16_bits(t["k"]), "v": gi.bf16_bits(t["v"]),
        "lam": t["lam"].numpy().copy(), "gate": gi.bf16_bits(t["gate"]),
    }


def _f64(bits):
    return gi.bf16_from_bits(bits).to(torch.float64)


def _run(inp, seqlens, window, rows=None):
    return oracle.prefill(inp["q_sig"], inp["q_noise"], inp["k"], inp["v"], inp["lam"], inp["gate"],
                          seqlens, window, rows=rows)


def _sdpa(q, k, v, seqlens, window):
    """Library attention per sequence: q [N, Hq, 192], k [N, Hkv, 192], v [N, Hkv, 128]
    (float64 torch), causal, optionally restricted to the last ``window`` keys."""
    outs, s0 = [], 0
    for length in seqlens:
        qq = q[s0:s0 + length].permute(1, 0, 2)[None]
        kk = k[s0:s0 + length].permute(1, 0, 2)[None]
        vv = v[s0:s0 + length].permute(1, 0, 2)[None]
        if window <= 0:
            o = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True, enable_gqa=True)
        else:
            t = torch.arange(length)[:, None]
            u = torch.arange(length)[None, :]
            mask = (u <= t) & (u > t - window)
            o = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, enable_gqa=True)
        outs.append(o[0].permute(1, 0, 2))
        s0 += length
    return torch.cat(outs, 0)


SEQS = (37, 1, 70)  # several sequences, ragged, one of length 1


@pytest.mark.parametrize("window", [0, 5, 16])
def test_library_special_case_lambda0_gate_open(window):
    """lambda = 0 and sigmoid(gate) = 1 (logit 40 rounds sigmoid to 1.0 in fp64):
    the output is plain causal GQA attention of the signal heads, which torch's
    SDPA computes with its own default 1/sqrt(192) scale and head grouping."""
    inp = _np_inputs(SEQS, 2, 11)
    inp["lam"][:] = 0.0
    inp["gate"][:] = gi.bf16_bits(torch.full((1,), 40.0, dtype=torch.bfloat16))[0]
    got = _run(inp, SEQS, window)
    ref = _sdpa(_f64(inp["q_sig"]), _f64(inp["k"]), _f64(inp["v"]), SEQS, window).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [0, 3])
def test_full_output_against_library_attention(window):
    """General lambda and gate: out = sigmoid(g) * (H_S - lambda * Repeat_4(H_N)) with
    H_S and H_N both from the library routine (noise head j on KV head j)."""
    inp = _np_inputs(SEQS, 3, 12)
    got = _run(inp, SEQS, window)
    hs = _sdpa(_f64(inp["q_sig"]), _f64(inp["k"]), _f64(inp["v"]), SEQS, window)
    hn = _sdpa(_f64(inp["q_noise"]), _f64(inp["k"]), _f64(inp["v"]), SEQS, window)
    lam = torch.from_numpy(inp["lam"]).to(torch.float64)
    gate = _f64(inp["gate"])
    ref = torch.sigmoid(gate) * (hs - lam[..., None] * hn.repeat_interleave(G, dim=1))
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_identical_paths_with_lambda_one_cancel_exactly():
    """Every signal query equal to its group's noise query and lambda = 1: D = 0 exactly."""
    inp = _np_inputs(SEQS, 2, 13)
    n = sum(SEQS)
    inp["q_sig"] = np.repeat(inp["q_noise"], G, axis=1).reshape(n, 2 * G, DQK).copy()
    inp["lam"][:] = 1.0
    got = _run(inp, SEQS, 0)
    assert np.all(got == 0.0)


def test_identical_paths_cancel_only_in_their_own_group():
    """Signal heads of group 0 copy noise head 1 instead: with lambda = 1 the output
    must NOT vanish (a swapped noise/KV group index would make it vanish)."""
    inp = _np_inputs(SEQS, 2, 13)
    inp["q_sig"][:, 0:G] = inp["q_noise"][:, 1:2]
    inp["lam"][:] = 1.0
    got = _run(inp, SEQS, 0)
    assert np.abs(got[:, 0:G]).max() > 1e-3


def test_gate_zero_halves_gate_open_exactly():
    """sigmoid(0) = 1/2 exactly and sigmoid(40) = 1.0 in fp64: out(g=0) * 2 == out(g=40)."""
    inp = _np_inputs(SEQS, 2, 14)
    inp["gate"][:] = 0
    half = _run(inp, SEQS, 0)
    inp["gate"][:] = gi.bf16_bits(torch.full((1,), 40.0, dtype=torch.bfloat16))[0]
    full = _run(inp, SEQS, 0)
    assert np.array_equal(half * 2.0, full)


def test_gate_is_elementwise_sigmoid():
    """Gate logit -40 gives out ~ D * e^-40 per element (and leaves neighbours alone)."""
    inp = _np_inputs((9,), 1, 15)
    base = _run(inp, (9,), 0)
    inp["gate"][:] = gi.bf16_bits(torch.full((1,), 40.0, dtype=torch.bfloat16))[0]
    d = _run(inp, (9,), 0)
    inp["gate"][4, 2, 7] = gi.bf16_bits(torch.full((1,), -40.0, dtype=torch.bfloat16))[0]
    closed = _run(inp, (9,), 0)
    assert closed[4, 2, 7] == pytest.approx(d[4, 2, 7] / (1.0 + math.exp(40.0)), rel=1e-14)
    mask = np.ones_like(closed, dtype=bool)
    mask[4, 2, 7] = False
    assert np.array_equal(closed[mask], d[mask])
    sig = 1.0 / (1.0 + np.exp(-_f64(gi.bf16_bits(gi.make_prefill_inputs((9,), 1, 15)["gate"])).numpy()))
    np.testing.assert_allclose(base, sig * d, rtol=1e-14, atol=0)


@pytest.mark.parametrize("window", [70, 71, 1000])
def test_window_at_least_length_equals_full_causal(window):
    inp = _np_inputs(SEQS, 2, 16)
    assert np.array_equal(_run(inp, SEQS, window), _run(inp, SEQS, 0))


def test_window_one_closed_form():
    """window = 1: each head sees only its own key, so H = v_t for every head and
    out = sigmoid(g) * (1 - lambda) * v_t."""
    inp = _np_inputs(SEQS, 2, 17)
    got = _run(inp, SEQS, 1)
    v = _f64(inp["v"]).numpy()                       # [N, 2, 128]
    lam = inp["lam"].astype(np.float64)              # [N, 8]
    sig = 1.0 / (1.0 + np.exp(-_f64(inp["gate"]).numpy()))
    ref = sig * (1.0 - lam[..., None]) * np.repeat(v, G, axis=1)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-15)


def test_first_row_of_each_sequence_closed_form():
    inp = _np_inputs(SEQS, 2, 18)
    starts = np.cumsum((0,) + SEQS[:-1])
    got = _run(inp, SEQS, 0, rows=starts)
    v = _f64(inp["v"]).numpy()[starts]
    lam = inp["lam"].astype(np.float64)[starts]
    sig = 1.0 / (1.0 + np.exp(-_f64(inp["gate"]).numpy()[starts]))
    ref = sig * (1.0 - lam[..., None]) * np.repeat(v, G, axis=1)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-15)


def test_constant_values_closed_form():
    """All value rows of a sequence equal: every softmax average returns that row."""
    inp = _np_inputs((50,), 2, 19)
    inp["v"][:] = inp["v"][7]
    got = _run(inp, (50,), 0)
    v = _f64(inp["v"]).numpy()[0]
    lam = inp["lam"].astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(-_f64(inp["gate"]).numpy()))
    ref = sig * (1.0 - lam[..., None]) * np.repeat(v[None], 50, axis=0).repeat(G, axis=1)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_uniform_scores_give_running_mean():
    """Zero queries give equal scores, so H_t is the mean of v_0..v_t (per group)."""
    inp = _np_inputs((20,), 2, 20)
    inp["q_sig"][:] = 0
    inp["q_noise"][:] = 0
    got = _run(inp, (20,), 6)
    v = _f64(inp["v"]).numpy()
    lam = inp["lam"].astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(-_f64(inp["gate"]).numpy()))
    h = np.stack([v[max(0, t - 5):t + 1].mean(0) for t in range(20)])   # [20, 2, 128]
    ref = sig * (1.0 - lam[..., None]) * np.repeat(h, G, axis=1)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_group_permutation_equivariance():
    """Permuting KV groups (K_j, V_j, noise j, signal 4j..4j+3, their lambda and gate)
    permutes the output groups, bit for bit."""
    hkv = 4
    inp = _np_inputs(SEQS, hkv, 21)
    perm = np.array([2, 0, 3, 1])
    sig_perm = (perm[:, None] * G + np.arange(G)[None]).reshape(-1)
    pin = {
        "q_sig": inp["q_sig"][:, sig_perm].copy(), "q_noise": inp["q_noise"][:, perm].copy(),
        "k": inp["k"][:, perm].copy(), "v": inp["v"][:, perm].copy(),
        "lam": inp["lam"][:, sig_perm].copy(), "gate": inp["gate"][:, sig_perm].copy(),
    }
    assert np.array_equal(_run(pin, SEQS, 4), _run(inp, SEQS, 4)[:, sig_perm])


def test_sequences_are_independent():
    """A packed batch gives the same rows as each sequence run alone."""
    inp = _np_inputs(SEQS, 2, 22)
    packed = _run(inp, SEQS, 0)
    s0 = 0
    for length in SEQS:
        sub = {k: v[s0:s0 + length].copy() for k, v in inp.items()}
        assert np.array_equal(_run(sub, (length,), 0), packed[s0:s0 + length])
        s0 += length


def _brute_force(inp, seqlens, window):
    """Materialise the masked score matrix of each sequence and head (numpy, fp64)."""
    qs, qn, k, v = (_f64(inp[n]).numpy() for n in ("q_sig", "q_noise", "k", "v"))
    lam = inp["lam"].astype(np.float64)
    gate = _f64(inp["gate"]).numpy()
    n_tok, hs = lam.shape
    out = np.zeros((n_tok, hs, DV))
    s0 = 0
    for length in seqlens:
        sl = slice(s0, s0 + length)
        t = np.arange(length)[:, None]
        u = np.arange(length)[None, :]
        vis = (u <= t) if window <= 0 else ((u <= t) & (u > t - window))

        def head(q, j):
            s = q[sl] @ k[sl, j].T / math.sqrt(DQK)
            s = np.where(vis, s, -np.inf)
            p = np.exp(s - s.max(1, keepdims=True))
            return (p @ v[sl, j]) / p.sum(1, keepdims=True)

        for j in range(hs // G):
            hn = head(qn[:, j], j)
            for i in range(G):
                h = j * G + i
                d = head(qs[:, h], j) - lam[sl, h][:, None] * hn
                out[sl, h] = d / (1.0 + np.exp(-gate[sl, h]))
        s0 += length
    return out


@pytest.mark.parametrize("window", [0, 1, 9])
def test_brute_force_tiny(window):
    inp = _np_inputs(SEQS, 2, 23)
    np.testing.assert_allclose(_run(inp, SEQS, window), _brute_force(inp, SEQS, window), rtol=0, atol=1e-12)


def test_row_selection_matches_full_run():
    inp = _np_inputs(SEQS, 2, 24)
    full = _run(inp, SEQS, 7)
    rows = np.array([0, 36, 37, 38, 100, 107])
    assert np.array_equal(_run(inp, SEQS, 7, rows=rows), full[rows])


@pytest.mark.parametrize("window", [0, 2, 300])
def test_decode_equals_last_prefill_row(window):
    """Decode of sequence b (query at L_b - 1, cache holding it) is the last prefill row of b."""
    lens = (5, 1, 40)
    inp = _np_inputs(lens, 2, 25)
    last = np.cumsum(lens) - 1
    cu = np.concatenate([[0], np.cumsum(lens)])
    pre = _run(inp, lens, window, rows=last)
    dec = oracle.decode(inp["q_sig"][last], inp["q_noise"][last], inp["k"], inp["v"], cu,
                        inp["lam"][last], inp["gate"][last], window)
    assert np.array_equal(dec, pre)


def test_rejects_bad_arguments():
    inp = _np_inputs((4,), 1, 26)
    with pytest.raises(ValueError):
        _run(inp, (5,), 0)                      # seqlens disagree with tensors
    with pytest.raises(ValueError):
        _run(inp, (4,), 0, rows=[4])            # row out of range
    with pytest.raises(ValueError):
        oracle.decode(inp["q_sig"][:1], inp["q_noise"][:1], inp["k"], inp["v"], [0, 0],
                      inp["lam"][:1], inp["gate"][:1], 0)   # empty cache row set
