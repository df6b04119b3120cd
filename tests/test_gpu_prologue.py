"""GPU parity of gdla_prologue (through the C ABI) against the fp64 prologue oracle.

Tolerance per output: rel_rms <= 5e-3 and max_abs <= 2e-2 of the output's largest
magnitude. The path rounds the RMSNorm'd c^Q and c^KV to bf16 before their
up-projections and stores every output (but lambda) in bf16: about two bf16
roundings (2^-9 relative each).
"""
import numpy as np
import pytest
import torch

import differential_latent_attention_b200 as gdla
import gdla_inputs as gi
import oracle

pytestmark = pytest.mark.gpu

NAMES = ("q_sig", "q_noise", "k", "v", "lam", "gate")
WEIGHTS = ("w_qa", "w_kva", "gamma_q", "gamma_kv", "w_qb", "w_uk", "w_uv", "w_lambda", "w_gate")


def _host(t):
    return gi.bf16_bits(t) if t.dtype == torch.bfloat16 else t.cpu().numpy()


def check_prologue(seqlens, hkv, seed):
    t = gi.make_prologue_inputs(seqlens, hkv, seed, device="cuda")
    got = gdla.prologue(t["x"], *[t[w] for w in WEIGHTS], seqlens)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    check_prologue_outputs(t, got, seqlens)


def check_prologue_outputs(t, got, seqlens):
    hkv = t["w_uk"].shape[0]
    ref = oracle.prologue(_host(t["x"]), *[_host(t[w]) for w in WEIGHTS], seqlens)
    report = {}
    for name in NAMES:
        g = got[name].float().cpu().numpy().astype(np.float64)
        r = ref[name]
        assert g.shape == r.shape, name
        d = g - r
        report[name] = (float(np.abs(d).max() / np.abs(r).max()), float(np.linalg.norm(d) / np.linalg.norm(r)))
    print(f"prologue seqlens={seqlens} hkv={hkv}: " + " ".join(f"{n}=({m:.1e},{e:.1e})" for n, (m, e) in report.items()))
    for name, (mx, rel) in report.items():
        assert rel <= 5e-3 and mx <= 2e-2, (name, mx, rel)


def test_small():
    check_prologue((37,), 1, 1)


def test_ragged_batch():
    check_prologue((5, 0, 130, 64), 2, 2)


def test_long_positions():
    check_prologue((2000,), 2, 3)


def test_sixteen_groups():
    check_prologue((300, 77), 16, 4)


def test_three_groups():
    # 4H = 12 lambda columns (one partly filled 64-column tile), 15 query heads
    check_prologue((129, 258), 3, 6)


def test_bench_size():
    # the bench's prologue workload in full: 4096 tokens, 16 KV groups (every output element)
    check_prologue((4096,), 16, 1)


def test_feeds_attention():
    """The prologue's outputs are accepted by attn_fwd as they are."""
    seqlens = (200,)
    t = gi.make_prologue_inputs(seqlens, 2, 5, device="cuda")
    o = gdla.prologue(t["x"], *[t[w] for w in WEIGHTS], seqlens)
    out = gdla.attn_fwd(o["q_sig"], o["q_noise"], o["k"], o["v"], o["lam"], o["gate"], seqlens, 0)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert gdla.device_error() == 0


def test_zero_hidden_state():
    """x = 0 (tokens 0 and 100 of two sequences zeroed, the rest random): those rows'
    projections vanish, RMSNorm of a zero vector is zero (no division by zero), the
    rotary part of zero stays zero, lambda = sigmoid(0) = 1/2, and the gate
    logits are zero; the other rows still match the oracle."""
    seqlens = (40, 90)
    t = gi.make_prologue_inputs(seqlens, 2, 8, device="cuda")
    zero_rows = [0, 40 + 60]
    t["x"][zero_rows] = 0
    o = gdla.prologue(t["x"], *[t[w] for w in WEIGHTS], seqlens)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    for name in ("q_sig", "q_noise", "k", "v", "gate"):
        assert torch.count_nonzero(o[name][zero_rows].float()).item() == 0, name
    assert float((o["lam"][zero_rows] - 0.5).abs().max()) <= 1e-6
    check_prologue_outputs(t, o, seqlens)
