"""GPU parity of gdla_attn_bwd (through the C ABI) against the fp64 backward oracle.

Tolerance (per gradient, over all elements): rel_rms <= 5e-3 (the forward's bar)
and max_abs <= 2e-2 of the gradient's largest magnitude. The backward multiplies bf16 operands the
forward does not have - dH (= dout sigma(g)), P and dS = P (dP - rowsum(dH H))
are each rounded to bf16 before a tensor-core product, and every gradient is
stored in bf16 - so each gradient carries about three bf16 roundings (2^-9
relative each, ~1.1e-3 rms) instead of the forward's one or two; dS further
loses relative precision where dP and rowsum(dH H) nearly cancel.
"""
import numpy as np
import pytest
import torch

import differential_latent_attention_b200 as gdla
import gdla_inputs as gi
import oracle

pytestmark = pytest.mark.gpu

NAMES = ("dq_sig", "dq_noise", "dk", "dv", "dlambda", "dgate")


def _run(seqlens, hkv, window, seed):
    t = gi.make_prefill_inputs(seqlens, hkv, seed, device="cuda")
    dout = gi.make_prefill_grad(seqlens, hkv, seed, device="cuda")
    g = gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, seqlens, window)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    ref = oracle.prefill_bwd(*[gi.bf16_bits(t[n]) for n in ("q_sig", "q_noise", "k", "v")], t["lam"].cpu().numpy(),
                             gi.bf16_bits(t["gate"]), gi.bf16_bits(dout), seqlens, window)
    return g, ref


def _errors(got, ref):
    got = got.float().cpu().numpy().astype(np.float64)
    d = got - ref
    scale = max(float(np.abs(ref).max()), 1e-30)
    return float(np.abs(d).max()) / scale, float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))


def check_bwd(seqlens, hkv, window, seed, rel_tol=5e-3, max_tol=2e-2):
    g, ref = _run(seqlens, hkv, window, seed)
    report = {}
    for name in NAMES:
        mx, rel = _errors(g[name], ref[name])
        report[name] = (mx, rel)
        assert np.isfinite(g[name].float().cpu().numpy()).all(), name
    print(f"bwd seqlens={seqlens} hkv={hkv} window={window}: " +
          " ".join(f"{n}=({m:.1e},{r:.1e})" for n, (m, r) in report.items()))
    for name, (mx, rel) in report.items():
        assert rel <= rel_tol and mx <= max_tol, (name, mx, rel)


def test_tiny_full():
    check_bwd((37,), 1, 0, 1)


@pytest.mark.parametrize("window", [0, 4, 128])
def test_ragged(window):
    check_bwd((9, 0, 23, 1, 130, 64), 2, window, 2 + window)


def test_several_tiles_and_ragged_tail():
    # 700 tokens: 6 key tiles of 128 (ragged last), 30 q tiles (ragged last), 59 steps of 12 tokens
    check_bwd((700,), 2, 0, 3)
    check_bwd((700,), 2, 128, 4)


@pytest.mark.parametrize("window", [200, 256, 300])
def test_window_schedules(window):
    # windows up to 256 recompute on the sliding schedule (48-token items, 64-key tiles),
    # longer ones on the one-tile schedule (24-token items, 128-key tiles)
    check_bwd((700, 333), 2, window, 10 + window)


def test_sixteen_groups():
    check_bwd((300, 77), 16, 0, 5)


@pytest.mark.parametrize("w", [gi.PREFILL_FULL, gi.SWA], ids=lambda w: w.name)
def test_bench_workload_two_groups(w):
    """The bench's own backward workloads in its launch (T = 4096 full causal, and 2 x 32768 at
    window 128, all 16 KV groups in one call). A group's gradients depend on its own five heads,
    K and V only, so the oracle checks the first and the last group, each as a one-group problem."""
    t = gi.make_prefill_inputs(w.seqlens, w.num_kv_heads, w.seed, device="cuda")
    dout = gi.make_prefill_grad(w.seqlens, w.num_kv_heads, w.seed, device="cuda")
    g = gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, w.seqlens, w.window)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    for j in (0, w.num_kv_heads - 1):
        sig, noi = slice(4 * j, 4 * j + 4), slice(j, j + 1)
        ref = oracle.prefill_bwd(gi.bf16_bits(t["q_sig"][:, sig]), gi.bf16_bits(t["q_noise"][:, noi]),
                                 gi.bf16_bits(t["k"][:, noi]), gi.bf16_bits(t["v"][:, noi]),
                                 t["lam"][:, sig].cpu().numpy(), gi.bf16_bits(t["gate"][:, sig]),
                                 gi.bf16_bits(dout[:, sig]), w.seqlens, w.window)
        got = {"dq_sig": g["dq_sig"][:, sig], "dq_noise": g["dq_noise"][:, noi], "dk": g["dk"][:, noi],
               "dv": g["dv"][:, noi], "dlambda": g["dlambda"][:, sig], "dgate": g["dgate"][:, sig]}
        report = {name: _errors(got[name], ref[name]) for name in NAMES}
        print(f"bwd {w.name} group {j}: " + " ".join(f"{n}=({m:.1e},{r:.1e})" for n, (m, r) in report.items()))
        for name, (mx, rel) in report.items():
            assert rel <= 5e-3 and mx <= 2e-2, (j, name, mx, rel)


def test_deterministic():
    seqlens, hkv = (200, 61), 2
    t = gi.make_prefill_inputs(seqlens, hkv, 9, device="cuda")
    dout = gi.make_prefill_grad(seqlens, hkv, 9, device="cuda")
    a = gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, seqlens, 0)
    ws = torch.full((gdla.attn_bwd_workspace_bytes(sum(seqlens), hkv),), 0xFF, dtype=torch.uint8, device="cuda")
    b = gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, seqlens, 0, workspace=ws)
    torch.cuda.synchronize()
    for name in NAMES:
        assert torch.equal(a[name], b[name]), name


def test_window_one_closed_form():
    """Window 1: every token attends only to itself (P = 1), so with s = sigmoid(g),
    D_i = (1 - lambda_i) v and dD_i = dout_i s_i:
        dgate_i = dout_i D_i s_i (1 - s_i),  dlambda_i = -sum_d dD_i v,
        dv = sum_i (1 - lambda_i) dD_i,  and dq, dk vanish (dS = P (dP - rowsum) = 0).
    The GPU gradients against those closed forms in fp64, not against the oracle."""
    seqlens = (37, 1, 130, 24)
    hkv = 2
    t = gi.make_prefill_inputs(seqlens, hkv, 41, device="cuda")
    dout = gi.make_prefill_grad(seqlens, hkv, 41, device="cuda")
    g = gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, seqlens, 1)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    s = torch.sigmoid(t["gate"].double().cpu())                              # [N, 4H, 128]
    lam = t["lam"].double().cpu()[..., None]                                 # [N, 4H, 1]
    v = t["v"].double().cpu().repeat_interleave(4, dim=1)                    # [N, 4H, 128]
    go = dout.double().cpu()
    dd = go * s
    ref = {"dgate": go * (1.0 - lam) * v * s * (1.0 - s),
           "dlambda": -(dd * v).sum(-1),
           "dv": ((1.0 - lam) * dd).reshape(-1, hkv, 4, 128).sum(2)}
    for name, r in ref.items():
        mx, rel = _errors(g[name], r.numpy())
        assert rel <= 5e-3 and mx <= 2e-2, (name, mx, rel)
    scale = float(g["dv"].float().abs().max())
    for name in ("dq_sig", "dq_noise", "dk"):
        assert float(g[name].float().abs().max()) <= 1e-3 * scale, name


def _permute_groups(x, perm, per_group):
    """Reorder the KV-group blocks (of `per_group` heads each) along dim 1."""
    n = x.shape[0]
    blocks = x.reshape(n, len(perm), per_group, *x.shape[2:])
    return blocks[:, list(perm)].reshape(x.shape).contiguous()


def test_group_permutation_and_long_window_bitwise():
    """Permuting the KV groups of every input permutes every gradient's groups bit for
    bit, and a window no shorter than the sequences gives the full-causal gradients bit
    for bit (the groups are independent and the masks drop nothing)."""
    seqlens = (300, 77, 1)
    hkv, perm = 3, (2, 0, 1)
    t = gi.make_prefill_inputs(seqlens, hkv, 43, device="cuda")
    dout = gi.make_prefill_grad(seqlens, hkv, 43, device="cuda")
    a = gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, seqlens, 0)
    sig = lambda x: _permute_groups(x, perm, 4)
    one = lambda x: _permute_groups(x, perm, 1)
    b = gdla.attn_bwd(sig(t["q_sig"]), one(t["q_noise"]), one(t["k"]), one(t["v"]), sig(t["lam"]),
                      sig(t["gate"]), sig(dout), seqlens, 0)
    c = gdla.attn_bwd(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], dout, seqlens, 4096)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    for name in NAMES:
        per = 1 if name in ("dq_noise", "dk", "dv") else 4
        assert torch.equal(_permute_groups(a[name], perm, per), b[name]), name
        assert torch.equal(a[name], c[name]), name
