"""Pins of the fp64 prologue oracle (``oracle.prologue``): the projections that make
the attention's inputs from the hidden state.

* against a composition of library routines in fp64: torch's linear and rms_norm and
  the rotary embedding of the transformers library (rotate-half, base 10000), on a
  ragged batch (positions restart per sequence);
* closed forms of the rotary embedding (unit vectors, position 0) and its
  relative-position property; RMSNorm's scale invariance;
* planted slips in the oracle (each a substituted function) must fail the first pin.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

H = 2                         # KV groups (small, for speed); the kernels take 16
HS, HQ = 4 * H, 5 * H
HIDDEN, QR, DC, DR = oracle.HIDDEN, oracle.Q_RANK, oracle.DC, oracle.DR


def _weights(seed):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, scale: (torch.randn(*s, generator=g, dtype=torch.float64) * scale)
    return {
        "w_qa": r(QR, HIDDEN, scale=HIDDEN ** -0.5), "w_kva": r(DC + DR, HIDDEN, scale=HIDDEN ** -0.5),
        "gamma_q": 1 + 0.1 * r(QR, scale=1.0), "gamma_kv": 1 + 0.1 * r(DC, scale=1.0),
        "w_qb": r(HQ * 192, QR, scale=QR ** -0.5), "w_uk": r(H, 128, DC, scale=DC ** -0.5),
        "w_uv": r(H, 128, DC, scale=DC ** -0.5), "w_lambda": r(HS, HIDDEN, scale=HIDDEN ** -0.5),
        "w_gate": r(HS * 128, HIDDEN, scale=HIDDEN ** -0.5)}


def library_prologue(x, w, seqlens):
    """The same projections from library routines (fp64)."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    cfg = LlamaConfig(hidden_size=64 * 4, num_attention_heads=4, head_dim=64, rope_theta=10000.0,
                      max_position_embeddings=1 << 16)
    rot = LlamaRotaryEmbedding(cfg)
    n = x.shape[0]
    pos = torch.cat([torch.arange(int(L)) for L in seqlens])[None]
    cos, sin = rot(x[None, None, :, :64], pos)                                   # [1, N, 64]
    cq = F.rms_norm(F.linear(x, w["w_qa"]), (QR,), w["gamma_q"], eps=1e-6)
    ckv_full = F.linear(x, w["w_kva"])
    ckv = F.rms_norm(ckv_full[:, :DC], (DC,), w["gamma_kv"], eps=1e-6)
    q = F.linear(cq, w["w_qb"]).reshape(n, HQ, 192)
    q_rope, _ = apply_rotary_pos_emb(q[None, :, :, 128:].transpose(1, 2), q[None, :, :, 128:].transpose(1, 2),
                                     cos, sin)                                  # [1, HQ, N, 64]
    q = torch.cat([q[..., :128], q_rope[0].transpose(0, 1)], -1)
    kr, _ = apply_rotary_pos_emb(ckv_full[None, None, :, DC:], ckv_full[None, None, :, DC:], cos, sin)
    k_nope = torch.stack([F.linear(ckv, w["w_uk"][j]) for j in range(H)], 1)
    v = torch.stack([F.linear(ckv, w["w_uv"][j]) for j in range(H)], 1)
    k = torch.cat([k_nope, kr[0, 0][:, None, :].expand(n, H, 64)], -1)
    lam = torch.sigmoid(F.linear(x, w["w_lambda"]))
    gate = F.linear(x, w["w_gate"]).reshape(n, HS, 128)
    return {"q_sig": q[:, :HS], "q_noise": q[:, HS:], "k": k, "v": v, "lam": lam, "gate": gate}


SEQLENS = (5, 0, 9, 3)


def _run_oracle(x, w):
    return oracle.prologue(x.numpy(), w["w_qa"].numpy(), w["w_kva"].numpy(), w["gamma_q"].numpy(),
                           w["gamma_kv"].numpy(), w["w_qb"].numpy(), w["w_uk"].numpy(), w["w_uv"].numpy(),
                           w["w_lambda"].numpy(), w["w_gate"].numpy(), SEQLENS)


def _worst(got, ref):
    return max(float(np.abs(got[n] - ref[n].numpy()).max() / max(np.abs(ref[n].numpy()).max(), 1e-30)) for n in ref)


def test_prologue_matches_library_composition():
    w = _weights(1)
    x = torch.randn(sum(SEQLENS), HIDDEN, generator=torch.Generator().manual_seed(2), dtype=torch.float64)
    ref = library_prologue(x, w, SEQLENS)
    got = _run_oracle(x, w)
    for name in ref:
        assert got[name].shape == tuple(ref[name].shape), name
    # the library rotary tables are computed in fp32
    assert _worst(got, ref) < 1e-5


def test_rope_closed_forms_and_relative_position():
    e = np.eye(64)
    for p in (0, 1, 7):
        out = oracle.rope(e[[0, 1, 33]], np.array([p, p, p]))
        f1 = 10000.0 ** (-1 / 32)
        assert np.allclose(out[0, [0, 32]], [np.cos(p), np.sin(p)], atol=1e-15)
        assert np.allclose(out[1, [1, 33]], [np.cos(p * f1), np.sin(p * f1)], atol=1e-15)
        assert np.allclose(out[2, [1, 33]], [-np.sin(p * f1), np.cos(p * f1)], atol=1e-15)
    rng = np.random.default_rng(0)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    d1 = oracle.rope(q[None], [13])[0] @ oracle.rope(k[None], [5])[0]
    d2 = oracle.rope(q[None], [8])[0] @ k
    assert abs(d1 - d2) < 1e-12
    assert np.allclose(np.linalg.norm(oracle.rope(q[None], [123])), np.linalg.norm(q))


def test_rms_norm_scale_invariance():
    rng = np.random.default_rng(1)
    c = rng.standard_normal((3, 512))
    g = rng.standard_normal(512)
    assert np.allclose(oracle.rms_norm(c * 7.5, g), oracle.rms_norm(c, g), rtol=1e-6)  # up to eps / (2 mean c^2)
    assert np.allclose(np.sqrt(np.mean(oracle.rms_norm(c, np.ones(512)) ** 2, -1)), 1.0, rtol=1e-5)


def _rope_pairs_adjacent(xr, positions):
    xr = np.asarray(xr, dtype=np.float64)
    half = xr.shape[-1] // 2
    inv = oracle.ROPE_BASE ** (-np.arange(half) / half)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    shape = (ang.shape[0],) + (1,) * (xr.ndim - 2) + (half,)
    cos, sin = np.cos(ang).reshape(shape), np.sin(ang).reshape(shape)
    a, b = xr[..., 0::2], xr[..., 1::2]
    out = np.empty_like(xr)
    out[..., 0::2], out[..., 1::2] = a * cos - b * sin, a * sin + b * cos
    return out


MUTANTS = {
    "rope_adjacent_pairs": ("rope", _rope_pairs_adjacent),
    "rope_base_1e4_over_64": ("ROPE_BASE", 100000.0),
    "rms_without_gamma": ("rms_norm", None),
    "rms_eps_large": ("RMS_EPS", 1e-1),
    "positions_not_restarted": ("positions_of", lambda s: np.arange(int(sum(s)), dtype=np.int64)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_prologue_slip_is_caught(name, monkeypatch):
    attr, val = MUTANTS[name]
    if name == "rms_without_gamma":
        orig = oracle.rms_norm
        val = lambda c, g: orig(c, np.ones_like(np.asarray(g)))
    monkeypatch.setattr(oracle, attr, val)
    w = _weights(3)
    x = torch.randn(sum(SEQLENS), HIDDEN, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
    ref = library_prologue(x, w, SEQLENS)
    got = _run_oracle(x, w)
    assert _worst(got, ref) > 1e-3, f"mutant {name} not caught"


# Slips inside the body of oracle.prologue: each is a copy of its source with one
# substitution, compiled in the oracle module's namespace.
BODY_MUTANTS = {
    "rope_on_content_dims": ("np.concatenate([q[..., :DQK - ROPE], rope(q[..., DQK - ROPE:], pos)], axis=-1)",
                             "np.concatenate([rope(q[..., :ROPE], pos), q[..., ROPE:]], axis=-1)"),
    "k_rope_from_latent_dims": ("k_rope = rope(ckv_full[:, DC:], pos)", "k_rope = rope(ckv_full[:, :ROPE], pos)"),
    "w_uk_and_w_uv_swapped": ('k_nope = np.einsum("nc,hdc->nhd", ckv, _f64(w_uk))',
                              'k_nope = np.einsum("nc,hdc->nhd", ckv, _f64(w_uv))'),
    "lambda_without_sigmoid": ("lam = 1.0 / (1.0 + np.exp(-(x @ _f64(w_lambda).T)))", "lam = x @ _f64(w_lambda).T"),
    "noise_heads_first": ('{"q_sig": q[:, :hs], "q_noise": q[:, hs:]', '{"q_sig": q[:, hkv:], "q_noise": q[:, :hkv]'),
    "c_q_not_normalised": ("cq = rms_norm(x @ _f64(w_qa).T, gamma_q)", "cq = (x @ _f64(w_qa).T) * gamma_q"),
    "k_rope_not_rotated": ("k_rope = rope(ckv_full[:, DC:], pos)", "k_rope = ckv_full[:, DC:]"),
}


@pytest.mark.parametrize("name", sorted(BODY_MUTANTS))
def test_planted_slip_in_the_prologue_body_is_caught(name, monkeypatch):
    import inspect
    import textwrap
    old, new = BODY_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(oracle.prologue))
    assert src.count(old) == 1, name
    scope = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), scope)
    monkeypatch.setattr(oracle, "prologue", scope["prologue"])
    w = _weights(3)
    x = torch.randn(sum(SEQLENS), HIDDEN, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
    ref = library_prologue(x, w, SEQLENS)
    got = _run_oracle(x, w)
    assert _worst(got, ref) > 1e-3, f"mutant {name} not caught"
