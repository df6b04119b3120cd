"""Pin of the latent-cache decode oracle against the expanded decode oracle.

The compressed KV cache holds one row per token, c (512) and a rotary key kr
(64) shared by every KV head; KV head j is the up-projection
K_j = [W^UK_j c | kr], V_j = W^UV_j c. With the query's non-rotary part
absorbed (q_abs = [W^UK_j^T q_nope | q_rope]) the scores and outputs are the
same numbers computed in another order. The inputs here are small integers and
sparse +-1 projections, so every expanded and absorbed tensor is exact in bf16
and the two independent fp64 computations must agree to rounding. Slips planted in
copies of the latent oracle's own code must each break that agreement.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

DC, DR, DV, DQK, GROUP = 512, 64, 128, 192, 4


def _bits(x):
    """bf16 bit patterns of values that are exact in bf16."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), f), "value not exact in bf16"
    return bits


def _sparse_pm1(rng, rows, cols, per_row=2):
    w = np.zeros((rows, cols))
    for r in range(rows):
        w[r, rng.choice(cols, per_row, replace=False)] = rng.choice([-1.0, 1.0], per_row)
    return w


def _case(seed, lengths, hkv):
    rng = np.random.default_rng(seed)
    b, nk, hs = len(lengths), int(sum(lengths)), GROUP * hkv
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    c = rng.integers(-1, 2, (nk, DC)).astype(np.float64)
    kr = rng.integers(-1, 2, (nk, DR)).astype(np.float64)
    w_uk = np.stack([_sparse_pm1(rng, DV, DC) for _ in range(hkv)])   # [H, 128, 512]
    w_uv = np.stack([_sparse_pm1(rng, DV, DC) for _ in range(hkv)])
    q_nope_s = rng.integers(-1, 2, (b, hs, DV)).astype(np.float64)
    q_rope_s = rng.integers(-1, 2, (b, hs, DR)).astype(np.float64)
    q_nope_n = rng.integers(-1, 2, (b, hkv, DV)).astype(np.float64)
    q_rope_n = rng.integers(-1, 2, (b, hkv, DR)).astype(np.float64)
    lam = ((rng.integers(0, 1 << 24, (b, hs)) + 0.5) / (1 << 24)).astype(np.float32)
    gate = rng.integers(-8, 9, (b, hs, DV)) / 4.0
    return dict(cu=cu, c=c, kr=kr, w_uk=w_uk, w_uv=w_uv, q_nope_s=q_nope_s, q_rope_s=q_rope_s,
                q_nope_n=q_nope_n, q_rope_n=q_rope_n, lam=lam, gate=gate, hkv=hkv)


def _expanded(x, window):
    hkv = x["hkv"]
    k = np.concatenate([np.einsum("jde,ue->ujd", x["w_uk"], x["c"]),
                        np.repeat(x["kr"][:, None, :], hkv, axis=1)], axis=2)       # [Nk, H, 192]
    v = np.einsum("jde,ue->ujd", x["w_uv"], x["c"])                                  # [Nk, H, 128]
    q_sig = np.concatenate([x["q_nope_s"], x["q_rope_s"]], axis=2)
    q_noise = np.concatenate([x["q_nope_n"], x["q_rope_n"]], axis=2)
    return oracle.decode(_bits(q_sig), _bits(q_noise), _bits(k), _bits(v), x["cu"], x["lam"], _bits(x["gate"]),
                         window)


def _absorbed(x, window, w_uv=None, drop_rope=False, wrong_group=False):
    hkv = x["hkv"]
    group = np.arange(GROUP * hkv) // GROUP
    if wrong_group:
        group = (group + 1) % hkv
    q_abs_sig = np.concatenate([np.einsum("hde,bhd->bhe", x["w_uk"][group], x["q_nope_s"]),
                                0 * x["q_rope_s"] if drop_rope else x["q_rope_s"]], axis=2)
    q_abs_noise = np.concatenate([np.einsum("jde,bjd->bje", x["w_uk"], x["q_nope_n"]), x["q_rope_n"]], axis=2)
    ckv = np.concatenate([x["c"], x["kr"]], axis=1)
    return oracle.decode_latent(_bits(q_abs_sig), _bits(q_abs_noise), _bits(ckv), x["cu"],
                                _bits(x["w_uv"] if w_uv is None else w_uv), x["lam"], _bits(x["gate"]), window)


@pytest.mark.parametrize("window", [0, 1, 16])
def test_absorbed_latent_decode_equals_expanded_decode(window):
    x = _case(90 + window, (1, 7, 40, 129), 2)
    ref = _expanded(x, window)
    got = _absorbed(x, window)
    assert np.abs(ref).max() > 0.1
    assert np.abs(got - ref).max() <= 1e-12


@pytest.mark.parametrize("slip", ["w_uk_for_w_uv", "transposed_groups", "rope_dropped"])
def test_plausible_slips_break_the_equivalence(slip):
    x = _case(99, (7, 40, 129), 2)
    ref = _expanded(x, 0)
    if slip == "w_uk_for_w_uv":
        got = _absorbed(x, 0, w_uv=x["w_uk"])
    elif slip == "transposed_groups":
        got = _absorbed(x, 0, wrong_group=True)
    else:
        got = _absorbed(x, 0, drop_rope=True)
    assert np.abs(got - ref).max() > 1e-3


# Planted slips inside the latent oracle itself: each is a copy of the oracle source
# with one plausible mistake in the latent path (scale, rotary dims, value slice,
# W^UV layout or group, noise-head index, window edge, subtract sign, normalisation),
# built on the CPU; the expanded decode (untouched code) must then disagree.
LATENT_MUTANTS = {
    "scale_dropped": ("for (int e = 0; e < DL; ++e) s += qd[e] * bf16_to_double(r[e]);\n        s = s / root;",
                      "for (int e = 0; e < DL; ++e) s += qd[e] * bf16_to_double(r[e]);"),
    "rope_dims_dropped": ("for (int e = 0; e < DL; ++e) s += qd[e] * bf16_to_double(r[e]);",
                          "for (int e = 0; e < DC; ++e) s += qd[e] * bf16_to_double(r[e]);"),
    "values_from_wrong_slice": ("for (int e = 0; e < DC; ++e) o[e] += w * bf16_to_double(r[e]);",
                                "for (int e = 0; e < DC; ++e) o[e] += w * bf16_to_double(r[e + DR]);"),
    "up_projection_transposed": ("bf16_to_double(w_uv_j[(long)d * DC + e])", "bf16_to_double(w_uv_j[(long)e * DV + d])"),
    "noise_group_index": ("attend_latent(J->q_noise + (b * J->hkv + j) * DL,",
                          "attend_latent(J->q_noise + (b * J->hkv + (J->hkv - 1 - j)) * DL,"),
    "w_uv_group_dropped": ("const uint16_t *w_uv_j = J->w_uv + (long)j * DV * DC;", "const uint16_t *w_uv_j = J->w_uv;"),
    "window_off_by_one": ("if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;\n"
                          "        const long nkeys = (long)(t - lo + 1);\n        const uint16_t *rows = J->ckv",
                          "if (J->window > 0 && t - J->window + 2 > 0) lo = t - J->window + 2;\n"
                          "        const long nkeys = (long)(t - lo + 1);\n        const uint16_t *rows = J->ckv"),
    "subtract_sign": ("const double dd = hsig[d] - l * hn[d];", "const double dd = hsig[d] + l * hn[d];"),
    "normalisation_dropped": ("for (int e = 0; e < DC; ++e) o[e] /= den;", ""),
}
MUTANT_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "_build", "oracle_mutants")


def _build_latent_mutant(name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdla_oracle.c")).read()
    assert src.count(old) == 1, name
    os.makedirs(MUTANT_DIR, exist_ok=True)
    c = os.path.join(MUTANT_DIR, f"latent_{name}.c")
    so = os.path.join(MUTANT_DIR, f"liblatent_{name}.so")
    with open(c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", so, c, "-lm"],
                          env={**os.environ, "TMPDIR": MUTANT_DIR})
    lib = ctypes.CDLL(so)
    real = oracle._load()
    for fn in ("gdla_oracle_decode", "gdla_oracle_decode_latent"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    return lib


@pytest.mark.parametrize("name", sorted(LATENT_MUTANTS))
def test_planted_latent_slip_is_caught(name, monkeypatch):
    lib = _build_latent_mutant(name, *LATENT_MUTANTS[name])
    worst = 0.0
    for window in (0, 16):
        x = _case(95 + window, (1, 7, 40, 129), 2)
        ref = _expanded(x, window)               # the unmodified expanded decode
        monkeypatch.setattr(oracle, "_lib", lib)
        got = _absorbed(x, window)               # the mutant's latent path
        monkeypatch.undo()
        worst = max(worst, float(np.abs(got - ref).max()))
    assert worst > 1e-6, f"mutant {name} not caught (worst {worst:.2e})"
