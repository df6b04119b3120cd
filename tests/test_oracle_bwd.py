"""Pins of the fp64 backward oracle (``oracle.prefill_bwd``).

The backward is pinned to automatic differentiation: the GDLA forward is composed
from library operations in fp64 (torch's scaled-dot-product attention per head,
then the subtract and the sigmoid gate), torch autograd differentiates
sum(dout * out), and every gradient the oracle returns must match to ~1e-12
relative. The composition is checked against the forward oracle first, so the
autograd reference and the oracle see the same function. Planted slips in the
oracle's backward (each a copy of the source with one plausible mistake, built on
the CPU) must each fail the pin.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import gdla_inputs as gi
import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdla_oracle.c")
MUTANT_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "_build", "oracle_mutants")


def _as64(t):
    return t.to(torch.float64)


def torch_forward(q_sig, q_noise, k, v, lam, gate, seqlens, window):
    """GDLA forward from library ops in fp64 (differentiable): per sequence and group,
    SDPA of the 4 signal heads and the noise head over the shared K_j, V_j with a
    causal (windowed) boolean mask, then sigmoid(gate) * (H_S - lambda H_N)."""
    hkv = q_noise.shape[1]
    outs = []
    s0 = 0
    for L in seqlens:
        L = int(L)
        if L == 0:
            continue
        t = torch.arange(L)
        vis = t[None, :] <= t[:, None]
        if window > 0:
            vis &= t[None, :] > t[:, None] - window
        sl = slice(s0, s0 + L)
        per_group = []
        for j in range(hkv):
            qs = q_sig[sl, 4 * j:4 * j + 4].permute(1, 0, 2)          # [4, L, 192]
            qn = q_noise[sl, j:j + 1].permute(1, 0, 2)                 # [1, L, 192]
            kj = k[sl, j].unsqueeze(0)
            vj = v[sl, j].unsqueeze(0)
            q5 = torch.cat([qs, qn], 0)                                 # [5, L, 192]
            h = torch.nn.functional.scaled_dot_product_attention(
                q5, kj.expand(5, L, -1), vj.expand(5, L, -1), attn_mask=vis, scale=1.0 / np.sqrt(192.0))
            hs_, hn = h[:4], h[4:5]                                     # [4, L, 128], [1, L, 128]
            lam_j = lam[sl, 4 * j:4 * j + 4].permute(1, 0).unsqueeze(-1)  # [4, L, 1]
            d = hs_ - lam_j * hn
            g = gate[sl, 4 * j:4 * j + 4].permute(1, 0, 2)
            per_group.append((torch.sigmoid(g) * d).permute(1, 0, 2))   # [L, 4, 128]
        outs.append(torch.cat(per_group, 1))
        s0 += L
    return torch.cat(outs, 0)


def autograd_reference(inp, dout, seqlens, window):
    leaves = {name: _as64(inp[name]).clone().requires_grad_(True)
              for name in ("q_sig", "q_noise", "k", "v", "lam", "gate")}
    out = torch_forward(leaves["q_sig"], leaves["q_noise"], leaves["k"], leaves["v"], leaves["lam"],
                        leaves["gate"], seqlens, window)
    (out * _as64(dout)).sum().backward()
    return out.detach().numpy(), {
        "dq_sig": leaves["q_sig"].grad.numpy(), "dq_noise": leaves["q_noise"].grad.numpy(),
        "dk": leaves["k"].grad.numpy(), "dv": leaves["v"].grad.numpy(),
        "dlambda": leaves["lam"].grad.numpy(), "dgate": leaves["gate"].grad.numpy()}


def oracle_grads(inp, dout, seqlens, window, fn=None):
    bits = [gi.bf16_bits(inp[n]) for n in ("q_sig", "q_noise", "k", "v")]
    args = bits + [inp["lam"].numpy(), gi.bf16_bits(inp["gate"]), gi.bf16_bits(dout), seqlens, window]
    return (fn or oracle.prefill_bwd)(*args)


CASES = [((37,), 1, 0), ((37,), 1, 5), ((9, 0, 23, 1), 2, 0), ((9, 0, 23, 1), 2, 4), ((30,), 3, 1)]


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("seqlens,hkv,window", CASES)
def test_backward_matches_autograd(seqlens, hkv, window):
    inp = gi.make_prefill_inputs(seqlens, hkv, 11 + hkv + window)
    dout = gi.make_prefill_grad(seqlens, hkv, 11 + hkv + window)
    out_t, ref = autograd_reference(inp, dout, seqlens, window)
    # the composition is the forward oracle's function
    fwd = oracle.prefill(*[gi.bf16_bits(inp[n]) for n in ("q_sig", "q_noise", "k", "v")], inp["lam"].numpy(),
                         gi.bf16_bits(inp["gate"]), seqlens, window)
    assert _rel(fwd, out_t) < 1e-12
    got = oracle_grads(inp, dout, seqlens, window)
    for name, r in ref.items():
        assert got[name].shape == r.shape, name
        assert _rel(got[name], r) < 1e-11, (name, _rel(got[name], r))


def test_gradient_of_a_masked_key_is_zero_for_rows_that_cannot_see_it():
    """The last key of a sequence is seen only by the last query row: zeroing the
    output gradient of that row leaves dk, dv of the key exactly zero."""
    seqlens = (12,)
    inp = gi.make_prefill_inputs(seqlens, 1, 5)
    dout = gi.make_prefill_grad(seqlens, 1, 5)
    dout[-1] = 0
    g = oracle_grads(inp, dout, seqlens, 0)
    assert np.all(g["dk"][-1] == 0) and np.all(g["dv"][-1] == 0)
    assert np.any(g["dk"][-2] != 0)


BWD_MUTANTS = {
    "drow_dropped": ("const double ds = p[u] * (dp[u] - drow);", "const double ds = p[u] * dp[u];"),
    "dlambda_sign": ("dl -= ddd * hh[GROUP][d];", "dl += ddd * hh[GROUP][d];"),
    "dnoise_without_lambda": ("dh[GROUP][d] -= l * ddd;", "dh[GROUP][d] -= ddd;"),
    "dgate_without_sigma_prime": ("go * dd * sg * (1.0 - sg)", "go * dd * sg"),
    "dk_unscaled": ("dkr[d] += ds * bf16_to_double(q[d]) / root;", "dkr[d] += ds * bf16_to_double(q[d]);"),
    "dq_unscaled": ("dq[d] += ds * bf16_to_double(kr[d]) / root;", "dq[d] += ds * bf16_to_double(kr[d]);"),
    "window_off_by_one": ("if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;\n"
                          "            const long nkeys = t - lo + 1;",
                          "if (J->window > 0 && t - J->window + 2 > 0) lo = t - J->window + 2;\n"
                          "            const long nkeys = t - lo + 1;"),
    "gate_sign": ("const double sg = 1.0 / (1.0 + exp(-g));", "const double sg = 1.0 / (1.0 + exp(g));"),
    "dD_without_gate": ("const double ddd = go * sg;", "const double ddd = go;"),
    "dv_from_wrong_head": ("for (int d = 0; d < DV; ++d) dvr[d] += p[u] * dh[d];",
                           "for (int d = 0; d < DV; ++d) dvr[d] += p[u] * dh[d] * (dq == J_unused ? 0 : 1);"),
}


def _build_bwd_mutant(name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    src = src.replace(old, new)
    if "J_unused" in new:  # a head-selection slip: dv accumulates only the signal heads
        src = src.replace(new, "for (int d = 0; d < DV; ++d) dvr[d] += p[u] * dh[d] * (is_noise ? 0.0 : 1.0);")
        src = src.replace("static void head_backward(const uint16_t *q,", "static void head_backward(int is_noise, const uint16_t *q,")
        src = src.replace("head_backward(q, krow, vrow,", "head_backward(h == GROUP, q, krow, vrow,")
    os.makedirs(MUTANT_DIR, exist_ok=True)
    c = os.path.join(MUTANT_DIR, f"bwd_{name}.c")
    so = os.path.join(MUTANT_DIR, f"libbwd_{name}.so")
    open(c, "w").write(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", so, c, "-lm"],
                          env={**os.environ, "TMPDIR": MUTANT_DIR})
    lib = ctypes.CDLL(so)
    p = ctypes.c_void_p
    lib.gdla_oracle_prefill_bwd.argtypes = [p, p, p, p, p, p, p, ctypes.c_int, ctypes.c_int, p, ctypes.c_int,
                                            p, p, p, p, p, p, ctypes.c_int]
    lib.gdla_oracle_prefill_bwd.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_planted_backward_slip_is_caught(name, monkeypatch):
    lib = _build_bwd_mutant(name, *BWD_MUTANTS[name])
    monkeypatch.setattr(oracle, "_lib", lib)
    seqlens, hkv, window = (9, 0, 23, 1), 2, 4
    inp = gi.make_prefill_inputs(seqlens, hkv, 3)
    dout = gi.make_prefill_grad(seqlens, hkv, 3)
    _, ref = autograd_reference(inp, dout, seqlens, window)
    got = oracle_grads(inp, dout, seqlens, window)
    worst = max(_rel(got[n], r) for n, r in ref.items())
    assert worst > 1e-6, f"mutant {name} not caught (worst rel {worst:.2e})"
