"""GDLA forward oracle (fp64, CPU): TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. The CUDA product path never
imports, links or calls it, and the two share no code.

The arithmetic lives in ``gdla_oracle.c`` (plain C, double precision); this
module only compiles it on demand and marshals numpy arrays through ctypes.
Parity status per function:

* ``prefill`` - pinned (closed forms, invariants, a library special case and
  brute force; see ``tests/test_oracle_pins.py``).
* ``decode`` - pinned through the decode == last prefill row identity and the
  same closed forms.
* ``decode_latent`` - pinned exactly to ``decode`` through an integer construction
  (``tests/test_oracle_latent.py``).
* ``prefill_bwd`` - pinned to fp64 automatic differentiation (torch autograd) of
  the forward composed from library operations, on full-causal, windowed and
  ragged inputs (``tests/test_oracle_bwd.py``).

The choice of lambda granularity (one scalar per token and signal head), the
absence of any normalisation after the subtract and the 1/sqrt(192) softmax
scale are readings where the pages are silent; no page value pins them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdla_oracle.so")
_lib = None
_lock = threading.Lock()

GROUP = 4
DQK = 192
DV = 128
DC = 512          # KV low-rank (latent) dim
DR = 64           # shared rotary key dim
DL = DC + DR      # width of a latent cache row and of an absorbed query


def build(force: bool = False) -> str:
    """Compile gdla_oracle.c into libgdla_oracle.so (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        # the compiler's intermediate files stay inside the repository
        scratch = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "_build", "tmp")
        os.makedirs(scratch, exist_ok=True)
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"], env={**os.environ, "TMPDIR": scratch})
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            p = ctypes.c_void_p
            lib.gdla_oracle_prefill.argtypes = [p, p, p, p, p, p, ctypes.c_int, ctypes.c_int, p,
                                                ctypes.c_int, p, ctypes.c_int64, p, ctypes.c_int]
            lib.gdla_oracle_prefill.restype = ctypes.c_int
            lib.gdla_oracle_decode.argtypes = [p, p, p, p, p, p, p, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, p, ctypes.c_int]
            lib.gdla_oracle_decode.restype = ctypes.c_int
            lib.gdla_oracle_decode_latent.argtypes = [p, p, p, p, p, p, p, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int, p, ctypes.c_int]
            lib.gdla_oracle_decode_latent.restype = ctypes.c_int
            lib.gdla_oracle_prefill_bwd.argtypes = [p, p, p, p, p, p, p, ctypes.c_int, ctypes.c_int, p,
                                                    ctypes.c_int, p, p, p, p, p, p, ctypes.c_int]
            lib.gdla_oracle_prefill_bwd.restype = ctypes.c_int
            _lib = lib
    return _lib


def default_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _bits(a, shape_tail, name):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"{name}: expected bf16 bit patterns as uint16, got {a.dtype}")
    if tuple(a.shape[1:]) != tuple(shape_tail):
        raise ValueError(f"{name}: expected trailing shape {shape_tail}, got {a.shape}")
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def prefill(q_sig, q_noise, k, v, lam, gate, seqlens, window, rows=None, num_threads=None):
    """Packed varlen GDLA prefill in fp64.

    q_sig [N, 4H, 192], q_noise [N, H, 192], k [N, H, 192], v [N, H, 128] and
    gate [N, 4H, 128] are uint16 arrays of bf16 bits; lam is float32 [N, 4H].
    ``rows`` selects packed token indices (default: all N). Returns float64
    [len(rows), 4H, 128].
    """
    hkv = q_noise.shape[1]
    hs = GROUP * hkv
    q_sig = _bits(q_sig, (hs, DQK), "q_sig")
    q_noise = _bits(q_noise, (hkv, DQK), "q_noise")
    k = _bits(k, (hkv, DQK), "k")
    v = _bits(v, (hkv, DV), "v")
    gate = _bits(gate, (hs, DV), "gate")
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    n = int(seqlens.sum())
    for name, a in (("q_sig", q_sig), ("q_noise", q_noise), ("k", k), ("v", v), ("gate", gate), ("lambda", lam)):
        if a.shape[0] != n:
            raise ValueError(f"{name}: leading dim {a.shape[0]} != sum(seqlens) {n}")
    if lam.shape != (n, hs):
        raise ValueError(f"lambda: expected shape {(n, hs)}, got {lam.shape}")
    if rows is None:
        rows = np.arange(n, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((rows.shape[0], hs, DV), dtype=np.float64)
    nt = int(num_threads or default_threads())
    rc = _load().gdla_oracle_prefill(_ptr(q_sig), _ptr(q_noise), _ptr(k), _ptr(v), _ptr(lam), _ptr(gate),
                                     hkv, int(seqlens.shape[0]), _ptr(seqlens), int(window),
                                     _ptr(rows), int(rows.shape[0]), _ptr(out), nt)
    if rc != 0:
        raise ValueError("gdla_oracle_prefill rejected its arguments")
    return out


def decode(q_sig, q_noise, k_cache, v_cache, cu_seqlens_k, lam, gate, window, num_threads=None):
    """Varlen GDLA decode in fp64: one query per sequence at position L_b - 1.

    q_sig [B, 4H, 192], q_noise [B, H, 192], gate [B, 4H, 128], lam [B, 4H];
    k_cache [Nk, H, 192] and v_cache [Nk, H, 128] packed by cu_seqlens_k [B+1].
    Returns float64 [B, 4H, 128].
    """
    hkv = q_noise.shape[1]
    hs = GROUP * hkv
    q_sig = _bits(q_sig, (hs, DQK), "q_sig")
    q_noise = _bits(q_noise, (hkv, DQK), "q_noise")
    k_cache = _bits(k_cache, (hkv, DQK), "k_cache")
    v_cache = _bits(v_cache, (hkv, DV), "v_cache")
    gate = _bits(gate, (hs, DV), "gate")
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens_k, dtype=np.int64))
    b = cu.shape[0] - 1
    if q_sig.shape[0] != b or q_noise.shape[0] != b or gate.shape[0] != b or lam.shape != (b, hs):
        raise ValueError("decode: per-sequence inputs must have leading dim B = len(cu_seqlens_k) - 1")
    if cu[-1] > k_cache.shape[0] or cu[-1] > v_cache.shape[0]:
        raise ValueError("decode: cache shorter than cu_seqlens_k[-1]")
    out = np.zeros((b, hs, DV), dtype=np.float64)
    nt = int(num_threads or default_threads())
    rc = _load().gdla_oracle_decode(_ptr(q_sig), _ptr(q_noise), _ptr(k_cache), _ptr(v_cache), _ptr(cu),
                                    _ptr(lam), _ptr(gate), b, hkv, int(window), _ptr(out), nt)
    if rc != 0:
        raise ValueError("gdla_oracle_decode rejected its arguments")
    return out


def decode_latent(q_abs_sig, q_abs_noise, ckv, cu_seqlens_k, w_uv, lam, gate, window, num_threads=None):
    """GDLA decode over the compressed KV cache with the projections absorbed, in fp64.

    q_abs_sig [B, 4H, 576] and q_abs_noise [B, H, 576]: queries as
    [W^UK_j^T q_nope (512) | q_rope (64)]; ckv [Nk, 576]: per token [c (512) | kr (64)],
    packed by cu_seqlens_k [B+1]; w_uv [H, 128, 512]; lam [B, 4H]; gate [B, 4H, 128].
    All bf16 inputs as uint16 bit patterns. Returns float64 [B, 4H, 128].
    """
    hkv = q_abs_noise.shape[1]
    hs = GROUP * hkv
    q_abs_sig = _bits(q_abs_sig, (hs, DL), "q_abs_sig")
    q_abs_noise = _bits(q_abs_noise, (hkv, DL), "q_abs_noise")
    ckv = _bits(ckv, (DL,), "ckv")
    w_uv = _bits(w_uv, (DV, DC), "w_uv")
    gate = _bits(gate, (hs, DV), "gate")
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens_k, dtype=np.int64))
    b = cu.shape[0] - 1
    if q_abs_sig.shape[0] != b or q_abs_noise.shape[0] != b or gate.shape[0] != b or lam.shape != (b, hs):
        raise ValueError("decode_latent: per-sequence inputs must have leading dim B = len(cu_seqlens_k) - 1")
    if w_uv.shape[0] != hkv:
        raise ValueError("decode_latent: w_uv needs one [128, 512] matrix per KV head")
    if cu[-1] > ckv.shape[0]:
        raise ValueError("decode_latent: cache shorter than cu_seqlens_k[-1]")
    out = np.zeros((b, hs, DV), dtype=np.float64)
    nt = int(num_threads or default_threads())
    rc = _load().gdla_oracle_decode_latent(_ptr(q_abs_sig), _ptr(q_abs_noise), _ptr(ckv), _ptr(cu), _ptr(w_uv),
                                           _ptr(lam), _ptr(gate), b, hkv, int(window), _ptr(out), nt)
    if rc != 0:
        raise ValueError("gdla_oracle_decode_latent rejected its arguments")
    return out


def prefill_bwd(q_sig, q_noise, k, v, lam, gate, dout, seqlens, window, num_threads=None):
    """Gradients of sum(dout * out) for the packed varlen GDLA prefill, in fp64.

    Inputs as ``prefill`` plus dout [N, 4H, 128] (uint16 bf16 bits). Returns a dict
    of float64 arrays: dq_sig [N, 4H, 192], dq_noise [N, H, 192], dk [N, H, 192],
    dv [N, H, 128], dlambda [N, 4H], dgate [N, 4H, 128].
    """
    hkv = q_noise.shape[1]
    hs = GROUP * hkv
    q_sig = _bits(q_sig, (hs, DQK), "q_sig")
    q_noise = _bits(q_noise, (hkv, DQK), "q_noise")
    k = _bits(k, (hkv, DQK), "k")
    v = _bits(v, (hkv, DV), "v")
    gate = _bits(gate, (hs, DV), "gate")
    dout = _bits(dout, (hs, DV), "dout")
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    n = int(seqlens.sum())
    for name, a in (("q_sig", q_sig), ("q_noise", q_noise), ("k", k), ("v", v), ("gate", gate),
                    ("dout", dout), ("lambda", lam)):
        if a.shape[0] != n:
            raise ValueError(f"{name}: leading dim {a.shape[0]} != sum(seqlens) {n}")
    if lam.shape != (n, hs):
        raise ValueError(f"lambda: expected shape {(n, hs)}, got {lam.shape}")
    g = {"dq_sig": np.zeros((n, hs, DQK)), "dq_noise": np.zeros((n, hkv, DQK)), "dk": np.zeros((n, hkv, DQK)),
         "dv": np.zeros((n, hkv, DV)), "dlambda": np.zeros((n, hs)), "dgate": np.zeros((n, hs, DV))}
    nt = int(num_threads or default_threads())
    rc = _load().gdla_oracle_prefill_bwd(_ptr(q_sig), _ptr(q_noise), _ptr(k), _ptr(v), _ptr(lam), _ptr(gate),
                                         _ptr(dout), hkv, int(seqlens.shape[0]), _ptr(seqlens), int(window),
                                         _ptr(g["dq_sig"]), _ptr(g["dq_noise"]), _ptr(g["dk"]), _ptr(g["dv"]),
                                         _ptr(g["dlambda"]), _ptr(g["dgate"]), nt)
    if rc != 0:
        raise ValueError("gdla_oracle_prefill_bwd rejected its arguments")
    return g


# ---------------------------------------------------------------------------
# Prologue: the projections that produce the attention's inputs from the hidden
# state (aitrends.kr/articles/94908, GDLA query-path paragraph: c^Q = RMSNorm(x W^Q_a)
# expanded to content and rotary queries; [c^KV; k^R] = x W^KV_a, c^KV RMSNorm'd once
# and expanded to 16 KV heads, k^R shared by every head; head-configuration paragraph:
# hidden 4096, query / KV low-rank 1024 / 512, rotary 64 of the 192 query-key dims;
# group-ratio paragraph: lambda_t = sigmoid(x_t W^lambda)). Readings where the pages
# are silent: RMSNorm eps 1e-6 with a learned weight; rotary embedding in the
# rotate-half form over the 64 rotary dims with base 10000, positions counted from
# 0 in each sequence; the element-wise gate logits are x W^G (one per signal head
# and value dim); query heads ordered signal 0..4H-1, then noise 0..H-1.
# Plain numpy fp64; matmul is the library primitive of each projection step.
# ---------------------------------------------------------------------------
HIDDEN = 4096
Q_RANK = 1024
ROPE = 64
ROPE_BASE = 10000.0
RMS_EPS = 1e-6


def _f64(a):
    """bf16 bit patterns (uint16) or float arrays -> float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def rms_norm(c, gamma):
    """RMSNorm over the last axis: c / sqrt(mean(c^2) + eps) * gamma."""
    c = np.asarray(c, dtype=np.float64)
    return c / np.sqrt(np.mean(c * c, axis=-1, keepdims=True) + RMS_EPS) * np.asarray(gamma, dtype=np.float64)


def rope(xr, positions):
    """Rotary embedding of the last axis (64 dims) in the rotate-half form: the pair
    (i, i + 32) is rotated by positions * base^(-i / 32)."""
    xr = np.asarray(xr, dtype=np.float64)
    half = xr.shape[-1] // 2
    inv = ROPE_BASE ** (-np.arange(half, dtype=np.float64) / half)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]       # [N, 32]
    shape = (ang.shape[0],) + (1,) * (xr.ndim - 2) + (half,)
    cos, sin = np.cos(ang).reshape(shape), np.sin(ang).reshape(shape)
    a, b = xr[..., :half], xr[..., half:]
    return np.concatenate([a * cos - b * sin, a * sin + b * cos], axis=-1)


def positions_of(seqlens):
    return np.concatenate([np.arange(int(L), dtype=np.int64) for L in seqlens]) if len(seqlens) else np.zeros(0)


def prologue(x, w_qa, w_kva, gamma_q, gamma_kv, w_qb, w_uk, w_uv, w_lambda, w_gate, seqlens):
    """The attention inputs from the hidden state x [N, 4096], in fp64.

    Weights are [out_features, in_features] (bf16 bits or floats): w_qa [1024, 4096],
    w_kva [576, 4096], w_qb [5H*192, 1024] (per query head [content 128 | rotary 64]),
    w_uk, w_uv [H, 128, 512], w_lambda [4H, 4096], w_gate [4H*128, 4096]; gamma_q [1024],
    gamma_kv [512]. Returns dict q_sig [N, 4H, 192], q_noise [N, H, 192], k [N, H, 192],
    v [N, H, 128], lam [N, 4H], gate [N, 4H, 128] (float64).
    """
    x = _f64(x)
    hkv = np.asarray(w_uk).shape[0]
    hs = GROUP * hkv
    pos = positions_of(seqlens)
    assert pos.shape[0] == x.shape[0]
    cq = rms_norm(x @ _f64(w_qa).T, gamma_q)                                   # [N, 1024]
    ckv_full = x @ _f64(w_kva).T                                               # [N, 576]
    ckv = rms_norm(ckv_full[:, :DC], gamma_kv)                                 # [N, 512]
    k_rope = rope(ckv_full[:, DC:], pos)                                       # [N, 64]
    q = (cq @ _f64(w_qb).T).reshape(x.shape[0], hs + hkv, DQK)                 # [N, 5H, 192]
    q = np.concatenate([q[..., :DQK - ROPE], rope(q[..., DQK - ROPE:], pos)], axis=-1)
    k_nope = np.einsum("nc,hdc->nhd", ckv, _f64(w_uk))                          # [N, H, 128]
    v = np.einsum("nc,hdc->nhd", ckv, _f64(w_uv))                               # [N, H, 128]
    k = np.concatenate([k_nope, np.broadcast_to(k_rope[:, None, :], (x.shape[0], hkv, ROPE))], axis=-1)
    lam = 1.0 / (1.0 + np.exp(-(x @ _f64(w_lambda).T)))
    gate = (x @ _f64(w_gate).T).reshape(x.shape[0], hs, DV)
    return {"q_sig": q[:, :hs], "q_noise": q[:, hs:], "k": k, "v": v, "lam": lam, "gate": gate}
