"""ctypes binding of libgdla.so: argument marshalling only.

Every step of the GDLA core runs in the library's CUDA kernels; PyTorch only
provides device memory and the current CUDA stream. There is no fallback: if
libgdla.so is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

from . import _build

GROUP, DQK, DV = 4, 192, 128
MAX_KV_HEADS = 64

STATUS = {0: "GDLA_OK", 1: "GDLA_ERR_INVALID_ARG", 2: "GDLA_ERR_UNSUPPORTED", 3: "GDLA_ERR_WORKSPACE",
          4: "GDLA_ERR_CUDA"}
EXPORTED = ("gdla_attn_fwd", "gdla_attn_bwd_workspace_bytes", "gdla_attn_bwd", "gdla_prologue_workspace_bytes",
            "gdla_prologue", "gdla_decode_workspace_bytes", "gdla_attn_decode", "gdla_attn_decode_noalloc",
            "gdla_decode_latent_workspace_bytes", "gdla_attn_decode_latent", "gdla_device_error",
            "gdla_selftest_wait_timeout", "gdla_status_string", "gdla_version")
DC, DR = 512, 64
DL = DC + DR
LATENT_MAX_KV_HEADS = 16
SELFTEST_SITE = 0x30001  # GDLA_SELFTEST_SITE

_lib = None
_lock = threading.Lock()


class GDLAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {library().gdla_status_string(status).decode()}")


def library():
    """The loaded libgdla.so (raises if it has not been built)."""
    global _lib
    lib = _lib
    if lib is not None:
        return lib
    with _lock:
        if _lib is None:
            path = _build.LIB_PATH
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing; build it with `python -m "
                                   f"differential_latent_attention_b200._build` (no fallback path exists)")
            lib = ctypes.CDLL(path)
            p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            lib.gdla_attn_fwd.argtypes = [p, p, p, p, p, p, p, i, p, i, i, p]
            lib.gdla_attn_fwd.restype = i
            lib.gdla_attn_bwd_workspace_bytes.argtypes = [ctypes.c_longlong, i]
            lib.gdla_attn_bwd_workspace_bytes.restype = sz
            lib.gdla_attn_bwd.argtypes = [p, p, p, p, p, p, p, p, p, p, p, p, p, i, p, i, i, p, sz, p]
            lib.gdla_attn_bwd.restype = i
            lib.gdla_prologue_workspace_bytes.argtypes = [ctypes.c_longlong]
            lib.gdla_prologue_workspace_bytes.restype = sz
            lib.gdla_prologue.argtypes = [p] * 16 + [i, p, i, p, sz, p]
            lib.gdla_prologue.restype = i
            lib.gdla_decode_workspace_bytes.argtypes = [i, i, i, i]
            lib.gdla_decode_workspace_bytes.restype = sz
            lib.gdla_attn_decode.argtypes = [p, p, p, p, p, i, i, p, p, p, i, i, i, p, sz, p]
            lib.gdla_attn_decode.restype = i
            lib.gdla_attn_decode_noalloc.argtypes = [p, p, p, p, p, i, i, p, p, p, i, i, i, p]
            lib.gdla_attn_decode_noalloc.restype = i
            lib.gdla_decode_latent_workspace_bytes.argtypes = [i, i, i, i]
            lib.gdla_decode_latent_workspace_bytes.restype = sz
            lib.gdla_attn_decode_latent.argtypes = [p, p, p, p, i, i, p, p, p, p, i, i, i, p, sz, p]
            lib.gdla_attn_decode_latent.restype = i
            lib.gdla_device_error.argtypes = [i]
            lib.gdla_device_error.restype = i
            lib.gdla_selftest_wait_timeout.argtypes = [p]
            lib.gdla_selftest_wait_timeout.restype = i
            lib.gdla_status_string.argtypes = [i]
            lib.gdla_status_string.restype = ctypes.c_char_p
            lib.gdla_version.argtypes = []
            lib.gdla_version.restype = i
            _lib = lib
    return _lib


# Arguments are passed to the C ABI as plain integers (the argtypes convert them).
def _ptr(t):
    return t.data_ptr() if t is not None else 0


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _on_one_device(stream, named):
    """Every tensor of a call on one CUDA device, and the launch stream on it too: the
    library launches on that stream and its kernels dereference every pointer there.
    ``named`` holds (name, tensor) pairs already checked to be CUDA tensors (None skipped)."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        d = t.get_device()
        if dev is None:
            dev = d
        elif d != dev:
            raise ValueError(f"{name} is on cuda:{d}, the call's other tensors on cuda:{dev}")
    sdev = stream.device.index if stream is not None else torch.cuda.current_device()
    if dev is not None and sdev != dev:
        raise ValueError(f"the tensors are on cuda:{dev} but the launch stream is on cuda:{sdev}")


def _check_workspace(ws):
    if ws is None:
        return
    if not isinstance(ws, torch.Tensor) or not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")


def _check(t, name, dtype, shape):
    # common case first: one combined test per call, the detailed ones only to explain a failure
    if type(t) is torch.Tensor and t.dtype is dtype and t.shape == shape and t.is_cuda and t.is_contiguous():
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def attn_fwd(q_sig, q_noise, k, v, lam, gate, seqlens, window=0, out=None, stream=None):
    """Packed varlen GDLA prefill (calls ``gdla_attn_fwd``).

    q_sig [N, 4H, 192], q_noise [N, H, 192], k [N, H, 192], v [N, H, 128] and
    gate [N, 4H, 128] are bf16 CUDA tensors, lam [N, 4H] fp32; ``seqlens`` is a
    host sequence of per-sequence lengths summing to N. Returns out [N, 4H, 128]
    bf16 (written into ``out`` when given).
    """
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
    n = int(lens.sum(dtype=np.int64))
    hkv = q_noise.shape[1] if q_noise.dim() == 3 else -1
    hs = GROUP * hkv
    _check(q_sig, "q_sig", torch.bfloat16, (n, hs, DQK))
    _check(q_noise, "q_noise", torch.bfloat16, (n, hkv, DQK))
    _check(k, "k", torch.bfloat16, (n, hkv, DQK))
    _check(v, "v", torch.bfloat16, (n, hkv, DV))
    _check(lam, "lam", torch.float32, (n, hs))
    _check(gate, "gate", torch.bfloat16, (n, hs, DV))
    if out is None:
        out = torch.empty((n, hs, DV), dtype=torch.bfloat16, device=q_sig.device)
    _check(out, "out", torch.bfloat16, (n, hs, DV))
    _on_one_device(stream, (("q_sig", q_sig), ("q_noise", q_noise), ("k", k), ("v", v), ("lam", lam),
                            ("gate", gate), ("out", out)))
    st = library().gdla_attn_fwd(_ptr(q_sig), _ptr(q_noise), _ptr(k), _ptr(v), _ptr(lam), _ptr(gate), _ptr(out),
                                 int(lens.shape[0]), lens.__array_interface__["data"][0], hkv, int(window),
                                 _stream(stream))
    if st != 0:
        raise GDLAError(st, "gdla_attn_fwd")
    return out


def attn_bwd_workspace_bytes(total_tokens, num_kv_heads):
    return int(library().gdla_attn_bwd_workspace_bytes(int(total_tokens), int(num_kv_heads)))


def attn_bwd(q_sig, q_noise, k, v, lam, gate, dout, seqlens, window=0, grads=None, workspace=None, stream=None):
    """Packed varlen GDLA prefill backward (calls ``gdla_attn_bwd``).

    Inputs as ``attn_fwd`` plus dout [N, 4H, 128] bf16 (the gradient of out).
    Returns a dict of dq_sig, dq_noise, dk, dv, dgate (bf16) and dlambda (fp32),
    written into ``grads`` when given; ``workspace`` (uint8 CUDA tensor) is
    allocated here when not given.
    """
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
    n = int(lens.sum(dtype=np.int64))
    hkv = q_noise.shape[1] if q_noise.dim() == 3 else -1
    hs = GROUP * hkv
    _check(q_sig, "q_sig", torch.bfloat16, (n, hs, DQK))
    _check(q_noise, "q_noise", torch.bfloat16, (n, hkv, DQK))
    _check(k, "k", torch.bfloat16, (n, hkv, DQK))
    _check(v, "v", torch.bfloat16, (n, hkv, DV))
    _check(lam, "lam", torch.float32, (n, hs))
    _check(gate, "gate", torch.bfloat16, (n, hs, DV))
    _check(dout, "dout", torch.bfloat16, (n, hs, DV))
    shapes = {"dq_sig": ((n, hs, DQK), torch.bfloat16), "dq_noise": ((n, hkv, DQK), torch.bfloat16),
              "dk": ((n, hkv, DQK), torch.bfloat16), "dv": ((n, hkv, DV), torch.bfloat16),
              "dlambda": ((n, hs), torch.float32), "dgate": ((n, hs, DV), torch.bfloat16)}
    if grads is None:
        grads = {name: torch.empty(shape, dtype=dt, device=q_sig.device) for name, (shape, dt) in shapes.items()}
    for name, (shape, dt) in shapes.items():
        _check(grads[name], name, dt, shape)
    need = attn_bwd_workspace_bytes(n, hkv)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q_sig.device)
    _check_workspace(workspace)
    _on_one_device(stream, [("q_sig", q_sig), ("q_noise", q_noise), ("k", k), ("v", v), ("lam", lam),
                            ("gate", gate), ("dout", dout), ("workspace", workspace)] + list(grads.items()))
    ws_bytes = workspace.numel() * workspace.element_size()
    st = library().gdla_attn_bwd(_ptr(q_sig), _ptr(q_noise), _ptr(k), _ptr(v), _ptr(lam), _ptr(gate), _ptr(dout),
                                 _ptr(grads["dq_sig"]), _ptr(grads["dq_noise"]), _ptr(grads["dk"]), _ptr(grads["dv"]),
                                 _ptr(grads["dlambda"]), _ptr(grads["dgate"]), int(lens.shape[0]),
                                 lens.__array_interface__["data"][0], hkv, int(window), workspace.data_ptr(),
                                 ws_bytes, _stream(stream))
    if st != 0:
        raise GDLAError(st, "gdla_attn_bwd")
    return grads


def prologue_workspace_bytes(total_tokens):
    return int(library().gdla_prologue_workspace_bytes(int(total_tokens)))


def prologue(x, w_qa, w_kva, gamma_q, gamma_kv, w_qb, w_uk, w_uv, w_lambda, w_gate, seqlens, outs=None,
             workspace=None, stream=None):
    """The attention inputs from the hidden state (calls ``gdla_prologue``).

    x [N, 4096] bf16; weights [out, in] bf16: w_qa [1024, 4096], w_kva [576, 4096],
    w_qb [5H*192, 1024], w_uk / w_uv [H, 128, 512], w_lambda [4H, 4096],
    w_gate [4H*128, 4096]; gamma_q [1024], gamma_kv [512] fp32. Returns a dict
    q_sig, q_noise, k, v, lam, gate in the layouts ``attn_fwd`` takes.
    """
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
    n = int(lens.sum(dtype=np.int64))
    hkv = w_uk.shape[0] if w_uk.dim() == 3 else -1
    hs = GROUP * hkv
    _check(x, "x", torch.bfloat16, (n, 4096))
    _check(w_qa, "w_qa", torch.bfloat16, (1024, 4096))
    _check(w_kva, "w_kva", torch.bfloat16, (576, 4096))
    _check(gamma_q, "gamma_q", torch.float32, (1024,))
    _check(gamma_kv, "gamma_kv", torch.float32, (512,))
    _check(w_qb, "w_qb", torch.bfloat16, ((hs + hkv) * DQK, 1024))
    _check(w_uk, "w_uk", torch.bfloat16, (hkv, DV, 512))
    _check(w_uv, "w_uv", torch.bfloat16, (hkv, DV, 512))
    _check(w_lambda, "w_lambda", torch.bfloat16, (hs, 4096))
    _check(w_gate, "w_gate", torch.bfloat16, (hs * DV, 4096))
    shapes = {"q_sig": ((n, hs, DQK), torch.bfloat16), "q_noise": ((n, hkv, DQK), torch.bfloat16),
              "k": ((n, hkv, DQK), torch.bfloat16), "v": ((n, hkv, DV), torch.bfloat16),
              "lam": ((n, hs), torch.float32), "gate": ((n, hs, DV), torch.bfloat16)}
    if outs is None:
        outs = {name: torch.empty(shape, dtype=dt, device=x.device) for name, (shape, dt) in shapes.items()}
    for name, (shape, dt) in shapes.items():
        _check(outs[name], name, dt, shape)
    if workspace is None:
        workspace = torch.empty(max(prologue_workspace_bytes(n), 1), dtype=torch.uint8, device=x.device)
    _check_workspace(workspace)
    _on_one_device(stream, [("x", x), ("w_qa", w_qa), ("w_kva", w_kva), ("gamma_q", gamma_q), ("gamma_kv", gamma_kv),
                            ("w_qb", w_qb), ("w_uk", w_uk), ("w_uv", w_uv), ("w_lambda", w_lambda),
                            ("w_gate", w_gate), ("workspace", workspace)] + list(outs.items()))
    st = library().gdla_prologue(_ptr(x), _ptr(w_qa), _ptr(w_kva), _ptr(gamma_q), _ptr(gamma_kv), _ptr(w_qb),
                                 _ptr(w_uk), _ptr(w_uv), _ptr(w_lambda), _ptr(w_gate), _ptr(outs["q_sig"]),
                                 _ptr(outs["q_noise"]), _ptr(outs["k"]), _ptr(outs["v"]), _ptr(outs["lam"]),
                                 _ptr(outs["gate"]), int(lens.shape[0]), lens.__array_interface__["data"][0], hkv,
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream))
    if st != 0:
        raise GDLAError(st, "gdla_prologue")
    return outs


def decode_workspace_bytes(batch, num_kv_heads, max_seqlen_k, window=0):
    return int(library().gdla_decode_workspace_bytes(int(batch), int(num_kv_heads), int(max_seqlen_k),
                                                     int(window)))


def attn_decode(q_sig, q_noise, k_cache, v_cache, cu_seqlens_k, max_seqlen_k, lam, gate, window=0, out=None,
                workspace=None, stream=None):
    """Varlen GDLA decode (calls ``gdla_attn_decode``).

    One query per sequence: q_sig [B, 4H, 192], q_noise [B, H, 192], lam [B, 4H],
    gate [B, 4H, 128]; k_cache [Nk, H, 192] and v_cache [Nk, H, 128] hold the
    sequences back to back as given by the int32 CUDA tensor cu_seqlens_k [B+1].
    ``workspace`` (uint8 CUDA tensor) is allocated here when not given.
    """
    b = q_sig.shape[0]
    hkv = q_noise.shape[1] if q_noise.dim() == 3 else -1
    hs = GROUP * hkv
    nk = k_cache.shape[0]
    _check(q_sig, "q_sig", torch.bfloat16, (b, hs, DQK))
    _check(q_noise, "q_noise", torch.bfloat16, (b, hkv, DQK))
    _check(k_cache, "k_cache", torch.bfloat16, (nk, hkv, DQK))
    _check(v_cache, "v_cache", torch.bfloat16, (nk, hkv, DV))
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32, (b + 1,))
    _check(lam, "lam", torch.float32, (b, hs))
    _check(gate, "gate", torch.bfloat16, (b, hs, DV))
    if out is None:
        out = torch.empty((b, hs, DV), dtype=torch.bfloat16, device=q_sig.device)
    _check(out, "out", torch.bfloat16, (b, hs, DV))
    need = decode_workspace_bytes(b, hkv, max_seqlen_k, window)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_sig.device)
    _check_workspace(workspace)
    _on_one_device(stream, (("q_sig", q_sig), ("q_noise", q_noise), ("k_cache", k_cache), ("v_cache", v_cache),
                            ("cu_seqlens_k", cu_seqlens_k), ("lam", lam), ("gate", gate), ("out", out),
                            ("workspace", workspace)))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = library().gdla_attn_decode(_ptr(q_sig), _ptr(q_noise), _ptr(k_cache), _ptr(v_cache), _ptr(cu_seqlens_k),
                                    int(nk), int(max_seqlen_k), _ptr(lam), _ptr(gate), _ptr(out), int(b), hkv,
                                    int(window), _ptr(workspace), ws_bytes, _stream(stream))
    if st != 0:
        raise GDLAError(st, "gdla_attn_decode")
    return out


def decode_latent_workspace_bytes(batch, num_kv_heads, max_seqlen_k, window=0):
    return int(library().gdla_decode_latent_workspace_bytes(int(batch), int(num_kv_heads), int(max_seqlen_k),
                                                            int(window)))


def attn_decode_latent(q_abs_sig, q_abs_noise, ckv, cu_seqlens_k, max_seqlen_k, w_uv, lam, gate, window=0,
                       out=None, workspace=None, stream=None):
    """GDLA decode over the compressed KV cache (calls ``gdla_attn_decode_latent``).

    q_abs_sig [B, 4H, 576] and q_abs_noise [B, H, 576] bf16 (queries with W^UK
    absorbed), ckv [Nk, 576] bf16 ([c | k_rope] per token, sequences packed as
    given by the int32 CUDA tensor cu_seqlens_k [B+1]), w_uv [H, 128, 512] bf16,
    lam [B, 4H] fp32, gate [B, 4H, 128] bf16. ``workspace`` (uint8 CUDA tensor)
    is allocated here when not given.
    """
    b = q_abs_sig.shape[0]
    hkv = q_abs_noise.shape[1] if q_abs_noise.dim() == 3 else -1
    hs = GROUP * hkv
    nk = ckv.shape[0]
    _check(q_abs_sig, "q_abs_sig", torch.bfloat16, (b, hs, DL))
    _check(q_abs_noise, "q_abs_noise", torch.bfloat16, (b, hkv, DL))
    _check(ckv, "ckv", torch.bfloat16, (nk, DL))
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32, (b + 1,))
    _check(w_uv, "w_uv", torch.bfloat16, (hkv, DV, DC))
    _check(lam, "lam", torch.float32, (b, hs))
    _check(gate, "gate", torch.bfloat16, (b, hs, DV))
    if out is None:
        out = torch.empty((b, hs, DV), dtype=torch.bfloat16, device=q_abs_sig.device)
    _check(out, "out", torch.bfloat16, (b, hs, DV))
    need = decode_latent_workspace_bytes(b, hkv, max_seqlen_k, window)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_abs_sig.device)
    _check_workspace(workspace)
    _on_one_device(stream, (("q_abs_sig", q_abs_sig), ("q_abs_noise", q_abs_noise), ("ckv", ckv),
                            ("cu_seqlens_k", cu_seqlens_k), ("w_uv", w_uv), ("lam", lam), ("gate", gate),
                            ("out", out), ("workspace", workspace)))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = library().gdla_attn_decode_latent(_ptr(q_abs_sig), _ptr(q_abs_noise), _ptr(ckv), _ptr(cu_seqlens_k),
                                           int(nk), int(max_seqlen_k), _ptr(w_uv), _ptr(lam), _ptr(gate),
                                           _ptr(out), int(b), hkv, int(window), _ptr(workspace), ws_bytes,
                                           _stream(stream))
    if st != 0:
        raise GDLAError(st, "gdla_attn_decode_latent")
    return out


def device_error(clear=True) -> int:
    """Code recorded by a kernel whose bounded wait ran out (0 = none); synchronises."""
    return int(library().gdla_device_error(1 if clear else 0))


def selftest_wait_timeout(stream=None):
    """Enqueue the failure-path self-test (a bounded wait that runs out after about a
    second and records SELFTEST_SITE in the device failure word)."""
    st = library().gdla_selftest_wait_timeout(_stream(stream))
    if st != 0:
        raise GDLAError(st, "gdla_selftest_wait_timeout")
