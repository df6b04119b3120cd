"""gdla_attn_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin inside another runtime that forbids allocation on its
execution path, a service with a fixed pre-reserved memory budget) only hold
their input and output buffers, so they cannot supply the split-KV workspace
of gdla_attn_decode. The no-allocation entry point keeps that scratch in a
fixed-size device array inside the library. These tests call it through the
C ABI and compare it, bit for bit, with the regular entry point (given a
NaN-filled workspace) on the same inputs, for calls in a row (the array keeps
the previous call's contents, which must not leak into the next result), and
check that sizes needing more scratch than the array holds are refused before
anything runs.

This file is named so that pytest collects it last.
"""
import ctypes
import os
import re

import pytest
import torch

import differential_latent_attention_b200 as gdla
import gdla_inputs as gi
from _parity import gpu_decode

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _scratch_limit():
    hdr = open(os.path.join(ROOT, "include", "gdla.h")).read()
    m = re.search(r"#define\s+GDLA_DECODE_STATIC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", hdr)
    return int(m.group(1)) << int(m.group(2))


def _noalloc(d, max_len, window, out):
    lib = gdla.library()
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    hkv = d["q_noise"].shape[1]
    return lib.gdla_attn_decode_noalloc(
        p(d["q_sig"]), p(d["q_noise"]), p(d["k_cache"]), p(d["v_cache"]), p(d["cu_seqlens_k"]),
        d["k_cache"].shape[0], max_len, p(d["lam"]), p(d["gate"]), p(out), d["q_sig"].shape[0], hkv, window,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [
    # (KV lengths, KV heads, window, max_seqlen_k, seed): both need split-KV scratch
    ((3000, 70, 5000, 1), 2, 0, 5000, 60),
    ((1500, 4100, 9), 3, 0, 8192, 61),
]


def _reference(d, max_len, window):
    """gdla_attn_decode on the same inputs, its caller-owned workspace filled with
    NaN so that a slot read before it is written would show."""
    hkv = d["q_noise"].shape[1]
    need = gdla.decode_workspace_bytes(d["q_sig"].shape[0], hkv, max_len, window)
    ws = torch.full((max(need, 4) // 4,), float("nan"), dtype=torch.float32, device="cuda").view(torch.uint8)
    return gpu_decode(d, max_len, window, workspace=ws)


def _run_and_compare(d, max_len, window, what):
    ref = _reference(d, max_len, window)
    out = torch.full_like(ref, float("nan"))
    assert _noalloc(d, max_len, window, out) == 0
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
    # the same kernels on the same inputs: the results must agree bit for bit
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), what


def test_two_calls_in_a_row_match_the_workspace_entry_point():
    limit = _scratch_limit()
    for lengths, hkv, window, max_len, seed in CASES:
        need = gdla.decode_workspace_bytes(len(lengths), hkv, max_len, window)
        assert 0 < need <= limit
        d = gi.make_decode_inputs(lengths, hkv, seed, device="cuda")
        _run_and_compare(d, max_len, window, f"no-alloc decode {lengths}")


def test_previous_contents_of_the_scratch_do_not_leak():
    """The fixed array keeps the last call's split partials. A long batch fills
    every split slot; the same batch shape with short caches then leaves most
    splits empty (their slots keep the old partials, which the combine must not
    read); a long batch with new inputs follows. Each call must match the
    workspace entry point bit for bit."""
    hkv, max_len = 2, 8192
    long_a = gi.make_decode_inputs((8192, 8000, 6000, 8100), hkv, 66, device="cuda")
    short = gi.make_decode_inputs((5, 1030, 1, 64), hkv, 67, device="cuda")
    long_b = gi.make_decode_inputs((8192, 7001, 8192, 2049), hkv, 68, device="cuda")
    assert gdla.decode_workspace_bytes(4, hkv, max_len, 0) <= _scratch_limit()
    _run_and_compare(long_a, max_len, 0, "long batch")
    _run_and_compare(short, max_len, 0, "short caches after a long batch")
    _run_and_compare(long_b, max_len, 0, "long batch after short caches")


def test_single_split_needs_no_scratch():
    d = gi.make_decode_inputs((300, 129, 5), 2, 62, device="cuda")
    assert gdla.decode_workspace_bytes(3, 2, 300, 128) == 0
    ref = gpu_decode(d, 300, 128)
    out = torch.empty_like(ref)
    assert _noalloc(d, 300, 128, out) == 0
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), "no-alloc window decode"


def test_sizes_beyond_the_scratch_limit_are_refused():
    # 64 sequences x 16 KV heads up to 32768 keys needs ~85 MB of split scratch
    lengths = (64,) * 64
    d = gi.make_decode_inputs(lengths, 16, 63, device="cuda")
    assert gdla.decode_workspace_bytes(64, 16, 32768, 0) > _scratch_limit()
    out = torch.full((64, 64, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(d, 32768, 0, out) == 3          # GDLA_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
