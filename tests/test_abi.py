"""The C-ABI library on the CPU: it loads, exports every symbol include/gdla.h
declares, and rejects bad arguments on the host before launching anything
(fake, aligned device addresses are never dereferenced on these paths)."""
import ctypes
import os
import re

import numpy as np
import pytest

import differential_latent_attention_b200 as gdla
from differential_latent_attention_b200 import _build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # 16-byte aligned; never dereferenced by the host checks exercised here


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return gdla.library()


def _declared():
    hdr = open(os.path.join(ROOT, "include", "gdla.h")).read()
    return set(re.findall(r"GDLA_API\s+[\w\s\*]*?\b(gdla_\w+)\s*\(", hdr))


def test_header_and_binding_agree():
    assert _declared() == set(ops.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert lib.gdla_version() == 1


def test_status_strings(lib):
    for code, name in ops.STATUS.items():
        assert lib.gdla_status_string(code).decode().startswith(name)
    assert b"unknown" in lib.gdla_status_string(99)


def _fwd(lib, seqlens, hkv=1, window=0, ptrs=None):
    lens = np.asarray(seqlens, dtype=np.int32)
    p = ptrs or [FAKE] * 7
    return lib.gdla_attn_fwd(*[ctypes.c_void_p(x) for x in p], len(lens),
                             lens.ctypes.data_as(ctypes.c_void_p) if len(lens) else None, hkv, window, None)


def test_fwd_argument_checks(lib):
    assert _fwd(lib, [4], hkv=0) == 2
    assert _fwd(lib, [4], hkv=65) == 2
    assert _fwd(lib, [4, -1]) == 1
    assert lib.gdla_attn_fwd(*[ctypes.c_void_p(FAKE)] * 7, 0, None, 1, 0, None) == 1      # batch < 1
    assert _fwd(lib, [0, 0]) == 0                                                       # nothing to do
    for i in range(7):
        p = [FAKE] * 7
        p[i] = 0
        assert _fwd(lib, [4], ptrs=p) == 1                                               # null
        p[i] = FAKE + 8
        assert _fwd(lib, [4], ptrs=p) == 1                                               # misaligned
    assert _fwd(lib, [2 ** 30, 2 ** 30]) == 1                                            # N >= 2^31


def _dec(lib, ws=FAKE, ws_bytes=1 << 40, batch=2, hkv=1, nk=10, max_len=5, window=0, ptrs=None, cu=FAKE):
    p = ptrs or [FAKE] * 4
    tail = [FAKE] * 3
    return lib.gdla_attn_decode(*[ctypes.c_void_p(x) for x in p], ctypes.c_void_p(cu), nk, max_len,
                                *[ctypes.c_void_p(x) for x in tail], batch, hkv, window,
                                ctypes.c_void_p(ws), ws_bytes, None)


def test_decode_argument_checks(lib):
    assert _dec(lib, batch=0) == 1
    assert _dec(lib, nk=0) == 1
    assert _dec(lib, max_len=0) == 1
    assert _dec(lib, hkv=65) == 2
    assert _dec(lib, cu=0) == 1
    assert _dec(lib, cu=FAKE + 2) == 1
    p = [FAKE] * 4
    p[2] = FAKE + 4
    assert _dec(lib, ptrs=p) == 1
    need = lib.gdla_decode_workspace_bytes(2, 1, 5000, 0)
    assert need > 0
    assert _dec(lib, max_len=5000, ws=0) == 3
    assert _dec(lib, max_len=5000, ws_bytes=need - 1) == 3
    assert _dec(lib, max_len=5000, ws=FAKE + 16) == 3                                    # not 256-byte aligned


def test_decode_workspace_sizes(lib):
    assert lib.gdla_decode_workspace_bytes(64, 16, 32768, 128) == 0      # window: one split
    assert lib.gdla_decode_workspace_bytes(64, 16, 900, 0) == 0          # short cache: one split
    big = lib.gdla_decode_workspace_bytes(64, 16, 32768, 0)
    assert big == 64 * 16 * 32 * 5 * 130 * 4
    assert lib.gdla_decode_workspace_bytes(0, 16, 32768, 0) == 0
    assert lib.gdla_decode_workspace_bytes(1, 16, 0, 0) == 0
    # splits never exceed 64 and the workspace grows with them
    assert lib.gdla_decode_workspace_bytes(1, 1, 1 << 20, 0) == 64 * 5 * 130 * 4


def test_binding_rejects_cpu_tensors():
    import torch
    t = torch.zeros((4, 4, 192), dtype=torch.bfloat16)
    with pytest.raises((ValueError, TypeError)):
        gdla.attn_fwd(t, t[:, :1], t[:, :1], t[:, :1, :128], torch.zeros(4, 4), t[..., :128], [4])


def _lat(lib, ws=FAKE, ws_bytes=1 << 40, batch=2, hkv=1, nk=10, max_len=5, window=0, ptrs=None, cu=FAKE):
    p = ptrs or [FAKE] * 3
    tail = [FAKE] * 4   # w_uv, lambda, gate, out
    return lib.gdla_attn_decode_latent(*[ctypes.c_void_p(x) for x in p], ctypes.c_void_p(cu), nk, max_len,
                                       *[ctypes.c_void_p(x) for x in tail], batch, hkv, window,
                                       ctypes.c_void_p(ws), ws_bytes, None)


def test_latent_decode_argument_checks(lib):
    assert _lat(lib, batch=0) == 1
    assert _lat(lib, nk=0) == 1
    assert _lat(lib, max_len=0) == 1
    assert _lat(lib, hkv=17) == 2                   # 5 * 16 query heads per CTA at most
    assert _lat(lib, hkv=0) == 2
    assert _lat(lib, cu=0) == 1
    assert _lat(lib, cu=FAKE + 2) == 1
    p = [FAKE] * 3
    p[2] = FAKE + 8
    assert _lat(lib, ptrs=p) == 1
    need = lib.gdla_decode_latent_workspace_bytes(2, 1, 5000, 0)
    assert need > 0
    assert _lat(lib, max_len=5000, ws=0) == 3
    assert _lat(lib, max_len=5000, ws_bytes=need - 1) == 3
    assert _lat(lib, max_len=5000, ws=FAKE + 16) == 3


def test_latent_workspace_sizes(lib):
    # per (sequence, split): 80 head rows x (512 latent dims + max and sum) fp32
    per = 80 * (512 + 2) * 4
    assert lib.gdla_decode_latent_workspace_bytes(64, 16, 32768, 0) == 64 * 16 * per   # 16 splits of 2,048 keys
    assert lib.gdla_decode_latent_workspace_bytes(64, 16, 32768, 128) == 64 * 1 * per   # a window: one split
    assert lib.gdla_decode_latent_workspace_bytes(1, 16, 1 << 20, 0) == 32 * per        # at most 32 splits
    assert lib.gdla_decode_latent_workspace_bytes(1, 17, 4096, 0) == 0
    assert lib.gdla_decode_latent_workspace_bytes(0, 16, 4096, 0) == 0


def _bwd(lib, lens, hkv=1, window=0, ptrs=None, ws=FAKE, ws_bytes=1 << 40):
    arr = (ctypes.c_int32 * len(lens))(*lens)
    p = ptrs or [FAKE] * 13
    return lib.gdla_attn_bwd(*[ctypes.c_void_p(x) for x in p], len(lens), arr, hkv, window, ctypes.c_void_p(ws),
                             ws_bytes, None)


def test_bwd_argument_checks(lib):
    assert _bwd(lib, [4], hkv=0) == 2
    assert _bwd(lib, [4], hkv=65) == 2
    assert _bwd(lib, [4, -1]) == 1
    assert lib.gdla_attn_bwd(*[ctypes.c_void_p(FAKE)] * 13, 0, None, 1, 0, ctypes.c_void_p(FAKE), 1, None) == 1
    assert _bwd(lib, [0, 0]) == 0                                                        # nothing to do
    for i in range(13):
        p = [FAKE] * 13
        p[i] = 0
        assert _bwd(lib, [4], ptrs=p) == 1                                                # null
        p[i] = FAKE + 8
        assert _bwd(lib, [4], ptrs=p) == 1                                                # misaligned
    assert _bwd(lib, [2 ** 30, 2 ** 30]) == 1                                             # N >= 2^31
    need = lib.gdla_attn_bwd_workspace_bytes(4, 1)
    assert _bwd(lib, [4], ws=0) == 3
    assert _bwd(lib, [4], ws_bytes=need - 1) == 3
    assert _bwd(lib, [4], ws=FAKE + 16) == 3                                              # not 256-byte aligned


def test_bwd_workspace_sizes(lib):
    # dH_S [N, 4H, 128] and dH_N [N, H, 128] bf16, row statistics [N, H, 16] fp32, each 256-byte aligned
    a = lambda b: (b + 255) // 256 * 256
    n, h = 4096, 16
    assert lib.gdla_attn_bwd_workspace_bytes(n, h) == a(n * 4 * h * 256) + a(n * h * 256) + a(n * h * 64)
    assert lib.gdla_attn_bwd_workspace_bytes(37, 3) == a(37 * 12 * 256) + a(37 * 3 * 256) + a(37 * 3 * 64)
    assert lib.gdla_attn_bwd_workspace_bytes(-1, 16) == 0
    assert lib.gdla_attn_bwd_workspace_bytes(4, 0) == 0
    assert lib.gdla_attn_bwd_workspace_bytes(4, 65) == 0


def _pro(lib, lens, hkv=1, ptrs=None, ws=FAKE, ws_bytes=1 << 40):
    arr = (ctypes.c_int32 * len(lens))(*lens)
    p = ptrs or [FAKE] * 16
    return lib.gdla_prologue(*[ctypes.c_void_p(x) for x in p], len(lens), arr, hkv, ctypes.c_void_p(ws), ws_bytes,
                             None)


def test_prologue_argument_checks(lib):
    assert _pro(lib, [4], hkv=0) == 2
    assert _pro(lib, [4], hkv=65) == 2
    assert _pro(lib, [1] * 1025) == 2                                                     # more sequences than a plan holds
    assert _pro(lib, [4, -1]) == 1
    assert lib.gdla_prologue(*[ctypes.c_void_p(FAKE)] * 16, 0, None, 1, ctypes.c_void_p(FAKE), 1, None) == 1
    assert _pro(lib, [0, 0]) == 0                                                         # nothing to do
    for i in range(16):
        p = [FAKE] * 16
        p[i] = 0
        assert _pro(lib, [4], ptrs=p) == 1                                                # null
        p[i] = FAKE + 8
        assert _pro(lib, [4], ptrs=p) == 1                                                # misaligned
    assert _pro(lib, [2 ** 30, 2 ** 30]) == 1                                             # N >= 2^31
    need = lib.gdla_prologue_workspace_bytes(4)
    assert _pro(lib, [4], ws=0) == 3
    assert _pro(lib, [4], ws_bytes=need - 1) == 3
    assert _pro(lib, [4], ws=FAKE + 16) == 3


def test_prologue_workspace_sizes(lib):
    # c^Q * gamma and c^KV * gamma (bf16), partial sums of squares [N, 16], rotated k^R [N, 64] bf16,
    # rotary table [N, 64] fp32, each 256-byte aligned
    a = lambda b: (b + 255) // 256 * 256
    for n in (4096, 37):
        assert lib.gdla_prologue_workspace_bytes(n) == (a(n * 2048) + a(n * 1024) + a(n * 64) + a(n * 128) +
                                                        a(n * 256))
    assert lib.gdla_prologue_workspace_bytes(-1) == 0


class _OnDevice:
    """Stands in for a CUDA tensor's device index (the binding's device check reads only that)."""

    def __init__(self, index):
        self.index = index

    def get_device(self):
        return self.index


class _StreamOn:
    def __init__(self, index):
        import torch
        self.device = torch.device("cuda", index)


def test_binding_wants_one_device_for_tensors_and_stream():
    ops._on_one_device(_StreamOn(1), [("a", _OnDevice(1)), ("b", None), ("c", _OnDevice(1))])
    with pytest.raises(ValueError, match="c is on cuda:0"):
        ops._on_one_device(_StreamOn(1), [("a", _OnDevice(1)), ("c", _OnDevice(0))])
    with pytest.raises(ValueError, match="launch stream is on cuda:0"):
        ops._on_one_device(_StreamOn(0), [("a", _OnDevice(1))])


def test_binding_rejects_a_host_workspace():
    import torch
    ops._check_workspace(None)
    with pytest.raises(ValueError, match="workspace"):
        ops._check_workspace(torch.empty(16, dtype=torch.uint8))
