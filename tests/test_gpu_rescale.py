"""Online-softmax rescaling on the GPU. With N(0,1) inputs the running row
maximum settles after the first key tile, so the O rescale (taken when the
maximum grows by more than 2^8) would hardly run. Here key magnitudes grow
along each sequence, so every key tile raises the maximum by far more than
that and O is rescaled on every tile; with magnitudes falling along the
sequence the first tile holds the maximum and later weights underflow. Both
must match the fp64 oracle."""
import numpy as np
import pytest
import torch

import gdla_inputs as gi
import oracle
from _parity import assert_close, check_prefill, decode_host_args, gpu_decode

pytestmark = pytest.mark.gpu


def _scale_rows(x, positions, rising):
    """Multiply row u of x (dim 0) by 1 + pos/16 (rising) or 1 + (L - pos)/16, in bf16."""
    pos = torch.as_tensor(positions, dtype=torch.float32, device=x.device)
    c = 1.0 + (pos if rising else pos.max() - pos) / 16.0
    return (x.float() * c.view(-1, *([1] * (x.dim() - 1)))).to(torch.bfloat16)


@pytest.mark.parametrize("rising", [True, False], ids=["rising", "falling"])
@pytest.mark.parametrize("window", [0, 200, 1000])
def test_prefill_key_scale_drift(rising, window):
    seqlens = (700, 300)
    t = gi.make_prefill_inputs(seqlens, 2, 70 + window, device="cuda")
    positions = np.concatenate([np.arange(L) for L in seqlens])
    t["k"] = _scale_rows(t["k"], positions, rising)
    check_prefill(seqlens, 2, window, 0, t=t, what=f"prefill rising={rising} window={window}")


@pytest.mark.parametrize("rising", [True, False], ids=["rising", "falling"])
@pytest.mark.parametrize("window", [0, 128])
def test_decode_key_scale_drift(rising, window):
    lengths = (3000, 5000, 129)
    d = gi.make_decode_inputs(lengths, 2, 80 + window, device="cuda")
    positions = np.concatenate([np.arange(L) for L in lengths])
    d["k_cache"] = _scale_rows(d["k_cache"], positions, rising)
    out = gpu_decode(d, max(lengths), window)
    torch.cuda.synchronize()
    ref = oracle.decode(*decode_host_args(d), window)
    assert_close(out.float().cpu().numpy(), ref, f"decode rising={rising} window={window}")
