"""The kernels' failure path on the GPU, without a fault: a bounded wait on an
mbarrier that nothing arrives on runs out (after about a second), records its
site in the device failure word and returns; the host reads the code, clears
it, and the same context then computes a correct result."""
import pytest
import torch

import differential_latent_attention_b200 as gdla
from differential_latent_attention_b200 import ops
from _parity import check_prefill

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    assert gdla.device_error(clear=True) in (0, ops.SELFTEST_SITE)
    ops.selftest_wait_timeout()
    assert gdla.device_error(clear=False) == ops.SELFTEST_SITE   # synchronises: the kernel returned
    assert gdla.device_error(clear=True) == ops.SELFTEST_SITE
    assert gdla.device_error(clear=True) == 0                    # cleared
    # the context is intact: a regular call still matches the oracle and records nothing
    check_prefill((70, 130), 2, 0, 19)
    torch.cuda.synchronize()
    assert gdla.device_error() == 0
