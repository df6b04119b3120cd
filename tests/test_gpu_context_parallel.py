"""Context parallelism on the GPU with NCCL. Only one GPU is available to a test, so
this runs one rank: the Ulysses all-to-alls (over NCCL, bf16) and the SWA entry
(no halo on one rank) must reproduce attn_fwd bit for bit. The multi-rank exchange
logic is covered on CPU (test_context_parallel.py, gloo, 2 and 4 ranks)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(port, q):
    import torch.distributed as dist
    from datetime import timedelta
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=120))
    import differential_latent_attention_b200 as gdla
    from differential_latent_attention_b200 import context_parallel as cp
    import gdla_inputs as gi
    T, hkv = 1000, 4
    t = gi.make_prefill_inputs((T,), hkv, 5, device="cuda")
    args = (t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"])
    ok = []
    ref = gdla.attn_fwd(*args, (T,), 0)
    ok.append(torch.equal(cp.full_forward_ulysses(*args), ref))
    ref = gdla.attn_fwd(*args, (T,), 128)
    ok.append(torch.equal(cp.swa_forward_cp(*args, 128), ref))
    torch.cuda.synchronize()
    ok.append(gdla.device_error() == 0)
    dist.destroy_process_group()
    q.put(ok)


def test_single_rank_matches_attn_fwd():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_worker, args=(_free_port(), q))
    p.start()
    ok = q.get(timeout=300)
    p.join(timeout=120)
    assert p.exitcode == 0
    assert ok == [True, True, True]
