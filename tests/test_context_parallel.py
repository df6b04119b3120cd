"""Context parallelism (differential_latent_attention_b200.context_parallel) on CPU:
gloo ranks (world size 2 and 4), the local attention supplied by the fp64 oracle.
Each rank holds a contiguous chunk of one sequence; the chunks of the output,
gathered, must equal the oracle on the whole sequence exactly (the same keys are
visited in the same order, so the fp64 sums are identical)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_attn(q_sig, q_noise, k, v, lam, gate, seqlens, window):
    """attn_fwd's signature over CPU tensors holding bf16 values (as float32)."""
    import gdla_inputs as gi
    import oracle
    bits = [gi.bf16_bits(t.to(torch.bfloat16)) for t in (q_sig, q_noise, k, v)]
    out = oracle.prefill(*bits, lam.numpy().astype(np.float32), gi.bf16_bits(gate.to(torch.bfloat16)), seqlens,
                         window, num_threads=2)
    return torch.from_numpy(out)


def _inputs(T, hkv, seed):
    import gdla_inputs as gi
    t = gi.make_prefill_inputs((T,), hkv, seed)
    # float32 carriers of the bf16 values (gloo moves float32; the oracle re-reads them exactly)
    return {k: (v.to(torch.float32) if v.dtype == torch.bfloat16 else v) for k, v in t.items()}


def _worker(rank, world, port, mode, T, hkv, window, q):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    from differential_latent_attention_b200 import context_parallel as cp
    t = _inputs(T, hkv, 3)
    c = T // world
    chunk = {k: v[rank * c:(rank + 1) * c].contiguous() for k, v in t.items()}
    args = (chunk["q_sig"], chunk["q_noise"], chunk["k"], chunk["v"], chunk["lam"], chunk["gate"])
    if mode == "swa":
        out = cp.swa_forward_cp(*args, window, attn=_oracle_attn)
    else:
        out = cp.full_forward_ulysses(*args, attn=_oracle_attn)
    q.put((rank, out.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("mode,world,window", [("swa", 2, 8), ("swa", 4, 8), ("swa", 4, 25),
                                               ("ulysses", 2, 0), ("ulysses", 4, 0)])
def test_chunks_equal_the_whole_sequence(mode, world, window):
    T, hkv = 96, 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, T, hkv, window, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = np.concatenate([parts[r] for r in range(world)], 0)
    t = _inputs(T, hkv, 3)
    ref = _oracle_attn(t["q_sig"], t["q_noise"], t["k"], t["v"], t["lam"], t["gate"], (T,), window).numpy()
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


def _error_worker(rank, world, port, q):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from differential_latent_attention_b200 import context_parallel as cp
    caught = []
    for hkv, window, fn in ((4, 60, "swa"), (4, 0, "swa"), (3, 0, "ulysses")):
        t = _inputs(96, hkv, 5)
        c = 96 // world
        chunk = [t[k][rank * c:(rank + 1) * c].contiguous() for k in ("q_sig", "q_noise", "k", "v", "lam", "gate")]
        try:
            if fn == "swa":
                cp.swa_forward_cp(*chunk, window, attn=_oracle_attn)
            else:
                cp.full_forward_ulysses(*chunk, attn=_oracle_attn)
        except ValueError:
            caught.append((hkv, window, fn))
    dist.barrier()   # every rank raised before any exchange, so the group is still in step
    q.put((rank, caught))
    dist.destroy_process_group()


def test_unsupported_splits_raise_on_every_rank_before_any_exchange():
    """A chunk shorter than the window's halo, a window of 0 for the halo scheme and a
    KV-group count the world size does not divide each raise ValueError on every rank,
    before any collective (the ranks stay in step and finish a barrier afterwards)."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_error_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == [(4, 60, "swa"), (4, 0, "swa"), (3, 0, "ulysses")], res[r]
