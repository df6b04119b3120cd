"""Context parallelism for long sequences (aitrends.kr/articles/94908, context-parallel
paragraph: full-attention layers cost Theta(L^2) and use Ulysses, the sequence <-> head
all-to-all; sliding-window layers cost Theta(L W) and only need each rank's W-token
neighbourhood, so the received K/V drops from Theta(L) to Theta(W)).

One sequence of T tokens is split in contiguous chunks over the R ranks of a process
group: rank r holds tokens [r C, (r+1) C), C = T / R, of every input tensor. Each rank
calls the same function with its chunk and gets its chunk of the output.

* ``swa_forward_cp`` (window W): one exchange step. Rank r sends the K and V rows of its
  last W - 1 tokens to rank r + 1 and receives rank r - 1's; it then runs the local
  windowed prefill over [halo; chunk] with zero query rows in front (their outputs are
  dropped), so every token sees exactly its W keys. Needs C >= W - 1.
* ``full_forward_ulysses`` (full causal): an all-to-all turns the R sequence chunks of all
  H KV groups into the whole sequence of H / R groups (a group's 4 signal heads, its
  noise head, K, V, lambda and gate move together), the local full-causal prefill runs on
  those groups, and a second all-to-all returns each rank its chunk of all 4H output
  heads. Needs H % R == 0.

The collectives are torch.distributed (NCCL on GPUs); the attention is this package's
``attn_fwd`` unless ``attn`` is given (same signature, used by the CPU tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .ops import DQK, DV


def _attn(attn):
    if attn is not None:
        return attn
    from .ops import attn_fwd
    return attn_fwd


def swa_forward_cp(q_sig, q_noise, k, v, lam, gate, window, group=None, attn=None):
    """Sliding-window GDLA over one sequence split in contiguous chunks across ``group``.

    Inputs are this rank's chunk: q_sig [C, 4H, 192], q_noise [C, H, 192], k [C, H, 192],
    v [C, H, 128], lam [C, 4H], gate [C, 4H, 128]. Returns this rank's out [C, 4H, 128].
    """
    if window <= 0:
        raise ValueError("swa_forward_cp needs a window > 0 (full causal: full_forward_ulysses)")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    c = q_sig.shape[0]
    halo = window - 1
    if c < halo:
        raise ValueError(f"chunk of {c} tokens is shorter than the halo of {halo} (window - 1)")
    if halo == 0 or world == 1:
        return _attn(attn)(q_sig, q_noise, k, v, lam, gate, (c,), window)
    # halo exchange: the last window-1 K/V rows go to the next rank (one send/recv pair per tensor)
    send_kv = torch.cat([k[c - halo:].reshape(halo, -1), v[c - halo:].reshape(halo, -1)], 1).contiguous()
    recv_kv = torch.empty_like(send_kv)
    peer = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    ops = []
    if rank + 1 < world:
        ops.append(dist.P2POp(dist.isend, send_kv, peer(rank + 1), group))
    if rank > 0:
        ops.append(dist.P2POp(dist.irecv, recv_kv, peer(rank - 1), group))
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    hkv = q_noise.shape[1]
    if rank == 0:
        return _attn(attn)(q_sig, q_noise, k, v, lam, gate, (c,), window)
    kd = hkv * DQK
    k_halo = recv_kv[:, :kd].reshape(halo, hkv, DQK)
    v_halo = recv_kv[:, kd:].reshape(halo, hkv, DV)
    pad = lambda t: torch.cat([torch.zeros((halo,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device), t], 0)
    out = _attn(attn)(pad(q_sig), pad(q_noise), torch.cat([k_halo, k], 0), torch.cat([v_halo, v], 0), pad(lam),
                      pad(gate), (halo + c,), window)
    return out[halo:]


def _to_groups(x, world, group):
    """[C, heads, ...] (this rank's tokens, all groups; heads group-major) -> all-to-all ->
    [world * C, heads / world, ...] (all tokens, this rank's block of groups)."""
    c = x.shape[0]
    tail = tuple(x.shape[2:])
    xs = x.reshape((c, world, -1) + tail).transpose(0, 1).contiguous()  # [world (dest), C, heads/world, ...]
    out = torch.empty_like(xs)
    dist.all_to_all_single(out, xs, group=group)                          # [world (source chunk), C, ...]
    return out.reshape((world * c,) + tuple(out.shape[2:]))


def _from_groups(y, world, group):
    """[world * C, heads / world, ...] (all tokens, this rank's groups) -> all-to-all ->
    [C, heads, ...] (this rank's tokens, all groups)."""
    c = y.shape[0] // world
    ys = y.reshape((world, c) + tuple(y.shape[1:])).contiguous()        # [world (dest chunk), C, ...]
    out = torch.empty_like(ys)
    dist.all_to_all_single(out, ys, group=group)                          # [world (source group block), C, ...]
    return out.transpose(0, 1).reshape((c, -1) + tuple(out.shape[3:]))


def full_forward_ulysses(q_sig, q_noise, k, v, lam, gate, group=None, attn=None):
    """Full-causal GDLA over one sequence split in contiguous chunks across ``group``
    (Ulysses: sequence <-> KV-group all-to-all before and after the attention).

    Inputs as ``swa_forward_cp``; H (KV groups) must be a multiple of the world size.
    Returns this rank's out [C, 4H, 128].
    """
    world = dist.get_world_size(group)
    hkv = q_noise.shape[1]
    if hkv % world:
        raise ValueError(f"{hkv} KV groups do not split over {world} ranks")
    qs, qn, kk, vv, ll, gg = (_to_groups(x, world, group) for x in (q_sig, q_noise, k, v, lam, gate))
    out = _attn(attn)(qs, qn, kk, vv, ll, gg, (qs.shape[0],), 0)
    return _from_groups(out, world, group)
