"""Sequence parallelism for the MoGA block over P ranks.

"MoGA: Mixture-of-Groups Attention for End-to-End Long Video Generation"
(paper-graph-ui summary, §3.4) trains with DeepSpeed-Ulysses sequence
parallelism: routing runs on each rank's own tokens, the routing results are
aggregated, and attention heads are exchanged all-to-all so that every rank
holds all tokens of a subset of the heads.  This module is that exchange
around the library's kernels:

1. each rank routes its n = N / P consecutive tokens (``ops.route``);
2. group ids and gates of all N tokens are all-gathered (N ints + N floats);
3. q, k, v go all-to-all from token shards [n, H, d_h] to head shards
   [N, H / P, d_h] (rank r keeps heads [r H/P, (r+1) H/P));
4. each rank sorts the gathered ids and runs the block (grouped attention,
   optionally STGA and the mean) for its heads over all N tokens
   (``ops.block``);
5. the outputs go all-to-all back to token shards [n, H, d_h].

The collectives are torch.distributed calls (NCCL on GPUs, gloo on the CPU);
``ops`` supplies the compute, by default the CUDA library.  Token order is
frame-major and shards are consecutive, so STGA windows stay whole on every
rank after the exchange.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch
import torch.distributed as dist


def seq_to_heads(t: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """[n, H, D] token shard -> [world * n, H / world, D] head shard (all-to-all)."""
    n, H, D = t.shape
    hp = H // world
    send = t.reshape(n, world, hp, D).permute(1, 0, 2, 3).contiguous()  # block p goes to rank p
    recv = torch.empty_like(send)                                        # block p came from rank p
    dist.all_to_all_single(recv, send, group=group)
    return recv.reshape(world * n, hp, D)


def heads_to_seq(t: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """[world * n, H / world, D] head shard -> [n, H, D] token shard (all-to-all)."""
    N, hp, D = t.shape
    n = N // world
    send = t.reshape(world, n, hp, D).contiguous()   # tokens of rank p go to rank p
    recv = torch.empty_like(send)                    # head block p came from rank p
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3).reshape(n, world * hp, D)


def all_gather_1d(t: torch.Tensor, world: int, group=None) -> torch.Tensor:
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.cat(parts)


class CudaOps:
    """The library's kernels as the compute of ``ulysses_layer``."""

    @staticmethod
    def route(x, W_r, b_r, M):
        from . import route
        r = route(x, W_r, b_r, M)
        return r["group_id"], r["gate"]

    @staticmethod
    def block(q, k, v, group_id, gate, M, grid=None, window=None):
        from . import group_attn, sort, stga_window_attn, sync_status
        s = sort(group_id, M)
        out = group_attn(q, k, v, s["perm"], s["offsets"], gate, M, out_scale=0.5 if window else 1.0)
        if window:
            stga_window_attn(q, k, v, grid, window, accumulate=True, out=out)
        sync_status(s["ws"])
        return out


def ulysses_layer(x: torch.Tensor, W_r: torch.Tensor, b_r: Optional[torch.Tensor], q: torch.Tensor,
                  k: torch.Tensor, v: torch.Tensor, M: int, grid: Optional[Sequence[int]] = None,
                  window: Optional[Sequence[int]] = None, group=None, ops=None):
    """The MoGA block on this rank's token shard; returns (out, group_id, gate)
    for the shard, equal to the single-device block's rows of these tokens.

    x [n, d], q/k/v [n, H, d_h] with n = N / P consecutive tokens and H a
    multiple of P; grid (T, Hg, Wg) describes all N tokens.  1 <= M <= 1024,
    the group limit of the library's routing and counting sort.
    """
    world = dist.get_world_size(group)
    n, H, _ = q.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    if not 1 <= M <= 1024:
        raise ValueError(f"M = {M} groups: routing and sorting take 1 to 1024")
    ops = ops or CudaOps
    gid_local, gate_local = ops.route(x, W_r, b_r, M)
    gid = all_gather_1d(gid_local, world, group)
    gate = all_gather_1d(gate_local, world, group)
    qh, kh, vh = (seq_to_heads(t, world, group) for t in (q, k, v))
    out_h = ops.block(qh, kh, vh, gid, gate, M, grid, window)
    return heads_to_seq(out_h, world, group), gid_local, gate_local
