"""Grouped attention and STGA window attention on the GPU against the oracle.

Grouped attention: "MoGA: Mixture-of-Groups Attention for End-to-End Long Video
Generation" (paper-graph-ui summary), §3.4 "Grouped Attention" (Eq. 5) and
Algorithm 1 steps 2-4; STGA: same section, "Spatial-Temporal Group Attention".
"""
import numpy as np
import pytest
import torch

import learned_token_group_b200 as moga
import oracle
from parity import compare_out, groups_to_perm, np_cpu
from workloads import custom, make_inputs

pytestmark = pytest.mark.gpu


def _qkv(N, H, d_h, seed, peaky=False):
    wl = custom(N, H=H, d_h=d_h, d=64, M=2, peaky=peaky)
    inp = make_inputs(wl, seed=seed, device="cuda")
    return inp["q"], inp["k"], inp["v"]


def _run_groups(q, k, v, gid, gate_np, M, out_scale=1.0):
    perm, offsets = groups_to_perm(gid, M)
    dev = q.device
    gate = None if gate_np is None else torch.from_numpy(gate_np.astype(np.float32)).to(dev)
    out = moga.group_attn(q, k, v, torch.from_numpy(perm).to(dev), torch.from_numpy(offsets).to(dev), gate, M,
                          out_scale=out_scale)
    ws = None
    torch.cuda.synchronize()
    return out


GROUP_CASES = [
    # (N, H, d_h, M, sizes or None)
    (1, 1, 64, 1, None),
    (200, 2, 64, 3, None),
    (300, 2, 128, 4, None),
    (1000, 1, 64, 4, None),
    (1500, 3, 128, 1, None),                          # M = 1: full attention
    (700, 2, 128, 7, [0, 1, 127, 128, 129, 0, 315]),   # empty, singleton, tile edges
    (2600, 1, 128, 3, [2048, 1, 551]),                # many KV tiles + ragged tail
    # segment ends around a unit of two 128-row query tiles: one row into the
    # third tile, a unit and a half, one row past it, two full units, one row
    # over, a single short tile
    (2100, 2, 128, 6, [257, 384, 385, 512, 513, 49]),
    # the largest group count the library takes: 1024 groups of a few tokens
    # (some empty), one short tile each
    (6000, 2, 128, 1024, None),
]


@pytest.mark.parametrize("N,H,d_h,M,sizes", GROUP_CASES)
def test_group_attn(N, H, d_h, M, sizes):
    rng = np.random.default_rng(N + 7 * M)
    if sizes is None:
        gid = rng.integers(0, M, size=N)
    else:
        assert sum(sizes) == N
        gid = rng.permutation(np.repeat(np.arange(M), sizes))
    gate = rng.uniform(1.0 / M, 1.0, size=N)
    q, k, v = _qkv(N, H, d_h, seed=N)
    out = _run_groups(q, k, v, gid, gate, M)
    ref = oracle.group_attention(np_cpu(q), np_cpu(k), np_cpu(v), gid, gate.astype(np.float32), M)
    compare_out(out, ref, groups=gid)


def test_group_attn_no_gate_and_scale():
    N, H, M = 400, 2, 3
    rng = np.random.default_rng(3)
    gid = rng.integers(0, M, size=N)
    q, k, v = _qkv(N, H, 128, seed=5)
    out = _run_groups(q, k, v, gid, None, M, out_scale=0.5)
    ref = 0.5 * oracle.group_attention(np_cpu(q), np_cpu(k), np_cpu(v), gid, np.ones(N), M)
    compare_out(out, ref, groups=gid)


def test_group_attn_peaky_rescaling():
    # each query's own key dominates: exercises the online-softmax max tracking
    N, H, M = 1100, 2, 2
    rng = np.random.default_rng(9)
    gid = rng.integers(0, M, size=N)
    q, k, v = _qkv(N, H, 128, seed=21, peaky=True)
    gate = np.ones(N)
    out = _run_groups(q, k, v, gid, gate, M)
    ref = oracle.group_attention(np_cpu(q), np_cpu(k), np_cpu(v), gid, gate, M)
    compare_out(out, ref, groups=gid)


def test_group_attn_permutation_equivariance():
    # property at any size: shuffling tokens shuffles the output rows
    N, H, M = 900, 2, 5
    rng = np.random.default_rng(4)
    gid = rng.integers(0, M, size=N)
    gate = rng.uniform(0.2, 1, size=N)
    q, k, v = _qkv(N, H, 128, seed=8)
    a = _run_groups(q, k, v, gid, gate, M)
    pi = rng.permutation(N)
    pit = torch.from_numpy(pi).cuda()
    b = _run_groups(q[pit].contiguous(), k[pit].contiguous(), v[pit].contiguous(), gid[pi], gate[pi], M)
    diff = (a[pit].float() - b.float()).abs().max().item()
    assert diff <= 2e-2


STGA_CASES = [
    # (grid, window, H, d_h)
    ((3, 10, 12), (3, 8, 8), 2, 128),
    ((2, 5, 6), (2, 4, 4), 1, 64),
    ((1, 4, 6), (1, 4, 6), 2, 128),      # window = whole grid: full attention
    ((6, 30, 52), (3, 8, 8), 2, 128),    # the 480p latent grid, clipped edges
    ((2, 9, 7), (5, 16, 16), 1, 128),    # window larger than the grid
    # whole-frame windows: runs of consecutive tokens, read in place
    ((2, 30, 52), (1, 30, 52), 2, 128),  # per-frame attention, 1560 tokens (ragged tail)
    ((5, 30, 52), (2, 30, 52), 1, 64),   # two frames per window, last window clipped
    ((3, 7, 9), (2, 20, 20), 2, 64),     # wider than the frame, shorter than the clip
    # windows of up to 192 tokens loaded as whole boxes: every clip kind, box
    # sizes that use one or two query tiles, a second tile with one live warp
    ((5, 10, 12), (3, 8, 8), 3, 128),    # T not a multiple of wt: clipped in time too
    ((4, 30, 52), (3, 8, 8), 1, 64),     # d_h 64 on the 480p grid
    ((2, 9, 20), (2, 4, 8), 2, 128),     # 64-token boxes
    ((3, 16, 40), (1, 8, 16), 2, 128),   # 128-token boxes: one query tile
    ((3, 13, 23), (3, 6, 10), 2, 128),   # 180-token boxes, clipped in rows and columns
    ((2, 25, 25), (1, 12, 12), 2, 128),  # 144 tokens: the second tile's last warp holds no row
    ((3, 5, 6), (3, 8, 8), 2, 128),      # box larger than the grid in rows and columns
    ((2, 8, 8), (3, 8, 8), 2, 128),      # fewer frames than the window's extent
    ((1, 1, 1), (3, 8, 8), 3, 64),       # a single token
]


@pytest.mark.parametrize("grid,window,H,d_h", STGA_CASES)
def test_stga(grid, window, H, d_h):
    N = grid[0] * grid[1] * grid[2]
    q, k, v = _qkv(N, H, d_h, seed=N + 1)
    out = moga.stga_window_attn(q, k, v, grid, window)
    torch.cuda.synchronize()
    ref = oracle.stga_attention(np_cpu(q), np_cpu(k), np_cpu(v), *grid, window)
    win = np.zeros(N, dtype=np.int64)
    for i, idx in enumerate(oracle.stga_windows(*grid, window)):
        win[idx] = i
    compare_out(out, ref, groups=win)


def test_stga_unit_window_is_v():
    grid = (2, 3, 4)
    q, k, v = _qkv(24, 2, 64, seed=2)
    out = moga.stga_window_attn(q, k, v, grid, (1, 1, 1))
    torch.cuda.synchronize()
    assert (out.float() - v.float()).abs().max().item() == 0.0


@pytest.mark.parametrize("window", [(3, 8, 8), (1, 10, 12)])
def test_stga_accumulate(window):
    grid = (3, 10, 12)
    N = 360
    q, k, v = _qkv(N, 2, 128, seed=77)
    base = torch.randn((N, 2, 128), device="cuda").to(torch.bfloat16)
    out = base.clone()
    moga.stga_window_attn(q, k, v, grid, window, accumulate=True, out=out)
    torch.cuda.synchronize()
    ref = np_cpu(base).astype(np.float64) + 0.5 * oracle.stga_attention(np_cpu(q), np_cpu(k), np_cpu(v), *grid,
                                                                         window)
    compare_out(out, ref)
