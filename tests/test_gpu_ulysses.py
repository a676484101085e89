"""moga_sort (the counting sort of caller-given group ids) and the
sequence-parallel block on one GPU.

moga_sort must reproduce the oracle's stable counting sort bit for bit and
report ids outside [0, M).  The sequence-parallel path (ulysses_layer) with a
single rank over NCCL exchanges nothing: its routing and output are compared
with the oracle (group ids with the near-tie rule, gate, and per group the
block output), and it must also equal moga_layer bit for bit (same routing,
same sort, same kernels in the same order).  Its two-rank exchange is checked
on the CPU (tests/test_multirank_cpu.py).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import learned_token_group_b200 as moga
import oracle
from parity import GATE_TOL_BF16, MARGIN, compare_out, np_cpu
from workloads import custom, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,M", [(0, 4), (1, 3), (127, 2), (1000, 7), (4097, 64), (20000, 300), (5000, 1024)])
def test_sort_matches_oracle(N, M):
    rng = np.random.default_rng(N + M)
    gid = rng.integers(0, M, size=N).astype(np.int32)
    res = moga.sort(torch.from_numpy(gid).cuda(), M)
    moga.sync_status(res["ws"])
    perm, offsets, mx = oracle.counting_sort(gid, M)
    assert np.array_equal(np_cpu(res["offsets"]), offsets)
    assert int(np_cpu(res["max_seqlen"])[0]) == mx
    if N:
        assert np.array_equal(np_cpu(res["perm"]), perm)


def test_sort_reports_bad_ids():
    gid = torch.zeros(500, dtype=torch.int32, device="cuda")
    gid[17] = 4                                   # M = 4: one id out of range
    res = moga.sort(gid, 4)
    with pytest.raises(moga.MogaError) as e:
        moga.sync_status(res["ws"])
    assert e.value.status == 6
    assert int(np_cpu(res["offsets"])[-1]) == 499  # the bad token is left out


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("window", [None, (3, 8, 8)])
def test_sequence_parallel_single_rank_equals_layer(window):
    from learned_token_group_b200.ulysses import ulysses_layer
    grid = (3, 16, 20)
    wl = custom(960, H=4, d_h=128, d=256, M=5, x_kind="clustered", grid=grid, window=window, name="sp")
    inp = make_inputs(wl, seed=12, device="cuda")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out, gid, gate = ulysses_layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M,
                                       grid, window)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = moga.moga_layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M,
                          grid if window else None, window)
    moga.sync_status(ref["ws"])
    # against the oracle
    ref_gid, ref_gate, margin = oracle.route(np_cpu(inp["x"]), np_cpu(inp["W_r"]), None)
    g = np_cpu(gid).astype(np.int64)
    assert not ((g != ref_gid) & (margin >= MARGIN)).any()
    same = g == ref_gid
    assert np.abs(np_cpu(gate)[same] - ref_gate[same]).max() <= GATE_TOL_BF16
    q, k, v = (np_cpu(inp[n]) for n in "qkv")
    want = oracle.group_attention(q, k, v, g, np_cpu(gate).astype(np.float64), wl.M)
    if window:
        want = 0.5 * (want + oracle.stga_attention(q, k, v, *grid, window))
    compare_out(out, want, groups=g)
    # and bit for bit against the single-device block
    assert torch.equal(gid, ref["group_id"]) and torch.equal(gate, ref["gate"])
    assert torch.equal(out, ref["out"])
