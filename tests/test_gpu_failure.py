"""Failure detection on the GPU without faulting it.

* A bounded device wait that runs out (the test hook withholds a K tile, so a
  barrier that nothing completes is waited on) must come back as
  MOGA_ERR_TIMEOUT from moga_sync_status, and the CUDA context must stay usable:
  the next call is checked against the oracle.
* Out-of-range offsets or permutation entries are skipped on the device and
  reported as MOGA_ERR_DEVICE_CHECK.
"""
import ctypes

import numpy as np
import pytest
import torch

import learned_token_group_b200 as moga
import oracle
from parity import compare_out, groups_to_perm, np_cpu
from workloads import custom, make_inputs

pytestmark = pytest.mark.gpu

TIMEOUT, DEVICE_CHECK = 5, 6


def _case(N=700, H=2, M=3, seed=3):
    inp = make_inputs(custom(N, H=H, d_h=128, d=64, M=M), seed=seed, device="cuda")
    rng = np.random.default_rng(seed)
    gid = rng.integers(0, M, size=N)
    gate = rng.uniform(1.0 / M, 1.0, size=N)
    perm, offsets = groups_to_perm(gid, M)
    t = lambda a: torch.from_numpy(a).cuda()
    return inp, gid, gate, t(perm), t(offsets), t(gate.astype(np.float32))


def _ws(N, H, M):
    return moga.workspace(moga.get_lib().moga_group_attn_workspace_size(N, H, 128, M), "cuda")


def _status(ws):
    return moga.get_lib().moga_sync_status(ctypes.c_void_p(ws.data_ptr()),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_wait_timeout_reported_and_context_survives():
    lib = moga.get_lib()
    N, H, M = 700, 2, 3
    inp, gid, gate, perm, offsets, gate_t = _case(N, H, M)
    ws = _ws(N, H, M)
    old = lib.moga_set_wait_limit_ns(50_000_000)
    try:
        assert lib.moga_debug_inject(1) == 0
        moga.group_attn(inp["q"], inp["k"], inp["v"], perm, offsets, gate_t, M, ws=ws)
        assert _status(ws) == TIMEOUT
    finally:
        lib.moga_debug_inject(0)
        lib.moga_set_wait_limit_ns(old)
    assert _status(ws) == 0                      # the status word was cleared by the read
    out = moga.group_attn(inp["q"], inp["k"], inp["v"], perm, offsets, gate_t, M, ws=ws)
    moga.sync_status(ws)
    ref = oracle.group_attention(np_cpu(inp["q"]), np_cpu(inp["k"]), np_cpu(inp["v"]), gid, gate, M)
    compare_out(out, ref, groups=gid)


def test_bad_offsets_reported():
    N, H, M = 500, 1, 4
    inp, gid, gate, perm, offsets, gate_t = _case(N, H, M)
    bad = offsets.clone()
    bad[-1] = N - 1                              # offsets[M] != N
    ws = _ws(N, H, M)
    moga.group_attn(inp["q"], inp["k"], inp["v"], perm, bad, gate_t, M, ws=ws)
    assert _status(ws) == DEVICE_CHECK


def test_bad_perm_reported():
    N, H, M = 500, 1, 4
    inp, gid, gate, perm, offsets, gate_t = _case(N, H, M)
    bad = perm.clone()
    bad[7] = N                                   # one out-of-range token index
    ws = _ws(N, H, M)
    moga.group_attn(inp["q"], inp["k"], inp["v"], bad, offsets, gate_t, M, ws=ws)
    assert _status(ws) == DEVICE_CHECK
    assert _status(ws) == 0


@pytest.mark.parametrize("window", [(3, 8, 8), (2, 10, 12), (2, 30, 52)])
def test_window_kernels_time_out_cleanly(window):
    """The same hook on the STGA kernels: the whole-window box kernel (3x8x8),
    the general in-place plan (240-token windows) and the tiled loads of whole
    frames.  Each producer gives up, the bounded waits run out, the status
    says so, and the next call matches the oracle."""
    lib = moga.get_lib()
    grid = (4, 30, 52)
    N = 4 * 30 * 52
    inp = make_inputs(custom(N, H=2, d_h=128, d=64, M=2), seed=8, device="cuda")
    ws = moga.workspace(lib.stga_window_attn_workspace_size(*grid, (ctypes.c_int * 3)(*window), 2, 128), "cuda")
    old = lib.moga_set_wait_limit_ns(50_000_000)
    try:
        assert lib.moga_debug_inject(1) == 0
        moga.stga_window_attn(inp["q"], inp["k"], inp["v"], grid, window, ws=ws)
        assert _status(ws) == TIMEOUT
    finally:
        lib.moga_debug_inject(0)
        lib.moga_set_wait_limit_ns(old)
    out = moga.stga_window_attn(inp["q"], inp["k"], inp["v"], grid, window, ws=ws)
    moga.sync_status(ws)
    ref = oracle.stga_attention(np_cpu(inp["q"]), np_cpu(inp["k"]), np_cpu(inp["v"]), *grid, window)
    compare_out(out, ref)
