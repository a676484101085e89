"""The whole MoGA block (moga_layer, C ABI) on the GPU against the oracle.

"MoGA: Mixture-of-Groups Attention for End-to-End Long Video Generation"
(paper-graph-ui summary), §3.4: router (Eqs. 2-4), grouped attention (Eq. 5,
Algorithm 1), STGA, and the mean of the two branches.

Small workloads are compared on every output row.  At full size the oracle
computes a seeded sample of rows exactly (each sampled row still sees its whole
group / window), in the launch configuration the benchmark times: every row of
the two smallest non-empty groups, 256 rows of every other group and 1,024
STGA rows spread over whole and clipped windows, on all heads.
"""
import numpy as np
import pytest
import torch

import learned_token_group_b200 as moga
import oracle
from parity import GATE_TOL_BF16, GATE_TOL_F32, check_route, compare_out, np_cpu, sample_rows
from workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu


def _layer(wl, seed):
    inp = make_inputs(wl, seed=seed, device="cuda")
    res = moga.moga_layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M, wl.grid,
                          wl.window)
    moga.sync_status(res["ws"])
    return inp, res


def test_layer_empty_input():
    """N = 0 tokens: nothing to route or attend; the call succeeds, the
    offsets are all zero and nothing is written."""
    wl = custom(64, H=2, d_h=128, d=128, M=5, name="empty")
    inp = make_inputs(wl, seed=1, device="cuda")
    cut = {k: (v[:0] if k in ("x", "q", "k", "v") else v) for k, v in inp.items()}
    res = moga.moga_layer(cut["x"], cut["W_r"], cut["b_r"], cut["q"], cut["k"], cut["v"], wl.M)
    moga.sync_status(res["ws"])
    assert res["out"].shape == (0, 2, 128)
    assert np.array_equal(np_cpu(res["offsets"]), np.zeros(wl.M + 1, dtype=np.int32))


def test_layer_max_groups():
    """The largest group count (M = 1024, the SIMT router): every token's
    group and gate against the oracle, and every row of the output."""
    wl = custom(4096, H=2, d_h=128, d=256, M=1024, x_kind="clustered", name="m1024")
    inp, res = _layer(wl, seed=3)
    gid, info = check_route(res, inp["x"], inp["W_r"], inp["b_r"], wl.M, GATE_TOL_BF16)
    gate = np_cpu(res["gate"]).astype(np.float64)
    q, k, v = (np_cpu(inp[n]) for n in "qkv")
    compare_out(res["out"], oracle.group_attention(q, k, v, gid, gate, wl.M), groups=gid)


SMALL = [
    WORKLOADS["tiny"],
    custom(384, H=2, d_h=128, d=256, M=4, x_kind="clustered", grid=(3, 8, 16), window=(3, 8, 8), name="small_stga"),
    custom(2 * 30 * 52, H=1, d_h=64, d=128, M=6, x_kind="clustered", grid=(2, 30, 52), window=(3, 8, 8),
           name="frame_grid"),
    custom(1000, H=2, d_h=128, d=128, M=1, name="m1_full"),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_layer_small(wl):
    inp, res = _layer(wl, seed=1)
    gid, info = check_route(res, inp["x"], inp["W_r"], inp["b_r"], wl.M,
                            GATE_TOL_F32 if wl.x_dtype == "f32" else GATE_TOL_BF16)
    gate = np_cpu(res["gate"]).astype(np.float64)
    q, k, v = (np_cpu(inp[n]) for n in "qkv")
    moga_ref = oracle.group_attention(q, k, v, gid, gate, wl.M)
    ref = moga_ref
    if wl.window is not None:
        ref = 0.5 * (moga_ref + oracle.stga_attention(q, k, v, *wl.grid, wl.window))
    compare_out(res["out"], ref, groups=gid)


@pytest.mark.parametrize("name", ["wan_32k", "video_187k", "skew_187k", "minute_580k"])
def test_layer_workload(name):
    wl = WORKLOADS[name]
    inp, res = _layer(wl, seed=0)
    gid, info = check_route(res, inp["x"], inp["W_r"], inp["b_r"], wl.M, GATE_TOL_BF16)
    rng = np.random.default_rng(123)
    # every row of the two smallest groups, 256 rows of every other group and
    # 1,024 STGA rows over all window kinds (whole and clipped), on every head
    # (at 580k the oracle needs about 3 s of host time per head)
    rows = sample_rows(gid, wl.M, wl.grid, wl.window, rng, per_group=256, stga_rows=1024)
    heads = list(range(wl.H))
    gate = np_cpu(res["gate"]).astype(np.float64)
    # the oracle reads only the rows/heads it needs, straight from the seeded inputs
    q, k, v = inp["q"], inp["k"], inp["v"]
    moga_ref = oracle.group_attention(q, k, v, gid, gate, wl.M, rows=rows, heads=heads)
    stga_ref = oracle.stga_attention(q, k, v, *wl.grid, wl.window, rows=rows, heads=heads)
    ref = 0.5 * (moga_ref + stga_ref)          # [len(rows), len(heads), d_h]
    out = res["out"][torch.from_numpy(rows).cuda()][:, heads]
    compare_out(out, ref, groups=gid[rows])
    print(f"{name}: checked {rows.size} rows x {len(heads)} heads; near-ties {info['n_near']}")


@pytest.mark.parametrize("name", ["wan_32k"])
def test_layer_bitwise_deterministic(name):
    """Two runs on the same inputs give identical bits (no order-dependent
    reductions anywhere on the path)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=4, device="cuda")
    layer = moga.MogaLayer(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window, torch.bfloat16, "cuda")
    outs = []
    for _ in range(2):
        layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"])
        moga.sync_status(layer.ws)
        outs.append((layer.out.clone(), layer.perm.clone(), layer.gate.clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


THREE = [
    custom(384, H=2, d_h=128, d=256, M=4, x_kind="clustered", grid=(3, 8, 16), window=(3, 8, 8), name="small3"),
    custom(2 * 30 * 52, H=1, d_h=64, d=128, M=6, x_kind="clustered", grid=(2, 30, 52), window=(3, 8, 8),
           name="frame_grid3"),
]


@pytest.mark.parametrize("wl", THREE, ids=[w.name for w in THREE])
def test_layer_three_branches(wl):
    """MoGA + STGA + per-frame attention, averaged (moga_layer_ex, branches = 3)."""
    inp = make_inputs(wl, seed=2, device="cuda")
    res = moga.moga_layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M, wl.grid,
                          wl.window, per_frame=True)
    moga.sync_status(res["ws"])
    gid, _ = check_route(res, inp["x"], inp["W_r"], inp["b_r"], wl.M, GATE_TOL_BF16)
    gate = np_cpu(res["gate"]).astype(np.float64)
    q, k, v = (np_cpu(inp[n]) for n in "qkv")
    ref = (oracle.group_attention(q, k, v, gid, gate, wl.M) + oracle.stga_attention(q, k, v, *wl.grid, wl.window)
           + oracle.frame_attention(q, k, v, *wl.grid)) / 3
    compare_out(res["out"], ref, groups=gid)


@pytest.mark.parametrize("name,heads_all", [("wan_32k", False), ("video_187k", True)])
def test_layer_three_branches_sampled(name, heads_all):
    """The three-branch block at full size, in the launch configuration of
    the bench's widened row: sampled rows of every group and of every window
    kind, compared in full (whole group, window and frame attended)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=3, device="cuda")
    res = moga.moga_layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M, wl.grid,
                          wl.window, per_frame=True)
    moga.sync_status(res["ws"])
    gid, _ = check_route(res, inp["x"], inp["W_r"], inp["b_r"], wl.M, GATE_TOL_BF16)
    rows = sample_rows(gid, wl.M, wl.grid, wl.window, np.random.default_rng(5), per_group=64, stga_rows=256)
    heads = list(range(wl.H)) if heads_all else [0, wl.H - 1]
    gate = np_cpu(res["gate"]).astype(np.float64)
    q, k, v = inp["q"], inp["k"], inp["v"]
    ref = (oracle.group_attention(q, k, v, gid, gate, wl.M, rows=rows, heads=heads)
           + oracle.stga_attention(q, k, v, *wl.grid, wl.window, rows=rows, heads=heads)
           + oracle.frame_attention(q, k, v, *wl.grid, rows=rows, heads=heads)) / 3
    out = res["out"][torch.from_numpy(rows).cuda()][:, heads]
    compare_out(out, ref, groups=gid[rows])


def test_layer_replays_in_a_cuda_graph():
    """A whole layer (router, sort, gathers, both attention kernels) captured
    into a CUDA graph replays to the same bits as eager calls, also after the
    inputs are overwritten in place."""
    wl = WORKLOADS["wan_32k"]
    inp = make_inputs(wl, seed=5, device="cuda")
    layer = moga.MogaLayer(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window, torch.bfloat16, "cuda")
    args = lambda: (inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"])
    layer(*args())
    moga.sync_status(layer.ws)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer(*args())
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer(*args())
    for seed in (5, 6):
        new = make_inputs(wl, seed=seed, device="cuda")
        for key in ("x", "q", "k", "v"):
            inp[key].copy_(new[key])
        layer.out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        moga.sync_status(layer.ws)
        got = layer.out.clone()
        layer(*args())
        moga.sync_status(layer.ws)
        assert torch.equal(got, layer.out)
