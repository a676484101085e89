"""Router + counting sort on the GPU against the oracle (moga_route, C ABI).

Router and gate: "MoGA: Mixture-of-Groups Attention for End-to-End Long Video
Generation" (paper-graph-ui summary), §3.4 "MoGA Router", Eqs. 2-4; counting
sort: "MoGA Pseudocode and Kernel Integration", Algorithm 1 step 2.
"""
import numpy as np
import pytest
import torch

import learned_token_group_b200 as moga
from parity import GATE_TOL_BF16, GATE_TOL_F32, check_route, np_cpu
from workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # (N, d, M, dtype, kind)
    (1, 64, 4, "bf16", "normal"),
    (127, 64, 1, "bf16", "normal"),
    (129, 128, 5, "bf16", "normal"),
    (1000, 256, 16, "bf16", "clustered"),
    (3000, 512, 64, "bf16", "skew"),
    (2000, 320, 300, "bf16", "normal"),      # M beyond the tensor-core path: SIMT router
    (4097, 1536, 8, "bf16", "clustered"),
    (5000, 104, 24, "bf16", "normal"),       # d not a multiple of 64: zero-filled K tail
    (777, 64, 7, "f32", "normal"),
]


@pytest.mark.parametrize("N,d,M,dt,kind", CASES)
def test_route_small(N, d, M, dt, kind):
    wl = custom(N, d=d, M=M, x_dtype=dt, x_kind=kind)
    inp = make_inputs(wl, seed=11, device="cuda", with_qkv=False)
    res = moga.route(inp["x"], inp["W_r"], inp["b_r"], M)
    torch.cuda.synchronize()
    check_route(res, inp["x"], inp["W_r"], inp["b_r"], M, GATE_TOL_F32 if dt == "f32" else GATE_TOL_BF16)


def test_route_empty():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.randn((4, 64), device="cuda").to(torch.bfloat16)
    res = moga.route(x, W, None, 4)
    torch.cuda.synchronize()
    assert np_cpu(res["offsets"]).tolist() == [0] * 5 and int(np_cpu(res["max_seqlen"])[0]) == 0


def test_route_ties_lowest_group():
    # x = 0 gives equal logits everywhere: every token goes to group 0, gate 1/M
    x = torch.zeros((300, 128), dtype=torch.bfloat16, device="cuda")
    W = torch.randn((12, 128), device="cuda").to(torch.bfloat16)
    res = moga.route(x, W, None, 12)
    torch.cuda.synchronize()
    assert (np_cpu(res["group_id"]) == 0).all()
    assert np.allclose(np_cpu(res["gate"]), 1 / 12, atol=1e-7)
    assert np_cpu(res["perm"]).tolist() == list(range(300))


@pytest.mark.parametrize("name", ["tiny", "wan_32k", "video_187k", "skew_187k", "minute_580k"])
def test_route_workload(name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=0, device="cuda", with_qkv=False)
    res = moga.route(inp["x"], inp["W_r"], inp["b_r"], wl.M)
    torch.cuda.synchronize()
    gid, info = check_route(res, inp["x"], inp["W_r"], inp["b_r"], wl.M,
                            GATE_TOL_F32 if wl.x_dtype == "f32" else GATE_TOL_BF16)
    counts = np.bincount(gid, minlength=wl.M)
    print(f"{name}: group sizes {counts.tolist()} near-ties {info['n_near']} flipped {info['n_flipped']}")
    if name == "skew_187k":
        assert (counts[56:] == 0).all()
        assert sorted(counts[48:56].tolist()) == [1, 2, 3, 5, 8, 13, 21, 34]


@pytest.mark.parametrize("name", ["tiny", "wan_32k", "skew_187k"])
def test_route_balance_stats(name):
    """moga_route_ex: routing identical to moga_route, plus P_i and the balance
    metric against the oracle, bitwise repeatable."""
    import oracle
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=0, device="cuda", with_qkv=False)
    res = moga.route_stats(inp["x"], inp["W_r"], inp["b_r"], wl.M)
    ref = moga.route(inp["x"], inp["W_r"], inp["b_r"], wl.M)
    again = moga.route_stats(inp["x"], inp["W_r"], inp["b_r"], wl.M)
    torch.cuda.synchronize()
    for key in ("group_id", "perm", "offsets", "gate"):
        assert np.array_equal(np_cpu(res[key]), np_cpu(ref[key]))
    F, P, b = oracle.balance_stats(np_cpu(inp["x"]), np_cpu(inp["W_r"]),
                                   None if inp["b_r"] is None else np_cpu(inp["b_r"]))
    pm = np_cpu(res["prob_mean"]).astype(np.float64)
    assert np.abs(pm - P).max() <= 1e-5, np.abs(pm - P).max()
    assert abs(float(np_cpu(res["balance"])[0]) - b) <= 1e-4 * max(1.0, b)
    assert np.array_equal(np_cpu(again["prob_mean"]), np_cpu(res["prob_mean"]))
    assert np.array_equal(np_cpu(again["balance"]), np_cpu(res["balance"]))
    print(f"{name}: balance metric {b:.4f} (GPU {float(np_cpu(res['balance'])[0]):.4f})")
