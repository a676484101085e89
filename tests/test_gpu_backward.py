"""Training path on the GPU against the oracle: the forward that keeps the
log-sum-exp (moga_layer_train) and the block's gradients (moga_layer_backward).

"MoGA: Mixture-of-Groups Attention for End-to-End Long Video Generation"
(paper-graph-ui summary), section 3.4, "MoGA Router" and "Grouped Attention":
the hard assignment is held fixed; the router learns through the gate of
Eq. 5, q, k, v through each branch's attention.

Tolerances (bf16 operands, fp32 accumulation; the arithmetic behind them):
* lse: fp32 scores of bf16 inputs and an fp32 sum, |err| <= LSE_ABS.
* dq, dk, dv (bf16): P, dS and dO enter the tensor core as bf16 (relative
  rounding 2^-9 each) and the result is rounded to bf16 once per branch
  (twice with STGA): about sqrt(3) * 2^-9 ~ 3.4e-3 of the norm for
  independent roundings, so GRAD_REL_L2 = 1e-2 leaves a factor of three; no
  element may be off by more than GRAD_MAX_REL of the tensor's largest
  magnitude (a few ulps of bf16 at that magnitude).
* dx, dW_r, db_r: the gate gradient sums dout * o over H * d_h products of
  bf16 values (o rounded to bf16), then the router's fp32 arithmetic:
  ROUTER_REL_L2 of the tensor's norm.
"""
import numpy as np
import pytest
import torch

import learned_token_group_b200 as moga
import oracle
from parity import check_route, compare_out, np_cpu
from workloads import custom, make_inputs

pytestmark = pytest.mark.gpu

LSE_ABS = 2e-3
GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2
ROUTER_REL_L2 = 1e-2


def _run(wl, seed, with_bias=True):
    inp = make_inputs(wl, seed=seed, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed + 7)
    b_r = (0.1 * torch.randn(wl.M, generator=gen, device="cuda")) if with_bias else None
    dout = torch.randn((wl.N, wl.H, wl.d_h), generator=gen, device="cuda").to(torch.bfloat16)
    sv = moga.layer_train(inp["x"], inp["W_r"], b_r, inp["q"], inp["k"], inp["v"], wl.M, wl.grid, wl.window)
    g = moga.layer_backward(dout, sv, inp["x"], inp["W_r"], b_r, inp["q"], inp["k"], inp["v"], wl.M, wl.grid,
                            wl.window)
    moga.sync_status(sv["ws"])
    moga.sync_status(g["ws"])
    return inp, b_r, dout, sv, g


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _check_grads(g, ref, what=""):
    errs = {}
    for name in ("dq", "dk", "dv"):
        a = np_cpu(g[name]).astype(np.float64)
        b = ref[name]
        assert np.isfinite(a).all(), f"{what}{name}: non-finite"
        rel = _rel(a, b)
        mx = float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))
        errs[name] = (rel, mx)
        assert rel <= GRAD_REL_L2, f"{what}{name}: rel-L2 {rel:.3e}"
        assert mx <= GRAD_MAX_REL, f"{what}{name}: max error {mx:.3e} of max |ref|"
    for name in ("dx", "dW_r", "db_r"):
        if g[name] is None:
            continue
        a = np_cpu(g[name]).astype(np.float64)
        assert np.isfinite(a).all(), f"{what}{name}: non-finite"
        rel = _rel(a, ref[name])
        errs[name] = (rel,)
        assert rel <= ROUTER_REL_L2, f"{what}{name}: rel-L2 {rel:.3e}"
    return errs


def _check_forward(wl, inp, sv, b_r):
    x, W, q, k, v = (np_cpu(inp[n]) for n in ("x", "W_r", "q", "k", "v"))
    b = None if b_r is None else np_cpu(b_r)
    gid, _ = check_route({n: sv[n] for n in ("group_id", "gate", "perm", "offsets")}, inp["x"], inp["W_r"], b_r,
                         wl.M, 1e-4 if wl.x_dtype == "bf16" else 1e-5)
    ref = oracle.moga_layer(x, W, b, q, k, v, wl.M, grid=wl.grid, window=wl.window)
    compare_out(sv["o_moga"], ref["moga"], groups=gid, what="o_moga")
    if wl.window is not None:
        compare_out(sv["o_stga"], ref["stga"], what="o_stga")
    compare_out(sv["out"], ref["out"], what="out")
    # log-sum-exp at sorted positions (groups) and window positions (STGA)
    lse = np_cpu(sv["lse_moga"])
    perm = np_cpu(sv["perm"]).astype(np.int64)
    off = np_cpu(sv["offsets"]).astype(np.int64)
    worst = 0.0
    for m in range(wl.M):
        idx = perm[off[m]:off[m + 1]]
        if idx.size == 0:  # an empty group has no rows to check
            continue
        for h in range(wl.H):
            r = oracle.attention_lse(q[idx, h].astype(np.float64), k[idx, h].astype(np.float64))
            worst = max(worst, float(np.abs(lse[h, off[m]:off[m + 1]] - r).max()))
    assert worst <= LSE_ABS, f"lse_moga error {worst:.3e}"
    if wl.window is not None:
        lse_s = np_cpu(sv["lse_stga"])
        pos = 0
        for idx in oracle.stga_windows(*wl.grid, wl.window):
            for h in range(wl.H):
                r = oracle.attention_lse(q[idx, h].astype(np.float64), k[idx, h].astype(np.float64))
                assert np.abs(lse_s[h, pos:pos + idx.size] - r).max() <= LSE_ABS
            pos += idx.size
    return gid


def _reference(wl, inp, b_r, dout):
    x, W, q, k, v = (np_cpu(inp[n]) for n in ("x", "W_r", "q", "k", "v"))
    return oracle.moga_layer_backward(x, W, None if b_r is None else np_cpu(b_r), q, k, v, wl.M, np_cpu(dout),
                                      grid=wl.grid, window=wl.window)


CASES = [
    # groups only, ragged tiles, d_h 128
    (custom(700, H=2, d_h=128, d=64, M=3), 1),
    # groups + STGA on a small grid, d_h 64
    (custom(360, H=2, d_h=64, d=64, M=4, grid=(3, 10, 12), window=(3, 8, 8)), 2),
    # the 480p latent grid, clustered tokens: groups of thousands of tokens
    (custom(9360, H=2, d_h=128, d=256, M=5, x_kind="clustered", grid=(6, 30, 52), window=(3, 8, 8)), 3),
    # fp32 router input (the tiny configuration's dtype)
    (custom(1024, H=1, d_h=64, d=64, M=4, x_dtype="f32"), 4),
    # windows larger than two tiles (whole frames)
    (custom(3120, H=1, d_h=128, d=64, M=2, grid=(2, 30, 52), window=(1, 30, 52)), 5),
    # router gradients over 40 groups: dW_r in three chunks of 16 groups, the last partial
    (custom(1500, H=1, d_h=64, d=128, M=40, x_kind="clustered"), 6),
    # bf16 router input with M > 256: the logits come from the SIMT router
    (custom(1200, H=1, d_h=64, d=64, M=300), 7),
    # d_h 128 with 40 groups: the dK/dV pass reads its group table from global memory
    (custom(1600, H=2, d_h=128, d=128, M=40, x_kind="clustered"), 8),
]


@pytest.mark.parametrize("wl,seed", CASES, ids=[f"{c[0].N}_{c[0].d_h}_{c[0].window}" for c in CASES])
def test_backward(wl, seed):
    inp, b_r, dout, sv, g = _run(wl, seed)
    gid = _check_forward(wl, inp, sv, b_r)
    _, _, margin = oracle.route(np_cpu(inp["x"]), np_cpu(inp["W_r"]), np_cpu(b_r))
    assert (gid == oracle.route(np_cpu(inp["x"]), np_cpu(inp["W_r"]), np_cpu(b_r))[0]).all(), \
        "a token's group differs from the oracle's; pick inputs without near-ties"
    ref = _reference(wl, inp, b_r, dout)
    errs = _check_grads(g, ref)
    print(wl.N, wl.d_h, wl.window, {k_: tuple(f"{e:.2e}" for e in v_) for k_, v_ in errs.items()})


def test_backward_without_bias():
    wl = custom(500, H=1, d_h=128, d=64, M=3)
    inp, b_r, dout, sv, g = _run(wl, 11, with_bias=False)
    assert g["db_r"] is None
    ref = _reference(wl, inp, None, dout)
    _check_grads(g, ref)


def test_backward_one_group_router_silent():
    # one group: the gate is identically 1, so the router gets no gradient
    wl = custom(300, H=1, d_h=64, d=64, M=1)
    inp, b_r, dout, sv, g = _run(wl, 12)
    assert float(g["dW_r"].abs().max()) < 1e-6 and float(g["db_r"].abs().max()) < 1e-6
    assert float(g["dx"].float().abs().max()) < 1e-6
    ref = _reference(wl, inp, b_r, dout)
    _check_grads(g, ref)


def test_autograd_function_matches_calls():
    wl = custom(360, H=2, d_h=64, d=64, M=4, grid=(3, 10, 12), window=(3, 8, 8))
    inp, b_r, dout, sv, g = _run(wl, 2)
    leaves = {n: inp[n].clone().requires_grad_(True) for n in ("x", "W_r", "q", "k", "v")}
    b = b_r.clone().requires_grad_(True)
    out = moga.MogaFunction.apply(leaves["x"], leaves["W_r"], b, leaves["q"], leaves["k"], leaves["v"], wl.M,
                                  wl.grid, wl.window)
    out.backward(dout)
    torch.cuda.synchronize()
    assert torch.equal(out, sv["out"])
    for n, gn in (("x", "dx"), ("q", "dq"), ("k", "dk"), ("v", "dv")):
        assert torch.equal(leaves[n].grad, g[gn]), n
    assert torch.equal(leaves["W_r"].grad.float(), g["dW_r"].to(leaves["W_r"].dtype).float())
    assert torch.equal(b.grad, g["db_r"])


def test_backward_is_deterministic():
    wl = custom(9360, H=2, d_h=128, d=256, M=5, x_kind="clustered", grid=(6, 30, 52), window=(3, 8, 8))
    _, _, _, _, g1 = _run(wl, 3)
    _, _, _, _, g2 = _run(wl, 3)
    for n in ("dx", "dW_r", "db_r", "dq", "dk", "dv"):
        assert torch.equal(g1[n], g2[n]), n


def test_backward_full_size_sampled():
    """video_187k (187,200 tokens, 12 heads, M = 16, STGA 3x8x8) in the
    launch configuration `bench.py --train` times, checked on samples the
    oracle computes exactly: dq of sampled query rows of every group (each row
    against its whole group, plus its STGA window), dk and dv of every token
    of the small groups (whole-group backward, plus each token's window), and
    dx of sampled tokens (their gate gradient over all 12 heads).  Group
    membership is the GPU's assignment, which the routing check above pins
    (the backward holds the assignment fixed)."""
    from workloads import WORKLOADS
    wl = WORKLOADS["video_187k"]
    inp, b_r, dout, sv, g = _run(wl, 0, with_bias=False)
    route_res = {n: sv[n] for n in ("group_id", "gate", "perm", "offsets")}
    gid, _ = check_route(route_res, inp["x"], inp["W_r"], None, wl.M, 1e-4)
    x64 = np_cpu(inp["x"]).astype(np.float64)
    W64 = np_cpu(inp["W_r"]).astype(np.float64)
    r = x64 @ W64.T
    p = np.exp(r - r.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    gate = p[np.arange(wl.N), gid]
    w = 0.5
    rng = np.random.default_rng(5)
    heads = [0, wl.H - 1]
    windows = oracle.stga_windows(*wl.grid, wl.window)
    win_of = np.empty(wl.N, dtype=np.int64)
    for wi, idx in enumerate(windows):
        win_of[idx] = wi
    rows_of = lambda t, idx, h: np_cpu(t[torch.as_tensor(idx, device="cuda"), h]).astype(np.float64)
    win_cache = {}

    def window_grads(wi, h):
        key = (wi, h)
        if key not in win_cache:
            idx = windows[wi]
            win_cache[key] = (idx,) + oracle.attention_rows_backward(
                rows_of(inp["q"], idx, h), rows_of(inp["k"], idx, h), rows_of(inp["v"], idx, h),
                w * rows_of(dout, idx, h))[:3]
        return win_cache[key]

    got_q, ref_q, got_kv, ref_kv = [], [], [], []
    sizes = np.bincount(gid, minlength=wl.M)
    for m in range(wl.M):
        idx = np.nonzero(gid == m)[0]
        if idx.size == 0:
            continue
        rows = np.sort(rng.choice(idx, size=min(16, idx.size), replace=False))
        for h in heads:
            K, V = rows_of(inp["k"], idx, h), rows_of(inp["v"], idx, h)
            dOr = w * gate[rows][:, None] * rows_of(dout, rows, h)
            dq = oracle.attention_dq_rows(rows_of(inp["q"], rows, h), K, V, dOr)[0]
            for a, t in enumerate(rows):
                widx, wq, _, _ = window_grads(win_of[t], h)
                dq[a] += wq[np.searchsorted(widx, t)]
            ref_q.append(dq)
            got_q.append(np_cpu(g["dq"][torch.as_tensor(rows, device="cuda"), h]).astype(np.float64))
            if 100 <= sizes[m] <= 3000:   # small groups: dk, dv of every token
                Q = rows_of(inp["q"], idx, h)
                dO = w * gate[idx][:, None] * rows_of(dout, idx, h)
                _, dk, dv, _ = oracle.attention_rows_backward(Q, K, V, dO)
                for a, t in enumerate(idx):
                    widx, _, wk, wv = window_grads(win_of[t], h)
                    j = np.searchsorted(widx, t)
                    dk[a] += wk[j]
                    dv[a] += wv[j]
                tt = torch.as_tensor(idx, device="cuda")
                ref_kv.append(np.concatenate([dk, dv], axis=1))
                got_kv.append(np.concatenate([np_cpu(g["dk"][tt, h]), np_cpu(g["dv"][tt, h])], axis=1))
    assert got_kv, "no group of 100-3000 tokens to check dk and dv on"
    for what, got, ref in (("dq", got_q, ref_q), ("dk|dv", got_kv, ref_kv)):
        a, b = np.concatenate(got), np.concatenate(ref)
        rel = _rel(a, b)
        mx = float(np.abs(a - b).max() / np.abs(b).max())
        assert rel <= GRAD_REL_L2 and mx <= GRAD_MAX_REL, f"{what}: rel-L2 {rel:.3e}, max {mx:.3e}"
    # dx of sampled tokens of three groups: the gate gradient sums all heads
    got_x, ref_x = [], []
    for m in np.argsort(sizes)[-3:]:
        idx = np.nonzero(gid == m)[0]
        rows = np.sort(rng.choice(idx, size=8, replace=False))
        dgate = np.zeros(rows.size)
        for h in range(wl.H):
            K, V = rows_of(inp["k"], idx, h), rows_of(inp["v"], idx, h)
            A = oracle.attention_rows(rows_of(inp["q"], rows, h), K, V)
            dgate += w * (rows_of(dout, rows, h) * A).sum(axis=1)
        onehot = np.zeros((rows.size, wl.M))
        onehot[np.arange(rows.size), gid[rows]] = 1.0
        dr = (dgate * gate[rows])[:, None] * (onehot - p[rows])
        ref_x.append(dr @ W64)
        got_x.append(np_cpu(g["dx"][torch.as_tensor(rows, device="cuda")]).astype(np.float64))
    rel = _rel(np.concatenate(got_x), np.concatenate(ref_x))
    assert rel <= ROUTER_REL_L2, f"dx: rel-L2 {rel:.3e}"


@pytest.mark.parametrize("wl,window", [
    (custom(360, H=2, d_h=64, d=64, M=4, grid=(3, 10, 12), window=(3, 8, 8)), (3, 8, 8)),
    (custom(3120, H=1, d_h=128, d=64, M=3, grid=(2, 30, 52), window=(3, 8, 8)), (3, 8, 8)),
    (custom(360, H=2, d_h=128, d=64, M=4, grid=(3, 10, 12)), None),     # MoGA + per-frame only
])
def test_backward_three_branches(wl, window):
    """The block with the per-frame branch (moga_layer_train_ex /
    moga_layer_backward_ex): out is the mean of the branches that are on and
    each branch's share of dout is dout divided by their number."""
    inp = make_inputs(wl, seed=21, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(22)
    b_r = 0.1 * torch.randn(wl.M, generator=gen, device="cuda")
    dout = torch.randn((wl.N, wl.H, wl.d_h), generator=gen, device="cuda").to(torch.bfloat16)
    args = (inp["x"], inp["W_r"], b_r, inp["q"], inp["k"], inp["v"], wl.M, wl.grid, window)
    sv = moga.layer_train(*args, per_frame=True)
    g = moga.layer_backward(dout, sv, *args)
    moga.sync_status(g["ws"])
    x, W, q, k, v = (np_cpu(inp[n]) for n in ("x", "W_r", "q", "k", "v"))
    ref = oracle.moga_layer(x, W, np_cpu(b_r), q, k, v, wl.M, grid=wl.grid, window=window, per_frame=True)
    compare_out(sv["o_frame"], ref["frame"], what="o_frame")
    compare_out(sv["out"], ref["out"], what="out")
    gref = oracle.moga_layer_backward(x, W, np_cpu(b_r), q, k, v, wl.M, np_cpu(dout), grid=wl.grid, window=window,
                                      per_frame=True)
    _check_grads(g, gref)


def test_backward_with_balancing_loss():
    """balance_alpha adds the group balancing loss (alpha * M * sum_i F_i P_i,
    "Group Balancing Loss") to the router's gradient; q, k, v are unaffected."""
    wl = custom(700, H=2, d_h=128, d=64, M=5, x_kind="clustered")
    inp, b_r, dout, sv, g0 = _run(wl, 31)
    args = (inp["x"], inp["W_r"], b_r, inp["q"], inp["k"], inp["v"], wl.M, wl.grid, wl.window)
    g = moga.layer_backward(dout, sv, *args, balance_alpha=0.1)
    moga.sync_status(g["ws"])
    for n in ("dq", "dk", "dv"):
        assert torch.equal(g[n], g0[n]), n
    x, W, q, k, v = (np_cpu(inp[n]) for n in ("x", "W_r", "q", "k", "v"))
    ref = oracle.moga_layer_backward(x, W, np_cpu(b_r), q, k, v, wl.M, np_cpu(dout), balance_alpha=0.1)
    _check_grads(g, ref)
    # with dout = 0 the balancing term is the router's whole gradient (and
    # q, k, v get none), so the term is compared on its own
    zero = torch.zeros_like(dout)
    gz = moga.layer_backward(zero, sv, *args, balance_alpha=0.5)
    moga.sync_status(gz["ws"])
    refz = oracle.moga_layer_backward(x, W, np_cpu(b_r), q, k, v, wl.M, np_cpu(zero), balance_alpha=0.5)
    assert np.abs(refz["dW_r"]).max() > 0
    for n in ("dq", "dk", "dv"):
        assert float(gz[n].float().abs().max()) == 0.0, n
    for n in ("dx", "dW_r", "db_r"):
        rel = _rel(np_cpu(gz[n]).astype(np.float64), refz[n])
        assert rel <= ROUTER_REL_L2, f"{n}: rel-L2 {rel:.3e}"
