"""Shot-aware STGA (stga_shot_attn, C ABI) on the GPU against the oracle.

"MoGA: Mixture-of-Groups Attention for End-to-End Long Video Generation"
(paper-graph-ui summary), §3.4 "Spatial-Temporal Group Attention (STGA)":
temporal groups never cross a shot cut; keys and values, not queries, of a
shot's boundary windows see latent frames of the adjacent shots.  Small grids
are compared on every row; the 480p / 120-frame grid on sampled rows of the
boundary windows, in the configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import learned_token_group_b200 as moga
import oracle
from parity import compare_out, np_cpu
from workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu


def _qkv(N, H, d_h, seed):
    inp = make_inputs(custom(N, H=H, d_h=d_h, d=64, M=2), seed=seed, device="cuda")
    return inp["q"], inp["k"], inp["v"]


def _window_ids(grid, window, shots, ap, an):
    N = grid[0] * grid[1] * grid[2]
    win = np.zeros(N, dtype=np.int64)
    for i, (qi, _) in enumerate(oracle.shot_windows(*grid, window, shots, ap, an)):
        win[qi] = i
    return win


CASES = [
    # (grid, window, shots, aug_prev, aug_next, H, d_h)
    ((9, 8, 16), (3, 8, 8), [0, 4, 9], 2, 2, 2, 128),        # cut inside a temporal window
    ((6, 30, 52), (0, 15, 26), [0, 2, 6], 2, 2, 1, 64),      # the pages' 2x2 partition, whole shots
    ((5, 4, 6), (2, 4, 3), [0, 1, 2, 3, 4, 5], 2, 2, 2, 128),  # one-frame shots: augmentation clipped
    ((7, 10, 12), (2, 8, 8), [0, 3, 7], 1, 3, 1, 128),       # unequal augmentation
    ((4, 9, 7), (0, 16, 16), [0, 4], 2, 2, 2, 64),           # one shot, window larger than a frame
]


@pytest.mark.parametrize("grid,window,shots,ap,an,H,d_h", CASES)
def test_shot_stga(grid, window, shots, ap, an, H, d_h):
    N = grid[0] * grid[1] * grid[2]
    q, k, v = _qkv(N, H, d_h, seed=N + len(shots))
    ss = torch.tensor(shots, dtype=torch.int32, device="cuda")
    out, ws = moga.stga_shot_attn(q, k, v, grid, window, ss, ap, an)
    moga.sync_status(ws)
    ref = oracle.stga_shot_attention(np_cpu(q), np_cpu(k), np_cpu(v), *grid, window, shots, ap, an)
    compare_out(out, ref, groups=_window_ids(grid, window, shots, ap, an))


def test_shot_stga_accumulate_and_scale():
    grid, window, shots = (6, 10, 12), (2, 8, 8), [0, 3, 6]
    N = 720
    q, k, v = _qkv(N, 2, 128, seed=5)
    base = _qkv(N, 2, 128, seed=6)[0]
    out = base.clone()
    ss = torch.tensor(shots, dtype=torch.int32, device="cuda")
    _, ws = moga.stga_shot_attn(q, k, v, grid, window, ss, 2, 2, out_scale=1 / 3, accumulate=True, out=out)
    moga.sync_status(ws)
    ref = np_cpu(base).astype(np.float64) + oracle.stga_shot_attention(np_cpu(q), np_cpu(k), np_cpu(v), *grid,
                                                                        window, shots, 2, 2) / 3
    compare_out(out, ref)


@pytest.mark.parametrize("window,plain,bitwise", [((3, 8, 8), (3, 8, 8), False),       # different kernels
                                                  ((0, 30, 52), (6, 30, 52), True)])   # same tiled kernel
def test_one_shot_equals_plain_stga(window, plain, bitwise):
    """With a single shot there is nothing to augment: the result is the
    plain STGA branch.  Whole-shot windows and plain whole-clip windows run
    the same kernel over the same tiles, so they agree bit for bit.  For
    3x8x8 windows plain STGA runs the whole-window box kernel (one softmax
    step over 192 keys) while shot windows are copied by rows (two key
    tiles), so the two are compared with the oracle instead."""
    grid = (6, 30, 52)
    q, k, v = _qkv(9360, 2, 128, seed=9)
    ss = torch.tensor([0, 6], dtype=torch.int32, device="cuda")
    a, ws = moga.stga_shot_attn(q, k, v, grid, window, ss, 2, 2)
    moga.sync_status(ws)
    b = moga.stga_window_attn(q, k, v, grid, plain)
    torch.cuda.synchronize()
    if bitwise:
        assert torch.equal(a, b)
    else:
        ref = oracle.stga_attention(np_cpu(q), np_cpu(k), np_cpu(v), *grid, plain)
        compare_out(a, ref)
        compare_out(b, ref)


def test_bad_shot_boundaries_are_reported():
    grid, window = (6, 8, 8), (2, 8, 8)
    q, k, v = _qkv(384, 1, 128, seed=3)
    for shots in ([0, 4, 2, 6], [1, 3, 6], [0, 3, 5]):          # not increasing, not from 0, not to T
        ss = torch.tensor(shots, dtype=torch.int32, device="cuda")
        out = torch.zeros_like(q)
        _, ws = moga.stga_shot_attn(q, k, v, grid, window, ss, 2, 2, out=out)
        with pytest.raises(moga.MogaError) as e:
            moga.sync_status(ws)
        assert e.value.status == 6                               # MOGA_ERR_DEVICE_CHECK
        assert out.float().abs().max().item() == 0.0             # nothing was written
    ss = torch.tensor([0, 3, 6], dtype=torch.int32, device="cuda")
    _, ws = moga.stga_shot_attn(q, k, v, grid, window, ss, 2, 2)
    moga.sync_status(ws)                                         # the context is still usable


# Shot split of the 120-frame 480p grid used by the benchmark's shot-aware row.
VIDEO_SHOTS = [0, 24, 40, 60, 88, 100, 120]


@pytest.mark.parametrize("window", [(0, 15, 26), (3, 8, 8)])
def test_shot_stga_video_sampled(window):
    wl = WORKLOADS["video_187k"]
    inp = make_inputs(wl, seed=0, device="cuda")
    ss = torch.tensor(VIDEO_SHOTS, dtype=torch.int32, device="cuda")
    out, ws = moga.stga_shot_attn(inp["q"], inp["k"], inp["v"], wl.grid, window, ss, 2, 2)
    moga.sync_status(ws)
    T, Hg, Wg = wl.grid
    rng = np.random.default_rng(7)
    rows = []
    for s in VIDEO_SHOTS[:-1] + [VIDEO_SHOTS[-1] - 1]:         # frames at every cut, both sides
        for f in {max(s - 1, 0), min(s, T - 1)}:
            rows.append(f * Hg * Wg + rng.choice(Hg * Wg, size=24, replace=False))
    rows.append(rng.choice(wl.N, size=64, replace=False))
    rows = np.unique(np.concatenate(rows))
    heads = [0, wl.H - 1]
    ref = oracle.stga_shot_attention(inp["q"], inp["k"], inp["v"], *wl.grid, window, VIDEO_SHOTS, 2, 2,
                                     rows=rows, heads=heads)
    got = out[torch.from_numpy(rows).cuda()][:, heads]
    compare_out(got, ref, groups=_window_ids(wl.grid, window, VIDEO_SHOTS, 2, 2)[rows])


@pytest.mark.parametrize("per_frame", [True, False])
def test_layer_shots_block(per_frame):
    """moga_layer_shots: the mean of MoGA, shot-aware STGA and (optionally)
    per-frame attention, against the oracle's branches combined the same way."""
    grid, window, shots = (6, 8, 16), (0, 4, 8), [0, 2, 6]
    wl = custom(768, H=2, d_h=128, d=128, M=4, x_kind="clustered", grid=grid, name="shots_block")
    inp = make_inputs(wl, seed=17, device="cuda")
    ss = torch.tensor(shots, dtype=torch.int32, device="cuda")
    res = moga.moga_layer_shots(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M, grid, window,
                                ss, 2, 2, per_frame=per_frame)
    moga.sync_status(res["ws"])
    gid = np_cpu(res["group_id"]).astype(np.int64)
    gate = np_cpu(res["gate"]).astype(np.float64)
    q, k, v = (np_cpu(inp[n]) for n in ("q", "k", "v"))
    ref = oracle.group_attention(q, k, v, gid, gate, wl.M) + oracle.stga_shot_attention(q, k, v, *grid, window,
                                                                                       shots, 2, 2)
    if per_frame:
        ref = ref + oracle.frame_attention(q, k, v, *grid)
    ref = ref / (3 if per_frame else 2)
    compare_out(res["out"], ref, groups=gid)
