"""Pins of the CPU oracle to things other than itself.

Each ``check_*`` function takes the oracle module and raises AssertionError
when the oracle disagrees with a closed form, a library routine, brute force
on a tiny input or an invariant of the method.  The plain tests run every
check on the real oracle; ``test_planted_mistakes_are_caught`` runs them on
copies of the oracle with one plausible mistake planted (on the CPU) and
requires that some check fails, so the pins are known to bite.

Method source: "MoGA: Mixture-of-Groups Attention for End-to-End Long Video
Generation" (paper-graph-ui summary), section 3.4 (Eqs. 1-5, Algorithm 1, STGA).
"""
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers that are independent of the oracle
# ----------------------------------------------------------------------------
def _sdpa(q, k, v):
    """Library attention (torch CPU, float64): q,k,v [L, H, E] -> [L, H, E]."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float64).transpose(1, 0, 2)))
    o = torch.nn.functional.scaled_dot_product_attention(t(q)[None], t(k)[None], t(v)[None])[0]
    return o.numpy().transpose(1, 0, 2)


def _brute_route(x, W, b):
    """Pure-Python loops: logits, softmax, first argmax, gate."""
    N, d = len(x), len(x[0])
    M = len(W)
    gid, gate = [], []
    for i in range(N):
        r = [sum(float(x[i][c]) * float(W[m][c]) for c in range(d)) + (float(b[m]) if b is not None else 0.0)
             for m in range(M)]
        best = 0
        for m in range(1, M):
            if r[m] > r[best]:
                best = m
        z = sum(math.exp(rm - r[best]) for rm in r)
        gid.append(best)
        gate.append(1.0 / z)
    return np.array(gid), np.array(gate)


def _brute_masked_dense(q, k, v, gid, gate):
    """Pure-Python masked dense attention: key j is visible to query i iff
    both tokens carry the same group id; output scaled by the gate."""
    N, H, E = q.shape
    out = np.zeros((N, H, E))
    for i in range(N):
        for h in range(H):
            s = []
            for j in range(N):
                if gid[j] == gid[i]:
                    s.append((j, sum(float(q[i, h, c]) * float(k[j, h, c]) for c in range(E)) / math.sqrt(E)))
            mx = max(val for _, val in s)
            w = [(j, math.exp(val - mx)) for j, val in s]
            z = sum(wj for _, wj in w)
            for c in range(E):
                out[i, h, c] = gate[i] * sum(wj * float(v[j, h, c]) for j, wj in w) / z
    return out


def _brute_stga(q, k, v, grid, window):
    """Pure-Python window attention: tokens share a window iff their
    (t // wt, h // wh, w // ww) coordinates agree."""
    T, Hg, Wg = grid
    wt, wh, ww = window
    N, H, E = q.shape
    coord = []
    for i in range(N):
        t, rem = divmod(i, Hg * Wg)
        hh, w = divmod(rem, Wg)
        coord.append((t // wt, hh // wh, w // ww))
    out = np.zeros((N, H, E))
    for i in range(N):
        keys = [j for j in range(N) if coord[j] == coord[i]]
        for h in range(H):
            s = [sum(float(q[i, h, c]) * float(k[j, h, c]) for c in range(E)) / math.sqrt(E) for j in keys]
            mx = max(s)
            w = [math.exp(a - mx) for a in s]
            z = sum(w)
            for c in range(E):
                out[i, h, c] = sum(wj * float(v[j, h, c]) for j, wj in zip(keys, w)) / z
    return out


def _brute_shot_stga(q, k, v, grid, window, shot_start, aug_prev, aug_next):
    """Pure-Python shot-aware window attention from coordinates: key j is
    visible to query i iff both lie in the same spatial tile and j's frame is
    in i's temporal window, or in the previous shot's last aug_prev frames
    when i's window starts its shot, or in the next shot's first aug_next
    frames when i's window ends its shot."""
    T, Hg, Wg = grid
    wt, wh, ww = window
    s = list(shot_start)
    N, H, E = q.shape

    def coords(i):
        t, rem = divmod(i, Hg * Wg)
        hh, w = divmod(rem, Wg)
        return t, hh, w

    def visible(i, jj):
        t, hh, w = coords(i)
        t2, h2, w2 = coords(jj)
        if h2 // wh != hh // wh or w2 // ww != w // ww:
            return False
        sh = max(n for n in range(len(s) - 1) if s[n] <= t)
        step = wt if wt > 0 else s[sh + 1] - s[sh]
        a = s[sh] + ((t - s[sh]) // step) * step
        b = min(s[sh + 1], a + step)
        if a <= t2 < b:
            return True
        if a == s[sh] and sh > 0 and max(s[sh - 1], s[sh] - aug_prev) <= t2 < s[sh]:
            return True
        if b == s[sh + 1] and sh + 1 < len(s) - 1 and s[sh + 1] <= t2 < min(s[sh + 2], s[sh + 1] + aug_next):
            return True
        return False

    out = np.zeros((N, H, E))
    for i in range(N):
        keys = [jj for jj in range(N) if visible(i, jj)]
        for h in range(H):
            sc = [sum(float(q[i, h, c]) * float(k[jj, h, c]) for c in range(E)) / math.sqrt(E) for jj in keys]
            mx = max(sc)
            w = [math.exp(a - mx) for a in sc]
            z = sum(w)
            for c in range(E):
                out[i, h, c] = sum(wj * float(v[jj, h, c]) for jj, wj in zip(keys, w)) / z
    return out


def _read_golden(name):
    sections, cur = {}, None
    env = {"e": math.e, "log": math.log, "__builtins__": {}}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                cur = sections.setdefault(line.strip("[]"), {})
                continue
            key, expr = line.split("=", 1)
            cur[key.strip()] = eval(expr, env)  # fixture expressions only
    return sections


# ----------------------------------------------------------------------------
# checks
# ----------------------------------------------------------------------------
def check_route_closed_form(o):
    # W_r = I, x = a * e_k: r = a e_k, so p_k = e^a / (e^a + M - 1).
    M, a = 5, 2.0
    x = np.zeros((3 * M, M))
    for i in range(3 * M):
        x[i, i % M] = a
    gid, gate, margin = o.route(x, np.eye(M))
    assert np.array_equal(gid, np.arange(3 * M) % M)
    assert np.allclose(gate, math.exp(a) / (math.exp(a) + M - 1), rtol=0, atol=1e-15)
    assert np.allclose(margin, a)


def check_route_ties_and_M1(o):
    gid, gate, _ = o.route(np.zeros((4, 3)), np.ones((6, 3)))
    assert np.array_equal(gid, np.zeros(4)) and np.allclose(gate, 1 / 6)
    # logits (1, 3, 3, 0): the first of the two maxima wins
    W = np.array([[1.0], [3.0], [3.0], [0.0]])
    gid, gate, _ = o.route(np.ones((1, 1)), W)
    assert gid[0] == 1
    assert abs(gate[0] - math.exp(3) / (math.exp(1) + 2 * math.exp(3) + 1)) < 1e-15
    rng = np.random.default_rng(1)
    gid, gate, margin = o.route(rng.normal(size=(7, 4)), rng.normal(size=(1, 4)))
    assert np.all(gid == 0) and np.all(gate == 1.0) and np.all(np.isinf(margin))


def check_route_brute(o):
    rng = np.random.default_rng(2)
    x = rng.normal(size=(16, 8))
    W = rng.normal(size=(3, 8)) / math.sqrt(8)
    b = rng.normal(size=3)
    g0, p0 = _brute_route(x.tolist(), W.tolist(), b.tolist())
    gid, gate, margin = o.route(x, W, b)
    assert np.array_equal(gid, g0)
    assert np.allclose(gate, p0, rtol=0, atol=1e-13)
    assert np.all(gate >= 1 / 3 - 1e-15) and np.all(gate <= 1)
    r = x @ W.T + b
    srt = np.sort(r, axis=1)
    assert np.allclose(margin, srt[:, -1] - srt[:, -2])


def check_counting_sort(o):
    rng = np.random.default_rng(3)
    for N, M in [(0, 3), (1, 1), (50, 7), (1000, 16), (333, 64)]:
        g = rng.integers(0, max(1, M // 2), size=N).astype(np.int32)  # upper groups empty
        perm, offsets, mx = o.counting_sort(g, M)
        assert np.array_equal(perm, np.argsort(g, kind="stable"))
        assert np.array_equal(np.sort(perm), np.arange(N))
        assert offsets[0] == 0 and offsets[-1] == N and np.all(np.diff(offsets) >= 0)
        assert np.array_equal(np.diff(offsets), np.bincount(g, minlength=M))
        assert mx == (np.bincount(g, minlength=M).max() if N else 0)
        for m in range(M):
            seg = perm[offsets[m]:offsets[m + 1]]
            assert np.all(g[seg] == m) and np.all(np.diff(seg) > 0)


def check_full_attention_when_M1(o):
    rng = np.random.default_rng(4)
    q, k, v = (rng.normal(size=(40, 3, 16)) for _ in range(3))
    x = rng.normal(size=(40, 5))
    res = o.moga_layer(x, rng.normal(size=(1, 5)), None, q, k, v, 1)
    assert np.all(res["gate"] == 1.0)
    assert np.allclose(res["out"], _sdpa(q, k, v), rtol=0, atol=1e-12)


def check_group_equals_subset_attention(o):
    rng = np.random.default_rng(5)
    N, H, E, M = 60, 2, 8, 4
    q, k, v = (rng.normal(size=(N, H, E)) for _ in range(3))
    gid = rng.integers(0, M, size=N)
    gate = rng.uniform(0.25, 1.0, size=N)
    out = o.group_attention(q, k, v, gid, gate, M)
    for m in range(M):
        idx = np.nonzero(gid == m)[0]
        if idx.size:
            ref = _sdpa(q[idx], k[idx], v[idx]) * gate[idx][:, None, None]
            assert np.allclose(out[idx], ref, rtol=0, atol=1e-12)


def check_special_cases(o):
    rng = np.random.default_rng(6)
    N, H, E, M = 30, 2, 4, 3
    q, k = rng.normal(size=(N, H, E)), rng.normal(size=(N, H, E))
    gid = np.array([0] * 12 + [1] * 17 + [2])           # group 2 is a single token
    gid = gid[rng.permutation(N)]
    gate = rng.uniform(1 / M, 1, size=N)
    v = rng.normal(size=(N, H, E))
    # constant V inside each group -> out = gate * v
    vc = np.zeros_like(v)
    for m in range(M):
        vc[gid == m] = rng.normal(size=(1, H, E))
    out = o.group_attention(q, k, vc, gid, gate, M)
    assert np.allclose(out, gate[:, None, None] * vc, rtol=0, atol=1e-12)
    # q = 0 -> uniform weights -> out = gate * mean of the group's V
    out = o.group_attention(np.zeros_like(q), k, v, gid, gate, M)
    for m in range(M):
        idx = gid == m
        assert np.allclose(out[idx], gate[idx][:, None, None] * v[idx].mean(0), rtol=0, atol=1e-12)
    # singleton group -> out = gate * own v
    s = np.nonzero(gid == 2)[0][0]
    out = o.group_attention(q, k, v, gid, gate, M)
    assert np.allclose(out[s], gate[s] * v[s], rtol=0, atol=1e-14)


def check_brute_force_tiny(o):
    rng = np.random.default_rng(7)
    N, H, E, M, d = 24, 2, 4, 3, 6
    x = rng.normal(size=(N, d))
    W = rng.normal(size=(M, d))
    q, k, v = (rng.normal(size=(N, H, E)) for _ in range(3))
    res = o.moga_layer(x, W, None, q, k, v, M)
    g0, p0 = _brute_route(x.tolist(), W.tolist(), None)
    ref = _brute_masked_dense(q, k, v, g0, p0)
    assert np.array_equal(res["group_id"], g0)
    assert np.allclose(res["out"], ref, rtol=0, atol=1e-12)


def check_permutation_equivariance(o):
    rng = np.random.default_rng(8)
    N, H, E, M, d = 48, 2, 8, 5, 6
    x = rng.normal(size=(N, d))
    W = rng.normal(size=(M, d))
    q, k, v = (rng.normal(size=(N, H, E)) for _ in range(3))
    pi = rng.permutation(N)
    a = o.moga_layer(x, W, None, q, k, v, M)["out"]
    b = o.moga_layer(x[pi], W, None, q[pi], k[pi], v[pi], M)["out"]
    assert np.allclose(a[pi], b, rtol=0, atol=1e-12)


def check_stga(o):
    rng = np.random.default_rng(9)
    grid = (3, 10, 12)
    N = 360
    q, k, v = (rng.normal(size=(N, 1, 8)) for _ in range(3))
    # window = whole grid -> full attention
    assert np.allclose(o.stga_attention(q, k, v, *grid, grid), _sdpa(q, k, v), rtol=0, atol=1e-12)
    # window (1,1,1) -> out = v
    assert np.allclose(o.stga_attention(q, k, v, *grid, (1, 1, 1)), v, rtol=0, atol=1e-14)
    # clipped edge windows against brute force (10 = 4+4+2, 12 = 8+4)
    small = (2, 5, 6)
    n = 60
    qs, ks, vs = q[:n], k[:n], v[:n]
    ref = _brute_stga(qs, ks, vs, small, (2, 4, 4))
    assert np.allclose(o.stga_attention(qs, ks, vs, *small, (2, 4, 4)), ref, rtol=0, atol=1e-12)
    sets = o.stga_windows(*grid, (3, 8, 8))
    assert sorted(np.concatenate(sets).tolist()) == list(range(N)) and len(sets) == 4


def check_layer_combine(o):
    rng = np.random.default_rng(10)
    grid, N = (2, 4, 6), 48
    x = rng.normal(size=(N, 5))
    W = rng.normal(size=(3, 5))
    q, k, v = (rng.normal(size=(N, 2, 8)) for _ in range(3))
    res = o.moga_layer(x, W, None, q, k, v, 3, grid=grid, window=(1, 2, 3))
    ref_stga = _brute_stga(q, k, v, grid, (1, 2, 3))
    g0, p0 = _brute_route(x.tolist(), W.tolist(), None)
    ref = 0.5 * (_brute_masked_dense(q, k, v, g0, p0) + ref_stga)
    assert np.allclose(res["out"], ref, rtol=0, atol=1e-12)
    # M = 1 and a whole-grid window: both branches are full attention
    res = o.moga_layer(x, W[:1], None, q, k, v, 1, grid=grid, window=grid)
    assert np.allclose(res["out"], _sdpa(q, k, v), rtol=0, atol=1e-12)


def check_golden(o):
    g = _read_golden("worked_example.txt")
    inp, exp = g["input"], g["expect"]
    x = np.array(inp["x"], float)
    q, k, v = (np.array(inp[n], float).reshape(4, 1, 1) for n in ("q", "k", "v"))
    res = o.moga_layer(x, np.array(inp["W_r"], float), None, q, k, v, inp["M"])
    assert res["group_id"].tolist() == exp["group_id"]
    assert np.allclose(res["gate"], exp["gate"], rtol=0, atol=1e-15)
    assert res["perm"].tolist() == exp["perm"] and res["offsets"].tolist() == exp["offsets"]
    assert res["max_seqlen"] == exp["max_seqlen"]
    assert np.allclose(res["out"][:, 0, 0], exp["moga"], rtol=0, atol=1e-14)
    s = _read_golden("stga_example.txt")
    T, Hg, Wg = s["input"]["grid"]
    v = np.array(s["input"]["v"], float).reshape(6, 1, 1)
    out = o.stga_attention(np.zeros_like(v), np.ones_like(v), v, T, Hg, Wg, s["input"]["window"])
    assert np.allclose(out[:, 0, 0], s["expect"]["stga"], rtol=0, atol=1e-14)


def check_three_branch_mean(o):
    rng = np.random.default_rng(11)
    # brute force: frames are windows (1, Hg, Wg); the block output is the mean of three branches
    grid, N = (3, 3, 4), 36
    x = rng.normal(size=(N, 5))
    W = rng.normal(size=(3, 5))
    q, k, v = (rng.normal(size=(N, 2, 4)) for _ in range(3))
    res = o.moga_layer(x, W, None, q, k, v, 3, grid=grid, window=(2, 2, 2), per_frame=True)
    g0, p0 = _brute_route(x.tolist(), W.tolist(), None)
    ref = (_brute_masked_dense(q, k, v, g0, p0) + _brute_stga(q, k, v, grid, (2, 2, 2))
           + _brute_stga(q, k, v, grid, (1, 3, 4))) / 3
    assert np.allclose(res["out"], ref, rtol=0, atol=1e-12)
    # one frame, M = 1, whole-grid window: every branch is full attention
    grid1 = (1, 4, 5)
    q1, k1, v1 = (rng.normal(size=(20, 2, 8)) for _ in range(3))
    res = o.moga_layer(rng.normal(size=(20, 3)), rng.normal(size=(1, 3)), None, q1, k1, v1, 1,
                       grid=grid1, window=grid1, per_frame=True)
    assert np.allclose(res["out"], _sdpa(q1, k1, v1), rtol=0, atol=1e-12)


def check_balance_stats(o):
    M = 4
    # W = 0: every p(i|x) = 1/M, all tokens tie into group 0 -> F = e_0, P = 1/M, metric 1
    F, P, b = o.balance_stats(np.ones((10, 3)), np.zeros((M, 3)))
    assert np.allclose(F, [1, 0, 0, 0]) and np.allclose(P, 0.25) and abs(b - 1.0) < 1e-15
    # confident and balanced: x = 60 e_{i mod M}, W = I -> F = P = 1/M, metric -> 1
    x = np.zeros((8 * M, M))
    x[np.arange(8 * M), np.arange(8 * M) % M] = 60.0
    F, P, b = o.balance_stats(x, np.eye(M))
    assert np.allclose(F, 1 / M) and np.allclose(P, 1 / M, atol=1e-20) and abs(b - 1.0) < 1e-12
    # collapsed and confident: everything in group 2 -> metric -> M
    x = np.zeros((12, M))
    x[:, 2] = 60.0
    F, P, b = o.balance_stats(x, np.eye(M))
    assert abs(b - M) < 1e-12
    # brute force on a random case
    rng = np.random.default_rng(12)
    x, W, bias = rng.normal(size=(15, 6)), rng.normal(size=(3, 6)), rng.normal(size=3)
    g0, _ = _brute_route(x.tolist(), W.tolist(), bias.tolist())
    p_all = []
    for i in range(15):
        r = [sum(x[i, c] * W[m, c] for c in range(6)) + bias[m] for m in range(3)]
        z = sum(math.exp(v - max(r)) for v in r)
        p_all.append([math.exp(v - max(r)) / z for v in r])
    Fb = np.bincount(g0, minlength=3) / 15
    Pb = np.mean(p_all, axis=0)
    F, P, b = o.balance_stats(x, W, bias)
    assert np.allclose(F, Fb) and np.allclose(P, Pb, atol=1e-14) and abs(b - 3 * np.sum(Fb * Pb)) < 1e-13


def check_shot_stga(o):
    rng = np.random.default_rng(21)
    # brute force: temporal windows inside shots, augmented keys at the cuts
    for grid, window, shots, aug in (((5, 3, 4), (2, 2, 3), [0, 2, 5], (1, 2)),
                                     ((6, 2, 3), (0, 2, 2), [0, 1, 3, 6], (2, 2)),
                                     ((7, 2, 2), (2, 1, 2), [0, 3, 4, 7], (2, 1))):
        N = grid[0] * grid[1] * grid[2]
        q, k, v = (rng.normal(size=(N, 2, 3)) for _ in range(3))
        out = o.stga_shot_attention(q, k, v, *grid, window, shots, *aug)
        assert np.allclose(out, _brute_shot_stga(q, k, v, grid, window, shots, *aug), rtol=0, atol=1e-12)
    # one shot: plain STGA, whatever the augmentation
    q, k, v = (rng.normal(size=(6 * 4 * 4, 2, 4)) for _ in range(3))
    plain = o.stga_attention(q, k, v, 6, 4, 4, (3, 2, 2))
    assert np.allclose(o.stga_shot_attention(q, k, v, 6, 4, 4, (3, 2, 2), [0, 6], 2, 2), plain, rtol=0, atol=1e-13)
    # cuts on window boundaries and no augmentation: plain STGA again
    assert np.allclose(o.stga_shot_attention(q, k, v, 6, 4, 4, (3, 2, 2), [0, 3, 6], 0, 0), plain, rtol=0,
                       atol=1e-13)
    # queries are not augmented: every token appears in exactly one query set,
    # and key sets are query sets plus boundary frames only
    pairs = o.shot_windows(9, 2, 2, (2, 2, 2), [0, 4, 9], 2, 2)
    allq = np.sort(np.concatenate([a for a, _ in pairs]))
    assert np.array_equal(allq, np.arange(36))
    assert all(np.isin(a, b).all() for a, b in pairs)
    # perturbations: the frame before the previous shot's last two is invisible
    # to the next shot's first window; the last frame before the cut is visible
    grid, shots = (8, 2, 2), [0, 4, 8]
    q, k, v = (rng.normal(size=(32, 1, 4)) for _ in range(3))
    base = o.stga_shot_attention(q, k, v, *grid, (0, 2, 2), shots, 2, 2)
    first_win = np.arange(16, 32)                          # shot 1, frames 4..7, the only tile
    k2, v2 = k.copy(), v.copy()
    k2[4:8] += 3.0                                         # frame 1 (4 tokens) of shot 0
    v2[4:8] -= 2.0
    assert np.allclose(o.stga_shot_attention(q, k2, v2, *grid, (0, 2, 2), shots, 2, 2)[first_win],
                       base[first_win], rtol=0, atol=0)
    k3 = k.copy()
    k3[12:16] += 3.0                                       # frame 3: shot 0's last frame
    assert not np.allclose(o.stga_shot_attention(q, k3, v, *grid, (0, 2, 2), shots, 2, 2)[first_win],
                           base[first_win])


def _fd_problem(seed, M=3, window=(1, 2, 3), per_frame=True, bias=True):
    rng = np.random.default_rng(seed)
    grid, N, d, H, E = (2, 3, 4), 24, 5, 2, 4
    x = rng.normal(size=(N, d))
    W = rng.normal(size=(M, d))
    b = rng.normal(size=M) if bias else None
    q, k, v = (rng.normal(size=(N, H, E)) for _ in range(3))
    dout = rng.normal(size=(N, H, E))
    return dict(x=x, W_r=W, b_r=b, q=q, k=k, v=v, M=M, grid=grid, window=window, per_frame=per_frame, dout=dout)


def check_backward_finite_differences(o):
    """Every gradient of L = sum(dout * out) against central differences of
    the (separately pinned) forward, on sampled coordinates of every input."""
    for seed, kw in ((30, {}), (31, {"window": None, "per_frame": False}), (32, {"per_frame": False}),
                     (33, {"window": None})):
        pr = _fd_problem(seed, **kw)
        fwd_args = {k_: pr[k_] for k_ in ("x", "W_r", "b_r", "q", "k", "v")}
        M, grid, window, pf, dout = pr["M"], pr["grid"], pr["window"], pr["per_frame"], pr["dout"]

        def loss(a):
            res = o.moga_layer(a["x"], a["W_r"], a["b_r"], a["q"], a["k"], a["v"], M, grid=grid, window=window,
                               per_frame=pf)
            return float(np.sum(dout * res["out"]))

        _, _, margin = o.route(pr["x"], pr["W_r"], pr["b_r"])
        assert margin.min() > 1e-4          # a step of 1e-6 cannot move a token to another group
        g = o.moga_layer_backward(pr["x"], pr["W_r"], pr["b_r"], pr["q"], pr["k"], pr["v"], M, dout, grid=grid,
                                  window=window, per_frame=pf)
        names = {"x": "dx", "W_r": "dW_r", "b_r": "db_r", "q": "dq", "k": "dk", "v": "dv"}
        rng = np.random.default_rng(seed + 100)
        eps = 1e-6
        for name, gname in names.items():
            base = fwd_args[name]
            flat = base.reshape(-1)
            for c in rng.choice(flat.size, size=min(flat.size, 12), replace=False):
                a = dict(fwd_args)
                plus = flat.copy()
                plus[c] += eps
                minus = flat.copy()
                minus[c] -= eps
                a[name] = plus.reshape(base.shape)
                lp = loss(a)
                a[name] = minus.reshape(base.shape)
                lm = loss(a)
                num = (lp - lm) / (2 * eps)
                ana = g[gname].reshape(-1)[c]
                assert abs(num - ana) <= 1e-6 * (1 + abs(num)), (seed, gname, int(c), num, ana)


def check_balance_loss_gradient(o):
    """The balancing-loss term of the router gradient against central
    differences of alpha * M * sum_i F_i P_i computed with ``balance_stats``
    (F held at the unperturbed assignment)."""
    rng = np.random.default_rng(80)
    N, d, M, alpha = 30, 6, 4, 0.7
    x = rng.normal(size=(N, d))
    W = rng.normal(size=(M, d))
    b = rng.normal(size=M)
    q, k, v = (rng.normal(size=(N, 1, 4)) for _ in range(3))
    zero = np.zeros((N, 1, 4))
    g = o.moga_layer_backward(x, W, b, q, k, v, M, zero, balance_alpha=alpha)
    F0, _, _ = o.balance_stats(x, W, b)

    def loss(xx, WW, bb):
        _, P, _ = o.balance_stats(xx, WW, bb)
        return alpha * M * float(np.sum(F0 * P))

    eps = 1e-6
    for name, arr, gname in (("x", x, "dx"), ("W_r", W, "dW_r"), ("b_r", b, "db_r")):
        flat = arr.reshape(-1)
        for c in rng.choice(flat.size, size=min(flat.size, 10), replace=False):
            pl, mi = flat.copy(), flat.copy()
            pl[c] += eps
            mi[c] -= eps
            args_p = {"x": x, "W_r": W, "b_r": b}
            args_m = dict(args_p)
            args_p[name] = pl.reshape(arr.shape)
            args_m[name] = mi.reshape(arr.shape)
            num = (loss(args_p["x"], args_p["W_r"], args_p["b_r"]) - loss(args_m["x"], args_m["W_r"], args_m["b_r"])) / (2 * eps)
            ana = g[gname].reshape(-1)[c]
            assert abs(num - ana) <= 1e-7 * (1 + abs(num)), (gname, int(c), num, ana)


def check_backward_dense_autograd(o):
    """The same gradients from torch autograd (float64) through a dense
    formulation: every branch as N x N attention with a membership mask."""
    pr = _fd_problem(40, M=4)
    t = {k_: torch.tensor(pr[k_], dtype=torch.float64, requires_grad=True)
         for k_ in ("x", "W_r", "b_r", "q", "k", "v")}
    N, H, E = pr["q"].shape
    T, Hg, Wg = pr["grid"]
    r = t["x"] @ t["W_r"].T + t["b_r"]
    p = torch.softmax(r, dim=1)
    gid = torch.argmax(r.detach(), dim=1)
    gate = p.gather(1, gid[:, None])[:, 0]
    tok = torch.arange(N)
    tt, hh, ww = tok // (Hg * Wg), (tok // Wg) % Hg, tok % Wg
    wt, wh, wwid = pr["window"]
    win = (tt // wt) * 1000 + (hh // wh) * 100 + ww // wwid
    masks = [gid[:, None] == gid[None, :], win[:, None] == win[None, :], tt[:, None] == tt[None, :]]

    def dense(mask):
        s = torch.einsum("ihe,jhe->hij", t["q"], t["k"]) / math.sqrt(E)
        s = s.masked_fill(~mask[None], float("-inf"))
        return torch.einsum("hij,jhe->ihe", torch.softmax(s, dim=2), t["v"])

    out = (gate[:, None, None] * dense(masks[0]) + dense(masks[1]) + dense(masks[2])) / 3
    (out * torch.tensor(pr["dout"])).sum().backward()
    g = o.moga_layer_backward(pr["x"], pr["W_r"], pr["b_r"], pr["q"], pr["k"], pr["v"], pr["M"], pr["dout"],
                              grid=pr["grid"], window=pr["window"], per_frame=True)
    for name, gname in (("x", "dx"), ("W_r", "dW_r"), ("b_r", "db_r"), ("q", "dq"), ("k", "dk"), ("v", "dv")):
        assert np.allclose(g[gname], t[name].grad.numpy(), rtol=1e-9, atol=1e-11), gname


def check_backward_special_cases(o):
    pr = _fd_problem(50, M=1, window=None, per_frame=False)
    g = o.moga_layer_backward(pr["x"], pr["W_r"], pr["b_r"], pr["q"], pr["k"], pr["v"], 1, pr["dout"])
    # one group: the gate is identically 1, so the router gets no gradient
    assert np.abs(g["dW_r"]).max() == 0 and np.abs(g["db_r"]).max() == 0 and np.abs(g["dx"]).max() == 0
    # a token alone in its group: out = gate * v, so dv = gate * dout and dq = dk = 0
    rng = np.random.default_rng(51)
    N, d, H, E = 6, 3, 1, 4
    x = np.eye(N, d) * 5.0
    x[3:] = 0.0
    x[3:, 0] = 5.0                     # tokens 0, 3, 4, 5 -> group 0; 1 -> group 1; 2 -> group 2
    W = np.eye(3, d)
    q, k, v, dout = (rng.normal(size=(N, H, E)) for _ in range(4))
    g = o.moga_layer_backward(x, W, None, q, k, v, 3, dout)
    _, gate, _ = o.route(x, W, None)
    assert np.allclose(g["dv"][1], gate[1] * dout[1], rtol=0, atol=1e-14)
    assert np.abs(g["dq"][1]).max() < 1e-15 and np.abs(g["dk"][1]).max() < 1e-15


def check_attention_lse(o):
    from scipy.special import logsumexp
    rng = np.random.default_rng(60)
    q, K = rng.normal(size=(7, 16)) * 3, rng.normal(size=(33, 16)) * 3
    ref = logsumexp(q @ K.T / 4.0, axis=1)
    assert np.allclose(o.attention_lse(q, K), ref, rtol=0, atol=1e-12)


def check_dq_rows(o):
    """Row-wise dQ equals the dQ rows of the whole-set backward, and torch
    autograd of Eq. 1 (float64) for those rows."""
    rng = np.random.default_rng(70)
    Q, K, V, dO = (rng.normal(size=(40, 8)) for _ in range(4))
    rows = np.array([0, 7, 39])
    dq, out = o.attention_dq_rows(Q[rows], K, V, dO[rows])
    full = o.attention_rows_backward(Q, K, V, dO)
    assert np.allclose(dq, full[0][rows], rtol=1e-12, atol=1e-12)
    assert np.allclose(out, full[3][rows], rtol=1e-12, atol=1e-12)
    tq = torch.tensor(Q[rows], requires_grad=True)
    o_t = torch.softmax(tq @ torch.tensor(K).T / math.sqrt(8), dim=1) @ torch.tensor(V)
    (o_t * torch.tensor(dO[rows])).sum().backward()
    assert np.allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)


CHECKS = [check_route_closed_form, check_route_ties_and_M1, check_route_brute, check_counting_sort,
          check_full_attention_when_M1, check_group_equals_subset_attention, check_special_cases,
          check_brute_force_tiny, check_permutation_equivariance, check_stga, check_layer_combine,
          check_golden, check_three_branch_mean, check_balance_stats, check_shot_stga,
          check_backward_finite_differences, check_backward_dense_autograd, check_backward_special_cases,
          check_attention_lse, check_dq_rows, check_balance_loss_gradient]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_oracle_pin(check):
    check(oracle)


# ----------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one check
# ----------------------------------------------------------------------------
def _wrong_scale(q_rows, K, V):
    s = (q_rows @ K.T) / K.shape[1]
    p = np.exp(s - s.max(1, keepdims=True))
    return (p / p.sum(1, keepdims=True)) @ V


def _no_max_transpose(q_rows, K, V):                   # softmax over the wrong axis
    s = (q_rows @ K.T) / math.sqrt(K.shape[1])
    p = np.exp(s - s.max(0, keepdims=True))
    return (p / p.sum(0, keepdims=True)) @ V


def _route_last_argmax(x, W_r, b_r=None):
    gid, gate, margin = _ORIG_ROUTE(x, W_r, b_r)
    W = np.asarray(W_r, float)
    r = np.asarray(x, float) @ W.T + (0 if b_r is None else np.asarray(b_r, float))
    last = r.shape[1] - 1 - np.argmax(r[:, ::-1], axis=1)
    return last.astype(np.int32), gate, margin


def _route_gate_of_group0(x, W_r, b_r=None):
    gid, gate, margin = _ORIG_ROUTE(x, W_r, b_r)
    W = np.asarray(W_r, float)
    r = np.asarray(x, float) @ W.T
    e = np.exp(r - r.max(1, keepdims=True))
    return gid, (e / e.sum(1, keepdims=True))[:, 0], margin


def _unstable_sort(group_id, M):
    perm, offsets, mx = _ORIG_SORT(group_id, M)
    out = perm.copy()
    for m in range(M):
        out[offsets[m]:offsets[m + 1]] = out[offsets[m]:offsets[m + 1]][::-1]
    return out, offsets, mx


def _no_gate(q, k, v, group_id, gate, M, rows=None, heads=None):
    return _ORIG_GA(q, k, v, group_id, np.ones(len(group_id)), M, rows, heads)


def _windows_off_by_one(T, Hg, Wg, window):
    return _ORIG_WIN(T, Hg, Wg, (window[0], window[1], window[2] + 1))


def _shot_aug_on_queries(T, Hg, Wg, window, shot_start, aug_prev=2, aug_next=2):
    return [(b, b) for _, b in _ORIG_SHOT(T, Hg, Wg, window, shot_start, aug_prev, aug_next)]


def _shot_aug_short(T, Hg, Wg, window, shot_start, aug_prev=2, aug_next=2):
    return _ORIG_SHOT(T, Hg, Wg, window, shot_start, max(aug_prev - 1, 0), aug_next)


def _shot_ignores_cuts(T, Hg, Wg, window, shot_start, aug_prev=2, aug_next=2):
    return _ORIG_SHOT(T, Hg, Wg, window, [0, T], aug_prev, aug_next)


def _bwd_no_jacobian_term(Q, K, V, dO):            # dS = P * dP, the row-sum term dropped
    c = 1.0 / math.sqrt(K.shape[1])
    S = (Q @ K.T) * c
    P = np.exp(S - S.max(1, keepdims=True))
    P = P / P.sum(1, keepdims=True)
    dS = P * (dO @ V.T)
    return (dS @ K) * c, (dS.T @ Q) * c, P.T @ dO, P @ V


def _bwd_dk_untransposed(Q, K, V, dO):              # dK = dS Q instead of dS^T Q
    dq, dk, dv, O = _ORIG_ABWD(Q, K, V, dO)
    c = 1.0 / math.sqrt(K.shape[1])
    S = (Q @ K.T) * c
    P = np.exp(S - S.max(1, keepdims=True))
    P = P / P.sum(1, keepdims=True)
    dP = dO @ V.T
    dS = P * (dP - (P * dP).sum(1, keepdims=True))
    return dq, (dS @ Q) * c, dv, O


def _bwd_router_sign(*a, **kw):                     # gradient ascent on the router
    g = _ORIG_LBWD(*a, **kw)
    for n in ("dx", "dW_r", "db_r"):
        g[n] = -g[n]
    return g


def _bwd_balance_sign(*a, **kw):                   # the balancing term added with the wrong sign
    alpha = kw.get("balance_alpha", 0.0)
    if not alpha:
        return _ORIG_LBWD(*a, **kw)
    g0 = _ORIG_LBWD(*a, **dict(kw, balance_alpha=0.0))
    g1 = _ORIG_LBWD(*a, **kw)
    return {n: (2 * g0[n] - g1[n]) if n in ("dx", "dW_r", "db_r") else g1[n] for n in g1}


def _lse_no_scale(q_rows, K):
    s = q_rows @ K.T
    m = s.max(axis=1)
    return m + np.log(np.exp(s - m[:, None]).sum(axis=1))


_ORIG_ABWD = oracle.attention_rows_backward
_ORIG_LBWD = oracle.moga_layer_backward
_ORIG_SHOT = oracle.shot_windows
_ORIG_GA = oracle.group_attention
_ORIG_WIN = oracle.stga_windows
_ORIG_ROUTE = oracle.route
_ORIG_SORT = oracle.counting_sort

MUTANTS = {
    "scale_1_over_d": ("attention_rows", _wrong_scale),
    "softmax_wrong_axis": ("attention_rows", _no_max_transpose),
    "argmax_last_on_ties": ("route", _route_last_argmax),
    "gate_of_wrong_group": ("route", _route_gate_of_group0),
    "unstable_group_order": ("counting_sort", _unstable_sort),
    "gate_dropped": ("group_attention", _no_gate),
    "window_width_off_by_one": ("stga_windows", _windows_off_by_one),
    "shot_augments_queries": ("shot_windows", _shot_aug_on_queries),
    "shot_augmentation_short": ("shot_windows", _shot_aug_short),
    "shot_cuts_ignored": ("shot_windows", _shot_ignores_cuts),
    "bwd_softmax_jacobian_term_dropped": ("attention_rows_backward", _bwd_no_jacobian_term),
    "bwd_dk_untransposed": ("attention_rows_backward", _bwd_dk_untransposed),
    "bwd_router_sign_flipped": ("moga_layer_backward", _bwd_router_sign),
    "lse_without_scale": ("attention_lse", _lse_no_scale),
    "balance_gradient_sign_flipped": ("moga_layer_backward", _bwd_balance_sign),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(oracle, attr, fn)
    caught = []
    for check in CHECKS:
        try:
            check(oracle)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"planted mistake {name} went unnoticed by every pin"
