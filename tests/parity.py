"""Comparison helpers shared by the GPU parity tests (no method arithmetic).

Tolerances (written here once, used by every parity test):
* group_id: bit-exact, except tokens whose oracle top-1/top-2 logit margin is
  below MARGIN (counted, reported and excluded).
* perm, offsets, max_seqlen: bit-exact against the oracle's counting sort of
  the GPU's own group_id (and against the oracle's routing when no excluded
  token flipped).
* gate: |gpu - oracle| <= GATE_TOL_F32 (fp32 inputs) / GATE_TOL_BF16.
* bf16 attention outputs: max-abs <= OUT_MAX_ABS and relative L2 <= OUT_REL_L2,
  checked per group (outputs of large groups are small, so a global max-abs
  bound alone would be loose).
"""
import numpy as np
import torch

import oracle

MARGIN = 1e-3
GATE_TOL_F32 = 1e-5
GATE_TOL_BF16 = 1e-4
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 1e-2


def np_cpu(t):
    t = t.detach()
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.cpu().numpy()


def check_route(res, x, W_r, b_r, M, gate_tol):
    """Checks a moga_route result against the oracle; returns (gid_gpu, ref)."""
    ref_gid, ref_gate, margin = oracle.route(np_cpu(x), np_cpu(W_r), None if b_r is None else np_cpu(b_r))
    gid = np_cpu(res["group_id"]).astype(np.int64)
    N = gid.shape[0]
    near = margin < MARGIN
    bad = (gid != ref_gid) & ~near
    assert not bad.any(), f"{bad.sum()} group ids differ away from near-ties (first at {np.nonzero(bad)[0][:5]})"
    assert ((gid >= 0) & (gid < M)).all()
    same = gid == ref_gid
    gate = np_cpu(res["gate"])
    err = np.abs(gate[same] - ref_gate[same]).max() if same.any() else 0.0
    assert err <= gate_tol, f"gate error {err}"
    assert (gate >= 1.0 / M - 1e-6).all() and (gate <= 1.0 + 1e-6).all()
    perm_ref, off_ref, mx_ref = oracle.counting_sort(gid, M)
    assert np.array_equal(np_cpu(res["perm"]), perm_ref), "perm differs from the stable counting sort"
    assert np.array_equal(np_cpu(res["offsets"]), off_ref), "offsets differ"
    if "max_seqlen" in res:
        assert int(np_cpu(res["max_seqlen"])[0]) == mx_ref
    if same.all():
        p2, o2, _ = oracle.counting_sort(ref_gid, M)
        assert np.array_equal(np_cpu(res["perm"]), p2) and np.array_equal(np_cpu(res["offsets"]), o2)
    return gid, {"gid": ref_gid, "gate": ref_gate, "margin": margin, "n_near": int(near.sum()),
                 "n_flipped": int((~same).sum())}


def compare_out(out_gpu, ref, groups=None, rows=None, heads=None, what="out"):
    """Per-group max-abs / rel-L2 check of bf16 outputs against float64 refs."""
    o = np_cpu(out_gpu).astype(np.float64)
    if rows is not None:
        rows = np.asarray(rows)
        o, ref = o[rows], ref[rows]
        groups = None if groups is None else np.asarray(groups)[rows]
    if heads is not None:
        o, ref = o[:, heads], ref[:, heads]
    assert np.isfinite(o).all(), f"{what}: non-finite GPU output"
    keys = [None] if groups is None else np.unique(groups)
    worst = (0.0, 0.0)
    for g in keys:
        sel = slice(None) if g is None else (groups == g)
        a, b = o[sel], ref[sel]
        mad = float(np.abs(a - b).max()) if a.size else 0.0
        rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)) if a.size else 0.0
        assert mad <= OUT_MAX_ABS, f"{what}: group {g} max-abs {mad:.3e}"
        assert rel <= OUT_REL_L2, f"{what}: group {g} rel-L2 {rel:.3e}"
        worst = (max(worst[0], mad), max(worst[1], rel))
    return worst


def groups_to_perm(gid, M):
    """Test-side input construction (numpy library calls, not the oracle)."""
    gid = np.asarray(gid, dtype=np.int64)
    perm = np.argsort(gid, kind="stable").astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(np.bincount(gid, minlength=M))]).astype(np.int32)
    return perm, offsets


def sample_rows(gid, M, grid, window, rng, per_group=256, stga_rows=1024):
    """Seeded row sample for full-size parity checks.

    Every row of the two smallest non-empty groups, ``per_group`` random rows
    of every other group (all of them when the group is smaller), and, with a
    window, ``stga_rows`` tokens spread evenly over the window kinds the grid
    has: whole windows, and windows clipped in rows, in columns, in both, and
    (when T is not a multiple of the temporal extent) in time.  Each sampled
    row is later compared in full: its whole group / window is attended.
    """
    gid = np.asarray(gid)
    rows = []
    counts = np.bincount(gid, minlength=M)
    nonempty = [int(m) for m in np.argsort(counts, kind="stable") if counts[m] > 0]
    for m in nonempty[:2]:
        rows.append(np.nonzero(gid == m)[0])
    for m in nonempty[2:]:
        idx = np.nonzero(gid == m)[0]
        rows.append(rng.choice(idx, size=min(per_group, idx.size), replace=False))
    if window is not None and stga_rows:
        T, Hg, Wg = grid
        wt, wh, ww = window
        tok = np.arange(T * Hg * Wg)
        t, h, w = tok // (Hg * Wg), (tok // Wg) % Hg, tok % Wg
        ct = (t // wt) * wt + wt > T
        ch = (h // wh) * wh + wh > Hg
        cw = (w // ww) * ww + ww > Wg
        kind = ct.astype(np.int64) * 4 + ch * 2 + cw
        kinds = np.unique(kind)
        per = max(1, stga_rows // kinds.size)
        for kd in kinds:
            idx = np.nonzero(kind == kd)[0]
            rows.append(rng.choice(idx, size=min(per, idx.size), replace=False))
    return np.unique(np.concatenate(rows))
