"""CPU oracle for one Mixture-of-Groups Attention (MoGA) layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the package's smoke
check and the benchmark's CPU-baseline / reference arm may import this module.
It shares no code with the CUDA library: it is plain numpy in float64, written
from the method's definitions, and slow on purpose so that a reader can check
each step against the text by eye.

Source of every definition: "MoGA: Mixture-of-Groups Attention for End-to-End
Long Video Generation" (arXiv 2510.18692), as summarised on the paper-graph-ui
page of that title, §3.4 "Detailed, Sentence-Based Technical Breakdown":

* Eq. 1  SA(q, K, V) = softmax(q K^T / sqrt(d)) V         ("Vanilla Self-Attention")
* Eq. 2  r = Router(x) = x W_r (+ b), W_r in R^{d x M}      ("MoGA Router")
* Eq. 3  p(i|x) = softmax(r)_i                              ("MoGA Router")
* Eq. 4  g(x) = argmax_i p(i|x)                             ("MoGA Router")
* Eq. 5  MoGA(x) = p(g(x)|x) * SA(q, K_g(x), V_g(x))        ("Grouped Attention")
* Algorithm 1: route, permute Q/K/V into contiguous per-group segments
  (cu_seqlen, max_seqlen, permute index), attend per segment, un-permute
  ("MoGA Pseudocode and Kernel Integration").
* STGA: attention inside fixed local spatio-temporal windows; the block output
  is the mean of the MoGA and STGA outputs ("Spatial-Temporal Group Attention").

Readings where the pages leave a step open (each one is pinned by a test):

* softmax scale: 1/sqrt(d_h) per head (Algorithm 1 hands each head to
  FlashAttention, whose default scale is 1/sqrt(head dim)).
* argmax ties: the lowest group index wins.  softmax is strictly increasing, so
  argmax p = argmax r; it is taken on r, where rounding cannot create ties.
* order inside a group: original token index ascending (a stable sort), which
  makes the permutation unique.  ``perm[j]`` = original index of the token at
  sorted position j (the inverse of the pages' original-to-permuted index).
* STGA windows: non-overlapping boxes of (wt, wh, ww) tokens anchored at the
  grid origin, clipped at the grid edges; token index (t*Hg + h)*Wg + w.
* shot-aware STGA: temporal groups never cross a shot boundary.  Within each
  shot, temporal windows of wt frames tile the shot from its first frame and
  are clipped at its last (wt = 0: one window per shot).  Keys and values, not
  queries, of a shot's first temporal window are augmented with the last
  aug_prev frames of the previous shot, and those of its last temporal window
  with the first aug_next frames of the next shot, in the window's spatial tile
  (the pages say "two latent frames from adjacent shots": aug_prev = aug_next
  = 2 by default, each clipped to the neighbouring shot's length).
* combine: out = (MoGA + STGA) / 2 when STGA is on, MoGA alone otherwise; with
  the per-frame branch (attention inside each latent frame) the block output
  is the plain mean of all branches that are on.
* gradients ("MoGA Router" and "Grouped Attention": the argmax is not
  differentiable; gradients reach the router through the gate p(g(x)|x) of
  Eq. 5 and reach q, k, v through the attention given the hard assignment).
  The assignment g(x) is held fixed; no straight-through term is added.

Every function here is pinned by ``tests/test_oracle_pins.py`` to something
other than itself (closed forms, a library attention routine, numpy's stable
argsort, brute force on tiny inputs, invariants).  No function is unpinned.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "route", "balance_stats", "counting_sort", "attention_rows", "group_attention",
    "stga_windows", "stga_attention", "frame_attention", "moga_layer",
    "shot_windows", "stga_shot_attention", "attention_lse", "attention_rows_backward",
    "moga_layer_backward", "attention_dq_rows",
]

_ROW_BLOCK = 16384


def _f64(a) -> np.ndarray:
    """Exact upcast to float64 (accepts numpy arrays or torch CPU tensors)."""
    if hasattr(a, "detach"):
        a = a.detach()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def route(x, W_r, b_r=None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Router, softmax gate and hard assignment (Eqs. 2-4).

    x: [N, d]; W_r: [M, d] (row i is group i's prototype, i.e. the transposed
    d x M matrix of Eq. 2); b_r: [M] or None.
    Returns (group_id int32 [N], gate float64 [N], margin float64 [N]) where
    gate = p(g(x)|x) and margin = r_(1) - r_(2), the gap between the largest
    and second largest logit (infinite when M == 1).
    """
    W = _f64(W_r)
    M = W.shape[0]
    b = np.zeros(M) if b_r is None else _f64(b_r)
    N = x.shape[0]
    gid = np.empty(N, dtype=np.int32)
    gate = np.empty(N, dtype=np.float64)
    margin = np.empty(N, dtype=np.float64)
    for r0 in range(0, N, _ROW_BLOCK):
        r1 = min(N, r0 + _ROW_BLOCK)
        r = _f64(x[r0:r1]) @ W.T + b                      # Eq. 2
        e = np.exp(r - r.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)              # Eq. 3
        g = np.argmax(r, axis=1)                          # Eq. 4, first max wins
        gid[r0:r1] = g
        gate[r0:r1] = p[np.arange(r1 - r0), g]
        if M == 1:
            margin[r0:r1] = np.inf
        else:
            top2 = np.sort(r, axis=1)[:, -2:]
            margin[r0:r1] = top2[:, 1] - top2[:, 0]
    return gid, gate, margin


def balance_stats(x, W_r, b_r=None):
    """Group-balancing statistics ("Group Balancing Loss", Eq. 6).

    Reading taken (the pages' P_i definition and their limiting values
    disagree): F_i = fraction of tokens whose argmax group is i, P_i = mean of
    p(i|x) over ALL tokens, metric = M * sum_i F_i * P_i (1 when balanced and
    confident, M when collapsed onto one group).  Returns (F, P, metric).
    """
    W = _f64(W_r)
    M = W.shape[0]
    b = np.zeros(M) if b_r is None else _f64(b_r)
    N = x.shape[0]
    counts = np.zeros(M)
    psum = np.zeros(M)
    for r0 in range(0, N, _ROW_BLOCK):
        r = _f64(x[r0:r0 + _ROW_BLOCK]) @ W.T + b
        e = np.exp(r - r.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        psum += p.sum(axis=0)
        counts += np.bincount(np.argmax(r, axis=1), minlength=M)
    F = counts / N
    P = psum / N
    return F, P, float(M * np.sum(F * P))


def counting_sort(group_id, M: int) -> Tuple[np.ndarray, np.ndarray, int]:
    """Algorithm 1 step 2 index part: group tokens into contiguous segments.

    Returns (perm int32 [N], offsets int32 [M+1], max_seqlen) where
    offsets is the cu_seqlen array (exclusive prefix sum of the group sizes,
    offsets[M] = N) and perm lists group 0's tokens in index order, then
    group 1's, and so on.
    """
    g = np.asarray(group_id, dtype=np.int64)
    counts = np.array([(g == m).sum() for m in range(M)], dtype=np.int64)
    offsets = np.zeros(M + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.concatenate([np.nonzero(g == m)[0] for m in range(M)] + [np.zeros(0, np.int64)])
    max_seqlen = int(counts.max()) if M > 0 else 0
    return perm.astype(np.int32), offsets.astype(np.int32), max_seqlen


def attention_rows(q_rows: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Eq. 1 for a block of queries of one head: softmax(q K^T / sqrt(d_h)) V.

    q_rows [r, d_h], K and V [n, d_h]; float64 throughout, max-subtracted
    softmax over the n keys of each row.
    """
    d_h = K.shape[1]
    s = (q_rows @ K.T) / math.sqrt(d_h)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


def _attend_sets(q, k, v, sets: Iterable[np.ndarray], row_pos, heads, scale_rows,
                 out: np.ndarray, q_block: int = 512):
    """Attention of each token set's queries to the same set's keys/values.

    row_pos[i] is the output row of token i (or -1 when token i is not
    requested); heads lists the heads to compute, in output order.
    """
    for idx in sets:
        if idx.size == 0:
            continue
        qi = idx[row_pos[idx] >= 0]
        if qi.size == 0:
            continue
        for hp, h in enumerate(heads):
            Kh = _f64(k[idx, h])
            Vh = _f64(v[idx, h])
            for b0 in range(0, qi.size, q_block):
                rows = qi[b0:b0 + q_block]
                o = attention_rows(_f64(q[rows, h]), Kh, Vh)
                if scale_rows is not None:
                    o = o * scale_rows[rows][:, None]
                out[row_pos[rows], hp] = o
    return out


def _row_layout(N, H, d_h, rows, heads):
    """Output buffer and token -> output-row map for full or sampled runs."""
    heads = list(range(H)) if heads is None else [int(h) for h in heads]
    row_pos = np.full(N, -1, dtype=np.int64)
    if rows is None:
        row_pos[:] = np.arange(N)
        n_out = N
    else:
        rows = np.asarray(rows, dtype=np.int64)
        row_pos[rows] = np.arange(rows.size)
        n_out = rows.size
    return np.full((n_out, len(heads), d_h), np.nan), row_pos, heads


def group_attention(q, k, v, group_id, gate, M: int,
                    rows: Optional[Sequence[int]] = None,
                    heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """MoGA output, Eq. 5, computed directly in original token order.

    out[i, h] = gate[i] * SA(q[i,h], K_{g(i),h}, V_{g(i),h}) where K_g, V_g hold
    the keys/values of every token routed to g(i).  q, k, v: [N, H, d_h]
    arrays or tensors (any float type; upcast exactly to float64, and only the
    rows a group needs are read).  Returns [N, H, d_h]; with ``rows`` (distinct
    token indices) and/or ``heads`` only those are computed and the result is
    [len(rows), len(heads), d_h] in the given order.
    """
    N, H, d_h = q.shape
    g = np.asarray(group_id, dtype=np.int64)
    gate = _f64(gate)
    out, row_pos, hs = _row_layout(N, H, d_h, rows, heads)
    sets = (np.nonzero(g == m)[0] for m in range(M))
    return _attend_sets(q, k, v, sets, row_pos, hs, gate, out)


def stga_windows(T: int, Hg: int, Wg: int, window) -> List[np.ndarray]:
    """Token index sets of the STGA windows (non-overlapping, clipped at edges).

    Windows are enumerated with the temporal block outermost, then rows, then
    columns; tokens inside a window are listed in index order.
    """
    wt, wh, ww = window
    sets = []
    for t0 in range(0, T, wt):
        for h0 in range(0, Hg, wh):
            for w0 in range(0, Wg, ww):
                ts = np.arange(t0, min(T, t0 + wt))
                hs = np.arange(h0, min(Hg, h0 + wh))
                ws = np.arange(w0, min(Wg, w0 + ww))
                idx = ((ts[:, None, None] * Hg + hs[None, :, None]) * Wg
                       + ws[None, None, :]).reshape(-1)
                sets.append(np.sort(idx))
    return sets


def stga_attention(q, k, v, T: int, Hg: int, Wg: int, window,
                   rows: Optional[Sequence[int]] = None,
                   heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """STGA: full attention inside each spatio-temporal window (no gate).

    Output layout as for ``group_attention``.
    """
    N, H, d_h = q.shape
    assert T * Hg * Wg == N
    out, row_pos, hs = _row_layout(N, H, d_h, rows, heads)
    return _attend_sets(q, k, v, stga_windows(T, Hg, Wg, window), row_pos, hs, None, out)


def frame_attention(q, k, v, T: int, Hg: int, Wg: int, rows=None, heads=None) -> np.ndarray:
    """Per-frame branch: full attention among the tokens of each latent frame
    (the STGA definition with a window of one whole frame)."""
    return stga_attention(q, k, v, T, Hg, Wg, (1, Hg, Wg), rows=rows, heads=heads)


def _tile_tokens(frames: np.ndarray, hs: np.ndarray, ws: np.ndarray, Hg: int, Wg: int) -> np.ndarray:
    """Token indices (t*Hg + h)*Wg + w of a box of frames x rows x columns, sorted."""
    idx = ((frames[:, None, None] * Hg + hs[None, :, None]) * Wg + ws[None, None, :]).reshape(-1)
    return np.sort(idx)


def shot_windows(T: int, Hg: int, Wg: int, window, shot_start: Sequence[int],
                 aug_prev: int = 2, aug_next: int = 2) -> List[Tuple[np.ndarray, np.ndarray]]:
    """(query tokens, key/value tokens) of every shot-aware STGA window
    ("Spatial-Temporal Group Attention": frames of different shots are in
    distinct temporal groups; keys and values, not queries, see two latent
    frames of the adjacent shots).

    shot_start: 0 = s_0 < s_1 < ... < s_S = T; shot j holds frames
    [s_j, s_{j+1}).  Windows go shot by shot, then temporal window, then
    spatial rows, then columns; the query sets cover every token once.
    """
    wt, wh, ww = (int(w) for w in window)
    s = [int(v) for v in shot_start]
    assert s[0] == 0 and s[-1] == T and all(a < b for a, b in zip(s, s[1:]))
    S = len(s) - 1
    pairs = []
    for j in range(S):
        a, b = s[j], s[j + 1]
        step = wt if wt > 0 else b - a
        for t0 in range(a, b, step):
            t1 = min(b, t0 + step)
            extra = []
            if t0 == a and j > 0:                     # first window of the shot
                extra.append(np.arange(max(s[j - 1], a - aug_prev), a))
            if t1 == b and j < S - 1:                 # last window of the shot
                extra.append(np.arange(b, min(s[j + 2], b + aug_next)))
            own = np.arange(t0, t1)
            kv_frames = np.concatenate([own] + extra) if extra else own
            for h0 in range(0, Hg, wh):
                for w0 in range(0, Wg, ww):
                    hs = np.arange(h0, min(Hg, h0 + wh))
                    ws = np.arange(w0, min(Wg, w0 + ww))
                    pairs.append((_tile_tokens(own, hs, ws, Hg, Wg),
                                  _tile_tokens(kv_frames, hs, ws, Hg, Wg)))
    return pairs


def stga_shot_attention(q, k, v, T: int, Hg: int, Wg: int, window, shot_start,
                        aug_prev: int = 2, aug_next: int = 2,
                        rows: Optional[Sequence[int]] = None,
                        heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """Shot-aware STGA: each query attends to its window's tokens plus the
    window's boundary frames of the adjacent shots (see ``shot_windows``).

    Output layout as for ``group_attention``.
    """
    N, H, d_h = q.shape
    assert T * Hg * Wg == N
    out, row_pos, hs = _row_layout(N, H, d_h, rows, heads)
    for qidx, kidx in shot_windows(T, Hg, Wg, window, shot_start, aug_prev, aug_next):
        qi = qidx[row_pos[qidx] >= 0]
        if qi.size == 0:
            continue
        for hp, h in enumerate(hs):
            o = attention_rows(_f64(q[qi, h]), _f64(k[kidx, h]), _f64(v[kidx, h]))
            out[row_pos[qi], hp] = o
    return out


def moga_layer(x, W_r, b_r, q, k, v, M: int, grid=None, window=None,
               rows=None, heads=None, per_frame: bool = False):
    """One visual attention block: route, group attention, optional STGA and
    per-frame branches, and the arithmetic mean of the branches that are on.

    Returns a dict with group_id, gate, margin, perm, offsets, max_seqlen,
    moga (Eq. 5 output), stga / frame (or None) and out (the block output).
    """
    gid, gate, margin = route(x, W_r, b_r)
    perm, offsets, max_seqlen = counting_sort(gid, M)
    moga = group_attention(q, k, v, gid, gate, M, rows=rows, heads=heads)
    branches = [moga]
    stga = frame = None
    if window is not None:
        T, Hg, Wg = grid
        stga = stga_attention(q, k, v, T, Hg, Wg, window, rows=rows, heads=heads)
        branches.append(stga)
    if per_frame:
        T, Hg, Wg = grid
        frame = frame_attention(q, k, v, T, Hg, Wg, rows=rows, heads=heads)
        branches.append(frame)
    out = branches[0] if len(branches) == 1 else sum(branches) / len(branches)
    return {"group_id": gid, "gate": gate, "margin": margin, "perm": perm,
            "offsets": offsets, "max_seqlen": max_seqlen, "moga": moga,
            "stga": stga, "frame": frame, "out": out}


# ----------------------------------------------------------------------------- training
def attention_lse(q_rows: np.ndarray, K: np.ndarray) -> np.ndarray:
    """Natural-log log-sum-exp of each query row's scaled scores q K^T / sqrt(d_h)
    (the normaliser of Eq. 1's softmax), written out as max + log(sum(exp))."""
    s = (q_rows @ K.T) / math.sqrt(K.shape[1])
    m = s.max(axis=1)
    return m + np.log(np.exp(s - m[:, None]).sum(axis=1))


def attention_rows_backward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray):
    """Gradients of Eq. 1 over one token set of one head, given dO = dL/dO.

    With S = Q K^T / sqrt(d_h), P = softmax_rows(S), O = P V:
      dV = P^T dO;   dP = dO V^T;
      dS = P * (dP - rowsum(P * dP))        (Jacobian of the row softmax);
      dQ = dS K / sqrt(d_h);   dK = dS^T Q / sqrt(d_h).
    Returns (dQ, dK, dV, O), float64.
    """
    c = 1.0 / math.sqrt(K.shape[1])
    S = (Q @ K.T) * c
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=1, keepdims=True)
    O = P @ V
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
    return (dS @ K) * c, (dS.T @ Q) * c, dV, O


def moga_layer_backward(x, W_r, b_r, q, k, v, M: int, dout, grid=None, window=None,
                        per_frame: bool = False, balance_alpha: float = 0.0):
    """Gradients of L = sum(dout * out) + alpha * M * sum_i F_i P_i for the
    block of ``moga_layer`` (the second term is the group balancing loss of
    Eq. 6 in the reading of ``balance_stats``; F_i, a count of argmax
    assignments, is piecewise constant and carries no gradient).

    out = mean over the branches that are on of: MoGA (Eq. 5: gate * SA within
    the token's group), STGA (SA within each window), per-frame (SA within each
    frame).  Each branch's share of dout is dout / (number of branches).  The
    group assignment is held fixed (see the module notes); the gate
    p = softmax(x W_r^T + b)_g carries the router's gradient:
      dgate_i = sum_{h,c} w * dout[i,h,c] * SA_i[h,c];
      dr_ij   = dgate_i * p_ig * ([j == g] - p_ij)      (softmax Jacobian)
              + alpha * M / N * p_ij * (F_j - sum_k F_k p_ik)   (balancing loss);
      dW_r = dr^T x;  db_r = sum_i dr_i;  dx = dr W_r   (the router's part of dx).
    Returns a dict of float64 arrays dx [N, d], dW_r [M, d], db_r [M],
    dq, dk, dv [N, H, d_h], plus dgate [N].
    """
    X = _f64(x)
    W = _f64(W_r)
    b = np.zeros(M) if b_r is None else _f64(b_r)
    Q, Kt, Vt, dOut = _f64(q), _f64(k), _f64(v), _f64(dout)
    N, H, d_h = Q.shape
    r = X @ W.T + b                                         # Eq. 2
    e = np.exp(r - r.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)                    # Eq. 3
    g = np.argmax(r, axis=1)                                # Eq. 4
    gate = p[np.arange(N), g]
    nb = 1 + (window is not None) + bool(per_frame)
    w = 1.0 / nb
    dq = np.zeros_like(Q)
    dk = np.zeros_like(Q)
    dv = np.zeros_like(Q)
    dgate = np.zeros(N)

    def branch(sets, scale_rows):
        for idx in sets:
            if idx.size == 0:
                continue
            for h in range(H):
                dO = w * dOut[idx, h]
                if scale_rows is not None:
                    dO = dO * scale_rows[idx][:, None]
                gq, gk, gv, O = attention_rows_backward(Q[idx, h], Kt[idx, h], Vt[idx, h], dO)
                dq[idx, h] += gq
                dk[idx, h] += gk
                dv[idx, h] += gv
                if scale_rows is not None:                  # d/dgate of gate * SA
                    dgate[idx] += w * (dOut[idx, h] * O).sum(axis=1)

    branch([np.nonzero(g == m)[0] for m in range(M)], gate)
    if window is not None:
        branch(stga_windows(*grid, window), None)
    if per_frame:
        branch(stga_windows(*grid, (1, grid[1], grid[2])), None)
    onehot = np.zeros((N, M))
    onehot[np.arange(N), g] = 1.0
    dr = (dgate * gate)[:, None] * (onehot - p)
    if balance_alpha:
        F = np.bincount(g, minlength=M) / N
        dr += (balance_alpha * M / N) * p * (F[None, :] - (p @ F)[:, None])
    return {"dx": dr @ W, "dW_r": dr.T @ X, "db_r": dr.sum(axis=0),
            "dq": dq, "dk": dk, "dv": dv, "dgate": dgate}


def attention_dq_rows(Q_rows: np.ndarray, K: np.ndarray, V: np.ndarray, dO_rows: np.ndarray):
    """dQ of selected query rows of one head, each row on its own (the rows of
    ``attention_rows_backward`` computed without the other queries).

    For a query row q with scores s = q K^T / sqrt(d_h), p = softmax(s),
    o = p V and its output gradient g:  dp = g V^T,
    ds = p * (dp - sum(p * dp)),  dq = ds K / sqrt(d_h).
    Returns (dq [r, d_h], o [r, d_h]).
    """
    c = 1.0 / math.sqrt(K.shape[1])
    S = (Q_rows @ K.T) * c
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=1, keepdims=True)
    dP = dO_rows @ V.T
    dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
    return (dS @ K) * c, P @ V
