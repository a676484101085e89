"""Seeded synthetic inputs for the MoGA layer.

This module only draws random numbers and lays them out. It holds none of the
method's arithmetic: no routing, sorting or attention happens here.  Both the
CUDA path (through its tests and ``bench.py``) and the CPU oracle consume what
it produces, so the two sides always see the same input bits.

Shapes follow the workloads the MoGA pages describe (MoGA: Mixture-of-Groups
Attention for End-to-End Long Video Generation, §3.4 "Vanilla Self-Attention":
480p latent grid of 30x52 tokens per latent frame; §4 hyper-parameters: 187k
tokens for 30 s on Wan2.1-1.3B, about 580k tokens for the minute-long model).

Recipe (all draws from one ``torch.Generator`` seeded with ``seed``, in the
fixed order below):

* ``normal``     x ~ N(0, 1); W_r ~ N(0, 1/d); no bias.
* ``clustered``  8 centroids c_k ~ N(0, I_d); each token picks k uniformly;
                 x = c_k + 0.5 * eps.  W_r ~ N(0, 1/d); no bias.  Groups come
                 out uneven and some may be empty when M > 8.
* ``skew``       M - 8 live groups with centroids c_k ~ N(0, I_d); W_r row k is
                 c_k / |c_k| (rows of the 8 dead groups are random unit rows
                 with bias -30, so they stay empty).  Token clusters are drawn
                 from a Zipf(s = 1.5) law over the first M - 16 groups (group 0
                 takes about 40 % of the tokens); then 87 random tokens are
                 reassigned so that the next 8 groups hold exactly
                 1, 2, 3, 5, 8, 13, 21, 34 tokens.  x = c_k + 0.5 * eps.
* q, k, v ~ N(0, 1), stored in bf16, layout [N, H, d_h].
  ``peaky=True`` instead draws z ~ N(0,1) and sets q = 2 z, k = 2 (z + 0.1 n),
  so each query's own key dominates its softmax row.

x and W_r are bf16 except for the ``tiny`` workload, which is fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "custom"]


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    H: int
    d_h: int
    d: int
    M: int
    x_dtype: str                      # "f32" or "bf16"
    x_kind: str                       # "normal" | "clustered" | "skew"
    grid: Optional[Tuple[int, int, int]] = None    # (T, Hg, Wg), N = T*Hg*Wg
    window: Optional[Tuple[int, int, int]] = None  # STGA window (wt, wh, ww)
    peaky: bool = False

    def describe(self) -> str:
        g = "x".join(map(str, self.grid)) if self.grid else "none"
        w = "x".join(map(str, self.window)) if self.window else "none"
        return (f"N={self.N} H={self.H} d_h={self.d_h} d={self.d} M={self.M} "
                f"x={self.x_kind}/{self.x_dtype} grid={g} window={w}")


# Latent grid of a 480p frame after the VAE (8x8) and patchify (2x2): 30 x 52.
WORKLOADS = {
    "tiny": Workload("tiny", 1024, 1, 64, 64, 4, "f32", "normal"),
    "wan_32k": Workload("wan_32k", 32760, 12, 128, 1536, 8, "bf16", "clustered",
                        (21, 30, 52), (3, 8, 8)),
    "video_187k": Workload("video_187k", 187200, 12, 128, 1536, 16, "bf16", "clustered",
                           (120, 30, 52), (3, 8, 8)),
    "minute_580k": Workload("minute_580k", 580320, 40, 128, 5120, 32, "bf16", "clustered",
                            (372, 30, 52), (3, 8, 8)),
    "skew_187k": Workload("skew_187k", 187200, 12, 128, 1536, 64, "bf16", "skew",
                          (120, 30, 52), (3, 8, 8)),
    # video_187k with 4 heads: q/k/v still exceed L2 (192 MB each) while the
    # device footprint stays near 2 GB, for hardware-counter captures.
    "profile_187k_h4": Workload("profile_187k_h4", 187200, 4, 128, 1536, 16, "bf16", "clustered",
                                (120, 30, 52), (3, 8, 8)),
    # the same with 2 heads, for full captures of the training kernels
    # (gathered q/k/v/dO copies of 96 MB each; about 1.5 GB on the device)
    "profile_187k_h2": Workload("profile_187k_h2", 187200, 2, 128, 1536, 16, "bf16", "clustered",
                                (120, 30, 52), (3, 8, 8)),
}

_FORCED = (1, 2, 3, 5, 8, 13, 21, 34)   # sizes of the forced small groups (skew)
_N_CENTROIDS = 8                        # centroids of the clustered recipe


def custom(N, H=1, d_h=64, d=64, M=4, x_dtype="bf16", x_kind="normal",
           grid=None, window=None, peaky=False, name="custom") -> Workload:
    if grid is not None:
        assert grid[0] * grid[1] * grid[2] == N, "grid must cover N tokens"
    return Workload(name, N, H, d_h, d, M, x_dtype, x_kind,
                    tuple(grid) if grid else None, tuple(window) if window else None, peaky)


def _randn(shape, gen, device, chunk_elems=1 << 28):
    """fp32 N(0,1) draws, produced in row chunks to bound temporary memory."""
    rows = shape[0]
    per_row = int(math.prod(shape[1:])) if len(shape) > 1 else 1
    step = max(1, chunk_elems // max(per_row, 1))
    out = torch.empty(shape, dtype=torch.float32, device=device)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 device=device, dtype=torch.float32)
    return out


def _randn_bf16(shape, gen, device, chunk_elems=1 << 28):
    rows = shape[0]
    per_row = int(math.prod(shape[1:])) if len(shape) > 1 else 1
    step = max(1, chunk_elems // max(per_row, 1))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def _x_from_centroids(cent, idx, gen, device, out_dtype, chunk_rows=16384):
    N, d = idx.shape[0], cent.shape[1]
    x = torch.empty((N, d), dtype=out_dtype, device=device)
    for r0 in range(0, N, chunk_rows):
        r1 = min(N, r0 + chunk_rows)
        eps = torch.randn((r1 - r0, d), generator=gen, device=device, dtype=torch.float32)
        x[r0:r1] = (cent[idx[r0:r1]] + 0.5 * eps).to(out_dtype)
    return x


def make_inputs(wl: Workload, seed: int = 0, device="cpu", with_qkv: bool = True):
    """Draw the inputs of one MoGA layer.

    Returns a dict with ``x`` [N,d], ``W_r`` [M,d] (nn.Linear layout),
    ``b_r`` [M] fp32 or None, and (when ``with_qkv``) ``q``, ``k``, ``v``
    [N,H,d_h] bf16.  Everything lives on ``device``.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    xdt = torch.float32 if wl.x_dtype == "f32" else torch.bfloat16
    N, d, M = wl.N, wl.d, wl.M
    b_r = None
    if wl.x_kind == "normal":
        x = _randn((N, d), gen, device).to(xdt)
        W = (_randn((M, d), gen, device) / math.sqrt(d)).to(xdt)
    elif wl.x_kind == "clustered":
        cent = _randn((_N_CENTROIDS, d), gen, device)
        idx = torch.randint(0, _N_CENTROIDS, (N,), generator=gen, device=device)
        x = _x_from_centroids(cent, idx, gen, device, xdt)
        W = (_randn((M, d), gen, device) / math.sqrt(d)).to(xdt)
    elif wl.x_kind == "skew":
        n_forced, n_dead = len(_FORCED), 8
        live = M - n_dead
        zipf_groups = live - n_forced
        assert zipf_groups >= 1 and N > sum(_FORCED), "skew recipe needs M >= 17, N > 87"
        cent = _randn((live, d), gen, device)
        dead = _randn((n_dead, d), gen, device)
        W32 = torch.cat([cent / cent.norm(dim=1, keepdim=True),
                         dead / dead.norm(dim=1, keepdim=True)], 0)
        W = W32.to(xdt)
        b_r = torch.zeros(M, dtype=torch.float32, device=device)
        b_r[live:] = -30.0
        ranks = torch.arange(1, zipf_groups + 1, device=device, dtype=torch.float64)
        pz = (ranks ** -1.5)
        pz = (pz / pz.sum()).to(torch.float32)
        idx = torch.multinomial(pz, N, replacement=True, generator=gen)
        pos = torch.randperm(N, generator=gen, device=device)[: sum(_FORCED)]
        o = 0
        for j, cnt in enumerate(_FORCED):
            idx[pos[o:o + cnt]] = zipf_groups + j
            o += cnt
        x = _x_from_centroids(cent, idx, gen, device, xdt)
    else:
        raise ValueError(f"unknown x_kind {wl.x_kind!r}")
    out = {"x": x.contiguous(), "W_r": W.contiguous(), "b_r": b_r}
    if with_qkv:
        shp = (N, wl.H, wl.d_h)
        if wl.peaky:
            z = _randn(shp, gen, device)
            n = _randn(shp, gen, device)
            out["q"] = (2.0 * z).to(torch.bfloat16)
            out["k"] = (2.0 * (z + 0.1 * n)).to(torch.bfloat16)
            del z, n
            out["v"] = _randn_bf16(shp, gen, device)
        else:
            out["q"] = _randn_bf16(shp, gen, device)
            out["k"] = _randn_bf16(shp, gen, device)
            out["v"] = _randn_bf16(shp, gen, device)
    return out


def with_window(wl: Workload, window) -> Workload:
    return replace(wl, window=tuple(window) if window else None)
