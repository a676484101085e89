"""Python binding of the MoGA layer library (``libmoga.so``, C ABI in moga.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and the current CUDA stream.  There
is no CPU fallback: if the library is missing or a call fails, an exception
is raised.

Method: "MoGA: Mixture-of-Groups Attention for End-to-End Long Video
Generation" (paper-graph-ui summary, §3.4: router Eqs. 2-4, grouped attention
Eq. 5, Algorithm 1, STGA).
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence

import torch

__all__ = ["MogaError", "get_lib", "LIB_PATH", "HEADER_PATH", "route", "group_attn", "stga_window_attn",
           "moga_layer", "sync_status", "workspace", "MogaLayer", "exported_names", "kernel_launches",
           "set_timing_events", "STAGES", "Pipeline", "stga_shot_attn", "moga_layer_shots", "sort",
           "layer_train", "layer_backward", "MogaFunction"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoga.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moga.h")

MOGA_F32, MOGA_BF16 = 0, 1
STATUS = {0: "MOGA_OK", 1: "MOGA_ERR_INVALID_ARG", 2: "MOGA_ERR_UNSUPPORTED", 3: "MOGA_ERR_WORKSPACE",
          4: "MOGA_ERR_CUDA", 5: "MOGA_ERR_TIMEOUT", 6: "MOGA_ERR_DEVICE_CHECK"}


class MogaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


_lib = None
_P, _I64, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def get_lib():
    """Loads libmoga.so (raises ImportError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m learned_token_group_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "moga_status_string": (ctypes.c_char_p, [_I]),
        "moga_version": (_I, []),
        "moga_set_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
        "moga_route_workspace_size": (_SZ, [_I64, _I]),
        "moga_route": (_I, [_P, _P, _P, _I, _I64, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_group_attn_workspace_size": (_SZ, [_I64, _I, _I, _I]),
        "moga_group_attn": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I, _I, _I, _F, _P, _P, _SZ, _P]),
        "stga_window_attn_workspace_size": (_SZ, [_I, _I, _I, _P, _I, _I]),
        "stga_window_attn": (_I, [_P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _P, _P, _SZ, _P]),
        "moga_layer_workspace_size": (_SZ, [_I64, _I, _I, _I, _I, _I, _I, _P]),
        "moga_layer": (_I, [_P, _P, _P, _I, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _P,
                            _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_sync_status": (_I, [_P, _P]),
        "moga_layer_ex_workspace_size": (_SZ, [_I64, _I, _I, _I, _I]),
        "moga_route_ex_workspace_size": (_SZ, [_I64, _I]),
        "moga_route_ex": (_I, [_P, _P, _P, _I, _I64, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_layer_ex": (_I, [_P, _P, _P, _I, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _P, _I,
                               _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_kernel_launches": (ctypes.c_uint64, []),
        "moga_route_noalloc": (_I, [_P, _P, _P, _I, _I64, _I, _I, _P, _P, _P, _P, _P, _P]),
        "moga_route_noalloc_status": (_I, [_P]),
        "moga_set_timing_events": (_I, [_I, _P, _P]),
        "moga_debug_inject": (_I, [_I]),
        "stga_shot_attn_workspace_size": (_SZ, [_I, _I, _I, _P, _I, _I, _I, _I, _I]),
        "stga_shot_attn": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _SZ, _P]),
        "moga_layer_shots_workspace_size": (_SZ, [_I64, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I, _I]),
        "moga_layer_shots": (_I, [_P, _P, _P, _I, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _P, _P, _I, _I,
                                  _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_sort_workspace_size": (_SZ, [_I64, _I]),
        "moga_sort": (_I, [_P, _I64, _I, _P, _P, _P, _P, _SZ, _P]),
        "moga_pipe_create": (_I, [_I64, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I, ctypes.POINTER(_P)]),
        "moga_pipe_submit": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "moga_pipe_sync": (_I, [_P]),
        "moga_pipe_destroy": (_I, [_P]),
        "moga_layer_train_workspace_size": (_SZ, [_I64, _I, _I, _I, _I, _I, _I, _P]),
        "moga_layer_train": (_I, [_P, _P, _P, _I, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _P,
                                  _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_layer_backward_workspace_size": (_SZ, [_I64, _I, _I, _I, _I]),
        "moga_layer_train_ex_workspace_size": (_SZ, [_I64, _I, _I, _I, _I, _I, _I, _P, _I]),
        "moga_layer_train_ex": (_I, [_P, _P, _P, _I, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _P, _I,
                                     _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_layer_backward_ex": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _P, _I, _F,
                                        _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
        "moga_layer_backward": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _I, _P,
                                     _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def exported_names():
    """Function names declared in include/moga.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:moga|stga)_[a-z_0-9]+)\s*\(", text)))


# ----------------------------------------------------------------------------- helpers
def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(st: int, what: str):
    if st != 0:
        raise MogaError(st, what)


def _int3(w):
    return (ctypes.c_int * 3)(*[int(v) for v in w])


def _dev_tensor(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def workspace(nbytes: int, device) -> torch.Tensor:
    """Zero-filled device workspace (the status word must start clear)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


STAGES = {"router": 0, "sort": 1, "gather": 2, "group_attn": 3, "stga_prep": 4, "stga_attn": 5}


def kernel_launches() -> int:
    """Kernels launched by the library so far in this process."""
    return int(get_lib().moga_kernel_launches())


def set_timing_events(stage: str, begin=None, end=None) -> None:
    """Attach (or detach, with None) a torch.cuda.Event pair to a stage."""
    b = None if begin is None else ctypes.c_void_p(begin.cuda_event)
    e = None if end is None else ctypes.c_void_p(end.cuda_event)
    _check(get_lib().moga_set_timing_events(STAGES[stage], b, e), "moga_set_timing_events")


def sync_status(ws: torch.Tensor) -> None:
    """Synchronises the current stream and raises if a kernel flagged an error."""
    _check(get_lib().moga_sync_status(_ptr(ws), _stream(ws.device)), "device status")


# ----------------------------------------------------------------------------- calls
def route(x: torch.Tensor, W_r: torch.Tensor, b_r: Optional[torch.Tensor], M: int, out=None, ws=None):
    """moga_route: returns dict(group_id, gate, perm, offsets, max_seqlen) on x's device."""
    lib = get_lib()
    _dev_tensor(x, "x")
    _dev_tensor(W_r, "W_r", x.dtype)
    if b_r is not None:
        _dev_tensor(b_r, "b_r", torch.float32)
    dt = {torch.float32: MOGA_F32, torch.bfloat16: MOGA_BF16}[x.dtype]
    N, d = x.shape
    dev = x.device
    if out is None:
        out = {"group_id": torch.empty(N, dtype=torch.int32, device=dev),
               "gate": torch.empty(N, dtype=torch.float32, device=dev),
               "perm": torch.empty(N, dtype=torch.int32, device=dev),
               "offsets": torch.empty(M + 1, dtype=torch.int32, device=dev),
               "max_seqlen": torch.empty(1, dtype=torch.int32, device=dev)}
    need = lib.moga_route_workspace_size(N, M)
    if ws is None:
        ws = workspace(need, dev)
    st = lib.moga_route(_ptr(x), _ptr(W_r), _ptr(b_r), dt, N, d, M, _ptr(out["group_id"]), _ptr(out["gate"]),
                        _ptr(out["perm"]), _ptr(out["offsets"]), _ptr(out["max_seqlen"]), _ptr(ws), ws.numel(),
                        _stream(dev))
    _check(st, "moga_route")
    return out


def sort(group_id: torch.Tensor, M: int, ws=None):
    """Counting sort of caller-given group ids (moga_sort): dict(perm, offsets, max_seqlen, ws)."""
    lib = get_lib()
    _dev_tensor(group_id, "group_id", torch.int32)
    N = group_id.numel()
    dev = group_id.device
    if ws is None:
        ws = workspace(lib.moga_sort_workspace_size(N, M), dev)
    res = {"perm": torch.empty(N, dtype=torch.int32, device=dev),
           "offsets": torch.empty(M + 1, dtype=torch.int32, device=dev),
           "max_seqlen": torch.empty(1, dtype=torch.int32, device=dev), "ws": ws}
    st = lib.moga_sort(_ptr(group_id), N, M, _ptr(res["perm"]), _ptr(res["offsets"]), _ptr(res["max_seqlen"]),
                       _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "moga_sort")
    return res


def route_stats(x: torch.Tensor, W_r: torch.Tensor, b_r: Optional[torch.Tensor], M: int):
    """moga_route_ex: routing plus balancing statistics.

    Returns dict(group_id, gate, perm, offsets, max_seqlen, prob_mean [M], balance [1]).
    """
    lib = get_lib()
    _dev_tensor(x, "x")
    _dev_tensor(W_r, "W_r", x.dtype)
    dt = {torch.float32: MOGA_F32, torch.bfloat16: MOGA_BF16}[x.dtype]
    N, d = x.shape
    dev = x.device
    out = {"group_id": torch.empty(N, dtype=torch.int32, device=dev),
           "gate": torch.empty(N, dtype=torch.float32, device=dev),
           "perm": torch.empty(N, dtype=torch.int32, device=dev),
           "offsets": torch.empty(M + 1, dtype=torch.int32, device=dev),
           "max_seqlen": torch.empty(1, dtype=torch.int32, device=dev),
           "prob_mean": torch.empty(M, dtype=torch.float32, device=dev),
           "balance": torch.empty(1, dtype=torch.float32, device=dev)}
    ws = workspace(lib.moga_route_ex_workspace_size(N, M), dev)
    st = lib.moga_route_ex(_ptr(x), _ptr(W_r), _ptr(b_r), dt, N, d, M, _ptr(out["group_id"]), _ptr(out["gate"]),
                           _ptr(out["perm"]), _ptr(out["offsets"]), _ptr(out["max_seqlen"]), _ptr(out["prob_mean"]),
                           _ptr(out["balance"]), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "moga_route_ex")
    return out


def group_attn(q, k, v, perm, offsets, gate, M: int, out_scale: float = 1.0, out=None, ws=None):
    """moga_group_attn: out[perm[j]] = out_scale * gate * SA within each segment."""
    lib = get_lib()
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(perm, "perm", torch.int32)
    _dev_tensor(offsets, "offsets", torch.int32)
    if gate is not None:
        _dev_tensor(gate, "gate", torch.float32)
    N, H, d_h = q.shape
    if out is None:
        out = torch.empty_like(q)
    need = lib.moga_group_attn_workspace_size(N, H, d_h, M)
    if ws is None:
        ws = workspace(need, q.device)
    st = lib.moga_group_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(perm), _ptr(offsets), _ptr(gate), N, H, d_h, M,
                             float(out_scale), _ptr(out), _ptr(ws), ws.numel(), _stream(q.device))
    _check(st, "moga_group_attn")
    return out


def stga_window_attn(q, k, v, grid: Sequence[int], window: Sequence[int], accumulate: bool = False,
                     out=None, ws=None):
    """stga_window_attn over a (T, Hg, Wg) grid with (wt, wh, ww) windows."""
    lib = get_lib()
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, n, torch.bfloat16)
    N, H, d_h = q.shape
    T, Hg, Wg = (int(g) for g in grid)
    w3 = _int3(window)
    if out is None:
        if accumulate:
            raise ValueError("accumulate=True needs an existing out tensor")
        out = torch.empty_like(q)
    need = lib.stga_window_attn_workspace_size(T, Hg, Wg, w3, H, d_h)
    if ws is None:
        ws = workspace(need, q.device)
    st = lib.stga_window_attn(_ptr(q), _ptr(k), _ptr(v), T, Hg, Wg, w3, H, d_h, int(bool(accumulate)),
                              _ptr(out), _ptr(ws), ws.numel(), _stream(q.device))
    _check(st, "stga_window_attn")
    return out


def stga_shot_attn(q, k, v, grid: Sequence[int], window: Sequence[int], shot_start: torch.Tensor,
                   aug_prev: int = 2, aug_next: int = 2, out_scale: float = 1.0, accumulate: bool = False,
                   out=None, ws=None):
    """Shot-aware STGA over a (T, Hg, Wg) grid (stga_shot_attn in moga.h).

    shot_start: device int32 [nshots + 1] frame boundaries (0 ... T); window
    (wt, wh, ww) with wt = 0 for one temporal window per shot.
    """
    lib = get_lib()
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(shot_start, "shot_start", torch.int32)
    N, H, d_h = q.shape
    T, Hg, Wg = (int(g) for g in grid)
    w3 = _int3(window)
    nshots = shot_start.numel() - 1
    if out is None:
        if accumulate:
            raise ValueError("accumulate=True needs an existing out tensor")
        out = torch.empty_like(q)
    if ws is None:
        ws = workspace(lib.stga_shot_attn_workspace_size(T, Hg, Wg, w3, nshots, aug_prev, aug_next, H, d_h),
                       q.device)
    st = lib.stga_shot_attn(_ptr(q), _ptr(k), _ptr(v), T, Hg, Wg, w3, _ptr(shot_start), nshots, int(aug_prev),
                            int(aug_next), H, d_h, float(out_scale), int(bool(accumulate)), _ptr(out), _ptr(ws),
                            ws.numel(), _stream(q.device))
    _check(st, "stga_shot_attn")
    return out, ws


def moga_layer_shots(x, W_r, b_r, q, k, v, M: int, grid, window, shot_start: torch.Tensor, aug_prev: int = 2,
                     aug_next: int = 2, per_frame: bool = True, res=None):
    """The pages' visual block in one call: MoGA, shot-aware STGA and (per_frame)
    the per-frame branch, averaged.  Returns dict(out, group_id, gate, perm,
    offsets, ws); pass that dict back as ``res`` to reuse its buffers."""
    lib = get_lib()
    N, d = x.shape
    _, H, d_h = q.shape
    for n, t in (("x", x), ("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, n)
    _dev_tensor(shot_start, "shot_start", torch.int32)
    T, Hg, Wg = (int(g) for g in grid)
    w3 = _int3(window)
    nshots = shot_start.numel() - 1
    dev = x.device
    x_dt = {torch.float32: MOGA_F32, torch.bfloat16: MOGA_BF16}[x.dtype]
    need = lib.moga_layer_shots_workspace_size(N, H, d_h, M, T, Hg, Wg, w3, nshots, aug_prev, aug_next,
                                               int(bool(per_frame)))
    if res is None or res["ws"].numel() < need:
        res = {"out": torch.empty((N, H, d_h), dtype=torch.bfloat16, device=dev),
               "group_id": torch.empty(N, dtype=torch.int32, device=dev),
               "gate": torch.empty(N, dtype=torch.float32, device=dev),
               "perm": torch.empty(N, dtype=torch.int32, device=dev),
               "offsets": torch.empty(M + 1, dtype=torch.int32, device=dev), "ws": workspace(need, dev)}
    ws = res["ws"]
    st = lib.moga_layer_shots(_ptr(x), _ptr(W_r), _ptr(b_r), x_dt, _ptr(q), _ptr(k), _ptr(v), N, d, H, d_h, M, T,
                              Hg, Wg, w3, _ptr(shot_start), nshots, int(aug_prev), int(aug_next),
                              int(bool(per_frame)), _ptr(res["out"]), _ptr(res["group_id"]), _ptr(res["gate"]),
                              _ptr(res["perm"]), _ptr(res["offsets"]), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "moga_layer_shots")
    return res


class MogaLayer:
    """Preallocated outputs + workspace for repeated calls of one visual block.

    window: STGA window (or None); per_frame: add the per-frame branch (the
    block output is then the mean of all branches that are on).
    """

    def __init__(self, N, d, H, d_h, M, grid=None, window=None, x_dtype=torch.bfloat16, device="cuda",
                 per_frame: bool = False):
        lib = get_lib()
        self.N, self.d, self.H, self.d_h, self.M = N, d, H, d_h, M
        self.grid = tuple(grid) if grid is not None else (0, 0, 0)
        self.window = tuple(window) if window is not None else None
        self.branches = (1 if self.window else 0) | (2 if per_frame else 0)
        self.x_dt = {torch.float32: MOGA_F32, torch.bfloat16: MOGA_BF16}[x_dtype]
        self.device = torch.device(device)
        self._w3 = _int3(self.window) if self.window else None
        need = lib.moga_layer_ex_workspace_size(N, H, d_h, M, self.branches)
        self.ws = workspace(need, self.device)
        self.out = torch.empty((N, H, d_h), dtype=torch.bfloat16, device=self.device)
        self.group_id = torch.empty(N, dtype=torch.int32, device=self.device)
        self.gate = torch.empty(N, dtype=torch.float32, device=self.device)
        self.perm = torch.empty(N, dtype=torch.int32, device=self.device)
        self.offsets = torch.empty(M + 1, dtype=torch.int32, device=self.device)

    def __call__(self, x, W_r, b_r, q, k, v):
        lib = get_lib()
        if self.branches & 2:
            st = lib.moga_layer_ex(_ptr(x), _ptr(W_r), _ptr(b_r), self.x_dt, _ptr(q), _ptr(k), _ptr(v), self.N,
                                   self.d, self.H, self.d_h, self.M, *self.grid, self._w3, self.branches,
                                   _ptr(self.out), _ptr(self.group_id), _ptr(self.gate), _ptr(self.perm),
                                   _ptr(self.offsets), _ptr(self.ws), self.ws.numel(), _stream(self.device))
            _check(st, "moga_layer_ex")
        else:
            st = lib.moga_layer(_ptr(x), _ptr(W_r), _ptr(b_r), self.x_dt, _ptr(q), _ptr(k), _ptr(v), self.N,
                                self.d, self.H, self.d_h, self.M, *self.grid, self._w3, _ptr(self.out),
                                _ptr(self.group_id), _ptr(self.gate), _ptr(self.perm), _ptr(self.offsets),
                                _ptr(self.ws), self.ws.numel(), _stream(self.device))
            _check(st, "moga_layer")
        return self.out


def moga_layer(x, W_r, b_r, q, k, v, M: int, grid=None, window=None, per_frame: bool = False):
    """One MoGA block: returns dict(out, group_id, gate, perm, offsets, ws)."""
    N, d = x.shape
    _, H, d_h = q.shape
    for n, t in (("x", x), ("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, n)
    layer = MogaLayer(N, d, H, d_h, M, grid, window, x.dtype, x.device, per_frame=per_frame)
    layer(x, W_r, b_r, q, k, v)
    return {"out": layer.out, "group_id": layer.group_id, "gate": layer.gate, "perm": layer.perm,
            "offsets": layer.offsets, "ws": layer.ws}


def layer_train(x, W_r, b_r, q, k, v, M: int, grid=None, window=None, ws=None, res=None, per_frame: bool = False):
    """Training forward of one block (moga_layer_train_ex in moga.h): returns
    dict(out, o_moga, o_stga, o_frame, lse_moga, lse_stga, lse_frame,
    group_id, gate, perm, offsets, ws); everything but out is what
    ``layer_backward`` needs.  per_frame adds the per-frame branch (out is the
    mean of the branches).  ``res``: a previous result of the same shapes
    whose buffers are reused."""
    lib = get_lib()
    N, d = x.shape
    _, H, d_h = q.shape
    for n, t in (("x", x), ("W_r", W_r), ("q", q), ("k", k), ("v", v)):
        _dev_tensor(t, n)
    dev = q.device
    grid3 = tuple(int(g) for g in grid) if grid is not None else (0, 0, 0)
    w3 = _int3(window) if window is not None else None
    x_dt = {torch.float32: MOGA_F32, torch.bfloat16: MOGA_BF16}[x.dtype]
    mat = lambda: torch.empty((N, H, d_h), dtype=torch.bfloat16, device=dev)
    if res is not None:
        ws = res["ws"] if ws is None else ws
    vec = lambda: torch.empty((H, N), dtype=torch.float32, device=dev)
    r = dict(res) if res is not None else {"out": mat(), "o_moga": mat(), "o_stga": mat() if window is not None else None,
         "o_frame": mat() if per_frame else None,
         "lse_moga": vec(), "lse_stga": vec() if window is not None else None, "lse_frame": vec() if per_frame else None,
         "group_id": torch.empty(N, dtype=torch.int32, device=dev),
         "gate": torch.empty(N, dtype=torch.float32, device=dev),
         "perm": torch.empty(N, dtype=torch.int32, device=dev),
         "offsets": torch.empty(M + 1, dtype=torch.int32, device=dev)}
    need = lib.moga_layer_train_ex_workspace_size(N, H, d_h, M, *grid3, w3, int(bool(per_frame)))
    if ws is None or ws.numel() < need:
        ws = workspace(need, dev)
    st = lib.moga_layer_train_ex(_ptr(x), _ptr(W_r), _ptr(b_r), x_dt, _ptr(q), _ptr(k), _ptr(v), N, d, H, d_h, M,
                                 *grid3, w3, int(bool(per_frame)), _ptr(r["out"]), _ptr(r["o_moga"]),
                                 _ptr(r["o_stga"]), _ptr(r["o_frame"]), _ptr(r["lse_moga"]), _ptr(r["lse_stga"]),
                                 _ptr(r["lse_frame"]), _ptr(r["group_id"]), _ptr(r["gate"]), _ptr(r["perm"]),
                                 _ptr(r["offsets"]), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "moga_layer_train_ex")
    r["per_frame"] = bool(per_frame)
    r["ws"] = ws
    return r


def layer_backward(dout, saved, x, W_r, b_r, q, k, v, M: int, grid=None, window=None, ws=None, grads=None,
                   balance_alpha: float = 0.0):
    """Gradients of one block (moga_layer_backward_ex in moga.h) from dout and
    the dict ``layer_train`` returned: dict(dx, dW_r, db_r, dq, dk, dv, ws).
    db_r is None when b_r is None.  balance_alpha adds the group balancing
    loss alpha * M * sum_i F_i P_i to the router's gradient.  ``grads``: a
    previous result of the same shapes whose buffers are reused."""
    lib = get_lib()
    N, d = x.shape
    _, H, d_h = q.shape
    _dev_tensor(dout, "dout", torch.bfloat16)
    dev = q.device
    grid3 = tuple(int(g) for g in grid) if grid is not None else (0, 0, 0)
    w3 = _int3(window) if window is not None else None
    x_dt = {torch.float32: MOGA_F32, torch.bfloat16: MOGA_BF16}[x.dtype]
    if grads is not None:
        ws = grads["ws"] if ws is None else ws
    g = dict(grads) if grads is not None else {"dx": torch.empty_like(x),
         "dW_r": torch.empty((M, d), dtype=torch.float32, device=dev),
         "db_r": torch.empty(M, dtype=torch.float32, device=dev) if b_r is not None else None,
         "dq": torch.empty_like(q), "dk": torch.empty_like(q), "dv": torch.empty_like(q)}
    need = lib.moga_layer_backward_workspace_size(N, d, H, d_h, M)
    if ws is None or ws.numel() < need:
        ws = workspace(need, dev)
    s = saved
    pf = int(bool(s.get("per_frame", False)))
    st = lib.moga_layer_backward_ex(_ptr(dout), _ptr(x), _ptr(W_r), _ptr(b_r), x_dt, _ptr(q), _ptr(k), _ptr(v), N,
                                    d, H, d_h, M, *grid3, w3, pf, float(balance_alpha), _ptr(s["o_moga"]),
                                    _ptr(s["o_stga"]),
                                    _ptr(s.get("o_frame")), _ptr(s["lse_moga"]), _ptr(s["lse_stga"]),
                                    _ptr(s.get("lse_frame")), _ptr(s["group_id"]), _ptr(s["gate"]),
                                    _ptr(s["perm"]), _ptr(s["offsets"]), _ptr(g["dx"]), _ptr(g["dW_r"]),
                                    _ptr(g["db_r"]), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(ws),
                                    ws.numel(), _stream(dev))
    _check(st, "moga_layer_backward_ex")
    g["ws"] = ws
    return g


class MogaFunction(torch.autograd.Function):
    """The block as an autograd function: out = MogaFunction.apply(x, W_r,
    b_r, q, k, v, M, grid, window, per_frame, balance_alpha).  Forward runs
    ``layer_train``, backward ``layer_backward``; the group assignment is held
    fixed, so gradients reach the router through the gate (and, with
    balance_alpha, through the group balancing loss, which the caller adds to
    its loss as alpha * M * sum_i F_i P_i)."""

    @staticmethod
    def forward(ctx, x, W_r, b_r, q, k, v, M, grid=None, window=None, per_frame=False, balance_alpha=0.0):
        r = layer_train(x.contiguous(), W_r.contiguous(), b_r, q.contiguous(), k.contiguous(), v.contiguous(), M,
                        grid, window, per_frame=per_frame)
        ctx.save_for_backward(x, W_r, q, k, v)
        ctx.b_r = b_r
        ctx.saved = {n: r[n] for n in ("o_moga", "o_stga", "o_frame", "lse_moga", "lse_stga", "lse_frame",
                                       "group_id", "gate", "perm", "offsets", "per_frame")}
        ctx.args = (M, grid, window, balance_alpha)
        return r["out"]

    @staticmethod
    def backward(ctx, dout):
        x, W_r, q, k, v = ctx.saved_tensors
        M, grid, window, alpha = ctx.args
        g = layer_backward(dout.contiguous().to(torch.bfloat16), ctx.saved, x, W_r, ctx.b_r, q, k, v, M, grid,
                           window, balance_alpha=alpha)
        db = g["db_r"] if ctx.b_r is not None else None
        return g["dx"], g["dW_r"].to(W_r.dtype), db, g["dq"], g["dk"], g["dv"], None, None, None, None, None


def _host_tensor(t: torch.Tensor, name: str, dtype, shape):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


class Pipeline:
    """Host-to-host pipeline of one visual block (moga_pipe_* in moga.h).

    ``submit`` enqueues one step on host tensors (page-locked ones make the
    copies asynchronous) and returns at once; consecutive steps overlap their
    copies with their neighbours' compute.  ``sync`` waits for every submitted
    step; the host tensors handed to ``submit`` are kept alive until then.
    """

    def __init__(self, N, d, H, d_h, M, grid=None, window=None, x_dtype=torch.bfloat16, device="cuda",
                 per_frame: bool = False):
        lib = get_lib()
        self.N, self.d, self.H, self.d_h, self.M = N, d, H, d_h, M
        self.x_dtype = x_dtype
        grid = tuple(grid) if grid is not None else (0, 0, 0)
        self.window = tuple(window) if window is not None else None
        self.branches = (1 if self.window else 0) | (2 if per_frame else 0)
        x_dt = {torch.float32: MOGA_F32, torch.bfloat16: MOGA_BF16}[x_dtype]
        handle = ctypes.c_void_p()
        with torch.cuda.device(torch.device(device)):
            st = lib.moga_pipe_create(N, d, H, d_h, M, x_dt, *grid, _int3(self.window) if self.window else None,
                                      self.branches, ctypes.byref(handle))
        _check(st, "moga_pipe_create")
        self._h = handle
        self._keep = []

    def submit(self, x, W_r, b_r, q, k, v, out, group_id=None, gate=None):
        N, d, H, d_h, M = self.N, self.d, self.H, self.d_h, self.M
        _host_tensor(x, "x", self.x_dtype, (N, d))
        _host_tensor(W_r, "W_r", self.x_dtype, (M, d))
        if b_r is not None:
            _host_tensor(b_r, "b_r", torch.float32, (M,))
        for n, t in (("q", q), ("k", k), ("v", v), ("out", out)):
            _host_tensor(t, n, torch.bfloat16, (N, H, d_h))
        if group_id is not None:
            _host_tensor(group_id, "group_id", torch.int32, (N,))
        if gate is not None:
            _host_tensor(gate, "gate", torch.float32, (N,))
        st = get_lib().moga_pipe_submit(self._h, _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(out), _ptr(group_id), _ptr(gate))
        self._keep.append((x, W_r, b_r, q, k, v, out, group_id, gate))
        _check(st, "moga_pipe_submit")

    def sync(self):
        st = get_lib().moga_pipe_sync(self._h)
        self._keep.clear()
        _check(st, "moga_pipe_sync")

    def close(self):
        if self._h:
            get_lib().moga_pipe_destroy(self._h)
            self._h = None
            self._keep.clear()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
