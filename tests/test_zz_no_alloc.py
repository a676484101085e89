"""moga_route_noalloc: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc themselves (their framework's allocator
owns the GPU, or they replay a fixed launch sequence).  moga_route_noalloc
gives them the router and counting sort with the library's own fixed device
scratch instead of a caller workspace.  This test calls it through the C ABI
and checks it on consecutive calls of different sizes, so that contents left
behind by one call cannot leak into the next: against the oracle (group ids
with the near-tie rule, gate, and perm/offsets bit-exact against the oracle's
counting sort), against moga_route, and through moga_route_noalloc_status,
which must report no device-side condition.  It lives in
its own file, collected last, and passes alone or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import learned_token_group_b200 as moga
from parity import GATE_TOL_BF16, GATE_TOL_F32, check_route, np_cpu
from workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu

WORKSPACE_ERR = 3


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(inp, M):
    lib = moga.get_lib()
    x = inp["x"]
    N, d = x.shape
    dev = x.device
    out = {"group_id": torch.empty(N, dtype=torch.int32, device=dev),
           "gate": torch.empty(N, dtype=torch.float32, device=dev),
           "perm": torch.empty(N, dtype=torch.int32, device=dev),
           "offsets": torch.empty(M + 1, dtype=torch.int32, device=dev),
           "max_seqlen": torch.empty(1, dtype=torch.int32, device=dev)}
    dt = 0 if x.dtype == torch.float32 else 1
    st = lib.moga_route_noalloc(_p(x), _p(inp["W_r"]), _p(inp["b_r"]), dt, N, d, M, _p(out["group_id"]),
                                _p(out["gate"]), _p(out["perm"]), _p(out["offsets"]), _p(out["max_seqlen"]),
                                ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert st == 0, moga.STATUS.get(st, st)
    return out


CASES = [
    (WORKLOADS["wan_32k"], 5),
    (custom(3000, d=512, M=64, x_kind="skew"), 6),
    (WORKLOADS["tiny"], 7),                     # fp32 input: SIMT router
    (WORKLOADS["wan_32k"], 5),                  # the first case again, after smaller ones
]


def test_noalloc_matches_route_on_consecutive_calls():
    for wl, seed in CASES:
        inp = make_inputs(wl, seed=seed, device="cuda", with_qkv=False)
        ref = moga.route(inp["x"], inp["W_r"], inp["b_r"], wl.M)
        got = _noalloc(inp, wl.M)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        assert moga.get_lib().moga_route_noalloc_status(stream) == 0
        tol = GATE_TOL_F32 if wl.x_dtype == "f32" else GATE_TOL_BF16
        check_route(got, inp["x"], inp["W_r"], inp["b_r"], wl.M, tol)
        for key in ("group_id", "perm", "offsets", "max_seqlen"):
            assert np.array_equal(np_cpu(got[key]), np_cpu(ref[key])), f"{wl.name}: {key} differs"
        assert np.abs(np_cpu(got["gate"]) - np_cpu(ref["gate"])).max() <= tol


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = moga.get_lib()
    fake = ctypes.c_void_p(1 << 20)           # never dereferenced: the size check comes first
    for N, M in [(128 * 262145, 1), (600000, 64)]:
        st = lib.moga_route_noalloc(fake, fake, None, 1, N, 64, M, fake, fake, fake, fake, fake, None)
        assert st == WORKSPACE_ERR
