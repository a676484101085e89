"""Host pipeline (moga_pipe_* in the C ABI) on the GPU.

The pipeline runs the same visual block as moga_layer_ex on host-resident
inputs, overlapping the copies of consecutive steps with their neighbours'
compute.  Every step must return exactly what the device-resident call
returns on the same inputs (same kernels, same order), and consecutive steps
on different inputs must not disturb one another (two device slots are
reused in turn).
"""
import pytest
import torch

import learned_token_group_b200 as moga
from workloads import custom, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    (custom(2 * 30 * 52, H=2, d_h=128, d=256, M=6, x_kind="clustered", grid=(2, 30, 52), window=(3, 8, 8),
            name="pipe_stga"), False),
    (custom(384, H=2, d_h=64, d=128, M=4, x_kind="clustered", grid=(3, 8, 16), window=(3, 8, 8),
            name="pipe_three"), True),
    (custom(1000, H=1, d_h=128, d=64, M=5, x_dtype="f32", name="pipe_moga_only"), False),
]


@pytest.mark.parametrize("wl,per_frame", CASES, ids=[c[0].name for c in CASES])
def test_pipeline_matches_device_calls(wl, per_frame):
    xdt = torch.float32 if wl.x_dtype == "f32" else torch.bfloat16
    pipe = moga.Pipeline(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window, xdt, "cuda", per_frame=per_frame)
    steps = []
    for seed in (11, 12, 13, 14, 15):          # more steps than slots: both slots are reused
        inp = make_inputs(wl, seed=seed, device="cpu")
        host = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
        out = torch.empty((wl.N, wl.H, wl.d_h), dtype=torch.bfloat16).pin_memory()
        gid = torch.empty(wl.N, dtype=torch.int32).pin_memory()
        gate = torch.empty(wl.N, dtype=torch.float32).pin_memory()
        pipe.submit(host["x"], host["W_r"], host["b_r"], host["q"], host["k"], host["v"], out, gid, gate)
        steps.append((inp, out, gid, gate))
    pipe.sync()
    for inp, out, gid, gate in steps:
        dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
        ref = moga.moga_layer(dev["x"], dev["W_r"], dev["b_r"], dev["q"], dev["k"], dev["v"], wl.M, wl.grid,
                              wl.window, per_frame=per_frame)
        moga.sync_status(ref["ws"])
        assert torch.equal(out, ref["out"].cpu())
        assert torch.equal(gid, ref["group_id"].cpu())
        assert torch.equal(gate, ref["gate"].cpu())
    pipe.close()


def test_pipeline_outputs_optional_and_reusable():
    wl = CASES[0][0]
    pipe = moga.Pipeline(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window, torch.bfloat16, "cuda")
    inp = make_inputs(wl, seed=3, device="cpu")
    host = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    outs = [torch.empty((wl.N, wl.H, wl.d_h), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for rnd in range(2):                        # sync between rounds, then reuse the same pipeline
        for o in outs:
            pipe.submit(host["x"], host["W_r"], host["b_r"], host["q"], host["k"], host["v"], o)
        pipe.sync()
        assert torch.equal(outs[0], outs[1])
    with pytest.raises(ValueError):
        pipe.submit(host["x"].cuda(), host["W_r"], host["b_r"], host["q"], host["k"], host["v"], outs[0])
    pipe.close()
