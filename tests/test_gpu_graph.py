"""CUDA-graph capture of the whole-layer entry points.

Every call of the C ABI launches on the caller's stream, reads its problem
sizes from device memory (expert offsets) and never synchronises or
allocates, so a captured layer step replays without the host. These tests
capture moe_layer_fwd + moe_layer_bwd (BF16, with a ragged expert mix and
a zero-token expert) and moe_layer_fwd (MXFP8 and NVFP4, with a shared
expert) in a CUDA graph, replay it, and require every output to equal the eager run bit
for bit (the kernels are deterministic: fixed-order reductions, no atomics
on floating point).
"""
import pytest
import torch

from helpers import empty
from mixture_experts_layer_aux_b200.synthetic import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _same(a, b):
    if a is None:
        return b is None
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a, b)


def _bf16_layer(moe, wl, d):
    """Buffers and a closure running fwd (saving for bwd) then bwd through the C ABI."""
    cfg = moe.make_config(wl, save_for_bwd=1)
    T, H, E, k, F = wl.T, wl.H, wl.E, wl.k, wl.F
    o = dict(y=empty((T, H), torch.bfloat16), aux=empty((1,), torch.float32), idx=empty((T, k), torch.int32),
             gates=empty((T, k), torch.float32), counts=empty((E,), torch.int32),
             offsets=empty((E + 1,), torch.int32), dX=empty((T, H), torch.bfloat16),
             dW_r=empty((E, H), torch.bfloat16), dW_g=empty((E, F, H), torch.bfloat16),
             dW_u=empty((E, F, H), torch.bfloat16), dW_d=empty((E, H, F), torch.bfloat16),
             dlogits=empty((T, E), torch.float32))
    ws = moe.workspace(moe.moe_layer_workspace_size(cfg))
    saved = moe.workspace(moe.moe_layer_saved_size(cfg))
    wsb = moe.workspace(moe.moe_layer_bwd_workspace_size(cfg))

    def step():
        moe.moe_layer_fwd(cfg, d["x"], d["W_r"], d.get("logit_bias"), d["W_g"], d["W_u"], d["W_d"], None, None,
                          None, None, None, None, None, None, None, o["y"], o["aux"], o["idx"], o["gates"],
                          o["counts"], o["offsets"], saved, ws)
        moe.moe_layer_bwd(cfg, d["dY"], 0.01, d["x"], d["W_r"], d["W_g"], d["W_u"], d["W_d"], saved, o["dX"],
                          o["dW_r"], o["dW_g"], o["dW_u"], o["dW_d"], o["dlogits"], wsb)
    return o, step


def _capture_and_compare(moe, make):
    o1, step1 = make()
    step1()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    o2, step2 = make()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step2()  # warm-up on a side stream before capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for v in o2.values():
        if v is not None:
            v.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step2()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    for name in o1:
        assert _same(o1[name], o2[name]), f"{name}: graph replay differs from the eager run"


def test_layer_fwd_bwd_graph_replay_equals_eager(moe):
    wl = Workload("graph", T=777, H=512, E=16, k=4, F=512, bwd=True)
    d = make_inputs(wl, device="cuda", seed=11)
    bias = torch.zeros(wl.E, device="cuda")
    bias[-1] = -30.0  # one expert without tokens
    d["logit_bias"] = bias
    _capture_and_compare(moe, lambda: _bf16_layer(moe, wl, d))


def test_layer_fwd_mxfp8_graph_replay_equals_eager(moe):
    wl = Workload("graph_mx", T=640, H=512, E=8, k=2, F=256, S=1, score="sigmoid", route_scale=2.5, aux=False,
                  dtype="mxfp8")
    d = make_inputs(wl, device="cuda", seed=12)
    q = {}
    for name in ["W_g", "W_u", "W_d", "W_gs", "W_us", "W_ds"]:
        w = d[name]
        codes = torch.empty(w.shape, dtype=torch.uint8, device="cuda")
        sf = torch.empty(w.shape[:-1] + (w.shape[-1] // 32,), dtype=torch.uint8, device="cuda")
        moe.moe_quantize_mxfp8(w, codes, sf)
        q[name] = (codes, sf)
    torch.cuda.synchronize()

    def make():
        cfg = moe.make_config(wl)
        o = dict(y=empty((wl.T, wl.H), torch.bfloat16), idx=empty((wl.T, wl.k), torch.int32),
                 gates=empty((wl.T, wl.k), torch.float32))
        ws = moe.workspace(moe.moe_layer_workspace_size(cfg))

        def step():
            moe.moe_layer_fwd(cfg, d["x"], d["W_r"], None, q["W_g"][0], q["W_u"][0], q["W_d"][0], q["W_g"][1],
                              q["W_u"][1], q["W_d"][1], q["W_gs"][0], q["W_us"][0], q["W_ds"][0], q["W_gs"][1],
                              q["W_us"][1], q["W_ds"][1], o["y"], None, o["idx"], o["gates"], None, None, None, ws)
        return o, step
    _capture_and_compare(moe, make)


def test_layer_fwd_nvfp4_graph_replay_equals_eager(moe):
    wl = Workload("graph_nv", T=640, H=512, E=8, k=2, F=256, S=1, score="sigmoid", route_scale=2.5, aux=False,
                  dtype="nvfp4")
    d = make_inputs(wl, device="cuda", seed=13)
    q = {}
    for name in ["W_g", "W_u", "W_d", "W_gs", "W_us", "W_ds"]:
        w = d[name]
        R, C = w.shape[-2], w.shape[-1]
        packed = torch.empty(w.shape[:-1] + (C // 2,), dtype=torch.uint8, device="cuda")
        sf = torch.empty(moe.moe_nvfp4_sf_bytes(w.numel() // (R * C), R, C), dtype=torch.uint8, device="cuda")
        moe.moe_quantize_nvfp4(w, packed, sf)
        q[name] = (packed, sf)
    torch.cuda.synchronize()

    def make():
        cfg = moe.make_config(wl)
        o = dict(y=empty((wl.T, wl.H), torch.bfloat16), idx=empty((wl.T, wl.k), torch.int32),
                 gates=empty((wl.T, wl.k), torch.float32))
        ws = moe.workspace(moe.moe_layer_workspace_size(cfg))

        def step():
            moe.moe_layer_fwd(cfg, d["x"], d["W_r"], None, q["W_g"][0], q["W_u"][0], q["W_d"][0], q["W_g"][1],
                              q["W_u"][1], q["W_d"][1], q["W_gs"][0], q["W_us"][0], q["W_ds"][0], q["W_gs"][1],
                              q["W_us"][1], q["W_ds"][1], o["y"], None, o["idx"], o["gates"], None, None, None, ws)
        return o, step
    _capture_and_compare(moe, make)
