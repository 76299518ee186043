"""moe_permute_noalloc: the permutation for callers that cannot allocate.

Some callers cannot give the library device memory (a framework that owns all
of HBM through its own pool, code in a host callback where cudaMalloc would
stall or is not allowed). moe_permute_noalloc keeps its scratch in one array
compiled into the library instead of a caller workspace. This checks it
through the C ABI against moe_permute on the same inputs, on two calls in a
row (the second call reuses the array the first one left behind), and that a
size beyond the array is refused. This file sorts last so that a failure here
comes after every other test has run; it passes alone in a fresh process too.
"""
import pytest
import torch

from mixture_experts_layer_aux_b200.synthetic import random_gates, random_routing, randn_bf16

pytestmark = pytest.mark.gpu


def _run(moe, fn, cfg, x, idx, g, mx=False):
    T, k, E, H = cfg.T, cfg.k, cfg.E, cfg.H
    rows = T * k
    out = dict(counts=torch.empty(E, dtype=torch.int32, device="cuda"),
               offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
               row_of=torch.empty(T, k, dtype=torch.int32, device="cuda"),
               src_of=torch.empty(rows, dtype=torch.int32, device="cuda"),
               row_gate=torch.empty(rows, dtype=torch.float32, device="cuda"),
               xp=torch.empty(rows, H, dtype=torch.uint8 if mx else torch.bfloat16, device="cuda"),
               xp_sf=torch.empty(rows, H // 32, dtype=torch.uint8, device="cuda") if mx else None)
    args = (cfg, x, idx, g, out["counts"], out["offsets"], out["row_of"], out["src_of"], out["row_gate"], out["xp"],
            out["xp_sf"])
    if fn == "ws":
        ws = moe.workspace(moe.moe_permute_workspace_size(cfg))
        moe.moe_permute(*args, ws)
    else:
        moe.moe_permute_noalloc(*args)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("mx", [False, True])
def test_noalloc_permute_matches_workspace_permute_on_two_calls(moe, mx):
    cases = [(8192, 512, 128, 8, 4, 0.0), (1000, 256, 64, 8, 10, 0.6)]  # a big call, then a smaller one
    for i, (T, H, E, k, zero, hot) in enumerate(cases):
        cfg = moe.make_config(T=T, H=H, E=E, k=k, F=128, expert_dtype=1 if mx else 0)
        x = randn_bf16((T, H), 1.0, seed=10 + i, device="cuda")
        idx = random_routing(T, E, k, seed=20 + i, zero_experts=zero, hot=hot).cuda()
        g = random_gates(T, k, seed=30 + i).cuda()
        ref = _run(moe, "ws", cfg, x, idx, g, mx)
        got = _run(moe, "noalloc", cfg, x, idx, g, mx)
        for name in ref:
            if ref[name] is not None:
                assert torch.equal(got[name], ref[name]), (i, name)
    assert moe.moe_get_device_status() == 0


def test_noalloc_permute_refuses_sizes_beyond_its_array(moe):
    cap = moe.moe_permute_noalloc_scratch_capacity()
    assert cap == 8 << 20
    T, E, k = 1 << 20, 512, 8          # ranks alone need 32 MiB
    cfg = moe.make_config(T=T, H=256, E=E, k=k, F=128)
    assert moe.moe_permute_workspace_size(cfg) > cap
    # every pointer is NULL: the size check refuses the call first (status 2, unsupported); should that check
    # ever stop refusing, the NULL inputs are refused on the host (status 1) and no kernel is launched
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_permute_noalloc(cfg, None, None, None, None, None, None, None, None, None, None)
    assert ei.value.status == 2
