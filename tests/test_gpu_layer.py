"""Whole-layer parity of the CUDA path (moe_layer_fwd / moe_layer_bwd through
the C ABI) with the oracle, on the workload shapes and on small cases that the
oracle finishes in seconds.

Routing: the GPU's fp32 logits and the oracle's differ by summation order, so
top-k indices may legitimately differ on a near-tie. The tests require the
logits to agree within 1e-4 rms, every index disagreement to be a near-tie
(logit gap within that bound), and compare floating outputs only on tokens
whose routing agrees (all of them, in practice).
"""
import pytest
import torch

from helpers import TOL_BF16, check_bf16, empty, err_rms
from mixture_experts_layer_aux_b200.synthetic import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def run_fwd(moe, wl, d, save=False):
    cfg = moe.make_config(wl, save_for_bwd=int(save))
    T, E, k, H = wl.T, wl.E, wl.k, wl.H
    out = dict(y=empty((T, H), torch.bfloat16), idx=empty((T, k), torch.int32), gates=empty((T, k), torch.float32),
               counts=empty((E,), torch.int32), offsets=empty((E + 1,), torch.int32))
    out["aux"] = empty((1,), torch.float32) if cfg.compute_aux else None
    ws = moe.workspace(moe.moe_layer_workspace_size(cfg))
    saved = moe.workspace(moe.moe_layer_saved_size(cfg)) if save else None
    moe.moe_layer_fwd(cfg, d["x"], d["W_r"], d.get("logit_bias"), d["W_g"], d["W_u"], d["W_d"], None, None, None,
                      d.get("W_gs"), d.get("W_us"), d.get("W_ds"), None, None, None, out["y"], out["aux"],
                      out["idx"], out["gates"], out["counts"], out["offsets"], saved, ws, expert_bias=d.get("expert_bias"))
    torch.cuda.synchronize()
    out["saved"] = saved
    out["cfg"] = cfg
    return out


def routing_agreement(oracle, wl, h, gpu_idx):
    """Oracle logits + routing; returns (route dict, tokens whose indices agree)."""
    logits = oracle.router_logits(h["x"], h["W_r"], h.get("logit_bias"))
    r = oracle.route(logits, wl.k, wl.score, wl.norm_topk, wl.route_scale, with_aux=wl.aux and wl.score == "softmax",
                     capacity_factor=wl.capacity_factor, expert_bias=h.get("expert_bias"), n_group=wl.n_group,
                     topk_group=wl.topk_group)
    same = (gpu_idx.cpu() == r["idx"]).all(1)
    bound = 1e-4 * float(logits.pow(2).mean().sqrt())
    # selection values: the logits, or (DeepSeek-V3 variant) score + bias, whose slope is at most 1/4 of the logits'
    sel = r["sel"] if r.get("sel") is not None else logits
    for t in (~same).nonzero().flatten().tolist():
        gi, ri = gpu_idx[t].cpu(), r["idx"][t]
        # experts in disagreeing slots (a swap of slot order leaves the sets equal)
        a = sorted(set(gi[gi != ri].tolist()) | set(ri[gi != ri].tolist()))
        gap = (sel[t, a].max() - sel[t, a].min()).item()
        if wl.n_group > 1 and gap > 2 * bound:
            # a near-tie between groups moves whole groups: check the group scores around the cut
            G = wl.E // wl.n_group
            gs = torch.topk(sel[t].view(wl.n_group, G), min(2, G), dim=-1).values.sum(-1).sort(descending=True).values
            gap = (gs[wl.topk_group - 1] - gs[wl.topk_group]).item()
        assert gap <= 2 * bound, f"token {t}: routing differs by more than a near-tie (gap {gap})"
    assert int((~same).sum()) <= max(2, wl.T // 1000)
    return r, same


def host(d):
    return {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in d.items()}


def check_fwd(moe, oracle, wl, n_sample=None, seed=0):
    d = make_inputs(wl, device="cuda", seed=seed)
    out = run_fwd(moe, wl, d)
    h = host(d)
    r, same = routing_agreement(oracle, wl, h, out["idx"])
    if bool(same.all()):
        assert torch.equal(out["counts"].cpu(), r["counts"])
        assert torch.equal(out["offsets"].cpu(), r["offsets"])
    gen = torch.Generator().manual_seed(seed + 99)
    if n_sample is None or n_sample >= wl.T:
        toks = torch.arange(wl.T, dtype=torch.int32)
    else:
        toks = torch.randperm(wl.T, generator=gen)[:n_sample].sort().values.to(torch.int32)
    toks = toks[same[toks.long()]]
    shared = (h["W_gs"], h["W_us"], h["W_ds"]) if wl.S else None
    y_ref = oracle.moe_fwd_tokens(h["x"], h["W_g"], h["W_u"], h["W_d"], r["idx_kept"], r["gates"], toks,
                                  shared=shared, recipe="bf16")
    e = check_bf16(out["y"].cpu()[toks.long()], y_ref, terms=wl.k + wl.S)[0]
    ge = (out["gates"].cpu().double()[toks.long()] - r["gates"][toks.long()]).abs().max().item()
    assert ge <= 1e-5, ge
    if out["aux"] is not None:
        assert abs(out["aux"].item() - r["aux"]) <= 1e-4 * abs(r["aux"])
    assert moe.moe_get_device_status() == 0
    return e


def test_layer_fwd_tiny_full_oracle(moe, oracle):
    check_fwd(moe, oracle, WORKLOADS["tiny"])


@pytest.mark.parametrize("wl", [Workload("ragged", T=333, H=512, E=16, k=4, F=384),
                                Workload("shared", T=200, H=256, E=8, k=2, F=256, S=1, score="sigmoid",
                                         route_scale=2.5, aux=False),
                                Workload("k1", T=77, H=256, E=4, k=1, F=128)])
def test_layer_fwd_small_cases_full_oracle(moe, oracle, wl):
    check_fwd(moe, oracle, wl)


@pytest.mark.parametrize("cf", [0.6, 1.0])
def test_layer_fwd_capacity_factor_full_oracle(moe, oracle, cf):
    """Each expert keeps its first ceil(cf T k / E) pairs in token order; dropped pairs add nothing."""
    wl = Workload("capacity", T=600, H=512, E=8, k=2, F=512, skew=True, capacity_factor=cf)
    check_fwd(moe, oracle, wl)


def test_permute_capacity_maps_bit_exact(moe, oracle):
    """Capacity through moe_permute alone: kept counts, offsets and maps equal the oracle's, bit for bit."""
    from mixture_experts_layer_aux_b200.synthetic import random_routing
    T, E, k, H = 1000, 16, 4, 256
    wl = Workload("cap-perm", T=T, H=H, E=E, k=k, F=128, capacity_factor=0.7)
    cfg = moe.make_config(wl)
    idx = random_routing(T, E, k, seed=4, hot=0.5)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(2)).bfloat16()
    xd, idd = x.cuda(), idx.cuda()
    counts, offsets = empty((E,), torch.int32), empty((E + 1,), torch.int32)
    row_of, src_of = empty((T, k), torch.int32), empty((T * k,), torch.int32)
    xp = torch.zeros(T * k, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(cfg, xd, idd, None, counts, offsets, row_of, src_of, None, xp, None,
                    moe.workspace(moe.moe_permute_workspace_size(cfg)))
    torch.cuda.synchronize()
    keep, C = oracle.capacity_keep(idx, E, 0.7)
    assert int((keep == 0).sum()) > 0
    kc, off, ro, so = oracle.maps(idx, E, keep)
    assert torch.equal(counts.cpu(), kc) and torch.equal(offsets.cpu(), off) and torch.equal(row_of.cpu(), ro)
    n = int(off[-1])
    assert torch.equal(src_of.cpu()[:n], so[:n])
    assert torch.equal(xp.cpu()[:n].view(torch.int16), x[so[:n].long()].view(torch.int16))
    assert moe.moe_get_device_status() == 0


@pytest.mark.parametrize("wl", [
    Workload("dsv3-router", T=600, H=512, E=64, k=6, F=256, score="sigmoid", route_scale=2.5, aux=False,
             n_group=8, topk_group=4, sel_bias=True),
    Workload("bias-only", T=300, H=256, E=16, k=2, F=256, score="sigmoid", route_scale=2.5, aux=False,
             sel_bias=True)])
def test_layer_fwd_deepseek_router_variant_full_oracle(moe, oracle, wl):
    """Selection on sigmoid score + per-expert bias within the best expert groups; gates from the scores."""
    check_fwd(moe, oracle, wl)


def test_layer_fwd_is_deterministic(moe):
    wl = Workload("det", T=1000, H=512, E=32, k=4, F=256)
    d = make_inputs(wl, device="cuda", seed=5)
    a = run_fwd(moe, wl, d)
    b = run_fwd(moe, wl, d)
    assert torch.equal(a["y"].view(torch.int16), b["y"].view(torch.int16))
    assert torch.equal(a["aux"], b["aux"])


# ------------------------------------------------------------------ backward


def run_bwd(moe, wl, d, fwd, d_aux):
    cfg = fwd["cfg"]
    T, H, E, F = wl.T, wl.H, wl.E, wl.F
    o = dict(dX=empty((T, H), torch.bfloat16), dW_r=empty((E, H), torch.bfloat16),
             dW_g=empty((E, F, H), torch.bfloat16), dW_u=empty((E, F, H), torch.bfloat16),
             dW_d=empty((E, H, F), torch.bfloat16), dlogits=empty((T, E), torch.float32))
    ws = moe.workspace(moe.moe_layer_bwd_workspace_size(cfg))
    moe.moe_layer_bwd(cfg, d["dY"], d_aux, d["x"], d["W_r"], d["W_g"], d["W_u"], d["W_d"], fwd["saved"], o["dX"],
                      o["dW_r"], o["dW_g"], o["dW_u"], o["dW_d"], o["dlogits"], ws)
    torch.cuda.synchronize()
    return o


def check_bwd(moe, oracle, wl, seed=0, d_aux=0.01, n_tok=None, experts=None):
    d = make_inputs(wl, device="cuda", seed=seed, with_dy=True)
    fwd = run_fwd(moe, wl, d, save=True)
    g = run_bwd(moe, wl, d, fwd, d_aux)
    h = host(d)
    r, same = routing_agreement(oracle, wl, h, fwd["idx"])
    if n_tok is None:
        assert bool(same.all()), "full backward parity needs identical routing"
        toks = torch.arange(wl.T, dtype=torch.int32)
    else:
        toks = torch.randperm(wl.T, generator=torch.Generator().manual_seed(seed))[:n_tok].sort().values
        toks = toks[same[toks]].to(torch.int32)
        # experts touched by a near-tie flip get a different token set on the two sides
        flipped = set(fwd["idx"].cpu()[~same].flatten().tolist()) | set(r["idx"][~same].flatten().tolist())
        experts = [e for e in experts if e not in flipped]
    aux_on = wl.aux and wl.score == "softmax"
    dx, dl, _ = oracle.moe_bwd_tokens(h["x"], h["W_r"], h["W_g"], h["W_u"], h["W_d"], h["dY"], r, toks,
                                      score=wl.score, norm=wl.norm_topk, route_scale=wl.route_scale, aux_on=aux_on,
                                      d_aux=d_aux, recipe="bf16")
    res = {}
    res["dX"] = check_bf16(g["dX"].cpu()[toks.long()], dx, terms=wl.k + 1)[0]
    res["dlogits"] = err_rms(g["dlogits"].cpu()[toks.long()], dl)
    if experts is None:
        experts = list(range(wl.E))
    dWg, dWu, dWd = oracle.moe_bwd_expert_dw(h["x"], h["W_g"], h["W_u"], h["W_d"], h["dY"], r["idx_kept"],
                                             r["gates"], experts, recipe="bf16")
    ex = torch.tensor(experts).long()
    for name, ref in (("dW_g", dWg), ("dW_u", dWu), ("dW_d", dWd)):
        # the bar applies over the compared tensor (every compared expert's slice)
        res[name] = check_bf16(g[name].cpu()[ex], ref, terms=2)[0]
        for q, e in enumerate(experts):
            if int(r["kept_counts"][e]) == 0:
                assert (g[name][e] == 0).all(), (name, e)   # exact zeros for an expert with no token
            else:
                # and no expert, however small, may be grossly off relative to its own size
                assert err_rms(g[name][e].cpu(), ref[q].float().bfloat16().double()) <= 0.1, (name, e)
    if n_tok is None:
        res["dW_r"] = check_bf16(g["dW_r"].cpu(), oracle.router_dwr(dl, h["x"], round_dl=True))[0]
    else:
        # property at any size: dW_r = bf16(dlogits)^T x (with the GPU's own dlogits)
        dl16 = g["dlogits"].double().cpu().float().bfloat16().double()
        res["dW_r"] = check_bf16(g["dW_r"].cpu(), dl16.T @ h["x"].double())[0]
    # bf16 outputs were asserted by check_bf16 above; dlogits is fp32
    assert res["dlogits"] <= TOL_BF16, res
    print(wl.name, {k: round(v, 4) for k, v in res.items()})
    assert moe.moe_get_device_status() == 0
    return res


def test_layer_bwd_small_full_oracle(moe, oracle):
    wl = Workload("bwd-small", T=256, H=256, E=8, k=2, F=512, skew=True, bwd=True)
    check_bwd(moe, oracle, wl)


def test_layer_bwd_ragged_full_oracle(moe, oracle):
    wl = Workload("bwd-ragged", T=700, H=512, E=16, k=4, F=256, skew=True, bwd=True)
    check_bwd(moe, oracle, wl, seed=3, d_aux=0.5)


def test_layer_bwd_capacity_factor_full_oracle(moe, oracle):
    wl = Workload("bwd-capacity", T=512, H=256, E=8, k=2, F=512, skew=True, bwd=True, capacity_factor=0.8)
    check_bwd(moe, oracle, wl, seed=2, d_aux=0.3)


def test_layer_bwd_deepseek_router_variant_full_oracle(moe, oracle):
    """Backward through selection on sigmoid score + per-expert bias within the best expert groups."""
    wl = Workload("bwd-dsv3-router", T=512, H=256, E=32, k=4, F=256, score="sigmoid", route_scale=2.5, aux=False,
                  bwd=True, n_group=4, topk_group=2, sel_bias=True)
    check_bwd(moe, oracle, wl, seed=5, d_aux=0.0)


# ------------------------------------------------------------------ MXFP8 layer


def run_fwd_mx(moe, wl, d):
    cfg = moe.make_config(wl)
    T, E, k, H = wl.T, wl.E, wl.k, wl.H
    q = {}
    for name in ["W_g", "W_u", "W_d"] + (["W_gs", "W_us", "W_ds"] if wl.S else []):
        w = d[name]
        codes = torch.empty(w.shape, dtype=torch.uint8, device="cuda")
        sf = torch.empty(w.shape[:-1] + (w.shape[-1] // 32,), dtype=torch.uint8, device="cuda")
        moe.moe_quantize_mxfp8(w, codes, sf)
        q[name] = (codes, sf)
    y = empty((T, H), torch.bfloat16)
    idx = empty((T, k), torch.int32)
    gates = empty((T, k), torch.float32)
    ws = moe.workspace(moe.moe_layer_workspace_size(cfg))
    sh = [None] * 6
    if wl.S:
        sh = [q["W_gs"][0], q["W_us"][0], q["W_ds"][0], q["W_gs"][1], q["W_us"][1], q["W_ds"][1]]
    moe.moe_layer_fwd(cfg, d["x"], d["W_r"], d.get("logit_bias"), q["W_g"][0], q["W_u"][0], q["W_d"][0], q["W_g"][1],
                      q["W_u"][1], q["W_d"][1], *sh, y, None, idx, gates, None, None, None, ws,
                      expert_bias=d.get("expert_bias"))
    torch.cuda.synchronize()
    return y, idx, gates


def check_fwd_mx(moe, oracle, wl, n_sample=None, seed=0):
    d = make_inputs(wl, device="cuda", seed=seed)
    y, idx, gates = run_fwd_mx(moe, wl, d)
    logits = oracle.router_logits(d["x"].cpu(), d["W_r"].cpu(), None)
    r, same = routing_agreement(oracle, wl, {"x": d["x"].cpu(), "W_r": d["W_r"].cpu(),
                                             "expert_bias": None if d.get("expert_bias") is None
                                             else d["expert_bias"].cpu()}, idx)
    if n_sample is None:
        toks = torch.arange(wl.T, dtype=torch.int32)
    else:
        toks = torch.randperm(wl.T, generator=torch.Generator().manual_seed(seed + 7))[:n_sample].sort().values
        toks = toks.to(torch.int32)
    toks = toks[same[toks.long()]]
    # the oracle quantises the bf16 weights itself, only the experts the sampled tokens use
    need = sorted(set(r["idx"][toks.long()].flatten().tolist()))
    mx = {}
    for name in ("W_g", "W_u", "W_d"):
        W = d[name]
        codes = torch.zeros(W.shape, dtype=torch.uint8)
        sf = torch.zeros(W.shape[:-1] + (W.shape[-1] // 32,), dtype=torch.uint8)
        for e in need:
            c_, s_ = oracle.mxfp8_quantize(W[e].cpu())
            codes[e], sf[e] = c_, s_
        mx[name] = (codes, sf)
    for name in ("W_gs", "W_us", "W_ds"):
        if wl.S:
            mx[name] = oracle.mxfp8_quantize(d[name].cpu())
    shared = (mx["W_gs"][0], mx["W_us"][0], mx["W_ds"][0], mx["W_gs"][1], mx["W_us"][1], mx["W_ds"][1]) if wl.S \
        else None
    y_ref = oracle.moe_fwd_tokens(d["x"].cpu(), mx["W_g"][0], mx["W_u"][0], mx["W_d"][0], r["idx_kept"], r["gates"],
                                  toks, recipe="mxfp8", sf_g=mx["W_g"][1], sf_u=mx["W_u"][1], sf_d=mx["W_d"][1],
                                  shared=shared)
    e = check_bf16(y.cpu()[toks.long()], y_ref, tol=6e-2, terms=wl.k + wl.S)
    assert moe.moe_get_device_status() == 0
    return e


def test_layer_fwd_mxfp8_small_full_oracle(moe, oracle):
    wl = Workload("mx-small", T=256, H=512, E=16, k=4, F=256, S=1, score="sigmoid", route_scale=2.5, dtype="mxfp8",
                  aux=False)
    check_fwd_mx(moe, oracle, wl)


def test_layer_fwd_mxfp8_deepseek_router_variant(moe, oracle):
    wl = Workload("mx-dsv3-router", T=256, H=512, E=32, k=4, F=256, S=1, score="sigmoid", route_scale=2.5,
                  aux=False, dtype="mxfp8", n_group=4, topk_group=2, sel_bias=True)
    check_fwd_mx(moe, oracle, wl)


def test_layer_fwd_mxfp8_deepseek_router_with_capacity(moe, oracle):
    # the DeepSeek-V3 router variant with a capacity factor that drops pairs (dropped pairs: no row, no output)
    wl = Workload("mx-dsv3-cap", T=320, H=512, E=32, k=4, F=256, S=1, score="sigmoid", route_scale=2.5,
                  aux=False, dtype="mxfp8", n_group=4, topk_group=2, sel_bias=True, capacity_factor=1.0)
    check_fwd_mx(moe, oracle, wl)

