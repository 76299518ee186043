"""NVFP4 path (E2M1 elements, E4M3 scales per 16, per-matrix encode scales) against the oracle.

The quantisers are bit-exact (codes, scale bytes and the fp32 encode scales).
The GEMMs and the layer compare within TOL_NVFP4 with the oracle's nvfp4
recipe, which quantises the same bf16 inputs at the same points; elements that
differ more are single E2M1 rounding decisions taken differently (check_nv).
"""
import pytest
import torch

from helpers import TOL_NVFP4, check_bf16, check_nv, e_of_rows, empty
from mixture_experts_layer_aux_b200.synthetic import (WORKLOADS, Workload, make_inputs, random_gates, random_routing,
                                                      randn_bf16)
from test_gpu_layer import routing_agreement

pytestmark = pytest.mark.gpu


def _status_clean(moe):
    assert moe.moe_get_device_status(clear=True) == 0


def _gpu_quant_w(moe, w):
    """moe_quantize_nvfp4 of a [batch, R, C] or [R, C] bf16 weight -> (packed, sf buffer)."""
    R, C = w.shape[-2], w.shape[-1]
    batch = w.numel() // (R * C)
    packed = torch.empty(w.shape[:-1] + (C // 2,), dtype=torch.uint8, device="cuda")
    sf = torch.empty(moe.moe_nvfp4_sf_bytes(batch, R, C), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_nvfp4(w.cuda().contiguous(), packed, sf)
    return packed, sf


def _split_sf(sf, batch, R, C):
    """moe_quantize_nvfp4's scale buffer -> (row-major scales [batch, R, C/16] uint8, G [batch] fp32).

    The buffer holds the scales tiled: byte ((r/128) * C/64 + c/4) * 512 + 16 (r%32) + 4 ((r%128)/32) + c%4
    for global row r and 16-block c."""
    n = batch * R * (C // 16)
    s = sf.cpu()
    r = torch.arange(batch * R).view(-1, 1)
    c = torch.arange(C // 16).view(1, -1)
    idx = ((r // 128) * (C // 64) + c // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + c % 4
    return s[:n][idx].view(batch, R, C // 16), s[n:].view(torch.float32)


def _decoded_scales(oracle, sf_bytes):
    e4 = torch.tensor([oracle.e4m3_decode(c) for c in range(256)], dtype=torch.float64)
    return e4[sf_bytes.long()].repeat_interleave(16, dim=-1)


# ------------------------------------------------------------------ quantisers


@pytest.mark.parametrize("batch,R,C", [(3, 128, 256), (2, 384, 7168), (1, 128, 2048)])
def test_quantize_nvfp4_weights_bit_exact(moe, oracle, batch, R, C):
    w = randn_bf16((batch, R, C), 0.02, seed=R + C, scale_rows=True)
    w[0, 0, :16] = 0  # an all-zero block
    if R > 3:
        w[0, 1, :16] = torch.tensor([1e-40] * 8 + [-3e-39] * 8).to(torch.bfloat16)  # bf16 subnormals
        w[0, 2, :16] = torch.tensor([6.0, -5.0, 3.5, 0.25] + [1.0] * 12).to(torch.bfloat16)
    if batch > 1:
        w[1] = 0  # an all-zero matrix: G = 1, every scale 0
    packed, sf = _gpu_quant_w(moe, w)
    torch.cuda.synchronize()
    q, s, G = oracle.nvfp4_quantize(w, per_matrix=True)
    s_gpu, G_gpu = _split_sf(sf, batch, R, C)
    assert torch.equal(G_gpu, G.view(-1))
    assert torch.equal(s_gpu, s.view(batch, R, C // 16))
    assert torch.equal(packed.cpu(), q)
    _status_clean(moe)


@pytest.mark.parametrize("R,K", [(64, 256), (1000, 7168), (3, 2048)])
def test_quantize_nvfp4_activations_bit_exact(moe, oracle, R, K):
    x = randn_bf16((R, K), 1.0, seed=R + 3, scale_rows=True)
    x[0, 16:32] = 0
    dst = empty((R, K // 2), torch.uint8)
    sf = empty((R, K // 16), torch.uint8)
    moe.moe_quantize_nvfp4_act(x.cuda(), dst, sf)
    torch.cuda.synchronize()
    q, s, _ = oracle.nvfp4_quantize(x)
    assert torch.equal(sf.cpu(), s)
    assert torch.equal(dst.cpu(), q)


@pytest.mark.parametrize("T,H,E,k", [(300, 256, 8, 2), (1024, 7168, 256, 8), (300, 4864, 16, 4)])
def test_permute_nvfp4_bit_exact(moe, oracle, T, H, E, k):
    idx = random_routing(T, E, k, seed=T + 2)
    x = randn_bf16((T, H), 1.0, seed=T + 6, scale_rows=True)
    x[0, :32] = 0
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=256, expert_dtype=moe.MOE_DT_NVFP4)
    rows = T * k
    offsets = empty((E + 1,), torch.int32)
    row_of, src_of = empty((T, k), torch.int32), empty((rows,), torch.int32)
    xp = empty((rows, H // 2), torch.uint8)
    xsf = empty((rows, H // 16), torch.uint8)
    ws = moe.workspace(moe.moe_permute_workspace_size(cfg))
    moe.moe_permute(cfg, x.cuda(), idx.cuda(), None, None, offsets, row_of, src_of, None, xp, xsf, ws)
    torch.cuda.synchronize()
    _, _, ro, so = oracle.maps(idx, E)
    assert torch.equal(src_of.cpu(), so)
    q, s, _ = oracle.nvfp4_quantize(x[so.long()].contiguous())
    assert torch.equal(xsf.cpu(), s)
    assert torch.equal(xp.cpu(), q)
    _status_clean(moe)


# ------------------------------------------------------------------ grouped GEMMs

NV_CASES = [
    # T, H, E, k, F, zero experts, hot fraction: ragged expert sizes, an empty expert, several tiles
    (300, 512, 4, 2, 512, 1, 0.0),
    (513, 1024, 16, 4, 256, 3, 0.3),
    (64, 7168, 8, 8, 2048, 0, 0.0),
]


@pytest.mark.parametrize("T,H,E,k,F,zero,hot", NV_CASES)
def test_grouped_gemm_nvfp4_matches_oracle(moe, oracle, T, H, E, k, F, zero, hot):
    idx = random_routing(T, E, k, seed=T + F + 3, zero_experts=zero, hot=hot)
    counts, offsets, _, _ = oracle.maps(idx, E)
    rows = T * k
    xp = randn_bf16((rows, H), 1.0, seed=rows + 3)
    g = random_gates(rows, 1, seed=rows + 4).flatten() * 2.5
    Wg = randn_bf16((E, F, H), 0.02, seed=21)
    Wu = randn_bf16((E, F, H), 0.02, seed=22)
    Wd = randn_bf16((E, H, F), 0.02, seed=23)
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=F, expert_dtype=moe.MOE_DT_NVFP4)
    xq = empty((rows, H // 2), torch.uint8)
    xs = empty((rows, H // 16), torch.uint8)
    moe.moe_quantize_nvfp4_act(xp.cuda(), xq, xs)
    (gq, gs), (uq, us), (dq, ds) = _gpu_quant_w(moe, Wg), _gpu_quant_w(moe, Wu), _gpu_quant_w(moe, Wd)
    ap = empty((rows, F // 2), torch.uint8)
    ap_sf = empty((rows, F // 16), torch.uint8)
    o = empty((rows, H), torch.bfloat16)
    ws = moe.workspace(256)
    off = offsets.cuda()
    moe.moe_grouped_gemm_fwd(cfg, 0, xq, xs, gq, gs, uq, us, off, g.cuda(), ap, ap_sf, None, ws)
    moe.moe_grouped_gemm_fwd(cfg, 1, ap, ap_sf, dq, ds, None, None, off, None, o, None, None, ws)
    torch.cuda.synchronize()
    # the oracle quantises the same bf16 weights itself (bit-identical codes, tested above)
    Q = {n: oracle.nvfp4_quantize(w, per_matrix=True) for n, w in (("g", Wg), ("u", Wu), ("d", Wd))}
    e_of = e_of_rows(offsets)
    ref = oracle.expert_rows(xp, e_of, g.double(), Q["g"][0], Q["u"][0], Q["d"][0], recipe="nvfp4",
                             sf_g=Q["g"][1:], sf_u=Q["u"][1:], sf_d=Q["d"][1:], want=("zg", "zu", "ap", "o"))
    R = int(offsets[-1])
    ap_dq = oracle.nvfp4_decode(ap.cpu(), ap_sf.cpu())[:R]
    s_got = _decoded_scales(oracle, ap_sf.cpu())[:R]
    # the oracle's own block scales of ap: its pre-quantisation values g silu(z_g) z_u through its quantiser
    pre = g.double()[:R, None] * torch.nn.functional.silu(ref["zg"]) * ref["zu"]
    ref_q, ref_sf, _ = oracle.nvfp4_quantize(pre.float())
    s_ref = _decoded_scales(oracle, ref_sf)
    same = (oracle.nvfp4_decode(ref_q, ref_sf) == ref["ap"]).double().mean().item()
    assert same > 0.999, same  # (fp64 silu here and in the oracle may differ in the last bit)
    codes_same = (ap.cpu()[:R] == ref_q).double().mean().item()
    assert codes_same > 0.99, codes_same
    check_nv(ap_dq, ref["ap"], s_got, s_ref)
    check_bf16(o[:R], ref["o"], tol=TOL_NVFP4)
    _status_clean(moe)


# ------------------------------------------------------------------ layer


def run_fwd_nv(moe, wl, d):
    cfg = moe.make_config(wl)
    T, k, H = wl.T, wl.k, wl.H
    q = {}
    for name in ["W_g", "W_u", "W_d"] + (["W_gs", "W_us", "W_ds"] if wl.S else []):
        q[name] = _gpu_quant_w(moe, d[name])
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


def check_fwd_nv(moe, oracle, wl, n_sample=None, seed=0):
    d = make_inputs(wl, device="cuda", seed=seed)
    y, idx, gates = run_fwd_nv(moe, wl, d)
    r, same = routing_agreement(oracle, wl, {"x": d["x"].cpu(), "W_r": d["W_r"].cpu(),
                                             "expert_bias": None if d.get("expert_bias") is None
                                             else d["expert_bias"].cpu()}, idx)
    if n_sample is None:
        toks = torch.arange(wl.T, dtype=torch.int32)
    else:
        toks = torch.randperm(wl.T, generator=torch.Generator().manual_seed(seed + 7))[:n_sample].sort().values
        toks = toks.to(torch.int32)
    toks = toks[same[toks.long()]]
    # the oracle quantises the bf16 weights itself, only the experts the sampled tokens use (G per expert)
    need = sorted(set(r["idx"][toks.long()].flatten().tolist()) - {-1})
    nv = {}
    for name in ("W_g", "W_u", "W_d"):
        W = d[name]
        packed = torch.zeros(W.shape[:-1] + (W.shape[-1] // 2,), dtype=torch.uint8)
        sf = torch.zeros(W.shape[:-1] + (W.shape[-1] // 16,), dtype=torch.uint8)
        G = torch.ones(W.shape[0], dtype=torch.float32)
        for e in need:
            p_, s_, g_ = oracle.nvfp4_quantize(W[e].cpu(), per_matrix=True)
            packed[e], sf[e], G[e] = p_, s_, g_
        nv[name] = (packed, sf, G)
    for name in ("W_gs", "W_us", "W_ds"):
        if wl.S:
            nv[name] = oracle.nvfp4_quantize(d[name].cpu(), per_matrix=True)
    shared = (nv["W_gs"][0], nv["W_us"][0], nv["W_ds"][0], nv["W_gs"][1:], nv["W_us"][1:], nv["W_ds"][1:]) \
        if wl.S else None
    y_ref = oracle.moe_fwd_tokens(d["x"].cpu(), nv["W_g"][0], nv["W_u"][0], nv["W_d"][0], r["idx_kept"], r["gates"],
                                  toks, recipe="nvfp4", sf_g=nv["W_g"][1:], sf_u=nv["W_u"][1:], sf_d=nv["W_d"][1:],
                                  shared=shared)
    e = check_bf16(y.cpu()[toks.long()], y_ref, tol=TOL_NVFP4, terms=wl.k + wl.S)
    assert moe.moe_get_device_status() == 0
    return e


def test_layer_fwd_nvfp4_small_full_oracle(moe, oracle):
    wl = Workload("nv-small", T=256, H=512, E=16, k=4, F=256, S=1, score="sigmoid", route_scale=2.5, dtype="nvfp4",
                  aux=False)
    check_fwd_nv(moe, oracle, wl)


def test_layer_fwd_nvfp4_softmax_ragged_full_oracle(moe, oracle):
    wl = Workload("nv-ragged", T=333, H=768, E=12, k=3, F=512, dtype="nvfp4", aux=True)
    check_fwd_nv(moe, oracle, wl)


def test_layer_fwd_nvfp4_deepseek_router_and_capacity_full_oracle(moe, oracle):
    # the DeepSeek-V3 router variant (selection bias, 4 groups, 2 kept) with a capacity factor that drops pairs
    wl = Workload("nv-dsv3-cap", T=320, H=512, E=32, k=4, F=256, S=1, score="sigmoid", route_scale=2.5, aux=False,
                  dtype="nvfp4", n_group=4, topk_group=2, sel_bias=True, capacity_factor=1.0)
    check_fwd_nv(moe, oracle, wl)

