"""Stage-by-stage parity of the CUDA path (through the C ABI) with the oracle.

Inputs are seeded synthetic tensors fed identically to both sides; no oracle
input comes from the GPU. Integer and byte results (top-k indices, counts,
offsets, maps, MXFP8 codes and scales) must be bit-exact; floating results
must be within TOL * rms(ref).
"""
import pytest
import torch

from helpers import TOL_BF16, check_bf16, e_of_rows, empty, err_rms
from mixture_experts_layer_aux_b200.synthetic import (random_gates, random_logits, random_routing, randn_bf16,
                                                      skew_bias)

pytestmark = pytest.mark.gpu


def _status_clean(moe):
    assert moe.moe_get_device_status(clear=True) == 0


# ------------------------------------------------------------------ router


@pytest.mark.parametrize("T,H,E,bias", [(512, 256, 8, False), (300, 512, 128, True), (1000, 4096, 128, False),
                                        (129, 7168, 256, True), (1, 256, 8, False),
                                        # E <= 16: logits computed inside the top-k kernel; a ragged last round
                                        # of 16-byte chunks (H = 384: 48 chunks over 32 lanes), an odd T, fewer
                                        # chunks than lanes (H = 128), and the Mixtral shape
                                        (333, 384, 16, True), (77, 128, 4, True), (4096, 4096, 8, False)])
def test_router_logits_match_oracle(moe, oracle, T, H, E, bias):
    x = randn_bf16((T, H), 1.0, seed=T, device="cuda")
    W_r = randn_bf16((E, H), 0.02, seed=T + 1, device="cuda")
    b = skew_bias(E).cuda() if bias else None
    k = min(8, E)
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=128)
    logits = empty((T, E), torch.float32)
    idx = empty((T, k), torch.int32)
    gates = empty((T, k), torch.float32)
    ws = moe.workspace(moe.moe_router_workspace_size(cfg))
    moe.moe_router_topk(cfg, x, W_r, b, logits, None, idx, gates, None, None, ws)
    torch.cuda.synchronize()
    ref = oracle.router_logits(x.cpu(), W_r.cpu(), None if b is None else b.cpu())
    e = err_rms(logits, ref)
    assert e <= 1e-4, e
    # indices: identical to the oracle's own routing except on near-ties whose
    # logit gap is below the logit error bound
    ridx = oracle.topk(ref, k)
    diff = (idx.cpu() != ridx).any(1).nonzero().flatten().tolist()
    bound = 1e-4 * float(ref.pow(2).mean().sqrt())
    for t in diff:
        vals = ref[t]
        gi, ri = idx[t].cpu(), ridx[t]
        a = sorted(set(gi[gi != ri].tolist()) | set(ri[gi != ri].tolist()))
        gap = max(vals[a]) - min(vals[a])
        assert gap <= 2 * bound, (t, gap)
    assert len(diff) <= max(2, T // 1000)
    _status_clean(moe)


ROUTING_CASES = [
    # T, E, k, score, norm, scale, ties
    (512, 8, 2, "softmax", True, 1.0, False),
    (4096, 8, 2, "softmax", True, 1.0, True),
    (8192, 128, 8, "softmax", True, 1.0, False),
    (8192, 128, 8, "softmax", True, 1.0, True),
    (8192, 256, 8, "sigmoid", True, 2.5, False),
    (777, 256, 8, "sigmoid", True, 2.5, True),
    (33, 512, 16, "softmax", False, 1.0, False),
    (1, 4, 4, "softmax", True, 1.0, True),
]


@pytest.mark.parametrize("T,E,k,score,norm,scale,ties", ROUTING_CASES)
def test_routing_from_logits_bit_exact(moe, oracle, T, E, k, score, norm, scale, ties):
    l = random_logits(T, E, seed=T + E, ties=ties)
    aux_on = score == "softmax"
    cfg = moe.make_config(T=T, H=256, E=E, k=k, F=128, score=0 if score == "softmax" else 1, norm_topk=int(norm),
                          route_scale=scale, compute_aux=int(aux_on))
    lg = l.cuda()
    probs = empty((T, E), torch.float32)
    idx = empty((T, k), torch.int32)
    gates = empty((T, k), torch.float32)
    counts = empty((E,), torch.int32)
    aux = empty((1,), torch.float32) if aux_on else None
    ws = moe.workspace(moe.moe_router_workspace_size(cfg))
    moe.moe_router_topk(cfg, None, None, None, lg, probs, idx, gates, counts, aux, ws)
    torch.cuda.synchronize()
    r = oracle.route(l.double(), k, score, norm, scale, with_aux=aux_on)
    assert torch.equal(idx.cpu(), r["idx"])
    assert torch.equal(counts.cpu(), r["counts"])
    assert (gates.cpu().double() - r["gates"]).abs().max().item() <= 2e-6 * max(1.0, scale)
    assert (probs.cpu().double() - r["probs"]).abs().max().item() <= 2e-6
    if aux_on:
        assert abs(aux.item() - r["aux"]) <= 1e-5 * abs(r["aux"])
    _status_clean(moe)


@pytest.mark.parametrize("T,E,k,n_group,topk_group", [(4096, 256, 8, 8, 4), (1000, 64, 6, 8, 3), (333, 32, 4, 0, 0),
                                                      (64, 16, 4, 16, 4)])
def test_routing_deepseek_variant_from_logits(moe, oracle, T, E, k, n_group, topk_group):
    """Selection on the fp32 score + bias (group-limited): the oracle selects on the same fp32
    values (the GPU's scores plus the bias, added in fp32) and both sides add a group's two largest
    values exactly (in double), so the indices must agree bit for bit on every token."""
    l = random_logits(T, E, seed=T + E + 5)
    g = torch.Generator().manual_seed(E)
    b = ((torch.rand(E, generator=g) - 0.5) * 0.2).float()
    cfg = moe.make_config(T=T, H=256, E=E, k=k, F=128, score=1, norm_topk=1, route_scale=2.5, n_group=n_group,
                          topk_group=topk_group)
    probs, idx, gates = empty((T, E), torch.float32), empty((T, k), torch.int32), empty((T, k), torch.float32)
    ws = moe.workspace(moe.moe_router_workspace_size(cfg))
    moe.moe_router_topk(cfg, None, None, None, l.cuda(), probs, idx, gates, None, None, ws, expert_bias=b.cuda())
    torch.cuda.synchronize()
    r = oracle.route(l.double(), k, "sigmoid", True, 2.5, with_aux=False, expert_bias=b.double(), n_group=n_group,
                     topk_group=topk_group)
    assert (probs.cpu().double() - r["probs"]).abs().max().item() <= 2e-6
    sel32 = (probs.cpu() + b).double()                       # the GPU's selection values, exactly
    ref = oracle.topk_grouped(sel32, k, n_group, topk_group)
    assert torch.equal(idx.cpu(), ref)
    ok = (idx.cpu() == r["idx"]).all(1)
    gref = r["gates"][ok]
    assert (gates.cpu().double()[ok] - gref).abs().max().item() <= 5e-6
    _status_clean(moe)


# ------------------------------------------------------------------ permute


PERMUTE_CASES = [
    # T, H, E, k, zero_experts, hot
    (512, 256, 8, 2, 0, 0.0),
    (4096, 4096, 8, 2, 0, 0.0),
    (8192, 4096, 128, 8, 4, 0.0),
    (1000, 512, 64, 8, 10, 0.6),
    (1, 256, 4, 4, 0, 0.0),
    (130, 7168, 256, 8, 0, 0.0),
    (257, 256, 16, 1, 15, 0.0),  # every token on expert 0
    # more rank blocks x experts than the scan stages in shared memory (its two-pass path): without and with
    # rows long enough for the permute kernel's shared-memory staging
    (8192, 128, 512, 2, 37, 0.0),
    (7000, 2048, 512, 2, 5, 0.0),
    # rows past the permute kernel's register chunks and shared-memory slot (H > 4096): a ragged last group
    (300, 4480, 16, 2, 0, 0.0),
]


@pytest.mark.parametrize("T,H,E,k,zero,hot", PERMUTE_CASES)
def test_permute_bit_exact(moe, oracle, T, H, E, k, zero, hot):
    idx = random_routing(T, E, k, seed=T, zero_experts=zero, hot=hot)
    g = random_gates(T, k, seed=T)
    x = randn_bf16((T, H), 1.0, seed=T + 3)
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=128)
    rows = T * k
    counts, offsets = empty((E,), torch.int32), empty((E + 1,), torch.int32)
    row_of, src_of = empty((T, k), torch.int32), empty((rows,), torch.int32)
    row_gate = empty((rows,), torch.float32)
    xp = empty((rows, H), torch.bfloat16)
    ws = moe.workspace(moe.moe_permute_workspace_size(cfg))
    moe.moe_permute(cfg, x.cuda(), idx.cuda(), g.cuda(), counts, offsets, row_of, src_of, row_gate, xp, None, ws)
    torch.cuda.synchronize()
    c, o, ro, so = oracle.maps(idx, E)
    assert torch.equal(counts.cpu(), c)
    assert torch.equal(offsets.cpu(), o)
    assert torch.equal(row_of.cpu(), ro)
    assert torch.equal(src_of.cpu(), so)
    gflat = torch.empty(rows, dtype=torch.float32)
    gflat[ro.flatten().long()] = g.flatten()
    assert torch.equal(row_gate.cpu(), gflat)
    assert torch.equal(xp.cpu().view(torch.int16), x[so.long()].view(torch.int16))
    _status_clean(moe)


@pytest.mark.parametrize("T,H,E,k", [(300, 256, 8, 2), (1024, 7168, 256, 8), (300, 4480, 16, 4)])
def test_permute_mxfp8_bit_exact(moe, oracle, T, H, E, k):
    idx = random_routing(T, E, k, seed=T + 1)
    x = randn_bf16((T, H), 1.0, seed=T + 5, scale_rows=True)
    x[0, :64] = 0  # an all-zero block
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=128, expert_dtype=1)
    rows = T * k
    offsets = empty((E + 1,), torch.int32)
    row_of, src_of = empty((T, k), torch.int32), empty((rows,), torch.int32)
    xp = empty((rows, H), torch.uint8)
    xsf = empty((rows, H // 32), torch.uint8)
    ws = moe.workspace(moe.moe_permute_workspace_size(cfg))
    moe.moe_permute(cfg, x.cuda(), idx.cuda(), None, None, offsets, row_of, src_of, None, xp, xsf, ws)
    torch.cuda.synchronize()
    _, _, ro, so = oracle.maps(idx, E)
    assert torch.equal(src_of.cpu(), so)
    q, s = oracle.mxfp8_quantize(x[so.long()].contiguous())
    assert torch.equal(xsf.cpu(), s)
    assert torch.equal(xp.cpu(), q)
    _status_clean(moe)


@pytest.mark.parametrize("R,K", [(64, 256), (1000, 7168), (3, 2048)])
def test_quantize_mxfp8_bit_exact(moe, oracle, R, K):
    w = randn_bf16((R, K), 0.02, seed=R, scale_rows=True)
    w[0, 32:64] = 0
    if R > 2:
        w[1, :32] = torch.tensor([1e-40] * 16 + [-3e-39] * 16).to(torch.bfloat16)  # bf16 subnormals
        w[2, :32] = torch.tensor([448.0, 500.0, -1e30] + [1.0] * 29).to(torch.bfloat16)
    dst = empty((R, K), torch.uint8)
    sf = empty((R, K // 32), torch.uint8)
    moe.moe_quantize_mxfp8(w.cuda(), dst, sf)
    torch.cuda.synchronize()
    q, s = oracle.mxfp8_quantize(w)
    assert torch.equal(sf.cpu(), s)
    assert torch.equal(dst.cpu(), q)


# ------------------------------------------------------------------ unpermute


@pytest.mark.parametrize("T,H,k,extra", [(512, 256, 2, False), (8192, 4096, 8, False), (100, 7168, 8, True),
                                         (1, 256, 1, True)])
def test_unpermute_matches_oracle(moe, oracle, T, H, k, extra):
    E = 16
    idx = random_routing(T, E, k, seed=T + 7)
    _, _, ro, _ = oracle.maps(idx, E)
    o = randn_bf16((T * k, H), 1.0, seed=T + 8)
    ex = randn_bf16((T, H), 1.0, seed=T + 9) if extra else None
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=128)
    y = empty((T, H), torch.bfloat16)
    moe.moe_unpermute(cfg, o.cuda(), ro.cuda(), None if ex is None else ex.cuda(), y)
    torch.cuda.synchronize()
    ref = oracle.unpermute(o.double(), ro, None if ex is None else ex.double())
    d = (y.cpu().double() - ref).abs()
    # fp32 sum then one bf16 rounding: within 2^-8 relative (plus fp32 noise)
    assert (d <= ref.abs() * 2.0 ** -8 + 1e-6).all()
    assert err_rms(y, ref) <= TOL_BF16


# ------------------------------------------------------------------ grouped GEMMs


GEMM_CASES = [
    # T, H, E, k, F, zero_experts, hot
    (300, 256, 8, 2, 512, 2, 0.0),
    (200, 512, 4, 1, 256, 0, 0.95),   # one expert holds almost every row
    (100, 256, 16, 4, 384, 3, 0.0),   # F a multiple of 128 only
    (1000, 1024, 32, 8, 1536, 0, 0.3),
    (2100, 512, 4, 2, 512, 1, 0.0),   # large experts (1400 rows): the SM-pair kernel's own regime
]


@pytest.fixture(params=["default", "pair"])
def fwd_kernel(request, monkeypatch):
    """Run the forward GEMMs with the library's own kernel choice (the one-SM, 128-row
    tile kernel unless MOE_B200_PAIR_MIN_ROWS opts in), or forced onto the SM-pair
    (256-row tile) kernel."""
    if request.param == "pair":
        monkeypatch.setenv("MOE_B200_PAIR_MIN_ROWS", "0")
    else:
        monkeypatch.delenv("MOE_B200_PAIR_MIN_ROWS", raising=False)
    return request.param


@pytest.mark.parametrize("T,H,E,k,F,zero,hot", GEMM_CASES)
def test_grouped_gemm_fwd_matches_oracle(moe, oracle, fwd_kernel, T, H, E, k, F, zero, hot):
    idx = random_routing(T, E, k, seed=T + F, zero_experts=zero, hot=hot)
    counts, offsets, _, _ = oracle.maps(idx, E)
    rows = T * k
    xp = randn_bf16((rows, H), 1.0, seed=rows)
    g = random_gates(rows, 1, seed=rows).flatten()
    Wg = randn_bf16((E, F, H), 0.02, seed=1)
    Wu = randn_bf16((E, F, H), 0.02, seed=2)
    Wd = randn_bf16((E, H, F), 0.02, seed=3)
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=F)
    ap = empty((rows, F), torch.bfloat16)
    save = empty((rows, 2 * F), torch.bfloat16)
    o = empty((rows, H), torch.bfloat16)
    ws = moe.workspace(moe.moe_grouped_gemm_workspace_size(cfg, 0))
    dev = dict(xp=xp.cuda(), g=g.cuda(), Wg=Wg.cuda(), Wu=Wu.cuda(), Wd=Wd.cuda(), off=offsets.cuda())
    moe.moe_grouped_gemm_fwd(cfg, 0, dev["xp"], None, dev["Wg"], None, dev["Wu"], None, dev["off"], dev["g"], ap, None,
                             save, ws)
    moe.moe_grouped_gemm_fwd(cfg, 1, ap, None, dev["Wd"], None, None, None, dev["off"], None, o, None, None, ws)
    torch.cuda.synchronize()
    ref = oracle.expert_rows(xp, e_of_rows(offsets), g.double(), Wg, Wu, Wd, recipe="bf16",
                             want=("zg", "zu", "ap", "o"))
    check_bf16(ap, ref["ap"])
    check_bf16(save[:, :F].contiguous(), ref["zg"])
    check_bf16(save[:, F:].contiguous(), ref["zu"])
    check_bf16(o, ref["o"])
    _status_clean(moe)


# ------------------------------------------------------------------ MXFP8 grouped GEMMs


MX_CASES = [
    # T, H, E, k, F, zero_experts, hot
    (300, 256, 8, 2, 256, 2, 0.0),
    (200, 512, 4, 1, 384, 0, 0.9),
    (513, 1024, 16, 4, 512, 3, 0.3),
]


def _gpu_quant(moe, w):
    codes = torch.empty(w.shape, dtype=torch.uint8, device="cuda")
    sf = torch.empty(w.shape[:-1] + (w.shape[-1] // 32,), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8(w.cuda().contiguous(), codes, sf)
    return codes, sf


@pytest.mark.parametrize("T,H,E,k,F,zero,hot", MX_CASES)
def test_grouped_gemm_mxfp8_matches_oracle(moe, oracle, T, H, E, k, F, zero, hot):
    from helpers import check_mx
    idx = random_routing(T, E, k, seed=T + F + 1, zero_experts=zero, hot=hot)
    counts, offsets, _, _ = oracle.maps(idx, E)
    rows = T * k
    xp = randn_bf16((rows, H), 1.0, seed=rows + 1)
    g = random_gates(rows, 1, seed=rows + 2).flatten() * 2.5
    Wg = randn_bf16((E, F, H), 0.02, seed=11)
    Wu = randn_bf16((E, F, H), 0.02, seed=12)
    Wd = randn_bf16((E, H, F), 0.02, seed=13)
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=F, expert_dtype=1)
    xq, xs = _gpu_quant(moe, xp)
    (gq, gs), (uq, us), (dq, ds) = _gpu_quant(moe, Wg), _gpu_quant(moe, Wu), _gpu_quant(moe, Wd)
    ap = empty((rows, F), torch.uint8)
    ap_sf = empty((rows, F // 32), torch.uint8)
    o = empty((rows, H), torch.bfloat16)
    ws = moe.workspace(256)
    off = offsets.cuda()
    moe.moe_grouped_gemm_fwd(cfg, 0, xq, xs, gq, gs, uq, us, off, g.cuda(), ap, ap_sf, None, ws)
    moe.moe_grouped_gemm_fwd(cfg, 1, ap, ap_sf, dq, ds, None, None, off, None, o, None, None, ws)
    torch.cuda.synchronize()
    # the oracle quantises the same bf16 weights itself (bit-identical codes, tested above)
    Q = {n: oracle.mxfp8_quantize(w) for n, w in (("g", Wg), ("u", Wu), ("d", Wd))}
    ref = oracle.expert_rows(xp, e_of_rows(offsets), g.double(), Q["g"][0], Q["u"][0], Q["d"][0], recipe="mxfp8",
                             sf_g=Q["g"][1], sf_u=Q["u"][1], sf_d=Q["d"][1], want=("ap", "o"))
    ap_dq = oracle.mxfp8_decode(ap.cpu(), ap_sf.cpu())
    scale = torch.pow(2.0, ap_sf.cpu().double() - 127).repeat_interleave(32, 1)
    check_mx(ap_dq, ref["ap"], scale)
    check_bf16(o, ref["o"], tol=6e-2)
    _status_clean(moe)
