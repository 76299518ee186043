"""Transposed MXFP8 operands of the MXFP8 backward, against the oracle's quantiser.

Weights are quantised along their rows after a transpose (W^T in blocks of 32
along the original row dimension); the weight-gradient activations are
quantised along each expert's tokens into a transposed buffer whose expert
segments start on 128-row boundaries. Byte results are compared bit for bit
with the oracle's quantiser applied to the transposed (and zero-padded) bf16
source; the recomputed activation (mode 2) is compared within one E4M3 step,
since its fp32 value is computed on the GPU.
"""
import pytest
import torch

from helpers import check_mx, empty
from mixture_experts_layer_aux_b200.synthetic import random_routing, randn_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,R,C,extra", [(3, 64, 96, 0), (2, 256, 512, 64), (1, 32, 8, 0)])
def test_weight_transpose_quantise_bit_exact(moe, oracle, B, R, C, extra):
    w = randn_bf16((B, R, C), 0.02, seed=R + C)
    ldd = R + extra
    dst = torch.full((B, C, ldd), 0xAB, dtype=torch.uint8, device="cuda")
    sf = torch.full((B, C, ldd // 32), 0xCD, dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8_t(w.cuda(), dst, sf, ldd=ldd)
    torch.cuda.synchronize()
    codes, scales = oracle.mxfp8_quantize(w.transpose(1, 2).contiguous())
    assert torch.equal(dst.cpu()[:, :, :R], codes)
    assert torch.equal(sf.cpu()[:, :, :R // 32], scales)
    if extra:                                                   # the rest of each row is untouched
        assert bool((dst.cpu()[:, :, R:] == 0xAB).all()) and bool((sf.cpu()[:, :, R // 32:] == 0xCD).all())
    assert moe.moe_get_device_status() == 0


def untile(sf_tiled, C, ldd):
    """The tiled scale layout of the grouped transposed quantiser -> natural [C, ldd/32]."""
    r = torch.arange(C)[:, None]
    j = torch.arange(ldd // 32)[None, :]
    pos = ((r // 128) * (ldd // 128) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4
    return sf_tiled.reshape(-1)[pos.reshape(-1)].reshape(C, ldd // 32)


def _grouped_case(moe, T, E, k, C, zero, hot, seed):
    idx = random_routing(T, E, k, seed=seed, zero_experts=zero, hot=hot)
    cnt = torch.bincount(idx.flatten().long(), minlength=E)
    off = torch.zeros(E + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(cnt, 0)
    cfg = moe.make_config(T=T, H=256, E=E, k=k, F=128)
    ldd = moe.moe_mxfp8_t_padded_rows(cfg)
    padded = ((cnt + 127) // 128) * 128
    poff_ref = torch.zeros(E + 1, dtype=torch.int32)
    poff_ref[1:] = torch.cumsum(padded, 0)
    return cfg, off, poff_ref, ldd


def _expected_segments(oracle, rows_src, off, poff, E, C, ldd):
    """dst/sf the oracle's quantiser gives: per expert, its rows transposed, zero-padded to 128."""
    codes = torch.zeros((C, ldd), dtype=torch.uint8)
    scales = torch.zeros((C, ldd // 32), dtype=torch.uint8)
    for e in range(E):
        n = int(off[e + 1] - off[e])
        if n == 0:
            continue
        npad = ((n + 127) // 128) * 128
        seg = torch.zeros((npad, C), dtype=rows_src.dtype)
        seg[:n] = rows_src[int(off[e]):int(off[e + 1])]
        c_, s_ = oracle.mxfp8_quantize(seg.T.contiguous())
        p = int(poff[e])
        codes[:, p:p + npad] = c_
        scales[:, p // 32:(p + npad) // 32] = s_
    return codes, scales


@pytest.mark.parametrize("T,E,k,C,zero,hot", [(300, 8, 2, 128, 0, 0.0), (1000, 16, 4, 384, 3, 0.5),
                                              (64, 4, 1, 128, 3, 0.0)])
@pytest.mark.parametrize("mode", [0, 1])
def test_grouped_transpose_quantise_bit_exact(moe, oracle, T, E, k, C, zero, hot, mode):
    cfg, off, poff_ref, ldd = _grouped_case(moe, T, E, k, C, zero, hot, seed=T + mode)
    rows = T * k
    g = torch.Generator().manual_seed(C)
    if mode == 0:
        src = randn_bf16((rows, C), 1.0, seed=C + 1)
        src_of = None
        rows_src = src
    else:
        src = randn_bf16((T, C), 1.0, seed=C + 2)
        src_of = torch.randint(0, T, (rows,), generator=g, dtype=torch.int32)
        rows_src = src[src_of.long()]
    dst = torch.zeros((C, ldd), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((C, ldd // 32), dtype=torch.uint8, device="cuda")
    poff = empty((cfg.E + 1,), torch.int32)
    moe.moe_quantize_mxfp8_t_grouped(cfg, mode, src.cuda(), None if src_of is None else src_of.cuda(), None,
                                     off.cuda(), poff, C, dst, ldd, sf)
    torch.cuda.synchronize()
    assert torch.equal(poff.cpu(), poff_ref)
    codes, scales = _expected_segments(oracle, rows_src, off, poff_ref, E, C, ldd)
    tot = int(poff_ref[-1])
    assert torch.equal(dst.cpu()[:, :tot], codes[:, :tot])
    assert torch.equal(untile(sf.cpu(), C, ldd)[:, :tot // 32], scales[:, :tot // 32])
    assert moe.moe_get_device_status() == 0


def test_grouped_transpose_of_recomputed_activation(moe, oracle):
    T, E, k, F = 500, 8, 2, 128
    cfg, off, poff_ref, ldd = _grouped_case(moe, T, E, k, F, 1, 0.3, seed=7)
    rows = T * k
    gu = randn_bf16((rows, 2 * F), 1.5, seed=9)
    rg = torch.rand(rows, generator=torch.Generator().manual_seed(3)) * 0.9 + 0.05
    dst = torch.zeros((F, ldd), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((F, ldd // 32), dtype=torch.uint8, device="cuda")
    poff = empty((E + 1,), torch.int32)
    moe.moe_quantize_mxfp8_t_grouped(cfg, 2, gu.cuda(), None, rg.cuda(), off.cuda(), poff, F, dst, ldd, sf)
    torch.cuda.synchronize()
    zg, zu = gu[:, :F].double(), gu[:, F:].double()
    ap = rg.double()[:, None] * torch.nn.functional.silu(zg) * zu      # the gate-folded activation, fp64
    codes, scales = _expected_segments(oracle, ap.float(), off, poff_ref, E, F, ldd)
    tot = int(poff_ref[-1])
    sfn = untile(sf.cpu(), F, ldd)
    got = oracle.mxfp8_decode(dst.cpu()[:, :tot], sfn[:, :tot // 32])
    ref = oracle.mxfp8_decode(codes[:, :tot], scales[:, :tot // 32])
    scale = torch.pow(2.0, sfn[:, :tot // 32].double() - 127.0).repeat_interleave(32, dim=1)
    check_mx(got, ref, scale)
    assert moe.moe_get_device_status() == 0


# ------------------------------------------------------------------ MXFP8 backward GEMMs


def _routing(T, E, k, zero, hot, seed):
    idx = random_routing(T, E, k, seed=seed, zero_experts=zero, hot=hot)
    cnt = torch.bincount(idx.flatten().long(), minlength=E)
    off = torch.zeros(E + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(cnt, 0)
    return off


def _dq(oracle, codes, sf):
    return oracle.mxfp8_decode(codes.cpu(), sf.cpu())


@pytest.mark.parametrize("which", ["down", "gateup"])
def test_wgrad_mxfp8_grouped_along_tokens(moe, oracle, which):
    """dW[e] = AT[:, seg e] BT[:, seg e]^T over the transposed MXFP8 operands (decoded, fp64)."""
    from helpers import check_bf16
    T, E, k, H, F = 600, 8, 2, 256, 256
    off = _routing(T, E, k, 1, 0.4, seed=5)                       # expert 7 gets no token
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=F)
    rows, ldp = T * k, moe.moe_mxfp8_t_padded_rows(cfg)
    M, N = (H, F) if which == "down" else (2 * F, H)
    a_rows = randn_bf16((rows, M), 1.0, seed=11)
    b_rows = randn_bf16((rows, N), 1.0, seed=12)
    bufs = {}
    for name, src, C in (("A", a_rows, M), ("B", b_rows, N)):
        d = torch.zeros((C, ldp), dtype=torch.uint8, device="cuda")
        s = torch.zeros((C, ldp // 32), dtype=torch.uint8, device="cuda")
        poff = empty((E + 1,), torch.int32)
        moe.moe_quantize_mxfp8_t_grouped(cfg, 0, src.cuda(), None, None, off.cuda(), poff, C, d, ldp, s)
        bufs[name] = (d, s)
    if which == "down":
        dW0, dW1 = empty((E, H, F), torch.bfloat16), None
    else:
        dW0, dW1 = empty((E, F, H), torch.bfloat16), empty((E, F, H), torch.bfloat16)
    moe.moe_grouped_gemm_wgrad_mxfp8(cfg, 1 if which == "down" else 0, *bufs["A"], *bufs["B"], poff, ldp, dW0, dW1)
    torch.cuda.synchronize()
    A = oracle.mxfp8_decode(bufs["A"][0].cpu(), untile(bufs["A"][1].cpu(), M, ldp))
    B = oracle.mxfp8_decode(bufs["B"][0].cpu(), untile(bufs["B"][1].cpu(), N, ldp))
    p = poff.cpu()
    ref = torch.stack([A[:, int(p[e]):int(p[e + 1])] @ B[:, int(p[e]):int(p[e + 1])].T for e in range(E)])
    got = dW0.cpu() if which == "down" else torch.cat([dW0.cpu(), dW1.cpu()], dim=1)
    check_bf16(got, ref)
    assert bool((got[7] == 0).all())                              # no token: exact zeros
    assert moe.moe_get_device_status() == 0


def test_dgrad_mxfp8_down_swiglu_backward_and_gateup(moe, oracle):
    """dgate/dup and dg from MXFP8 dY . W_d^T with the SwiGLU backward on saved bf16 z; then
    dXp from MXFP8 dgate|dup . [W_g^T | W_u^T]. References in fp64 over the decoded operands."""
    from helpers import check_bf16, err_rms
    T, E, k, H, F = 400, 4, 2, 256, 256
    off = _routing(T, E, k, 0, 0.0, seed=6)
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=F, expert_dtype=1)
    rows = T * k
    dYp = randn_bf16((rows, H), 1.0, seed=21)
    Wd = randn_bf16((E, H, F), 0.02, seed=22)
    Wg = randn_bf16((E, F, H), 0.02, seed=23)
    Wu = randn_bf16((E, F, H), 0.02, seed=24)
    gu = randn_bf16((rows, 2 * F), 1.0, seed=25)
    rg = torch.rand(rows, generator=torch.Generator().manual_seed(26)) * 0.9 + 0.05
    dq = torch.empty((rows, H), dtype=torch.uint8, device="cuda")
    dq_sf = torch.empty((rows, H // 32), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8(dYp.cuda(), dq, dq_sf)
    wdt = torch.empty((E, F, H), dtype=torch.uint8, device="cuda")
    wdt_sf = torch.empty((E, F, H // 32), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8_t(Wd.cuda(), wdt, wdt_sf)
    wgu = torch.empty((E, H, 2 * F), dtype=torch.uint8, device="cuda")
    wgu_sf = torch.empty((E, H, 2 * F // 32), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8_t(Wg.cuda(), wgu, wgu_sf, ldd=2 * F)
    moe.moe_quantize_mxfp8_t(Wu.cuda(), wgu, wgu_sf, ldd=2 * F, col0=F)
    dgu = empty((rows, 2 * F), torch.bfloat16)
    dg = empty((rows,), torch.float32)
    ws = moe.workspace(rows * (F // 128) * 4)
    offd = off.cuda()
    moe.moe_grouped_gemm_dgrad_mxfp8(cfg, 1, dq, dq_sf, wdt, wdt_sf, offd, gu.cuda(), rg.cuda(), dgu, dg, ws)
    torch.cuda.synchronize()
    v = torch.empty((rows, F), dtype=torch.float64)
    A, Bd = _dq(oracle, dq, dq_sf), _dq(oracle, wdt, wdt_sf)
    for e in range(E):
        sl = slice(int(off[e]), int(off[e + 1]))
        v[sl] = A[sl] @ Bd[e].T
    zg, zu = gu[:, :F].double(), gu[:, F:].double()
    sg = torch.sigmoid(zg)
    g = rg.double()[:, None]
    ref_dgu = torch.cat([g * v * zu * sg * (1 + zg * (1 - sg)), g * v * zg * sg], dim=1)
    check_bf16(dgu.cpu(), ref_dgu)
    ref_dg = (v * torch.nn.functional.silu(zg) * zu).sum(1)
    assert err_rms(dg.cpu(), ref_dg) <= 1e-4
    # gate/up dgrad on the GPU's dgate|dup
    gq = torch.empty((rows, 2 * F), dtype=torch.uint8, device="cuda")
    gq_sf = torch.empty((rows, 2 * F // 32), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8(dgu, gq, gq_sf)
    dxp = empty((rows, H), torch.bfloat16)
    moe.moe_grouped_gemm_dgrad_mxfp8(cfg, 0, gq, gq_sf, wgu, wgu_sf, offd, None, None, dxp, None, ws)
    torch.cuda.synchronize()
    G, W = _dq(oracle, gq, gq_sf), _dq(oracle, wgu, wgu_sf)
    ref = torch.empty((rows, H), dtype=torch.float64)
    for e in range(E):
        sl = slice(int(off[e]), int(off[e + 1]))
        ref[sl] = G[sl] @ W[e].T
    check_bf16(dxp.cpu(), ref)
    assert moe.moe_get_device_status() == 0


# ------------------------------------------------------------------ MXFP8 layer backward


def _mx_layer(moe, oracle, wl, seed, d_aux=0.2):
    from helpers import TOL_MXFP8, check_bf16, err_rms
    from mixture_experts_layer_aux_b200.synthetic import make_inputs
    d = make_inputs(wl, device="cuda", seed=seed, with_dy=True)
    T, H, E, k, F = wl.T, wl.H, wl.E, wl.k, wl.F
    cfg = moe.make_config(wl, save_for_bwd=1)
    q = {}
    for n in ("W_g", "W_u", "W_d"):
        c_ = torch.empty(d[n].shape, dtype=torch.uint8, device="cuda")
        s_ = torch.empty(d[n].shape[:-1] + (d[n].shape[-1] // 32,), dtype=torch.uint8, device="cuda")
        moe.moe_quantize_mxfp8(d[n], c_, s_)
        q[n] = (c_, s_)
    wdt = torch.empty((E, F, H), dtype=torch.uint8, device="cuda")
    wdt_sf = torch.empty((E, F, H // 32), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8_t(d["W_d"], wdt, wdt_sf)
    wgu = torch.empty((E, H, 2 * F), dtype=torch.uint8, device="cuda")
    wgu_sf = torch.empty((E, H, 2 * F // 32), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_mxfp8_t(d["W_g"], wgu, wgu_sf, ldd=2 * F)
    moe.moe_quantize_mxfp8_t(d["W_u"], wgu, wgu_sf, ldd=2 * F, col0=F)
    y = empty((T, H), torch.bfloat16)
    idx = empty((T, k), torch.int32)
    aux = empty((1,), torch.float32) if cfg.compute_aux else None
    saved = moe.workspace(moe.moe_layer_saved_size(cfg))
    moe.moe_layer_fwd(cfg, d["x"], d["W_r"], d.get("logit_bias"), q["W_g"][0], q["W_u"][0], q["W_d"][0],
                      q["W_g"][1], q["W_u"][1], q["W_d"][1], None, None, None, None, None, None, y, aux, idx, None,
                      None, None, saved, moe.workspace(moe.moe_layer_workspace_size(cfg)),
                      expert_bias=d.get("expert_bias"))
    o = dict(dX=empty((T, H), torch.bfloat16), dW_r=empty((E, H), torch.bfloat16),
             dW_g=empty((E, F, H), torch.bfloat16), dW_u=empty((E, F, H), torch.bfloat16),
             dW_d=empty((E, H, F), torch.bfloat16), dlogits=empty((T, E), torch.float32))
    moe.moe_layer_bwd_mxfp8(cfg, d["dY"], d_aux, d["x"], d["W_r"], wdt, wdt_sf, wgu, wgu_sf, saved, o["dX"],
                            o["dW_r"], o["dW_g"], o["dW_u"], o["dW_d"], o["dlogits"],
                            moe.workspace(moe.moe_layer_bwd_mxfp8_workspace_size(cfg)))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    # oracle: the MXFP8 backward recipe on the same routing
    h = {n: (v.cpu() if torch.is_tensor(v) else v) for n, v in d.items()}
    logits = oracle.router_logits(h["x"], h["W_r"], h.get("logit_bias"))
    r = oracle.route(logits, k, wl.score, wl.norm_topk, wl.route_scale, with_aux=wl.aux and wl.score == "softmax",
                     expert_bias=h.get("expert_bias"), n_group=wl.n_group, topk_group=wl.topk_group)
    assert torch.equal(idx.cpu(), r["idx"]), "full-oracle parity needs identical routing"
    # the oracle quantises the bf16 weights itself (forward operands along K; W_d^T along H, W_g^T and
    # W_u^T along F), and the GPU's codes must be the same bytes
    mx = {n: oracle.mxfp8_quantize(h[n]) for n in ("W_g", "W_u", "W_d")}
    mx.update(W_dT=oracle.mxfp8_quantize(h["W_d"].transpose(1, 2).contiguous()),
              W_gT=oracle.mxfp8_quantize(h["W_g"].transpose(1, 2).contiguous()),
              W_uT=oracle.mxfp8_quantize(h["W_u"].transpose(1, 2).contiguous()))
    for n in ("W_g", "W_u", "W_d"):
        assert torch.equal(q[n][0].cpu(), mx[n][0]) and torch.equal(q[n][1].cpu(), mx[n][1]), n
    assert torch.equal(wdt.cpu(), mx["W_dT"][0]) and torch.equal(wdt_sf.cpu(), mx["W_dT"][1])
    assert torch.equal(wgu.cpu(), torch.cat([mx["W_gT"][0], mx["W_uT"][0]], dim=2))
    assert torch.equal(wgu_sf.cpu(), torch.cat([mx["W_gT"][1], mx["W_uT"][1]], dim=2))
    aux_on = wl.aux and wl.score == "softmax"
    dx, dl, _ = oracle.moe_bwd_tokens(h["x"], h["W_r"], None, None, None, h["dY"], r, score=wl.score,
                                      norm=wl.norm_topk, route_scale=wl.route_scale, aux_on=aux_on, d_aux=d_aux,
                                      recipe="mxfp8", mx=mx)
    # MXFP8 tolerance throughout: a bf16 rounding flip upstream of an MXFP8 operand can move one of its
    # codes by a step
    res = {"dX": check_bf16(o["dX"].cpu(), dx, tol=TOL_MXFP8, terms=k + 1)[0], "dlogits": err_rms(o["dlogits"].cpu(), dl)}
    dWg, dWu, dWd = oracle.moe_bwd_expert_dw(h["x"], None, None, None, h["dY"], r["idx"], r["gates"],
                                             list(range(E)), recipe="mxfp8", mx=mx)
    for name, ref in (("dW_g", dWg), ("dW_u", dWu), ("dW_d", dWd)):
        res[name] = check_bf16(o[name].cpu(), ref, tol=TOL_MXFP8, terms=2)[0]
    res["dW_r"] = check_bf16(o["dW_r"].cpu(), oracle.router_dwr(dl, h["x"], round_dl=True), tol=TOL_MXFP8)[0]
    assert res["dlogits"] <= TOL_MXFP8, res
    print(wl.name, {kk: round(vv, 4) for kk, vv in res.items()})
    return res


def test_layer_bwd_mxfp8_full_oracle(moe, oracle):
    from mixture_experts_layer_aux_b200.synthetic import Workload
    wl = Workload("mx-bwd", T=384, H=256, E=8, k=2, F=256, dtype="mxfp8", skew=True, bwd=True)
    _mx_layer(moe, oracle, wl, seed=3)


def test_layer_bwd_mxfp8_sigmoid_router(moe, oracle):
    from mixture_experts_layer_aux_b200.synthetic import Workload
    wl = Workload("mx-bwd-sig", T=256, H=512, E=16, k=4, F=256, dtype="mxfp8", score="sigmoid", route_scale=2.5,
                  aux=False, bwd=True)
    _mx_layer(moe, oracle, wl, seed=4, d_aux=0.0)


def test_layer_bwd_mxfp8_deepseek_router_variant(moe, oracle):
    """Backward through the DeepSeek-V3 router shape: selection on sigmoid score + per-expert bias
    within the best expert groups, gates from the unbiased scores."""
    from mixture_experts_layer_aux_b200.synthetic import Workload
    wl = Workload("mx-bwd-dsv3-router", T=256, H=512, E=32, k=4, F=256, dtype="mxfp8", score="sigmoid",
                  route_scale=2.5, aux=False, bwd=True, n_group=4, topk_group=2, sel_bias=True)
    _mx_layer(moe, oracle, wl, seed=6, d_aux=0.0)
