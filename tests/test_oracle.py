"""Pins of the CPU oracle against things other than itself (no GPU).

Each test ties one oracle function to an independent fact: a dense brute
force, a library routine (torch fp64 matmul / sort / float8 cast, numpy's
half-even rounding), a closed form, an invariant, central finite differences,
or hand-computed OCP MX and NVFP4 values (tests/golden/mxfp8_ocp_cases.txt,
tests/golden/nvfp4_cases.txt). A plausible mistake anywhere in the
oracle (a dropped term, a wrong sign or index, a transposed operand) fails at
least one of them.
"""
import math
import os

import pytest
import torch

from mixture_experts_layer_aux_b200.synthetic import Workload, make_inputs, random_logits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_ocp_cases.txt")


def small(T=24, H=64, E=6, k=2, F=96, **kw):
    return Workload("small", T=T, H=H, E=E, k=k, F=F, **kw)


def ref_swiglu(x, Wg, Wu, Wd):
    """torch fp64: W_d (silu(W_g x) * (W_u x)) for rows of x."""
    zg = x @ Wg.T
    zu = x @ Wu.T
    return (torch.nn.functional.silu(zg) * zu) @ Wd.T


# --------------------------------------------------------------- routing


def test_router_logits_match_torch_fp64_matmul(oracle):
    wl = small(T=33, H=96, E=7)
    inp = make_inputs(wl, seed=1)
    bias = torch.linspace(-1, 1, wl.E)
    l = oracle.router_logits(inp["x"], inp["W_r"], bias)
    ref = (inp["x"].double() @ inp["W_r"].double().T + bias.double()).float().double()
    # fp64 sums in a different order may round to an adjacent fp32
    assert torch.allclose(l, ref, rtol=2e-7, atol=1e-9)
    l64 = oracle.router_logits(inp["x"], inp["W_r"], None, round_f32=False)
    assert torch.allclose(l64, inp["x"].double() @ inp["W_r"].double().T, rtol=1e-13, atol=1e-13)


def test_scores_match_torch(oracle):
    l = random_logits(17, 9, seed=3).double()
    assert torch.allclose(oracle.scores(l, "softmax"), torch.softmax(l, dim=1), rtol=1e-14, atol=1e-16)
    assert torch.allclose(oracle.scores(l, "sigmoid"), torch.sigmoid(l), rtol=1e-14, atol=1e-16)


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("E,k", [(8, 2), (128, 8), (5, 5), (1, 1)])
def test_topk_matches_stable_sort(oracle, E, k, ties):
    l = random_logits(64, E, seed=E + k, ties=ties).double()
    idx = oracle.topk(l, k)
    ref = torch.sort(-l, dim=1, stable=True).indices[:, :k].to(torch.int32)
    assert torch.equal(idx, ref)


def test_topk_all_equal_logits_picks_lowest_indices(oracle):
    l = torch.zeros(5, 16, dtype=torch.float64)
    idx = oracle.topk(l, 4)
    assert torch.equal(idx, torch.arange(4, dtype=torch.int32).repeat(5, 1))
    r = oracle.route(l, 4)
    assert torch.allclose(r["gates"], torch.full((5, 4), 0.25, dtype=torch.float64), rtol=0, atol=1e-16)
    # uniform probabilities: aux = E * sum_e f_e / E = 1 for any f
    assert r["aux"] == pytest.approx(1.0, abs=1e-14)


def test_gates_sum_to_route_scale(oracle):
    l = random_logits(40, 32, seed=5).double()
    r = oracle.route(l, 8, "softmax", True, 1.0)
    assert torch.allclose(r["gates"].sum(1), torch.ones(40, dtype=torch.float64), atol=1e-14)
    r = oracle.route(l, 8, "sigmoid", True, 2.5)
    assert torch.allclose(r["gates"].sum(1), torch.full((40,), 2.5, dtype=torch.float64), atol=1e-14)
    # softmax renormalised over the selected = softmax of the selected logits
    r = oracle.route(l, 8, "softmax", True, 1.0)
    sel = torch.gather(l, 1, r["idx"].long())
    assert torch.allclose(r["gates"], torch.softmax(sel, dim=1), atol=1e-15)
    # sigmoid: g = 2.5 * sigma(l_sel) / sum sigma(l_sel)
    r = oracle.route(l, 8, "sigmoid", True, 2.5)
    sg = torch.sigmoid(torch.gather(l, 1, r["idx"].long()))
    assert torch.allclose(r["gates"], 2.5 * sg / sg.sum(1, keepdim=True), atol=1e-15)


def test_aux_matches_vectorised_closed_form(oracle):
    T, E, k = 50, 12, 3
    l = random_logits(T, E, seed=7).double()
    r = oracle.route(l, k)
    counts = torch.bincount(r["idx"].flatten().long(), minlength=E).double()
    ref = E * ((counts / (T * k)) * torch.softmax(l, 1).mean(0)).sum().item()
    assert r["aux"] == pytest.approx(ref, rel=1e-13)
    # perfectly balanced counts and uniform P: aux = 1
    s = torch.full((T, E), 1.0 / E, dtype=torch.float64)
    c = torch.full((E,), T * k // E, dtype=torch.int32)
    assert oracle.aux(s, c, k) == pytest.approx(T * k // E * E / (T * k), abs=1e-14)


@pytest.mark.parametrize("T,E,k,zero", [(64, 8, 2, 0), (300, 128, 8, 4), (1, 4, 4, 0), (77, 16, 1, 3)])
def test_maps_match_stable_sort_and_invariants(oracle, T, E, k, zero):
    from mixture_experts_layer_aux_b200.synthetic import random_routing
    idx = random_routing(T, E, k, seed=T, zero_experts=zero)
    counts, offsets, row_of, src_of = oracle.maps(idx, E)
    flat = idx.flatten().long()
    srt = torch.sort(flat, stable=True)
    assert torch.equal(counts.long(), torch.bincount(flat, minlength=E))
    assert torch.equal(offsets[1:].long(), torch.cumsum(counts.long(), 0)) and offsets[0] == 0
    assert int(counts.sum()) == T * k == int(offsets[-1])
    assert torch.equal(src_of.long(), srt.indices // k)
    ref_row = torch.empty(T * k, dtype=torch.long)
    ref_row[srt.indices] = torch.arange(T * k)
    assert torch.equal(row_of.flatten().long(), ref_row)
    # bijection and src_of[row_of[t,j]] == t
    assert torch.equal(torch.sort(row_of.flatten()).values.long(), torch.arange(T * k))
    assert torch.equal(src_of[row_of.flatten().long()].long(), torch.arange(T).repeat_interleave(k))
    if zero:
        assert (counts[E - zero:] == 0).all()


def test_permute_then_unpermute_is_k_times_identity(oracle):
    from mixture_experts_layer_aux_b200.synthetic import random_routing
    T, E, k, H = 40, 8, 3, 16
    idx = random_routing(T, E, k, seed=2)
    _, _, row_of, src_of = oracle.maps(idx, E)
    x = torch.randn(T, H, dtype=torch.float64)
    xp = x[src_of.long()]                     # permute = gather by src_of
    y = oracle.unpermute(xp, row_of)
    assert torch.equal(y, k * x) or torch.allclose(y, k * x, rtol=1e-15, atol=0)
    # one-hot selection: only slot 0 rows non-zero -> recovers x exactly
    o = torch.zeros_like(xp)
    o[row_of[:, 0].long()] = x
    assert torch.equal(oracle.unpermute(o, row_of), x)


def test_unpermute_sums_every_slot_and_the_shared_row(oracle):
    """unpermute-sum = each token's k rows gathered by torch indexing and summed, plus the shared
    expert's row of that token when one is given."""
    from mixture_experts_layer_aux_b200.synthetic import random_routing
    T, E, k, H = 30, 5, 3, 16
    idx = random_routing(T, E, k, seed=7)
    _, _, row_of, _ = oracle.maps(idx, E)
    g = torch.Generator().manual_seed(8)
    o = torch.randn(T * k, H, generator=g, dtype=torch.float64)
    sh = torch.randn(T, H, generator=g, dtype=torch.float64)
    gathered = o[row_of.long()].sum(1)
    assert torch.allclose(oracle.unpermute(o, row_of), gathered, rtol=1e-14, atol=1e-14)
    assert torch.allclose(oracle.unpermute(o, row_of, sh), gathered + sh, rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------- experts


def test_single_expert_is_plain_swiglu_mlp(oracle):
    wl = small(T=9, H=64, E=1, k=1, F=96)
    inp = make_inputs(wl, seed=4)
    r = oracle.layer_fwd(wl, inp)
    assert torch.equal(r["idx"], torch.zeros(9, 1, dtype=torch.int32))
    assert torch.allclose(r["gates"], torch.ones(9, 1, dtype=torch.float64))
    ref = ref_swiglu(inp["x"].double(), inp["W_g"][0].double(), inp["W_u"][0].double(), inp["W_d"][0].double())
    assert torch.allclose(r["y"], ref, rtol=1e-12, atol=1e-14)


def test_k_equals_E_is_dense_softmax_mixture(oracle):
    wl = small(T=11, H=32, E=4, k=4, F=64)
    inp = make_inputs(wl, seed=5)
    r = oracle.layer_fwd(wl, inp)
    l = r["logits"]
    p = torch.softmax(l, 1)
    ref = torch.zeros(11, 32, dtype=torch.float64)
    for e in range(4):
        ref += p[:, e:e + 1] * ref_swiglu(inp["x"].double(), inp["W_g"][e].double(), inp["W_u"][e].double(),
                                          inp["W_d"][e].double())
    assert torch.allclose(r["y"], ref, rtol=1e-12, atol=1e-14)


def test_per_token_loop_equals_dense_masked_brute_force(oracle):
    wl = small(T=30, H=64, E=6, k=2, F=96)
    inp = make_inputs(wl, seed=6)
    r = oracle.layer_fwd(wl, inp)
    gd = torch.zeros(wl.T, wl.E, dtype=torch.float64)
    gd.scatter_(1, r["idx"].long(), r["gates"])
    yd = oracle.moe_fwd_dense(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], gd)
    assert torch.allclose(r["y"], yd, rtol=1e-12, atol=1e-13)


def test_fold_before_down_projection_equals_after(oracle):
    wl = small(T=20, H=64, E=5, k=3, F=96)
    inp = make_inputs(wl, seed=7)
    r = oracle.layer_fwd(wl, inp)
    y_fold = oracle.moe_fwd_tokens(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], r["idx"], r["gates"], fold=True)
    y_post = oracle.moe_fwd_tokens(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], r["idx"], r["gates"], fold=False)
    assert torch.allclose(y_fold, y_post, rtol=1e-12, atol=1e-13)
    # ...and the fold really changes the intermediate (g applied): ap = g * a
    assert not torch.equal(y_fold, torch.zeros_like(y_fold))


def test_row_stage_composes_to_per_token_loop(oracle):
    """permute (gather by src_of) -> per-row expert stage -> unpermute-sum equals the per-token loop."""
    wl = small(T=25, H=64, E=5, k=2, F=64)
    inp = make_inputs(wl, seed=8)
    r = oracle.layer_fwd(wl, inp)
    off = r["offsets"].long()
    e_of = torch.bucketize(torch.arange(wl.T * wl.k), off[1:], right=True).to(torch.int32)
    g_of = torch.empty(wl.T * wl.k, dtype=torch.float64)
    g_of[r["row_of"].flatten().long()] = r["gates"].flatten()
    xp = inp["x"][r["src_of"].long()].contiguous()
    st = oracle.expert_rows(xp, e_of, g_of, inp["W_g"], inp["W_u"], inp["W_d"])
    y = oracle.unpermute(st["o"], r["row_of"])
    assert torch.allclose(y, r["y"], rtol=1e-13, atol=1e-14)


def test_shared_expert_adds_plain_mlp(oracle):
    wl = small(T=10, H=64, E=4, k=2, F=64, S=1, score="sigmoid", route_scale=2.5, aux=False)
    inp = make_inputs(wl, seed=9)
    r = oracle.layer_fwd(wl, inp)
    y0 = oracle.moe_fwd_tokens(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], r["idx"], r["gates"])
    sh = ref_swiglu(inp["x"].double(), inp["W_gs"].double(), inp["W_us"].double(), inp["W_ds"].double())
    assert torch.allclose(r["y"], y0 + sh, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------- MXFP8


def _golden():
    elems, scales, blocks = [], [], []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        tag, rest = line.split(" ", 1)
        if tag == "elem":
            v, c = rest.split()
            elems.append((float(v), int(c, 16)))
        elif tag == "scale":
            a, b = rest.split()
            scales.append((float(a), int(b)))
        elif tag == "block":
            head, tail = rest.split(" : ")
            name, byte = head.split()
            vals, codes = tail.split(" => ")
            blocks.append((name, int(byte), [float(v) for v in vals.split()], [int(c, 16) for c in codes.split()]))
    return elems, scales, blocks


def test_mxfp8_golden_elements_and_scales(oracle):
    elems, scales, _ = _golden()
    assert len(elems) > 20 and len(scales) > 5
    for v, c in elems:
        assert oracle.e4m3_encode(v) == c, (v, hex(oracle.e4m3_encode(v)), hex(c))
    for a, b in scales:
        assert oracle.mx_scale_byte(a) == b, (a, oracle.mx_scale_byte(a), b)


def test_mxfp8_golden_blocks(oracle):
    _, _, blocks = _golden()
    for name, byte, vals, codes in blocks:
        v = torch.zeros(1, 32, dtype=torch.float32)
        v[0, :len(vals)] = torch.tensor(vals, dtype=torch.float32)
        q, s = oracle.mxfp8_quantize(v)
        assert int(s[0, 0]) == byte, name
        exp = codes + [0] * (32 - len(codes))
        assert q[0].tolist() == exp, (name, [hex(c) for c in q[0].tolist()])


def test_e4m3_decode_matches_torch_float8(oracle):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64)
    mine = torch.tensor([oracle.e4m3_decode(c) for c in range(256)], dtype=torch.float64)
    nan = torch.isnan(ref)
    assert torch.equal(torch.isnan(mine), nan)
    assert torch.equal(mine[~nan], ref[~nan])


def test_e4m3_encode_matches_torch_cast_in_range(oracle):
    g = torch.Generator().manual_seed(0)
    v = (torch.rand(4000, generator=g, dtype=torch.float64) * 2 - 1) * 448.0
    v = torch.cat([v, v * 1e-3, torch.tensor([0.0009765625, 0.0029296875, 1.0625, 1.1875, 15.5, -0.3])])
    v32 = v.float()
    ref = v32.to(torch.float8_e4m3fn).view(torch.uint8)
    mine = torch.tensor([oracle.e4m3_encode(float(x)) for x in v32], dtype=torch.uint8)
    assert torch.equal(mine, ref)


def test_mxfp8_roundtrip_error_bound(oracle):
    g = torch.Generator().manual_seed(1)
    v = torch.randn(64, 256, generator=g) * torch.logspace(-6, 6, 64).unsqueeze(1)
    q, s = oracle.mxfp8_quantize(v)
    dq = oracle.mxfp8_decode(q, s)
    X = torch.pow(2.0, s.double() - 127.0).repeat_interleave(32, 1)
    a = (v.double() / X).abs()
    assert (a < 512).all()                                   # scale puts amax in [256, 512)
    blk_amax = a.view(64, 8, 32).amax(-1)
    assert ((blk_amax >= 256) & (blk_amax < 512)).all()
    e = torch.floor(torch.log2(a.clamp_min(2.0 ** -9))).clamp_min(-6)
    half_ulp = torch.pow(2.0, e - 4) * X
    err = (dq - v.double()).abs()
    inrange = a <= 448
    assert (err[inrange] <= half_ulp[inrange] * (1 + 1e-12)).all()
    assert torch.equal(dq[~inrange].abs(), 448.0 * X[~inrange])


def test_mxfp8_bf16_and_fp32_entry_points_agree(oracle):
    g = torch.Generator().manual_seed(2)
    v = (torch.randn(16, 128, generator=g) * 0.02).bfloat16()
    a = oracle.mxfp8_quantize(v)
    b = oracle.mxfp8_quantize(v.float())
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# --------------------------------------------------------------- group-limited routing (DeepSeek-V3 variant)


def _torch_grouped_topk(sel, k, n_group, topk_group):
    """The same rule with library sorts: group score = sum of the two largest in the group;
    the topk_group best groups (stable descending sort: lower index first on ties); then the
    k best experts of those groups."""
    T, E = sel.shape
    G = E // n_group
    grp = sel.view(T, n_group, G)
    gscore = torch.topk(grp, min(2, G), dim=-1).values.sum(-1)
    gorder = torch.sort(-gscore, dim=1, stable=True).indices[:, :topk_group]
    mask = torch.zeros(T, n_group, dtype=torch.bool)
    mask.scatter_(1, gorder, True)
    v = torch.where(mask.repeat_interleave(G, dim=1), sel, torch.full_like(sel, -float("inf")))
    return torch.sort(-v, dim=1, stable=True).indices[:, :k].to(torch.int32)


@pytest.mark.parametrize("E,n_group,topk_group,k", [(16, 4, 2, 3), (32, 8, 4, 8), (12, 3, 1, 2), (8, 8, 3, 3)])
def test_grouped_topk_matches_library_sorts(oracle, E, n_group, topk_group, k):
    g = torch.Generator().manual_seed(E + k)
    sel = torch.rand(64, E, generator=g, dtype=torch.float64)
    sel[::7, :] = torch.round(sel[::7, :] * 4) / 4            # some rows with many exact ties
    idx = oracle.topk_grouped(sel, k, n_group, topk_group)
    assert torch.equal(idx, _torch_grouped_topk(sel, k, n_group, topk_group))


def test_grouped_topk_without_groups_or_bias_is_plain_topk(oracle):
    l = random_logits(50, 16, seed=8).double()
    s = oracle.scores(l, "sigmoid")
    assert torch.equal(oracle.topk_grouped(s, 4, 0, 0), oracle.topk(l, 4))    # sigmoid is increasing
    assert torch.equal(oracle.topk_grouped(s, 4, 4, 4), oracle.topk(l, 4))    # every group kept


def test_selection_bias_moves_selection_not_gates(oracle):
    l = random_logits(40, 16, seed=9).double()
    b = torch.zeros(16, dtype=torch.float64)
    b[5] = 10.0                                               # expert 5 wins every token's selection
    r = oracle.route(l, 3, "sigmoid", True, 2.5, with_aux=False, expert_bias=b)
    assert bool((r["idx"][:, 0] == 5).all())
    s = torch.sigmoid(l)                                      # gates from the unbiased scores
    ref = s.gather(1, r["idx"].long())
    ref = ref / ref.sum(1, keepdim=True) * 2.5
    assert torch.allclose(r["gates"], ref, rtol=1e-13, atol=0)


# --------------------------------------------------------------- capacity factor


def _stable_rank_within_expert(idx, E):
    """Position of each (t, j) among its expert's pairs in token order, by a library stable sort."""
    flat = idx.flatten().long()
    order = torch.sort(flat, stable=True).indices
    counts = torch.bincount(flat, minlength=E)
    starts = torch.cumsum(counts, 0) - counts
    rank = torch.empty_like(flat)
    rank[order] = torch.arange(flat.numel()) - starts[flat[order]]
    return rank.view(idx.shape), counts


@pytest.mark.parametrize("cf", [0.5, 0.77, 1.0, 1.25, 100.0])   # 0.77: cf T k / E = 15.4, so C rounds up
def test_capacity_keep_matches_stable_sort_rank_and_maps_invariants(oracle, cf):
    from mixture_experts_layer_aux_b200.synthetic import random_routing
    T, E, k = 60, 6, 2
    idx = random_routing(T, E, k, seed=3, hot=0.6)
    keep, C = oracle.capacity_keep(idx, E, cf)
    cf32 = float(torch.tensor(cf, dtype=torch.float32))  # the configuration carries cf as float32
    assert C == min(T * k, math.ceil(cf32 * T * k / E))
    rank, counts = _stable_rank_within_expert(idx, E)
    assert torch.equal(keep.bool(), rank < C)
    kc, off, row_of, src_of = oracle.maps(idx, E, keep)
    assert torch.equal(kc.long(), torch.clamp(counts, max=C))
    assert int(off[-1]) == int(kc.sum())
    kept = keep.bool()
    assert bool((row_of[~kept] == -1).all())
    rows = row_of[kept].long()
    assert torch.equal(torch.sort(rows).values, torch.arange(int(off[-1])))      # a bijection onto the kept rows
    tok = torch.arange(T).unsqueeze(1).expand(T, k)
    assert torch.equal(src_of[rows].long(), tok[kept])
    # a kept row sits in its expert's segment at its rank
    e = idx[kept].long()
    assert torch.equal(rows, off[e].long() + rank[kept])
    if cf >= 100.0:                                                              # no drops: the dropless maps
        c0, o0, r0, s0 = oracle.maps(idx, E)
        assert torch.equal(row_of, r0) and torch.equal(off, o0)


def test_capacity_forward_equals_dense_brute_force_without_dropped_pairs(oracle):
    """y with capacity = the dense all-experts mixture whose gate matrix is zero at dropped pairs."""
    wl = small(T=40, H=64, E=4, k=2, F=96, capacity_factor=0.75)
    inp = make_inputs(wl, seed=21)
    r = oracle.layer_fwd(wl, inp)
    assert r["keep"] is not None and int((r["keep"] == 0).sum()) > 0            # some pairs are dropped
    gd = torch.zeros(wl.T, wl.E, dtype=torch.float64)
    gd.scatter_(1, r["idx"].long(), r["gates"] * r["keep"].double())
    yd = oracle.moe_fwd_dense(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], gd)
    assert torch.allclose(r["y"], yd, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------- backward


def _fd_setup(score, norm, scale, aux_on, seed=0, T=8, H=16, E=4, k=2, F=32):
    g = torch.Generator().manual_seed(seed)
    t = dict(
        x=torch.randn(T, H, generator=g, dtype=torch.float64),
        W_r=torch.randn(E, H, generator=g, dtype=torch.float64) * 0.4,
        W_g=torch.randn(E, F, H, generator=g, dtype=torch.float64) * 0.3,
        W_u=torch.randn(E, F, H, generator=g, dtype=torch.float64) * 0.3,
        W_d=torch.randn(E, H, F, generator=g, dtype=torch.float64) * 0.3,
        dY=torch.randn(T, H, generator=g, dtype=torch.float64),
    )
    cfg = dict(k=k, score=score, norm=norm, scale=scale, aux_on=aux_on, d_aux=0.7 if aux_on else 0.0)
    return t, cfg


def _loss(o, t, cfg, logits=None):
    if logits is None:
        logits = o.router_logits(t["x"], t["W_r"], None, round_f32=False)
    r = o.route(logits, cfg["k"], cfg["score"], cfg["norm"], cfg["scale"], with_aux=cfg["aux_on"],
                capacity_factor=cfg.get("cf", 0.0), expert_bias=cfg.get("expert_bias"),
                n_group=cfg.get("n_group", 0), topk_group=cfg.get("topk_group", 0))
    y = o.moe_fwd_tokens(t["x"], t["W_g"], t["W_u"], t["W_d"], r["idx_kept"], r["gates"])
    L = (t["dY"] * y).sum().item()
    if cfg["aux_on"]:
        L += cfg["d_aux"] * r["aux"]
    return L, r


@pytest.mark.parametrize("score,norm,scale,aux_on,cf", [("softmax", True, 1.0, True, 0.0),
                                                        ("sigmoid", True, 2.5, False, 0.0),
                                                        ("softmax", False, 1.0, True, 0.0),
                                                        ("softmax", True, 1.0, True, 0.75)])
def test_backward_matches_central_finite_differences(oracle, score, norm, scale, aux_on, cf):
    t, cfg = _fd_setup(score, norm, scale, aux_on)
    cfg["cf"] = cf
    r = _fd_check(oracle, t, cfg)
    if cf > 0:
        assert int((r["keep"] == 0).sum()) > 0                                  # the case drops pairs


@pytest.mark.parametrize("norm,n_group,topk_group", [(True, 4, 2), (False, 4, 2), (True, 0, 0)])
def test_backward_deepseek_router_matches_central_finite_differences(oracle, norm, n_group, topk_group):
    """Sigmoid scores, selection on score + per-expert bias within the best groups, gates from the
    unbiased scores: the bias and the group limit move the selection only, so the derivative at a
    fixed selection is the sigmoid router's."""
    t, cfg = _fd_setup("sigmoid", norm, 2.5, False, seed=5, E=8, k=3)
    cfg.update(expert_bias=torch.tensor([0.3, -0.2, 0.0, 0.5, -0.4, 0.1, 0.25, -0.1]), n_group=n_group,
               topk_group=topk_group)
    r = _fd_check(oracle, t, cfg)
    plain = oracle.route(r["logits"], 3, "sigmoid", norm, 2.5, with_aux=False)
    assert not torch.equal(r["idx"], plain["idx"])                             # the variant changes selection


def _fd_check(o, t, cfg):
    """Analytic gradients of the oracle's backward against central differences of its forward loss, on
    inputs and weights, and on the logits themselves; entries whose perturbation changes the selection
    are skipped. Returns the routing at the unperturbed point."""
    score, norm, scale, aux_on = cfg["score"], cfg["norm"], cfg["scale"], cfg["aux_on"]
    L0, r = _loss(o, t, cfg)
    E = t["W_r"].shape[0]
    dx, dl, dg = o.moe_bwd_tokens(t["x"], t["W_r"], t["W_g"], t["W_u"], t["W_d"], t["dY"], r, score=score,
                                  norm=norm, route_scale=scale, aux_on=aux_on, d_aux=cfg["d_aux"])
    dWg, dWu, dWd = o.moe_bwd_expert_dw(t["x"], t["W_g"], t["W_u"], t["W_d"], t["dY"], r["idx_kept"], r["gates"],
                                        list(range(E)))
    dWr = o.router_dwr(dl, t["x"])
    grads = dict(x=dx, W_r=dWr, W_g=dWg, W_u=dWu, W_d=dWd)
    h = 1e-6
    g = torch.Generator().manual_seed(11)
    checked = 0
    for name, G in grads.items():
        P = t[name]
        flat = P.view(-1)
        for i in torch.randperm(flat.numel(), generator=g)[:12].tolist():
            old = flat[i].item()
            flat[i] = old + h
            Lp, rp = _loss(o, t, cfg)
            flat[i] = old - h
            Lm, rm = _loss(o, t, cfg)
            flat[i] = old
            if not (torch.equal(rp["idx"], r["idx"]) and torch.equal(rm["idx"], r["idx"])):
                continue                              # selection changed: not differentiable here
            fd = (Lp - Lm) / (2 * h)
            an = G.reshape(-1)[i].item()
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, fd, an)
            checked += 1
    assert checked >= 40
    # dlogits against finite differences in the logits themselves
    l0 = o.router_logits(t["x"], t["W_r"], None, round_f32=False)
    for tt in range(l0.shape[0]):
        for e in range(E):
            lp = l0.clone(); lp[tt, e] += h
            lm = l0.clone(); lm[tt, e] -= h
            Lp, rp = _loss(o, t, cfg, lp)
            Lm, rm = _loss(o, t, cfg, lm)
            if not (torch.equal(rp["idx"], r["idx"]) and torch.equal(rm["idx"], r["idx"])):
                continue
            fd = (Lp - Lm) / (2 * h)
            assert abs(fd - dl[tt, e].item()) <= 1e-6 * max(1.0, abs(fd)), (tt, e, fd, dl[tt, e].item())
    return r


def test_zero_token_expert_gets_exact_zero_weight_grads(oracle):
    from mixture_experts_layer_aux_b200.synthetic import random_routing
    wl = small(T=12, H=32, E=5, k=2, F=32)
    inp = make_inputs(wl, seed=12, with_dy=True)
    idx = random_routing(12, 5, 2, seed=1, zero_experts=2)
    gts = torch.full((12, 2), 0.5, dtype=torch.float64)
    dWg, dWu, dWd = oracle.moe_bwd_expert_dw(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], idx, gts,
                                             [3, 4, 0])
    assert (dWg[:2] == 0).all() and (dWu[:2] == 0).all() and (dWd[:2] == 0).all()
    assert dWd[2].abs().sum() > 0


def test_weight_grad_of_down_is_gated_outer_product_sum(oracle):
    """dW_d[e] = sum over e's tokens of g * dY_t (x) a_t, checked with torch fp64."""
    wl = small(T=14, H=32, E=3, k=2, F=32)
    inp = make_inputs(wl, seed=13, with_dy=True)
    r = oracle.layer_fwd(wl, inp)
    _, _, dWd = oracle.moe_bwd_expert_dw(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], r["idx"],
                                         r["gates"], [1])
    x, dY = inp["x"].double(), inp["dY"].double()
    ref = torch.zeros(32, 32, dtype=torch.float64)
    for t in range(14):
        for j in range(2):
            if int(r["idx"][t, j]) == 1:
                a = torch.nn.functional.silu(x[t] @ inp["W_g"][1].double().T) * (x[t] @ inp["W_u"][1].double().T)
                ref += r["gates"][t, j] * torch.outer(dY[t], a)
    assert torch.allclose(dWd[0], ref, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------- precision recipes


def test_bf16_round_matches_torch_cast(oracle):
    g = torch.Generator().manual_seed(3)
    v = torch.randn(5000, generator=g, dtype=torch.float64) * torch.logspace(-30, 30, 5000, dtype=torch.float64)
    # exact ties of the fp32 -> bf16 step: low 16 bits of the fp32 pattern = 0x8000
    ties = (torch.randint(0, 2 ** 15, (200,), generator=g, dtype=torch.int32) * 65536 + 32768).view(torch.float32)
    v = torch.cat([v, ties.double(), torch.tensor([0.0, -0.0, 1.0, -3.5, 65504.0])])
    ref = v.float().bfloat16().double()
    mine = torch.tensor([oracle.bf16_round(float(x)) for x in v], dtype=torch.float64)
    assert torch.equal(mine, ref)


def test_bf16_recipe_rounds_operand_and_output(oracle):
    """ap is the bf16 value of the exact g*silu(zg)*zu; o is the bf16 value of W_d ap
    (torch fp64 matmul as the library routine)."""
    from mixture_experts_layer_aux_b200.synthetic import random_gates, randn_bf16
    R, H, F, E = 40, 64, 96, 3
    xp = randn_bf16((R, H), 1.0, seed=1)
    e_of = torch.arange(R, dtype=torch.int32) % E
    g = random_gates(R, 1, seed=2).flatten().double()
    Wg, Wu, Wd = (randn_bf16((E, F, H), 0.02, seed=3), randn_bf16((E, F, H), 0.02, seed=4),
                  randn_bf16((E, H, F), 0.02, seed=5))
    ex = oracle.expert_rows(xp, e_of, g, Wg, Wu, Wd, want=("ap", "o"))
    b = oracle.expert_rows(xp, e_of, g, Wg, Wu, Wd, recipe="bf16", want=("zg", "ap", "o"))
    assert torch.equal(b["ap"], ex["ap"].float().bfloat16().double())
    o_ref = torch.stack([Wd[int(e_of[r])].double() @ b["ap"][r] for r in range(R)])
    assert torch.allclose(b["o"], o_ref.float().bfloat16().double(), rtol=0, atol=0) or \
        (b["o"] - o_ref.float().bfloat16().double()).abs().max() <= 2.0 ** -8 * o_ref.abs().max()
    assert not torch.equal(b["o"], ex["o"])


def test_bf16_recipe_forward_composes_and_stays_near_exact(oracle):
    wl = small(T=25, H=64, E=5, k=2, F=64)
    inp = make_inputs(wl, seed=8)
    r = oracle.layer_fwd(wl, inp)
    yb = oracle.moe_fwd_tokens(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], r["idx"], r["gates"], recipe="bf16")
    off = r["offsets"].long()
    e_of = torch.bucketize(torch.arange(wl.T * wl.k), off[1:], right=True).to(torch.int32)
    g_of = torch.empty(wl.T * wl.k, dtype=torch.float64)
    g_of[r["row_of"].flatten().long()] = r["gates"].flatten()
    xp = inp["x"][r["src_of"].long()].contiguous()
    st = oracle.expert_rows(xp, e_of, g_of, inp["W_g"], inp["W_u"], inp["W_d"], recipe="bf16")
    assert torch.allclose(oracle.unpermute(st["o"], r["row_of"]), yb, rtol=1e-14, atol=1e-15)
    rms = r["y"].pow(2).mean().sqrt()
    assert (yb - r["y"]).abs().max() <= 0.02 * rms


def test_bf16_recipe_backward_stays_near_exact(oracle):
    wl = small(T=30, H=64, E=4, k=2, F=64)
    inp = make_inputs(wl, seed=9, with_dy=True)
    r = oracle.layer_fwd(wl, inp)
    args = (inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], r)
    dx0, dl0, _ = oracle.moe_bwd_tokens(*args, d_aux=0.3)
    dx1, dl1, _ = oracle.moe_bwd_tokens(*args, d_aux=0.3, recipe="bf16")
    for a, b in ((dx0, dx1), (dl0, dl1)):
        rms = a.pow(2).mean().sqrt()
        assert 0 < (a - b).abs().max() <= 0.03 * rms
    w0 = oracle.moe_bwd_expert_dw(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], r["idx"], r["gates"], [0, 1])
    w1 = oracle.moe_bwd_expert_dw(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], r["idx"], r["gates"], [0, 1],
                                  recipe="bf16")
    for a, b in zip(w0, w1):
        rms = a.pow(2).mean().sqrt()
        assert 0 < (a - b).abs().max() <= 0.03 * rms
    # the router-gradient operand: dl rounded to bf16
    d_r = oracle.router_dwr(dl0, inp["x"], round_dl=True)
    assert torch.allclose(d_r, dl0.float().bfloat16().double().T @ inp["x"].double(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------- MXFP8 backward


def _mxq(t):
    """MXFP8 round trip along the last dim (fp32 in), with the pinned quantiser."""
    c, s = oracle_mod().mxfp8_quantize(t.float().contiguous())
    return oracle_mod().mxfp8_decode(c, s)


def _mxq_rows(t):
    """MXFP8 round trip along dim 0 in blocks of 32 rows (zero-padded at the end)."""
    n = t.shape[0]
    pad = (-n) % 32
    tp = torch.cat([t, torch.zeros(pad, t.shape[1], dtype=t.dtype)]) if pad else t
    return _mxq(tp.T.contiguous()).T[:n]


def oracle_mod():
    import oracle
    return oracle


def _mx_bwd_case(seed=31):
    wl = small(T=40, H=64, E=3, k=2, F=64, bwd=True)
    inp = make_inputs(wl, seed=seed, with_dy=True)
    o = oracle_mod()
    mx = {n: o.mxfp8_quantize(inp[n]) for n in ("W_g", "W_u", "W_d")}
    mx["W_dT"] = o.mxfp8_quantize(inp["W_d"].transpose(1, 2).contiguous())
    mx["W_gT"] = o.mxfp8_quantize(inp["W_g"].transpose(1, 2).contiguous())
    mx["W_uT"] = o.mxfp8_quantize(inp["W_u"].transpose(1, 2).contiguous())
    return wl, inp, mx


@pytest.mark.parametrize("recipe", ["mxfp8", "mxfp8-q"])
def test_mxfp8_forward_composes_from_quantised_operands(oracle, recipe):
    """recipe mxfp8 = fp64 products of x rounded to MXFP8 along H, the MXFP8 weights, the gate-folded
    activation (and the shared expert's activation) rounded to MXFP8 along F, and bf16 expert outputs
    (torch fp64 + the pinned quantiser; a missing rounding point fails it). mxfp8-q: the same MXFP8
    quantisation points with unrounded expert outputs."""
    wl = small(T=16, H=64, E=4, k=2, F=64, S=1)
    inp = make_inputs(wl, seed=45)
    r = oracle.route(oracle.router_logits(inp["x"], inp["W_r"]), wl.k, "softmax", True, 1.0)
    names = ("W_g", "W_u", "W_d", "W_gs", "W_us", "W_ds")
    mx = {n: oracle.mxfp8_quantize(inp[n]) for n in names}
    y = oracle.moe_fwd_tokens(inp["x"], mx["W_g"][0], mx["W_u"][0], mx["W_d"][0], r["idx"], r["gates"],
                              recipe=recipe, sf_g=mx["W_g"][1], sf_u=mx["W_u"][1], sf_d=mx["W_d"][1],
                              shared=(mx["W_gs"][0], mx["W_us"][0], mx["W_ds"][0], mx["W_gs"][1], mx["W_us"][1],
                                      mx["W_ds"][1]))
    dec = {n: oracle.mxfp8_decode(*mx[n]) for n in names}
    xq = _mxq(inp["x"].double())
    silu = torch.nn.functional.silu
    bf = (lambda t: t) if recipe.endswith("-q") else (lambda t: t.float().bfloat16().double())  # noqa: E731
    ref = torch.zeros(wl.T, wl.H, dtype=torch.float64)
    for t in range(wl.T):
        for j in range(wl.k):
            e = int(r["idx"][t, j])
            zg, zu = dec["W_g"][e] @ xq[t], dec["W_u"][e] @ xq[t]
            ap = _mxq(((silu(zg) * zu) * float(r["gates"][t, j])).unsqueeze(0))[0]
            ref[t] += bf(dec["W_d"][e] @ ap)
        zg, zu = dec["W_gs"] @ xq[t], dec["W_us"] @ xq[t]
        ref[t] += bf(dec["W_ds"] @ _mxq((silu(zg) * zu).unsqueeze(0))[0])
    assert torch.allclose(y, ref, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("recipe", ["mxfp8", "mxfp8-q"])
def test_mxfp8_backward_composes_from_quantised_operands(oracle, recipe):
    """The MXFP8 backward equals fp64 products of the operands rounded at the recipe's points:
    dY and x along H, W_d^T along H, dgate/dup to bf16 then along F, W_g^T / W_u^T along F, and
    for the weight gradients every operand along the expert's tokens (torch fp64 + the pinned
    quantiser; a transposed operand or a missing rounding point fails it). mxfp8-q: the same MXFP8
    quantisation points, with none of the bf16 roundings (saved z, dgate/dup, dXp, router path)."""
    wl, inp, mx = _mx_bwd_case()
    r = oracle.route(oracle.router_logits(inp["x"], inp["W_r"]).double(), wl.k, with_aux=False)
    dx, dl, dg = oracle.moe_bwd_tokens(inp["x"], inp["W_r"], None, None, None, inp["dY"], r, aux_on=False,
                                       recipe=recipe, mx=mx)
    dWg, dWu, dWd = oracle.moe_bwd_expert_dw(inp["x"], None, None, None, inp["dY"], r["idx"], r["gates"],
                                             list(range(wl.E)), recipe=recipe, mx=mx)
    dec = {n: oracle.mxfp8_decode(*mx[n]) for n in mx}
    x, dY = inp["x"].double(), inp["dY"].double()
    xq, dYq = _mxq(x), _mxq(dY)
    bf = (lambda t: t) if recipe.endswith("-q") else (lambda t: t.float().bfloat16().double())
    silu = torch.nn.functional.silu
    ref_dx = torch.zeros_like(x)
    rows = {e: [] for e in range(wl.E)}
    for t in range(wl.T):
        for j in range(wl.k):
            e, g = int(r["idx"][t, j]), float(r["gates"][t, j])
            zg, zu = bf(xq[t] @ dec["W_g"][e].T), bf(xq[t] @ dec["W_u"][e].T)
            v = dec["W_dT"][e] @ dYq[t]
            sg = torch.sigmoid(zg)
            dzg = bf(g * v * zu * sg * (1 + zg * (1 - sg)))
            dzu = bf(g * v * silu(zg))
            assert abs(float(v @ (silu(zg) * zu)) - float(dg[t, j])) <= 1e-12 * max(1.0, abs(float(dg[t, j])))
            ref_dx[t] += bf(dec["W_gT"][e] @ _mxq(dzg[None])[0] + dec["W_uT"][e] @ _mxq(dzu[None])[0])
            rows[e].append((t, g * silu(zg) * zu, dzg, dzu))
    router = bf(bf(dl) @ inp["W_r"].double())                 # the router path, rounded as under bf16
    assert torch.allclose(dx, ref_dx + router, rtol=0, atol=1e-12)
    for e in range(wl.E):
        ts = torch.tensor([q[0] for q in rows[e]])
        A = _mxq_rows(torch.stack([q[1] for q in rows[e]]))
        DZG = _mxq_rows(torch.stack([q[2] for q in rows[e]]))
        DZU = _mxq_rows(torch.stack([q[3] for q in rows[e]]))
        X, DY = _mxq_rows(x[ts]), _mxq_rows(dY[ts])
        assert torch.allclose(dWd[e], DY.T @ A, rtol=1e-12, atol=1e-13)
        assert torch.allclose(dWg[e], DZG.T @ X, rtol=1e-12, atol=1e-13)
        assert torch.allclose(dWu[e], DZU.T @ X, rtol=1e-12, atol=1e-13)


def test_mxfp8_backward_stays_near_exact(oracle):
    wl, inp, mx = _mx_bwd_case(seed=32)
    r = oracle.route(oracle.router_logits(inp["x"], inp["W_r"]).double(), wl.k, with_aux=False)
    args = (inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], r)
    dx_e, _, _ = oracle.moe_bwd_tokens(*args, aux_on=False)
    dx_m, _, _ = oracle.moe_bwd_tokens(*args, aux_on=False, recipe="mxfp8", mx=mx)
    gw_e = oracle.moe_bwd_expert_dw(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], r["idx"], r["gates"],
                                    [0, 1, 2])
    gw_m = oracle.moe_bwd_expert_dw(inp["x"], None, None, None, inp["dY"], r["idx"], r["gates"], [0, 1, 2],
                                    recipe="mxfp8", mx=mx)
    rms = lambda t: float(t.pow(2).mean().sqrt())
    assert rms(dx_m - dx_e) <= 0.08 * rms(dx_e)
    for a, b in zip(gw_m, gw_e):
        assert rms(a - b) <= 0.12 * rms(b)


# --------------------------------------------------------------- NVFP4

GOLDEN_NV = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_cases.txt")


def _golden_nv():
    elems, scales, blocks = [], [], []
    with open(GOLDEN_NV) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            kind, rest = line.split(None, 1)
            if kind == "elem":
                v, c = rest.split()
                elems.append((float(v), int(c, 16)))
            elif kind == "scale":
                a, G, b = rest.split()
                scales.append((float(a), float(G), int(b, 16)))
            else:
                head, tail = rest.split(" : ")
                name, G, byte = head.split()
                vals, codes = tail.split(" => ")
                blocks.append((name, float(G), int(byte, 16), [float(v) for v in vals.split()],
                               [int(c, 16) for c in codes.split()]))
    return elems, scales, blocks


def test_nvfp4_golden_elements_and_scales(oracle):
    elems, scales, _ = _golden_nv()
    assert len(elems) > 20 and len(scales) > 5
    for v, c in elems:
        assert oracle.e2m1_encode(v) == c, (v, hex(oracle.e2m1_encode(v)), hex(c))
    for a, G, b in scales:
        assert oracle.nvfp4_scale_byte(a, G) == b, (a, G, hex(oracle.nvfp4_scale_byte(a, G)), hex(b))


def _nv_quantize_block(vals, G):
    """One 16-block through the oracle's matrix quantiser with a given G (via a 1-matrix tensor)."""
    import oracle
    v = torch.zeros(1, 16, dtype=torch.float32)
    v[0, :len(vals)] = torch.tensor(vals, dtype=torch.float32)
    packed = torch.empty(1, 8, dtype=torch.uint8)
    sc = torch.empty(1, 1, dtype=torch.uint8)
    src = v.bfloat16()
    assert torch.equal(src.float(), v), "golden block values must be exact in bf16"
    oracle.lib().oc_nvfp4_quantize_bf16(1, 16, oracle._p(src), float(G), oracle._p(packed), oracle._p(sc))
    codes = torch.stack([packed[0] & 15, packed[0] >> 4], dim=-1).flatten().tolist()
    return int(sc[0, 0]), codes


def test_nvfp4_golden_blocks(oracle):
    _, _, blocks = _golden_nv()
    for name, G, byte, vals, codes in blocks:
        sb, got = _nv_quantize_block(vals, G)
        assert sb == byte, (name, hex(sb), hex(byte))
        assert got == codes + [0] * (16 - len(codes)), (name, got)


def test_e2m1_decode_is_the_ocp_value_table(oracle):
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert [oracle.e2m1_decode(c) for c in range(8)] == mags
    assert [oracle.e2m1_decode(8 + c) for c in range(8)] == [-m for m in mags]


def _e2m1_generic(u: torch.Tensor) -> torch.Tensor:
    """Round fp64 magnitudes to a 2-bit-significand float with exponents 0..2 and
    subnormal quantum 0.5, half to even, saturated at 6 (numpy's half-even round)."""
    import numpy as np
    a = np.abs(u.numpy())
    q = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    r = np.minimum(np.round(a / q) * q, 6.0)
    return torch.from_numpy(np.copysign(r, u.numpy()))


def test_e2m1_encode_matches_generic_half_even_rounding(oracle):
    g = torch.Generator().manual_seed(5)
    u = torch.cat([(torch.rand(3000, generator=g, dtype=torch.float64) * 2 - 1) * 7.5,
                   torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 7.0, 0.0])])
    mine = torch.tensor([oracle.e2m1_decode(oracle.e2m1_encode(float(x))) for x in u], dtype=torch.float64)
    assert torch.equal(mine, _e2m1_generic(u))


def test_nvfp4_quantizer_matches_library_casts_and_error_bound(oracle):
    """Scales against torch's float8_e4m3fn cast of (amax/6)*G, elements against the generic
    half-even rounding of v*(G/scale) in fp32; each element within half a grid step of v."""
    g = torch.Generator().manual_seed(6)
    w = (torch.randn(3, 24, 64, generator=g) * torch.tensor([0.02, 1.0, 30.0]).view(3, 1, 1)).bfloat16()
    packed, sc, G = oracle.nvfp4_quantize(w, per_matrix=True)
    assert G.shape == (3,)
    for b in range(3):
        v = w[b].float()
        amax_t = v.abs().max()
        assert float(G[b]) == float(torch.tensor(2688.0, dtype=torch.float32) / amax_t)
        blk = v.view(24, 4, 16)
        s_f = (blk.abs().amax(-1) / 6.0) * G[b]
        ref_sb = s_f.to(torch.float8_e4m3fn)
        assert torch.equal(sc[b].view(24, 4), ref_sb.view(torch.uint8))
        sd = ref_sb.float()
        r = torch.where(sd > 0, G[b] / sd, torch.zeros_like(sd))
        u = (blk * r.unsqueeze(-1)).double()
        dec = oracle.nvfp4_decode(packed[b], sc[b])  # code * scale (G not divided out)
        assert torch.equal(dec.view(24, 4, 16) / sd.double().unsqueeze(-1).clamp_min(1e-300)
                           * (sd.double().unsqueeze(-1) > 0), _e2m1_generic(u) * (sd.double().unsqueeze(-1) > 0))
        # the block holding the tensor's amax gets the largest scale
        assert int(sc[b].max()) == 0x7E
        # round trip within half a grid step (or the saturation gap above 6)
        full = oracle.nvfp4_decode(packed[b], sc[b], G[b]).view(24, 4, 16)
        step = torch.where(u.abs() < 2, 0.5, torch.where(u.abs() < 4, 1.0, 2.0))
        # (+ 1e-6 |u|: u = v * (G / scale) carries fp32 rounding)
        bound = (torch.where(u.abs() <= 6, step / 2, u.abs() - 6) + 1e-6 * u.abs()) \
            * (sd.double() / G[b].double()).unsqueeze(-1)
        assert ((full - blk.double()).abs() <= bound).all()


def test_nvfp4_matrix_decode_in_expert_rows_matches_fp64_weights(oracle):
    """The oracle's NVFP4 matrix reader (nibble order, scale index, G per expert) equals
    the table decode of the same codes fed as fp64 matrices."""
    wl = small(T=10, H=64, E=3, k=2, F=32)
    inp = make_inputs(wl, seed=41)
    nv = {n: oracle.nvfp4_quantize(inp[n], per_matrix=True) for n in ("W_g", "W_u", "W_d")}
    dec = {n: oracle.nvfp4_decode(*nv[n]) for n in nv}
    xp = inp["x"][torch.arange(10) % 10]
    e_of = torch.tensor([0, 1, 2, 1, 0, 2, 2, 1, 0, 0], dtype=torch.int32)
    g_of = torch.rand(10, dtype=torch.float64)
    a = oracle.expert_rows(xp, e_of, g_of, nv["W_g"][0], nv["W_u"][0], nv["W_d"][0],
                           sf_g=(nv["W_g"][1], nv["W_g"][2]), sf_u=(nv["W_u"][1], nv["W_u"][2]),
                           sf_d=(nv["W_d"][1], nv["W_d"][2]), want=("zg", "zu", "o"))
    b = oracle.expert_rows(xp, e_of, g_of, dec["W_g"], dec["W_u"], dec["W_d"], want=("zg", "zu", "o"))
    for key in ("zg", "zu", "o"):
        assert torch.allclose(a[key], b[key], rtol=1e-12, atol=1e-15), key


def _nv_roundtrip_ref(t: torch.Tensor) -> torch.Tensor:
    """NVFP4 round trip with G = 1 along the last dim, written with torch casts."""
    v = t.float().view(*t.shape[:-1], -1, 16)
    sd = (v.abs().amax(-1) / 6.0).to(torch.float8_e4m3fn).float()
    r = torch.where(sd > 0, 1.0 / sd, torch.zeros_like(sd))
    u = (v * r.unsqueeze(-1)).double()
    return (_e2m1_generic(u) * sd.double().unsqueeze(-1)).view(t.shape)


@pytest.mark.parametrize("recipe", ["nvfp4", "nvfp4-q"])
def test_nvfp4_forward_composes_from_quantised_operands(oracle, recipe):
    """recipe nvfp4 = fp64 products of NVFP4 x (G=1), NVFP4 weights (G per expert),
    the gate-folded activation rounded to NVFP4 (G=1) and bf16 expert outputs;
    nvfp4-q: the same quantisation points with unrounded expert outputs."""
    wl = small(T=16, H=64, E=4, k=2, F=48, S=1)
    inp = make_inputs(wl, seed=43)
    logits = oracle.router_logits(inp["x"], inp["W_r"])
    r = oracle.route(logits, wl.k, "softmax", True, 1.0)
    names = ("W_g", "W_u", "W_d", "W_gs", "W_us", "W_ds")
    nv = {n: oracle.nvfp4_quantize(inp[n], per_matrix=True) for n in names}
    y = oracle.moe_fwd_tokens(inp["x"], nv["W_g"][0], nv["W_u"][0], nv["W_d"][0], r["idx"], r["gates"],
                              recipe=recipe, sf_g=nv["W_g"][1:], sf_u=nv["W_u"][1:], sf_d=nv["W_d"][1:],
                              shared=(nv["W_gs"][0], nv["W_us"][0], nv["W_ds"][0], nv["W_gs"][1:],
                                      nv["W_us"][1:], nv["W_ds"][1:]))
    dec = {n: oracle.nvfp4_decode(*nv[n]) for n in names}
    xq = _nv_roundtrip_ref(inp["x"])
    ref = torch.zeros(wl.T, wl.H, dtype=torch.float64)
    bf = (lambda t: t) if recipe.endswith("-q") else (lambda t: t.float().bfloat16().double())  # noqa: E731
    for t in range(wl.T):
        for j in range(wl.k):
            e = int(r["idx"][t, j])
            zg, zu = dec["W_g"][e] @ xq[t], dec["W_u"][e] @ xq[t]
            ap = _nv_roundtrip_ref(float(r["gates"][t, j]) * torch.nn.functional.silu(zg) * zu)
            ref[t] += bf(dec["W_d"][e] @ ap)
        zg, zu = dec["W_gs"] @ xq[t], dec["W_us"] @ xq[t]
        ref[t] += bf(dec["W_ds"] @ _nv_roundtrip_ref(torch.nn.functional.silu(zg) * zu))
    assert torch.allclose(y, ref, rtol=1e-9, atol=1e-12)


def test_nvfp4_forward_stays_near_exact(oracle):
    """NVFP4 is coarse, but the recipe's output tracks the exact forward (a missing 1/G
    or a misplaced scale would be off by orders of magnitude)."""
    wl = small(T=32, H=128, E=4, k=2, F=64)
    inp = make_inputs(wl, seed=44)
    logits = oracle.router_logits(inp["x"], inp["W_r"])
    r = oracle.route(logits, wl.k, "softmax", True, 1.0)
    nv = {n: oracle.nvfp4_quantize(inp[n], per_matrix=True) for n in ("W_g", "W_u", "W_d")}
    y = oracle.moe_fwd_tokens(inp["x"], nv["W_g"][0], nv["W_u"][0], nv["W_d"][0], r["idx"], r["gates"],
                              recipe="nvfp4", sf_g=nv["W_g"][1:], sf_u=nv["W_u"][1:], sf_d=nv["W_d"][1:])
    y0 = oracle.moe_fwd_tokens(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], r["idx"], r["gates"])
    rms = y0.pow(2).mean().sqrt()
    rel = (y - y0).pow(2).mean().sqrt() / rms
    assert 0.01 < rel < 0.3, float(rel)


def test_nvfp4_bf16_and_fp32_entry_points_agree(oracle):
    g = torch.Generator().manual_seed(7)
    v = (torch.randn(16, 128, generator=g) * 0.5).bfloat16()
    a = oracle.nvfp4_quantize(v)
    b = oracle.nvfp4_quantize(v.float())
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# --------------------------------------------------------------- what a bf16 output can reach


def test_literal_bar_is_out_of_reach_of_a_correctly_rounded_bf16_weight_gradient(oracle):
    """The literal bar max |got - ref| <= 2e-2 rms(ref) cannot be met by any bf16 output of a tensor whose
    largest elements lie far out in its tail: the exact value rounded to bf16 (the best a bf16 output can
    be) already misses it. Shown on the oracle's exact weight gradient of a small expert (a few tokens make
    dW_d a sum of a few outer products, heavy-tailed), with the rounding error inside the bound 2^-8 max|v|
    that the format allows."""
    wl = small(T=64, H=128, E=8, k=2, F=128)
    inp = make_inputs(wl, seed=21, with_dy=True)
    t = torch.arange(64)
    idx = torch.stack([torch.zeros(64, dtype=torch.long), 2 + t % 6], dim=1).to(torch.int32)
    idx[:2, 1] = 1                                           # expert 1 gets two tokens
    g = torch.full((64, 2), 0.5, dtype=torch.float64)
    small_e = 1
    _, _, dWd = oracle.moe_bwd_expert_dw(inp["x"], inp["W_g"], inp["W_u"], inp["W_d"], inp["dY"], idx, g,
                                         [small_e])
    v = dWd[0]
    rms = float(v.pow(2).mean().sqrt())
    rounding = float((v.float().bfloat16().double() - v).abs().max())
    assert rounding <= 2.0 ** -8 * float(v.abs().max())
    assert rounding > 2e-2 * rms, (rounding / rms, float(v.abs().max()) / rms)
