"""The seeded synthetic inputs (no GPU): the recipe's shapes and distributions, its determinism, and the
skewed workload's routing (log-Zipf prior, four experts without tokens), checked with the oracle's router."""
import math

import torch

from mixture_experts_layer_aux_b200.synthetic import WORKLOADS, Workload, make_inputs, skew_bias


def test_recipe_is_deterministic_and_bf16():
    wl = Workload("s", T=64, H=128, E=8, k=2, F=64, S=1, bwd=True, sel_bias=True)
    a, b = make_inputs(wl, seed=5), make_inputs(wl, seed=5)
    c = make_inputs(wl, seed=6)
    for n in ("x", "W_r", "W_g", "W_u", "W_d", "W_gs", "W_us", "W_ds", "dY"):
        assert a[n].dtype == torch.bfloat16 and torch.equal(a[n], b[n]), n
        assert not torch.equal(a[n], c[n]), n
    assert a["W_g"].shape == (8, 64, 128) and a["W_d"].shape == (8, 128, 64) and a["W_ds"].shape == (128, 64)
    assert a["expert_bias"].shape == (8,) and bool((a["expert_bias"].abs() <= 0.1).all())


def test_recipe_distributions():
    wl = Workload("s", T=512, H=512, E=8, k=2, F=256, bwd=True)
    d = make_inputs(wl, seed=1)
    for n, std in (("x", 1.0), ("dY", 1.0), ("W_r", 0.02), ("W_g", 0.02), ("W_u", 0.02), ("W_d", 0.02)):
        v = d[n].double()
        assert abs(v.mean().item()) < 0.02 * std, n
        assert abs(v.std().item() / std - 1.0) < 0.02, n


def test_skew_bias_is_log_zipf_with_four_experts_pushed_out():
    b = skew_bias(128)
    assert b.dtype == torch.float32
    for e in (0, 1, 7, 123):
        assert b[e].item() == torch.tensor(-1.2 * math.log(e + 1.0), dtype=torch.float32).item()
    assert bool((b[124:] == -30.0).all())


def test_skewed_routing_leaves_experts_without_tokens(oracle):
    # the skewed workload's shape at fewer tokens: the pushed-out experts get none, the prior makes the
    # lowest-numbered experts the hottest
    wl = WORKLOADS["skewed"]
    small = Workload("skewed-small", T=1024, H=wl.H, E=wl.E, k=wl.k, F=64, skew=True)
    d = make_inputs(small, seed=0)
    r = oracle.route(oracle.router_logits(d["x"], d["W_r"], d["logit_bias"]), small.k)
    counts = r["counts"]
    assert int(counts.sum()) == small.T * small.k
    assert bool((counts[124:] == 0).all())
    assert int(counts[:8].sum()) > int(counts[64:124].sum())
