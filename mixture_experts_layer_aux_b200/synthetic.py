"""Seeded synthetic inputs for the MoE layer.

This module is shared by the tests, the bench and the oracle harness. It only
draws random tensors with the shapes and distributions of the workloads; it
holds none of the layer's arithmetic (no routing, no expert math).

Workloads (shapes of the models the Megatron-Core MoE pages benchmark; the
pages train on real data, which synthetic tensors of the same shape stand in
for):

  tiny     T=512  H=256  E=8   k=2 F=512   softmax, gates renormalised
  mixtral  T=4096 H=4096 E=8   k=2 F=14336 softmax top-2 renormalised
  qwen3    T=8192 H=4096 E=128 k=8 F=1536  softmax top-8 renormalised + aux loss
  dsv3     T=8192 H=7168 E=256 k=8 F=2048  + 1 shared expert, sigmoid scores,
           selected-normalised x2.5, MXFP8 expert operands (dsv3-nvfp4: the
           same with NVFP4 expert operands)
  skewed   qwen3 shape with a per-expert logit bias (log-Zipf s=1.2, and the
           last four experts pushed out), forward + backward with dY~N(0,1)

Recipe: one torch.Generator seeded with `seed` on the target device; tensors
are drawn in the fixed order x, W_r, W_g, W_u, W_d, [W_gs, W_us, W_ds], [dY],
each in fp32 and cast to bf16 with round-to-nearest-even. x~N(0,1), every
weight ~N(0, 0.02^2), dY~N(0,1). Large weights are drawn one expert at a time
so no fp32 copy of a whole weight tensor is ever held.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    F: int
    S: int = 0                 # shared experts (0 or 1)
    score: str = "softmax"     # "softmax" | "sigmoid"
    norm_topk: bool = True
    route_scale: float = 1.0
    dtype: str = "bf16"        # expert operand dtype: "bf16" | "mxfp8" | "nvfp4"
    aux: bool = True           # compute the load-balancing aux statistic
    skew: bool = False         # add the skew logit bias
    bwd: bool = False          # the workload includes the backward pass
    capacity_factor: float = 0.0  # > 0: each expert keeps its first ceil(cf T k / E) pairs
    n_group: int = 0           # > 1: group-limited routing over n_group groups of experts
    topk_group: int = 0        # groups kept per token when n_group > 1
    sel_bias: bool = False     # draw a per-expert selection bias (moves selection, not gates)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def rows(self) -> int:
        return self.T * self.k

    def expert_flops_fwd(self) -> float:
        """Algorithmic expert FLOPs of one forward pass (routed + shared)."""
        return 6.0 * self.H * self.F * (self.T * self.k + self.T * self.S)

    def expert_weight_bytes(self) -> float:
        """Bytes of the routed and shared expert weights (bf16; fp8 + 1/32 scale bytes; fp4 + 1/16)."""
        per = {"mxfp8": 1.0 + 1.0 / 32, "nvfp4": 0.5 + 1.0 / 16}.get(self.dtype, 2.0)
        return 3.0 * self.H * self.F * (self.E + self.S) * per

    def router_flops(self) -> float:
        return 2.0 * self.T * self.H * self.E


WORKLOADS = {
    "tiny": Workload("tiny", T=512, H=256, E=8, k=2, F=512),
    "mixtral": Workload("mixtral", T=4096, H=4096, E=8, k=2, F=14336),
    "qwen3": Workload("qwen3", T=8192, H=4096, E=128, k=8, F=1536),
    "dsv3": Workload("dsv3", T=8192, H=7168, E=256, k=8, F=2048, S=1,
                     score="sigmoid", route_scale=2.5, dtype="mxfp8", aux=False),
    "skewed": Workload("skewed", T=8192, H=4096, E=128, k=8, F=1536,
                       skew=True, bwd=True),
    # the ranked variants on the same shapes: DeepSeek-V3 routing (selection bias, 8 groups, 4 kept)
    # and the capacity factor (1.25) on the skewed fwd+bwd step
    "dsv3-grouped": Workload("dsv3-grouped", T=8192, H=7168, E=256, k=8, F=2048, S=1, score="sigmoid",
                             route_scale=2.5, dtype="mxfp8", aux=False, n_group=8, topk_group=4, sel_bias=True),
    # the DeepSeek-V3 forward with NVFP4 expert operands (E2M1 + E4M3 per 16, per-expert encode scales)
    "dsv3-nvfp4": Workload("dsv3-nvfp4", T=8192, H=7168, E=256, k=8, F=2048, S=1, score="sigmoid",
                           route_scale=2.5, dtype="nvfp4", aux=False),
    # the same with 64 experts and T=2048: the same ~256 rows per expert (so the same tile structure) on a
    # quarter of the weights, about 1.5 GB on the device
    "dsv3-nvfp4-e64": Workload("dsv3-nvfp4-e64", T=2048, H=7168, E=64, k=8, F=2048, S=1, score="sigmoid",
                               route_scale=2.5, dtype="nvfp4", aux=False),
    # the MXFP8 layer on the same small case (~1.9 GB on the device): the full ncu capture of the MXFP8 GEMM
    "dsv3-e64": Workload("dsv3-e64", T=2048, H=7168, E=64, k=8, F=2048, S=1, score="sigmoid", route_scale=2.5,
                         dtype="mxfp8", aux=False),
    # the token-side traffic of the Qwen3 shape (T=8192, H=4096, k=8) on 16 small experts, about 1.5 GB on the
    # device: the small case of the permutation and unpermute kernels' DRAM captures
    "qwen3-mem": Workload("qwen3-mem", T=8192, H=4096, E=16, k=8, F=512),
    # the token-side traffic of the DeepSeek-V3 MXFP8 shape (T=8192, H=7168, k=8, MXFP8 permutation) on 16 small
    # experts without the shared one, a few GB on the device: the small case of the MXFP8 permutation's captures
    "dsv3-mem": Workload("dsv3-mem", T=8192, H=7168, E=16, k=8, F=256, score="sigmoid", route_scale=2.5,
                         dtype="mxfp8", aux=False),
    # the MXFP8 backward on the DeepSeek-V3 routed experts (the backward has no shared expert)
    "dsv3-train": Workload("dsv3-train", T=8192, H=7168, E=256, k=8, F=2048, score="sigmoid", route_scale=2.5,
                           dtype="mxfp8", aux=False, bwd=True),
    # the same MXFP8 training step on 16 experts with the same ~256 rows each (~4 GB on the device): the small
    # case of the backward kernels' section captures
    "dsv3-train-e16": Workload("dsv3-train-e16", T=512, H=7168, E=16, k=8, F=2048, score="sigmoid", route_scale=2.5,
                               dtype="mxfp8", aux=False, bwd=True),
    "skewed-capacity": Workload("skewed-capacity", T=8192, H=4096, E=128, k=8, F=1536, skew=True, bwd=True,
                                capacity_factor=1.25),
}


def skew_bias(E: int) -> torch.Tensor:
    """Per-expert logit bias of the skewed workload (an input, fp32 [E]).

    log-Zipf prior with s=1.2 over expert rank e+1, and the last four experts
    pushed to -30 so that they receive no tokens at all.
    """
    b = torch.tensor([-1.2 * math.log(e + 1.0) for e in range(E)], dtype=torch.float32)
    if E > 4:
        b[E - 4:] = -30.0
    return b


def _randn_bf16(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if len(shape) == 3:
        # one expert at a time: bounded fp32 scratch
        for e in range(shape[0]):
            t = torch.randn(shape[1:], generator=gen, dtype=torch.float32, device=device)
            out[e].copy_(t.mul_(std))
    else:
        t = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
        out.copy_(t.mul_(std))
    return out


def make_inputs(wl: Workload, device="cpu", seed: int = 0, with_dy: bool | None = None) -> dict:
    """Draw the inputs of workload `wl` on `device` (see the module docstring)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, H, E, F = wl.T, wl.H, wl.E, wl.F
    d = {}
    d["x"] = _randn_bf16((T, H), 1.0, gen, device)
    d["W_r"] = _randn_bf16((E, H), 0.02, gen, device)
    d["W_g"] = _randn_bf16((E, F, H), 0.02, gen, device)
    d["W_u"] = _randn_bf16((E, F, H), 0.02, gen, device)
    d["W_d"] = _randn_bf16((E, H, F), 0.02, gen, device)
    if wl.S:
        d["W_gs"] = _randn_bf16((F, H), 0.02, gen, device)
        d["W_us"] = _randn_bf16((F, H), 0.02, gen, device)
        d["W_ds"] = _randn_bf16((H, F), 0.02, gen, device)
    if with_dy is None:
        with_dy = wl.bwd
    if with_dy:
        d["dY"] = _randn_bf16((T, H), 1.0, gen, device)
    d["logit_bias"] = skew_bias(E).to(device) if wl.skew else None
    # per-expert selection bias (drawn last so the other inputs do not change): uniform in
    # [-0.1, 0.1), the order of the balancing corrections a DeepSeek-V3-style router carries
    d["expert_bias"] = ((torch.rand((E,), generator=gen, device=device) - 0.5) * 0.2) if wl.sel_bias else None
    return d


def random_logits(T: int, E: int, device="cpu", seed: int = 0, std: float = 1.28,
                  ties: bool = False) -> torch.Tensor:
    """Seeded fp32 router logits [T,E] (input for the routing-stage tests).

    std 1.28 is the logit spread of x~N(0,1), W_r~N(0,0.02^2) at H=4096.
    With `ties`, values are rounded to a coarse grid so that many exact ties
    occur (tests the lowest-index tie-break).
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    l = torch.randn((T, E), generator=gen, dtype=torch.float32, device=device) * std
    if ties:
        l = torch.round(l * 2.0) / 2.0
    return l


def random_routing(T: int, E: int, k: int, device="cpu", seed: int = 0,
                   zero_experts: int = 0, hot: float = 0.0) -> torch.Tensor:
    """Seeded top-k expert indices [T,k] int32: k distinct experts per token.

    `zero_experts` experts (the highest-numbered ones) are never chosen;
    `hot` in [0,1) makes expert 0 appear in that fraction of tokens (skew).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    Eu = E - zero_experts
    assert Eu >= k
    keys = torch.rand((T, Eu), generator=gen)
    if hot > 0.0:
        hot_mask = torch.rand((T,), generator=gen) < hot
        keys[hot_mask, 0] = 2.0
    idx = torch.argsort(keys, dim=1, descending=True)[:, :k].to(torch.int32)
    return idx.contiguous().to(device)


def random_gates(T: int, k: int, device="cpu", seed: int = 0) -> torch.Tensor:
    """Seeded positive per-(token, slot) gate values [T,k] fp32."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    g = torch.rand((T, k), generator=gen) * 0.9 + 0.05
    return g.to(device)


def randn_bf16(shape, std: float = 1.0, seed: int = 0, device="cpu", scale_rows: bool = False) -> torch.Tensor:
    """Seeded N(0, std^2) tensor cast to bf16 (RNE). With scale_rows, each row
    is further multiplied by 2^u, u uniform in [-12, 12] (a wide dynamic range
    for quantiser tests)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    t = torch.randn(shape, generator=gen, dtype=torch.float32, device=device) * std
    if scale_rows:
        u = torch.randint(-12, 13, (shape[0],) + (1,) * (len(shape) - 1), generator=gen, device=device)
        t = t * torch.pow(2.0, u.to(torch.float32))
    return t.to(torch.bfloat16)
