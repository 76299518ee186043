"""Benchmark of the MoE layer on B200: one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral|qwen3|dsv3|skewed|tiny]
                  [--impl ours|reference]

A step is one pass of the layer (router -> permute -> grouped gate/up GEMM with
the fused SwiGLU and gate -> grouped down GEMM -> [shared expert] -> unpermute,
plus the backward for the fwd+bwd workload) over one batch of synthetic
tokens, with every input already resident in device memory. The stage entry
points of the C ABI are called in order on one stream, with CUDA events
between them, so each kernel's share of the step is measured live; `e2e`
times the public whole-layer call moe_layer_fwd with the step's tokens copied
from pinned host memory and the output copied back every step.

Inputs (weights >= 2.8 GB) are larger than the 126 MB L2, so no L2 flush is
needed between steps. Multi-GPU runs are data-parallel replicas (one process
per GPU, torchrun): each rank runs its own layer on its own tokens, there is
no collective in the data path, and the step time is the max over ranks.

--impl reference times the CPU oracle (the only reference this layer has) on
a bounded sample of tokens on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_aux_b200.synthetic import WORKLOADS, make_inputs  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def measured_traffic(workload: str):
    """DRAM bytes per launch of the gate/up GEMM from the committed ncu capture, or None when the
    capture is of another workload or the kernel's sources have changed since it was taken."""
    import hashlib
    import re
    p = os.path.join(ROOT, "profiles", "gemm_gateup_mixtral.md")
    if not os.path.exists(p):
        return None
    m = re.search(r"```json traffic\n(.*?)\n```", open(p).read(), re.S)
    if not m:
        return None
    meta = json.loads(m.group(1))
    if meta.get("workload") != workload:
        return None
    h = hashlib.sha256()
    for f in meta["sources"]:
        with open(os.path.join(ROOT, f)) as fh:
            h.update(code_tokens(fh.read()).encode())
    return meta["dram_bytes_per_launch"] if h.hexdigest() == meta["sources_sha256"] else None


def code_tokens(src: str) -> str:
    """C/CUDA source with its comments removed and every run of whitespace outside string and character
    literals folded to one space: edits to comments or layout leave it unchanged, any change to the code
    changes it."""
    out, i, n = [], 0, len(src)

    def sp():
        if out and out[-1] != " ":
            out.append(" ")

    while i < n:
        c = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            sp()
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif c.isspace():
            while i < n and src[i].isspace():
                i += 1
            sp()
        else:
            out.append(c)
            i += 1
    return "".join(out).strip()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


METRIC = "MoE-layer tokens/s (grouped-GEMM TFLOP/s as fraction of B200 peak in roofline), 1 GPU per replica"
DATA = "synthetic (seeded; x~N(0,1), weights~N(0,0.02^2), bf16)"


def workload_config(wl, ws):
    variant = (f" groups {wl.topk_group}/{wl.n_group}" if wl.n_group > 1 else "") + \
        (" +selection bias" if wl.sel_bias else "") + \
        (f" capacity {wl.capacity_factor}" if wl.capacity_factor > 0 else "")
    return {"workload": f"{wl.name}: {'fwd+bwd' if wl.bwd else 'fwd'} T={wl.T} H={wl.H} E={wl.E} k={wl.k} "
                        f"F={wl.F}{' +1 shared' if wl.S else ''} {wl.score} {wl.dtype}{variant}",
            "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "F": wl.F, "shared": wl.S,
            "parallelism": f"replicas x{ws} (no data-path collective)",
            "l2": (f"inputs larger than L2 (expert weights {wl.expert_weight_bytes() / 1e9:.1f} GB vs 126 MB), "
                   "no flush" if wl.expert_weight_bytes() > 126e6 else "weights fit in L2 (parity-size case)")}


def aggregate_tokens_per_s(tokens_per_rank, ws, ms_max):
    """Whole-job throughput: every rank's tokens over the slowest rank's step time."""
    return round(tokens_per_rank * ws / (ms_max * 1e-3), 1)


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, ws


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    """Max of a float over ranks (device tensor on nccl, host on gloo)."""
    if ws == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_done(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # the raw samples stay on disk for inspection: MOE_BENCH_CLOCKS_DIR, else the system temp directory
        d = os.environ.get("MOE_BENCH_CLOCKS_DIR") or os.path.join(tempfile.gettempdir(), "moe_bench_clocks")
        self.path = os.path.join(d, f"clocks_rank{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples"]}
        loaded = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our layer

class Layer:
    """Device buffers and the staged C-ABI calls of one layer step."""

    def __init__(self, moe, wl, seed=0):
        self.moe, self.wl = moe, wl
        self.cfg = moe.make_config(wl, save_for_bwd=int(wl.bwd))
        d = make_inputs(wl, device="cuda", seed=seed)
        T, H, E, k, F = wl.T, wl.H, wl.E, wl.k, wl.F
        rows = T * k
        # block-scaled operands (MXFP8, or NVFP4: two E2M1 codes per byte and a scale per 16)
        self.mx = wl.dtype in ("mxfp8", "nvfp4")
        self.nv = wl.dtype == "nvfp4"
        cw = (lambda K: K // 2) if self.nv else (lambda K: K)       # code bytes per row of K elements
        sw = (lambda K: K // 16) if self.nv else (lambda K: K // 32)  # scale bytes per row
        if self.mx:
            q = {}
            if wl.bwd:
                # the backward's transposed MXFP8 weights: W_d^T [E,F,H] along H, W_g^T | W_u^T [E,H,2F] along F
                self.wdt = torch.empty((E, F, H), dtype=torch.uint8, device="cuda")
                self.wdt_sf = torch.empty((E, F, H // 32), dtype=torch.uint8, device="cuda")
                moe.moe_quantize_mxfp8_t(d["W_d"], self.wdt, self.wdt_sf)
                self.wgu = torch.empty((E, H, 2 * F), dtype=torch.uint8, device="cuda")
                self.wgu_sf = torch.empty((E, H, 2 * F // 32), dtype=torch.uint8, device="cuda")
                moe.moe_quantize_mxfp8_t(d["W_g"], self.wgu, self.wgu_sf, ldd=2 * F)
                moe.moe_quantize_mxfp8_t(d["W_u"], self.wgu, self.wgu_sf, ldd=2 * F, col0=F)
            for name in ["W_g", "W_u", "W_d"] + (["W_gs", "W_us", "W_ds"] if wl.S else []):
                w = d[name]
                codes = torch.empty(w.shape[:-1] + (cw(w.shape[-1]),), dtype=torch.uint8, device="cuda")
                if self.nv:
                    # one buffer: the block scales, then one fp32 encode scale per expert matrix
                    R, C = w.shape[-2], w.shape[-1]
                    sf = torch.empty(moe.moe_nvfp4_sf_bytes(w.numel() // (R * C), R, C), dtype=torch.uint8,
                                     device="cuda")
                    moe.moe_quantize_nvfp4(w, codes, sf)
                else:
                    sf = torch.empty(w.shape[:-1] + (w.shape[-1] // 32,), dtype=torch.uint8, device="cuda")
                    moe.moe_quantize_mxfp8(w, codes, sf)
                q[name] = (codes, sf)
                d[name] = None
            torch.cuda.synchronize()
            self.q = q
        self.d = d
        dev = "cuda"
        self.logits = torch.empty(T, E, dtype=torch.float32, device=dev)
        self.probs = torch.empty(T, E, dtype=torch.float32, device=dev)
        self.idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.gates = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.aux = torch.empty(1, dtype=torch.float32, device=dev) if self.cfg.compute_aux else None
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.row_of = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.src_of = torch.empty(rows, dtype=torch.int32, device=dev)
        self.row_gate = torch.empty(rows, dtype=torch.float32, device=dev)
        self.xp = torch.empty(rows, cw(H), dtype=torch.uint8, device=dev) if self.mx else \
            torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
        self.xp_sf = torch.empty(rows, sw(H), dtype=torch.uint8, device=dev) if self.mx else None
        self.ap = torch.empty(rows, cw(F), dtype=torch.uint8, device=dev) if self.mx else \
            torch.empty(rows, F, dtype=torch.bfloat16, device=dev)
        self.ap_sf = torch.empty(rows, sw(F), dtype=torch.uint8, device=dev) if self.mx else None
        self.o = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.ws_r = moe.workspace(moe.moe_router_workspace_size(self.cfg))
        self.ws_p = moe.workspace(moe.moe_permute_workspace_size(self.cfg))
        self.ws_g = moe.workspace(max(moe.moe_grouped_gemm_workspace_size(self.cfg, 0),
                                      moe.moe_grouped_gemm_workspace_size(self.cfg, 1)))
        self.ws_layer = moe.workspace(moe.moe_layer_workspace_size(self.cfg))
        self.saved = moe.workspace(moe.moe_layer_saved_size(self.cfg)) if wl.bwd else None
        if wl.bwd:
            self.dY = d["dY"]
            self.gateup = torch.empty(rows, 2 * F, dtype=torch.bfloat16, device=dev)
            self.dX = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
            self.dW_r = torch.empty(E, H, dtype=torch.bfloat16, device=dev)
            self.dW_g = torch.empty(E, F, H, dtype=torch.bfloat16, device=dev)
            self.dW_u = torch.empty(E, F, H, dtype=torch.bfloat16, device=dev)
            self.dW_d = torch.empty(E, H, F, dtype=torch.bfloat16, device=dev)
            self.ws_bwd = moe.workspace(moe.moe_layer_bwd_mxfp8_workspace_size(self.cfg) if self.mx
                                        else moe.moe_layer_bwd_workspace_size(self.cfg))
        if wl.S:
            self.off2 = torch.tensor([0, T], dtype=torch.int32, device=dev)
            self.as_ = torch.empty(T, cw(F), dtype=torch.uint8, device=dev) if self.mx else \
                torch.empty(T, F, dtype=torch.bfloat16, device=dev)
            self.as_sf = torch.empty(T, sw(F), dtype=torch.uint8, device=dev) if self.mx else None
            self.so = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
            self.cfg_sh = moe.make_config(wl, T=T, E=1, k=1, n_shared=0, compute_aux=0, save_for_bwd=0, n_group=0,
                                          topk_group=0, capacity_factor=0.0)
            if self.mx:
                self.xq = torch.empty(T, cw(H), dtype=torch.uint8, device=dev)
                self.xq_sf = torch.empty(T, sw(H), dtype=torch.uint8, device=dev)

    def w(self, name):
        return self.q[name] if self.mx else (self.d[name], None)

    # the timed step: staged C-ABI calls with events between stages
    STAGES_FWD = ("router", "permute", "gemm_gateup", "gemm_down", "shared", "unpermute")

    def step(self, ev=None):
        m, c, d = self.moe, self.cfg, self.d

        def mark(i):
            if ev is not None:
                ev[i].record()
        mark(0)
        m.moe_router_topk(c, d["x"], d["W_r"], d["logit_bias"], self.logits, self.probs, self.idx, self.gates,
                          self.counts, self.aux, self.ws_r, expert_bias=d.get("expert_bias"))
        mark(1)
        m.moe_permute(c, d["x"], self.idx, self.gates, None, self.offsets, self.row_of, self.src_of, self.row_gate,
                      self.xp, self.xp_sf, self.ws_p)
        mark(2)
        Wg, sg = self.w("W_g")
        Wu, su = self.w("W_u")
        Wd, sd = self.w("W_d")
        m.moe_grouped_gemm_fwd(c, 0, self.xp, self.xp_sf, Wg, sg, Wu, su, self.offsets, self.row_gate, self.ap,
                               self.ap_sf, self.gateup if self.wl.bwd else None, self.ws_g)
        mark(3)
        m.moe_grouped_gemm_fwd(c, 1, self.ap, self.ap_sf, Wd, sd, None, None, self.offsets, None, self.o, None, None,
                               self.ws_g)
        mark(4)
        extra = None
        if self.wl.S:
            cs = self.cfg_sh
            Wgs, sgs = self.w("W_gs")
            Wus, sus = self.w("W_us")
            Wds, sds = self.w("W_ds")
            xin, xsf = d["x"], None
            if self.nv:
                m.moe_quantize_nvfp4_act(d["x"], self.xq, self.xq_sf)
                xin, xsf = self.xq, self.xq_sf
            elif self.mx:
                m.moe_quantize_mxfp8(d["x"], self.xq, self.xq_sf)
                xin, xsf = self.xq, self.xq_sf
            m.moe_grouped_gemm_fwd(cs, 0, xin, xsf, Wgs, sgs, Wus, sus, self.off2, None, self.as_, self.as_sf, None,
                                   self.ws_g)
            m.moe_grouped_gemm_fwd(cs, 1, self.as_, self.as_sf, Wds, sds, None, None, self.off2, None, self.so, None,
                                   None, self.ws_g)
            extra = self.so
        mark(5)
        m.moe_unpermute(c, self.o, self.row_of, extra, self.y)
        mark(6)

    def launches_per_step(self):
        """Kernels of ours launched per step (as the ncu launch list shows them): router GEMM,
        top-k, finalize (+ aux when computed), rank, scan, scatter, gate/up GEMM, down GEMM,
        unpermute; + the shared expert's two GEMMs (and, block-scaled, its input quantiser); and
        for fwd+bwd the nine kernels of moe_layer_bwd (dY gather, down dgrad with the SwiGLU
        backward, two weight-gradient GEMMs, gate/up dgrad, router backward, two router
        GEMMs, dXp unpermute)."""
        n = 9 + (1 if self.cfg.compute_aux else 0)
        if self.wl.S:
            n += 2 + (1 if self.mx else 0)
        if self.wl.bwd:
            # MXFP8: dY gather-quantise, two dgrad GEMMs, dgate|dup quantiser, padded offsets, four
            # transposed quantisers, two weight-gradient GEMMs, router backward, two router GEMMs, unpermute
            n += 15 if self.mx else 9
        return n

    def layer_call(self, x, y, aux):
        m, c, d = self.moe, self.cfg, self.d
        Wg, sg = self.w("W_g")
        Wu, su = self.w("W_u")
        Wd, sd = self.w("W_d")
        sh = [None] * 6
        if self.wl.S:
            (a, sa), (b, sb), (e, se) = self.w("W_gs"), self.w("W_us"), self.w("W_ds")
            sh = [a, b, e, sa, sb, se]
        m.moe_layer_fwd(c, x, d["W_r"], d["logit_bias"], Wg, Wu, Wd, sg, su, sd, *sh, y, aux, None, None, None, None,
                        self.saved, self.ws_layer, expert_bias=d.get("expert_bias"))

    def bwd_call(self):
        m, c, d = self.moe, self.cfg, self.d
        if self.mx:
            m.moe_layer_bwd_mxfp8(c, self.dY, 0.01, d["x"], d["W_r"], self.wdt, self.wdt_sf, self.wgu, self.wgu_sf,
                                  self.saved, self.dX, self.dW_r, self.dW_g, self.dW_u, self.dW_d, None, self.ws_bwd)
            return
        m.moe_layer_bwd(c, self.dY, 0.01, d["x"], d["W_r"], d["W_g"], d["W_u"], d["W_d"], self.saved, self.dX,
                        self.dW_r, self.dW_g, self.dW_u, self.dW_d, None, self.ws_bwd)


def graph_replay(L, wl, args, st, ws):
    """Capture one whole step in a CUDA graph and time K replays (after W) with CUDA events."""
    def one():
        if wl.bwd:
            L.layer_call(L.d["x"], L.y, L.aux)
            L.bwd_call()
        else:
            L.step()
    side = torch.cuda.Stream()
    side.wait_stream(st)
    with torch.cuda.stream(side):
        one()  # warm the capture stream (tensor maps, function attributes)
    st.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        one()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, ws)
    del g
    return {"ms_per_step": round(ms, 4), "value": aggregate_tokens_per_s(wl.T, ws, ms), "unit": "tokens/s",
            "how": "one step captured in a CUDA graph, replayed K times"}


def run_ours(args, rank, ws):
    import mixture_experts_layer_aux_b200 as moe
    moe.load()
    wl = WORKLOADS[args.workload]
    P = peaks()
    L = Layer(moe, wl, seed=rank)
    st = torch.cuda.current_stream()
    T = wl.T
    nst = 7
    # warm-up
    for _ in range(args.warmup):
        if wl.bwd:
            L.layer_call(L.d["x"], L.y, L.aux)
            L.bwd_call()
        else:
            L.step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    # rows the experts compute: every (token, slot) pair, or the kept ones under a capacity factor
    # (read once, outside the timed region, from a staged routing + permutation)
    rows_kept = wl.T * wl.k
    if wl.capacity_factor > 0:
        L.step()
        torch.cuda.synchronize()
        rows_kept = int(L.offsets[-1].item())

    if wl.bwd:
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    else:
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for i in range(args.steps):
            if wl.bwd:
                ev[i][0].record(st)
                L.layer_call(L.d["x"], L.y, L.aux)
                ev[i][1].record(st)
                L.bwd_call()
                ev[i][2].record(st)
            else:
                L.step(ev[i])
        e1.record(st)
        torch.cuda.synchronize()
    barrier(ws)
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, ws)
    clocks = clk.summary()

    # per-stage times (average over the timed steps)
    if wl.bwd:
        names = ("fwd", "bwd")
    else:
        names = Layer.STAGES_FWD
    stage_ms = {}
    for j, n in enumerate(names):
        stage_ms[n] = sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)) / args.steps

    # dominant kernel: the grouped gate/up GEMM (2/3 of the expert FLOPs)
    F, H, rows = wl.F, wl.H, rows_kept
    flops_gateup = 4.0 * rows * H * F
    flops_down = 2.0 * rows * H * F
    if wl.dtype == "mxfp8":
        peak_t = P.get("bf16_tflops_sustained", P["bf16_tflops"]) * 2.0
        peak_note = "mxfp8 peak = 2 x measured sustained bf16 (nominal fp8:bf16 ratio)"
    elif wl.dtype == "nvfp4":
        peak_t = P.get("bf16_tflops_sustained", P["bf16_tflops"]) * 4.0
        peak_note = "nvfp4 peak = 4 x measured sustained bf16 (nominal fp4:bf16 ratio, 9 : 2.25 PFLOP/s dense)"
    else:
        peak_t = P.get("bf16_tflops_sustained", P["bf16_tflops"])
        peak_note = "measured sustained bf16 (cuBLAS, seconds-long loop)"
    roof = None
    kernels = {}
    if not wl.bwd:
        g_ms = stage_ms["gemm_gateup"]
        d_ms = stage_ms["gemm_down"]
        ach = flops_gateup / (g_ms * 1e-3) / 1e12
        roof = {"kernel": "grouped GEMM gate/up + SwiGLU epilogue", "bound": "tensor", "achieved": round(ach, 1),
                "peak": peak_t, "unit": "TFLOP/s", "frac": round(ach / peak_t, 4),
                "traffic": measured_traffic(wl.name) if wl.dtype == "bf16" else None,
                "peak_source": f"{P['source']}: {peak_note}"}
        hbm = P["hbm_gbs"]
        per_elem = {"mxfp8": 1 + 1 / 32, "nvfp4": 0.5 + 1 / 16}.get(wl.dtype, 2)
        perm_bytes = T * H * 2 + rows * H * per_elem + 16 * rows
        unperm_bytes = rows * H * 2 + T * H * 2 + (T * H * 2 if wl.S else 0)
        kernels = {
            "router_ms": round(stage_ms["router"], 4),
            "permute_ms": round(stage_ms["permute"], 4),
            "permute_GBps": round(perm_bytes / (stage_ms["permute"] * 1e-3) / 1e9, 1),
            "gemm_gateup_ms": round(g_ms, 4),
            "gemm_gateup_TFLOPs": round(ach, 1),
            "gemm_down_ms": round(d_ms, 4),
            "gemm_down_TFLOPs": round(flops_down / (d_ms * 1e-3) / 1e12, 1),
            "shared_ms": round(stage_ms["shared"], 4),
            "unpermute_ms": round(stage_ms["unpermute"], 4),
            "unpermute_GBps": round(unperm_bytes / (stage_ms["unpermute"] * 1e-3) / 1e9, 1),
            "grouped_gemm_TFLOPs": round((flops_gateup + flops_down) / ((g_ms + d_ms) * 1e-3) / 1e12, 1),
            "grouped_gemm_frac_of_peak": round((flops_gateup + flops_down) / ((g_ms + d_ms) * 1e-3) / 1e12 / peak_t,
                                               4),
            "hbm_peak_GBps": hbm,
        }
    else:
        tot = 3.0 * 6.0 * H * F * (rows_kept + wl.T * wl.S)  # algorithmic fwd + bwd expert FLOPs
        kernels = {"fwd_ms": round(stage_ms["fwd"], 4), "bwd_ms": round(stage_ms["bwd"], 4),
                   "expert_TFLOPs_fwd_bwd": round(tot / (ms * 1e-3) / 1e12, 1)}
        ach = tot / (ms * 1e-3) / 1e12
        roof = {"kernel": "whole fwd+bwd step (grouped GEMMs dominate)", "bound": "tensor", "achieved": round(ach, 1),
                "peak": peak_t, "unit": "TFLOP/s", "frac": round(ach / peak_t, 4), "traffic": None,
                "peak_source": f"{P['source']}: {peak_note}"}

    # the same step under CUDA-graph replay (one captured step, replayed K times)
    graph = graph_replay(L, wl, args, st, ws)

    # end to end: public whole-layer call, tokens H2D from pinned memory, y (+aux) D2H, every step. The copies
    # run on two copy streams (H2D, D2H) and overlap the neighbouring steps' compute, double-buffered as an
    # input pipeline would: step i's tokens go up while step i-1 computes, its output comes down while step
    # i+1 computes.
    x_host = L.d["x"].cpu().pin_memory()
    y_host = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    aux_host = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(L.d["x"]) for _ in range(2)]
    y_dev = [torch.empty_like(L.y) for _ in range(2)]
    aux_dev = [torch.empty_like(L.aux) if L.aux is not None else None for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_h2d = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(h2d_s):
            if i >= 2:
                h2d_s.wait_event(ev_comp[b])      # step i-2 has finished reading x_dev[b]
            x_dev[b].copy_(x_host, non_blocking=True)
            ev_h2d[b].record(h2d_s)
        st.wait_event(ev_h2d[b])
        if i >= 2:
            st.wait_event(ev_d2h[b])              # step i-2's output has left y_dev[b]
        L.layer_call(x_dev[b], y_dev[b], aux_dev[b])
        if wl.bwd:
            L.bwd_call()
        ev_comp[b].record(st)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_comp[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            if aux_dev[b] is not None:
                aux_host[b].copy_(aux_dev[b], non_blocking=True)
            ev_d2h[b].record(d2h_s)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(ws)
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(st)
    for i in range(args.steps):
        e2e_step(i)
    st.wait_event(ev_d2h[(args.steps - 1) % 2])
    a1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1) / args.steps, ws)
    h2d = x_host.numel() * 2
    d2h = y_host[0].numel() * 2 + (4 if L.aux is not None else 0)
    assert moe.moe_get_device_status() == 0

    cfg_line = workload_config(wl, ws)
    if wl.capacity_factor > 0:
        cfg_line["rows_computed"] = rows_kept  # of T*k: the pairs kept at the experts' capacity
    line = {
        "metric": METRIC,
        "value": aggregate_tokens_per_s(wl.T, ws, ms),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": DATA,
        "config": cfg_line,
        "roofline": roof,
        "kernels": kernels,
        "e2e": {"value": aggregate_tokens_per_s(wl.T, ws, e2e_ms), "unit": "tokens/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "api": "moe_layer_fwd" +
                (("+moe_layer_bwd_mxfp8" if L.mx else "+moe_layer_bwd") if wl.bwd else ""),
                "copies": "H2D and D2H on their own streams, overlapping the neighbouring steps (double-buffered)"},
        "graph": graph,
        "gpu_launches": L.launches_per_step() * args.steps,
        "clocks": clocks,
    }
    return line, L


class OracleTimer:
    """Times the oracle (as it stands) on a bounded sample of a workload's tokens on the host."""

    def __init__(self, wl, seed=0):
        import oracle
        oracle.build()
        self.oracle = oracle
        self.wl = wl
        # the sample's inputs on the host: x rows, the router, and every expert (tokens may pick any)
        d = make_inputs(wl, device="cuda" if torch.cuda.is_available() else "cpu", seed=seed)
        self.h = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in d.items()}
        del d
        self.mxw = None
        names = ["W_g", "W_u", "W_d"] + (["W_gs", "W_us", "W_ds"] if wl.S else [])
        if wl.dtype == "mxfp8":
            self.mxw = {n: oracle.mxfp8_quantize(self.h[n]) for n in names}
        elif wl.dtype == "nvfp4":
            self.mxw = {n: oracle.nvfp4_quantize(self.h[n], per_matrix=True) for n in names}

    def run(self, n):
        """Seconds the oracle's layer forward takes on the first n tokens."""
        toks = torch.arange(n, dtype=torch.int32)
        sub = dict(self.h)
        sub["x"] = self.h["x"][:n].contiguous()
        t0 = time.perf_counter()
        self.oracle.layer_fwd(self.wl.with_(T=n), sub, toks=toks, mx_weights=self.mxw)
        return time.perf_counter() - t0

    def sample_size(self, budget_s, max_tok):
        self.run(2)                       # warm: threads, page faults
        per_tok = self.run(4) / 4
        return int(max(2, min(max_tok, self.wl.T, budget_s / max(per_tok, 1e-6))))

    def describe(self, n, t, value):
        return {"value": value, "unit": "tokens/s", "cores": self.oracle.nthreads(), "kind": "oracle",
                "sample": f"{n} of {self.wl.T} tokens of the {self.wl.name} layer forward (router + top-k + "
                          f"experts), {t:.2f} s on the host per sample"}


def cpu_baseline(wl, budget_s=12.0, max_tok=256, seed=0):
    ot = OracleTimer(wl, seed)
    n = ot.sample_size(budget_s, max_tok)
    t = ot.run(n)
    return ot.describe(n, t, round(n / t, 3)), n, t


def run_reference(args, rank, ws):
    """The oracle on the host cores: each step times a bounded sample of the workload's tokens,
    sized so that warm-up plus timed steps stay within a few minutes."""
    if rank != 0:
        return None
    wl = WORKLOADS[args.workload]
    ot = OracleTimer(wl, seed=0)
    budget = max(0.05, min(4.0, 150.0 / (args.warmup + args.steps)))
    n = ot.sample_size(budget, 256)
    vals, tsum = [], 0.0
    for i in range(args.warmup + args.steps):
        t = ot.run(n)
        if i >= args.warmup:
            vals.append(t / n)
            tsum += t
    sec_per_tok = statistics.mean(vals)
    v = round(1.0 / sec_per_tok, 3)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec_per_tok * wl.T * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": DATA, "config": workload_config(wl, ws),
            "cpu_baseline": ot.describe(n, tsum / args.steps, v),
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="mixtral", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank, ws = dist_setup(args.gpus)
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        line = run_reference(args, rank, ws)
        if rank == 0:
            print(json.dumps(line), flush=True)
        dist_done(ws)
        return
    line, L = run_ours(args, rank, ws)
    del L
    torch.cuda.empty_cache()
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)[0]
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_done(ws)


if __name__ == "__main__":
    main()
