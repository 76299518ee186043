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
    """DRAM bytes per launch of the workload's gate/up GEMM from a committed ncu capture (a ```json traffic
    block in a profiles/*.md summary), or None when no capture is of this workload or the captured kernel's
    sources have changed since it was taken."""
    import glob
    import hashlib
    import re
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for block in re.findall(r"```json traffic\n(.*?)\n```", open(p).read(), re.S):
            meta = json.loads(block)
            if meta.get("workload") != workload:
                continue
            h = hashlib.sha256()
            for f in meta["sources"]:
                with open(os.path.join(ROOT, f)) as fh:
                    h.update(code_tokens(fh.read()).encode())
            return meta["dram_bytes_per_launch"] if h.hexdigest() == meta["sources_sha256"] else None
    return None


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
    """SM clock, power and throttle reasons sampled during a timed region.

    A background thread reads them through NVML (read-only queries) every ~2 ms, so even a timed region of
    a few tens of milliseconds gets tens of samples; where NVML is unavailable, nvidia-smi polls at its own
    rate instead. While it runs, the interpreter's thread switch interval is cut to 0.5 ms, so the launching
    thread cannot hold the sampler off for the default 5 ms. Nothing here changes any GPU setting."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples = []            # (sm_mhz, power_w, reasons bitmask)
        self.max_mhz = None
        self.how = None
        self.proc = self.thread = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def __enter__(self):
        import sys
        import threading
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(min(self._switch, 0.0005))
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._bits = {name: getattr(nv, attr) for name, attr in self.REASONS}
            self._stop = threading.Event()

            def poll():
                while not self._stop.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                             int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        pass
                    self._stop.wait(self.period)
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.how = f"NVML every {self.period * 1e3:.0f} ms"
        except Exception:
            self._start_smi()
        return self

    def _start_smi(self):
        d = os.environ.get("MOE_BENCH_CLOCKS_DIR") or os.path.join(tempfile.gettempdir(), "moe_bench_clocks")
        self.path = os.path.join(d, f"clocks_gpu{self.index}.csv")
        try:
            os.makedirs(d, exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            self.how = "nvidia-smi -lms 20"
        except (OSError, FileNotFoundError):
            self.proc = None

    def __exit__(self, *a):
        import sys
        sys.setswitchinterval(self._switch)
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
            self._read_smi()

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        self._bits = {n: 1 << i for i, n in enumerate(names)}
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
                pw = float(parts[3])
            except ValueError:
                continue
            mask = sum(1 << i for i, v in enumerate(parts[5:9]) if v.lower() == "active")
            self.samples.append((sm, pw, mask))
            self.max_mhz = mx

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"], "samples": 0,
                    "how": self.how}
        mx = self.max_mhz
        sm = [x[0] for x in self.samples]
        loaded = [x for x in self.samples if mx and x[0] > 0.5 * mx] or self.samples
        reasons = sorted({n for n, bit in self._bits.items() for x in self.samples if x[2] & bit})
        return {"sm_mhz": statistics.median([x[0] for x in loaded]), "sm_max_mhz": mx,
                "sm_mhz_min": min(sm), "power_w_max": round(max(x[1] for x in self.samples), 1),
                "reasons": reasons, "samples": len(self.samples), "how": self.how}


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
        top-k, finalize (+ aux when computed), rank, scan, permute, gate/up GEMM, down GEMM,
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


# measured on B200 by back-to-back MMA probes from shared memory (one CTA per SM): dense flop per SM clock
FLOP_PER_SM_CLK = {"bf16": 8190.0, "mxfp8": 16381.0}
N_SM = 148


def tensor_peak(P, dtype, timed_s):
    """Dense peak for a kernel timed inside a region of timed_s seconds: the burst cuBLAS bf16 figure for a
    region shorter than two seconds, the sustained one (a seconds-long loop under the power cap) for a
    longer one; MXFP8 and NVFP4 at the nominal 2x and 4x of bf16."""
    sustained = timed_s >= 2.0
    base = P.get("bf16_tflops_sustained", P["bf16_tflops"]) if sustained else P["bf16_tflops"]
    mult = {"mxfp8": 2.0, "nvfp4": 4.0}.get(dtype, 1.0)
    what = "sustained" if sustained else "burst"
    note = f"{P['source']} cuBLAS bf16 {what} ({base:g} TFLOP/s)" + (f" x {mult:g} for {dtype}" if mult != 1 else "")
    return base * mult, note


def clock_normalised(flops, ms, clocks, dtype):
    """Flop per SM clock per SM (from the median loaded SM clock), against the probe-measured MMA rate."""
    mhz = clocks.get("sm_mhz")
    per = FLOP_PER_SM_CLK.get(dtype)
    if not mhz or not ms:
        return None
    f = flops / (ms * 1e-3) / (mhz * 1e6) / N_SM
    out = {"flop_per_sm_clk": round(f, 1), "sm_mhz": mhz}
    if per:
        out.update(probe_flop_per_sm_clk=per, frac=round(f / per, 4))
    return out


def measure(moe, wl, args, ws, rank, P, headline):
    """Time K steps of workload wl (after W warm-up steps) and return its measurements; the headline
    workload also gets CUDA-graph replay and the end-to-end (host buffers) figure."""
    L = Layer(moe, wl, seed=rank)
    st = torch.cuda.current_stream()
    T = wl.T
    nst = 7
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
    timed_s = ms * args.steps * 1e-3

    names = ("fwd", "bwd") if wl.bwd else Layer.STAGES_FWD
    stage_ms = {}
    for j, n in enumerate(names):
        stage_ms[n] = sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)) / args.steps

    F, H, rows = wl.F, wl.H, rows_kept
    flops_gateup = 4.0 * rows * H * F
    flops_down = 2.0 * rows * H * F
    peak_t, peak_note = tensor_peak(P, wl.dtype, timed_s)
    hbm = P["hbm_gbs"]
    if not wl.bwd:
        g_ms, d_ms = stage_ms["gemm_gateup"], stage_ms["gemm_down"]
        ach = flops_gateup / (g_ms * 1e-3) / 1e12
        roof = {"kernel": "grouped GEMM gate/up + SwiGLU epilogue", "bound": "tensor", "achieved": round(ach, 1),
                "peak": round(peak_t, 1), "unit": "TFLOP/s", "frac": round(ach / peak_t, 4),
                "traffic": measured_traffic(wl.name),
                "peak_source": peak_note + " (of measured)" if P["source"] == "measured" else peak_note,
                "clock_normalised": clock_normalised(flops_gateup, g_ms, clocks, wl.dtype)}
        per_elem = {"mxfp8": 1 + 1 / 32, "nvfp4": 0.5 + 1 / 16}.get(wl.dtype, 2)
        perm_bytes = T * H * 2 + rows * H * per_elem + 16 * rows
        unperm_bytes = rows * H * 2 + T * H * 2 + (T * H * 2 if wl.S else 0)
        kernels = {
            "router_ms": round(stage_ms["router"], 4),
            "permute_ms": round(stage_ms["permute"], 4),
            "permute_GBps": round(perm_bytes / (stage_ms["permute"] * 1e-3) / 1e9, 1),
            "permute_frac_of_hbm": round(perm_bytes / (stage_ms["permute"] * 1e-3) / 1e9 / hbm, 4),
            "gemm_gateup_ms": round(g_ms, 4),
            "gemm_gateup_TFLOPs": round(ach, 1),
            "gemm_down_ms": round(d_ms, 4),
            "gemm_down_TFLOPs": round(flops_down / (d_ms * 1e-3) / 1e12, 1),
            "shared_ms": round(stage_ms["shared"], 4),
            "unpermute_ms": round(stage_ms["unpermute"], 4),
            "unpermute_GBps": round(unperm_bytes / (stage_ms["unpermute"] * 1e-3) / 1e9, 1),
            "unpermute_frac_of_hbm": round(unperm_bytes / (stage_ms["unpermute"] * 1e-3) / 1e9 / hbm, 4),
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
                "peak": round(peak_t, 1), "unit": "TFLOP/s", "frac": round(ach / peak_t, 4), "traffic": None,
                "peak_source": peak_note + " (of measured)" if P["source"] == "measured" else peak_note,
                "clock_normalised": clock_normalised(tot, ms, clocks, wl.dtype)}
    out = {"ms_per_step": round(ms, 4), "value": aggregate_tokens_per_s(wl.T, ws, ms), "unit": "tokens/s",
           "timed_s": round(timed_s, 4), "roofline": roof, "kernels": kernels, "clocks": clocks,
           "gpu_launches": L.launches_per_step() * args.steps, "rows_kept": rows_kept}
    if headline:
        out["graph"] = graph_replay(L, wl, args, st, ws)
        out["e2e"] = e2e(moe, L, wl, args, st, ws)
    del L
    torch.cuda.empty_cache()
    return out


def e2e(moe, L, wl, args, st, ws):
    """End to end through the public whole-layer call: tokens H2D from pinned memory, y (+aux) D2H, every
    step. The copies run on two copy streams (H2D, D2H) and overlap the neighbouring steps' compute,
    double-buffered as an input pipeline would: step i's tokens go up while step i-1 computes, its output
    comes down while step i+1 computes."""
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
    return {"value": aggregate_tokens_per_s(wl.T, ws, e2e_ms), "unit": "tokens/s", "ms_per_step": round(e2e_ms, 4),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "api": "moe_layer_fwd" +
            (("+moe_layer_bwd_mxfp8" if L.mx else "+moe_layer_bwd") if wl.bwd else ""),
            "copies": "H2D and D2H on their own streams, overlapping the neighbouring steps (double-buffered)"}


# the other configurations reported beside the headline workload, in the same run (one GPU)
OTHER_WORKLOADS = ("qwen3", "dsv3", "skewed", "dsv3-nvfp4", "dsv3-train")


def run_ours(args, rank, ws):
    import mixture_experts_layer_aux_b200 as moe
    moe.load()
    wl = WORKLOADS[args.workload]
    P = peaks()
    m = measure(moe, wl, args, ws, rank, P, headline=True)
    cfg_line = workload_config(wl, ws)
    if wl.capacity_factor > 0:
        cfg_line["rows_computed"] = m["rows_kept"]  # of T*k: the pairs kept at the experts' capacity
    line = {
        "metric": METRIC,
        "value": m["value"],
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": DATA,
        "config": cfg_line,
        "roofline": m["roofline"],
        "kernels": m["kernels"],
        "e2e": m["e2e"],
        "graph": m["graph"],
        "gpu_launches": m["gpu_launches"],
        "clocks": m["clocks"],
    }
    others = [w for w in (args.workloads.split(",") if args.workloads else []) if w and w != args.workload]
    if others and ws == 1:
        line["workloads"] = {}
        for name in others:
            o = measure(moe, WORKLOADS[name], args, ws, rank, P, headline=False)
            o["config"] = workload_config(WORKLOADS[name], ws)["workload"]
            o.pop("rows_kept")
            line["workloads"][name] = o
            line["gpu_launches"] += o["gpu_launches"]
    return line, None


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
    # a step is the bounded token sample; the whole workload's step time is only an extrapolation
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tsum / args.steps * 1e3, 1),
            "step": f"{n} of the workload's {wl.T} tokens (a bounded sample)",
            "extrapolated_full_step_ms": round(sec_per_tok * wl.T * 1e3, 1),
            "extrapolated_note": "per-token time of the sample x T, not measured",
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
    ap.add_argument("--workloads", default=",".join(OTHER_WORKLOADS),
                    help="other workloads measured in the same run (single GPU only); '' for none")
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
    line, _ = run_ours(args, rank, ws)
    torch.cuda.empty_cache()
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)[0]
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_done(ws)


if __name__ == "__main__":
    main()
