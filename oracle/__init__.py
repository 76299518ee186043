"""CPU oracle of the MoE layer -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package. The product path never does, and this package
imports nothing from the product (mixture_experts_layer_aux_b200).

The arithmetic lives in moe_oracle.c (plain per-token loops in fp64; each
function there cites the passage it follows). This module only marshals CPU
tensors into it and chains its steps in the order the pages give:

  score every expert -> keep the top-k -> sum gate(e) * Expert_e(x)
  ("Megatron-Core MoE -- 大规模稀疏专家并行实践", 实践案例 / 案例 1)

Parity status: every oracle function is pinned by a test in
tests/test_oracle.py against something other than itself (brute force,
closed forms, library routines, finite differences, hand-computed OCP MX
and NVFP4 values); none is "parity unpinned". tests/test_oracle_mutants.py
plants one mistake at a time in a scratch copy of moe_oracle.c and checks
that each fails at least one of those pins.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

OC_BF16, OC_MXFP8, OC_F64, OC_NVFP4 = 0, 1, 2, 3
# rounding points of the precision recipes (see moe_oracle.c); "mxfp8-q" / "nvfp4-q" keep only the
# block-scaled formats' quantisation points (no bf16 rounding anywhere else)
RECIPES = {"exact": 0, "mxfp8": 1, "bf16": 2, "nvfp4": 3, "mxfp8-q": 4, "nvfp4-q": 5}
MX_RECIPES = ("mxfp8", "mxfp8-q")


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (portable x86-64 code, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Mat(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("cols", ctypes.c_int32), ("rows", ctypes.c_int64),
                ("data", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("gs", ctypes.c_void_p),
                ("gs_rows", ctypes.c_int64)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            _lib.oc_e4m3_decode.restype = ctypes.c_double
            _lib.oc_e4m3_decode.argtypes = [ctypes.c_uint8]
            _lib.oc_e4m3_encode.restype = ctypes.c_uint8
            _lib.oc_e4m3_encode.argtypes = [ctypes.c_double]
            _lib.oc_mx_scale_byte.restype = ctypes.c_uint8
            _lib.oc_mx_scale_byte.argtypes = [ctypes.c_double]
            _lib.oc_aux.restype = ctypes.c_double
            _lib.oc_bf16_round.restype = ctypes.c_double
            _lib.oc_bf16_round.argtypes = [ctypes.c_double]
            _lib.oc_num_threads.restype = ctypes.c_int
            _lib.oc_e2m1_decode.restype = ctypes.c_double
            _lib.oc_e2m1_decode.argtypes = [ctypes.c_uint8]
            _lib.oc_e2m1_encode.restype = ctypes.c_uint8
            _lib.oc_e2m1_encode.argtypes = [ctypes.c_double]
            _lib.oc_nvfp4_global_scale.restype = ctypes.c_float
            _lib.oc_nvfp4_global_scale.argtypes = [ctypes.c_float]
            _lib.oc_nvfp4_scale_byte.restype = ctypes.c_uint8
            _lib.oc_nvfp4_scale_byte.argtypes = [ctypes.c_float, ctypes.c_float]
            _lib.oc_nvfp4_quantize_bf16.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_void_p, ctypes.c_float,
                                                    ctypes.c_void_p, ctypes.c_void_p]
            _lib.oc_nvfp4_quantize_f32.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_void_p, ctypes.c_float,
                                                   ctypes.c_void_p, ctypes.c_void_p]
            _lib.oc_bf16_amax.restype = ctypes.c_float
            _lib.oc_bf16_amax.argtypes = [ctypes.c_long, ctypes.c_void_p]
        return _lib


# ----------------------------------------------------------------- helpers

def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _chk(t, dtype):
    assert t.device.type == "cpu", "the oracle runs on host tensors only"
    assert t.dtype == dtype, (t.dtype, dtype)
    assert t.is_contiguous()
    return t


class Mat:
    """A row-major matrix the oracle can read: bf16, MXFP8 (codes+scales), NVFP4
    (packed codes + scales + per-matrix encode scales) or fp64.

    Keeps the backing tensors alive while the C side holds raw pointers.
    """

    def __init__(self, kind, data, sf=None, rows=None, cols=None, gs=None, gs_rows=0):
        self.kind, self.data, self.sf, self.gs = kind, data, sf, gs
        if cols is None:
            cols = data.shape[-1]
        if rows is None:
            rows = data.numel() // cols
        self.s = _Mat(kind, cols, rows, data.data_ptr(), 0 if sf is None else sf.data_ptr(),
                      0 if gs is None else gs.data_ptr(), gs_rows)

    @property
    def ref(self):
        return ctypes.byref(self.s)


def mat(t: torch.Tensor) -> Mat:
    """bf16 or fp64 tensor -> Mat (2-D view over the last dim)."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return Mat(OC_BF16, t.view(torch.int16))
    if t.dtype == torch.float64:
        return Mat(OC_F64, t)
    raise TypeError(t.dtype)


def mat_mx(codes: torch.Tensor, sf: torch.Tensor) -> Mat:
    return Mat(OC_MXFP8, _chk(codes.contiguous(), torch.uint8), _chk(sf.contiguous(), torch.uint8))


def mat_nv(packed: torch.Tensor, sf: torch.Tensor, gs: torch.Tensor | None) -> Mat:
    """NVFP4 matrix: packed [..., R, C/2], sf [..., R, C/16], gs [...] fp32 (one G per [R, C] matrix) or None."""
    packed = _chk(packed.contiguous(), torch.uint8)
    cols = 2 * packed.shape[-1]
    R = packed.shape[-2] if packed.dim() >= 2 else 1
    if gs is not None:
        gs = _chk(gs.reshape(-1).contiguous(), torch.float32)
    return Mat(OC_NVFP4, packed, _chk(sf.contiguous(), torch.uint8), rows=packed.numel() * 2 // cols, cols=cols,
               gs=gs, gs_rows=R)


def nthreads() -> int:
    return lib().oc_num_threads()


def bf16_round(v: float) -> float:
    """fp32-then-bf16 round-to-nearest-even of one value."""
    return float(lib().oc_bf16_round(float(v)))


def _recipe(r):
    return RECIPES[r] if isinstance(r, str) else int(r)


# ----------------------------------------------------------------- MXFP8

def e4m3_encode(v: float) -> int:
    return int(lib().oc_e4m3_encode(float(v)))


def e4m3_decode(c: int) -> float:
    return float(lib().oc_e4m3_decode(int(c)))


def mx_scale_byte(amax: float) -> int:
    return int(lib().oc_mx_scale_byte(float(amax)))


def mxfp8_quantize(src: torch.Tensor):
    """src [..., K] bf16 or fp32 (K % 32 == 0) -> (codes uint8 [..., K], scales uint8 [..., K/32])."""
    K = src.shape[-1]
    assert K % 32 == 0
    src = src.contiguous()
    rows = src.numel() // K
    codes = torch.empty(src.shape, dtype=torch.uint8)
    scales = torch.empty(tuple(src.shape[:-1]) + (K // 32,), dtype=torch.uint8)
    if src.dtype == torch.bfloat16:
        lib().oc_mxfp8_quantize_bf16(ctypes.c_long(rows), K, _p(src), _p(codes), _p(scales))
    elif src.dtype == torch.float32:
        lib().oc_mxfp8_quantize(ctypes.c_long(rows), K, _p(src), _p(codes), _p(scales))
    else:
        raise TypeError(src.dtype)
    return codes, scales


def mxfp8_decode(codes: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """Exact fp64 values of MXFP8 codes + scales (table lookup per code)."""
    table = torch.tensor([e4m3_decode(c) for c in range(256)], dtype=torch.float64)
    v = table[codes.long()]
    s = torch.pow(2.0, scales.to(torch.float64) - 127.0)
    return v * s.repeat_interleave(32, dim=-1)


# ----------------------------------------------------------------- NVFP4

def e2m1_encode(v: float) -> int:
    return int(lib().oc_e2m1_encode(float(v)))


def e2m1_decode(c: int) -> float:
    return float(lib().oc_e2m1_decode(int(c)))


def nvfp4_global_scale(amax: float) -> float:
    return float(lib().oc_nvfp4_global_scale(float(amax)))


def nvfp4_scale_byte(amax: float, G: float = 1.0) -> int:
    return int(lib().oc_nvfp4_scale_byte(float(amax), float(G)))


def nvfp4_quantize(src: torch.Tensor, per_matrix: bool = False):
    """src [..., K] bf16 or fp32 (K % 16 == 0) -> (packed uint8 [..., K/2], scales uint8 [..., K/16], G fp32).

    per_matrix (bf16 only): each [R, K] matrix of src [..., R, K] gets G = 6*448/amax(matrix)
    (G is then [...]); otherwise G = 1 (a 0-d tensor)."""
    K = src.shape[-1]
    assert K % 16 == 0
    src = src.contiguous()
    packed = torch.empty(tuple(src.shape[:-1]) + (K // 2,), dtype=torch.uint8)
    scales = torch.empty(tuple(src.shape[:-1]) + (K // 16,), dtype=torch.uint8)
    if src.dtype == torch.float32:
        assert not per_matrix
        lib().oc_nvfp4_quantize_f32(src.numel() // K, K, _p(src), 1.0, _p(packed), _p(scales))
        return packed, scales, torch.tensor(1.0, dtype=torch.float32)
    assert src.dtype == torch.bfloat16
    if not per_matrix:
        lib().oc_nvfp4_quantize_bf16(src.numel() // K, K, _p(src), 1.0, _p(packed), _p(scales))
        return packed, scales, torch.tensor(1.0, dtype=torch.float32)
    R = src.shape[-2]
    mats = src.view(-1, R, K)
    pk, sc = packed.view(-1, R, K // 2), scales.view(-1, R, K // 16)
    G = torch.empty(mats.shape[0], dtype=torch.float32)
    for b in range(mats.shape[0]):
        m = mats[b]
        G[b] = float(lib().oc_nvfp4_global_scale(lib().oc_bf16_amax(m.numel(), _p(m))))
        lib().oc_nvfp4_quantize_bf16(R, K, _p(m), float(G[b]), _p(pk[b]), _p(sc[b]))
    return packed, scales, G.view(src.shape[:-2])


def nvfp4_decode(packed: torch.Tensor, scales: torch.Tensor, G=None) -> torch.Tensor:
    """Exact-up-to-the-final-division fp64 values: E2M1 code * E4M3 scale / G (G per [R, K] matrix)."""
    e2 = torch.tensor([e2m1_decode(c) for c in range(16)], dtype=torch.float64)
    e4 = torch.tensor([e4m3_decode(c) for c in range(256)], dtype=torch.float64)
    lo, hi = (packed & 15).long(), (packed >> 4).long()
    codes = torch.stack([lo, hi], dim=-1).flatten(-2)
    v = e2[codes] * e4[scales.long()].repeat_interleave(16, dim=-1)
    if G is not None and G.dim() > 0:
        v = v / G.to(torch.float64).reshape(tuple(G.shape) + (1, 1))
    elif G is not None:
        v = v / float(G)
    return v


# ----------------------------------------------------------------- routing

def router_logits(x, W_r, bias=None, round_f32=True) -> torch.Tensor:
    """fp64 [T,E] (fp32-valued when round_f32): x W_r^T (+ bias)."""
    T, H = x.shape
    E = W_r.shape[0]
    out = torch.empty((T, E), dtype=torch.float64)
    mx, mw = mat(x), mat(W_r)
    b = None if bias is None else _chk(bias.to(torch.float32).contiguous(), torch.float32)
    lib().oc_router_logits(T, H, E, mx.ref, mw.ref, _p(b), int(round_f32), _p(out))
    return out


def scores(logits: torch.Tensor, score: str) -> torch.Tensor:
    l = _chk(logits.to(torch.float64).contiguous(), torch.float64)
    T, E = l.shape
    s = torch.empty_like(l)
    lib().oc_scores(T, E, 0 if score == "softmax" else 1, _p(l), _p(s))
    return s


def topk(logits: torch.Tensor, k: int) -> torch.Tensor:
    l = _chk(logits.to(torch.float64).contiguous(), torch.float64)
    T, E = l.shape
    idx = torch.empty((T, k), dtype=torch.int32)
    lib().oc_topk(T, E, k, _p(l), _p(idx))
    return idx


def topk_grouped(sel: torch.Tensor, k: int, n_group: int = 0, topk_group: int = 0) -> torch.Tensor:
    """Group-limited top-k on selection scores sel [T,E] (see oc_topk_grouped)."""
    v = _chk(sel.to(torch.float64).contiguous(), torch.float64)
    T, E = v.shape
    idx = torch.empty((T, k), dtype=torch.int32)
    lib().oc_topk_grouped(T, E, k, n_group, topk_group, _p(v), _p(idx))
    return idx


def gates(s: torch.Tensor, idx: torch.Tensor, norm: bool, route_scale: float) -> torch.Tensor:
    T, E = s.shape
    k = idx.shape[1]
    g = torch.empty((T, k), dtype=torch.float64)
    lib().oc_gates(T, E, k, int(norm), ctypes.c_double(route_scale), _p(_chk(s, torch.float64)),
                   _p(_chk(idx, torch.int32)), _p(g))
    return g


def maps(idx: torch.Tensor, E: int, keep: torch.Tensor | None = None):
    """-> counts [E], offsets [E+1], row_of [T,k], src_of [T*k] (all int32).

    With a capacity keep mask (uint8 [T,k]), only kept pairs get rows: counts are
    the kept counts and row_of is -1 for dropped pairs (src_of beyond offsets[E]
    is unused)."""
    idx = _chk(idx.contiguous(), torch.int32)
    T, k = idx.shape
    counts = torch.empty(E, dtype=torch.int32)
    offsets = torch.empty(E + 1, dtype=torch.int32)
    row_of = torch.empty((T, k), dtype=torch.int32)
    src_of = torch.full((T * k,), -1, dtype=torch.int32)
    if keep is None:
        lib().oc_maps(T, E, k, _p(idx), _p(counts), _p(offsets), _p(row_of), _p(src_of))
    else:
        keep = _chk(keep.contiguous(), torch.uint8)
        lib().oc_maps_kept(T, E, k, _p(idx), _p(keep), _p(counts), _p(offsets), _p(row_of), _p(src_of))
    return counts, offsets, row_of, src_of


def capacity_keep(idx: torch.Tensor, E: int, capacity_factor: float):
    """-> (keep uint8 [T,k], C): each expert keeps its first C = ceil(cf T k / E) pairs in
    token order (cf <= 0: no limit, C = T k). cf is the layer configuration's value, an
    IEEE float32 (so 0.6 means 0.60000002384...), and C is computed from it in double
    precision as ((cf T) k) / E."""
    idx = _chk(idx.contiguous(), torch.int32)
    T, k = idx.shape
    cf32 = float(torch.tensor(float(capacity_factor), dtype=torch.float32))
    keep = torch.empty((T, k), dtype=torch.uint8)
    C = lib().oc_capacity_keep(T, E, k, ctypes.c_double(cf32), _p(idx), _p(keep))
    return keep, int(C)


def aux(s_softmax: torch.Tensor, counts: torch.Tensor, k: int) -> float:
    T, E = s_softmax.shape
    return float(lib().oc_aux(T, E, k, _p(_chk(s_softmax, torch.float64)), _p(_chk(counts, torch.int32))))


def route(logits: torch.Tensor, k: int, score: str = "softmax", norm: bool = True,
          route_scale: float = 1.0, with_aux: bool = True, capacity_factor: float = 0.0,
          expert_bias: torch.Tensor | None = None, n_group: int = 0, topk_group: int = 0) -> dict:
    """All routing steps from given logits: scores, top-k, gates, maps, aux.

    counts are the router's (every selected pair; they feed aux). With a capacity
    factor > 0, pairs past an expert's capacity are dropped: keep marks the kept
    pairs, idx_kept is idx with -1 at dropped pairs, kept_counts / offsets /
    row_of / src_of describe the kept rows only."""
    E = logits.shape[1]
    s = scores(logits, score)
    if expert_bias is None and n_group <= 1:
        idx = topk(logits, k)
        sel = None
    else:
        # DeepSeek-V3 variant: selection on score + per-expert bias, group-limited
        sel = s + (expert_bias.to(torch.float64) if expert_bias is not None else 0.0)
        idx = topk_grouped(sel, k, n_group, topk_group)
    g = gates(s, idx, norm, route_scale)
    counts, offsets, row_of, src_of = maps(idx, E)
    out = dict(logits=logits, probs=s, idx=idx, gates=g, counts=counts, offsets=offsets,
               row_of=row_of, src_of=src_of, idx_kept=idx, kept_counts=counts, keep=None, capacity=idx.numel(),
               sel=sel)
    if capacity_factor > 0:
        keep, C = capacity_keep(idx, E, capacity_factor)
        kc, offsets, row_of, src_of = maps(idx, E, keep)
        out.update(keep=keep, capacity=C, idx_kept=torch.where(keep.bool(), idx, torch.full_like(idx, -1)),
                   kept_counts=kc, offsets=offsets, row_of=row_of, src_of=src_of)
    if with_aux and score == "softmax":
        out["aux"] = aux(s, counts, k)
    return out


# ----------------------------------------------------------------- experts

def _wmat(W, sf=None):
    """Expert weight [E, R, C] (or [R, C]) bf16 / fp64, MXFP8 codes with sf, or NVFP4
    packed codes with sf = (scales, G)."""
    if isinstance(sf, tuple):
        return mat_nv(W, sf[0], sf[1])
    if sf is not None:
        return mat_mx(W.reshape(-1, W.shape[-1]), sf.reshape(-1, sf.shape[-1]))
    return mat(W.reshape(-1, W.shape[-1]))


def moe_fwd_tokens(x, W_g, W_u, W_d, idx, g, toks=None, *, recipe="exact", fold=True,
                   sf_g=None, sf_u=None, sf_d=None, shared=None, return_shared=False):
    """Layer output rows y[toks] (fp64, unrounded) for given routing (idx [T,k], gates g [T,k] fp64).

    recipe: "exact" (no rounding), "bf16" (the BF16 recipe's rounding points),
    "mxfp8" (the weight tensors are MXFP8 codes and sf_* their scales) or "nvfp4"
    (the weights are packed NVFP4 codes, sf_* = (scales, G) pairs); "mxfp8-q" /
    "nvfp4-q" take the same operands but round nothing to bf16.
    shared = (W_gs, W_us, W_ds[, sf_gs, sf_us, sf_ds]) adds the always-on shared expert.
    """
    rc = _recipe(recipe)
    mx = rc in (RECIPES["mxfp8"], RECIPES["nvfp4"], RECIPES["mxfp8-q"], RECIPES["nvfp4-q"])
    T, H = x.shape
    E, F = W_g.shape[0], W_g.shape[1]
    k = idx.shape[1]
    if toks is None:
        toks = torch.arange(T, dtype=torch.int32)
    toks = _chk(toks.to(torch.int32).contiguous(), torch.int32)
    n = toks.numel()
    y = torch.empty((n, H), dtype=torch.float64)
    sh_out = torch.empty((n, H), dtype=torch.float64) if (shared is not None and return_shared) else None
    mxm, mg, mu, md = mat(x), _wmat(W_g, sf_g), _wmat(W_u, sf_u), _wmat(W_d, sf_d)
    S = 0
    sref = [None, None, None]
    if shared is not None:
        S = 1
        if mx:
            gs, us, ds, sgs, sus, sds = shared
            sm = [_wmat(gs, sgs), _wmat(us, sus), _wmat(ds, sds)]
        else:
            gs, us, ds = shared[:3]
            sm = [_wmat(gs), _wmat(us), _wmat(ds)]
        sref = [m.ref for m in sm]
    null = ctypes.c_void_p(0)
    lib().oc_moe_fwd_tokens(T, H, E, k, F, S, rc, int(fold), mxm.ref, mg.ref, mu.ref, md.ref,
                            sref[0] or null, sref[1] or null, sref[2] or null,
                            _p(_chk(idx.contiguous(), torch.int32)), _p(_chk(g.contiguous(), torch.float64)),
                            n, _p(toks), _p(y), _p(sh_out))
    return (y, sh_out) if return_shared else y


def moe_fwd_dense(x, W_g, W_u, W_d, gate_dense):
    T, H = x.shape
    E, F = W_g.shape[0], W_g.shape[1]
    y = torch.empty((T, H), dtype=torch.float64)
    mxm, mg, mu, md = mat(x), _wmat(W_g), _wmat(W_u), _wmat(W_d)
    lib().oc_moe_fwd_dense(T, H, E, F, mxm.ref, mg.ref, mu.ref, md.ref,
                           _p(_chk(gate_dense.contiguous(), torch.float64)), _p(y))
    return y


def expert_rows(xp, e_of, g_of, W_g, W_u, W_d, rows=None, *, recipe="exact", sf_g=None, sf_u=None, sf_d=None,
                want=("ap", "o")):
    """Per-row expert stage: row r of xp goes to expert e_of[r] with gate g_of[r].

    Returns a dict with any of zg, zu [n,F] (unrounded), ap [n,F] (= g * silu(zg) * zu,
    rounded per recipe) and o [n,H] = W_d[e] ap (bf16-rounded under the bf16 and
    mxfp8 recipes), all fp64, for the rows listed (default: all).
    """
    rc = _recipe(recipe)
    R, H = xp.shape
    F = W_g.shape[1]
    if rows is None:
        rows = torch.arange(R, dtype=torch.int32)
    rows = _chk(rows.to(torch.int32).contiguous(), torch.int32)
    n = rows.numel()
    out = {w: torch.empty((n, H if w == "o" else F), dtype=torch.float64) for w in want}
    mxp, mg, mu, md = mat(xp), _wmat(W_g, sf_g), _wmat(W_u, sf_u), _wmat(W_d, sf_d)
    lib().oc_expert_rows(H, F, rc, mxp.ref, _p(_chk(e_of.to(torch.int32).contiguous(), torch.int32)),
                         _p(_chk(g_of.to(torch.float64).contiguous(), torch.float64)), mg.ref, mu.ref, md.ref,
                         n, _p(rows), _p(out.get("zg")), _p(out.get("zu")), _p(out.get("ap")), _p(out.get("o")))
    return out


def unpermute(o, row_of, shared=None):
    R, H = o.shape
    T, k = row_of.shape
    y = torch.empty((T, H), dtype=torch.float64)
    lib().oc_unpermute(T, H, k, _p(_chk(o.contiguous(), torch.float64)), _p(_chk(row_of.contiguous(), torch.int32)),
                       _p(None if shared is None else _chk(shared.contiguous(), torch.float64)), _p(y))
    return y


# ----------------------------------------------------------------- backward

def _mx_mats(mx, names):
    return [_wmat(mx[n][0], mx[n][1]) for n in names]


def moe_bwd_tokens(x, W_r, W_g, W_u, W_d, dY, r: dict, toks=None, *, score="softmax", norm=True,
                   route_scale=1.0, aux_on=True, d_aux=0.0, recipe="exact", mx=None):
    """dX[toks] (fp64, expert + router paths), dlogits[toks] [n,E] and dg [n,k] for routing r
    (the dict returned by route()).

    recipe "mxfp8" (the MXFP8 backward) takes mx = dict of (codes, scales) pairs: W_g, W_u, W_d
    (the forward's, MXFP8 along their K) and W_dT [E,F,H], W_gT, W_uT [E,H,F] (transposed, MXFP8
    along H resp. F); W_g, W_u, W_d are then ignored. "mxfp8-q" takes the same operands and
    rounds nothing to bf16."""
    T, H = x.shape
    E, F = (mx["W_g"][0] if recipe in MX_RECIPES else W_g).shape[:2]
    k = r["idx"].shape[1]
    if toks is None:
        toks = torch.arange(T, dtype=torch.int32)
    toks = _chk(toks.to(torch.int32).contiguous(), torch.int32)
    n = toks.numel()
    dx = torch.empty((n, H), dtype=torch.float64)
    dl = torch.empty((n, E), dtype=torch.float64)
    dg = torch.empty((n, k), dtype=torch.float64)
    s_soft = r["probs"] if score == "softmax" else scores(r["logits"], "softmax")
    if recipe in MX_RECIPES:
        wg, wu, wd, wdt, wgt, wut = _mx_mats(mx, ["W_g", "W_u", "W_d", "W_dT", "W_gT", "W_uT"])
    else:
        wg, wu, wd = _wmat(W_g), _wmat(W_u), _wmat(W_d)
        wdt = wgt = wut = None
    mdy = mat(dY)
    ms = [mat(x), mat(W_r), wg, wu, wd]
    tr = [m.ref if m is not None else None for m in (wdt, wgt, wut)]
    lib().oc_moe_bwd_tokens(T, H, E, k, F, 0 if score == "softmax" else 1, int(norm), ctypes.c_double(route_scale),
                            int(aux_on), ctypes.c_double(d_aux), _recipe(recipe), *[m.ref for m in ms], *tr,
                            mdy.ref,
                            _p(r["idx"]), _p(_chk(r["probs"], torch.float64)), _p(s_soft), _p(r["counts"]),
                            _p(_chk(r["keep"].contiguous(), torch.uint8)) if r.get("keep") is not None else None,
                            n, _p(toks), _p(dx), _p(dl), _p(dg))
    return dx, dl, dg


def moe_bwd_expert_dw(x, W_g, W_u, W_d, dY, idx, g, experts, recipe="exact", mx=None):
    """dW_g, dW_u [n,F,H] and dW_d [n,H,F] (fp64) for the listed experts.

    recipe "mxfp8" / "mxfp8-q" take mx as moe_bwd_tokens does (W_g, W_u, W_d, W_dT are used)."""
    T, H = x.shape
    E, F = (mx["W_g"][0] if recipe in MX_RECIPES else W_g).shape[:2]
    k = idx.shape[1]
    experts = _chk(torch.as_tensor(experts, dtype=torch.int32).contiguous(), torch.int32)
    n = experts.numel()
    dWg = torch.empty((n, F, H), dtype=torch.float64)
    dWu = torch.empty((n, F, H), dtype=torch.float64)
    dWd = torch.empty((n, H, F), dtype=torch.float64)
    if recipe in MX_RECIPES:
        wg, wu, wd, wdt = _mx_mats(mx, ["W_g", "W_u", "W_d", "W_dT"])
    else:
        wg, wu, wd, wdt = _wmat(W_g), _wmat(W_u), _wmat(W_d), None
    mdy = mat(dY)
    ms = [mat(x), wg, wu, wd]
    lib().oc_moe_bwd_expert_dw(T, H, E, k, F, _recipe(recipe), *[m.ref for m in ms],
                               wdt.ref if wdt is not None else None, mdy.ref,
                               _p(_chk(idx.contiguous(), torch.int32)),
                               _p(_chk(g.contiguous(), torch.float64)), n, _p(experts), _p(dWg), _p(dWu), _p(dWd))
    return dWg, dWu, dWd


def router_dwr(dl: torch.Tensor, x: torch.Tensor, round_dl: bool = False) -> torch.Tensor:
    T, E = dl.shape
    H = x.shape[1]
    out = torch.empty((E, H), dtype=torch.float64)
    mx_ = mat(x)
    lib().oc_router_dwr(T, H, E, _p(_chk(dl.contiguous(), torch.float64)), int(round_dl), mx_.ref, _p(out))
    return out


# ----------------------------------------------------------------- whole layer

def layer_fwd(wl, inp: dict, toks=None, logits=None, mx_weights=None, recipe=None) -> dict:
    """Full forward of workload `wl` on host inputs `inp` (synthetic.make_inputs layout).

    Routing is computed for every token; outputs y are computed for `toks`
    (default all). logits may be given (fp64/fp32 [T,E]); else the oracle's own.
    mx_weights: for the MXFP8 recipe, the oracle-quantised weights
    dict(W_g=(codes, sf), W_u=..., W_d=..., [W_gs, W_us, W_ds]); for the NVFP4
    recipe dict(W_g=(packed, sf, G), ...).
    """
    if logits is None:
        logits = router_logits(inp["x"], inp["W_r"], inp.get("logit_bias"))
    r = route(logits.to(torch.float64), wl.k, wl.score, wl.norm_topk, wl.route_scale,
              with_aux=wl.aux and wl.score == "softmax", capacity_factor=getattr(wl, "capacity_factor", 0.0),
              expert_bias=inp.get("expert_bias"), n_group=getattr(wl, "n_group", 0),
              topk_group=getattr(wl, "topk_group", 0))
    mx = wl.dtype in ("mxfp8", "nvfp4")
    if recipe is None:
        recipe = wl.dtype if mx else "exact"
    kw = {}
    if mx:
        # MXFP8: (codes, scales) pairs; NVFP4: (packed, scales, G) triples
        W = {n: (w[0], w[1] if len(w) == 2 else (w[1], w[2])) for n, w in mx_weights.items()}
        kw = dict(sf_g=W["W_g"][1], sf_u=W["W_u"][1], sf_d=W["W_d"][1])
        wg, wu, wd = W["W_g"][0], W["W_u"][0], W["W_d"][0]
        shared = None
        if wl.S:
            shared = (W["W_gs"][0], W["W_us"][0], W["W_ds"][0], W["W_gs"][1], W["W_us"][1], W["W_ds"][1])
    else:
        wg, wu, wd = inp["W_g"], inp["W_u"], inp["W_d"]
        shared = (inp["W_gs"], inp["W_us"], inp["W_ds"]) if wl.S else None
    y = moe_fwd_tokens(inp["x"], wg, wu, wd, r["idx_kept"], r["gates"], toks, recipe=recipe, shared=shared, **kw)
    r["y"] = y
    return r
