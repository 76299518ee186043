"""The C-ABI library: loads, exports what include/moe.h declares, and rejects
bad arguments on the host before anything is launched (no GPU needed).

Every call below fails validation before any CUDA call, so the (fake,
never-dereferenced) pointer values are safe on any machine.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

OK, INVALID, UNSUPPORTED, ALIGN, WS = 0, 1, 2, 3, 4


@pytest.fixture(scope="module")
def lib():
    from mixture_experts_layer_aux_b200 import binding
    return binding.load()


@pytest.fixture(scope="module")
def B():
    from mixture_experts_layer_aux_b200 import binding
    binding.load()
    return binding


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_layer_entry_points():
    names = declared_functions()
    for n in ["moe_router_topk", "moe_permute", "moe_grouped_gemm_fwd", "moe_grouped_gemm_bwd", "moe_unpermute",
              "moe_layer_fwd", "moe_layer_bwd", "moe_quantize_mxfp8"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib, B):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in B.exported_symbols(), n   # and the binding wraps it


def test_library_is_built_for_sm100a():
    from mixture_experts_layer_aux_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)
    assert os.path.exists(build.LIB)


def test_status_strings(lib):
    for s in range(7):
        assert lib.moe_status_string(s)
    assert b"WORKSPACE" in lib.moe_status_string(WS)


def cfg(B, **kw):
    base = dict(T=512, H=256, E=8, k=2, F=512)
    base.update(kw)
    return B.make_config(**base)


FAKE = 0x10000  # aligned, never dereferenced (every call fails validation first)


def test_config_validation(lib, B):
    c = cfg(B)
    assert lib.moe_router_workspace_size(ctypes.byref(c)) > 0
    for bad, code in [(dict(k=9), UNSUPPORTED), (dict(k=0), INVALID), (dict(E=600, k=2), UNSUPPORTED),
                      (dict(H=200), UNSUPPORTED), (dict(F=100), UNSUPPORTED), (dict(T=0), INVALID),
                      (dict(score=5), INVALID), (dict(n_shared=2), UNSUPPORTED),
                      (dict(compute_aux=1, score=1), UNSUPPORTED), (dict(capacity_factor=-1.0), INVALID),
                      (dict(capacity_factor=float("nan")), INVALID), (dict(capacity_factor=float("inf")), INVALID),
                      (dict(n_group=3), INVALID), (dict(n_group=4, topk_group=0), INVALID),
                      (dict(n_group=4, topk_group=5), INVALID), (dict(n_group=33), INVALID),
                      (dict(n_group=4, topk_group=1, k=3), INVALID)]:
        c = cfg(B, **bad)
        assert lib.moe_router_workspace_size(ctypes.byref(c)) == 0
        rc = lib.moe_router_topk(ctypes.byref(c), FAKE, FAKE, None, None, FAKE, None, FAKE, FAKE, None, None, FAKE, 1 << 30,
                                 None)
        assert rc == code, (bad, rc)


def test_router_argument_errors(lib, B):
    c = cfg(B)
    ws = lib.moe_router_workspace_size(ctypes.byref(c))
    f = lib.moe_router_topk
    assert f(ctypes.byref(c), FAKE, FAKE, None, None, None, None, FAKE, FAKE, None, None, FAKE, ws, None) == INVALID
    assert f(ctypes.byref(c), FAKE, None, None, None, FAKE, None, FAKE, FAKE, None, None, FAKE, ws, None) == INVALID
    assert f(ctypes.byref(c), FAKE + 2, FAKE, None, None, FAKE, None, FAKE, FAKE, None, None, FAKE, ws, None) == ALIGN
    assert f(ctypes.byref(c), FAKE, FAKE, None, None, FAKE, None, FAKE, FAKE, None, None, FAKE, ws - 1, None) == WS
    assert f(ctypes.byref(c), FAKE, FAKE, None, None, FAKE, None, FAKE, FAKE, None, None, None, ws, None) == WS
    # aux requested without compute_aux
    assert f(ctypes.byref(c), FAKE, FAKE, None, None, FAKE, None, FAKE, FAKE, None, FAKE, FAKE, ws, None) == INVALID


def test_permute_argument_errors(lib, B):
    c = cfg(B)
    ws = lib.moe_permute_workspace_size(ctypes.byref(c))
    f = lib.moe_permute
    assert f(ctypes.byref(c), FAKE, None, None, None, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, ws, None) == INVALID
    assert f(ctypes.byref(c), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws, None) == INVALID
    assert f(ctypes.byref(c), FAKE + 4, FAKE, None, None, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, ws, None) == ALIGN
    assert f(ctypes.byref(c), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, ws - 1, None) == WS
    cm = cfg(B, expert_dtype=1)
    assert f(ctypes.byref(cm), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, ws, None) == INVALID


def test_gemm_and_layer_argument_errors(lib, B):
    c = cfg(B)
    g = lib.moe_grouped_gemm_fwd
    ws = lib.moe_grouped_gemm_workspace_size(ctypes.byref(c), 0)
    assert g(ctypes.byref(c), 7, FAKE, None, FAKE, None, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, ws,
             None) == INVALID
    assert g(ctypes.byref(c), 0, FAKE, None, FAKE, None, None, None, FAKE, FAKE, FAKE, None, None, FAKE, ws,
             None) == INVALID
    assert g(ctypes.byref(c), 0, FAKE, None, FAKE + 8, None, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, ws,
             None) == ALIGN
    assert g(ctypes.byref(c), 0, FAKE, None, FAKE, None, FAKE, None, FAKE, FAKE, FAKE, None, None, None, ws,
             None) == WS
    lw = lib.moe_layer_workspace_size(ctypes.byref(c))
    assert lw > lib.moe_layer_saved_size(ctypes.byref(c)) // 8
    L = lib.moe_layer_fwd
    args = [FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, None, None, None, None, None, None, None, None, FAKE, None,
            None, None, None, None, None]
    assert L(ctypes.byref(c), *args, FAKE, lw - 1, None) == WS
    args2 = list(args)
    args2[0] = None
    assert L(ctypes.byref(c), *args2, FAKE, lw, None) == INVALID
    cs = cfg(B, save_for_bwd=1)
    assert L(ctypes.byref(cs), *args, FAKE, lw, None) == INVALID     # saved buffer missing
    csh = cfg(B, n_shared=1)
    assert L(ctypes.byref(csh), *args, FAKE, lw, None) == INVALID    # shared weights missing
    u = lib.moe_unpermute
    assert u(ctypes.byref(c), FAKE, None, None, FAKE, None) == INVALID
    assert u(ctypes.byref(c), FAKE + 1, FAKE, None, FAKE, None) == ALIGN
    q = lib.moe_quantize_mxfp8
    assert q(FAKE, 4, 48, FAKE, FAKE, None) == UNSUPPORTED
    assert q(None, 4, 64, FAKE, FAKE, None) == INVALID
    bw = lib.moe_layer_bwd
    cb = cfg(B, save_for_bwd=1)
    bws = lib.moe_layer_bwd_workspace_size(ctypes.byref(cb))
    assert bw(ctypes.byref(cb), FAKE, ctypes.c_float(0.0), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
              FAKE, None, FAKE, bws - 1, None) == WS
    cbm = cfg(B, expert_dtype=1)
    assert bw(ctypes.byref(cbm), FAKE, ctypes.c_float(0.0), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
              FAKE, None, FAKE, bws, None) == UNSUPPORTED


def test_nvfp4_argument_errors(lib, B):
    # scale-buffer size: batch*R*C/16 scale bytes + batch fp32 encode scales
    assert lib.moe_nvfp4_sf_bytes(2, 3, 32) == 2 * 3 * 2 + 8
    assert lib.moe_nvfp4_sf_bytes(1, 4, 24) == 0
    q = lib.moe_quantize_nvfp4
    assert q(FAKE, 1, 128, 48, FAKE, FAKE, None) == UNSUPPORTED     # C % 64 != 0 (whole scale chunks)
    assert q(FAKE, 1, 100, 64, FAKE, FAKE, None) == UNSUPPORTED     # R % 128 != 0
    assert q(FAKE, 1, 128, 8, FAKE, FAKE, None) == INVALID          # C < 16
    assert q(None, 1, 128, 64, FAKE, FAKE, None) == INVALID
    assert q(FAKE, 1, 128, 64, FAKE, FAKE + 4, None) == ALIGN       # sf is bulk-copied: 16-byte aligned
    qa = lib.moe_quantize_nvfp4_act
    assert qa(FAKE, 4, 24, FAKE, FAKE, None) == UNSUPPORTED
    assert qa(FAKE + 8, 4, 32, FAKE, FAKE, None) == ALIGN
    c = cfg(B, H=512, F=384, expert_dtype=B.MOE_DT_NVFP4)           # NVFP4 needs F % 256 == 0
    lw = lib.moe_layer_workspace_size(ctypes.byref(c))
    L = lib.moe_layer_fwd
    args = [FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, None, None, None, FAKE, None,
            None, None, None, None, None]
    assert L(ctypes.byref(c), *args, FAKE, lw, None) == UNSUPPORTED
    cs = cfg(B, H=512, F=512, expert_dtype=B.MOE_DT_NVFP4, save_for_bwd=1)  # no NVFP4 backward
    assert lib.moe_layer_saved_size(ctypes.byref(cs)) == 0
    args_s = list(args)
    args_s[22] = FAKE  # saved
    assert L(ctypes.byref(cs), *args_s, FAKE, lib.moe_layer_workspace_size(ctypes.byref(cs)), None) == UNSUPPORTED
    g = lib.moe_grouped_gemm_fwd
    ws = lib.moe_grouped_gemm_workspace_size(ctypes.byref(c), 0)
    assert g(ctypes.byref(c), 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws,
             None) == UNSUPPORTED
    c2 = cfg(B, H=512, F=512, expert_dtype=B.MOE_DT_NVFP4)
    assert g(ctypes.byref(c2), 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws,
             None) == INVALID  # save_gateup is not supported


def test_backward_argument_errors(lib, B):
    # BF16 grouped backward GEMMs
    c = cfg(B)
    gb = lib.moe_grouped_gemm_bwd
    wsb = lib.moe_grouped_gemm_bwd_workspace_size(ctypes.byref(c), 1)
    assert gb(ctypes.byref(cfg(B, expert_dtype=1)), 1, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None,
              None, FAKE, wsb, None) == UNSUPPORTED
    assert gb(ctypes.byref(c), 1, None, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, wsb,
              None) == INVALID                                                      # dO missing
    assert gb(ctypes.byref(c), 1, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, None, FAKE, wsb,
              None) == INVALID                                                      # dgrad without W_d
    assert gb(ctypes.byref(c), 1, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, wsb - 1,
              None) == WS
    assert gb(ctypes.byref(c), 7, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, FAKE, wsb,
              None) == INVALID                                                      # no such GEMM
    # MXFP8 transposed quantisers
    qt = lib.moe_quantize_mxfp8_t
    assert qt(None, 1, 64, 64, FAKE, 64, FAKE, None) == INVALID
    assert qt(FAKE, 0, 64, 64, FAKE, 64, FAKE, None) == INVALID
    assert qt(FAKE, 1, 48, 64, FAKE, 64, FAKE, None) == UNSUPPORTED                # R % 32 != 0
    assert qt(FAKE, 1, 64, 12, FAKE, 64, FAKE, None) == UNSUPPORTED                # C % 8 != 0
    assert qt(FAKE, 1, 64, 64, FAKE, 32, FAKE, None) == UNSUPPORTED                # ldd < R
    assert qt(FAKE, 1, 64, 64, FAKE, 80, FAKE, None) == UNSUPPORTED                # ldd % 32 != 0
    assert qt(FAKE + 8, 1, 64, 64, FAKE, 64, FAKE, None) == ALIGN
    assert qt(FAKE, 1, 64, 64, FAKE + 8, 64, FAKE, None) == ALIGN                 # dst: 16-byte code runs
    cm = cfg(B, expert_dtype=1)
    ldp = lib.moe_mxfp8_t_padded_rows(ctypes.byref(cm))
    T, k, E = 512, 2, 8
    assert ldp == -(-(T * k + 128 * E) // 512) * 512                                # each expert padded to 128 rows
    assert lib.moe_mxfp8_t_padded_rows(ctypes.byref(cfg(B, k=0))) == 0
    qg = lib.moe_quantize_mxfp8_t_grouped
    assert qg(ctypes.byref(cm), 3, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, ldp, FAKE, None) == INVALID   # mode
    assert qg(ctypes.byref(cm), 1, FAKE, None, None, FAKE, FAKE, 256, FAKE, ldp, FAKE, None) == INVALID   # no src_of
    assert qg(ctypes.byref(cm), 2, FAKE, None, None, FAKE, FAKE, 256, FAKE, ldp, FAKE, None) == INVALID   # no gate
    assert qg(ctypes.byref(cm), 0, FAKE, None, None, FAKE, FAKE, 96, FAKE, ldp, FAKE, None) == UNSUPPORTED
    assert qg(ctypes.byref(cm), 0, FAKE, None, None, FAKE, FAKE, 256, FAKE, ldp - 512, FAKE, None) == INVALID
    assert qg(ctypes.byref(cm), 0, FAKE, None, None, FAKE, FAKE, 256, FAKE, ldp + 32, FAKE, None) == INVALID
    assert qg(ctypes.byref(cm), 0, FAKE + 4, None, None, FAKE, FAKE, 256, FAKE, ldp, FAKE, None) == ALIGN
    assert qg(ctypes.byref(cm), 0, FAKE, None, None, FAKE, FAKE, 256, FAKE + 4, ldp, FAKE, None) == ALIGN
    # MXFP8 grouped data- and weight-gradient GEMMs
    dg = lib.moe_grouped_gemm_dgrad_mxfp8
    need = T * k * (512 // 128) * 4
    assert dg(ctypes.byref(cfg(B, expert_dtype=1, F=384)), 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
              FAKE, need, None) == UNSUPPORTED                                      # F % 256 != 0
    assert dg(ctypes.byref(cm), 1, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == INVALID
    assert dg(ctypes.byref(cm), 1, FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need,
              None) == ALIGN
    assert dg(ctypes.byref(cm), 1, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, need,
              None) == INVALID                                                      # SwiGLU backward needs gate/up
    assert dg(ctypes.byref(cm), 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 4,
              None) == WS
    assert dg(ctypes.byref(cm), 7, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None, None, 0, None) == INVALID
    wg = lib.moe_grouped_gemm_wgrad_mxfp8
    assert wg(ctypes.byref(cm), 1, None, FAKE, FAKE, FAKE, FAKE, ldp, FAKE, None, None) == INVALID
    assert wg(ctypes.byref(cm), 1, FAKE, FAKE, FAKE, FAKE, FAKE, ldp - 512, FAKE, None, None) == INVALID
    assert wg(ctypes.byref(cm), 1, FAKE, FAKE, FAKE, FAKE, FAKE, ldp + 32, FAKE, None, None) == INVALID
    assert wg(ctypes.byref(cm), 0, FAKE, FAKE, FAKE, FAKE, FAKE, ldp, FAKE, None, None) == INVALID   # gate/up: dW_u
    assert wg(ctypes.byref(cm), 7, FAKE, FAKE, FAKE, FAKE, FAKE, ldp, FAKE, FAKE, None) == INVALID
    # MXFP8 layer backward
    lb = lib.moe_layer_bwd_mxfp8
    cmb = cfg(B, expert_dtype=1, save_for_bwd=1)
    lws = lib.moe_layer_bwd_mxfp8_workspace_size(ctypes.byref(cmb))
    assert lws > 0
    args = [FAKE, ctypes.c_float(0.0), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None]
    assert lb(ctypes.byref(cfg(B, save_for_bwd=1)), *args, FAKE, lws, None) == INVALID     # not an MXFP8 layer
    assert lb(ctypes.byref(cfg(B, expert_dtype=1, save_for_bwd=1, n_shared=1)), *args, FAKE, lws,
              None) == UNSUPPORTED                                                  # no shared-expert backward
    bad = list(args)
    bad[0] = None
    assert lb(ctypes.byref(cmb), *bad, FAKE, lws, None) == INVALID                  # dY missing
    bad = list(args)
    bad[2] = FAKE + 8
    assert lb(ctypes.byref(cmb), *bad, FAKE, lws, None) == ALIGN                    # x
    bad = list(args)
    bad[5] = FAKE + 2
    assert lb(ctypes.byref(cmb), *bad, FAKE, lws, None) == ALIGN                    # W_d^T scales: 4-byte aligned
    assert lb(ctypes.byref(cmb), *args, FAKE, lws - 1, None) == WS
