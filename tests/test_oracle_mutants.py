"""Planted mistakes in the CPU oracle, each caught by its pins (no GPU).

Every mutant below is one plausible slip in oracle/moe_oracle.c: a dropped term, a wrong sign, bound or
index, another rounding rule, a swapped operand. For each, a temporary copy of the oracle with that one
change is compiled and tests/test_oracle.py is run against it in a separate process; the run must end with
at least one failed pin. An unchanged copy run the same way must pass, so a broken harness cannot pass
these tests. Nothing here touches the CUDA path or the oracle in the tree.

Equivalent mutants (no entry point can observe them) are left out: e.g. reading every row of an NVFP4
weight with its first matrix's G, since the oracle reads expert weights only through per-expert slices.
"""
import concurrent.futures as cf
import os
import re
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

# (name, text in moe_oracle.c, replacement[, replace every occurrence])
MUTANTS = [
    # number formats
    ("bf16_round_ties_away", "u += 0x7fffu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    ("e4m3_decode_bias", "else v = ldexp(1.0 + m / 8.0, ef - 7);", "else v = ldexp(1.0 + m / 8.0, ef - 8);"),
    ("e4m3_ties_away", "else n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;", "else n = fl + 1.0;"),
    ("mx_scale_emax", "int b = e - 8 + 127;", "int b = e - 7 + 127;"),
    ("mx_matrix_scale_bias", "const double X = ldexp(1.0, (int)s[b] - 127);",
     "const double X = ldexp(1.0, (int)s[b] - 128);"),
    ("e2m1_ties_odd", "if (d < bd || (d == bd && (c & 1) == 0)) {", "if (d < bd || (d == bd && (c & 1) == 1)) {"),
    ("nvfp4_scale_divisor", "float s = amax / 6.0f;", "float s = amax / 4.0f;"),
    ("nvfp4_inverted_scale", "float r = sd > 0.0f ? G / sd : 0.0f;", "float r = sd > 0.0f ? sd / G : 0.0f;"),
    # routing
    ("router_bias_dropped", "if (bias) s += (double)bias[e];", "if (bias) s += 0.0;"),
    ("sigmoid_sign", "static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }",
     "static double sigmoid(double z) { return 1.0 / (1.0 + exp(z)); }"),
    ("softmax_denominator", "for (int e = 0; e < E; ++e) o[e] /= z;", "for (int e = 0; e < E; ++e) o[e] /= (z + 1.0);"),
    ("topk_ties_to_higher", "if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] >= l[best]) best = e;"),
    ("group_score_top1_only", "gscore[g] = (G >= 2) ? a1 + a2 : a1;", "gscore[g] = a1;"),
    ("gates_drop_route_scale", "gates[(long)t * k + j] = g * route_scale;", "gates[(long)t * k + j] = g;"),
    ("aux_f_over_T", "double f = (double)counts[e] / ((double)T * k);", "double f = (double)counts[e] / (double)T;"),
    ("capacity_off_by_one", "keep[p] = (uint8_t)(seen[e] < cap);", "keep[p] = (uint8_t)(seen[e] <= cap);"),
    ("capacity_floor", "double c = ceil(cf * (double)T * (double)k / (double)E);",
     "double c = floor(cf * (double)T * (double)k / (double)E);"),
    # permutation
    ("maps_unstable_order", "for (long p = 0; p < (long)T * k; ++p) {\n        int e = idx[p];\n        int r = fill[e]++;",
     "for (long p = (long)T * k - 1; p >= 0; --p) {\n        int e = idx[p];\n        int r = fill[e]++;"),
    ("src_of_slot_index", "src_of[r] = (int32_t)(p / k);", "src_of[r] = (int32_t)(p % k);", True),
    # experts, forward
    ("gate_up_swapped", "    matvec(Wu, xv, zu, rowbuf);\n    for (int f = 0; f < F; ++f) a[f] = silu(zg[f]) * zu[f];",
     "    matvec(Wu, xv, zu, rowbuf);\n    for (int f = 0; f < F; ++f) a[f] = silu(zu[f]) * zg[f];"),
    ("fold_drops_gate", "for (int f = 0; f < F; ++f) a[f] *= g;", "for (int f = 0; f < F; ++f) a[f] *= 1.0;"),
    # backward
    ("silu_grad_sign", "return s * (1.0 + z * (1.0 - s));", "return s * (1.0 - z * (1.0 - s));"),
    ("dzu_without_silu", "                dzu[f] = da * silu(zg[f]);", "                dzu[f] = da * zg[f];"),
    ("softmax_gate_path_sign", "dl[e] += g[j] * dg[j] - g[j] * sgd / route_scale;",
     "dl[e] += g[j] * dg[j] + g[j] * sgd / route_scale;"),
    ("sigmoid_gate_path_sign", "dl[e] += dsj * sj * (1.0 - sj);", "dl[e] -= dsj * sj * (1.0 - sj);"),
    ("softmax_unnormalised_drops_mean", "for (int e = 0; e < E; ++e) dl[e] += s[e] * (ds[e] - sds);",
     "for (int e = 0; e < E; ++e) dl[e] += s[e] * ds[e];"),
    ("aux_backward_drops_mean", "dl[e] += d_aux * ss[e] * (ce - sc);", "dl[e] += d_aux * ss[e] * ce;"),
    ("wd_grad_drops_gate", "for (int f = 0; f < F; ++f) a[f] *= gl[i];", "for (int f = 0; f < F; ++f) a[f] *= 1.0;"),
    ("dz_grad_drops_gate", "                double da = gl[i] * v[f];", "                double da = v[f];"),
    ("dwg_uses_dzu", "gG[(long)f * H + h] += cg * xv[h];", "gG[(long)f * H + h] += cu * xv[h];"),
    ("dx_drops_up_path", "                matvec_t_acc(&we_u, dzu, dxp, rowbuf);\n", ""),
    ("dx_drops_router_path", "            for (int h = 0; h < H; ++h) dxp[h] += c * rowbuf[h];",
     "            for (int h = 0; h < H; ++h) dxp[h] += 0.0 * c * rowbuf[h];"),
    ("router_dwr_transposed", "double c = dl[(long)t * E + e];", "double c = dl[(long)e * T + t];"),
    ("router_dwr_unrounded_dl", "if (round_dl) c = oc_bf16_round(c);", "if (0) c = oc_bf16_round(c);"),
    # precision recipes and block-scaled matrices
    ("mx_recipe_skips_x", "        if (is_mx(recipe)) mx_roundtrip(xv, H);\n        else if (is_nv(recipe)) nv_roundtrip(xv, H);"
     "\n        for (int h = 0; h < H; ++h) y[h] = 0.0;",
     "        if (0) mx_roundtrip(xv, H);\n        else if (is_nv(recipe)) nv_roundtrip(xv, H);"
     "\n        for (int h = 0; h < H; ++h) y[h] = 0.0;"),
    ("bf16_recipe_skips_act", "else if (recipe == OC_BF16R) round_vec(a, F, recipe);", "else if (0) round_vec(a, F, recipe);"),
    ("mx_roundtrip_scale_off", "        uint8_t sb = oc_mx_scale_byte(amax);\n        double X = ldexp(1.0, (int)sb - 127);"
     "\n        for (int i = 0; i < 32; ++i)",
     "        uint8_t sb = oc_mx_scale_byte(amax);\n        double X = ldexp(1.0, (int)sb - 126);"
     "\n        for (int i = 0; i < 32; ++i)"),
    ("mx_strided_ignores_stride", "t[i] = (float)v[(b0 + i) * stride];", "t[i] = (float)v[b0 + i];"),
    ("nv_roundtrip_drops_scale", "for (int i = 0; i < 16; ++i) v[b * 16 + i] = oc_e2m1_decode(c[i]) * sd;",
     "for (int i = 0; i < 16; ++i) v[b * 16 + i] = oc_e2m1_decode(c[i]);"),
    ("nvfp4_matrix_multiplies_G", "out[c] = g_e2m1[code] * g_e4m3[s[c / 16]] / G;",
     "out[c] = g_e2m1[code] * g_e4m3[s[c / 16]] * G;"),
    ("nvfp4_slice_keeps_first_G", "if (m->gs) s.gs = m->gs + r0 / m->gs_rows;", "if (m->gs) s.gs = m->gs;"),
    ("nvfp4_pack_nibbles_swapped", "(uint8_t)(c[2 * i] | (c[2 * i + 1] << 4))", "(uint8_t)(c[2 * i + 1] | (c[2 * i] << 4))",
     True),
    ("nvfp4_read_nibbles_swapped", "uint8_t code = (p[c / 2] >> (4 * (c & 1))) & 15;",
     "uint8_t code = (p[c / 2] >> (4 * (1 - (c & 1)))) & 15;"),
    # forward output
    ("shared_expert_dropped", "            for (int h = 0; h < H; ++h) y[h] += o[h];\n            if (shared_out)",
     "            for (int h = 0; h < H; ++h) y[h] += 0.0 * o[h];\n            if (shared_out)"),
    ("unfolded_path_drops_gate", "for (int h = 0; h < H; ++h) y[h] += g * o[h];", "for (int h = 0; h < H; ++h) y[h] += o[h];"),
    ("unpermute_drops_shared", "if (shared) s += shared[(long)t * H + h];", "if (shared) s += 0.0;"),
    ("unpermute_first_slot_only", "for (int j = 0; j < k; ++j) s += o[(long)row_of[(long)t * k + j] * H + h];",
     "for (int j = 0; j < 1; ++j) s += o[(long)row_of[(long)t * k + j] * H + h];"),
    # more number-format edges
    ("e4m3_no_subnormal_quantum", "    if (e < -6) e = -6;                     /* subnormal range shares the 2^-9 quantum */\n",
     ""),
    ("e4m3_saturates_too_high", "if (val > 448.0) val = 448.0;", "if (val > 480.0) val = 480.0;"),
    ("nvfp4_global_scale_constant", "return amax > 0.0f ? 2688.0f / amax : 1.0f;", "return amax > 0.0f ? 448.0f / amax : 1.0f;"),
    # grouped router
    ("group_filter_ignored", "if (!gkeep[e / G]) continue;", "if (0) continue;"),
    ("group_second_best_not_updated", "else if (v[e] > a2) { a2 = v[e]; }", "else if (0) { a2 = v[e]; }"),
    ("group_ties_to_higher", "if (best < 0 || gscore[g] > gscore[best]) best = g;", "if (best < 0 || gscore[g] >= gscore[best]) best = g;"),
    # aux and backward details
    ("aux_without_E", "    return (double)E * acc;", "    return acc;"),
    ("bwd_gates_unnormalised", "            if (norm) gj /= Z;\n            g[j] = gj * route_scale;",
     "            g[j] = gj * route_scale;"),
    ("bwd_dropped_pair_contributes", "dg[j] = 0.0; /* dropped at capacity: the output does not depend on its gate */\n"
     "                continue;", "dg[j] = 0.0; /* dropped at capacity: the output does not depend on its gate */"),
    ("sigmoid_unnormalised_drops_slope", "dl[e] += route_scale * dg[j] * sj * (1.0 - sj);",
     "dl[e] += route_scale * dg[j] * sj;"),
    ("expert_dw_silu_instead_of_grad", "DZG[(long)i * F + f] = da * zu[f] * silu_grad(zg[f]);",
     "DZG[(long)i * F + f] = da * zu[f] * silu(zg[f]);"),
    ("mx_dgrad_reads_forward_weight", "oc_mat wt_d = oc_slice(WdT, (int64_t)e * F, F);   /* W_d^T [F, H], MXFP8 along H */\n"
     "                matvec(&wt_d, dye, v, rowbuf);",
     "for (int f = 0; f < F; ++f) v[f] = 0.0;\n                matvec_t_acc(&we_d, dye, v, rowbuf);"),
    # the quantisation-points-only recipes
    ("mxq_skips_mx_quantisation", "static int is_mx(int recipe) { return recipe == OC_MX || recipe == OC_MXQ; }",
     "static int is_mx(int recipe) { return recipe == OC_MX; }"),
    ("nvq_skips_nv_quantisation", "static int is_nv(int recipe) { return recipe == OC_NV || recipe == OC_NVQ; }",
     "static int is_nv(int recipe) { return recipe == OC_NV; }"),
    ("q_recipes_round_expert_outputs", "if (recipe == OC_BF16R || recipe == OC_MX || recipe == OC_NV)\n",
     "if (recipe != OC_EXACT)\n"),
    ("mxq_rounds_saved_z_in_weight_grads", "                if (recipe == OC_MX)\n                    for (int f = 0; f < F; ++f) { zg[f]",
     "                if (is_mx(recipe))\n                    for (int f = 0; f < F; ++f) { zg[f]"),
]


def _run_pins(workdir: str, source: str):
    """Compile `source` as the oracle of a scratch tree and run tests/test_oracle.py against it."""
    os.makedirs(os.path.join(workdir, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), os.path.join(workdir, "oracle"))
    with open(os.path.join(workdir, "oracle", "moe_oracle.c"), "w") as f:
        f.write(source)
    os.makedirs(os.path.join(workdir, "tests"))
    for name in ("conftest.py", "test_oracle.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(workdir, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(workdir, "tests", "golden"))
    # the scratch tree's oracle first; the synthetic-input module from the repository
    env = dict(os.environ, PYTHONPATH=workdir + os.pathsep + ROOT, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "tests/test_oracle.py"],
                       cwd=workdir, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.fixture(scope="module")
def outcomes():
    with open(SRC) as f:
        src = f.read()
    jobs = {"(unchanged)": src}
    for m in MUTANTS:
        name, old, new = m[:3]
        every = len(m) > 3 and m[3]
        n = src.count(old)
        assert n == 1 or (every and n > 1), f"{name}: the text to change occurs {n} times"
        jobs[name] = src.replace(old, new)
    tmp = tempfile.mkdtemp(prefix="oracle_mutants_")
    try:
        with cf.ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1))) as ex:
            futs = {name: ex.submit(_run_pins, os.path.join(tmp, f"m{i}"), s) for i, (name, s) in enumerate(jobs.items())}
            yield {name: fu.result() for name, fu in futs.items()}
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def test_unchanged_oracle_passes_its_pins_in_the_harness(outcomes):
    rc, out = outcomes["(unchanged)"]
    assert rc == 0, out


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(outcomes, name):
    rc, out = outcomes[name]
    # a pin failed (not a crash, a build error or an error in a fixture)
    assert rc == 1 and re.search(r"\b1 failed\b", out) and not re.search(r"\berror", out.splitlines()[-1]), out
