"""Device-side checks of the routing metadata, fed host-made corrupted inputs.

The expert indices and the per-expert offsets are where a MoE layer's bugs live (the study notes' 案例 1
读法: index, capacity and alignment metadata). Both are produced on the device in the layer, so nothing on
the host can validate them; the kernels do:

  moe_permute           an expert index outside [0, E), or one a token already chose, is recorded as
                        status 0x202 (bad index) and that (token, slot) pair is dropped: it gets no row
                        (row_of = -1) and counts only the valid pairs;
  grouped GEMMs         offsets that are not monotone, start below 0 or end past the rows are recorded as
                        status 0x201 (bad offsets) and the GEMM computes nothing: no tile is loaded or stored.

Every output buffer sits between canary bytes, which must be untouched afterwards; the status word is read
and cleared, so the tests that follow start clean.
"""
import pytest
import torch

from mixture_experts_layer_aux_b200.synthetic import random_gates, random_routing, randn_bf16

pytestmark = pytest.mark.gpu

DEV_BAD_OFFSETS, DEV_BAD_INDEX = 0x201, 0x202
PAD = 4096  # canary bytes before and after every output


class Guarded:
    """A device buffer of `shape`/`dtype` with PAD canary bytes on both sides."""

    def __init__(self, shape, dtype, fill=0x5A):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((PAD + nbytes + PAD,), fill, dtype=torch.uint8, device="cuda")
        self.nbytes = nbytes
        self.t = self.raw[PAD:PAD + nbytes].view(dtype).view(shape)
        self.fill = fill

    def canaries_intact(self):
        r = self.raw.cpu()
        return bool((r[:PAD] == self.fill).all()) and bool((r[PAD + self.nbytes:] == self.fill).all())

    def untouched(self):
        return bool((self.raw.cpu() == self.fill).all())


def _read_status(moe):
    return moe.moe_get_device_status(clear=True)


@pytest.mark.parametrize("dtype", [0, 1])
def test_permute_flags_and_drops_bad_expert_indices(moe, oracle, dtype):
    T, H, E, k = 300, 256, 16, 4
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=128, expert_dtype=dtype)
    idx = random_routing(T, E, k, seed=41)
    bad = torch.zeros(T, k, dtype=torch.bool)
    idx[5, 2], bad[5, 2] = E + 3, True           # past the last expert
    idx[7, 1], bad[7, 1] = -2, True              # negative
    idx[11, 3], bad[11, 3] = int(idx[11, 0]), True   # a token choosing the same expert twice: the later slot
    idx[299, 0], bad[299, 0] = 1 << 30, True     # far out of range, in the last (partial) rank block
    x = randn_bf16((T, H), 1.0, seed=42)
    g = random_gates(T, k, seed=43)
    rows = T * k
    out = dict(counts=Guarded((E,), torch.int32), offsets=Guarded((E + 1,), torch.int32),
               row_of=Guarded((T, k), torch.int32), src_of=Guarded((rows,), torch.int32),
               row_gate=Guarded((rows,), torch.float32),
               xp=Guarded((rows, H), torch.uint8 if dtype else torch.bfloat16),
               xp_sf=Guarded((rows, H // 32), torch.uint8) if dtype else None)
    assert _read_status(moe) == 0
    moe.moe_permute(cfg, x.cuda(), idx.cuda(), g.cuda(), out["counts"].t, out["offsets"].t, out["row_of"].t,
                    out["src_of"].t, out["row_gate"].t, out["xp"].t, None if out["xp_sf"] is None else out["xp_sf"].t,
                    moe.workspace(moe.moe_permute_workspace_size(cfg)))
    torch.cuda.synchronize()
    assert _read_status(moe) == DEV_BAD_INDEX
    for name, buf in out.items():
        if buf is not None:
            assert buf.canaries_intact(), name
    # the valid pairs, as the oracle maps them with the bad ones dropped
    keep = (~bad).to(torch.uint8)
    kc, off, ro, so = oracle.maps(torch.where(bad, torch.zeros_like(idx), idx), E, keep)
    assert torch.equal(out["counts"].t.cpu(), kc) and torch.equal(out["offsets"].t.cpu(), off)
    assert torch.equal(out["row_of"].t.cpu(), ro)
    assert bool((out["row_of"].t.cpu()[bad] == -1).all())
    n = int(off[-1])
    assert n == rows - int(bad.sum())
    assert torch.equal(out["src_of"].t.cpu()[:n], so[:n])
    kp = keep.bool()
    rg_ref = torch.empty(n, dtype=torch.float32)
    rg_ref[ro[kp].long()] = g[kp]
    assert torch.equal(out["row_gate"].t.cpu()[:n], rg_ref)
    if dtype == 0:
        assert torch.equal(out["xp"].t.cpu()[:n].view(torch.int16), x[so[:n].long()].view(torch.int16))
    else:
        codes, sf = oracle.mxfp8_quantize(x[so[:n].long()])
        assert torch.equal(out["xp"].t.cpu()[:n], codes) and torch.equal(out["xp_sf"].t.cpu()[:n], sf)
    # rows past the valid ones are never written
    xb = out["xp"].raw.cpu()[PAD:PAD + out["xp"].nbytes].view(rows, -1)
    assert bool((xb[n:] == out["xp"].fill).all())
    assert _read_status(moe) == 0


def _offsets_cases(rows, E):
    good = torch.linspace(0, rows, E + 1).round().to(torch.int32)
    non_monotone = good.clone()
    non_monotone[3] = int(good[4])          # offsets[3] > offsets[4]
    non_monotone[4] = int(good[3])
    past_end = good.clone()
    past_end[-1] = rows + 128
    negative = good.clone()
    negative[0] = -128
    return {"non-monotone": non_monotone, "past the rows": past_end, "negative start": negative}


@pytest.mark.parametrize("case", ["non-monotone", "past the rows", "negative start"])
@pytest.mark.parametrize("which", [0, 1])
@pytest.mark.parametrize("dtype", [0, 1])
def test_grouped_gemm_flags_bad_offsets_and_writes_nothing(moe, case, which, dtype):
    T, H, E, k, F = 256, 512, 8, 2, 256
    rows = T * k
    cfg = moe.make_config(T=T, H=H, E=E, k=k, F=F, expert_dtype=dtype)
    off = _offsets_cases(rows, E)[case].cuda()
    K, N = (H, F) if which == 0 else (F, H)
    if dtype == 0:
        A = randn_bf16((rows, K), 1.0, seed=51, device="cuda")
        B0 = randn_bf16((E, N, K), 0.02, seed=52, device="cuda")
        B1 = randn_bf16((E, N, K), 0.02, seed=53, device="cuda") if which == 0 else None
        A_sf = B0_sf = B1_sf = None
    else:
        def q(t):
            c = torch.empty(t.shape, dtype=torch.uint8, device="cuda")
            s = torch.empty(t.shape[:-1] + (t.shape[-1] // 32,), dtype=torch.uint8, device="cuda")
            moe.moe_quantize_mxfp8(t, c, s)
            return c, s
        A, A_sf = q(randn_bf16((rows, K), 1.0, seed=51, device="cuda"))
        B0, B0_sf = q(randn_bf16((E, N, K), 0.02, seed=52, device="cuda"))
        B1, B1_sf = q(randn_bf16((E, N, K), 0.02, seed=53, device="cuda")) if which == 0 else (None, None)
    gate = torch.rand(rows, device="cuda") if which == 0 else None
    if dtype == 1 and which == 0:
        C, C_sf = Guarded((rows, N), torch.uint8), Guarded((rows, N // 32), torch.uint8)
    else:
        C, C_sf = Guarded((rows, N), torch.bfloat16), None
    save = Guarded((rows, 2 * F), torch.bfloat16) if which == 0 else None
    torch.cuda.synchronize()
    assert _read_status(moe) == 0
    moe.moe_grouped_gemm_fwd(cfg, which, A, A_sf, B0, B0_sf, B1, B1_sf, off, gate, C.t,
                             None if C_sf is None else C_sf.t, None if save is None else save.t,
                             moe.workspace(moe.moe_grouped_gemm_workspace_size(cfg, which)))
    torch.cuda.synchronize()
    assert _read_status(moe) == DEV_BAD_OFFSETS
    for b in (C, C_sf, save):
        if b is not None:
            assert b.untouched()
    assert _read_status(moe) == 0
