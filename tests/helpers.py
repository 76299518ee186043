"""Shared helpers of the GPU parity tests (comparison metrics, buffers)."""
import torch

# Floating-point bars: max |err| <= TOL * rms(ref) over the compared tensor.
TOL_BF16 = 2e-2
TOL_MXFP8 = 6e-2
# NVFP4 against an oracle that quantises at the same points: the block-scaled bar of MXFP8 (the two sides
# differ only by fp32-vs-fp64 accumulation and the rare E2M1 / E4M3 rounding decisions it moves)
TOL_NVFP4 = 6e-2


def rms(t: torch.Tensor) -> float:
    t = t.detach().double().cpu()
    return float(t.pow(2).mean().sqrt())


def err_rms(got: torch.Tensor, ref: torch.Tensor) -> float:
    """max |got - ref| / rms(ref) (both moved to host fp64)."""
    g = got.detach().double().cpu()
    r = ref.detach().double().cpu()
    assert g.shape == r.shape, (g.shape, r.shape)
    d = (g - r).abs().max().item() if g.numel() else 0.0
    den = float(r.pow(2).mean().sqrt()) if r.numel() else 1.0
    return d / max(den, 1e-30)


def e_of_rows(offsets: torch.Tensor) -> torch.Tensor:
    """Expert index of every row of the expert-contiguous order."""
    off = offsets.long().cpu()
    R = int(off[-1])
    return (torch.bucketize(torch.arange(R), off[1:], right=True)).to(torch.int32)


def empty(shape, dtype, device="cuda"):
    return torch.empty(shape, dtype=dtype, device=device)


def bf16_of(t: torch.Tensor) -> torch.Tensor:
    """fp64 -> fp32 -> bf16 (round to nearest even) -> fp64, via torch's casts."""
    return t.double().float().bfloat16().double()


def check_bf16(got: torch.Tensor, ref: torch.Tensor, tol: float = TOL_BF16, max_flip_frac: float = 1e-3,
               terms: int = 1):
    """Compare a bf16 kernel output with the oracle's value of the same tensor under identical quantisation.

    `ref` is the oracle's value before the output's own bf16 rounding, computed with the kernels' bf16
    rounding applied at every earlier point. Every element must lie within tol * rms(ref) of bf16(ref),
    except elements downstream of a rounding decision that the two sides took differently (their fp32 and
    fp64 values before a rounding point straddled a bf16 rounding boundary). Such an element is a sum of
    `terms` rounded contributions (the k experts' rows, a router term, ...); each flipped contribution moves
    it by one bf16 ulp of that contribution, which is at most one ulp of the largest element of its row,
    and its own rounding adds one more: it may differ by at most (terms + 1) such ulps, and at most
    max_flip_frac of the elements may do so.
    Returns (max |got - bf16(ref)| / rms, max |got - ref| / rms, flips).
    """
    g = got.detach().double().cpu()
    r = ref.detach().double().cpu()
    assert g.shape == r.shape, (g.shape, r.shape)
    r16 = bf16_of(r)
    den = max(float(r.pow(2).mean().sqrt()), 1e-30)
    d = (g - r16).abs()
    bad = d > tol * den
    flips = int(bad.sum())
    if flips:
        rows = r.reshape(-1, r.shape[-1]) if r.dim() >= 2 else r.reshape(1, -1)
        rowmax = rows.abs().amax(dim=1, keepdim=True).expand_as(rows).reshape(r.shape)
        mag = torch.maximum(torch.maximum(r16.abs(), g.abs()), rowmax).clamp_min(1e-38)
        ulp = torch.pow(2.0, torch.floor(torch.log2(mag)) - 7)
        allow = (terms + 1) * ulp * (1 + 1e-9)
        assert bool((d[bad] <= allow[bad]).all()), \
            f"elements beyond {tol}*rms more than {terms + 1} bf16 ulps of their row apart: " \
            f"max {float(d.max()) / den:.3g} rms"
        assert flips <= max(1, max_flip_frac * g.numel()), f"{flips} rounding-flip differences beyond {tol}*rms"
    return float(d.max()) / den, float((g - r).abs().max()) / den, flips


def e4m3_ulp(v: torch.Tensor) -> torch.Tensor:
    """Spacing of the E4M3 grid at |v| (v already divided by its block scale)."""
    a = v.abs().clamp_min(2.0 ** -6)
    return torch.pow(2.0, torch.floor(torch.log2(a)) - 3)


def check_mx(got_dq: torch.Tensor, ref_dq: torch.Tensor, scale: torch.Tensor, tol: float = 6e-2,
             max_flip_frac: float = 1e-2):
    """Compare dequantised MXFP8 kernel values with the oracle's MXFP8 values
    (identical quantisation). Elements beyond tol*rms(ref) must be one E4M3 step
    apart at their block scale (a rounding decision taken differently from
    slightly different fp32 inputs), and be at most max_flip_frac of all."""
    g = got_dq.double().cpu()
    r = ref_dq.double().cpu()
    s = scale.double().cpu()
    den = max(float(r.pow(2).mean().sqrt()), 1e-30)
    d = (g - r).abs()
    bad = d > tol * den
    flips = int(bad.sum())
    if flips:
        step = e4m3_ulp(torch.maximum(g.abs(), r.abs()) / s) * s
        assert bool((d[bad] <= step[bad] * (1 + 1e-9)).all()), f"MXFP8 values more than one step apart"
        assert flips <= max(1, max_flip_frac * g.numel()), f"{flips} MXFP8 step differences beyond {tol}*rms"
    return float(d.max()) / den, flips


def e2m1_step(u: torch.Tensor) -> torch.Tensor:
    """Spacing of the E2M1 grid around |u| (u already divided by its block scale)."""
    a = u.abs()
    return torch.where(a < 2, 0.5, torch.where(a < 4, 1.0, 2.0)).double()


def check_nv(got: torch.Tensor, ref: torch.Tensor, s_got: torch.Tensor, s_ref: torch.Tensor, tol: float = TOL_NVFP4,
             max_flip_frac: float = 1e-2):
    """Compare dequantised NVFP4 kernel values with the oracle's NVFP4 values of the same tensor
    (identical quantisation; s_* = each element's decoded block scale). Elements beyond tol*rms(ref)
    come from a rounding decision taken differently from slightly different fp32 inputs: they must be
    within one E2M1 step at the larger scale plus 6x the difference of the two block scales (a block
    scale that itself rounded the other way), and be at most max_flip_frac of all."""
    g, r = got.double().cpu(), ref.double().cpu()
    sg, sr = s_got.double().cpu(), s_ref.double().cpu()
    den = max(float(r.pow(2).mean().sqrt()), 1e-30)
    d = (g - r).abs()
    bad = d > tol * den
    flips = int(bad.sum())
    if flips:
        sm = torch.maximum(sg, sr)
        step = e2m1_step(torch.maximum(g.abs(), r.abs()) / sm.clamp_min(1e-30)) * sm + 6 * (sg - sr).abs()
        assert bool((d[bad] <= step[bad] * (1 + 1e-9)).all()), "NVFP4 values more than one step apart"
        assert flips <= max(1, max_flip_frac * g.numel()), f"{flips} NVFP4 step differences beyond {tol}*rms"
    return float(d.max()) / den, flips
