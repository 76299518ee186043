"""Shared helpers of the GPU parity tests (comparison metrics, buffers)."""
import torch

# Floating-point bars: max |err| <= TOL * rms(ref) over the compared tensor.
TOL_BF16 = 2e-2
TOL_MXFP8 = 6e-2


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
