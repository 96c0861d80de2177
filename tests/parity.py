"""Shared helpers for the GPU parity tests (comparison against the fp64 oracle)."""
import torch

# Tolerances on bf16 inputs with fp32 accumulation: max-abs error of O and of LSE.
O_TOL = 1e-2
LSE_TOL = 1e-3


def assert_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    """o_gpu bf16 (any device), o_ref float64 of the same shape; lse likewise (fp32 / fp64)."""
    og = o_gpu.detach().double().cpu()
    assert og.shape == o_ref.shape, (og.shape, o_ref.shape)
    assert torch.isfinite(og).all(), f"{what}: non-finite O"
    diff = (og - o_ref).abs()
    err = diff.max().item() if og.numel() else 0.0
    if err > O_TOL:
        i = int(diff.argmax())
        idx = torch.unravel_index(torch.tensor(i), diff.shape)
        raise AssertionError(f"{what}: max |O - oracle| = {err:.3e} > {O_TOL} at "
                             f"{tuple(int(x) for x in idx)}: gpu {og.flatten()[i].item():.6f} "
                             f"oracle {o_ref.flatten()[i].item():.6f}")
    lerr = 0.0
    if lse_ref is not None:
        lg = lse_gpu.detach().double().cpu()
        assert lg.shape == lse_ref.shape, (lg.shape, lse_ref.shape)
        assert torch.isfinite(lg).all(), f"{what}: non-finite LSE"
        lerr = (lg - lse_ref).abs().max().item() if lg.numel() else 0.0
        assert lerr <= LSE_TOL, f"{what}: max |LSE - oracle| = {lerr:.3e} > {LSE_TOL}"
    return err, lerr
