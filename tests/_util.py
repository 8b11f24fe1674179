"""Helpers shared by the test files: bf16 bit-pattern conversions and the
tolerance checks the parity tests use."""

import numpy as np
import torch


def bits_to_bf16(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def gemm_rows_close(gpu_bits, ref_bits, what=""):
    """bf16 outputs of an fp32-accumulated dot product against the oracle's
    (double accumulation rounded to fp32, then bf16). The two differ only by
    fp32 accumulation order before the final bf16 rounding, so each element
    may land one bf16 step (2^-8 relative) away, plus an absolute allowance of
    2^-12 of the row's RMS for elements that cancel to near zero. Returns the
    fraction of bit-identical elements."""
    g = bits_to_bf16(gpu_bits).double()
    r = bits_to_bf16(ref_bits).double()
    rms = r.pow(2).mean(dim=-1, keepdim=True).sqrt().clamp_min(1e-30)
    tol = r.abs() * 2.0 ** -7 + rms * 2.0 ** -12
    bad = (g - r).abs() > tol
    assert not bool(bad.any()), (
        f"{what}: {int(bad.sum())} elements out of tolerance; worst |d|={float((g - r).abs().max()):.3g}")
    return float((np.asarray(gpu_bits) == np.asarray(ref_bits)).mean())


def layer_output_close(gpu_bits, ref_bits, what="", scale_abs_by_rms=False):
    """End-to-end bound on the layer output: max |err| <= 2e-2 and
    relative L2 error <= 1e-2 against the oracle. With scale_abs_by_rms, the
    absolute bound is 2e-2 * max(1, rms(ref)) (used where one bf16 step of the
    output already exceeds 2e-2)."""
    g = bits_to_bf16(gpu_bits).double()
    r = bits_to_bf16(ref_bits).double()
    err = (g - r).abs()
    rms = float(r.pow(2).mean().sqrt())
    lim = 2e-2 * (max(1.0, rms) if scale_abs_by_rms else 1.0)
    rel = float((g - r).norm() / r.norm().clamp_min(1e-30))
    assert float(err.max()) <= lim, f"{what}: max|err| {float(err.max()):.4g} > {lim:.4g}"
    assert rel <= 1e-2, f"{what}: rel-L2 {rel:.4g} > 1e-2"
    return float(err.max()), rel
