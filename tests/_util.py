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


def bf16_step(x: torch.Tensor) -> torch.Tensor:
    """The spacing of bf16 values at |x| (one unit in the last place of an
    8-bit significand): 2^(floor(log2 |x|) - 7), and the subnormal spacing
    2^-133 below the smallest normal."""
    a = x.abs().clamp_min(2.0 ** -126)
    return torch.pow(2.0, torch.floor(torch.log2(a)) - 7)


def layer_output_close(gpu_bits, ref_bits, what="", scale_abs_by_rms=False, y_abs=None):
    """End-to-end bound on the layer output against the oracle: relative L2
    error <= 1e-2, and per element |err| <= A, with A = 2e-2 (2e-2 *
    max(1, rms(ref)) with scale_abs_by_rms, used where the outputs' scale makes
    one bf16 step exceed 2e-2 throughout).

    Where A is below what bf16 rounding allows, an element may instead be off
    by what the rounding points explain. Both sides round act, y and the output
    to bf16 from fp32 sums formed in different orders, so each y row may land
    up to two bf16 steps (2^-6 relative) from the oracle's: one from its own
    rounding, one from act elements that rounded the other way. The output is
    the convex combination sum_j w_j y_j (w >= 0, sum w = 1), formed the same
    way on both sides, then rounded once more: one bf16 step of the output.
    With y_abs[t, h] = sum_j w_j |y_j[h]| (from the GPU's y and weights) the
    allowance is step(out) + 2^-6 * y_abs; without it, two bf16 steps of the
    output. At most 1e-3 of the elements may need the allowance. Returns
    (max |err|, rel-L2, number of elements beyond A)."""
    g = bits_to_bf16(gpu_bits).double()
    r = bits_to_bf16(ref_bits).double()
    err = (g - r).abs()
    rms = float(r.pow(2).mean().sqrt())
    lim = 2e-2 * (max(1.0, rms) if scale_abs_by_rms else 1.0)
    rel = float((g - r).norm() / r.norm().clamp_min(1e-30))
    beyond = err > lim
    n_beyond = int(beyond.sum())
    step = bf16_step(torch.maximum(g.abs(), r.abs()))
    if y_abs is None:
        allow = 2 * step
    else:
        allow = step + 2.0 ** -6 * torch.as_tensor(y_abs, dtype=torch.float64).reshape(g.shape)
    bad = beyond & (err > allow)
    assert not bool(bad.any()), (
        f"{what}: {int(bad.sum())} elements beyond max({lim:.4g}, rounding allowance); max|err| {float(err.max()):.4g}")
    assert n_beyond <= 1e-3 * err.numel(), f"{what}: {n_beyond} elements beyond {lim:.4g}"
    assert rel <= 1e-2, f"{what}: rel-L2 {rel:.4g} > 1e-2"
    return float(err.max()), rel, n_beyond


def weighted_abs_y(y_bits, w, inv_perm, T, H, k):
    """sum_j w[t, j] |y[inv_perm[t*k + j], h]| as a [T, H] float32 tensor."""
    y = bits_to_bf16(y_bits).float().abs()
    rows = torch.as_tensor(np.asarray(inv_perm, np.int64).reshape(T, k))
    wt = torch.as_tensor(np.asarray(w, np.float32).reshape(T, k))
    acc = torch.zeros(T, H, dtype=torch.float32)
    for j in range(k):
        acc += wt[:, j:j + 1] * y[rows[:, j]]
    return acc
