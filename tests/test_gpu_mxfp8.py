"""MXFP8 weights (OCP MX v1.0: E4M3 + one E8M0 scale per 32 K) and MXFP4
weights (E2M1 + one E8M0 scale per 32 K, with MXFP8 activations) on the
block-scaled tensor-core MMA, against the CPU oracle through the C ABI.

Bit-exact: the MX quantisation of the activations. Within tolerance: the
GEMMs (fp32 accumulation order) and the layer. The down GEMM is fed the
oracle's quantised act, so it is checked on its own; the gate/up GEMM's
quantised act is compared with the quantisation of the oracle's act, code
by code, where a code may sit one E4M3 step away only when the two bf16 act
values straddle an E4M3 rounding point.
"""

import numpy as np
import pytest
import torch

import moe_synth
import oracle
import mixture_experts_expert_top_b200 as moe
from mixture_experts_expert_top_b200 import build as moe_build
from _util import bf16_bits, bits_to_bf16, gemm_rows_close, layer_output_close, weighted_abs_y

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    moe_build.build()
    moe.lib()
    yield
    assert moe.moe_get_device_error() == 0


def dev(x):
    return torch.as_tensor(x).contiguous().to(DEV)


def gpu_quantize(x):
    rows, K = x.shape
    q = torch.empty(rows, K, dtype=torch.uint8, device=DEV)
    s = torch.empty(rows, K // 32, dtype=torch.uint8, device=DEV)
    moe.moe_mx_quantize(dev(x), rows, K, q, s)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("rows,K", [(1, 32), (7, 96), (64, 2048), (300, 7168)])
def test_mx_quantize_is_bit_exact(rows, K):
    g = torch.Generator().manual_seed(rows + K)
    x = (torch.randn(rows, K, generator=g) * torch.exp(torch.randn(rows, 1, generator=g) * 6)).to(torch.bfloat16)
    x[0, :32] = 0                                             # an all-zero block
    if K >= 64:
        x[0, 32:64] = torch.tensor(2.0 ** -130)                 # subnormal-range block
        x[0, 33] = -1.9921875                                   # saturates to -448 * 2^e
    gq, gs = gpu_quantize(x)
    oq, os_ = oracle.mx_quantize(x)
    assert np.array_equal(gs, os_)
    assert np.array_equal(gq, oq)


MX_GEMM = [moe_synth.MoeConfig(f"{name}_{fmt}", T=T, H=H, I=I, E=E, k=k, fmt=fmt)
           for fmt in ("mxfp8", "mxfp4")
           for name, T, H, I, E, k in (("mx_bn32", 48, 1024, 384, 12, 4),     # 16 rows per expert
                                       ("mx_bn64", 96, 1024, 384, 24, 8),     # 32 rows per expert
                                       ("mx_bn128", 256, 512, 256, 16, 4))]   # 64 rows per expert


def _e4m3_step(v):
    """Spacing of E4M3 values at |v| (3 mantissa bits; 2^-9 below 2^-6)."""
    a = np.maximum(np.abs(v), 2.0 ** -6)
    return 2.0 ** (np.floor(np.log2(a)) - 3)


@pytest.mark.parametrize("cfg", MX_GEMM, ids=lambda c: c.name)
@pytest.mark.parametrize("gather", [False, True], ids=["rows", "perm"])
def test_mx_grouped_gemms_match_oracle(cfg, gather):
    inp = moe_synth.gen_inputs(cfg, seed=41)
    r = oracle.forward(inp, cfg.k, fmt=cfg.fmt)
    P = cfg.P
    sh = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt)
    offsets = dev(r["offsets"])
    if gather:      # hidden quantised once per token, rows read through perm
        xq, xs = oracle.mx_quantize(inp["hidden"])
        perm = dev(r["perm"])
    else:           # the permuted rows, quantised
        xq, xs = oracle.mx_quantize(oracle.gather(inp["hidden"], r["perm"], cfg.k))
        perm = None
    act_q = torch.empty(P, cfg.I, dtype=torch.uint8, device=DEV)
    act_s = torch.empty(P, cfg.I // 32, dtype=torch.uint8, device=DEV)
    moe.moe_grouped_gemm_swiglu_mx(dev(xq), dev(xs), perm, offsets, dev(inp["w_gu"]), dev(inp["w_gu_scales"]), sh,
                                   act_q, act_s)
    # down fed the oracle's quantised act: checked on its own
    aq, as_ = oracle.mx_quantize(r["act"])
    y = torch.empty(P, cfg.H, dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_gemm_down_mx(dev(aq), dev(as_), offsets, dev(inp["w_d"]), dev(inp["w_d_scales"]), sh, y)
    torch.cuda.synchronize()
    gemm_rows_close(bf16_bits(y), r["y"], "y")
    # gate/up: the quantised act equals the quantisation of the oracle's act,
    # except where the two bf16 acts (within the GEMM tolerance) straddle an
    # E4M3 rounding point: there one step apart
    gq, gs = act_q.cpu().numpy(), act_s.cpu().numpy()
    g_val = oracle.mx_dequantize(gq, gs)
    r_val = oracle.mx_dequantize(aq, as_)
    same = (gq == aq)
    assert same.mean() > 0.98, same.mean()
    diff = np.abs(g_val - r_val)
    assert np.all(diff <= 1.01 * _e4m3_step(r_val) * np.repeat(2.0 ** (as_.astype(np.int64) - 127), 32, axis=1)
                  + 1e-30), float(diff.max())


MX_LAYERS = [moe_synth.MoeConfig(f"{fmt}_{kind}", T=T, H=2048, I=768, E=128, k=8, fmt=fmt, logit_extra=extra)
             for fmt in ("mxfp8", "mxfp4")
             for kind, T, extra in (("decode", 64, "none"), ("prefill", 1024, "bias0.5"))]


@pytest.mark.parametrize("cfg", MX_LAYERS, ids=lambda c: c.name)
def test_mx_layer_matches_oracle(cfg):
    inp = moe_synth.gen_inputs(cfg, seed=0)
    d = {n: t.to(DEV) for n, t in inp.items()}
    sh = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt)
    ws = torch.empty(moe.moe_workspace_size(sh), dtype=torch.uint8, device=DEV)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    moe.moe_forward(d["hidden"], d["logits"], d["w_gu"], d["w_gu_scales"], d["w_d"], d["w_d_scales"], sh, out, ws)
    out2 = torch.empty_like(out)
    moe.moe_forward(d["hidden"], d["logits"], d["w_gu"], d["w_gu_scales"], d["w_d"], d["w_d_scales"], sh, out2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))        # deterministic
    r = oracle.forward(inp, cfg.k, fmt=cfg.fmt)
    y_abs = weighted_abs_y(r["y"], r["w"], r["inv_perm"], cfg.T, cfg.H, cfg.k)
    layer_output_close(bf16_bits(out), r["out"], cfg.name, y_abs=y_abs)
    assert moe.moe_forward_kernel_count(sh) == (5 if cfg.T <= 64 else 6)


def test_mx_entry_points_refuse_other_formats():
    sh = moe.Shape.of(16, 256, 128, 8, 2)                   # bf16 shape
    one = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    with pytest.raises(moe.MoeError):
        moe.moe_grouped_gemm_swiglu_mx(one, one, None, one.view(torch.int32), one, one, sh, one, one)
    shm = moe.Shape.of(16, 256, 128, 8, 2, "mxfp8")
    with pytest.raises(moe.MoeError):                        # the bf16 entry point refuses MXFP8
        moe.moe_grouped_gemm_down(torch.zeros(32, 128, dtype=torch.bfloat16, device=DEV), one.view(torch.int32),
                                  one, one, shm, torch.zeros(32, 256, dtype=torch.bfloat16, device=DEV))
