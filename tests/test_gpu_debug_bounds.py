"""The range-checking build (libmoe_b200_debug.so, compiled with
-DMOE_DEBUG_BOUNDS): on valid inputs it gives the release library's bits;
a permutation entry or an expert offset outside its range is caught by the
kernel's own check before it addresses memory, reported as device error 4,
and replaced by an in-range value. Only this build is given such inputs."""

import numpy as np
import pytest
import torch

import moe_synth
import oracle
import mixture_experts_expert_top_b200 as moe
from mixture_experts_expert_top_b200 import build as moe_build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _libs(cuda_device):
    moe_build.build()
    moe_build.build(debug_bounds=True)
    moe.lib()
    with moe.debug_bounds_library():
        moe.lib()
    yield
    assert moe.moe_get_device_error() == 0
    with moe.debug_bounds_library():
        assert moe.moe_get_device_error() == 0


def _forward(cfg, inp):
    d = {n: t.to(DEV) for n, t in inp.items()}
    shape = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt)
    ws = torch.empty(moe.moe_workspace_size(shape), dtype=torch.uint8, device=DEV)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=DEV)
    moe.moe_forward(d["hidden"], d["logits"], d["w_gu"], d.get("w_gu_scales"), d["w_d"], d.get("w_d_scales"),
                    shape, out, ws)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("cfg", [moe_synth.get_config("qwen3_decode"),
                                 moe_synth.get_config("qwen3_prefill", T=1024),
                                 moe_synth.MoeConfig("int4_small", T=48, H=1024, I=384, E=12, k=4, fmt="int4_g128")],
                         ids=lambda c: c.name)
def test_debug_build_gives_the_release_bits(cfg):
    inp = moe_synth.gen_inputs(cfg, seed=3)
    ref = _forward(cfg, inp)
    with moe.debug_bounds_library():
        got = _forward(cfg, inp)
        assert moe.moe_get_device_error() == 0
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_debug_build_flags_a_permutation_entry_out_of_range():
    cfg = moe_synth.get_config("qwen3_decode")
    inp = moe_synth.gen_inputs(cfg, seed=4)
    ids, _ = oracle.route(inp["logits"], cfg.k)
    _, offsets, perm, _ = oracle.permute(ids, cfg.E)
    perm = perm.copy()
    perm[5], perm[9] = cfg.P + 100, -3
    shape = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    assert moe.moe_forward_gathers_in_gemm(shape) == 1      # the GEMM reads rows through perm
    act = torch.empty(cfg.P, cfg.I, dtype=torch.bfloat16, device=DEV)
    with moe.debug_bounds_library():
        moe.moe_grouped_gemm_swiglu(inp["hidden"].to(DEV), torch.from_numpy(perm).to(DEV),
                                    torch.from_numpy(offsets).to(DEV), inp["w_gu"].to(DEV), None, shape, act)
        assert moe.moe_get_device_error() == 4
        assert moe.moe_get_device_error() == 0


@pytest.mark.parametrize("kind", ["decreasing", "past_the_end"])
def test_debug_build_flags_bad_expert_offsets(kind):
    E, H, I, T, k = 16, 256, 128, 64, 2
    P = T * k
    offsets = np.linspace(0, P, E + 1).astype(np.int32)
    if kind == "decreasing":
        offsets[4], offsets[5] = offsets[5], offsets[4]
    else:
        offsets[E] = P + 50
    g = torch.Generator().manual_seed(1)
    act = (torch.randn(P, I, generator=g)).to(torch.bfloat16).to(DEV)
    w_d = (torch.randn(E, H, I, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    y = torch.empty(P, H, dtype=torch.bfloat16, device=DEV)
    with moe.debug_bounds_library():
        moe.moe_grouped_gemm_down(act, torch.from_numpy(offsets).to(DEV), w_d, None, moe.Shape.of(T, H, I, E, k), y)
        assert moe.moe_get_device_error() == 4
        assert moe.moe_get_device_error() == 0
