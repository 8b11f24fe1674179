"""moe_forward_fused: the whole decode layer in one persistent kernel. On the
shapes it takes it runs moe_forward's arithmetic (same routing, permutation,
tiles, K order, epilogues and finalize order), so its output must equal
moe_forward's bit for bit, and the oracle's within the layer tolerance."""

import numpy as np
import pytest
import torch

import moe_synth
import oracle
import mixture_experts_expert_top_b200 as moe
from mixture_experts_expert_top_b200 import build as moe_build
from _util import bf16_bits, layer_output_close, weighted_abs_y

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    moe_build.build()
    moe.lib()
    yield
    assert moe.moe_get_device_error() == 0


class Case:
    def __init__(self, cfg, seed=0):
        self.cfg = cfg
        self.inp = moe_synth.gen_inputs(cfg, seed=seed)
        self.d = {n: t.to(DEV) for n, t in self.inp.items()}
        self.shape = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt, n_shared=cfg.n_shared)
        self.ws = torch.empty(moe.moe_workspace_size(self.shape), dtype=torch.uint8, device=DEV)

    def fused(self, hidden=None, logits=None):
        out = torch.empty(self.cfg.T, self.cfg.H, dtype=torch.bfloat16, device=DEV)
        moe.moe_forward_fused(self.d["hidden"] if hidden is None else hidden,
                              self.d["logits"] if logits is None else logits,
                              self.d["w_gu"], self.d["w_d"], self.shape, out, self.ws)
        return out

    def reference(self):
        out = torch.empty(self.cfg.T, self.cfg.H, dtype=torch.bfloat16, device=DEV)
        ws = torch.empty_like(self.ws)
        moe.moe_forward(self.d["hidden"], self.d["logits"], self.d["w_gu"], None, self.d["w_d"], None, self.shape,
                        out, ws)
        return out


FUSED = [moe_synth.get_config("tiny"),
         moe_synth.get_config("qwen3_decode"),
         moe_synth.get_config("shared_decode"),
         moe_synth.get_config("tiny", T=33, H=72, I=40, E=5, k=3),
         moe_synth.get_config("tiny", T=1, k=1),
         moe_synth.get_config("qwen3_decode", T=64, E=256, k=8)]


@pytest.mark.parametrize("cfg", FUSED, ids=lambda c: c.describe())
def test_fused_equals_forward_and_matches_oracle(cfg):
    c = Case(cfg)
    got = c.fused()
    ref = c.reference()
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    r = oracle.forward(c.inp, cfg.k, n_shared=cfg.n_shared)
    y_abs = weighted_abs_y(r["y"], r["w"], r["inv_perm"], cfg.T, cfg.H, cfg.k + cfg.n_shared)
    layer_output_close(bf16_bits(got), r["out"], cfg.name, y_abs=y_abs)


def test_fused_back_to_back_calls_reset_their_counters():
    # two batches alternating on one workspace with no synchronisation: each
    # call must start from zeroed completion counters and its own routing
    cfg = moe_synth.get_config("qwen3_decode")
    c = Case(cfg)
    h2 = moe_synth.gen_hidden(cfg, seed=5).to(DEV)
    l2 = moe_synth.gen_logits(cfg, seed=5).to(DEV)
    ref_a = c.fused().clone()
    ref_b = c.fused(h2, l2).clone()
    torch.cuda.synchronize()
    assert not torch.equal(ref_a.view(torch.int16), ref_b.view(torch.int16))
    outs = [c.fused() if i % 2 == 0 else c.fused(h2, l2) for i in range(6)]
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        assert torch.equal(o.view(torch.int16), (ref_a if i % 2 == 0 else ref_b).view(torch.int16)), i


def test_fused_refuses_shapes_it_does_not_take():
    dev_b = dict(dtype=torch.bfloat16, device=DEV)
    one = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    for sh in (moe.Shape.of(65, 256, 128, 8, 2), moe.Shape.of(16, 256, 128, 300, 2),
               moe.Shape.of(16, 256, 128, 8, 2, "int4_g128")):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_forward_fused(torch.zeros(sh.T, sh.H, **dev_b), torch.zeros(sh.T, sh.E, device=DEV),
                                  torch.zeros(8, **dev_b), torch.zeros(8, **dev_b), sh,
                                  torch.zeros(sh.T, sh.H, **dev_b), one)
        assert ei.value.status == 2          # MOE_ERR_UNSUPPORTED
