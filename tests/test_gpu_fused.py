"""moe_forward_fused: the whole decode layer in one persistent kernel (and
moe_forward on these shapes). It runs the step entry points' arithmetic (the
same routing, permutation, K order, epilogues and finalize order), so its
output and the routing and permutation it leaves in the workspace must equal
theirs bit for bit, and its output the oracle's within the layer tolerance."""

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

    def steps(self):
        """The layer through the step entry points, one kernel each."""
        c, d, sh = self.cfg, self.d, self.shape
        K, Et, P = c.k + c.n_shared, c.E + c.n_shared, c.P
        i32 = dict(dtype=torch.int32, device=DEV)
        s = {"ids": torch.empty(c.T, K, **i32), "w": torch.empty(c.T, K, dtype=torch.float32, device=DEV),
             "counts": torch.empty(Et, **i32), "offsets": torch.empty(Et + 1, **i32),
             "perm": torch.empty(P, **i32), "inv_perm": torch.empty(P, **i32),
             "act": torch.empty(P, c.I, dtype=torch.bfloat16, device=DEV),
             "y": torch.empty(P, c.H, dtype=torch.bfloat16, device=DEV),
             "out": torch.empty(c.T, c.H, dtype=torch.bfloat16, device=DEV)}
        pws = torch.empty(max(1, moe.moe_permute_workspace_size(sh)), dtype=torch.uint8, device=DEV)
        moe.moe_route(d["logits"], sh, s["ids"], s["w"])
        moe.moe_permute(s["ids"], sh, s["counts"], s["offsets"], s["perm"], s["inv_perm"], None, None, pws)
        moe.moe_grouped_gemm_swiglu(d["hidden"], s["perm"], s["offsets"], d["w_gu"], None, sh, s["act"])
        moe.moe_grouped_gemm_down(s["act"], s["offsets"], d["w_d"], None, sh, s["y"])
        moe.moe_finalize(s["y"], s["w"], s["inv_perm"], sh, s["out"])
        return s

    def workspace_view(self, name, n, dtype=torch.int32):
        """The routing / permutation moe_forward_fused left in the workspace:
        the layout is the library's (256-byte aligned regions in the order
        ids, w, counts, offsets, perm, inv_perm)."""
        c = self.cfg
        P, Et = c.P, c.E + c.n_shared
        sizes = [("ids", P * 4), ("w", P * 4), ("counts", Et * 4), ("offsets", (Et + 1) * 4), ("perm", P * 4),
                 ("inv_perm", P * 4)]
        o = 0
        for nm, b in sizes:
            if nm == name:
                return self.ws[o:o + n * 4].view(dtype)
            o = (o + b + 255) // 256 * 256
        raise KeyError(name)


FUSED = [moe_synth.get_config("tiny"),
         moe_synth.get_config("qwen3_decode"),
         moe_synth.get_config("shared_decode"),
         moe_synth.get_config("tiny", T=33, H=72, I=40, E=5, k=3),
         moe_synth.get_config("tiny", T=1, k=1),
         moe_synth.get_config("qwen3_decode", T=64, E=256, k=8),
         moe_synth.get_config("tiny", T=64, E=4, k=2),                # experts of about 32 tokens (N > 32)
         moe_synth.get_config("tiny", T=64, E=2, k=2),                # every token in both experts: N = 64
         moe_synth.get_config("tiny", T=16, H=384, I=192, E=8, k=2),  # last down tile has one 128-row half
         moe_synth.get_config("qwen3_decode", logit_extra="bias0.5"),   # 29 empty experts
         moe_synth.get_config("qwen3_decode", logit_extra="zipf1.2")]   # a few experts hold most tokens


@pytest.mark.parametrize("cfg", FUSED, ids=lambda c: c.describe())
def test_fused_equals_forward_and_matches_oracle(cfg):
    c = Case(cfg)
    assert moe.moe_forward_is_fused(c.shape)
    got = c.fused()
    ref = c.steps()
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), ref["out"].view(torch.int16))
    P, Et = cfg.P, cfg.E + cfg.n_shared
    for name, n in (("ids", P), ("counts", Et), ("offsets", Et + 1), ("perm", P), ("inv_perm", P)):
        assert torch.equal(c.workspace_view(name, n), ref[name].reshape(-1)), name
    assert torch.equal(c.workspace_view("w", P, torch.float32), ref["w"].reshape(-1))
    # moe_forward runs the same kernel
    out2 = torch.empty_like(got)
    moe.moe_forward(c.d["hidden"], c.d["logits"], c.d["w_gu"], None, c.d["w_d"], None, c.shape, out2, c.ws)
    torch.cuda.synchronize()
    assert torch.equal(out2.view(torch.int16), got.view(torch.int16))
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
