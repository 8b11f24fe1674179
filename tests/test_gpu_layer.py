"""The whole layer on the GPU (moe_forward through the C ABI) against the CPU
oracle, on every workload at its full size and on every element, plus
determinism, the host-buffer entry point and degenerate shapes.
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


class Layer:
    """Device copies of one workload's inputs and the step-by-step outputs."""

    def __init__(self, cfg, seed=0):
        self.cfg = cfg
        self.inp = moe_synth.gen_inputs(cfg, seed=seed)
        self.d = {n: t.to(DEV) for n, t in self.inp.items()}
        self.shape = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt, n_shared=cfg.n_shared)
        self.ws = torch.empty(moe.moe_workspace_size(self.shape), dtype=torch.uint8, device=DEV)

    def forward(self):
        out = torch.empty(self.cfg.T, self.cfg.H, dtype=torch.bfloat16, device=DEV)
        d = self.d
        moe.moe_forward(d["hidden"], d["logits"], d["w_gu"], d.get("w_gu_scales"), d["w_d"], d.get("w_d_scales"),
                        self.shape, out, self.ws)
        return out

    def steps(self):
        c, d = self.cfg, self.d
        P = c.P
        K, Et = c.k + c.n_shared, c.E + c.n_shared        # slots per token, experts in the weights
        i32 = dict(dtype=torch.int32, device=DEV)
        s = {"ids": torch.empty(c.T, K, **i32), "w": torch.empty(c.T, K, dtype=torch.float32, device=DEV),
             "counts": torch.empty(Et, **i32), "offsets": torch.empty(Et + 1, **i32),
             "perm": torch.empty(P, **i32), "inv_perm": torch.empty(P, **i32),
             "hp": torch.empty(P, c.H, dtype=torch.bfloat16, device=DEV),
             "act": torch.empty(P, c.I, dtype=torch.bfloat16, device=DEV),
             "y": torch.empty(P, c.H, dtype=torch.bfloat16, device=DEV),
             "out": torch.empty(c.T, c.H, dtype=torch.bfloat16, device=DEV)}
        pws = torch.empty(max(1, moe.moe_permute_workspace_size(self.shape)), dtype=torch.uint8, device=DEV)
        moe.moe_route(d["logits"], self.shape, s["ids"], s["w"])
        moe.moe_permute(s["ids"], self.shape, s["counts"], s["offsets"], s["perm"], s["inv_perm"], d["hidden"],
                        s["hp"], pws)
        moe.moe_grouped_gemm_swiglu(s["hp"], None, s["offsets"], d["w_gu"], d.get("w_gu_scales"), self.shape,
                                    s["act"])
        moe.moe_grouped_gemm_down(s["act"], s["offsets"], d["w_d"], d.get("w_d_scales"), self.shape, s["y"])
        moe.moe_finalize(s["y"], s["w"], s["inv_perm"], self.shape, s["out"])
        torch.cuda.synchronize()
        return s


WORKLOADS = ["tiny", "qwen3_decode", "qwen3_prefill", "skewed", "w4a16_decode"]
# shared experts beside the routed ones (GC-MoE abstract): 2 shared experts
# on a decode batch and on a prefill batch (the shared experts then take
# every token: 2048-row segments)
SHARED = [moe_synth.MoeConfig("shared_decode", T=64, H=2048, I=768, E=64, k=6, n_shared=2),
          moe_synth.MoeConfig("shared_prefill", T=2048, H=2048, I=768, E=64, k=6, n_shared=2,
                              logit_extra="bias0.5")]


@pytest.mark.parametrize("cfg", [moe_synth.get_config(n) for n in WORKLOADS] + SHARED, ids=lambda c: c.name)
def test_layer_matches_oracle_on_every_element(cfg):
    """Each workload at its full size, every element of every step:
    routing ids, counts, offsets, perm, inv_perm and the gather bit-exact;
    act on every row; y on every row, from the down GEMM fed the oracle's act
    so that it is checked alone; finalize of the GPU's own y bit-exact; and
    the layer output on every token within the layer's tolerance."""
    name = cfg.name
    L = Layer(cfg)
    out = L.forward()
    s = L.steps()
    # moe_forward and the step-by-step calls run the same arithmetic
    assert torch.equal(out.view(torch.int16), s["out"].view(torch.int16))
    r = oracle.forward(L.inp, cfg.k, fmt=cfg.fmt, n_shared=cfg.n_shared)
    for n in ("ids", "counts", "offsets", "perm", "inv_perm"):
        assert np.array_equal(s[n].cpu().numpy().reshape(-1), r[n].reshape(-1)), n
    if cfg.name == "skewed":
        assert (r["counts"] == 0).any()          # empty experts are exercised
    assert np.array_equal(bf16_bits(s["hp"]), oracle.gather(L.inp["hidden"], r["perm"], cfg.k + cfg.n_shared))
    gemm_rows_close(bf16_bits(s["act"]), r["act"], "act")
    y = torch.empty_like(s["y"])
    moe.moe_grouped_gemm_down(bits_to_bf16(r["act"]).to(DEV), s["offsets"], L.d["w_d"], L.d.get("w_d_scales"),
                              L.shape, y)
    torch.cuda.synchronize()
    gemm_rows_close(bf16_bits(y), r["y"], "y")
    K = cfg.k + cfg.n_shared
    fin = oracle.finalize(bf16_bits(s["y"]), s["w"].cpu().numpy(), s["inv_perm"].cpu().numpy(), cfg.T, cfg.H, K)
    assert np.array_equal(bf16_bits(s["out"]), fin)
    y_abs = weighted_abs_y(bf16_bits(s["y"]), s["w"].cpu().numpy(), s["inv_perm"].cpu().numpy(), cfg.T, cfg.H, K)
    layer_output_close(bf16_bits(out), r["out"], name, scale_abs_by_rms=cfg.fmt == "int4_g128", y_abs=y_abs)


def test_layer_is_deterministic():
    L = Layer(moe_synth.get_config("qwen3_decode"))
    first = L.forward().clone()
    for _ in range(9):
        assert torch.equal(L.forward().view(torch.int16), first.view(torch.int16))
    Lp = Layer(moe_synth.get_config("qwen3_prefill", T=2048))
    a = Lp.forward().clone()
    assert torch.equal(Lp.forward().view(torch.int16), a.view(torch.int16))


@pytest.mark.parametrize("name", ["qwen3_decode", "w4a16_decode", "qwen3_prefill"])
def test_back_to_back_calls_with_different_routing(name):
    # moe_forward starts each kernel before the previous one on the stream has
    # finished (programmatic dependent launch), and the decode down GEMM reads
    # the expert offsets before its wait. Alternating two batches whose routing
    # differs, with no synchronisation between the calls, would expose a kernel
    # that sees the previous call's offsets or rows.
    kw = {"T": 1024} if name == "qwen3_prefill" else {}
    cfg = moe_synth.get_config(name, **kw)
    A = Layer(cfg, seed=0)
    # B: other tokens and logits, the same weights and the same workspace
    B = Layer.__new__(Layer)
    B.cfg, B.shape, B.ws = cfg, A.shape, A.ws
    B.inp = dict(A.inp, hidden=moe_synth.gen_hidden(cfg, seed=7), logits=moe_synth.gen_logits(cfg, seed=7))
    B.d = dict(A.d, hidden=B.inp["hidden"].to(DEV), logits=B.inp["logits"].to(DEV))
    ref_a = A.steps()["out"].clone()
    ref_b = B.steps()["out"].clone()
    assert not torch.equal(ref_a.view(torch.int16), ref_b.view(torch.int16))
    outs = []
    for i in range(6):
        outs.append((A if i % 2 == 0 else B).forward())
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        ref = ref_a if i % 2 == 0 else ref_b
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), f"call {i}"


def _capture_forward(L, out):
    """moe_forward captured in a CUDA graph (programmatic launches become
    programmatic edges of the graph)."""
    try:
        g = torch.cuda.CUDAGraph(keep_graph=True)
    except TypeError:
        g = torch.cuda.CUDAGraph()
    d = L.d
    with torch.cuda.graph(g):
        moe.moe_forward(d["hidden"], d["logits"], d["w_gu"], d.get("w_gu_scales"), d["w_d"], d.get("w_d_scales"),
                        L.shape, out, L.ws, torch.cuda.current_stream())
    return g


@pytest.mark.parametrize("name", ["qwen3_decode", "qwen3_prefill"])
def test_forward_replays_from_a_cuda_graph(name):
    cfg = moe_synth.get_config(name, **({"T": 1024} if name == "qwen3_prefill" else {}))
    L = Layer(cfg)
    ref = L.forward().clone()
    out = torch.zeros_like(ref)
    g = _capture_forward(L, out)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # new tokens copied into the captured input buffers: the replay routes them afresh
    h2, l2 = moe_synth.gen_hidden(cfg, seed=9), moe_synth.gen_logits(cfg, seed=9)
    L.d["hidden"].copy_(h2)
    L.d["logits"].copy_(l2)
    g.replay()
    torch.cuda.synchronize()
    L2 = Layer.__new__(Layer)
    L2.cfg, L2.shape, L2.ws = cfg, L.shape, torch.empty_like(L.ws)
    L2.inp = dict(L.inp, hidden=h2, logits=l2)
    L2.d = dict(L.d)
    assert torch.equal(out.view(torch.int16), L2.steps()["out"].view(torch.int16))


def test_captured_forward_has_the_advertised_number_of_kernels():
    cudart = pytest.importorskip("cuda.bindings.runtime")
    L = Layer(moe_synth.get_config("qwen3_decode"))
    L.forward()
    out = torch.empty(L.cfg.T, L.cfg.H, dtype=torch.bfloat16, device=DEV)
    g = _capture_forward(L, out)
    try:
        raw = g.raw_cuda_graph()
    except Exception as e:      # noqa: BLE001 - torch without the raw handle
        pytest.skip(f"no raw CUDA graph handle: {e}")
    err, _, n = cudart.cudaGraphGetNodes(cudart.cudaGraph_t(init_value=int(raw)), 0)
    assert err == cudart.cudaError_t.cudaSuccess
    err, nodes, n = cudart.cudaGraphGetNodes(cudart.cudaGraph_t(init_value=int(raw)), n)
    kinds = [cudart.cudaGraphNodeGetType(nd)[1] for nd in nodes]
    kernels = sum(k == cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel for k in kinds)
    assert kernels == moe.moe_forward_kernel_count(L.shape) == 2      # counter reset + persistent kernel


@pytest.mark.parametrize("name,T", [("qwen3_decode", 64), ("qwen3_prefill", 8192), ("skewed", 4096),
                                    ("qwen3_prefill", 3000)])
def test_forward_host_matches_forward(name, T):
    # T >= 2048 runs in chunks on the library's copy streams: the same bits
    L = Layer(moe_synth.get_config(name, T=T))
    ref = L.forward()
    d, c = L.d, L.cfg
    ws = torch.empty(moe.moe_forward_host_workspace_size(L.shape), dtype=torch.uint8, device=DEV)
    h = L.inp["hidden"].pin_memory()
    lg = L.inp["logits"].pin_memory()
    out = torch.empty(c.T, c.H, dtype=torch.bfloat16).pin_memory()
    moe.moe_forward_host(h, lg, d["w_gu"], None, d["w_d"], None, L.shape, out, ws)
    assert torch.equal(out.view(torch.int16), ref.cpu().view(torch.int16))


EDGE = [
    moe_synth.get_config("tiny", T=1),
    moe_synth.get_config("tiny", T=1, k=1),
    moe_synth.get_config("tiny", E=1, k=1),
    moe_synth.get_config("tiny", k=8),
    moe_synth.get_config("tiny", T=33, H=72, I=40, E=5, k=3),
    moe_synth.get_config("skewed", T=300, H=512, I=320, E=64, k=6),
    moe_synth.MoeConfig("int4_small", T=20, H=256, I=128, E=6, k=2, fmt="int4_g128"),
    moe_synth.get_config("qwen3_decode", T=9000, H=64, I=64, E=128, k=1),   # multi-CTA permute
]


@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: f"T{c.T}H{c.H}I{c.I}E{c.E}k{c.k}{c.fmt}")
def test_layer_edge_shapes(cfg):
    L = Layer(cfg, seed=5)
    out = L.forward()
    r = oracle.forward(L.inp, cfg.k, fmt=cfg.fmt)
    layer_output_close(bf16_bits(out), r["out"], cfg.describe())


def test_zero_inputs_give_zero_output():
    cfg = moe_synth.get_config("qwen3_decode")
    L = Layer(cfg)
    L.d["hidden"].zero_()
    out = L.forward()
    assert torch.all(out.float() == 0)
    L.d["hidden"].copy_(L.inp["hidden"])
    L.d["w_d"].zero_()
    assert torch.all(L.forward().float() == 0)


def test_empty_batch():
    cfg = moe_synth.get_config("tiny", T=0)
    sh = moe.Shape.of(0, cfg.H, cfg.I, cfg.E, cfg.k)
    bf = dict(dtype=torch.bfloat16, device=DEV)
    moe.moe_forward(torch.empty(0, **bf), torch.empty(0, device=DEV), torch.empty(0, **bf), None,
                    torch.empty(0, **bf), None, sh, torch.empty(0, **bf), torch.empty(1, dtype=torch.uint8, device=DEV))
