"""Expert parallelism through the C ABI (moe_ep_count, moe_ep_dispatch,
moe_ep_local_offsets, moe_ep_combine), with R ranks emulated on one GPU by
one process: every rank's buffers are on the same device and the phases are
separated by device synchronisation, the barrier the steps ask for (no
kernel waits for another rank). Each rank's output must equal moe_forward on
that rank's tokens with all experts, bit for bit: every pair runs the same
arithmetic, only on the rank that owns its expert."""

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


def _ranks(cfg, Ts, seed0=100):
    out = []
    for r, T in enumerate(Ts):
        c = cfg.with_(T=T)
        out.append((moe_synth.gen_hidden(c, seed=seed0 + r), moe_synth.gen_logits(c, seed=seed0 + r)))
    return out


@pytest.mark.parametrize("R,Ts,extra", [(1, [48], "none"), (2, [16, 40], "none"), (4, [33, 64, 7, 20], "none"),
                                        (4, [64, 64, 64, 64], "bias0.5"), (8, [8, 1, 17, 64, 32, 5, 11, 40], "none"),
                                        (2, [0, 24], "none")],
                         ids=["R1", "R2", "R4", "R4_biased", "R8", "R2_empty_rank"])
def test_ep_equals_moe_forward_on_each_rank(R, Ts, extra):
    cfg = moe_synth.get_config("qwen3_decode").with_(logit_extra=extra)
    w = moe_synth.gen_inputs(cfg.with_(T=1), seed=0)
    w_gu, w_d = w["w_gu"].to(DEV), w["w_d"].to(DEV)
    E_loc = cfg.E // R
    ranks = [(h.to(DEV), l.to(DEV)) for h, l in _ranks(cfg, Ts)]
    outs = moe.ep_forward(ranks, [w_gu[r * E_loc:(r + 1) * E_loc] for r in range(R)],
                          [w_d[r * E_loc:(r + 1) * E_loc] for r in range(R)], cfg.k)
    assert moe.moe_get_device_error() == 0
    for r, (h, l) in enumerate(ranks):
        ref = moe.forward(h, l, w_gu, w_d, cfg.k)
        torch.cuda.synchronize()
        assert torch.equal(outs[r].view(torch.int16), ref.view(torch.int16)), r


def test_ep_rank_output_matches_oracle():
    cfg = moe_synth.get_config("qwen3_decode")
    w = moe_synth.gen_inputs(cfg.with_(T=1), seed=0)
    R, Ts = 2, [24, 40]
    ranks = _ranks(cfg, Ts)
    E_loc = cfg.E // R
    w_gu, w_d = w["w_gu"].to(DEV), w["w_d"].to(DEV)
    outs = moe.ep_forward([(h.to(DEV), l.to(DEV)) for h, l in ranks],
                          [w_gu[r * E_loc:(r + 1) * E_loc] for r in range(R)],
                          [w_d[r * E_loc:(r + 1) * E_loc] for r in range(R)], cfg.k)
    torch.cuda.synchronize()
    for r in range(R):
        inp = {"hidden": ranks[r][0], "logits": ranks[r][1], "w_gu": w["w_gu"], "w_d": w["w_d"]}
        ref = oracle.forward(inp, cfg.k)
        y_abs = weighted_abs_y(ref["y"], ref["w"], ref["inv_perm"], Ts[r], cfg.H, cfg.k)
        layer_output_close(bf16_bits(outs[r]), ref["out"], f"ep rank {r}", y_abs=y_abs)


def test_ep_capacity_overflow_raises_the_device_flag_and_writes_nothing_past_it():
    # a receive buffer one row too small: the dispatch skips the row that does
    # not fit and reports it (error 4); nothing outside the buffer is written
    cfg = moe_synth.get_config("tiny")               # T=16, H=128, I=64, E=8, k=2
    hid = moe_synth.gen_hidden(cfg, seed=3).to(DEV)
    lg = torch.zeros(cfg.T, cfg.E, device=DEV)
    lg[:, 0], lg[:, 1] = 2.0, 1.0                    # every token to experts 0 and 1 (both on rank 0)
    sh = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    P = cfg.P
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    wts = torch.empty(cfg.T, cfg.k, device=DEV)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(P, dtype=torch.int32, device=DEV)
    inv = torch.empty(P, dtype=torch.int32, device=DEV)
    pws = torch.empty(max(1, moe.moe_permute_workspace_size(sh)), dtype=torch.uint8, device=DEV)
    moe.moe_route(lg, sh, ids, wts)
    moe.moe_permute(ids, sh, counts, offsets, perm, inv, None, None, pws)
    cap = P - 1
    guard = 8
    rows = torch.full((cap + guard, cfg.H), 7.0, dtype=torch.bfloat16, device=DEV)
    src = torch.full((cap + guard,), -5, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(2, cfg.E // 2, dtype=torch.int32, device=DEV)
    cnt1 = torch.zeros_like(cnt)
    rows1 = torch.empty_like(rows)
    src1 = torch.empty_like(src)
    y_ret = torch.empty(P, cfg.H, dtype=torch.bfloat16, device=DEV)
    pe = moe.EpPeers()
    pe.world, pe.rank, pe.capacity = 2, 0, cap
    for q, (c, rw, s) in enumerate(((cnt, rows, src), (cnt1, rows1, src1))):
        pe.counts[q], pe.recv_rows[q], pe.recv_src[q] = c.data_ptr(), rw.data_ptr(), s.data_ptr()
        pe.y_ret[q], pe.pairs[q] = y_ret.data_ptr(), P
    moe.moe_ep_count(offsets, sh, pe)
    torch.cuda.synchronize()
    assert cnt[0].tolist()[:2] == [cfg.T, cfg.T]
    moe.moe_ep_dispatch(hid, perm, offsets, sh, pe)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 4
    assert torch.all(rows[cap:] == 7.0) and torch.all(src[cap:] == -5)
    assert torch.all(src[:cap] >= 0)
