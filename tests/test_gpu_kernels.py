"""Per-kernel parity of the CUDA path with the CPU oracle, through the C ABI.

Bit-exact: routing ids, counts, offsets, perm, inv_perm, the gather, the
W4A16 decode and finalize (fed the same y and weights). Within tolerance:
routing weights (expf vs exp in double) and the GEMM outputs (fp32
accumulation order; see _util.gemm_rows_close).
"""

import numpy as np
import pytest
import torch

import moe_synth
import oracle
import mixture_experts_expert_top_b200 as moe
from mixture_experts_expert_top_b200 import build as moe_build
from _util import bf16_bits, bits_to_bf16, gemm_rows_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    moe_build.build()
    moe.lib()
    yield
    assert moe.moe_get_device_error() == 0


def dev(x, dtype=None):
    t = torch.as_tensor(x)
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().to(DEV)


def run_route(logits, k, n_shared=0):
    T, E = logits.shape
    ids = torch.empty(T, k + n_shared, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k + n_shared, dtype=torch.float32, device=DEV)
    moe.moe_route(dev(logits), moe.Shape.of(T, 8, 8, E, k, n_shared=n_shared), ids, w)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


def run_permute(ids, E, H=8, hidden=None):
    T, k = ids.shape
    P = T * k
    sh = moe.Shape.of(T, H, 8, E, k)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(P, dtype=torch.int32, device=DEV)
    inv = torch.empty(P, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(1, moe.moe_permute_workspace_size(sh)), dtype=torch.uint8, device=DEV)
    hp = None
    if hidden is not None:
        hp = torch.empty(P, H, dtype=torch.bfloat16, device=DEV)
    moe.moe_permute(dev(ids, torch.int32), sh, counts, offsets, perm, inv,
                    None if hidden is None else dev(hidden), hp, ws)
    torch.cuda.synchronize()
    out = [x.cpu().numpy() for x in (counts, offsets, perm, inv)]
    return out + ([bf16_bits(hp)] if hidden is not None else [])


# ---------------------------------------------------------------- routing --

ROUTE_CASES = [(c.T, c.E, c.k, c.name) for c in moe_synth.CONFIGS.values()] + [
    (100, 8, 8, "k=E"), (33, 64, 1, "k=1"), (5, 1, 1, "E=1"), (40, 1024, 32, "E=1024,k=32"), (3, 33, 4, "E=33"),
]


@pytest.mark.parametrize("T,E,k,name", ROUTE_CASES, ids=[c[3] for c in ROUTE_CASES])
def test_route_matches_oracle(T, E, k, name):
    cfg = moe_synth.CONFIGS.get(name)
    logits = moe_synth.gen_logits(cfg) if cfg else torch.randn(T, E, generator=torch.Generator().manual_seed(T + E))
    gi, gw = run_route(logits, k)
    oi, ow = oracle.route(logits, k)
    assert np.array_equal(gi, oi)
    # The GPU forms x = l_j - l_0 in fp32 (rounding error up to |x| 2^-24,
    # which exp turns into the same relative error), then expf (<= 2 ulp), an
    # fp32 sum of k terms and one division; the oracle works in double.
    # Bound: 2^-24 (8 + 2 max_j |l_j - l_0|) relative, per token.
    lsel = np.take_along_axis(logits.numpy().astype(np.float64), oi.astype(np.int64), 1)
    spread = np.abs(lsel - lsel[:, :1]).max(1, keepdims=True)
    rel = np.abs(gw.astype(np.float64) - ow) / np.abs(ow)
    bound = 2.0 ** -24 * (8 + 2 * spread)
    assert np.all(rel <= bound), f"max relative error {rel.max():.3g}, worst ratio {(rel / bound).max():.3g}"
    assert np.all(np.abs(gw.astype(np.float64).sum(1) - 1) <= 1e-6)


def test_route_ties_go_to_the_lower_expert():
    logits = torch.zeros(8, 16)
    logits[1, 3] = logits[1, 9] = 1.0
    logits[2] = torch.arange(16) % 4 * 0.5
    logits[3, :] = -3.0
    logits[4, 15] = 5.0
    logits[6, :] = -1.0                       # -0 and +0 compare equal: the lower id goes first
    logits[6, 2], logits[6, 7] = -0.0, 0.0
    logits[7, :] = -1.0
    logits[7, 2], logits[7, 7] = 0.0, -0.0
    gi, gw = run_route(logits, 4)
    oi, ow = oracle.route(logits, 4)
    assert np.array_equal(gi, oi)
    assert np.array_equal(gi[3], [0, 1, 2, 3]) and np.all(gw[3] == 0.25)
    assert np.array_equal(gi[6][:2], [2, 7]) and np.array_equal(gi[7][:2], [2, 7])


@pytest.mark.parametrize("E", [6, 64, 256])
def test_route_orders_by_logit_where_probabilities_tie(E):
    """The rows where a rounded probability would tie distinct logits (far
    below the max, or underflowed), NaN logits and signed zeros. Row 0 pads
    the planted row with NaN (ranked last, after the row's own entries, by
    id), so its ids are the hand-derived order; rows 1 and 2 put the planted
    row in the top lanes or pad it with -1e30, and are compared with the
    oracle."""
    import test_oracle_pins as pins
    for row, k, expect in pins.ROUTE_EDGE_ROWS:
        n = len(row)
        logits = torch.full((3, E), -1e30)
        logits[0, :] = float("nan")
        logits[0, :n] = torch.tensor(row)
        logits[1, E - n:] = torch.tensor(row)
        logits[2, :n] = torch.tensor(row)
        gi, gw = run_route(logits, k)
        oi, ow = oracle.route(logits, k)
        assert np.array_equal(gi, oi), (row, gi, oi)
        assert gi[0].tolist() == expect
        assert np.allclose(gw, ow, rtol=2 ** -20, atol=0)


@pytest.mark.parametrize("T,E,k,S", [(37, 64, 6, 2), (5, 8, 2, 1), (300, 256, 8, 4), (9, 30, 1, 31)])
def test_route_appends_shared_expert_slots(T, E, k, S):
    """Shared experts: slots k..k+S-1 of every token hold experts E..E+S-1 with
    weight exactly 1; the routed slots are the routing without them."""
    logits = torch.randn(T, E, generator=torch.Generator().manual_seed(T + S))
    gi, gw = run_route(logits, k, S)
    oi, ow = run_route(logits, k)
    assert np.array_equal(gi[:, :k], oi) and np.array_equal(gw[:, :k], ow)
    assert np.array_equal(gi[:, k:], np.tile(np.arange(E, E + S, dtype=np.int32), (T, 1)))
    assert np.all(gw[:, k:] == 1.0)


# ---------------------------------------------------------------- permute --

# single CTA (P <= 8192); chunk counts scanned inside the scatter CTAs (<= 64
# chunks of 2048 pairs, E <= 512); separate scan CTA (more chunks, or E > 512)
PERMUTE_CASES = [(16, 8, 2), (64, 128, 8), (256, 256, 8), (1024, 8, 8), (1025, 64, 8), (8192, 128, 8),
                 (4096, 64, 6), (1, 4, 4), (3000, 1024, 3), (20000, 2, 1), (3000, 512, 4), (20000, 64, 8)]


@pytest.mark.parametrize("T,E,k", PERMUTE_CASES)
def test_permute_matches_oracle(T, E, k):
    g = torch.Generator().manual_seed(T * 7 + E)
    logits = torch.randn(T, E, generator=g)
    if E >= 16:     # skew the load so that some experts stay empty
        logits += torch.linspace(3, -3, E)[None, :]
    ids, _ = oracle.route(logits, k)
    counts, offsets, perm, inv = run_permute(ids, E)
    oc, oo, op, oinv = oracle.permute(ids, E)
    assert np.array_equal(counts, oc)
    assert np.array_equal(offsets, oo)
    assert np.array_equal(perm, op)
    assert np.array_equal(inv, oinv)


def test_permute_with_gather():
    cfg = moe_synth.get_config("qwen3_decode")
    hidden = moe_synth.gen_hidden(cfg)
    ids, _ = oracle.route(moe_synth.gen_logits(cfg), cfg.k)
    *_, perm, inv, hp = run_permute(ids, cfg.E, H=cfg.H, hidden=hidden)
    assert np.array_equal(hp, oracle.gather(hidden, perm, cfg.k))


def test_permute_flags_bad_expert_ids():
    ids = np.array([[0, 1], [2, 7], [1, 9]], np.int32)     # 9 is out of range for E = 8
    counts, offsets, perm, inv = run_permute(ids, 8)
    assert moe.moe_get_device_error() == 1
    assert counts.sum() == 5 and offsets[-1] == 5 and inv[5] == -1
    assert moe.moe_get_device_error() == 0                  # reading clears it


# -------------------------------------------------------------- finalize --

def run_finalize(y_bits, w, inv, T, H, k):
    out = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    moe.moe_finalize(dev(bits_to_bf16(y_bits)), dev(w, torch.float32), dev(inv, torch.int32),
                     moe.Shape.of(T, H, 8, max(k, 1), k), out)
    torch.cuda.synchronize()
    return bf16_bits(out)


@pytest.mark.parametrize("T,H,k", [(16, 128, 2), (64, 2048, 8), (333, 72, 6), (7, 7168, 8), (1, 8, 1), (50, 64, 32)])
def test_finalize_bit_exact(T, H, k):
    rng = np.random.default_rng(T * H + k)
    y = rng.standard_normal((T * k, H)).astype(np.float32)
    y[rng.random(y.shape) < 0.05] = 0.0
    y[rng.random(y.shape) < 0.02] *= 2.0 ** -130           # subnormal rows of values
    y_bits = bf16_bits(torch.from_numpy(y).to(torch.bfloat16))
    w = rng.random((T, k)).astype(np.float32)
    w[rng.random(w.shape) < 0.05] = 0.0
    inv = rng.permutation(T * k).astype(np.int32)
    assert np.array_equal(run_finalize(y_bits, w, inv, T, H, k), oracle.finalize(y_bits, w, inv, T, H, k))


def test_finalize_flags_out_of_range_rows():
    # A corrupted inverse permutation must not pass silently: an index outside
    # [0, T*k) contributes 0 (as a +0 row would) and raises device error 3.
    T, H, k = 5, 64, 3
    rng = np.random.default_rng(11)
    y_bits = bf16_bits(torch.from_numpy(rng.standard_normal((T * k, H)).astype(np.float32)).to(torch.bfloat16))
    w = rng.random((T, k)).astype(np.float32)
    inv = rng.permutation(T * k).astype(np.int32)
    inv[4], inv[9] = T * k, -2
    assert moe.moe_get_device_error() == 0
    out = run_finalize(y_bits, w, inv, T, H, k)
    assert moe.moe_get_device_error() == 3
    y_ext = np.concatenate([y_bits, np.zeros((1, H), np.uint16)])
    inv_ref = np.where((inv < 0) | (inv >= T * k), T * k, inv).astype(np.int32)
    assert np.array_equal(out, oracle.finalize(y_ext, w, inv_ref, T, H, k))


def test_finalize_special_cases_from_the_golden_file():
    import test_oracle_pins as pins
    for k, v, w, exp, why in pins._golden_finalize_cases():
        # replicate the one-element case across 8 lanes (one 16-byte vector)
        y = np.repeat(np.array(v, np.uint16).reshape(k, 1), 8, axis=1)
        wf = np.array(w, np.uint32).view(np.float32).reshape(1, k)
        out = run_finalize(y, wf, np.arange(k, dtype=np.int32), 1, 8, k)
        assert np.all(out == exp), why


# ---------------------------------------------------------- W4A16 decode --

@pytest.mark.parametrize("rows,K", [(4, 128), (300, 7168), (129, 2048)])
def test_dequant_int4_bit_exact(rows, K):
    g = torch.Generator().manual_seed(rows + K)
    q = torch.randint(0, 256, (rows, K // 2), generator=g, dtype=torch.uint8)
    s = (torch.rand(rows, K // 128, generator=g) * 0.018 + 0.002).to(torch.bfloat16)
    s[0, 0] = 2.0 ** -130 if rows > 1 else s[0, 0]      # subnormal-range scale
    out = torch.empty(rows, K, dtype=torch.bfloat16, device=DEV)
    moe.moe_dequant_int4(dev(q), dev(s), rows, K, out)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(out), oracle.dequant_int4(q, s))


# ----------------------------------------------------------- grouped GEMMs --

GEMM_CFGS = [
    moe_synth.get_config("tiny"),
    moe_synth.get_config("qwen3_decode"),
    moe_synth.get_config("qwen3_decode", T=200, E=16),                 # many rows per expert: several N blocks
    moe_synth.get_config("tiny", T=33, H=72, I=40, E=5, k=3),           # ragged H, I < 128
    moe_synth.get_config("skewed", T=96, H=256, I=192, E=16, k=3),      # uneven, empty experts
    moe_synth.get_config("qwen3_prefill", T=700, H=512, I=256, E=8, k=2),  # tokens-on-M kernel, ragged tail
    moe_synth.get_config("qwen3_prefill", T=1024, H=512, I=384, E=8, k=2),  # CTA-pair kernel
    moe_synth.get_config("qwen3_prefill", T=1100, H=264, I=200, E=4, k=2),  # CTA-pair, ragged H and I
    moe_synth.get_config("qwen3_decode", T=448, H=1024, I=384, E=64, k=8),  # weights on M, 128-token blocks
    moe_synth.MoeConfig("int4_bn64", T=96, H=1024, I=384, E=24, k=8, fmt="int4_g128"),  # int4, 64-token blocks
    # int4 with few rows per expert (gate/up decoded into TMEM, down into
    # warp-level MMA fragments): K = 640 and 384 end half-way through a 256-K
    # stage
    moe_synth.MoeConfig("int4_warp_ragged", T=40, H=640, I=384, E=10, k=3, fmt="int4_g128"),
    # uneven load: empty experts, experts past 32 rows (several token blocks)
    moe_synth.MoeConfig("int4_warp_zipf", T=64, H=512, I=256, E=16, k=4, fmt="int4_g128", logit_extra="zipf1.2"),
]


def gemm_case(cfg, seed=21):
    inp = moe_synth.gen_inputs(cfg, seed=seed)
    r = oracle.forward(inp, cfg.k, fmt=cfg.fmt)
    hp = oracle.gather(inp["hidden"], r["perm"], cfg.k)
    return inp, r, hp


def wdev(inp, name):
    return dev(inp[name]) if name in inp else None


@pytest.mark.parametrize("cfg", GEMM_CFGS, ids=lambda c: f"T{c.T}H{c.H}I{c.I}E{c.E}k{c.k}")
def test_grouped_gemm_swiglu_and_down_match_oracle(cfg):
    inp, r, hp = gemm_case(cfg)
    P = cfg.P
    sh = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt)
    offsets = dev(r["offsets"], torch.int32)
    act = torch.empty(P, cfg.I, dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_gemm_swiglu(dev(bits_to_bf16(hp)), None, offsets, wdev(inp, "w_gu"), wdev(inp, "w_gu_scales"),
                                sh, act)
    # the down GEMM is fed the oracle's act so that each GEMM is checked alone
    y = torch.empty(P, cfg.H, dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_gemm_down(dev(bits_to_bf16(r["act"])), offsets, wdev(inp, "w_d"), wdev(inp, "w_d_scales"), sh, y)
    torch.cuda.synchronize()
    gemm_rows_close(bf16_bits(act), r["act"], "act")
    gemm_rows_close(bf16_bits(y), r["y"], "y")


@pytest.mark.parametrize("cfg", [GEMM_CFGS[1], GEMM_CFGS[2], GEMM_CFGS[3], GEMM_CFGS[5], GEMM_CFGS[6], GEMM_CFGS[7],
                                 moe_synth.get_config("qwen3_prefill", T=3000, H=1024, I=512, E=6, k=2),
                                 moe_synth.MoeConfig("int4_gather", T=48, H=1024, I=384, E=12, k=4, fmt="int4_g128")],
                         ids=lambda c: f"T{c.T}H{c.H}I{c.I}E{c.E}k{c.k}{c.fmt}")
def test_grouped_gemm_swiglu_gathers_through_perm(cfg):
    """perm given: the GEMM reads hidden rows through perm (TMA gather4; at
    CTA-pair shapes the single-CTA kernel takes the call) and must give the
    same act as from the materialised permuted rows."""
    inp, r, hp = gemm_case(cfg)
    sh = moe.Shape.of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.fmt)
    offsets = dev(r["offsets"], torch.int32)
    act_g = torch.empty(cfg.P, cfg.I, dtype=torch.bfloat16, device=DEV)
    act_m = torch.empty(cfg.P, cfg.I, dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_gemm_swiglu(dev(inp["hidden"]), dev(r["perm"], torch.int32), offsets, wdev(inp, "w_gu"),
                                wdev(inp, "w_gu_scales"), sh, act_g)
    moe.moe_grouped_gemm_swiglu(dev(bits_to_bf16(hp)), None, offsets, wdev(inp, "w_gu"), wdev(inp, "w_gu_scales"),
                                sh, act_m)
    torch.cuda.synchronize()
    assert torch.equal(act_g.view(torch.int16), act_m.view(torch.int16))
    gemm_rows_close(bf16_bits(act_g), r["act"], "act (gathered)")


RAGGED_EXPERTS = [
    # (rows per expert, H, I): tails of 1, 15, 17 rows, one row past a 256-row
    # block, empty experts, and H / I that are not multiples of 64 or 128
    ([1, 15, 17, 255, 257, 0, 512, 16, 256, 33], 512, 384),
    ([257, 1, 0, 17, 255, 100], 264, 200),
    ([300, 700, 3, 0, 0, 129], 1024, 768),
]


@pytest.mark.parametrize("counts,H,I", RAGGED_EXPERTS, ids=lambda x: str(x))
def test_grouped_gemms_on_ragged_experts_match_oracle(counts, H, I):
    """Many rows per expert (weights on M across a CTA pair, token N set per
    tile at run time): every row of every expert against the oracle's FFN of
    that row, with experts whose row counts end anywhere in a 256-row block."""
    E = len(counts)
    P = sum(counts)
    assert P >= 64 * E            # the shapes that take the many-rows-per-expert kernels
    g = torch.Generator().manual_seed(P + H + I)
    a = (torch.randn(P, H, generator=g)).to(torch.bfloat16)
    w_gu = (torch.randn(E, 2 * I, H, generator=g) * 0.02).to(torch.bfloat16)
    w_d = (torch.randn(E, H, I, generator=g) * 0.02).to(torch.bfloat16)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    ref_act = np.zeros((P, I), np.uint16)
    ref_y = np.zeros((P, H), np.uint16)
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            ref_act[r], ref_y[r] = oracle.expert_ffn(a[r], w_gu[e], w_d[e], H, I)
    sh = moe.Shape.of(P, H, I, E, 1)
    d_off = dev(offsets)
    act = torch.empty(P, I, dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_gemm_swiglu(dev(a), None, d_off, dev(w_gu), None, sh, act)
    y = torch.empty(P, H, dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_gemm_down(dev(bits_to_bf16(ref_act)), d_off, dev(w_d), None, sh, y)
    torch.cuda.synchronize()
    gemm_rows_close(bf16_bits(act), ref_act, "act")
    gemm_rows_close(bf16_bits(y), ref_y, "y")


def test_grouped_gemm_int4_matches_oracle():
    cfg = moe_synth.MoeConfig("int4_mid", T=48, H=1024, I=384, E=12, k=4, fmt="int4_g128")
    test_grouped_gemm_swiglu_and_down_match_oracle(cfg)


# ------------------------------------------------------------ failure path --

def test_a_wait_that_never_completes_gives_up_and_reports_a_timeout():
    # One CTA waits on a pipeline barrier that nothing arrives on, with a
    # 20 ms limit: the wait must give up, raise code 2 and let the kernel end,
    # and the context must stay usable afterwards.
    assert moe.moe_get_device_error() == 0
    moe.moe_selftest_bounded_wait(20_000_000)
    assert moe.moe_get_device_error() == 2      # synchronises, reads and clears
    assert moe.moe_get_device_error() == 0
    logits = torch.randn(40, 64, generator=torch.Generator().manual_seed(3))
    gi, _ = run_route(logits, 6)
    oi, _ = oracle.route(logits, 6)
    assert np.array_equal(gi, oi)
