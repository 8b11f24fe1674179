"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a library routine, a closed form, an
invariant, an exactly computed value or a dense brute-force evaluation,
chosen so that a plausible slip in the oracle (a dropped term, a swapped
gate/up, a wrong index or sign, an unstable sort, an FTZ, a fused slot-0
multiply) fails at least one of them.

Sources of what is pinned: InfiniLM PR #500 Qwen3-MoE report §2.1-§2.2
(routing, bucketing, gather, grouped GEMMs with SwiGLU, weighted scatter) and
the FlashInfer PR #7196 analysis §1 (finalize arithmetic) and §2-§3 (W4A16).
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import moe_synth
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits_to_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- routing --

@pytest.mark.parametrize("T,E,k", [(37, 8, 2), (64, 128, 8), (5, 256, 8), (9, 6, 6), (3, 1, 1)])
def test_route_ids_are_a_stable_descending_sort(T, E, k):
    g = torch.Generator().manual_seed(T * 1000 + E)
    logits = torch.randn(T, E, generator=g)
    # plant exact ties so that "ties go to the lower expert id" is exercised
    logits[:, E // 2:] = torch.round(logits[:, E // 2:] * 2) / 2
    logits[0, :] = 0.25
    ids, _ = oracle.route(logits, k)
    ref = torch.sort(logits, dim=1, descending=True, stable=True).indices[:, :k]
    assert np.array_equal(ids, ref.numpy().astype(np.int32))


# Rows where the order of the logits and the order of any rounded probability
# part ways. Softmax is strictly increasing, so the k most probable experts are
# the k largest logits (InfiniLM PR #500 report §2.1, top-k softmax routing;
# ties to the lower expert id as the layer's statement of the problem fixes);
# each expected order below is read off the logits by hand.
ROUTE_EDGE_ROWS = [
    # distinct logits far below the max: their probabilities round to the same
    # double (1 + 1e-30 == 1 + 2e-30), but 2e-30 > 1e-30
    ([1.0, 1e-30, 2e-30, -1.0], 3, [0, 2, 1]),
    # probabilities of 0 and 1 underflow to 0.0 next to 1000; 1 > 0 still
    ([1000.0, 0.0, 1.0], 3, [0, 2, 1]),
    # NaN ranks as -inf; -0 and +0 tie and go to the lower id
    ([0.5, float("nan"), -0.0, 0.0, float("nan"), -2.0], 6, [0, 2, 3, 5, 1, 4]),
    ([0.0, -0.0, float("nan"), -float("inf"), 1.0], 4, [4, 0, 1, 2]),
]


@pytest.mark.parametrize("row,k,expect", ROUTE_EDGE_ROWS)
def test_route_orders_by_logit_where_probabilities_tie(row, k, expect):
    logits = torch.tensor([row], dtype=torch.float32)
    ids, w = oracle.route(logits, k)
    assert ids[0].tolist() == expect
    # library pin of the same reading: a stable descending sort of the logits
    # with NaN read as -inf and -0 as +0
    clean = torch.where(torch.isnan(logits), torch.tensor(-float("inf")), logits) + 0.0
    ref = torch.sort(clean, dim=1, descending=True, stable=True).indices[:, :k]
    assert ids[0].tolist() == ref[0].tolist()
    # weights: the renormalised softmax of the selected logits in double, with
    # NaN contributing exp(-inf) = 0
    sel = clean[0, ids[0].astype(np.int64)].double()
    p = torch.exp(sel - sel[0])
    assert np.allclose(w[0], (p / p.sum()).numpy(), rtol=2 ** -24, atol=0)
    assert abs(float(w[0].astype(np.float64).sum()) - 1.0) <= 1e-6


@pytest.mark.parametrize("T,E,k", [(50, 8, 2), (64, 128, 8), (40, 64, 6), (7, 256, 8)])
def test_route_weights_match_library_softmax(T, E, k):
    g = torch.Generator().manual_seed(E + k)
    logits = torch.randn(T, E, generator=g) * 2
    ids, w = oracle.route(logits, k)
    p = torch.softmax(logits.double(), dim=1)
    sel = torch.gather(p, 1, torch.from_numpy(ids).long())
    ref = (sel / sel.sum(dim=1, keepdim=True)).numpy()
    assert np.all(np.abs(w.astype(np.float64) - ref) <= 2.0 ** -24 * ref + 1e-30)
    # invariants: sum to one, non-increasing in slot order, in (0, 1]
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1.0) <= 1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)
    assert np.all((w > 0) & (w <= 1))


def test_route_closed_forms():
    g = torch.Generator().manual_seed(3)
    logits = torch.randn(20, 16, generator=g)
    # k = 1: the single weight is exactly 1
    ids, w = oracle.route(logits, 1)
    assert np.all(w == 1.0)
    assert np.array_equal(ids[:, 0], logits.argmax(1).numpy())
    # all-equal logits: experts 0..k-1, weights exactly 1/k (k a power of two)
    for k in (2, 8):
        ids, w = oracle.route(torch.full((4, 16), -1.5), k)
        assert np.array_equal(ids, np.tile(np.arange(k, dtype=np.int32), (4, 1)))
        assert np.all(w == np.float32(1.0 / k))
    # k = E: the weights are the full softmax, in descending order
    ids, w = oracle.route(logits, 16)
    p = torch.softmax(logits.double(), 1).numpy()
    ref = np.take_along_axis(p, ids.astype(np.int64), 1)
    assert np.allclose(w, ref, rtol=2 ** -23, atol=0)


def test_route_ignores_a_uniform_shift_of_the_logits():
    g = torch.Generator().manual_seed(4)
    logits = torch.randn(30, 64, generator=g)
    ids0, w0 = oracle.route(logits, 6)
    ids1, w1 = oracle.route(logits + 8.0, 6)     # exact in fp32 for |x| < 8
    assert np.array_equal(ids0, ids1)
    assert np.allclose(w0, w1, rtol=1e-6, atol=0)


# ---------------------------------------------------------------- permute --

@pytest.mark.parametrize("T,E,k", [(16, 8, 2), (64, 128, 8), (300, 64, 6), (1, 4, 4), (0, 8, 2)])
def test_permute_matches_bincount_and_stable_argsort(T, E, k):
    g = torch.Generator().manual_seed(T + E)
    logits = torch.randn(T, E, generator=g)
    ids, _ = oracle.route(logits, k) if T else (np.zeros((0, k), np.int32), None)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    flat = torch.from_numpy(ids.reshape(-1).astype(np.int64))
    assert np.array_equal(counts, torch.bincount(flat, minlength=E).numpy())
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(perm, torch.sort(flat, stable=True).indices.numpy())
    assert np.array_equal(inv[perm], np.arange(T * k))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(ids.reshape(-1)[seg] == e)
        assert np.all(np.diff(seg) > 0)


def test_permute_rejects_bad_ids():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 9]], np.int32), 8)
    with pytest.raises(ValueError):
        oracle.permute(np.array([[-1, 0]], np.int32), 8)


def test_gather_rows():
    h = torch.randn(5, 24).to(torch.bfloat16)
    perm = np.array([3, 0, 9, 4, 1, 2, 8, 5, 6, 7], np.int32)     # k = 2
    out = oracle.gather(h, perm, 2)
    assert np.array_equal(out, bf16_bits(h)[perm // 2])


# ---------------------------------------------------------- W4A16 decode --

def test_dequant_int4_matches_torch_rne():
    g = torch.Generator().manual_seed(5)
    rows, K = 6, 384
    q = torch.randint(0, 256, (rows, K // 2), generator=g, dtype=torch.uint8)
    s = (torch.rand(rows, K // 128, generator=g) * 0.018 + 0.002).to(torch.bfloat16)
    out = oracle.dequant_int4(q, s)
    lo = (q & 15).to(torch.int32)
    hi = (q >> 4).to(torch.int32)
    nib = torch.stack([lo, hi], dim=2).reshape(rows, K)        # low nibble = even K index
    val = torch.where(nib >= 8, nib - 16, nib)
    ref = (val.float() * s.float().repeat_interleave(128, dim=1)).to(torch.bfloat16)
    assert np.array_equal(out, bf16_bits(ref))


def test_dequant_int4_special_values():
    q = np.zeros((1, 64), np.uint8)
    q[0, 0] = 0x80          # element 0 -> 0, element 1 -> -8
    q[0, 1] = 0x7F          # element 2 -> -1, element 3 -> 7
    s = bf16_bits(torch.tensor([[2.0 ** -7]], dtype=torch.bfloat16))
    out = bits_to_bf16(oracle.dequant_int4(q, s)).float().numpy()[0]
    assert out[0] == 0.0 and not np.signbit(out[0])
    assert out[1] == -8 * 2.0 ** -7 and out[2] == -2.0 ** -7 and out[3] == 7 * 2.0 ** -7
    assert np.all(out[4:] == 0.0)


# ---------------------------------------------------------------- finalize --

def _golden_finalize_cases():
    cases = []
    with open(os.path.join(GOLDEN, "finalize_special_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v, w, exp, why = [c.strip() for c in line.split("|")]
            cases.append((int(k), [int(x, 16) for x in v.split()],
                          [int(x, 16) for x in w.split()], int(exp, 16), why))
    return cases


@pytest.mark.parametrize("case", _golden_finalize_cases(), ids=lambda c: c[4])
def test_finalize_golden_special_cases(case):
    k, v, w, exp, _ = case
    y = np.array(v, np.uint16).reshape(k, 1)
    wf = np.array(w, np.uint32).view(np.float32).reshape(1, k)
    out = oracle.finalize(y, wf, np.arange(k, dtype=np.int32), 1, 1, k)
    assert int(out[0, 0]) == exp, f"got {out[0,0]:04x} want {exp:04x}"


def _f32_rne(x: Fraction) -> float:
    """Exact Fraction -> nearest-even fp32 (normal range), by integer arithmetic."""
    if x == 0:
        return 0.0
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = math.floor(math.log2(x.numerator) - math.log2(x.denominator))
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    scaled = x / Fraction(2) ** (e - 23)        # in [2^23, 2^24)
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * float(Fraction(n) * Fraction(2) ** (e - 23))


def test_finalize_is_fused_after_slot_zero():
    """Random slots checked against exact rational arithmetic: slot 0 is one
    rounded multiply, later slots are single-rounding FMAs."""
    rng = np.random.default_rng(7)
    T, H, k = 40, 16, 6
    y = bf16_bits(torch.from_numpy(rng.standard_normal((T * k, H)).astype(np.float32)).to(torch.bfloat16))
    w = rng.random((T, k)).astype(np.float32)
    inv = rng.permutation(T * k).astype(np.int32)
    out = oracle.finalize(y, w, inv, T, H, k)
    yf = bits_to_bf16(y).float().numpy()
    n_unfused_differs = 0
    for t in range(T):
        for h in range(H):
            acc = _f32_rne(Fraction(float(yf[inv[t * k], h])) * Fraction(float(w[t, 0])))
            unf = acc
            for j in range(1, k):
                v = Fraction(float(yf[inv[t * k + j], h]))
                acc = _f32_rne(v * Fraction(float(w[t, j])) + Fraction(acc))
                unf = _f32_rne(Fraction(_f32_rne(v * Fraction(float(w[t, j])))) + Fraction(unf))
            ref = bf16_bits(torch.tensor([acc], dtype=torch.float32).to(torch.bfloat16))[0]
            n_unfused_differs += acc != unf
            assert out[t, h] == ref, (t, h)
    assert n_unfused_differs > 0    # the vectors do separate fused from unfused


def test_finalize_metamorphic_scaling():
    rng = np.random.default_rng(8)
    T, H, k = 8, 32, 4
    yt = torch.from_numpy(rng.standard_normal((T * k, H)).astype(np.float32)).to(torch.bfloat16)
    w = rng.random((T, k)).astype(np.float32)
    inv = np.arange(T * k, dtype=np.int32)
    a = bits_to_bf16(oracle.finalize(bf16_bits(yt), w, inv, T, H, k)).float()
    b = bits_to_bf16(oracle.finalize(bf16_bits(yt * 2), w, inv, T, H, k)).float()
    assert torch.equal(b, a * 2)


# ------------------------------------------------- FFN / the whole layer --

def dense_brute_force(inp, k, fmt="bf16", n_shared=0):
    """Every token through every expert in float64 (torch matmul), combined
    with weight 0 for unselected experts; routing from torch softmax/sort.
    Shared experts (the last n_shared of the weight arrays) get weight 1
    for every token. Rounding points as in the layer: fp32 accumulators,
    bf16 act and y."""
    x = inp["hidden"].double()
    logits = inp["logits"]
    T, H = x.shape
    E = logits.shape[1]
    Et = E + n_shared
    if fmt == "bf16":
        Wgu = inp["w_gu"].double()
        Wd = inp["w_d"].double()
    else:
        Wgu = torch.stack([bits_to_bf16(oracle.dequant_int4(inp["w_gu"][e], inp["w_gu_scales"][e]))
                           for e in range(Et)]).double()
        Wd = torch.stack([bits_to_bf16(oracle.dequant_int4(inp["w_d"][e], inp["w_d_scales"][e]))
                          for e in range(Et)]).double()
    I = Wd.shape[2]
    p = torch.softmax(logits.double(), 1)
    order = torch.sort(logits, dim=1, descending=True, stable=True).indices[:, :k]
    sel = torch.gather(p, 1, order)
    wsel = sel / sel.sum(1, keepdim=True)
    wfull = torch.zeros(T, Et, dtype=torch.float64).scatter_(1, order, wsel)
    wfull[:, E:] = 1.0
    out = torch.zeros(T, H, dtype=torch.float64)
    for e in range(Et):
        g = (x @ Wgu[e, :I].T).float().double()
        u = (x @ Wgu[e, I:].T).float().double()
        act = (g / (1 + torch.exp(-g)) * u).float().to(torch.bfloat16).double()
        y = (act @ Wd[e].T).float().to(torch.bfloat16).double()
        out += wfull[:, e:e + 1] * y
    return out


SHAPES = [
    moe_synth.get_config("tiny"),
    moe_synth.get_config("tiny", T=1),
    moe_synth.get_config("tiny", k=1),
    moe_synth.get_config("tiny", k=8),                 # k = E
    moe_synth.get_config("tiny", E=1, k=1),
    moe_synth.get_config("tiny", T=33, H=72, I=40, E=5, k=3),
    moe_synth.get_config("skewed", T=24, H=96, I=48, E=16, k=3),
    moe_synth.get_config("qwen3_prefill", T=20, H=64, I=32, E=12, k=4),
]


@pytest.mark.parametrize("cfg", SHAPES, ids=lambda c: f"T{c.T}H{c.H}I{c.I}E{c.E}k{c.k}")
def test_forward_matches_dense_brute_force(cfg):
    inp = moe_synth.gen_inputs(cfg, seed=11)
    r = oracle.forward(inp, cfg.k)
    ref = dense_brute_force(inp, cfg.k)
    out = bits_to_bf16(r["out"]).double()
    err = (out - ref).abs()
    # oracle: fp32 slot-ordered combine then bf16; brute force: float64 sum.
    assert torch.all(err <= ref.abs() * 2.0 ** -8 + 1e-6), float(err.max())
    assert np.array_equal(r["counts"].sum(), cfg.T * cfg.k)


@pytest.mark.parametrize("cfg", [moe_synth.get_config("tiny", n_shared=1),
                                 moe_synth.get_config("tiny", T=33, H=72, I=40, E=5, k=3, n_shared=2),
                                 moe_synth.get_config("skewed", T=24, H=96, I=48, E=16, k=3, n_shared=1)],
                         ids=lambda c: c.describe())
def test_forward_with_shared_experts_matches_dense_brute_force(cfg):
    # GC-MoE abstract: shared experts beside the routed ones, added with weight 1
    inp = moe_synth.gen_inputs(cfg, seed=17)
    r = oracle.forward(inp, cfg.k, n_shared=cfg.n_shared)
    ref = dense_brute_force(inp, cfg.k, n_shared=cfg.n_shared)
    out = bits_to_bf16(r["out"]).double()
    assert torch.all((out - ref).abs() <= ref.abs() * 2.0 ** -8 + 1e-6), float((out - ref).abs().max())
    # every token has its k routed slots, then experts E.. with weight exactly 1
    assert np.array_equal(r["ids"][:, cfg.k:], np.tile(np.arange(cfg.E, cfg.E + cfg.n_shared), (cfg.T, 1)))
    assert np.all(r["w"][:, cfg.k:] == 1.0)
    assert np.array_equal(r["counts"][cfg.E:], np.full(cfg.n_shared, cfg.T))
    # the routed slots are those of the layer without shared experts
    r0 = oracle.forward(dict(inp, w_gu=inp["w_gu"][:cfg.E], w_d=inp["w_d"][:cfg.E]), cfg.k)
    assert np.array_equal(r["ids"][:, :cfg.k], r0["ids"])
    assert np.array_equal(r["w"][:, :cfg.k], r0["w"])


def test_shared_expert_alone_when_routed_outputs_vanish():
    # routed W_down = 0 makes every routed y exactly +0, so the combine is
    # 0*w_0 (+) ... (+) 1*y_shared = y_shared: the output is the shared expert's
    # own bf16 output, bit for bit, for every token
    cfg = moe_synth.get_config("tiny", n_shared=1)
    inp = moe_synth.gen_inputs(cfg, seed=18)
    wd = inp["w_d"].clone()
    wd[:cfg.E] = 0
    r = oracle.forward(dict(inp, w_d=wd), cfg.k, n_shared=1)
    for t in range(cfg.T):
        _, y = oracle.expert_ffn(inp["hidden"][t], inp["w_gu"][cfg.E], wd[cfg.E], cfg.H, cfg.I)
        assert np.array_equal(bits_to_bf16(r["out"][t]).float().numpy(), bits_to_bf16(y).float().numpy())


def test_forward_int4_matches_dense_brute_force():
    cfg = moe_synth.MoeConfig("int4_small", T=12, H=256, I=128, E=6, k=2, fmt="int4_g128")
    inp = moe_synth.gen_inputs(cfg, seed=12)
    r = oracle.forward(inp, cfg.k, fmt=cfg.fmt)
    ref = dense_brute_force(inp, cfg.k, fmt=cfg.fmt)
    out = bits_to_bf16(r["out"]).double()
    assert torch.all((out - ref).abs() <= ref.abs() * 2.0 ** -8 + 1e-6)


def test_forward_closed_forms():
    cfg = moe_synth.get_config("tiny")
    inp = moe_synth.gen_inputs(cfg, seed=13)
    # hidden = 0 -> g = u = 0 -> act = 0 -> out = 0
    z = dict(inp, hidden=torch.zeros_like(inp["hidden"]))
    assert np.all((oracle.forward(z, cfg.k)["out"] & 0x7FFF) == 0)
    # W_down = 0 -> out = 0
    z = dict(inp, w_d=torch.zeros_like(inp["w_d"]))
    assert np.all((oracle.forward(z, cfg.k)["out"] & 0x7FFF) == 0)
    base = bits_to_bf16(oracle.forward(inp, cfg.k)["out"]).float()
    # doubling W_down doubles y exactly, hence the output
    z = dict(inp, w_d=inp["w_d"] * 2)
    assert torch.equal(bits_to_bf16(oracle.forward(z, cfg.k)["out"]).float(), base * 2)
    # doubling the up rows doubles act exactly (linear in u) ...
    I = cfg.I
    wgu = inp["w_gu"].clone()
    wgu[:, I:] *= 2
    assert torch.equal(bits_to_bf16(oracle.forward(dict(inp, w_gu=wgu), cfg.k)["out"]).float(), base * 2)
    # ... but doubling the gate rows does not (silu is not linear): gate/up not swapped
    wgu = inp["w_gu"].clone()
    wgu[:, :I] *= 2
    other = bits_to_bf16(oracle.forward(dict(inp, w_gu=wgu), cfg.k)["out"]).float()
    assert not torch.allclose(other, base * 2, rtol=1e-2, atol=1e-3)


def test_forward_k1_is_the_single_expert_output():
    cfg = moe_synth.get_config("tiny", k=1)
    inp = moe_synth.gen_inputs(cfg, seed=14)
    r = oracle.forward(inp, 1)
    for t in range(cfg.T):
        e = int(r["ids"][t, 0])
        _, y = oracle.expert_ffn(inp["hidden"][t], inp["w_gu"][e], inp["w_d"][e], cfg.H, cfg.I)
        assert np.array_equal(r["out"][t], y)


def test_forward_tokens_agrees_with_forward():
    cfg = moe_synth.get_config("tiny", T=40, E=8, k=3)
    inp = moe_synth.gen_inputs(cfg, seed=15)
    r = oracle.forward(inp, cfg.k)
    toks = [0, 7, 39, 21]
    ids, w, out = oracle.forward_tokens(inp, cfg.k, toks)
    assert np.array_equal(ids, r["ids"][toks])
    assert np.array_equal(w, r["w"][toks])
    assert np.array_equal(out, r["out"][toks])


def test_forward_intermediates_are_consistent():
    cfg = moe_synth.get_config("tiny", T=21)
    inp = moe_synth.gen_inputs(cfg, seed=16)
    r = oracle.forward(inp, cfg.k)
    hp = oracle.gather(inp["hidden"], r["perm"], cfg.k)
    for row in (0, 5, cfg.P - 1):
        p = int(r["perm"][row])
        e = int(r["ids"].reshape(-1)[p])
        act, y = oracle.expert_ffn(hp[row], inp["w_gu"][e], inp["w_d"][e], cfg.H, cfg.I)
        assert np.array_equal(act, r["act"][row]) and np.array_equal(y, r["y"][row])


# ------------------------------------------------------- input generator --

def test_synthetic_inputs_are_deterministic_and_shaped():
    cfg = moe_synth.get_config("tiny")
    a = moe_synth.gen_inputs(cfg, seed=0)
    b = moe_synth.gen_inputs(cfg, seed=0)
    c = moe_synth.gen_inputs(cfg, seed=1)
    for n in a:
        assert torch.equal(a[n], b[n])
    assert not torch.equal(a["hidden"], c["hidden"])
    assert a["w_gu"].shape == (8, 128, 128) and a["w_d"].shape == (8, 128, 64)
    # a single expert regenerates alone
    one = moe_synth.gen_expert_weights(cfg, 5, seed=0)
    assert torch.equal(one["w_gu"], a["w_gu"][5])


def test_synthetic_distributions():
    cfg = moe_synth.get_config("qwen3_decode")
    w = moe_synth.gen_expert_weights(cfg, 0)["w_gu"].float()
    assert abs(w.std().item() - 0.02) < 5e-4 and abs(w.mean().item()) < 5e-4
    lg = moe_synth.gen_logits(moe_synth.get_config("skewed"))
    col = lg.mean(0)
    assert torch.all(col[1:] < col[:-1] + 0.2)       # Zipf popularity falls with rank
    qcfg = moe_synth.MoeConfig("q", T=4, H=256, I=128, E=2, k=1, fmt="int4_g128")
    q = moe_synth.gen_expert_weights(qcfg, 0)
    nib = torch.cat([(q["w_gu"] & 15).flatten(), (q["w_gu"] >> 4).flatten()]).long()
    hist = torch.bincount(nib, minlength=16).double()
    assert hist.min() > 0.8 * hist.mean()
    s = q["w_gu_scales"].float()
    assert s.min() >= 0.0019 and s.max() <= 0.0201


def test_expert_ffn_is_gate_up_then_down():
    cfg = moe_synth.get_config("tiny")
    inp = moe_synth.gen_inputs(cfg, seed=17)
    act, y = oracle.expert_ffn(inp["hidden"][3], inp["w_gu"][2], inp["w_d"][2], cfg.H, cfg.I)
    assert np.array_equal(oracle.expert_down(act, inp["w_d"][2], cfg.H, cfg.I), y)


# ------------------------------------------------------------------ MXFP8 --
# OCP Microscaling Formats (MX) v1.0: E4M3 elements, one E8M0 scale (2^(c-127))
# per 32 consecutive elements; the block exponent is floor(log2 max|x|) - 8,
# elements are x / 2^e rounded to nearest even and saturated to +-448.

def _torch_e4m3_codes(v: torch.Tensor) -> np.ndarray:
    return v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_mx_quantize_matches_the_definition_and_torch_e4m3():
    g = torch.Generator().manual_seed(31)
    x = (torch.randn(64, 256, generator=g) * torch.exp(torch.randn(64, 1, generator=g) * 4)).to(torch.bfloat16)
    x[0, :32] = 0                                   # all-zero block: code 0, zero elements
    x[1, 5] = 2.0 ** -100                           # tiny next to the block's max
    q, sc = oracle.mx_quantize(x)
    xf = x.float()
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 32):
            blk = xf[r, 32 * b:32 * b + 32]
            amax = float(blk.abs().max())
            e = -127 if amax == 0 else max(-127, min(127, math.frexp(amax)[1] - 1 - 8))
            assert sc[r, b] == e + 127
            scaled = blk * 2.0 ** -e                 # exact in fp32 here
            assert float(scaled.abs().max()) < 512
            ref = _torch_e4m3_codes(scaled.clamp(-448, 448))   # torch: round to nearest even
            assert np.array_equal(q[r, 32 * b:32 * b + 32], ref), (r, b)


def test_e4m3_codes_decode_as_torch_and_saturate():
    # every finite code decodes to torch's float8_e4m3fn value (scale 2^0)
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    q = codes.reshape(-1, 1).repeat(32, 1)[:, :32]
    dec = oracle.mx_dequantize(q, np.full((q.shape[0], 1), 127, np.uint8))
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(dec[:, 0], ref)
    # saturation: a block whose max scales into [448, 512) keeps 448
    x = torch.zeros(1, 32, dtype=torch.bfloat16)
    x[0, 0] = 255.0 * 2 ** -7                     # 1.9921875: e = -8, scaled 510
    x[0, 1] = -1.0
    q, sc = oracle.mx_quantize(x)
    assert sc[0, 0] == 127 - 8 and q[0, 0] == 0x7E and q[0, 1] == 0xF8   # 448; -256 = -(1.0 * 2^8)
    # subnormal elements: 2^-9 steps below 2^-6 (scale 2^0 block with max 256)
    x = torch.zeros(1, 32, dtype=torch.bfloat16)
    x[0, 0], x[0, 1], x[0, 2] = 256.0, 3 * 2.0 ** -9, 2.0 ** -10
    q, sc = oracle.mx_quantize(x)
    assert sc[0, 0] == 127 and q[0, 1] == 3 and q[0, 2] == 0      # 2^-10 ties to even 0


def test_mxfp8_ffn_matches_dense_double_of_the_decoded_operands():
    cfg = moe_synth.MoeConfig("mx_small", T=6, H=128, I=64, E=3, k=2, fmt="mxfp8")
    inp = moe_synth.gen_inputs(cfg, seed=32)
    for e in range(cfg.E):
        wgu = oracle.mx_dequantize(inp["w_gu"][e], inp["w_gu_scales"][e])
        wd = oracle.mx_dequantize(inp["w_d"][e], inp["w_d_scales"][e])
        for t in range(cfg.T):
            act, y = oracle.expert_ffn(inp["hidden"][t], inp["w_gu"][e], inp["w_d"][e], cfg.H, cfg.I, fmt="mxfp8",
                                       w_gu_scales=inp["w_gu_scales"][e], w_d_scales=inp["w_d_scales"][e])
            xq = oracle.mx_dequantize(*oracle.mx_quantize(inp["hidden"][t:t + 1]))[0]
            g = np.float32(wgu[:cfg.I] @ xq).astype(np.float64)
            u = np.float32(wgu[cfg.I:] @ xq).astype(np.float64)
            a_ref = torch.from_numpy((g / (1 + np.exp(-g)) * u).astype(np.float32)).to(torch.bfloat16)
            assert np.array_equal(act, bf16_bits(a_ref))
            aq = oracle.mx_dequantize(*oracle.mx_quantize(a_ref[None]))[0]
            y_ref = torch.from_numpy(np.float32(wd @ aq)).to(torch.bfloat16)
            assert np.array_equal(y, bf16_bits(y_ref))


# ------------------------------------------------- MXFP4 weights (fmt 3) --

# The E2M1 element values of the OCP Microscaling Formats (MX) v1.0 spec
# (FP4 E2M1: bias 1, 1 mantissa bit, no infinities or NaN), by code 0..7;
# codes 8..15 are the same magnitudes negated.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _unpack_e2m1(q: np.ndarray) -> np.ndarray:
    """Codes [rows, K] from packed bytes [rows, K/2], even K in the low nibble."""
    lo, hi = q & 15, q >> 4
    return np.stack([lo, hi], axis=-1).reshape(q.shape[0], -1)


def _e2m1_table_values(codes: np.ndarray) -> np.ndarray:
    mag = np.array(E2M1_TABLE)[codes & 7]
    return np.where(codes & 8, -mag, mag)


def test_e2m1_codes_decode_as_the_mx_table_with_their_block_scale():
    codes = np.arange(16, dtype=np.uint8)
    q = np.zeros((16, 16), np.uint8)
    q[:, 0] = codes                         # element 0 (low nibble) = code, element 1 = 0
    q[:, 1] = codes << 4                    # element 3 (high nibble of byte 1) = code
    sc = np.full((16, 1), 127 + 3, np.uint8)   # scale 2^3
    dec = oracle.mx4_dequantize(q, sc)
    ref = _e2m1_table_values(codes.astype(np.int64)) * 8.0
    assert np.array_equal(dec[:, 0], ref)
    assert np.array_equal(dec[:, 3], ref)
    assert not dec[:, [1, 2]].any() and not dec[:, 4:].any()
    # code 8 is -0.0 (sign bit only)
    assert math.copysign(1.0, dec[8, 0]) == -1.0 and dec[8, 0] == 0.0
    # the scale applies per 32 elements: two blocks of one row with scales 2^-1 and 2^2
    q = np.full((1, 32), 0x22, np.uint8)                  # every element code 2 (1.0)
    dec = oracle.mx4_dequantize(q, np.array([[126, 129]], np.uint8))
    assert np.array_equal(dec[0], np.r_[np.full(32, 0.5), np.full(32, 4.0)])


def test_mxfp4_weight_ffn_matches_dense_double_of_the_table_decoded_operands():
    # FP4 weights (decoded here from the MX table, not by the oracle), FP8
    # activations (the oracle's MX quantisation, pinned above), double sums
    cfg = moe_synth.MoeConfig("mx4_small", T=5, H=128, I=64, E=3, k=2, fmt="mxfp4")
    inp = moe_synth.gen_inputs(cfg, seed=33)

    def table_decode(q, s):
        codes = _unpack_e2m1(q.numpy())
        return _e2m1_table_values(codes.astype(np.int64)) * np.repeat(
            2.0 ** (s.numpy().astype(np.int64) - 127), 32, axis=1)

    for e in range(cfg.E):
        wgu = table_decode(inp["w_gu"][e], inp["w_gu_scales"][e])
        wd = table_decode(inp["w_d"][e], inp["w_d_scales"][e])
        assert np.array_equal(wgu, oracle.mx4_dequantize(inp["w_gu"][e], inp["w_gu_scales"][e]))
        for t in range(cfg.T):
            act, y = oracle.expert_ffn(inp["hidden"][t], inp["w_gu"][e], inp["w_d"][e], cfg.H, cfg.I, fmt="mxfp4",
                                       w_gu_scales=inp["w_gu_scales"][e], w_d_scales=inp["w_d_scales"][e])
            xq = oracle.mx_dequantize(*oracle.mx_quantize(inp["hidden"][t:t + 1]))[0]
            g = np.float32(wgu[:cfg.I] @ xq).astype(np.float64)
            u = np.float32(wgu[cfg.I:] @ xq).astype(np.float64)
            a_ref = torch.from_numpy((g / (1 + np.exp(-g)) * u).astype(np.float32)).to(torch.bfloat16)
            assert np.array_equal(act, bf16_bits(a_ref))
            aq = oracle.mx_dequantize(*oracle.mx_quantize(a_ref[None]))[0]
            y_ref = torch.from_numpy(np.float32(wd @ aq)).to(torch.bfloat16)
            assert np.array_equal(y, bf16_bits(y_ref))


def test_mxfp4_layer_equals_its_steps_and_zero_down_weights_give_zero():
    cfg = moe_synth.MoeConfig("mx4_layer", T=8, H=128, I=64, E=4, k=2, fmt="mxfp4")
    inp = moe_synth.gen_inputs(cfg, seed=34)
    r = oracle.forward(inp, cfg.k, fmt="mxfp4")
    # every permuted row's act/y equals the single-expert evaluation
    ids = r["ids"].reshape(-1)
    for row in range(cfg.P):
        pair = int(r["perm"][row])
        t, e = pair // cfg.k, int(ids[pair])
        act, y = oracle.expert_ffn(inp["hidden"][t], inp["w_gu"][e], inp["w_d"][e], cfg.H, cfg.I, fmt="mxfp4",
                                   w_gu_scales=inp["w_gu_scales"][e], w_d_scales=inp["w_d_scales"][e])
        assert np.array_equal(r["act"][row], act) and np.array_equal(r["y"][row], y)
    z = dict(inp)
    z["w_d"] = torch.zeros_like(inp["w_d"])        # code 0 = +0.0 for every weight
    rz = oracle.forward(z, cfg.k, fmt="mxfp4")
    assert not (rz["out"] & 0x7FFF).any()
