"""Python access to the CPU oracle of the MoE expert-FFN layer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU baseline call this package; the product path never does.
The arithmetic lives in moe_oracle.c (plain C, fp64 accumulation); this
module only marshals arrays through ctypes. bf16 data crosses as uint16 bit
patterns.

Functions follow the layer's steps (InfiniLM PR #500 Qwen3-MoE report §2.2;
FlashInfer PR #7196 analysis §1 for finalize, §2-§3 for W4A16):
  route, permute, gather, dequant_int4, expert_ffn, expert_down, finalize,
  forward, forward_tokens.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.oracle_route.argtypes = [vp, i32, i32, i32, vp, vp]
        L.oracle_permute.argtypes = [vp, i32, i32, vp, vp, vp, vp]
        L.oracle_gather.argtypes = [vp, vp, i32, i32, i32, vp]
        L.oracle_dequant_int4.argtypes = [vp, vp, i32, i32, vp]
        L.oracle_expert_ffn.argtypes = [i32, vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.oracle_expert_gate_up.argtypes = [i32, vp, vp, vp, i32, i32, vp]
        L.oracle_expert_down.argtypes = [i32, vp, vp, vp, i32, i32, vp]
        L.oracle_finalize.argtypes = [vp, vp, vp, i32, i32, i32, vp]
        L.oracle_forward.argtypes = [i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                     vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_forward_shared.argtypes = [i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                            vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_forward_tokens.argtypes = [i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                            vp, i32, vp, vp, vp]
        L.oracle_set_num_threads.argtypes = [i32]
        L.oracle_mx_quantize.argtypes = [vp, i32, i32, vp, vp]
        L.oracle_mx_dequantize.argtypes = [vp, vp, i32, i32, vp]
        L.oracle_mx4_dequantize.argtypes = [vp, vp, i32, i32, vp]
        for f in ("oracle_route", "oracle_permute", "oracle_forward", "oracle_forward_shared",
                  "oracle_forward_tokens", "oracle_num_threads"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


# ---- marshalling ---------------------------------------------------------

def _np(x, dtype) -> np.ndarray:
    """Contiguous numpy view/copy of a CPU tensor or array with the given dtype.
    bf16 tensors are reinterpreted as uint16 bit patterns."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            x = x.view(torch.int16)
        x = x.numpy()
    a = np.ascontiguousarray(x)
    if a.dtype != dtype:
        if dtype == np.uint16 and a.dtype == np.int16:
            a = a.view(np.uint16)
        else:
            a = a.astype(dtype)
    return a


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_tensor(a: np.ndarray) -> torch.Tensor:
    """uint16 bit patterns -> torch bf16 tensor (copy)."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16).copy()).view(torch.bfloat16)


def _fmt_code(fmt: str) -> int:
    if fmt == "bf16":
        return 0
    if fmt == "int4_g128":
        return 1
    if fmt == "mxfp8":
        return 2
    if fmt == "mxfp4":
        return 3
    raise ValueError(fmt)


def mx_quantize(x):
    """MXFP8 quantisation (OCP MX v1.0) of bf16 rows [rows, K], K % 32 == 0:
    (E4M3 codes [rows, K] uint8, E8M0 scale codes [rows, K/32] uint8)."""
    xa = _np(x, np.uint16)
    rows, K = xa.shape
    q = np.zeros((rows, K), np.uint8)
    sc = np.zeros((rows, K // 32), np.uint8)
    lib().oracle_mx_quantize(_p(xa), rows, K, _p(q), _p(sc))
    return q, sc


def mx_dequantize(q, scales) -> np.ndarray:
    """Decoded values (float64 [rows, K]) of MXFP8 codes and scales."""
    qa = _np(q, np.uint8)
    sa = _np(scales, np.uint8)
    rows, K = qa.shape
    out = np.zeros((rows, K), np.float64)
    lib().oracle_mx_dequantize(_p(qa), _p(sa), rows, K, _p(out))
    return out


def mx4_dequantize(q, scales) -> np.ndarray:
    """Decoded values (float64 [rows, K]) of MXFP4 weights: E2M1 codes packed
    two per byte [rows, K/2] (even K index in the low nibble) and E8M0 scale
    codes [rows, K/32]."""
    qa = _np(q, np.uint8)
    sa = _np(scales, np.uint8)
    rows, K = qa.shape[0], qa.shape[1] * 2
    out = np.zeros((rows, K), np.float64)
    lib().oracle_mx4_dequantize(_p(qa), _p(sa), rows, K, _p(out))
    return out


# ---- steps -----------------------------------------------------------------

def route(logits, k: int):
    """(ids [T,k] int32, w [T,k] fp32): softmax, top-k, renormalise."""
    lg = _np(logits, np.float32)
    T, E = lg.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    if lib().oracle_route(_p(lg), T, E, k, _p(ids), _p(w)):
        raise ValueError("oracle_route: bad arguments")
    return ids, w


def permute(ids, E: int):
    """(counts [E], offsets [E+1], perm [P], inv_perm [P]), all int32."""
    fl = _np(ids, np.int32).reshape(-1)
    P = fl.size
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(P, np.int32)
    inv = np.zeros(P, np.int32)
    if lib().oracle_permute(_p(fl), P, E, _p(counts), _p(offsets), _p(perm), _p(inv)):
        raise ValueError("oracle_permute: expert id out of range")
    return counts, offsets, perm, inv


def gather(hidden, perm, k: int) -> np.ndarray:
    h = _np(hidden, np.uint16)
    pm = _np(perm, np.int32).reshape(-1)
    out = np.zeros((pm.size, h.shape[1]), np.uint16)
    lib().oracle_gather(_p(h), _p(pm), pm.size, h.shape[1], k, _p(out))
    return out


def dequant_int4(q, scales) -> np.ndarray:
    """bf16 bit patterns [rows, K] of bf16(q * scale)."""
    qa = _np(q, np.uint8)
    sa = _np(scales, np.uint16)
    rows, kh = qa.shape
    out = np.zeros((rows, 2 * kh), np.uint16)
    lib().oracle_dequant_int4(_p(qa), _p(sa), rows, 2 * kh, _p(out))
    return out


def expert_ffn(x, w_gu, w_d, H: int, I: int, fmt: str = "bf16", w_gu_scales=None, w_d_scales=None):
    """One expert on one token row: (act [I], y [H]) as bf16 bit patterns."""
    f = _fmt_code(fmt)
    wdt = np.uint16 if f == 0 else np.uint8
    xa = _np(x, np.uint16).reshape(-1)
    gu = _np(w_gu, wdt)
    d = _np(w_d, wdt)
    sdt = np.uint16 if f == 1 else np.uint8
    sg = None if f == 0 else _np(w_gu_scales, sdt)
    sd = None if f == 0 else _np(w_d_scales, sdt)
    act = np.zeros(I, np.uint16)
    y = np.zeros(H, np.uint16)
    lib().oracle_expert_ffn(f, _p(xa), _p(gu), _p(sg), _p(d), _p(sd), H, I, _p(act), _p(y))
    return act, y


def expert_down(act, w_d, H: int, I: int, fmt: str = "bf16", w_d_scales=None):
    """The down projection of one act row [I] by expert weights: y [H] bf16 bits."""
    f = _fmt_code(fmt)
    wdt = np.uint16 if f == 0 else np.uint8
    aa = _np(act, np.uint16).reshape(-1)
    d = _np(w_d, wdt)
    sd = None if f == 0 else _np(w_d_scales, np.uint16 if f == 1 else np.uint8)
    y = np.zeros(H, np.uint16)
    lib().oracle_expert_down(f, _p(aa), _p(d), _p(sd), H, I, _p(y))
    return y


def finalize(y, w, inv_perm, T: int, H: int, k: int) -> np.ndarray:
    """out [T,H] bf16 bit patterns from y [P,H] bf16, w [T,k] fp32, inv_perm [P]."""
    ya = _np(y, np.uint16)
    wa = _np(w, np.float32)
    ia = _np(inv_perm, np.int32)
    out = np.zeros((T, H), np.uint16)
    lib().oracle_finalize(_p(ya), _p(wa), _p(ia), T, H, k, _p(out))
    return out


def _weights(inputs: Dict[str, torch.Tensor], fmt: str):
    f = _fmt_code(fmt)
    wdt = np.uint16 if f == 0 else np.uint8
    sdt = np.uint16 if f == 1 else np.uint8
    gu = _np(inputs["w_gu"], wdt)
    d = _np(inputs["w_d"], wdt)
    sg = None if f == 0 else _np(inputs["w_gu_scales"], sdt)
    sd = None if f == 0 else _np(inputs["w_d_scales"], sdt)
    return f, gu, sg, d, sd


def _inner(d: np.ndarray, f: int) -> int:
    """I from the down weights [E, H, I] (int4 and MXFP4: packed, I/2 bytes per row)."""
    return d.shape[2] * 2 if f in (1, 3) else d.shape[2]


def forward(inputs: Dict[str, torch.Tensor], k: int, fmt: str = "bf16", n_shared: int = 0) -> Dict[str, np.ndarray]:
    """The whole layer with every intermediate.

    inputs: hidden [T,H] bf16, logits [T,E] fp32, w_gu, w_d (+ scales for int4),
    as produced by moe_synth.gen_inputs; with n_shared > 0 the weight arrays
    hold E + n_shared experts, the last n_shared shared. Returns numpy arrays:
    ids, w ([T, k + n_shared]), counts, offsets (over E + n_shared experts),
    perm, inv_perm (int32 / fp32) and act, y, out (bf16 bit patterns).
    """
    f, gu, sg, d, sd = _weights(inputs, fmt)
    h = _np(inputs["hidden"], np.uint16)
    lg = _np(inputs["logits"], np.float32)
    T, H = h.shape
    E = lg.shape[1]
    I = _inner(d, f)
    K, Et = k + n_shared, E + n_shared
    P = T * K
    r = {
        "ids": np.zeros((T, K), np.int32), "w": np.zeros((T, K), np.float32),
        "counts": np.zeros(Et, np.int32), "offsets": np.zeros(Et + 1, np.int32),
        "perm": np.zeros(P, np.int32), "inv_perm": np.zeros(P, np.int32),
        "act": np.zeros((P, I), np.uint16), "y": np.zeros((P, H), np.uint16),
        "out": np.zeros((T, H), np.uint16),
    }
    rc = lib().oracle_forward_shared(f, _p(h), _p(lg), _p(gu), _p(sg), _p(d), _p(sd), T, H, I, E, k, n_shared,
                                     *[_p(r[n]) for n in ("ids", "w", "counts", "offsets", "perm",
                                                          "inv_perm", "act", "y", "out")])
    if rc:
        raise ValueError("oracle_forward: bad arguments")
    return r


def forward_tokens(inputs: Dict[str, torch.Tensor], k: int, tokens: Sequence[int], fmt: str = "bf16"):
    """The layer output for the listed tokens only: (ids, w, out_rows)."""
    f, gu, sg, d, sd = _weights(inputs, fmt)
    h = _np(inputs["hidden"], np.uint16)
    lg = _np(inputs["logits"], np.float32)
    T, H = h.shape
    E = lg.shape[1]
    I = _inner(d, f)
    tk = np.ascontiguousarray(np.asarray(tokens, np.int32))
    n = tk.size
    ids = np.zeros((n, k), np.int32)
    w = np.zeros((n, k), np.float32)
    out = np.zeros((n, H), np.uint16)
    rc = lib().oracle_forward_tokens(f, _p(h), _p(lg), _p(gu), _p(sg), _p(d), _p(sd), T, H, I, E, k,
                                     _p(tk), n, _p(ids), _p(w), _p(out))
    if rc:
        raise ValueError("oracle_forward_tokens: bad arguments")
    return ids, w, out
