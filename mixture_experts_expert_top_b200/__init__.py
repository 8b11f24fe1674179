"""Python binding of libmoe_b200, the B200 (sm_100a) MoE expert-FFN layer.

Argument marshalling only: every function here passes torch tensors' device
pointers and sizes to the C entry point of the same name (include/moe.h) and
raises MoeError on a non-OK status. All computation runs in the library's
CUDA kernels. If the library is missing this module raises on first use; it
has no fallback of any kind.

The layer: top-k softmax routing -> permute (bucket by expert, gather) ->
grouped GEMM gate/up + SwiGLU -> grouped GEMM down -> weighted finalize
(InfiniLM PR #500 Qwen3-MoE report §2.2; FlashInfer PR #7196 analysis §1-§2).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "MoeError", "Shape", "lib", "library_path", "FMT_BF16", "FMT_INT4_G128",
    "moe_workspace_size", "moe_permute_workspace_size", "moe_forward_host_workspace_size",
    "moe_route", "moe_permute", "moe_grouped_gemm_swiglu", "moe_grouped_gemm_down",
    "moe_finalize", "moe_forward", "moe_forward_host", "moe_dequant_int4",
    "moe_get_device_error", "moe_status_string", "moe_permute_noalloc", "moe_selftest_bounded_wait",
    "moe_forward_kernel_count", "moe_forward_gathers_in_gemm", "forward", "debug_bounds_library",
    "moe_mx_quantize", "moe_grouped_gemm_swiglu_mx", "moe_grouped_gemm_down_mx", "FMT_MXFP8", "FMT_MXFP4",
    "moe_forward_fused", "moe_forward_is_fused",
    "EP_MAX_RANKS", "EpPeers", "moe_ep_count", "moe_ep_dispatch", "moe_ep_local_offsets", "moe_ep_combine",
    "ep_forward",
]

HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(HERE, "libmoe_b200.so")

FMT_BF16 = 0
FMT_INT4_G128 = 1
FMT_MXFP8 = 2
FMT_MXFP4 = 3

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
          3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_FLAG"}


EP_MAX_RANKS = 8


class EpPeers(ctypes.Structure):
    """moe_ep_peers_t: every rank's expert-parallel buffers (device addresses)."""
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("counts", ctypes.c_void_p * EP_MAX_RANKS), ("recv_rows", ctypes.c_void_p * EP_MAX_RANKS),
                ("recv_src", ctypes.c_void_p * EP_MAX_RANKS), ("y_ret", ctypes.c_void_p * EP_MAX_RANKS),
                ("pairs", ctypes.c_int32 * EP_MAX_RANKS)]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Shape(ctypes.Structure):
    """moe_shape_t: E routed experts and top_k routed slots per token, plus
    n_shared shared experts (experts E.. of the weight arrays, one extra slot
    each with weight 1)."""
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("top_k", ctypes.c_int32), ("fmt", ctypes.c_int32),
                ("n_shared", ctypes.c_int32)]

    @classmethod
    def of(cls, T, H, I, E, top_k, fmt=FMT_BF16, n_shared=0) -> "Shape":
        if isinstance(fmt, str):
            fmt = {"bf16": FMT_BF16, "int4_g128": FMT_INT4_G128, "mxfp8": FMT_MXFP8, "mxfp4": FMT_MXFP4}[fmt]
        return cls(int(T), int(H), int(I), int(E), int(top_k), int(fmt), int(n_shared))

    @property
    def slots(self) -> int:
        return self.top_k + self.n_shared

    @property
    def experts(self) -> int:
        return self.E + self.n_shared


_lib: Optional[ctypes.CDLL] = None
_debug_lib: Optional[ctypes.CDLL] = None
_use_debug = False


def lib() -> ctypes.CDLL:
    """The loaded library (libmoe_b200.so; inside `debug_bounds_library()`,
    the range-checking build libmoe_b200_debug.so)."""
    global _lib, _debug_lib
    if _use_debug:
        if _debug_lib is None:
            _debug_lib = _load(True)
        return _debug_lib
    if _lib is None:
        _lib = _load(False)
    return _lib


class debug_bounds_library:
    """Context manager: the entry points of this module call the build made
    with -DMOE_DEBUG_BOUNDS (perm-derived rows and expert offsets range-checked
    in the kernels, device error 4 on a bad one) while it is active."""

    def __enter__(self):
        global _use_debug
        self._prev = _use_debug
        _use_debug = True
        return lib()

    def __exit__(self, *exc):
        global _use_debug
        _use_debug = self._prev
        return False


def _load(debug_bounds: bool) -> ctypes.CDLL:
    from . import build as _build
    path = _build.LIB_DEBUG if debug_bounds else library_path
    if not _build.up_to_date(debug_bounds):
        # a missing or stale library is rebuilt from the sources (needs nvcc); never skipped
        try:
            _build.build(debug_bounds=debug_bounds)
        except Exception as e:      # noqa: BLE001 - re-raised with the path
            raise RuntimeError(f"{path} is missing or older than its sources and could not be "
                               f"built ({e}): build it with `python -m mixture_experts_expert_top_b200.build`")
    L = ctypes.CDLL(path)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    sp = ctypes.POINTER(Shape)
    sigs = {
        "moe_workspace_size": ([sp], sz),
        "moe_permute_workspace_size": ([sp], sz),
        "moe_forward_host_workspace_size": ([sp], sz),
        "moe_route": ([vp, sp, vp, vp, vp], ctypes.c_int),
        "moe_permute": ([vp, sp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "moe_grouped_gemm_swiglu": ([vp, vp, vp, vp, vp, sp, vp, vp], ctypes.c_int),
        "moe_grouped_gemm_down": ([vp, vp, vp, vp, sp, vp, vp], ctypes.c_int),
        "moe_finalize": ([vp, vp, vp, sp, vp, vp], ctypes.c_int),
        "moe_forward": ([vp, vp, vp, vp, vp, vp, sp, vp, vp, sz, vp], ctypes.c_int),
        "moe_forward_host": ([vp, vp, vp, vp, vp, vp, sp, vp, vp, sz, vp], ctypes.c_int),
        "moe_dequant_int4": ([vp, vp, i32, i32, vp, vp], ctypes.c_int),
        "moe_mx_quantize": ([vp, i32, i32, vp, vp, vp], ctypes.c_int),
        "moe_forward_fused": ([vp, vp, vp, vp, sp, vp, vp, sz, vp], ctypes.c_int),
        "moe_grouped_gemm_swiglu_mx": ([vp, vp, vp, vp, vp, vp, sp, vp, vp, vp], ctypes.c_int),
        "moe_grouped_gemm_down_mx": ([vp, vp, vp, vp, vp, sp, vp, vp], ctypes.c_int),
        "moe_permute_noalloc": ([vp, sp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "moe_get_device_error": ([ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
        "moe_selftest_bounded_wait": ([ctypes.c_int64, vp], ctypes.c_int),
        "moe_forward_kernel_count": ([sp], ctypes.c_int32),
        "moe_forward_gathers_in_gemm": ([sp], ctypes.c_int32),
        "moe_forward_is_fused": ([sp], ctypes.c_int32),
        "moe_ep_count": ([vp, sp, ctypes.POINTER(EpPeers), vp], ctypes.c_int),
        "moe_ep_dispatch": ([vp, vp, vp, sp, ctypes.POINTER(EpPeers), vp], ctypes.c_int),
        "moe_ep_local_offsets": ([sp, ctypes.POINTER(EpPeers), vp, vp], ctypes.c_int),
        "moe_ep_combine": ([vp, vp, sp, ctypes.POINTER(EpPeers), vp], ctypes.c_int),
        "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    }
    for name, (args, res) in sigs.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


# ---- marshalling helpers ---------------------------------------------------

BF16, F32, I32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def _p(t, *dtypes) -> Optional[int]:
    """Device (or host) address of a tensor, None for None. With dtypes, a
    tensor of another dtype is refused (the C ABI takes untyped pointers)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if dtypes and t.dtype not in dtypes:
        raise TypeError(f"libmoe_b200: expected a tensor of {' or '.join(map(str, dtypes))}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe_b200 must be contiguous")
    return t.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise MoeError(status, where)


def _shape(shape) -> Shape:
    if isinstance(shape, Shape):
        return shape
    return Shape.of(*shape)


# ---- entry points (same names as the C ABI) --------------------------------

def moe_workspace_size(shape) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(_shape(shape))))


def moe_permute_workspace_size(shape) -> int:
    return int(lib().moe_permute_workspace_size(ctypes.byref(_shape(shape))))


def moe_forward_host_workspace_size(shape) -> int:
    return int(lib().moe_forward_host_workspace_size(ctypes.byref(_shape(shape))))


def moe_route(logits, shape, topk_ids, topk_w, stream=None) -> None:
    _check(lib().moe_route(_p(logits, F32), ctypes.byref(_shape(shape)), _p(topk_ids, I32), _p(topk_w, F32),
                           _s(stream)),
           "moe_route")


def moe_permute(topk_ids, shape, counts, offsets, perm, inv_perm, hidden=None, hidden_perm=None,
                ws=None, stream=None) -> None:
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().moe_permute(_p(topk_ids, I32), ctypes.byref(_shape(shape)), _p(counts, I32), _p(offsets, I32),
                             _p(perm, I32), _p(inv_perm, I32), _p(hidden, BF16), _p(hidden_perm, BF16), _p(ws),
                             nbytes, _s(stream)),
           "moe_permute")


def moe_permute_noalloc(topk_ids, shape, counts, offsets, perm, inv_perm, hidden=None, hidden_perm=None,
                        stream=None) -> None:
    """moe_permute without a workspace: its scratch is a fixed array inside the
    library (for callers that cannot allocate device memory)."""
    _check(lib().moe_permute_noalloc(_p(topk_ids, I32), ctypes.byref(_shape(shape)), _p(counts, I32),
                                     _p(offsets, I32), _p(perm, I32), _p(inv_perm, I32), _p(hidden, BF16),
                                     _p(hidden_perm, BF16), _s(stream)),
           "moe_permute_noalloc")


def moe_grouped_gemm_swiglu(a, perm, offsets, w_gu, w_gu_scales, shape, act, stream=None) -> None:
    _check(lib().moe_grouped_gemm_swiglu(_p(a, BF16), _p(perm, I32), _p(offsets, I32), _p(w_gu, BF16, U8),
                                         _p(w_gu_scales, BF16, U8), ctypes.byref(_shape(shape)), _p(act, BF16),
                                         _s(stream)),
           "moe_grouped_gemm_swiglu")


def moe_grouped_gemm_down(act, offsets, w_d, w_d_scales, shape, y, stream=None) -> None:
    _check(lib().moe_grouped_gemm_down(_p(act, BF16), _p(offsets, I32), _p(w_d, BF16, U8), _p(w_d_scales, BF16, U8),
                                       ctypes.byref(_shape(shape)), _p(y, BF16), _s(stream)),
           "moe_grouped_gemm_down")


def moe_finalize(y, topk_w, inv_perm, shape, out, stream=None) -> None:
    _check(lib().moe_finalize(_p(y, BF16), _p(topk_w, F32), _p(inv_perm, I32), ctypes.byref(_shape(shape)),
                              _p(out, BF16), _s(stream)),
           "moe_finalize")


def moe_forward(hidden, logits, w_gu, w_gu_scales, w_d, w_d_scales, shape, out, ws, stream=None) -> None:
    nbytes = ws.numel() * ws.element_size()
    _check(lib().moe_forward(_p(hidden, BF16), _p(logits, F32), _p(w_gu, BF16, U8), _p(w_gu_scales, BF16, U8),
                             _p(w_d, BF16, U8), _p(w_d_scales, BF16, U8), ctypes.byref(_shape(shape)), _p(out, BF16),
                             _p(ws), nbytes, _s(stream)),
           "moe_forward")


def moe_forward_host(hidden_host, logits_host, w_gu, w_gu_scales, w_d, w_d_scales, shape, out_host, ws,
                     stream=None) -> None:
    nbytes = ws.numel() * ws.element_size()
    _check(lib().moe_forward_host(_p(hidden_host, BF16), _p(logits_host, F32), _p(w_gu, BF16, U8),
                                  _p(w_gu_scales, BF16, U8), _p(w_d, BF16, U8), _p(w_d_scales, BF16, U8),
                                  ctypes.byref(_shape(shape)), _p(out_host, BF16), _p(ws), nbytes, _s(stream)),
           "moe_forward_host")


def moe_forward_fused(hidden, logits, w_gu, w_d, shape, out, ws, stream=None) -> None:
    nbytes = ws.numel() * ws.element_size()
    _check(lib().moe_forward_fused(_p(hidden, BF16), _p(logits, F32), _p(w_gu, BF16), _p(w_d, BF16),
                                   ctypes.byref(_shape(shape)), _p(out, BF16), _p(ws), nbytes, _s(stream)),
           "moe_forward_fused")


def moe_mx_quantize(x, rows: int, K: int, q, scales, stream=None) -> None:
    _check(lib().moe_mx_quantize(_p(x, BF16), int(rows), int(K), _p(q, U8), _p(scales, U8), _s(stream)),
           "moe_mx_quantize")


def moe_grouped_gemm_swiglu_mx(a_q, a_scales, perm, offsets, w_gu, w_gu_scales, shape, act_q, act_scales,
                               stream=None) -> None:
    _check(lib().moe_grouped_gemm_swiglu_mx(_p(a_q, U8), _p(a_scales, U8), _p(perm, I32), _p(offsets, I32),
                                            _p(w_gu, U8), _p(w_gu_scales, U8), ctypes.byref(_shape(shape)),
                                            _p(act_q, U8), _p(act_scales, U8), _s(stream)),
           "moe_grouped_gemm_swiglu_mx")


def moe_grouped_gemm_down_mx(act_q, act_scales, offsets, w_d, w_d_scales, shape, y, stream=None) -> None:
    _check(lib().moe_grouped_gemm_down_mx(_p(act_q, U8), _p(act_scales, U8), _p(offsets, I32), _p(w_d, U8),
                                          _p(w_d_scales, U8), ctypes.byref(_shape(shape)), _p(y, BF16), _s(stream)),
           "moe_grouped_gemm_down_mx")


def moe_dequant_int4(q, scales, rows: int, K: int, out, stream=None) -> None:
    _check(lib().moe_dequant_int4(_p(q, U8), _p(scales, BF16), int(rows), int(K), _p(out, BF16), _s(stream)),
           "moe_dequant_int4")


def moe_forward_kernel_count(shape) -> int:
    return int(lib().moe_forward_kernel_count(ctypes.byref(_shape(shape))))


def moe_forward_is_fused(shape) -> bool:
    v = int(lib().moe_forward_is_fused(ctypes.byref(_shape(shape))))
    if v < 0:
        raise MoeError(1, "moe_forward_is_fused: invalid shape")
    return v == 1


def moe_forward_gathers_in_gemm(shape) -> bool:
    v = int(lib().moe_forward_gathers_in_gemm(ctypes.byref(_shape(shape))))
    if v < 0:
        raise MoeError(1, "moe_forward_gathers_in_gemm: invalid shape")
    return v == 1


def moe_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    _check(lib().moe_selftest_bounded_wait(int(limit_ns), _s(stream)), "moe_selftest_bounded_wait")


def moe_get_device_error() -> int:
    code = ctypes.c_int32(0)
    _check(lib().moe_get_device_error(ctypes.byref(code)), "moe_get_device_error")
    return int(code.value)


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


# ---- convenience -----------------------------------------------------------

def forward(hidden: torch.Tensor, logits: torch.Tensor, w_gu: torch.Tensor, w_d: torch.Tensor, top_k: int,
            w_gu_scales: Optional[torch.Tensor] = None, w_d_scales: Optional[torch.Tensor] = None,
            out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_forward on device tensors; allocates out and the workspace with
    torch when they are not given. hidden [T,H] bf16, logits [T,E] fp32,
    w_gu [E+S,2I,H] bf16 (or uint8: int4 [E+S,2I,H/2] with bf16 scales, MXFP8
    [E+S,2I,H] or MXFP4 [E+S,2I,H/2] with uint8 scales), w_d likewise:
    weight arrays with more experts than logits columns hold S shared experts
    after the E routed ones."""
    T, H = hidden.shape
    E = logits.shape[1]
    if w_gu.dtype != torch.uint8:
        fmt = FMT_BF16
    elif w_gu_scales is None or w_gu_scales.dtype != torch.uint8:
        fmt = FMT_INT4_G128
    else:
        fmt = FMT_MXFP4 if w_gu.shape[2] * 2 == H else FMT_MXFP8
    I = w_d.shape[2] * (2 if fmt in (FMT_INT4_G128, FMT_MXFP4) else 1)
    shape = Shape.of(T, H, I, E, top_k, fmt, n_shared=w_gu.shape[0] - E)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=hidden.device)
    if ws is None:
        ws = torch.empty(max(moe_workspace_size(shape), 1), dtype=torch.uint8, device=hidden.device)
    moe_forward(hidden, logits, w_gu, w_gu_scales, w_d, w_d_scales, shape, out, ws, stream)
    return out


# ---- expert parallelism -----------------------------------------------------

def moe_ep_count(offsets, shape, peers: EpPeers, stream=None) -> None:
    _check(lib().moe_ep_count(_p(offsets, I32), ctypes.byref(_shape(shape)), ctypes.byref(peers), _s(stream)),
           "moe_ep_count")


def moe_ep_dispatch(hidden, perm, offsets, shape, peers: EpPeers, stream=None) -> None:
    _check(lib().moe_ep_dispatch(_p(hidden, BF16), _p(perm, I32), _p(offsets, I32), ctypes.byref(_shape(shape)),
                                 ctypes.byref(peers), _s(stream)), "moe_ep_dispatch")


def moe_ep_local_offsets(shape, peers: EpPeers, offsets_local, stream=None) -> None:
    _check(lib().moe_ep_local_offsets(ctypes.byref(_shape(shape)), ctypes.byref(peers), _p(offsets_local, I32),
                                      _s(stream)), "moe_ep_local_offsets")


def moe_ep_combine(y_local, offsets_local, shape, peers: EpPeers, stream=None) -> None:
    _check(lib().moe_ep_combine(_p(y_local, BF16), _p(offsets_local, I32), ctypes.byref(_shape(shape)),
                                ctypes.byref(peers), _s(stream)), "moe_ep_combine")


def ep_forward(ranks, w_gu_shards, w_d_shards, top_k: int, devices=None):
    """The layer with its experts split over len(ranks) ranks driven from one
    process: rank r holds tokens ranks[r] = (hidden [T_r,H] bf16, logits
    [T_r,E] fp32) and the weights of experts r*E/R .. (r+1)*E/R - 1
    (w_gu_shards[r] [E/R,2I,H], w_d_shards[r] [E/R,H,I], bf16), all on device
    devices[r] (default: the current device for every rank, i.e. R ranks
    emulated on one GPU; ranks on different GPUs need peer access between
    them). The phases (route and permute, count, dispatch, local GEMMs,
    combine, finalize) are separated by a synchronisation of every rank's
    device, the barrier moe_ep_peers_t's steps ask for. Returns each rank's
    out [T_r,H] bf16."""
    R = len(ranks)
    if not 1 <= R <= EP_MAX_RANKS:
        raise ValueError(f"1 <= ranks <= {EP_MAX_RANKS}")
    devs = [torch.device(d) for d in (devices or [torch.cuda.current_device()] * R)]
    H = ranks[0][0].shape[1]
    E = ranks[0][1].shape[1]
    E_loc, I = w_d_shards[0].shape[0], w_d_shards[0].shape[2]
    if E_loc * R != E:
        raise ValueError("the weight shards must split the E experts evenly")
    k = int(top_k)
    Ts = [int(h.shape[0]) for h, _ in ranks]
    capacity = ((sum(Ts) * k + k - 1) // k) * k          # every pair of every rank at one owner
    i32 = torch.int32
    st = []
    for r, (h, lg) in enumerate(ranks):
        d = devs[r]
        P = Ts[r] * k
        st.append({
            "shape": Shape.of(Ts[r], H, I, E, k),
            "ids": torch.empty(Ts[r], k, dtype=i32, device=d), "w": torch.empty(Ts[r], k, device=d),
            "counts_g": torch.empty(E, dtype=i32, device=d), "offsets": torch.empty(E + 1, dtype=i32, device=d),
            "perm": torch.empty(P, dtype=i32, device=d), "inv": torch.empty(P, dtype=i32, device=d),
            "counts": torch.zeros(R, E_loc, dtype=i32, device=d),
            "recv_rows": torch.empty(capacity, H, dtype=torch.bfloat16, device=d),
            "recv_src": torch.empty(capacity, dtype=i32, device=d),
            "y_ret": torch.empty(max(P, 1), H, dtype=torch.bfloat16, device=d),
            "off_loc": torch.empty(E_loc + 1, dtype=i32, device=d),
            "act": torch.empty(capacity, I, dtype=torch.bfloat16, device=d),
            "y_loc": torch.empty(capacity, H, dtype=torch.bfloat16, device=d),
            "out": torch.empty(Ts[r], H, dtype=torch.bfloat16, device=d),
            "pws": torch.empty(max(1, moe_permute_workspace_size(Shape.of(Ts[r], H, I, E, k))), dtype=torch.uint8,
                               device=d),
        })
    shape_loc = Shape.of(capacity // k, H, I, E_loc, k)

    def peers(r):
        pe = EpPeers()
        pe.world, pe.rank, pe.capacity = R, r, capacity
        for q in range(R):
            pe.counts[q] = st[q]["counts"].data_ptr()
            pe.recv_rows[q] = st[q]["recv_rows"].data_ptr()
            pe.recv_src[q] = st[q]["recv_src"].data_ptr()
            pe.y_ret[q] = st[q]["y_ret"].data_ptr()
            pe.pairs[q] = Ts[q] * k
        return pe

    def barrier():
        for d in set(devs):
            torch.cuda.synchronize(d)

    def each(fn):
        for r in range(R):
            with torch.cuda.device(devs[r]):
                fn(r)
        barrier()

    def route_permute(r):
        h, lg = ranks[r]
        s = st[r]
        moe_route(lg, s["shape"], s["ids"], s["w"])
        moe_permute(s["ids"], s["shape"], s["counts_g"], s["offsets"], s["perm"], s["inv"], None, None, s["pws"])

    def local_gemms(r):
        s = st[r]
        moe_ep_local_offsets(s["shape"], peers(r), s["off_loc"])
        moe_grouped_gemm_swiglu(s["recv_rows"], None, s["off_loc"], w_gu_shards[r], None, shape_loc, s["act"])
        moe_grouped_gemm_down(s["act"], s["off_loc"], w_d_shards[r], None, shape_loc, s["y_loc"])

    def finalize(r):
        s = st[r]
        ident = torch.arange(Ts[r] * k, dtype=i32, device=devs[r])
        moe_finalize(s["y_ret"], s["w"], ident, s["shape"], s["out"])

    each(route_permute)
    each(lambda r: moe_ep_count(st[r]["offsets"], st[r]["shape"], peers(r)))
    each(lambda r: moe_ep_dispatch(ranks[r][0], st[r]["perm"], st[r]["offsets"], st[r]["shape"], peers(r)))
    each(local_gemms)
    each(lambda r: moe_ep_combine(st[r]["y_loc"], st[r]["off_loc"], st[r]["shape"], peers(r)))
    each(finalize)
    return [s["out"] for s in st]
