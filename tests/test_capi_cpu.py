"""The C-ABI library without a GPU: it loads, exports every entry point that
include/moe.h declares, and rejects bad arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

import moe_synth
import mixture_experts_expert_top_b200 as moe
from mixture_experts_expert_top_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    moe_build.build()


def declared_entry_points():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)
    return names


def test_header_declares_the_layer_entry_points():
    names = declared_entry_points()
    for n in ("moe_route", "moe_permute", "moe_grouped_gemm_swiglu", "moe_grouped_gemm_down",
              "moe_finalize", "moe_forward", "moe_workspace_size", "moe_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(moe.library_path)
    for n in declared_entry_points():
        assert hasattr(lib, n), n


def test_debug_bounds_library_builds_and_exports_every_declared_symbol():
    # the -DMOE_DEBUG_BOUNDS build of the same sources (range checks in the
    # kernels, device error 4) is a drop-in replacement for the release library
    path = moe_build.build(debug_bounds=True)
    assert path != moe.library_path
    lib = ctypes.CDLL(path)
    for n in declared_entry_points():
        assert hasattr(lib, n), n
    with moe.debug_bounds_library() as L:
        assert moe.lib() is L
        assert moe.moe_workspace_size(moe.Shape.of(64, 2048, 768, 128, 8)) == \
            ctypes.CDLL(moe.library_path).moe_workspace_size(ctypes.byref(moe.Shape.of(64, 2048, 768, 128, 8)))
    assert moe.lib() is not L


def test_binding_names_match_the_header():
    for n in declared_entry_points():
        assert callable(getattr(moe, n)), n


def test_status_strings():
    assert moe.moe_status_string(0) == "ok"
    assert "workspace" in moe.moe_status_string(3)
    assert moe.moe_status_string(99) == "unknown status"


@pytest.mark.parametrize("shape,ok", [
    ((16, 128, 64, 8, 2, 0), True),
    ((0, 128, 64, 8, 2, 0), True),
    ((16, 128, 64, 8, 9, 0), False),       # k > E
    ((16, 128, 64, 0, 1, 0), False),       # E = 0
    ((16, 130, 64, 8, 2, 0), False),       # H not a multiple of 8
    ((16, 128, 64, 2048, 2, 0), False),    # E > 1024
    ((16, 128, 64, 64, 33, 0), False),     # k > 32
    ((16, 192, 128, 8, 2, 1), False),      # int4 needs H % 128 == 0
    ((16, 256, 128, 8, 2, 1), True),
    ((-1, 128, 64, 8, 2, 0), False),
    ((16, 128, 64, 8, 2, 7), False),       # unknown format
])
def test_workspace_size_validates_the_shape(shape, ok):
    n = moe.moe_workspace_size(moe.Shape.of(*shape))
    assert (n > 0) == ok or (shape[0] == 0 and n >= 0)


def test_workspace_grows_with_tokens():
    a = moe.moe_workspace_size(moe.Shape.of(64, 2048, 768, 128, 8))
    b = moe.moe_workspace_size(moe.Shape.of(128, 2048, 768, 128, 8))
    assert b > a > 64 * 8 * (2048 * 2 + 768 * 2)
    assert moe.moe_forward_host_workspace_size(moe.Shape.of(64, 2048, 768, 128, 8)) > a
    assert moe.moe_permute_workspace_size(moe.Shape.of(64, 2048, 768, 128, 8)) == 0
    assert moe.moe_permute_workspace_size(moe.Shape.of(8192, 2048, 768, 128, 8)) == 32 * 128 * 4


def test_bad_arguments_are_rejected_before_any_launch():
    L = moe.lib()
    sh = moe.Shape.of(16, 128, 64, 8, 2)
    byref = ctypes.byref
    # null pointers
    assert L.moe_route(None, byref(sh), None, None, None) == 1
    assert L.moe_finalize(None, None, None, byref(sh), None, None) == 1
    assert L.moe_forward(None, None, None, None, None, None, byref(sh), None, None, 0, None) == 1
    # misaligned perm for the fused gather
    assert L.moe_grouped_gemm_swiglu(16, 18, 16, 16, None, byref(sh), 16, None) == 1
    # misaligned hidden
    assert L.moe_forward(17, 16, 16, None, 16, None, byref(sh), 16, 256, 1 << 30, None) == 1
    # scales given for bf16 weights
    assert L.moe_grouped_gemm_down(16, 16, 16, 16, byref(sh), 16, None) == 1
    # int4 without scales
    sh4 = moe.Shape.of(16, 256, 128, 8, 2, moe.FMT_INT4_G128)
    assert L.moe_grouped_gemm_down(16, 16, 16, None, byref(sh4), 16, None) == 1
    # workspace too small
    assert L.moe_forward(16, 16, 16, None, 16, None, byref(sh), 16, 256, 1024, None) == 3
    # k > E
    bad = moe.Shape.of(16, 128, 64, 8, 9)
    assert L.moe_route(16, byref(bad), 16, 16, None) == 1
    # permute: hidden without hidden_perm
    assert L.moe_permute(16, byref(sh), 16, 16, 16, 16, 16, None, None, 0, None) == 1
    # dequant: K not a multiple of 128
    assert L.moe_dequant_int4(16, 16, 4, 100, 16, None) == 1
    # bounded-wait self-test: limit outside 1 ns .. 1 s
    assert L.moe_selftest_bounded_wait(0, None) == 1
    assert L.moe_selftest_bounded_wait(2_000_000_000, None) == 1


def test_empty_batch_is_a_no_op():
    L = moe.lib()
    sh = moe.Shape.of(0, 128, 64, 8, 2)
    byref = ctypes.byref
    assert L.moe_route(None, byref(sh), None, None, None) == 0
    assert L.moe_permute(None, byref(sh), None, None, None, None, None, None, None, 0, None) == 0
    assert L.moe_forward(None, None, None, None, None, None, byref(sh), None, None, 0, None) == 0
    assert L.moe_finalize(None, None, None, byref(sh), None, None) == 0


def test_forward_kernel_count():
    # bf16 decode batches: the counter reset and the persistent kernel; else
    # one-CTA route+permute for T <= 64; the decode-shaped gate/up reads its
    # token rows through perm; prefill shapes add two bucketing kernels (three
    # past 64 chunks of 2048 pairs or 512 experts) and the gather
    sh = lambda c: moe.Shape.of(c.T, c.H, c.I, c.E, c.k, c.fmt, n_shared=c.n_shared)
    count = lambda c: moe.moe_forward_kernel_count(sh(c))
    assert count(moe_synth.get_config("qwen3_decode")) == 2
    assert count(moe_synth.get_config("tiny")) == 2
    assert count(moe_synth.get_config("shared_decode")) == 2
    assert count(moe_synth.get_config("mxfp8_decode")) == 5
    assert count(moe_synth.get_config("mxfp4_decode")) == 5
    assert count(moe_synth.get_config("qwen3_decode", T=65)) == 5            # past the persistent kernel's batch
    assert count(moe_synth.get_config("w4a16_decode")) == 5
    fused = lambda c: moe.moe_forward_is_fused(sh(c))
    assert fused(moe_synth.get_config("qwen3_decode")) and fused(moe_synth.get_config("shared_decode"))
    assert not fused(moe_synth.get_config("w4a16_decode")) and not fused(moe_synth.get_config("mxfp8_decode"))
    assert not fused(moe_synth.get_config("mxfp4_decode"))
    assert not fused(moe_synth.get_config("qwen3_prefill"))
    assert not fused(moe_synth.get_config("qwen3_decode", E=300))                # more experts than it takes
    assert count(moe_synth.get_config("qwen3_prefill")) == 7
    assert count(moe_synth.get_config("skewed")) == 7
    assert count(moe_synth.get_config("qwen3_prefill", T=20000)) == 8           # 79 chunks: separate scan
    assert moe.moe_forward_gathers_in_gemm(sh(moe_synth.get_config("qwen3_decode")))
    assert moe.moe_forward_gathers_in_gemm(sh(moe_synth.get_config("w4a16_decode")))
    assert not moe.moe_forward_gathers_in_gemm(sh(moe_synth.get_config("qwen3_prefill")))
    assert count(moe_synth.get_config("tiny", T=0)) == 0
    assert moe.moe_forward_kernel_count(moe.Shape.of(16, 128, 64, 8, 9)) == -1     # k > E


def test_binding_refuses_tensors_of_the_wrong_dtype():
    # checked in the binding before the library is called: no GPU needed
    import torch
    sh = moe.Shape.of(4, 128, 64, 8, 2)
    f32 = torch.zeros(4, 8)
    with pytest.raises(TypeError):
        moe.moe_route(f32.to(torch.float64), sh, torch.zeros(4, 2, dtype=torch.int32), torch.zeros(4, 2))
    with pytest.raises(TypeError):
        moe.moe_finalize(torch.zeros(8, 128), torch.zeros(4, 2), torch.zeros(8, dtype=torch.int32), sh,
                         torch.zeros(4, 128, dtype=torch.bfloat16))


C_CLIENT = r"""
#include <stddef.h>
#include <stdio.h>
#include <string.h>
#include "moe.h"

int main(void) {
    moe_shape_t s;
    s.T = 64; s.H = 2048; s.I = 768; s.E = 128; s.top_k = 8; s.fmt = MOE_W_BF16; s.n_shared = 0;
    size_t ws = moe_workspace_size(&s);
    moe_shape_t bad = s;
    bad.top_k = 129;
    int rc = 0;
    if (ws == 0) rc = 1;
    if (moe_workspace_size(&bad) != 0) rc = 2;
    if (moe_forward_kernel_count(&s) != 2 || moe_forward_is_fused(&s) != 1) rc = 3;
    if (strcmp(moe_status_string(MOE_OK), "ok") != 0) rc = 4;
    /* T = 0 enqueues nothing and succeeds without a GPU */
    s.T = 0;
    if (moe_forward(NULL, NULL, NULL, NULL, NULL, NULL, &s, NULL, NULL, 0, NULL) != MOE_OK) rc = 5;
    printf("%zu %d %zu %zu\n", ws, rc, sizeof(moe_ep_peers_t), offsetof(moe_ep_peers_t, pairs));
    return rc;
}
"""


def test_the_header_compiles_as_c99_and_a_c_program_links_and_runs(tmp_path):
    # the boundary is a C ABI: plain C must be able to include moe.h, link
    # libmoe_b200.so and call the host-side entry points (no GPU needed)
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    moe_build.build()
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    inc = os.path.join(os.path.dirname(os.path.dirname(moe.__file__)), "include")
    libdir = os.path.dirname(moe.library_path)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", inc, str(src), "-o", str(exe),
                        "-L", libdir, "-l:libmoe_b200.so", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.stdout, r.stderr)
    out = r.stdout.split()
    assert int(out[0]) > 0
    # the binding's moe_ep_peers_t has the C layout
    assert int(out[2]) == ctypes.sizeof(moe.EpPeers) and int(out[3]) == moe.EpPeers.pairs.offset


def test_ep_entry_points_validate_on_the_host():
    # refused before anything is enqueued: no GPU needed (addresses are never used)
    sh = moe.Shape.of(16, 128, 64, 8, 2)
    pe = moe.EpPeers()
    pe.world, pe.rank, pe.capacity = 3, 0, 32            # 8 experts do not split over 3 ranks
    for q in range(3):
        pe.counts[q] = pe.recv_rows[q] = pe.recv_src[q] = pe.y_ret[q] = 1 << 20
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_count(1 << 20, sh, pe, stream=0)
    assert ei.value.status == 2
    pe.world, pe.rank = 2, 2                             # rank outside the world
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_count(1 << 20, sh, pe, stream=0)
    assert ei.value.status == 1
    pe.rank = 1
    pe.recv_rows[1] = (1 << 20) + 8                      # receive rows not 16-byte aligned
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_dispatch(1 << 20, 1 << 20, 1 << 20, sh, pe, stream=0)
    assert ei.value.status == 1
    shs = moe.Shape.of(16, 128, 64, 8, 2, n_shared=1)    # shared experts are not dispatched
    pe.recv_rows[1] = 1 << 20
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_local_offsets(shs, pe, 1 << 20, stream=0)
    assert ei.value.status == 2


@pytest.mark.parametrize("shape,status", [
    ((16, 128, 64, 8, 9, 0), 1),            # k > E: invalid
    ((16, 128, 64, 0, 1, 0), 1),            # E = 0: invalid
    ((16, 128, 64, 8, 2, 7), 1),            # unknown format: invalid
    ((16, 128, 64, 2048, 2, 0), 2),         # E > 1024: outside the library's limits
    ((16, 128, 64, 64, 33, 0), 2),          # k > 32
    ((16, 130, 64, 8, 2, 0), 2),            # H not a multiple of 8
    ((16, 192, 128, 8, 2, 1), 2),           # int4 needs H % 128 == 0
    ((300_000_000, 128, 64, 16, 8, 0), 2),  # T * k >= 2^31
])
def test_shape_checks_return_the_documented_status(shape, status):
    L = moe.lib()
    assert L.moe_route(16, ctypes.byref(moe.Shape.of(*shape)), 16, 16, None) == status


def test_noalloc_permute_refuses_shapes_beyond_its_scratch_before_any_launch():
    # ceil(600000 / 2048) = 293 chunks x 1024 experts > 65536 scratch entries
    L = moe.lib()
    sh = moe.Shape.of(600000, 8, 8, 1024, 1)
    assert L.moe_permute_noalloc(16, ctypes.byref(sh), 16, 16, 16, 16, None, None, None) == 2
