"""moe_permute_noalloc: the permute for callers that cannot allocate device
memory (a plugin inside a framework that owns every allocation and passes no
workspace, or a hot loop that must not call cudaMalloc because it can
synchronise the device). It takes its scratch from an array built into the
library. It must produce exactly what moe_permute produces with a caller
workspace. Two calls in a row with different inputs are checked, because
every call shares that one array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import mixture_experts_expert_top_b200 as moe
from mixture_experts_expert_top_b200 import build as moe_build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    moe_build.build()
    moe.lib()
    yield
    assert moe.moe_get_device_error() == 0


def _ids(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g) + torch.linspace(2, -2, E)[None, :]
    return torch.sort(logits, dim=1, descending=True, stable=True).indices[:, :k].to(torch.int32).contiguous()


def _outputs(T, E, k, H):
    i32 = dict(dtype=torch.int32, device=DEV)
    P = T * k
    return [torch.full((E,), -7, **i32), torch.full((E + 1,), -7, **i32), torch.full((P,), -7, **i32),
            torch.full((P,), -7, **i32), torch.zeros(P, H, dtype=torch.bfloat16, device=DEV)]


# 12 and 12 chunks of 2048 pairs: chunk counts scanned inside the scatter
# CTAs; 79 chunks: a separate scan kernel writes back into the scratch array;
# 256 chunks x 128 experts = 32768 entries, half of the array
@pytest.mark.parametrize("T,E,k,H", [(4096, 64, 6, 64), (3000, 128, 8, 32), (20000, 64, 8, 16), (65536, 128, 8, 8)])
def test_noalloc_permute_matches_permute_on_two_calls_in_a_row(T, E, k, H):
    shape = moe.Shape.of(T, H, 64, E, k)
    assert moe.moe_permute_workspace_size(shape) > 0      # the scratch path is the one under test
    ws = torch.empty(moe.moe_permute_workspace_size(shape), dtype=torch.uint8, device=DEV)
    for call, seed in enumerate((1, 2)):                    # the second call sees the first call's scratch
        ids = _ids(T, E, k, seed + T).to(DEV)
        hidden = torch.randn(T, H, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16).to(DEV)
        ref = _outputs(T, E, k, H)
        got = _outputs(T, E, k, H)
        moe.moe_permute(ids, shape, *ref[:4], hidden, ref[4], ws)
        moe.moe_permute_noalloc(ids, shape, *got[:4], hidden, got[4])
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "perm", "inv_perm", "hidden_perm"), ref, got):
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b), f"call {call}: {name}"
        assert int(got[1][-1]) == T * k


def test_noalloc_permute_rejects_calls_beyond_its_scratch():
    # ceil(600000 / 2048) = 293 chunks x 1024 experts > 65536 entries
    shape = moe.Shape.of(600000, 8, 8, 1024, 1)
    one = torch.zeros(4, dtype=torch.int32, device=DEV)
    status = moe.lib().moe_permute_noalloc(one.data_ptr(), moe.ctypes.byref(shape), one.data_ptr(), one.data_ptr(),
                                           one.data_ptr(), one.data_ptr(), None, None, None)
    assert status == 2      # MOE_ERR_UNSUPPORTED, nothing enqueued
