"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device memory.

Such callers (a plug-in inside a host application that owns all device buffers, a serving loop
that must not call cudaMalloc/cudaFree) pass only inputs and outputs; the scratch comes from the
library's static device array. These tests call the entry point through the C ABI and require
its outputs to equal, bit for bit (dispatch is integer and byte work), those of moe_dispatch with
a caller workspace, on two calls in a row with different problems, so the second call runs on the
scratch the first one left behind.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_layer_57_b200 import moe
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu


def _problem(seed, T, E, k, d):
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, E + 1) ** 1.1
    p /= p.sum()
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    return to_dev(ids), x.cuda()


def test_noalloc_matches_workspace_dispatch_twice(cuda_ok):
    cases = [(1, 5000, 64, 2, 256, 1.0), (2, 777, 128, 1, 1024, 1.25)]
    for seed, T, E, k, d, cf in cases:
        ids, x = _problem(seed, T, E, k, d)
        C = moe.moe_capacity(T, E, k, cf)
        ref = moe.moe_dispatch(x, ids, E, C)
        got = moe.moe_dispatch_noalloc(x, ids, E, C)
        torch.cuda.synchronize()
        for name in ("slot", "expert_counts", "expert_offsets"):
            assert torch.equal(got[name], ref[name]), name
        total = int(ref["expert_offsets"][-1])
        assert torch.equal(got["row_token"][:total], ref["row_token"][:total])
        assert torch.equal(got["x_packed"][:total].view(torch.int16),
                           ref["x_packed"][:total].view(torch.int16))
        assert moe.moe_last_launch_count() == 3


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_ok):
    # T*k = 2^20 pairs need 4 MiB of ranks alone: more than the built-in array
    L = moe.lib()
    fake = 0x10000
    st = L.moe_dispatch_noalloc(fake, 1, 1 << 20, 64, fake, 8, 1, 1 << 20, fake, fake, fake, fake,
                                fake, 1 << 20, None)
    assert st == 3   # MOE_ERR_WORKSPACE_TOO_SMALL
    assert ctypes.c_char_p(L.moe_status_string(st)).value == b"MOE_ERR_WORKSPACE_TOO_SMALL"
