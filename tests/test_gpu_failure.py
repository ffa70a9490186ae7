"""Failure detection on the GPU without a fault: a bounded wait that cannot complete gives up.

moe_selftest_bounded_wait launches the grouped expert GEMM on a one-tile problem whose TMA role
issues no copy, so the MMA role waits on a barrier nobody arrives at (and the epilogue on an
accumulator that never fills). With a 1 ms limit every wait gives up, the kernel records
MOE_DEVERR_TIMEOUT in the workspace's status block, stops its roles, frees TMEM and returns: the
host reads the code, and the context stays usable for a normal layer call on a fresh workspace,
whose result is then checked against the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import check_out, dev_inputs, run_layer

pytestmark = pytest.mark.gpu

MOE_DEVERR_TIMEOUT = 1


def test_bounded_wait_expires_and_context_survives(cuda_ok):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ws = moe.moe_selftest_bounded_wait(1_000_000)          # 1 ms
    code = moe.moe_get_device_error(ws)                    # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert code == MOE_DEVERR_TIMEOUT
    assert elapsed < 5.0, f"the kernel took {elapsed:.2f} s to give up"
    assert moe.moe_last_launch_count() == 1

    # the device is still healthy: a normal layer on a fresh workspace matches the oracle
    w = synth.WORKLOADS[2].with_(T=300, d_model=256, d_ff=512, E=8)
    inp = synth.make_inputs(w)
    got = run_layer(w, dev_inputs(inp))
    assert got["device_error"] == 0
    ref = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                               add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha,
                               logits_in=got["logits"])
    assert np.array_equal(got["slot"], ref["slot"])
    check_out(got["out"], ref["out_exact"], True, True, what="after the expired wait")


def test_selftest_argument_checks(cuda_ok):
    L = moe.lib()
    ws = moe.workspace(moe.MOE_SELFTEST_WS_BYTES, "cuda")
    assert L.moe_selftest_bounded_wait(ws.data_ptr(), ws.numel(), 10, None) == 1   # limit too short
    assert L.moe_selftest_bounded_wait(ws.data_ptr(), 1024, 1_000_000, None) == 3  # ws too small
    assert L.moe_selftest_bounded_wait(None, ws.numel(), 1_000_000, None) == 1
    assert moe.moe_get_device_error(ws) == 0                                       # nothing ran
