"""Wide expert GEMM tiles on CTA pairs (cta_group::2 MMAs of M = 256 over two SMs) against one CTA
per tile, and against the oracle.

Layers whose capacity picks 256-token tiles (compute-bound expert GEMMs, as in the top-2 E = 8
workload) run their two expert GEMM layers on CTA pairs unless MOE_PAIR_MMA=0. The pair kernel
forms every output element from the same products in the same K order as the one-CTA kernel, so
the layer outputs must agree bit for bit; the oracle bounds both. Ragged expert segments, an odd
feature-tile count (d_ff = 768: the last 256-feature tile half past the expert's rows) and a
partial last token tile are covered.
"""
import os

import numpy as np
import pytest

import synth
from tests.helpers import check_out, dev_inputs, oracle_layer, run_layer

pytestmark = pytest.mark.gpu


def _run(w, d, pair: str, **kw):
    old = os.environ.get("MOE_PAIR_MMA")
    os.environ["MOE_PAIR_MMA"] = pair
    try:
        return run_layer(w, d, want_losses=True, **kw)
    finally:
        if old is None:
            os.environ.pop("MOE_PAIR_MMA", None)
        else:
            os.environ["MOE_PAIR_MMA"] = old


@pytest.mark.parametrize("kw", [dict(T=2048, d_model=512, d_ff=1024),
                                dict(T=1500, E=6, d_model=256, d_ff=768),
                                dict(T=1100, E=4, k=1, d_model=256, d_ff=512)])
def test_pair_tiles_equal_single_and_oracle(cuda_ok, kw):
    import mixture_experts_layer_57_b200.moe as moe
    w = synth.WORKLOADS[4].with_(**kw)
    assert moe.moe_capacity(w.T, w.E, w.k, w.capacity_factor) > 128  # 256-token tiles
    inp = synth.make_inputs(w)
    d = dev_inputs(inp)
    single = _run(w, d, "0")
    pair = _run(w, d, "1")
    assert single["device_error"] == 0 and pair["device_error"] == 0
    for name in ("out", "expert_ids", "slot", "gates"):
        assert np.array_equal(pair[name], single[name]), name
    ref = oracle_layer(inp, w, logits_in=pair["logits"])
    check_out(pair["out"], ref["out_exact"], True, True, what=f"pair {kw}")


def test_pair_tiles_full_size_equal_single(cuda_ok):
    w = synth.WORKLOADS[4]
    inp = synth.make_inputs(w)
    d = dev_inputs(inp)
    single = _run(w, d, "0")
    pair = _run(w, d, "1")
    assert single["device_error"] == 0 and pair["device_error"] == 0
    assert np.array_equal(pair["out"], single["out"])
