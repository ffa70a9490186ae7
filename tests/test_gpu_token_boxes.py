"""Co-scheduled PR-MoE layers whose experts hold few tokens: every expert tile loads only the token
rows its MMAs read (a TMA box of 32, 64 or 128 rows, the smallest that holds the tile's MMA N,
its rows rounded up to 16).

Routing is forced: W_r is the identity on the first E features and each token carries 8.0 in the
feature of its expert (0 in the other E - 1), so expert e's logit is 8 for its tokens and 0
otherwise. Expert loads of 32 / 33 / 64 / 65 / 150 tokens (capacity 128, 128-token tiles) put tiles
on both sides of each box boundary and drop 22 tokens of the last expert; loads of 16 / 32 / 33 /
64 / 90 (capacity 64, 64-token tiles: boxes of 32 or 64 rows) drop 26. The layer must match the
oracle and, bit for bit, the sequential launches (MOE_COSCHEDULE=0, which load whole boxes).
"""
import os

import numpy as np
import pytest

import synth
from tests.helpers import check_out, dev_inputs, oracle_layer, run_layer

pytestmark = pytest.mark.gpu

# (expert loads, capacity factor giving the capacity)
CASES = {128: ((32, 33, 64, 65, 150), 1.86),  # ceil(344 / 5 * 1.86) = 128
         64: ((16, 32, 33, 64, 90), 1.36)}    # ceil(235 / 5 * 1.36) = 64
BF16_EIGHT = 0x4100  # 8.0 in bfloat16


def forced_inputs(d_model: int, d_ff: int, seed: int, capacity: int = 128):
    loads, cf = CASES[capacity]
    E = len(loads)
    T = sum(loads)
    w = synth.WORKLOADS[3].with_(T=T, E=E, d_model=d_model, d_ff=d_ff, capacity_factor=cf,
                                 seed=seed)
    inp = synth.make_inputs(w)
    inp.pop("router_bias", None)
    expert_of = np.repeat(np.arange(E), loads)
    np.random.default_rng(seed).shuffle(expert_of)  # first-come order decides the drops
    x = inp["x"].copy()
    x[:, :E] = 0
    x[np.arange(T), expert_of] = BF16_EIGHT
    inp["x"] = x
    wr = np.zeros((E, d_model), dtype=np.float32)
    wr[np.arange(E), np.arange(E)] = 1.0
    inp["w_router"] = wr
    return w, inp, expert_of


def _run(w, d, cosched: str):
    old = os.environ.get("MOE_COSCHEDULE")
    os.environ["MOE_COSCHEDULE"] = cosched
    try:
        return run_layer(w, d)
    finally:
        if old is None:
            os.environ.pop("MOE_COSCHEDULE", None)
        else:
            os.environ["MOE_COSCHEDULE"] = old


@pytest.mark.parametrize("d_model,d_ff,seed,capacity", [(256, 512, 1, 128), (128, 768, 2, 128),
                                                       (256, 512, 3, 64)])
def test_short_token_boxes(cuda_ok, d_model, d_ff, seed, capacity):
    import mixture_experts_layer_57_b200.moe as moe
    w, inp, expert_of = forced_inputs(d_model, d_ff, seed, capacity)
    loads = CASES[capacity][0]
    assert moe.moe_capacity(w.T, w.E, w.k, w.capacity_factor) == capacity
    d = dev_inputs(inp)
    co = _run(w, d, "1")
    seq = _run(w, d, "0")
    assert co["device_error"] == 0 and seq["device_error"] == 0
    np.testing.assert_array_equal(co["expert_ids"][:, 0], expert_of)
    np.testing.assert_array_equal(co["expert_counts"], np.array(loads, dtype=np.int32))
    kept = np.minimum(np.array(loads), capacity)
    np.testing.assert_array_equal(np.diff(co["expert_offsets"]), kept)
    for name in ("out", "slot", "gates"):
        assert np.array_equal(co[name], seq[name]), name
    ref = oracle_layer(inp, w, logits_in=co["logits"])
    check_out(co["out"], ref["out_exact"], True, True, what=f"token boxes d={d_model} f={d_ff}")
