"""End-to-end GPU parity of moe_layer_forward against the oracle.

Routing and dispatch (ids, slots, demand counts, offsets) are bit-exact given the GPU's fp32
logits; the oracle runs the whole layer on those logits and its outputs are compared within the
tolerances of tests/helpers.py. Full-size workloads compare every token's routing and at least
128 output rows spread over the path's cases (a kept token of every touched expert, the first and
last rows and the token-tile boundaries of the largest segments, dropped and partially dropped
tokens); reduced versions of each workload compare every output row.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.helpers import check_out, dev_inputs, oracle_layer, run_layer, spread_tokens, to_dev

pytestmark = pytest.mark.gpu


def layer_parity(w: synth.Workload, inp=None, d_inp=None, n_sample=None, out_dtype=None,
                 add_input_residual=None, seed=0):
    inp = synth.make_inputs(w) if inp is None else inp
    d_inp = dev_inputs(inp) if d_inp is None else d_inp
    got = run_layer(w, d_inp, out_dtype=out_dtype, add_input_residual=add_input_residual)
    assert got["device_error"] == 0
    res = w.add_input_residual if add_input_residual is None else add_input_residual
    # routing from the GPU's logits: bit-exact
    rng = np.random.default_rng(seed)
    if n_sample is None or n_sample >= w.T:
        tokens = np.arange(w.T)
    else:
        ids_probe = oracle.route(got["logits"], w.k)[0]
        slot_probe, _ = oracle.assign_slots(ids_probe, w.E,
                                            oracle.capacity(w.T, w.E, w.k, w.capacity_factor))
        tokens = spread_tokens(w, ids_probe, slot_probe, n_sample, rng)
    bf16 = w.dtype == "bf16"
    out_bf16 = bf16 if out_dtype is None else out_dtype == torch.bfloat16
    ref = oracle_layer(inp, w, tokens, add_input_residual=res, logits_in=got["logits"],
                       out_bf16=out_bf16)
    assert np.array_equal(got["expert_ids"], ref["ids"])
    np.testing.assert_allclose(got["gates"], ref["gates"], rtol=2e-6, atol=1e-12)
    assert np.array_equal(got["slot"], ref["slot"])
    assert np.array_equal(got["expert_counts"], ref["counts"])
    off = np.concatenate([[0], np.cumsum(np.minimum(ref["counts"], ref["C"]))])
    assert np.array_equal(got["expert_offsets"], off.astype(np.int32))
    E = w.E
    np.testing.assert_array_equal(got["lb_stats"][:E], ref["f"].astype(np.float32))
    np.testing.assert_allclose(got["lb_stats"][E:2 * E], ref["Q"], rtol=1e-5, atol=1e-9)
    max_abs, rel = check_out(got["out"][tokens], ref["out_exact"], bf16, out_bf16, what=w.name)
    return dict(got=got, ref=ref, tokens=tokens, max_abs=max_abs, rel=rel)


def test_workload1_tiny_fp32_full(cuda_ok):
    r = layer_parity(synth.WORKLOADS[1])
    assert (r["got"]["slot"] < 0).any()          # capacity 16 binds: some tokens overflow


@pytest.mark.parametrize("cfg,T", [(2, 1024), (3, 512), (4, 512), (5, 32)])
def test_reduced_workloads_all_rows(cuda_ok, cfg, T):
    w = synth.WORKLOADS[cfg]
    shrink = dict(T=T)
    if cfg in (2, 3):
        shrink.update(d_model=512, d_ff=1024)
    if cfg == 4:
        shrink.update(d_model=1024, d_ff=2048)
    if cfg == 5:
        shrink.update(d_ff=2048)
    w = w.with_(**shrink)
    layer_parity(w)
    layer_parity(w, out_dtype=torch.float32)


@pytest.mark.parametrize("cfg,n", [(2, 256), (3, 160), (4, 128), (5, 32)])
def test_full_workloads_sampled(cuda_ok, cfg, n):
    w = synth.WORKLOADS[cfg]
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    r = layer_parity(w, inp, d_inp, n_sample=n, seed=cfg)
    assert len(r["tokens"]) >= min(n, w.T)
    r32 = layer_parity(w, inp, d_inp, n_sample=n // 2, out_dtype=torch.float32, seed=cfg + 10)
    print(f"workload {cfg}: bf16-out max-abs {r['max_abs']:.3e} rel-L2 {r['rel']:.3e}; "
          f"fp32-out max-abs {r32['max_abs']:.3e} rel-L2 {r32['rel']:.3e}")


@pytest.mark.parametrize("shape", [
    dict(T=2048, d_model=1024, d_ff=2048, E=16),    # capacity 128: 128-token expert tiles
    dict(T=1000, d_model=512, d_ff=1024, E=128),    # capacity 8: 16-token expert tiles, ragged T
    dict(T=300, d_model=256, d_ff=128, E=4),        # one 128-feature tile per expert
    dict(T=600, d_model=256, d_ff=512, E=8, capacity_factor=0.0),  # no expert rows at all
])
def test_prmoe_coscheduled_equals_sequential(cuda_ok, monkeypatch, shape):
    # the expert and dense GEMM layers co-scheduled in one launch each (default) give the same
    # bits as the sequential launches with the combine fused into the dense layer 2 epilogue;
    # both match the oracle
    w = synth.WORKLOADS[3].with_(**shape)
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    co = layer_parity(w, inp, d_inp)["got"]
    monkeypatch.setenv("MOE_COSCHEDULE", "0")
    seq = layer_parity(w, inp, d_inp)["got"]
    # co-scheduled: two GEMM launches and the combine; sequential: four GEMM launches, or only
    # the dense MLP's two when no expert keeps a row
    no_rows = int(co["expert_offsets"][-1]) == 0
    assert co["launches"] == seq["launches"] + (1 if no_rows else -1)
    assert np.array_equal(co["out"], seq["out"])
    for name in ("expert_ids", "gates", "slot", "expert_offsets", "lb_stats"):
        assert np.array_equal(co[name], seq[name]), name


def test_prmoe_both_residual_conventions(cuda_ok):
    w = synth.WORKLOADS[3].with_(T=384, d_model=256, d_ff=512)
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    layer_parity(w, inp, d_inp, add_input_residual=False)
    layer_parity(w, inp, d_inp, add_input_residual=True)


@pytest.mark.parametrize("name,kw", [
    ("T=1", dict(T=1)),
    ("k=E", dict(k=4, E=4, capacity_factor=1.0)),
    ("C=0", dict(capacity_factor=0.0)),
    ("C>=Tk", dict(capacity_factor=1000.0)),
    ("ragged T", dict(T=1001)),
    ("E=1", dict(E=1, k=1)),
    ("top1 C=0", dict(k=1, capacity_factor=0.0)),
    ("top1 ragged T", dict(k=1, T=777, capacity_factor=0.7)),
])
def test_edge_cases(cuda_ok, name, kw):
    base = dict(T=200, d_model=128, d_ff=256, E=8, k=2, capacity_factor=1.0, dtype="bf16",
                w_router_std=0.1, w_std=0.05, b_std=0.05, seed=77)
    base.update(kw)
    w = synth.Workload("edge", **base)
    r = layer_parity(w)
    if name in ("C=0", "top1 C=0"):
        assert np.array_equal(r["got"]["out"], synth.make_inputs(w)["x"])


@pytest.mark.parametrize("k,res,out32", [(1, False, False), (1, False, True), (1, True, True),
                                         (2, False, False)])
def test_residual_and_output_type_variants(cuda_ok, k, res, out32):
    w = synth.Workload("variants", T=333, d_model=128, d_ff=256, E=8, k=k, capacity_factor=0.8,
                       dtype="bf16", w_router_std=0.1, w_std=0.05, b_std=0.05, seed=79)
    r = layer_parity(w, add_input_residual=res, out_dtype=torch.float32 if out32 else None)
    dropped = (r["got"]["slot"] < 0).all(1)
    assert dropped.any()
    if not res:   # a token dropped by every choice has no residual: its output is zero
        assert np.all(r["got"]["out"][dropped] == 0)


def test_all_tokens_to_one_expert(cuda_ok):
    # a huge logit bias on expert 5: every first choice is 5, capacity keeps the first C tokens
    w = synth.Workload("collapse", T=300, d_model=64, d_ff=128, E=8, k=1, capacity_factor=2.0,
                       dtype="bf16", w_router_std=0.01, w_std=0.05, b_std=0.05, seed=78)
    inp = synth.make_inputs(w)
    inp["router_bias"] = np.zeros(8, dtype=np.float32)
    inp["router_bias"][5] = 50.0
    r = layer_parity(w, inp)
    g = r["got"]
    assert (g["expert_ids"][:, 0] == 5).all()
    assert g["expert_counts"][5] == 300 and (g["slot"][:75, 0] == np.arange(75)).all()
    assert (g["slot"][75:, 0] == -1).all()
    assert abs(g["lb_stats"][-1] - w.aux_alpha * 8) < 1e-4    # collapse: aux ~ alpha * E


def test_determinism_bitwise(cuda_ok):
    w = synth.WORKLOADS[4].with_(T=1024, d_model=512, d_ff=1024)
    d_inp = dev_inputs(synth.make_inputs(w))
    a = run_layer(w, d_inp)
    b = run_layer(w, d_inp)
    for n in ("out", "logits", "expert_ids", "gates", "slot", "expert_counts", "lb_stats"):
        assert np.array_equal(a[n], b[n]), n


def test_launch_count(cuda_ok):
    w = synth.WORKLOADS[3].with_(T=256, d_model=128, d_ff=256)
    got = run_layer(w, dev_inputs(synth.make_inputs(w)))
    # router 2 (prep: weight split + zeroed accumulators; tensor-core logits with softmax, top-k,
    # the statistics and the dispatch ranks in the epilogue), dispatch 2 (scan, scatter), the
    # expert and dense layers co-scheduled 2, the combine 1
    assert got["launches"] == 7
    w1 = synth.WORKLOADS[2].with_(T=256, d_model=128, d_ff=256)
    got = run_layer(w1, dev_inputs(synth.make_inputs(w1)))
    assert got["launches"] == 6      # top-1: the combine is fused into the experts' layer 2
    w2 = synth.WORKLOADS[4].with_(T=256, d_model=128, d_ff=256)
    got = run_layer(w2, dev_inputs(synth.make_inputs(w2)))
    assert got["launches"] == 7      # top-2: gather combine kernel


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_profiled_forward_matches_and_labels_stages(cuda_ok, cfg):
    from mixture_experts_layer_57_b200 import moe
    w = synth.WORKLOADS[cfg].with_(T=256, d_model=128, d_ff=256)
    d_inp = dev_inputs(synth.make_inputs(w))
    ref = run_layer(w, d_inp)
    dense = (d_inp["dense_w1"], d_inp["dense_b1"], d_inp["dense_w2"], d_inp["dense_b2"]) if w.dense else None
    args = moe.layer_args(d_inp["x"], d_inp["w_router"], d_inp["w1"], d_inp["b1"], d_inp["w2"],
                          d_inp["b2"], k=w.k, capacity_factor=w.capacity_factor,
                          router_bias=d_inp.get("router_bias"), dense=dense,
                          add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha)
    out = torch.empty(w.T, w.d_model, dtype=torch.bfloat16, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(12)]
    names = moe.moe_layer_forward_profiled(args, out, evs)
    torch.cuda.synchronize()
    want = {2: ["start", "router", "dispatch", "expert_gemm1", "expert_gemm2_combine"],
            3: ["start", "router", "dispatch", "experts_dense_gemm1", "experts_dense_gemm2",
                "combine"],
            4: ["start", "router", "dispatch", "expert_gemm1", "expert_gemm2", "combine"]}[cfg]
    assert names == want
    assert all(evs[i].elapsed_time(evs[i + 1]) >= 0 for i in range(len(names) - 1))
    from tests.helpers import to_host
    assert np.array_equal(to_host(out), ref["out"])
