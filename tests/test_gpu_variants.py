"""GPU parity of the routing variants against the oracle: renormalised top-k gates, the router
z-loss and the CoV^2 of Importance and Load (moe_router_topk_ex), overflow by priority
(moe_dispatch_priority), and both inside moe_layer_forward.

Ids, slots, counts and offsets are bit-exact (the oracle decides on the GPU's fp32 logits and, for
the priority order, on the GPU's fp32 router probabilities, which rank the pairs before and
after any renormalisation of the gates); renormalised gates match to 2e-6 relative; z-loss
and CoV^2 of Importance to 1e-5 relative (fp32 per-token terms, fixed-point sums); CoV^2 of Load
to 1e-6 (integer counts).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import check_out, dev_inputs, run_layer, to_dev, to_host
from tests.test_gpu_dispatch import make_ids

pytestmark = pytest.mark.gpu


def check_losses(got, ref, what=""):
    z, ci, cl = ref
    assert abs(got[0] - z) <= 1e-5 * abs(z) + 1e-6, (what, got[0], z)
    assert abs(got[1] - ci) <= 1e-5 * abs(ci) + 1e-7, (what, got[1], ci)
    assert abs(got[2] - cl) <= 1e-6 * abs(cl) + 1e-9, (what, got[2], cl)


def router_ex(w: synth.Workload, inp: dict, renormalize: bool):
    r = moe.moe_router_topk(to_dev(inp["x"]), to_dev(inp["w_router"]), w.k,
                            router_bias=to_dev(inp.get("router_bias")), aux_alpha=w.aux_alpha,
                            renormalize=renormalize, router_losses=True, probs=True)
    assert moe.moe_get_device_error(r["ws"]) == 0
    return {n: to_host(r[n]) for n in ("logits", "expert_ids", "gates", "lb_stats", "router_losses",
                                       "probs")}


def router_only(w):
    return {k: v for k, v in synth.make_inputs(w.with_(d_ff=8)).items()
            if not k.startswith(("w1", "w2", "b1", "b2", "dense"))}


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("renormalize", [False, True])
def test_router_variants_workloads(cuda_ok, cfg, renormalize):
    w = synth.WORKLOADS[cfg]
    inp = router_only(w)
    got = router_ex(w, inp, renormalize)
    ids, gates = oracle.route(got["logits"], w.k)
    assert np.array_equal(got["expert_ids"], ids)
    # the probabilities output is the softmax p of each choice, renormalised or not
    np.testing.assert_allclose(got["probs"], gates, rtol=2e-6, atol=1e-12)
    if renormalize:
        gates = oracle.renormalize_gates(gates)
        np.testing.assert_allclose(got["gates"].sum(1), 1.0, rtol=1e-5)
    else:
        assert np.array_equal(got["probs"], got["gates"])
    np.testing.assert_allclose(got["gates"], gates, rtol=2e-6, atol=1e-12)
    # the losses from the GPU's own logits and gates
    check_losses(got["router_losses"], oracle.router_losses(got["logits"], got["expert_ids"],
                                                            got["gates"]), w.name)
    # lb_stats keep the softmax p (not the renormalised gates)
    f, Q, _ = oracle.lb_stats(got["logits"], ids, w.aux_alpha)
    np.testing.assert_allclose(got["lb_stats"][w.E:2 * w.E], Q, rtol=1e-5, atol=1e-9)


@pytest.mark.parametrize("T,d,E,k,dt", [
    (1, 64, 4, 1, "bf16"), (300, 40, 37, 3, "f32"), (257, 1032, 1024, 8, "bf16"),
    (130, 8, 1, 1, "bf16"), (64, 16, 8, 8, "f32"), (5000, 200, 200, 2, "bf16"),
])
def test_router_variants_edge_shapes(cuda_ok, T, d, E, k, dt):
    w = synth.Workload("t", T=T, d_model=d, d_ff=8, E=E, k=k, capacity_factor=1.0, dtype=dt,
                       w_router_std=0.3, router_bias="normal", router_bias_std=0.5, seed=T + E)
    inp = synth.make_inputs(w)
    got = router_ex(w, inp, True)
    ids, gates = oracle.route(got["logits"], k)
    assert np.array_equal(got["expert_ids"], ids)
    np.testing.assert_allclose(got["gates"], oracle.renormalize_gates(gates), rtol=2e-6, atol=1e-12)
    check_losses(got["router_losses"], oracle.router_losses(got["logits"], ids, got["gates"]))
    if E == 1:
        # one expert: every gate renormalises to 1, Importance = Load = T, both CoV^2 = 0
        assert (got["gates"] == 1.0).all()
        assert got["router_losses"][1] == 0.0 and got["router_losses"][2] == 0.0


def test_router_z_loss_closed_form(cuda_ok):
    # equal logits: log sum exp = l + log E for every token, so z-loss = (l + log E)^2
    T, d, E = 200, 64, 16
    x = np.zeros((T, d), dtype=np.float32)
    w_r = np.zeros((E, d), dtype=np.float32)
    b = np.full(E, 0.75, dtype=np.float32)
    r = moe.moe_router_topk(to_dev(x), to_dev(w_r), 2, router_bias=to_dev(b), router_losses=True)
    z = float(to_host(r["router_losses"])[0])
    assert abs(z - (0.75 + np.log(E)) ** 2) <= 1e-5 * z


def check_priority_dispatch(x_host, ids, probs, E, C):
    T, k = ids.shape
    r = moe.moe_dispatch(to_dev(x_host), to_dev(ids), E, C, priority_probs=to_dev(probs))
    assert moe.moe_get_device_error(r["ws"]) == 0
    slot, counts = oracle.assign_slots_priority(ids, probs, E, C)
    assert np.array_equal(to_host(r["slot"]), slot)
    assert np.array_equal(to_host(r["expert_counts"]), counts)
    off = np.concatenate([[0], np.cumsum(np.minimum(counts, C))]).astype(np.int32)
    assert np.array_equal(to_host(r["expert_offsets"]), off)
    total = int(off[-1])
    rt = to_host(r["row_token"])[:total]
    t_idx, j_idx = np.nonzero(slot >= 0)
    rows = off[ids[t_idx, j_idx]] + slot[t_idx, j_idx]
    assert np.array_equal(np.sort(rows), np.arange(total))
    assert np.array_equal(rt[rows], t_idx)
    assert np.array_equal(to_host(r["x_packed"])[:total], x_host[rt])
    return slot


@pytest.mark.parametrize("T,E,k,kind,cf,levels", [
    (4096, 128, 1, "zipf", 1.0, 0), (8192, 8, 2, "zipf", 1.25, 0), (1000, 37, 3, "uniform", 1.0, 4),
    (777, 1024, 8, "uniform", 1.0, 0), (3000, 16, 4, "one_expert", 1.0, 3), (1, 4, 1, "uniform", 1.0, 0),
    (300, 5, 5, "uniform", 100.0, 0), (300, 6, 2, "uniform", 0.0, 0), (2500, 2, 1, "one_expert", 0.5, 2),
])
def test_priority_dispatch_bit_exact(cuda_ok, T, E, k, kind, cf, levels):
    rng = np.random.default_rng(T * 11 + E)
    ids = make_ids(rng, T, E, k, kind)
    gates = rng.random((T, k)).astype(np.float32)
    if levels:
        gates = (np.floor(gates * levels) / levels).astype(np.float32)  # many equal gates: ties
    C = moe.moe_capacity(T, E, k, cf)
    x = rng.integers(0, 1 << 16, size=(T, 72), dtype=np.uint16)
    x[(x & 0x7f80) == 0x7f80] = 0
    slot = check_priority_dispatch(x, ids, gates, E, C)
    if kind == "one_expert" and C < T:
        # the hot expert keeps exactly its C largest gates
        hot = E // 2
        t_hot, j_hot = np.nonzero(ids == hot)
        kept = slot[t_hot, j_hot] >= 0
        assert kept.sum() == C
        assert gates[t_hot, j_hot][kept].min() >= gates[t_hot, j_hot][~kept].max()


def test_priority_matches_capacity_example(cuda_ok):
    # comparison article, "Top-1 routing decision" and "Expert Capacity Overflow" examples: the
    # printed logits routed on the GPU (x = logits, W_r = identity), then capacity 2 by priority:
    # expert 0 keeps tokens 3 and 0 (largest probabilities) and drops token 1
    from tests.conftest import golden
    g = golden("capacity_overflow.json")
    t = golden("top1_four_tokens.json")
    x = np.array(t["logits"], dtype=np.float32)
    r = moe.moe_router_topk(to_dev(x), to_dev(np.eye(2, dtype=np.float32)), 1)
    ids, gates = to_host(r["expert_ids"]), to_host(r["gates"])
    assert ids[:, 0].tolist() == t["top1_experts"]
    C = moe.moe_capacity(g["tokens_per_batch"], g["num_experts"], 1, g["capacity_factor"])
    assert C == g["capacity"]
    feat = np.arange(4 * 8, dtype=np.float32).reshape(4, 8)
    slot = check_priority_dispatch(feat, ids, gates, 2, C)
    assert [tk for tk in (3, 0, 1) if slot[tk, 0] >= 0] == g["page_priority_order_kept_E0"]
    assert [tk for tk in range(4) if slot[tk, 0] < 0] == g["page_priority_order_dropped"]


def assert_priority_active(got, E, C):
    """Every expert keeps the pairs of its C largest router probabilities (before any
    renormalisation), and at least one expert keeps a different set than first-come would."""
    ids, slot, p = got["expert_ids"], got["slot"], got["topk_probs"]
    fc, _ = oracle.assign_slots(ids, E, C)
    differs = False
    for e in np.unique(ids):
        t_e, j_e = np.nonzero(ids == e)
        kept = slot[t_e, j_e] >= 0
        if kept.all() or not kept.any():
            continue
        assert p[t_e, j_e][kept].min() >= p[t_e, j_e][~kept].max(), e
        differs |= not np.array_equal(kept, fc[t_e, j_e] >= 0)
    assert differs, "priority kept the same pairs as first-come"


def layer_variant_parity(w: synth.Workload, overflow_priority=True, renormalize=True):
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    got = run_layer(w, d_inp, overflow_priority=overflow_priority, renormalize=renormalize,
                    want_losses=True)
    assert got["device_error"] == 0
    bf16 = w.dtype == "bf16"
    ref = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                               add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha,
                               logits_in=got["logits"], out_bf16=bf16,
                               overflow_priority=overflow_priority, renormalize=renormalize,
                               probs_in=got["topk_probs"])
    assert np.array_equal(got["expert_ids"], ref["ids"])
    ids, gates = oracle.route(got["logits"], w.k)
    np.testing.assert_allclose(got["topk_probs"], gates, rtol=2e-6, atol=1e-12)
    if renormalize:
        gates = oracle.renormalize_gates(gates)
    np.testing.assert_allclose(got["gates"], gates, rtol=2e-6, atol=1e-12)
    assert np.array_equal(got["slot"], ref["slot"])
    assert np.array_equal(got["expert_counts"], ref["counts"])
    off = np.concatenate([[0], np.cumsum(np.minimum(ref["counts"], ref["C"]))])
    assert np.array_equal(got["expert_offsets"], off.astype(np.int32))
    check_losses(got["router_losses"], (ref["z_loss"], ref["cov2_importance"], ref["cov2_load"]),
                 w.name)
    check_out(got["out"], ref["out_exact"], bf16, bf16, what=w.name)
    return got, ref


def test_layer_priority_renorm_tiny_fp32(cuda_ok):
    w = synth.WORKLOADS[1]
    got, ref = layer_variant_parity(w)
    assert (got["slot"] < 0).any()
    assert (got["gates"] == 1.0).all()  # top-1 gates renormalise to 1, the ranking does not
    assert_priority_active(got, w.E, ref["C"])


def test_layer_priority_renorm_page_example(cuda_ok):
    # comparison article, "Expert Capacity Overflow": capacity 2 for expert 0's three tokens; by
    # router probability t3 (0.859) and t0 (0.817) keep it and t1 (0.669) overflows. The layer
    # routes the printed logits (x = logits, W_r = identity) with renormalised top-1 gates, which
    # are all 1.0; the ranking still follows the probabilities, unlike first-come (drops t3).
    from tests.conftest import golden
    g = golden("capacity_overflow.json")
    t = golden("top1_four_tokens.json")
    w = synth.Workload("page", T=4, d_model=2, d_ff=8, E=2, k=1, capacity_factor=1.0, dtype="f32",
                       w_router_std=1.0, w_std=0.3, b_std=0.1, seed=3)
    inp = synth.make_inputs(w)
    inp["x"] = np.array(t["logits"], dtype=np.float32)
    inp["w_router"] = np.eye(2, dtype=np.float32)
    for renorm in (True, False):
        got = run_layer(w, dev_inputs(inp), overflow_priority=True, renormalize=renorm)
        assert got["device_error"] == 0
        slot = got["slot"][:, 0]
        assert [tk for tk in (3, 0, 1) if slot[tk] >= 0] == g["page_priority_order_kept_E0"]
        assert [tk for tk in range(4) if slot[tk] < 0] == g["page_priority_order_dropped"]
        fc = run_layer(w, dev_inputs(inp), overflow_priority=False, renormalize=renorm)
        assert [tk for tk in range(4) if fc["slot"][tk, 0] < 0] == g["first_come_reading_dropped"]
        assert not np.array_equal(got["slot"], fc["slot"])
        if renorm:
            assert (got["gates"] == 1.0).all()
        ref = oracle.layer_forward(inp, 4, 2, 8, 2, 1, 1.0, logits_in=got["logits"],
                                   overflow_priority=True, renormalize=renorm,
                                   probs_in=got["topk_probs"])
        assert np.array_equal(got["slot"], ref["slot"])
        check_out(got["out"], ref["out_exact"], False, False, what="page example")


@pytest.mark.parametrize("cfg,T,policy", [
    (2, 1024, (True, True)), (2, 1024, (True, False)), (2, 1024, (False, True)),
    (3, 512, (True, True)), (4, 512, (True, True)), (5, 32, (True, True)),
])
def test_layer_variants_reduced(cuda_ok, cfg, T, policy):
    w = synth.WORKLOADS[cfg]
    shrink = dict(T=T)
    if cfg in (2, 3):
        shrink.update(d_model=512, d_ff=1024)
    if cfg == 4:
        shrink.update(d_model=1024, d_ff=2048)
    w = w.with_(**shrink)
    got, ref = layer_variant_parity(w, *policy)
    if policy[0]:
        # the priority path changes which pairs are kept, not how many
        slot_fc, _ = oracle.assign_slots(got["expert_ids"], w.E, ref["C"])
        assert (slot_fc >= 0).sum() == (got["slot"] >= 0).sum()
        assert_priority_active(got, w.E, ref["C"])


def test_layer_priority_all_tokens_to_one_expert(cuda_ok):
    # a router bias that sends every token to expert 3: the kept tokens are those of largest gate
    w = synth.WORKLOADS[2].with_(T=600, d_model=256, d_ff=512)
    inp = synth.make_inputs(w)
    inp["router_bias"] = np.zeros(w.E, dtype=np.float32)
    inp["router_bias"][3] = 8.0
    got = run_layer(w, dev_inputs(inp), overflow_priority=True, want_losses=True)
    C = moe.moe_capacity(w.T, w.E, w.k, w.capacity_factor)
    assert (got["expert_ids"][:, 0] == 3).all()
    kept = got["slot"][:, 0] >= 0
    assert kept.sum() == C
    assert got["gates"][kept, 0].min() >= got["gates"][~kept, 0].max()
    assert abs(got["router_losses"][2] - (w.E - 1)) <= 1e-5 * (w.E - 1)  # CoV^2 of one-hot load
