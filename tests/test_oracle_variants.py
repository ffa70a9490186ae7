"""Pins of the oracle's routing variants and extra router statistics (the "next" items of the
routing: probability-priority overflow, renormalised gates, z-loss, Importance/Load CoV^2)."""
import itertools
import math

import numpy as np
import pytest

import oracle
from tests.conftest import golden


def test_z_loss_page_example():
    g = golden("router_z_loss.json")
    tol = g["print_tolerance"]
    for tok in g["tokens"]:
        l = np.array([tok["logits"]], dtype=np.float32)
        ids = np.zeros((1, 1), dtype=np.int32)
        gates = np.ones((1, 1), dtype=np.float32)
        z, _, _ = oracle.router_losses(l, ids, gates)
        lz = math.sqrt(z)
        assert abs(math.exp(lz) - tok["Z"]) < tol
        assert abs(lz - tok["logZ"]) < tol
        if "L_z" in tok:
            assert abs(z - tok["L_z"]) < tol


def test_z_loss_is_mean_over_tokens_and_shift_behaviour():
    # closed forms: L_z of E equal logits c is (c + ln E)^2; the loss averages over tokens
    l = np.array([[0.0] * 4, [1.0] * 4], dtype=np.float32)
    z, _, _ = oracle.router_losses(l, np.zeros((2, 1), np.int32), np.ones((2, 1), np.float32))
    assert abs(z - ((math.log(4)) ** 2 + (1 + math.log(4)) ** 2) / 2) < 1e-12


def test_cov2_hand_worked():
    # Load = [3, 1, 0]: mean 4/3, population variance 42/27, CoV^2 = 0.875
    ids = np.array([[0], [0], [1], [0]], dtype=np.int32)
    gates = np.array([[0.5], [0.25], [1.0], [0.25]], dtype=np.float32)
    l = np.zeros((4, 3), dtype=np.float32)
    _, ci, cl = oracle.router_losses(l, ids, gates)
    assert abs(cl - 0.875) < 1e-12
    # Importance = [1.0, 1.0, 0.0]: mean 2/3, variance 2/9, CoV^2 = 0.5
    assert abs(ci - 0.5) < 1e-12
    # uniform load: CoV^2 = 0
    _, _, cl2 = oracle.router_losses(np.zeros((3, 3), np.float32), np.array([[0], [1], [2]], np.int32),
                                     np.ones((3, 1), np.float32))
    assert cl2 == 0.0


def test_priority_overflow_page_example():
    g = golden("capacity_overflow.json")
    t = golden("top1_four_tokens.json")
    logits = np.array(t["logits"], dtype=np.float32)
    ids, gates = oracle.route(logits, 1)
    slot, counts = oracle.assign_slots_priority(ids, gates, 2, g["capacity"])
    kept_e0 = [tk for tk in (3, 0, 1) if slot[tk, 0] >= 0]
    assert kept_e0 == g["page_priority_order_kept_E0"]
    assert [tk for tk in range(4) if slot[tk, 0] < 0] == g["page_priority_order_dropped"]
    assert slot[3, 0] == 0 and slot[0, 0] == 1 and slot[2, 0] == 0
    assert counts.tolist() == g["demand"]


def test_priority_overflow_page_example_with_renormalised_gates():
    # the article ranks E0's tokens by router probability; renormalising a top-1 gate makes it
    # 1.0 for every token, but the ranking still follows the probability: keep t3 and t0, drop t1
    import synth
    g = golden("capacity_overflow.json")
    t = golden("top1_four_tokens.json")
    logits = np.array(t["logits"], dtype=np.float32)
    w = synth.Workload("page", T=4, d_model=8, d_ff=8, E=2, k=1, capacity_factor=1.0, dtype="f32",
                       w_router_std=1.0, w_std=0.3, b_std=0.1, seed=3)
    inp = synth.make_inputs(w)
    for renorm in (False, True):
        r = oracle.layer_forward(inp, 4, 8, 8, 2, 1, 1.0, logits_in=logits, overflow_priority=True,
                                 renormalize=renorm)
        assert [tk for tk in (3, 0, 1) if r["slot"][tk, 0] >= 0] == g["page_priority_order_kept_E0"]
        assert [tk for tk in range(4) if r["slot"][tk, 0] < 0] == g["page_priority_order_dropped"]
        assert r["slot"][3, 0] == 0 and r["slot"][0, 0] == 1 and r["slot"][2, 0] == 0
        if renorm:
            assert r["gates"].ravel().tolist() == [1.0, 1.0, 1.0, 1.0]


def test_priority_ranks_by_probability_not_renormalised_gate():
    # token 0 picks E0 (p 0.5) then E1 (p 0.4): renormalised E1 gate 0.4/0.9 = 0.444;
    # token 1 picks E1 (p 0.35) then E2 (p 0.30): renormalised E1 gate 0.35/0.65 = 0.538.
    # E1 has one place: by router probability token 0 (0.4 > 0.35) keeps it, although token 1's
    # renormalised gate is the larger one.
    import synth
    p = np.array([[0.5, 0.4, 0.05, 0.05], [0.29, 0.35, 0.30, 0.06]])
    logits = np.log(p).astype(np.float32)
    w = synth.Workload("rank", T=2, d_model=8, d_ff=8, E=4, k=2, capacity_factor=0.5, dtype="f32",
                       w_router_std=1.0, w_std=0.3, b_std=0.1, seed=4)
    inp = synth.make_inputs(w)
    r = oracle.layer_forward(inp, 2, 8, 8, 4, 2, 0.5, logits_in=logits, overflow_priority=True,
                             renormalize=True)
    assert r["C"] == 1
    assert r["ids"].tolist() == [[0, 1], [1, 2]]
    assert r["gates"][1, 0] > r["gates"][0, 1]          # renormalised: token 1's E1 gate is larger
    assert r["slot"][0, 1] == 0 and r["slot"][1, 0] == -1  # but token 0 keeps E1's place
    raw_ids, raw = oracle.route(logits, 2)
    s2, _ = oracle.assign_slots_priority(raw_ids, raw, 4, 1)
    assert np.array_equal(r["slot"], s2)


def priority_brute(ids, gates, E, C):
    T, k = ids.shape
    slot = np.full((T, k), -1, dtype=np.int32)
    for e in range(E):
        members = [p for p in range(T * k) if ids.flat[p] == e]
        members.sort(key=lambda p: (-float(gates.flat[p]), p))
        for r, p in enumerate(members):
            if r < C:
                slot.flat[p] = r
    return slot


@pytest.mark.parametrize("seed", range(4))
def test_priority_overflow_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    T, E, k = 120, 5, 2
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    gates = (rng.integers(0, 6, size=(T, k)) / 8.0).astype(np.float32)  # many equal gates
    for C in (0, 1, 9, 30, 1000):
        slot, counts = oracle.assign_slots_priority(ids, gates, E, C)
        assert np.array_equal(slot, priority_brute(ids, gates, E, C))
        assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))


def test_priority_equals_first_come_when_gates_equal():
    rng = np.random.default_rng(7)
    ids = rng.integers(0, 4, size=(50, 1)).astype(np.int32)
    gates = np.full((50, 1), 0.5, dtype=np.float32)
    a, _ = oracle.assign_slots_priority(ids, gates, 4, 6)
    b, _ = oracle.assign_slots(ids, 4, 6)
    assert np.array_equal(a, b)


def test_renormalized_gates():
    g = oracle.renormalize_gates(np.array([[0.5, 0.3], [0.2, 0.2], [0.7, 0.1]], dtype=np.float32))
    assert np.allclose(g, [[0.625, 0.375], [0.5, 0.5], [0.875, 0.125]], atol=1e-7)
    one = oracle.renormalize_gates(np.array([[0.3], [0.9]], dtype=np.float32))
    assert one.tolist() == [[1.0], [1.0]]
    # k = E: the full softmax already sums to one
    l = np.random.default_rng(1).normal(size=(6, 4)).astype(np.float32)
    _, gates = oracle.route(l, 4)
    assert np.allclose(oracle.renormalize_gates(gates), gates, rtol=1e-6)


def test_layer_with_variants_matches_composition():
    import synth
    w = synth.Workload("t", T=40, d_model=8, d_ff=12, E=4, k=2, capacity_factor=0.5, dtype="f32",
                       w_router_std=0.8, w_std=0.3, b_std=0.1, seed=21)
    inp = synth.make_inputs(w)
    r = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                             overflow_priority=True, renormalize=True)
    ids, probs = oracle.route(r["logits"], 2)
    gates = oracle.renormalize_gates(probs)
    assert np.array_equal(r["gates"], gates)
    slot, _ = oracle.assign_slots_priority(ids, probs, 4, r["C"])
    assert np.array_equal(r["slot"], slot)
    z, ci, cl = oracle.router_losses(r["logits"], ids, gates)
    assert (r["z_loss"], r["cov2_importance"], r["cov2_load"]) == (z, ci, cl)
    # outputs: x + sum over kept choices of gate * FFN_e(x)
    for t in (0, 7, 39):
        ref = inp["x"][t].astype(np.float64).copy()
        for j in range(2):
            if slot[t, j] >= 0:
                e = ids[t, j]
                y = oracle.ffn(inp["x"][t], inp["w1"][e], inp["b1"][e], inp["w2"][e], inp["b2"][e])
                ref += float(gates[t, j]) * y.astype(np.float64)
        assert np.allclose(r["out_exact"][t], ref, atol=1e-9)
