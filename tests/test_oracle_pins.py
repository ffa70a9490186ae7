"""Pins of the CPU oracle against what the pages print and what mathematics fixes.

Each test checks one oracle function against a value the oracle did not produce:
a worked example printed on a page (fixtures under tests/golden/, each citing its
page and section), a textbook constant, or an independent library routine.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import golden


# ---------------------------------------------------------------- router softmax / top-k

def test_router_softmax_page_example():
    g = golden("router_softmax_example.json")
    x = np.array([g["x"]], dtype=np.float32)
    w = np.array(g["w_router"], dtype=np.float32)
    logits = oracle.router_logits(x, w)
    assert logits[0].tolist() == g["logits"]
    ids, gates, probs = oracle.route(logits, 1, want_probs=True)
    tol = g["print_precision"]
    assert np.allclose(np.exp(logits[0].astype(np.float64)), g["exp_logits_printed"], atol=tol)
    assert abs(np.exp(logits[0].astype(np.float64)).sum() - g["sum_exp_printed"]) < tol
    assert np.allclose(probs[0], g["probs_printed"], atol=tol)
    assert ids[0, 0] == g["top1_expert"]
    assert abs(gates[0, 0] - g["probs_printed"][1]) < tol


def test_top1_four_tokens_page_example():
    g = golden("top1_four_tokens.json")
    logits = np.array(g["logits"], dtype=np.float32)
    ids, gates, probs = oracle.route(logits, 1, want_probs=True)
    assert ids[:, 0].tolist() == g["top1_experts"]
    assert np.allclose(probs, g["probs_printed"], atol=g["print_tolerance"])
    # gates are the (unrenormalised) probability of the chosen expert
    for t in range(4):
        assert gates[t, 0] == np.float32(probs[t, ids[t, 0]])


def test_three_expert_table_page_example():
    g = golden("three_expert_top1.json")
    scores = np.array(g["scores"], dtype=np.float32)
    ids, _ = oracle.route(scores, 1)
    assert ids[:, 0].tolist() == g["top1_experts"]


def test_softmax_closed_form_two_experts():
    # For two experts p_0 = 1 / (1 + exp(l_1 - l_0)) (logistic function).
    rng = np.random.default_rng(0)
    l = rng.normal(size=(50, 2)).astype(np.float32)
    _, _, p = oracle.route(l, 1, want_probs=True)
    ref = 1.0 / (1.0 + np.exp(l[:, 1].astype(np.float64) - l[:, 0].astype(np.float64)))
    assert np.allclose(p[:, 0], ref, rtol=0, atol=1e-15)
    assert np.allclose(p.sum(1), 1.0, atol=1e-15)


def test_router_logits_against_library_matmul():
    # Non-square W_r (E != d) with a bias catches a transposed operand or a dropped bias.
    rng = np.random.default_rng(1)
    T, d, E = 7, 5, 3
    x = rng.normal(size=(T, d)).astype(np.float32)
    w = rng.normal(size=(E, d)).astype(np.float32)
    b = rng.normal(size=E).astype(np.float32)
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b.astype(np.float64)
    got = oracle.router_logits(x, w, b)
    assert np.array_equal(got, ref.astype(np.float32))


def test_router_logits_bf16_input_widening():
    rng = np.random.default_rng(2)
    T, d, E = 4, 9, 6
    xf = torch.randn(T, d).to(torch.bfloat16)
    xbits = xf.view(torch.int16).numpy().view(np.uint16).copy()
    w = rng.normal(size=(E, d)).astype(np.float32)
    ref = xf.double().numpy() @ w.astype(np.float64).T
    got = oracle.router_logits(xbits, w)
    assert np.array_equal(got, ref.astype(np.float32))


def test_topk_ties_go_to_lowest_index_and_order():
    logits = np.array([[1.0, 1.0, 0.0, 1.0], [0.0, 2.0, 2.0, -1.0], [3.0, 1.0, 2.0, 0.0]], dtype=np.float32)
    ids, _ = oracle.route(logits, 1)
    assert ids[:, 0].tolist() == [0, 1, 0]
    ids, _ = oracle.route(logits, 3)
    assert ids.tolist() == [[0, 1, 3], [1, 2, 0], [0, 2, 1]]


def test_topk_equals_brute_force_sort():
    rng = np.random.default_rng(3)
    l = rng.integers(-3, 4, size=(200, 7)).astype(np.float32)  # many ties
    for k in (1, 2, 4, 7):
        ids, gates, p = oracle.route(l, k, want_probs=True)
        for t in range(l.shape[0]):
            order = sorted(range(7), key=lambda e: (-l[t, e], e))[:k]
            assert ids[t].tolist() == order
            assert gates[t].tolist() == [np.float32(p[t, e]) for e in order]


# ---------------------------------------------------------------- capacity and slots

def test_capacity_page_example():
    g = golden("capacity_overflow.json")
    C = oracle.capacity(g["tokens_per_batch"], g["num_experts"], 1, g["capacity_factor"])
    assert C == g["capacity"]
    ids = np.array(g["top1_experts"], dtype=np.int32)[:, None]
    slot, counts = oracle.assign_slots(ids, g["num_experts"], C)
    assert counts.tolist() == g["demand"]
    kept = [int(((ids[:, 0] == e) & (slot[:, 0] >= 0)).sum()) for e in range(2)]
    assert kept == g["kept"]
    dropped = [t for t in range(4) if slot[t, 0] < 0]
    assert dropped == g["first_come_reading_dropped"]
    assert slot[2, 0] == 0  # E1 keeps t2


@pytest.mark.parametrize("T,E,k,cf,C", [
    (16384, 128, 1, 1.0, 128), (8192, 8, 2, 1.25, 2560), (32, 128, 1, 2.0, 1),
    (64, 4, 1, 1.0, 16), (10, 3, 1, 1.0, 4), (1, 8, 1, 1.0, 1), (100, 7, 2, 0.0, 0),
    (5, 2, 2, 1e9, 5000000000),
])
def test_capacity_formula(T, E, k, cf, C):
    # ceil(k * T / E * cf), values worked by hand
    assert oracle.capacity(T, E, k, cf) == C


@pytest.mark.parametrize("T,E,k,cf,C", [
    (100, 10, 1, 1.1, 11), (1000, 100, 1, 1.1, 11), (30, 10, 1, 1.1, 4), (20, 10, 1, 1.15, 3),
    (700, 10, 1, 0.7, 49), (300, 100, 1, 0.7, 3), (60, 20, 1, 1.1, 4), (8, 8, 1, 1.001, 2),
])
def test_capacity_decimal_factor(T, E, k, cf, C):
    # a decimal factor held in binary (1.1 is stored slightly above 1.1) still gives the capacity
    # of the decimal number: 100 tokens / 10 experts x 1.1 = 11 exactly, so C = 11, not 12
    assert oracle.capacity(T, E, k, cf) == C


def test_capacity_matches_exact_decimal_arithmetic():
    # ceil(k T / E x cf) in exact rational arithmetic on the decimal factor, over a grid of shapes
    from fractions import Fraction
    rng = np.random.default_rng(11)
    factors = ["1.0", "1.1", "1.2", "1.25", "1.5", "2.0", "0.5", "0.7", "1.3", "0.9", "1.05", "0.3",
               "0.01", "3.3", "1.001", "1.123456"]
    cases = [(T, E, k) for T in range(1, 130, 3) for E in (1, 2, 3, 7, 8, 10, 16, 64, 128)
             for k in (1, 2)]
    cases += [(int(rng.integers(1, 2 ** 30)), int(rng.integers(1, 1025)), int(rng.integers(1, 9)))
              for _ in range(300)]
    for T, E, k in cases:
        for cf in factors:
            exact = -((-Fraction(k * T, E) * Fraction(cf)).__floor__())
            assert oracle.capacity(T, E, k, float(cf)) == exact, (T, E, k, cf)


# ---------------------------------------------------------------- number formats

@pytest.mark.parametrize("v,bits", [
    (1.0, 0x3F80), (1.0 + 2.0 ** -8, 0x3F80), (1.0 + 3 * 2.0 ** -8, 0x3F82),
    (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81), (-1.0 - 3 * 2.0 ** -8, 0xBF82), (3.0, 0x4040),
    (0.0, 0x0000), (-0.0, 0x8000), (2.0 ** -133, 0x0001), (2.0 ** -134, 0x0000),
    (1.5 * 2.0 ** -133, 0x0002), (3.3895313892515355e38, 0x7F7F), (1e39, 0x7F80),
    (-1e39, 0xFF80), (2.0 ** -126, 0x0080),
])
def test_round_bf16_worked_values(v, bits):
    assert int(oracle.round_bf16(v)) == bits


def test_round_bf16_matches_library_on_float_inputs():
    # For inputs that are exact fp32 values, direct rounding equals the library's
    # fp32 -> bf16 round-to-nearest-even conversion.
    g = torch.Generator().manual_seed(4)
    f = torch.cat([torch.randn(4000, generator=g) * s for s in (1e-3, 1.0, 1e3)])
    f = torch.cat([f, (torch.arange(-300, 300) * 2.0 ** -9 + 1.0)])
    ref = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_bf16(f.double().numpy())
    assert np.array_equal(got, ref)


def test_bf16_widening_exact():
    bits = np.array([0x3F80, 0xBF82, 0x0001, 0x7F7F, 0x4049], dtype=np.uint16)
    want = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.bf16_to_float(bits), want)


@pytest.mark.parametrize("z,want", [
    # GeLU(z) = z * Phi(z); Phi from the standard normal table
    (0.0, 0.0), (1.0, 0.8413447460685429), (-1.0, -0.15865525393145707),
    (2.0, 2 * 0.9772498680518208), (-2.0, -2 * 0.022750131948179195),
    (0.5, 0.5 * 0.6914624612740131), (3.0, 3 * 0.9986501019683699),
])
def test_gelu_standard_normal_table(z, want):
    assert abs(oracle.gelu(z) - want) < 1e-15 * max(1.0, abs(want))


# ---------------------------------------------------------------- combine / PR-MoE

def test_prmoe_residual_page_example():
    g = golden("prmoe_residual.json")
    dense = np.array([g["h_fixed"]], dtype=np.float32)
    y = np.array([[g["r_A"]]], dtype=np.float32)   # [T=1, k=1, d=2]
    gates = np.array([[g["gate"]]], dtype=np.float32)
    slot = np.array([[0]], dtype=np.int32)
    out = oracle.combine(gates, slot, y, dense=dense)
    assert np.allclose(out[0], g["output"], atol=1e-6)


def test_combine_drops_overflowed_pairs_and_sums_choices():
    y = np.array([[[1.0, 2.0], [10.0, 20.0]], [[3.0, 4.0], [30.0, 40.0]]], dtype=np.float32)
    gates = np.array([[0.5, 0.25], [0.75, 0.125]], dtype=np.float32)
    slot = np.array([[0, -1], [3, 7]], dtype=np.int32)
    res = np.array([[100.0, 200.0], [300.0, 400.0]], dtype=np.float32)
    out = oracle.combine(gates, slot, y, residual=res)
    assert out.tolist() == [[100.5, 201.0], [300 + 2.25 + 3.75, 400 + 3.0 + 5.0]]


# ---------------------------------------------------------------- load-balance statistics

def test_lb_uniform_routing_gives_alpha():
    g = golden("load_balance_loss.json")
    E = 8
    # each token has equal logits -> p = 1/E; top-1 choices cycle over experts -> f = 1/E
    T = 8 * E
    logits = np.zeros((T, E), dtype=np.float32)
    ids = np.array([[t % E] for t in range(T)], dtype=np.int32)
    f, Q, aux = oracle.lb_stats(logits, ids, alpha=0.37)
    assert np.allclose(f, 1 / E) and np.allclose(Q, 1 / E)
    assert abs(aux / 0.37 - g["uniform_loss_over_alpha"]) < 1e-12


def test_lb_collapse_gives_alpha_times_E():
    E, T = 16, 50
    logits = np.zeros((T, E), dtype=np.float32)
    logits[:, 3] = 60.0
    ids, _ = oracle.route(logits, 1)
    f, Q, aux = oracle.lb_stats(logits, ids, alpha=0.5)
    assert f[3] == 1.0 and abs(Q[3] - 1.0) < 1e-12
    assert abs(aux - 0.5 * E) < 1e-9


def test_lb_hand_worked_case():
    # logits [[0,0],[ln 3,0]]: p = [.5,.5], [.75,.25]; top-1 both expert 0 (tie -> lowest).
    logits = np.array([[0.0, 0.0], [math.log(3.0), 0.0]], dtype=np.float32)
    ids, _ = oracle.route(logits, 1)
    assert ids[:, 0].tolist() == [0, 0]
    f, Q, aux = oracle.lb_stats(logits, ids, alpha=1.0)
    p1 = 1.0 / (1.0 + math.exp(-float(np.float32(math.log(3.0)))))
    assert f.tolist() == [1.0, 0.0]
    assert abs(Q[0] - (0.5 + p1) / 2) < 1e-15
    assert abs(aux - 2 * (0.5 + p1) / 2) < 1e-15


def test_lb_top2_uses_first_choice():
    logits = np.array([[3.0, 2.0, 1.0], [1.0, 3.0, 2.0]], dtype=np.float32)
    ids, _ = oracle.route(logits, 2)
    f, Q, _ = oracle.lb_stats(logits, ids, alpha=1.0)
    assert f.tolist() == [0.5, 0.5, 0.0]
    assert abs(Q.sum() - 1.0) < 1e-15
