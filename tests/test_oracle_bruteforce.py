"""Pins of the CPU oracle by independent formulations and special cases.

* Dispatch: the slot counter is checked against the one-hot dispatch-mask
  formulation [T, E, C] that the fused gating kernel of the DeepSpeed-MoE notes
  (§4.4) replaces, and by exhaustive enumeration of all routings on tiny inputs.
* FFN: with one expert and room for every token the layer is a textbook dense
  MLP; computed here with numpy matrix products and scipy's erf.
* Identities: k = E with unlimited capacity is the dense softmax mixture
  sum_e p_e E_e(x); capacity 0 leaves only the residual.
"""
import itertools

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth


def mask_formulation(ids: np.ndarray, E: int, C: int):
    """Dispatch mask [T, E, C] built by sorting (expert, pair index) — no running counter."""
    T, k = ids.shape
    pairs = [(int(ids[t, j]), t * k + j) for t in range(T) for j in range(k)]
    order = sorted(pairs)
    mask = np.zeros((T, E, max(C, 0)), dtype=np.int8)
    slot = np.full((T, k), -1, dtype=np.int32)
    pos_in_expert = {}
    for e, p in order:
        c = pos_in_expert.get(e, 0)
        pos_in_expert[e] = c + 1
        t, j = divmod(p, k)
        if c < C:
            mask[t, e, c] = 1
            slot[t, j] = c
    demand = np.array([pos_in_expert.get(e, 0) for e in range(E)], dtype=np.int32)
    return mask, slot, demand


@pytest.mark.parametrize("seed", range(6))
def test_slots_equal_mask_formulation_random(seed):
    rng = np.random.default_rng(seed)
    T, E, k = 300, 5, 2
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    for C in (0, 1, 7, 60, 120, 1000):
        slot, counts = oracle.assign_slots(ids, E, C)
        mask, slot_ref, demand = mask_formulation(ids, E, C)
        assert np.array_equal(slot, slot_ref)
        assert np.array_equal(counts, demand)
        # the mask is a partial permutation: each kept pair owns exactly one cell
        assert mask.sum() == (slot >= 0).sum() == np.minimum(demand, C).sum()


def test_slots_exhaustive_tiny():
    # every top-1 routing of 6 tokens over 3 experts, and every top-2 routing of 4
    # tokens over 3 experts, at every capacity from 0 to the token count
    cases = [(6, 3, 1, list(itertools.product(range(3), repeat=6)))]
    choices2 = [c for c in itertools.permutations(range(3), 2)]
    cases.append((4, 3, 2, list(itertools.product(choices2, repeat=4))))
    n = 0
    for T, E, k, routings in cases:
        for r in routings:
            ids = np.array(r, dtype=np.int32).reshape(T, k)
            for C in range(0, T * k + 1):
                slot, counts = oracle.assign_slots(ids, E, C)
                _, slot_ref, demand = mask_formulation(ids, E, C)
                assert np.array_equal(slot, slot_ref) and np.array_equal(counts, demand)
                n += 1
    assert n > 10000


def gelu_np(z):
    return 0.5 * z * (1.0 + scipy.special.erf(z / np.sqrt(2.0)))


def dense_mlp_np(x, w1, b1, w2, b2):
    return gelu_np(x @ w1.T + b1) @ w2.T + b2


def _f64(a):
    return synth.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def test_single_expert_is_textbook_mlp_fp32():
    w = synth.Workload("t", T=20, d_model=12, d_ff=28, E=1, k=1, capacity_factor=1.0, dtype="f32",
                       w_router_std=1.0, w_std=0.3, b_std=0.1, seed=11)
    inp = synth.make_inputs(w)
    r = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor)
    assert (r["slot"] >= 0).all() and np.all(r["gates"] == 1.0)
    x = _f64(inp["x"])
    ref = x + dense_mlp_np(x, _f64(inp["w1"][0]), _f64(inp["b1"][0]), _f64(inp["w2"][0]), _f64(inp["b2"][0]))
    assert np.max(np.abs(r["out_exact"] - ref)) < 1e-6


def test_single_expert_is_textbook_mlp_bf16():
    # bf16: h is rounded to bf16 before the second layer (storage type of that operand)
    w = synth.Workload("t", T=16, d_model=16, d_ff=40, E=1, k=1, capacity_factor=1.0, dtype="bf16",
                       w_std=0.25, b_std=0.1, seed=12)
    inp = synth.make_inputs(w)
    r = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor)
    x = _f64(inp["x"])
    h = gelu_np(x @ _f64(inp["w1"][0]).T + _f64(inp["b1"][0]))
    h_bf = torch.from_numpy(h).float().to(torch.bfloat16).double().numpy()   # library rounding
    y = (h_bf @ _f64(inp["w2"][0]).T + _f64(inp["b2"][0])).astype(np.float32).astype(np.float64)
    ref = x + y
    # a rare h can round to the neighbouring bf16 (double rounding in the library path):
    # allow one bf16 ulp of h times the largest |W2| entry per element
    tol = np.abs(_f64(inp["w2"][0])).max() * np.abs(h).max() * 2 ** -7 * 2 + 1e-6
    assert np.max(np.abs(r["out_exact"] - ref)) < tol
    exact = np.isclose(r["out_exact"], ref, rtol=0, atol=1e-6).mean()
    assert exact > 0.95


def test_dense_mixture_identity_k_equals_E():
    # k = E and unlimited capacity: out = x + sum_e p_e E_e(x) with p = softmax(W_r x + b)
    w = synth.Workload("t", T=9, d_model=6, d_ff=10, E=3, k=3, capacity_factor=100.0, dtype="f32",
                       w_router_std=0.7, router_bias="normal", router_bias_std=0.5, w_std=0.4,
                       b_std=0.2, seed=13)
    inp = synth.make_inputs(w)
    r = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor)
    x = _f64(inp["x"])
    logits = (x @ inp["w_router"].astype(np.float64).T + inp["router_bias"].astype(np.float64))
    logits = logits.astype(np.float32).astype(np.float64)
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    ref = x.copy()
    for e in range(3):
        ye = dense_mlp_np(x, _f64(inp["w1"][e]), _f64(inp["b1"][e]), _f64(inp["w2"][e]), _f64(inp["b2"][e]))
        ref += p[:, e:e + 1].astype(np.float32).astype(np.float64) * ye
    assert np.max(np.abs(r["out_exact"] - ref)) < 1e-5


def test_capacity_zero_leaves_residual():
    for dt in ("f32", "bf16"):
        w = synth.Workload("t", T=12, d_model=8, d_ff=16, E=4, k=2, capacity_factor=0.0, dtype=dt, seed=14)
        inp = synth.make_inputs(w)
        r = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor)
        assert r["C"] == 0 and (r["slot"] < 0).all()
        assert np.array_equal(r["out"], inp["x"])


def test_prmoe_branch_is_dense_mlp_plus_gated_expert():
    w = synth.Workload("t", T=10, d_model=8, d_ff=12, E=3, k=1, capacity_factor=2.0, dtype="f32",
                       w_router_std=1.0, w_std=0.3, b_std=0.1, dense=True, add_input_residual=False,
                       seed=15)
    inp = synth.make_inputs(w)
    r = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                             add_input_residual=False)
    x = _f64(inp["x"])
    dense = dense_mlp_np(x, _f64(inp["dense_w1"]), _f64(inp["dense_b1"]), _f64(inp["dense_w2"]),
                         _f64(inp["dense_b2"])).astype(np.float32).astype(np.float64)
    ref = dense.copy()
    for t in range(w.T):
        if r["slot"][t, 0] >= 0:
            e = r["ids"][t, 0]
            ye = dense_mlp_np(x[t:t + 1], _f64(inp["w1"][e]), _f64(inp["b1"][e]), _f64(inp["w2"][e]),
                              _f64(inp["b2"][e]))
            ref[t] += float(r["gates"][t, 0]) * ye[0]
    assert np.max(np.abs(r["out_exact"] - ref)) < 1e-5


def test_token_subset_matches_full_run():
    w = synth.Workload("t", T=40, d_model=16, d_ff=24, E=4, k=2, capacity_factor=0.6, dtype="bf16", seed=16)
    inp = synth.make_inputs(w)
    full = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor)
    tok = np.array([39, 0, 17, 5])
    sub = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor, tokens=tok)
    assert np.array_equal(sub["out"], full["out"][tok])
    assert (full["slot"] < 0).any()   # capacity binds in this case


def test_given_logits_are_used_verbatim():
    w = synth.Workload("t", T=30, d_model=8, d_ff=8, E=5, k=1, capacity_factor=1.0, dtype="f32", seed=17)
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(0)
    li = rng.normal(size=(w.T, w.E)).astype(np.float32)
    r = oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor, logits_in=li)
    assert np.array_equal(r["logits"], li)
    assert np.array_equal(r["ids"][:, 0], li.argmax(1))


def test_init_variance_page_example():
    from tests.conftest import golden
    g = golden("router_init_variance.json")
    d = g["d"]
    for case in g["cases"]:
        w = synth.Workload("t", T=400, d_model=d, d_ff=8, E=64, k=1, capacity_factor=1.0, dtype="f32",
                           w_router_std=case["sigma"], seed=18)
        inp = synth.make_inputs(w)
        logits = oracle.router_logits(inp["x"], inp["w_router"]).astype(np.float64)
        assert abs(logits.var() / case["var_logits"] - 1) < 0.05
        assert abs(logits.std() - case["sd_logits"]) < 0.03 * case["sd_logits"]
