"""Pins of the oracle's backward pass (oracle_layer_backward) to things other than itself:

* central finite differences of the forward oracle's objective
  L = sum(dout * out) + aux_weight * aux + z_weight * z_loss, element by element, for every
  parameter and input of small fp32 layers (top-2 with drops, renormalised gates, PR-MoE dense
  branch, router bias, both extra loss terms);
* one expert that takes every token is a dense two-layer GeLU MLP: its gradients equal
  torch.autograd's (float64), and the router gets none (softmax over one expert is constant);
* closed forms: equal logits give a z-loss gradient of 2 (c + ln E) / E per router bias; the
  softmax backward sums to zero over the experts;
* the bf16 path differs from the fp32 path only through the bf16 rounding of h.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def margins_ok(inp, w, min_gap):
    logits = oracle.router_logits(inp["x"], inp["w_router"], inp.get("router_bias")).astype(np.float64)
    s = -np.sort(-logits, axis=1)
    gaps = s[:, :min(w.k + 1, w.E) - 0]
    return (np.diff(gaps, axis=1) < -min_gap).all()


def small_workload(seed, **kw):
    base = dict(T=8, d_model=6, d_ff=5, E=3, k=2, capacity_factor=0.75, dtype="f32",
                x_std=1.0, w_router_std=1.0, router_bias="normal", router_bias_std=0.5,
                w_std=0.4, b_std=0.2)
    base.update(kw)
    for s in range(seed, seed + 200):
        w = synth.Workload("fd", seed=s, **base)
        inp = synth.make_inputs(w)
        if margins_ok(inp, w, 0.05):
            return w, inp
    raise RuntimeError("no seed with clear routing margins")


PARAMS = ["x", "w_router", "router_bias", "w1", "b1", "w2", "b2",
          "dense_w1", "dense_b1", "dense_w2", "dense_b2"]
GRAD = {"x": "dx", "w_router": "dw_router", "router_bias": "db_router", "w1": "dw1", "b1": "db1",
        "w2": "dw2", "b2": "db2", "dense_w1": "dense_dw1", "dense_b1": "dense_db1",
        "dense_w2": "dense_dw2", "dense_b2": "dense_db2"}


@pytest.mark.parametrize("dense,renorm,priority,aux_w,z_w", [
    (False, False, False, 0.0, 0.0), (False, True, False, 0.7, 0.3), (True, False, False, 0.5, 0.0),
    (True, True, True, 0.0, 0.4),
])
def test_backward_matches_finite_differences(dense, renorm, priority, aux_w, z_w):
    w, inp = small_workload(11, dense=dense)
    rng = np.random.default_rng(3)
    dout = rng.normal(size=(w.T, w.d_model))
    kw = dict(add_input_residual=not dense, aux_alpha=0.05, aux_weight=aux_w, z_weight=z_w,
              overflow_priority=priority, renormalize=renorm)
    args = (w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor)
    g = oracle.layer_backward(inp, *args, dout, **kw)
    fwd = oracle.layer_forward(inp, *args, add_input_residual=kw["add_input_residual"],
                               overflow_priority=priority, renormalize=renorm)
    assert (fwd["slot"] < 0).any()               # some choices overflow
    eps = 2e-3
    checked = 0
    for name in PARAMS:
        if inp.get(name) is None:
            assert GRAD[name] not in g or g[GRAD[name]] is None or name == "router_bias"
            continue
        base = inp[name]
        grad = g[GRAD[name]]
        for idx in np.ndindex(base.shape):
            orig = base[idx]
            hi = np.float32(orig + eps)
            lo = np.float32(orig - eps)
            base[idx] = hi
            lp = oracle.layer_loss(inp, *args, dout, **kw)
            base[idx] = lo
            lm = oracle.layer_loss(inp, *args, dout, **kw)
            base[idx] = orig
            fd = (lp - lm) / (float(hi) - float(lo))
            an = grad[idx]
            assert abs(fd - an) <= 2e-3 + 2e-3 * abs(an), (name, idx, fd, an)
            checked += 1
    assert checked > 150


def test_one_expert_is_a_dense_mlp_torch_autograd():
    w = synth.Workload("mlp", T=7, d_model=5, d_ff=9, E=1, k=1, capacity_factor=2.0, dtype="f32",
                       x_std=1.0, w_std=0.5, b_std=0.3, seed=4)
    inp = synth.make_inputs(w)
    dout = np.random.default_rng(1).normal(size=(w.T, w.d_model))
    g = oracle.layer_backward(inp, w.T, w.d_model, w.d_ff, 1, 1, 2.0, dout,
                              add_input_residual=False, aux_weight=0.0, z_weight=0.0)
    t = {n: torch.tensor(inp[n].astype(np.float64), requires_grad=True)
         for n in ("x", "w1", "b1", "w2", "b2")}
    z = t["x"] @ t["w1"][0].T + t["b1"][0]
    h = torch.nn.functional.gelu(z, approximate="none")
    y = h @ t["w2"][0].T + t["b2"][0]
    (y * torch.tensor(dout)).sum().backward()
    for n, gn in (("x", "dx"), ("w1", "dw1"), ("b1", "db1"), ("w2", "dw2"), ("b2", "db2")):
        np.testing.assert_allclose(g[gn], t[n].grad.numpy().reshape(g[gn].shape), rtol=1e-9,
                                   atol=1e-10)
    assert np.abs(g["dw_router"]).max() == 0.0 and np.abs(g["db_router"]).max() == 0.0


def test_gelu_grad_against_textbook_values():
    # d/dz [z Phi(z)] = Phi(z) + z phi(z); Phi(0) = 1/2, Phi(1) = 0.8413447460685429,
    # phi(1) = 0.24197072451914337
    assert oracle.gelu_grad(0.0) == 0.5
    assert abs(oracle.gelu_grad(1.0) - (0.8413447460685429 + 0.24197072451914337)) < 1e-15
    assert abs(oracle.gelu_grad(-1.0) - (1 - 0.8413447460685429 - 0.24197072451914337)) < 1e-15
    h = 1e-6
    for z in (-3.0, -0.4, 0.7, 2.5):
        fd = (oracle.gelu(z + h) - oracle.gelu(z - h)) / (2 * h)
        assert abs(fd - oracle.gelu_grad(z)) < 1e-8


def test_z_loss_gradient_closed_form_equal_logits():
    T, d, E, c = 5, 4, 6, 0.75
    w = synth.Workload("z", T=T, d_model=d, d_ff=3, E=E, k=1, capacity_factor=1.0, dtype="f32",
                       seed=2)
    inp = synth.make_inputs(w)
    inp["w_router"] = np.zeros((E, d), dtype=np.float32)
    inp["router_bias"] = np.full(E, c, dtype=np.float32)
    g = oracle.layer_backward(inp, T, d, 3, E, 1, 1.0, np.zeros((T, d)), aux_weight=0.0,
                              z_weight=1.0)
    np.testing.assert_allclose(g["db_router"], 2 * (c + np.log(E)) / E, rtol=1e-12)


def test_softmax_backward_sums_to_zero_over_experts():
    w, inp = small_workload(40, E=5, k=2, T=12)
    dout = np.random.default_rng(5).normal(size=(w.T, w.d_model))
    g = oracle.layer_backward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor, dout,
                              aux_weight=0.4, z_weight=0.0)
    assert np.abs(g["dlogits"].sum(axis=1)).max() < 1e-12
    assert abs(g["db_router"].sum()) < 1e-12


def test_bf16_path_differs_only_through_h_rounding():
    w = synth.Workload("b", T=16, d_model=16, d_ff=24, E=4, k=2, capacity_factor=1.0,
                       dtype="bf16", seed=9, w_std=0.3, b_std=0.1, w_router_std=0.5)
    inp_b = synth.make_inputs(w)
    inp_f = {n: (oracle.bf16_to_float(v).astype(np.float32) if isinstance(v, np.ndarray)
                 and v.dtype == np.uint16 else v) for n, v in inp_b.items()}
    dout = np.random.default_rng(2).normal(size=(w.T, w.d_model))
    args = (w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor, dout)
    gb = oracle.layer_backward(inp_b, *args)
    gf = oracle.layer_backward(inp_f, *args)
    for n in ("dw1", "db1", "db2", "dw_router", "db_router", "dgates"):
        if n in ("dw_router", "db_router", "dgates"):
            # these see y, which uses the rounded h
            np.testing.assert_allclose(gb[n], gf[n], rtol=0.05, atol=0.05 * np.abs(gf[n]).max())
        else:
            assert np.array_equal(gb[n], gf[n]), n
    assert not np.array_equal(gb["dw2"], gf["dw2"])
    np.testing.assert_allclose(gb["dw2"], gf["dw2"], rtol=0, atol=2 ** -8 * np.abs(gf["dw2"]).max() * 4)
