"""GPU parity of the layer's backward pass (moe_layer_forward_train + moe_layer_backward) against
the oracle's chain rule (oracle.layer_backward, pinned by finite differences).

The oracle differentiates the same routing: it takes the GPU's fp32 logits and the chosen
experts' fp32 probabilities, so top-k, slots and the priority order are the GPU's. Tolerances (gradient g against the oracle's r, over
each tensor): fp32 layers, relative L2 <= 1e-5 and max |g - r| <= 1e-4 max |r|; bf16 layers (the
backward GEMM operands dY, dZ and GeLU'(z) are rounded to bf16, fp32 accumulation, dx returned
in bf16), relative L2 <= 1e-2 and max |g - r| <= 5e-2 max |r|.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import as_f64, dev_inputs, run_layer, to_dev, to_host

pytestmark = pytest.mark.gpu


def run_train(w: synth.Workload, d_inp: dict, dout_dev, aux_weight=0.0, z_weight=0.0,
              renormalize=False, overflow_priority=False):
    T, E, k, d, f = w.T, w.E, w.k, w.d_model, w.d_ff
    x = d_inp["x"]
    dense = None
    if w.dense:
        dense = (d_inp["dense_w1"], d_inp["dense_b1"], d_inp["dense_w2"], d_inp["dense_b2"])
    args = moe.layer_args(x, d_inp["w_router"], d_inp["w1"], d_inp["b1"], d_inp["w2"], d_inp["b2"],
                          k=k, capacity_factor=w.capacity_factor,
                          router_bias=d_inp.get("router_bias"), dense=dense,
                          add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha,
                          overflow_priority=overflow_priority, renormalize_gates=renormalize)
    dev = x.device
    aux = dict(logits=torch.empty(T, E, dtype=torch.float32, device=dev),
               expert_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               gates=torch.empty(T, k, dtype=torch.float32, device=dev),
               slot=torch.empty(T, k, dtype=torch.int32, device=dev),
               topk_probs=torch.empty(T, k, dtype=torch.float32, device=dev))
    out = torch.empty(T, d, dtype=x.dtype, device=dev)
    ws = moe.moe_layer_forward_train(args, out, aux=aux)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = dict(dx=torch.empty(T, d, dtype=x.dtype, device=dev),
                 dw_router=torch.empty(E, d, **f32), db_router=torch.empty(E, **f32),
                 dw1=torch.empty(E, f, d, **f32), dw2=torch.empty(E, d, f, **f32),
                 dgates=torch.empty(T, k, **f32), dlogits=torch.empty(T, E, **f32))
    if d_inp.get("b1") is not None:
        grads["db1"] = torch.empty(E, f, **f32)
    if d_inp.get("b2") is not None:
        grads["db2"] = torch.empty(E, d, **f32)
    if w.dense:
        grads.update(dense_dw1=torch.empty(f, d, **f32), dense_db1=torch.empty(f, **f32),
                     dense_dw2=torch.empty(d, f, **f32), dense_db2=torch.empty(d, **f32))
    moe.moe_layer_backward(args, dout_dev, grads, ws, aux_weight=aux_weight, z_weight=z_weight)
    assert moe.moe_get_device_error(ws) == 0
    r = {n: to_host(t) for n, t in grads.items()}
    r.update({n: to_host(t) for n, t in aux.items()})
    r["out"] = to_host(out)
    return r


def compare(name, got, ref, bf16):
    g = as_f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    rel = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(g - ref).max() / scale
    rel_tol, max_tol = (1e-2, 5e-2) if bf16 else (1e-5, 1e-4)
    assert rel <= rel_tol and mx <= max_tol, f"{name}: rel-L2 {rel:.3g}, max/scale {mx:.3g}"
    return rel


def backward_parity(w: synth.Workload, aux_weight=0.3, z_weight=0.1, renormalize=False,
                    overflow_priority=False, seed=0):
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    rng = np.random.default_rng(seed)
    bf16 = w.dtype == "bf16"
    dout = rng.normal(size=(w.T, w.d_model)).astype(np.float32)
    dout_h = oracle.round_bf16(dout) if bf16 else dout
    got = run_train(w, d_inp, to_dev(dout_h), aux_weight, z_weight, renormalize, overflow_priority)
    # forward of the training path = the inference forward, bit for bit
    fwd = run_layer(w, d_inp, overflow_priority=overflow_priority, renormalize=renormalize)
    assert np.array_equal(got["out"], fwd["out"])
    assert np.array_equal(got["expert_ids"], fwd["expert_ids"])
    ref = oracle.layer_backward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                                as_f64(dout_h), add_input_residual=w.add_input_residual,
                                aux_alpha=w.aux_alpha, aux_weight=aux_weight, z_weight=z_weight,
                                logits_in=got["logits"], probs_in=got["topk_probs"],
                                overflow_priority=overflow_priority, renormalize=renormalize)
    res = {}
    pairs = [("dx", "dx"), ("dw_router", "dw_router"), ("db_router", "db_router"),
             ("dw1", "dw1"), ("dw2", "dw2"), ("dgates", "dgates"), ("dlogits", "dlogits")]
    if "db1" in got:
        pairs.append(("db1", "db1"))
    if "db2" in got:
        pairs.append(("db2", "db2"))
    if w.dense:
        pairs += [(n, n) for n in ("dense_dw1", "dense_db1", "dense_dw2", "dense_db2")]
    for gname, rname in pairs:
        res[gname] = compare(gname, got[gname], ref[rname], bf16)
    return got, ref, res


def test_backward_tiny_fp32(cuda_ok):
    got, ref, _ = backward_parity(synth.WORKLOADS[1])
    assert (got["slot"] < 0).any()  # dropped tokens get no expert gradient


def test_backward_fp32_top2_dense_renorm(cuda_ok):
    w = synth.Workload("f32-top2-dense", T=200, d_model=48, d_ff=72, E=6, k=2,
                       capacity_factor=1.0, dtype="f32", w_router_std=0.5, router_bias="normal",
                       router_bias_std=0.5, dense=True, add_input_residual=False, seed=77)
    backward_parity(w, renormalize=True)


@pytest.mark.parametrize("cfg,T,shape,kw", [
    (2, 1024, dict(d_model=256, d_ff=512), {}),
    (3, 512, dict(d_model=256, d_ff=512), {}),
    (4, 512, dict(d_model=512, d_ff=1024), dict(renormalize=True, overflow_priority=True)),
    (5, 32, dict(d_model=256, d_ff=512), {}),
])
def test_backward_bf16_workloads_reduced(cuda_ok, cfg, T, shape, kw):
    w = synth.WORKLOADS[cfg].with_(T=T, **shape)
    backward_parity(w, **kw)


def test_backward_bf16_full_k(cuda_ok):
    # the headline workload's layer widths (K = 1024 into layer 1, K = 4096 into layer 2, and
    # d_ff = 4096 output features of the weight gradients) on a few hundred tokens; 8 experts keep
    # the oracle's float64 weight gradients small
    w = synth.WORKLOADS[2].with_(T=320, E=8, capacity_factor=1.0)
    got, _, _ = backward_parity(w, renormalize=True, overflow_priority=True)
    assert (got["slot"] < 0).any()


def test_backward_bf16_ragged_dims(cuda_ok):
    # d and d_ff not multiples of 64 (MN-major tails), top-2, drops
    w = synth.Workload("ragged", T=300, d_model=264, d_ff=200, E=5, k=2, capacity_factor=0.8,
                       dtype="bf16", w_router_std=0.3, router_bias="normal", router_bias_std=0.5,
                       seed=31)
    got, _, _ = backward_parity(w)
    assert (got["slot"] < 0).any()


def test_backward_bf16_one_hot_expert(cuda_ok):
    # every token routed to one expert: one long segment (many 64-row K blocks in the weight
    # gradient), the other experts get zero gradients
    w = synth.WORKLOADS[2].with_(T=700, d_model=256, d_ff=512, capacity_factor=200.0)
    inp = synth.make_inputs(w)
    inp["router_bias"] = np.zeros(w.E, dtype=np.float32)
    inp["router_bias"][5] = 8.0
    d_inp = dev_inputs(inp)
    dout = oracle.round_bf16(np.random.default_rng(1).normal(size=(w.T, w.d_model)))
    got = run_train(w, d_inp, to_dev(dout))
    assert (got["expert_ids"][:, 0] == 5).all()
    others = np.delete(got["dw1"], 5, axis=0)
    assert np.abs(others).max() == 0.0
    ref = oracle.layer_backward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                                as_f64(dout), aux_alpha=w.aux_alpha, logits_in=got["logits"],
                                probs_in=got["topk_probs"])
    for n in ("dw1", "dw2", "dx", "dw_router"):
        compare(n, got[n], ref[n], True)


def test_backward_deterministic(cuda_ok):
    w = synth.WORKLOADS[4].with_(T=256, d_model=256, d_ff=512)
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    dout = to_dev(oracle.round_bf16(np.random.default_rng(3).normal(size=(w.T, w.d_model))))
    a = run_train(w, d_inp, dout, 0.2, 0.1)
    b = run_train(w, d_inp, dout, 0.2, 0.1)
    for n in a:
        assert np.array_equal(a[n], b[n]), n


def test_backward_no_tokens_zeroes_gradients(cuda_ok):
    w = synth.WORKLOADS[2].with_(T=0, d_model=128, d_ff=256)
    d_inp = dev_inputs(synth.make_inputs(w.with_(T=4)))
    d_inp["x"] = d_inp["x"][:0]
    args = moe.layer_args(d_inp["x"], d_inp["w_router"], d_inp["w1"], d_inp["b1"], d_inp["w2"],
                          d_inp["b2"], k=1, capacity_factor=1.0)
    out = torch.empty(0, w.d_model, dtype=torch.bfloat16, device="cuda")
    ws = moe.moe_layer_forward_train(args, out)
    f32 = dict(dtype=torch.float32, device="cuda")
    g = dict(dx=torch.empty(0, w.d_model, dtype=torch.bfloat16, device="cuda"),
             dw_router=torch.full((w.E, w.d_model), 7.0, **f32),
             db_router=torch.full((w.E,), 7.0, **f32),
             dw1=torch.full((w.E, w.d_ff, w.d_model), 7.0, **f32),
             db1=torch.full((w.E, w.d_ff), 7.0, **f32),
             dw2=torch.full((w.E, w.d_model, w.d_ff), 7.0, **f32),
             db2=torch.full((w.E, w.d_model), 7.0, **f32))
    moe.moe_layer_backward(args, torch.empty(0, w.d_model, dtype=torch.bfloat16, device="cuda"),
                           g, ws)
    torch.cuda.synchronize()
    for n, t in g.items():
        if n != "dx":
            assert float(t.abs().max()) == 0.0, n
