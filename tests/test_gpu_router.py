"""GPU parity of moe_router_topk against the oracle.

Logits: within an fp32-accumulation bound of the oracle's double-accumulated logits.
Routing: given the GPU's own fp32 logits, expert ids are bit-exact and gates match the oracle's
double softmax to 2e-6 relative. Statistics: f exact, Q and aux to 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import as_f64, to_dev, to_host

pytestmark = pytest.mark.gpu


def logits_bound(x: np.ndarray, w: np.ndarray, b=None) -> np.ndarray:
    """Allowed |gpu - oracle| per logit: 8 * d * eps_fp32 * sum_i |x_i w_i| + fp32 rounding."""
    xf = np.abs(as_f64(x))
    s = xf @ np.abs(w.astype(np.float64)).T
    ref_mag = s + (np.abs(b.astype(np.float64)) if b is not None else 0)
    d = x.shape[1]
    return 8 * np.sqrt(d) * 2.0 ** -24 * ref_mag + 2.0 ** -23 * ref_mag + 1e-7


def run_router(w: synth.Workload, inp: dict, k=None, want_stats=True):
    k = w.k if k is None else k
    x = to_dev(inp["x"])
    r = moe.moe_router_topk(x, to_dev(inp["w_router"]), k, router_bias=to_dev(inp.get("router_bias")),
                            aux_alpha=w.aux_alpha, want_stats=want_stats)
    err = moe.moe_get_device_error(r["ws"])
    assert err == 0
    return {n: to_host(r[n]) for n in ("logits", "expert_ids", "gates") } | (
        {"lb_stats": to_host(r["lb_stats"])} if want_stats else {})


def check_router(w, inp, got, sample=None, k=None):
    k = w.k if k is None else k
    T, E = w.T, w.E
    rows = np.arange(T) if sample is None else sample
    ref_logits = oracle.router_logits(inp["x"][rows], inp["w_router"], inp.get("router_bias"))
    bound = logits_bound(inp["x"][rows], inp["w_router"], inp.get("router_bias"))
    diff = np.abs(got["logits"][rows].astype(np.float64) - ref_logits.astype(np.float64))
    assert (diff <= bound).all(), f"logits off by {diff.max()} (bound {bound[diff > bound].min()})"
    # routing decided on the GPU's logits
    ids, gates, p = oracle.route(got["logits"], k, want_probs=True)
    assert np.array_equal(got["expert_ids"], ids)
    np.testing.assert_allclose(got["gates"], gates, rtol=2e-6, atol=1e-12)
    if "lb_stats" in got:
        f, Q, aux = oracle.lb_stats(got["logits"], ids, w.aux_alpha)
        lb = got["lb_stats"].astype(np.float64)
        np.testing.assert_array_equal(lb[:E], f.astype(np.float32))
        np.testing.assert_allclose(lb[E:2 * E], Q, rtol=1e-5, atol=1e-9)
        assert abs(lb[2 * E] - aux) <= 1e-5 * abs(aux) + 1e-9
    return diff.max()


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_router_workloads(cuda_ok, cfg):
    w = synth.WORKLOADS[cfg]
    inp = {k: v for k, v in synth.make_inputs(w.with_(d_ff=8)).items() if not k.startswith(("w1", "w2", "b1", "b2"))}
    got = run_router(w, inp)
    rng = np.random.default_rng(cfg)
    sample = None if w.T <= 2048 else np.sort(rng.choice(w.T, 1024, replace=False))
    check_router(w, inp, got, sample)


@pytest.mark.parametrize("T,d,E,k,dt", [
    (1, 64, 4, 1, "bf16"), (300, 40, 37, 3, "f32"), (257, 1032, 1024, 8, "bf16"),
    (130, 8, 1, 1, "bf16"), (64, 16, 8, 8, "f32"), (1000, 200, 200, 2, "bf16"),
])
def test_router_edge_shapes(cuda_ok, T, d, E, k, dt):
    w = synth.Workload("t", T=T, d_model=d, d_ff=8, E=E, k=k, capacity_factor=1.0, dtype=dt,
                       w_router_std=0.3, router_bias="normal", router_bias_std=0.5, seed=T + E)
    inp = synth.make_inputs(w)
    got = run_router(w, inp)
    check_router(w, inp, got)


def test_router_exact_ties_lowest_index(cuda_ok):
    # x = 0 -> every logit equals its bias; equal biases tie and go to the lowest index
    T, d, E, k = 70, 16, 12, 4
    x = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    w = torch.randn(E, d, device="cuda")
    b = torch.tensor([0.0, 1.0, 1.0, 0.5, 1.0, 0.5] * 2, device="cuda")
    r = moe.moe_router_topk(x, w, k, router_bias=b)
    ids = to_host(r["expert_ids"])
    assert (ids == np.array([1, 2, 4, 7])).all()
    g = to_host(r["gates"])
    p = np.exp(np.array([0.0, 1, 1, .5, 1, .5] * 2))
    p /= p.sum()
    np.testing.assert_allclose(g[0], p[[1, 2, 4, 7]], rtol=2e-6)


def test_router_oracle_own_logits_ids(cuda_ok):
    # ids from the oracle's own logits agree except where the top-k margin is below 1e-4
    w = synth.WORKLOADS[2].with_(T=4096, d_ff=8)
    inp = synth.make_inputs(w)
    got = run_router(w, inp, want_stats=False)
    ref_logits = oracle.router_logits(inp["x"], inp["w_router"], None)
    ids, _ = oracle.route(ref_logits, 1)
    srt = np.sort(ref_logits, axis=1)
    margin = srt[:, -1] - srt[:, -2]
    ok = margin >= 1e-4
    assert np.array_equal(got["expert_ids"][ok], ids[ok])
    assert ok.mean() > 0.99


def test_router_zero_tokens(cuda_ok):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    r = moe.moe_router_topk(x, torch.randn(8, 64, device="cuda"), 2)
    assert moe.moe_last_launch_count() == 0
    assert r["expert_ids"].shape == (0, 2)


@pytest.mark.parametrize("cfg,T", [(2, 4096), (3, 1000), (4, 2048), (2, 64)])
def test_prepared_router_weight_gives_identical_layer(cuda_ok, cfg, T):
    # the router weight split once (moe_router_prepare) and passed to the layer gives the same
    # bits as the split done inside every call; at T <= 64 (fp32 GEMV router) it is ignored
    from tests.helpers import dev_inputs, run_layer
    w = synth.WORKLOADS[cfg].with_(T=T)
    if cfg in (3, 4):
        w = w.with_(d_model=1024, d_ff=2048)
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    plain = run_layer(w, d_inp, want_losses=True)
    prep = moe.moe_router_prepare(d_inp["w_router"])
    ready = run_layer(w, d_inp, want_losses=True, w_router_prepared=prep)
    assert plain["device_error"] == 0 and ready["device_error"] == 0
    for name in plain:
        if isinstance(plain[name], np.ndarray):
            assert np.array_equal(plain[name].view(np.uint8), ready[name].view(np.uint8)), name
    # the prepared weight is the exact split: hi + mid + lo == W_r
    E, d = inp["w_router"].shape
    dpad = (d + 63) // 64 * 64
    parts = to_host(prep).view(np.uint16).reshape(E, 3, dpad)[:, :, :d]
    widened = synth.bf16_bits_to_f32(parts).astype(np.float64)
    np.testing.assert_array_equal(widened.sum(1), inp["w_router"].astype(np.float64))


def _router_all(inp, k, renormalize, want_losses):
    r = moe.moe_router_topk(to_dev(inp["x"]), to_dev(inp["w_router"]), k,
                            router_bias=to_dev(inp.get("router_bias")), renormalize=renormalize,
                            router_losses=True if want_losses else None, probs=True)
    assert moe.moe_get_device_error(r["ws"]) == 0
    return {n: to_host(v) for n, v in r.items() if isinstance(v, torch.Tensor) and n != "ws"}


@pytest.mark.parametrize("T,d,E,k,renorm,extra", [
    (16384, 1024, 128, 1, False, False),   # the headline router: one tile per CTA
    (40000, 64, 128, 2, True, True),       # several tiles per CTA: stage 0 handed back and forth
    (20000, 256, 37, 3, False, True),      # E not a power of two, 64-expert tile
    (300, 128, 8, 2, True, True),          # 16-expert tile, ragged last tile
    (1000, 512, 32, 1, False, False),
])
def test_fused_router_equals_two_kernels(cuda_ok, monkeypatch, T, d, E, k, renorm, extra):
    # softmax, top-k and the statistics in the tensor-core kernel's epilogue give the bits of the
    # separate top-k kernel reading the logits back
    w = synth.Workload("fused", T=T, d_model=d, d_ff=8, E=E, k=k, capacity_factor=1.0,
                       dtype="bf16", w_router_std=0.05, router_bias="normal", router_bias_std=0.3,
                       seed=T + E)
    inp = synth.make_inputs(w)
    fused = _router_all(inp, k, renorm, extra)
    monkeypatch.setenv("MOE_FUSED_ROUTER", "0")
    two = _router_all(inp, k, renorm, extra)
    for name in two:
        assert np.array_equal(fused[name].view(np.uint8), two[name].view(np.uint8)), name
    # against the oracle: the probabilities output carries the unrenormalised gates
    check_router(w, inp, {**fused, "gates": fused["probs"]},
                 sample=np.arange(0, T, max(1, T // 512)), k=k)
    if renorm:
        np.testing.assert_allclose(fused["gates"].sum(1), 1.0, rtol=1e-5)


def test_fused_router_layer_without_logits_output(cuda_ok, monkeypatch):
    # the layer with no logits requested (nothing of them reaches global memory) gives the same
    # routing, dispatch and output as with them, and as the two-kernel router
    from tests.helpers import dev_inputs
    w = synth.WORKLOADS[2].with_(T=4096, d_model=512, d_ff=1024)
    d_inp = dev_inputs(synth.make_inputs(w))
    args = moe.layer_args(d_inp["x"], d_inp["w_router"], d_inp["w1"], d_inp["b1"], d_inp["w2"],
                          d_inp["b2"], k=w.k, capacity_factor=w.capacity_factor)

    def run(with_logits):
        aux = dict(expert_ids=torch.empty(w.T, 1, dtype=torch.int32, device="cuda"),
                   slot=torch.empty(w.T, 1, dtype=torch.int32, device="cuda"),
                   lb_stats=torch.empty(2 * w.E + 1, dtype=torch.float32, device="cuda"))
        if with_logits:
            aux["logits"] = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
        out = torch.empty(w.T, w.d_model, dtype=torch.bfloat16, device="cuda")
        ws = moe.workspace(moe.moe_layer_workspace_bytes(args), "cuda")
        moe.moe_layer_forward(args, out, aux=aux, ws=ws)
        assert moe.moe_get_device_error(ws) == 0
        return {n: to_host(t) for n, t in aux.items() if n != "logits"} | {"out": to_host(out)}

    a, b = run(False), run(True)
    monkeypatch.setenv("MOE_FUSED_ROUTER", "0")
    c = run(False)
    for n in a:
        assert np.array_equal(a[n], b[n]), n
        assert np.array_equal(a[n], c[n]), n
