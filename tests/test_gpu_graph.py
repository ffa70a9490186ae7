"""A layer call captured into a CUDA graph and replayed.

moe_layer_forward enqueues only device work on the caller's stream (programmatic dependent
launches, one memset, tensor maps encoded on the host at enqueue time), so it can be captured;
every replay must produce the eager call's outputs bit for bit, also after the inputs change in
place between replays (the graph holds pointers, not values).
"""
import numpy as np
import pytest
import torch

import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import dev_inputs, to_host

pytestmark = pytest.mark.gpu


def _layer(w, d):
    dense = None
    if w.dense:
        dense = (d["dense_w1"], d["dense_b1"], d["dense_w2"], d["dense_b2"])
    args = moe.layer_args(d["x"], d["w_router"], d["w1"], d["b1"], d["w2"], d["b2"], k=w.k,
                          capacity_factor=w.capacity_factor, router_bias=d.get("router_bias"),
                          dense=dense, add_input_residual=w.add_input_residual,
                          aux_alpha=w.aux_alpha)
    dev = d["x"].device
    aux = dict(expert_ids=torch.empty(w.T, w.k, dtype=torch.int32, device=dev),
               slot=torch.empty(w.T, w.k, dtype=torch.int32, device=dev),
               lb_stats=torch.empty(2 * w.E + 1, dtype=torch.float32, device=dev))
    out = torch.empty(w.T, w.d_model, dtype=d["x"].dtype, device=dev)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(args), dev)
    return args, aux, out, ws


@pytest.mark.parametrize("cfg,kw", [(2, dict(T=2048, d_model=512, d_ff=1024)),
                                    (3, dict(T=4096, E=32, d_model=512, d_ff=1024)),
                                    (4, dict(T=1024, d_model=256, d_ff=512)),
                                    (5, {})])
def test_layer_graph_replay(cuda_ok, cfg, kw):
    w = synth.WORKLOADS[cfg].with_(**kw)
    inp = synth.make_inputs(w)
    d = dev_inputs(inp)
    args, aux, out, ws = _layer(w, d)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.moe_layer_forward(args, out, aux=aux, ws=ws, stream=s)  # warm-up outside the capture
    s.synchronize()
    eager = {n: to_host(t) for n, t in aux.items()}
    eager["out"] = to_host(out)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        moe.moe_layer_forward(args, out, aux=aux, ws=ws, stream=s)
    out.zero_()
    for t in aux.values():
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws) == 0
    for n, t in aux.items():
        assert np.array_equal(to_host(t), eager[n]), n
    assert np.array_equal(to_host(out), eager["out"])
    # new token values in the same buffer: the replay must follow them
    d2 = dev_inputs(synth.make_inputs(w.with_(seed=w.seed + 11)))
    d["x"].copy_(d2["x"])
    g.replay()
    torch.cuda.synchronize()
    got = to_host(out)
    with torch.cuda.stream(s):
        moe.moe_layer_forward(args, out, aux=aux, ws=ws, stream=s)
    s.synchronize()
    assert np.array_equal(got, to_host(out))
    assert not np.array_equal(got, eager["out"])
    del g
