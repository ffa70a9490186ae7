"""The token-sharded layer's exchange through NCCL on the GPU, with a one-rank process group.

Every GPU run of this test suite has one GPU, so the exchange runs over a single NCCL rank: the
all-gather of the demands and the all-reduce of the integer statistics partials go through NCCL
on device buffers, on the layer's stream, between the begin and end halves of the layer. The
result must equal the single-GPU layer bit for bit and the oracle on the whole batch. (Two or more
NCCL ranks on one GPU would wait on one another inside NCCL's kernels, which is not run here; the
multi-rank exchange is tested with gloo ranks on the CPU.)
"""
import datetime
import socket

import numpy as np
import pytest
import torch

import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import dev_inputs, run_layer, to_host
from tests.test_gpu_shard import check_against_oracle

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture
def nccl_group(cuda_ok):
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        yield dist.group.WORLD
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cfg,T,renormalize", [(2, 2048, False), (3, 1000, False),
                                               (4, 768, True)])
def test_sharded_layer_over_nccl(nccl_group, cfg, T, renormalize):
    w = synth.WORKLOADS[cfg].with_(T=T, d_model=512, d_ff=1024)
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    whole = run_layer(w, d_inp, renormalize=renormalize, want_losses=True)
    dense = None
    if w.dense:
        dense = (d_inp["dense_w1"], d_inp["dense_b1"], d_inp["dense_w2"], d_inp["dense_b2"])
    args = moe.layer_args(d_inp["x"], d_inp["w_router"], d_inp["w1"], d_inp["b1"], d_inp["w2"],
                          d_inp["b2"], k=w.k, capacity_factor=w.capacity_factor,
                          router_bias=d_inp.get("router_bias"), dense=dense,
                          add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha,
                          renormalize_gates=renormalize)
    E, k = w.E, w.k
    dev = d_inp["x"].device
    aux = dict(logits=torch.empty(T, E, dtype=torch.float32, device=dev),
               topk_probs=torch.empty(T, k, dtype=torch.float32, device=dev),
               expert_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               gates=torch.empty(T, k, dtype=torch.float32, device=dev),
               slot=torch.empty(T, k, dtype=torch.int32, device=dev),
               expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
               expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               lb_stats=torch.empty(2 * E + 1, dtype=torch.float32, device=dev),
               router_losses=torch.empty(3, dtype=torch.float32, device=dev))
    out = torch.empty(T, w.d_model, dtype=d_inp["x"].dtype, device=dev)
    ws = moe.workspace(moe.moe_layer_shard_workspace_bytes(args, T), dev)
    moe.moe_layer_forward_sharded(args, T, out, group=nccl_group, aux=aux, ws=ws)
    assert moe.moe_get_device_error(ws) == 0
    torch.cuda.synchronize()
    got = {n: to_host(t) for n, t in aux.items()}
    got["out"] = to_host(out)
    for n in ("out", "expert_ids", "gates", "slot", "expert_counts", "expert_offsets", "lb_stats",
              "router_losses", "topk_probs"):
        assert np.array_equal(got[n], whole[n]), n
    sh = dict(out=got["out"], demand_all=got["expert_counts"][None, :], lb=[got["lb_stats"]],
              losses=[got["router_losses"]])
    for n in ("expert_ids", "gates", "slot", "logits", "topk_probs"):
        sh[n] = got[n]
    check_against_oracle(w, inp, [T], sh, renormalize)
