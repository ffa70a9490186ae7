"""GPU check of the token-sharded layer (moe_layer_forward_shard_begin / _end) against the oracle
on the whole batch, and against the whole-batch layer on one GPU.

The G shards run one after another on the one GPU: every shard's begin, then the exchange done by
hand (the demands stacked in shard order, the statistics partials summed), then every shard's end.
No kernel waits on another shard. Against the oracle (run on the whole batch from the shards' own
fp32 logits and probabilities): ids exact, gates to 2e-6, every token's global slot exact (local
slot + the earlier shards' demand), demand per expert exact, f exact and Q, aux, z-loss and CoV^2
within the single-GPU tolerances, every output row within the output tolerances. Against the
whole-batch layer: ids, gates and output rows bit for bit; lb_stats and router losses bit for bit
when the shards before the last hold multiples of 64 tokens.
"""
import numpy as np
import pytest
import torch

import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import check_out, dev_inputs, oracle_layer, run_layer, to_host

pytestmark = pytest.mark.gpu


def run_shards(w: synth.Workload, d_inp: dict, sizes, renormalize=False):
    assert sum(sizes) == w.T
    G = len(sizes)
    E, k = w.E, w.k
    dense = None
    if w.dense:
        dense = (d_inp["dense_w1"], d_inp["dense_b1"], d_inp["dense_w2"], d_inp["dense_b2"])
    shards = []
    t0 = 0
    for n in sizes:
        x = d_inp["x"][t0:t0 + n]
        args = moe.layer_args(x, d_inp["w_router"], d_inp["w1"], d_inp["b1"], d_inp["w2"],
                              d_inp["b2"], k=k, capacity_factor=w.capacity_factor,
                              router_bias=d_inp.get("router_bias"), dense=dense,
                              add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha,
                              renormalize_gates=renormalize)
        dev = x.device
        aux = dict(logits=torch.empty(n, E, dtype=torch.float32, device=dev),
                   topk_probs=torch.empty(n, k, dtype=torch.float32, device=dev),
                   expert_ids=torch.empty(n, k, dtype=torch.int32, device=dev),
                   gates=torch.empty(n, k, dtype=torch.float32, device=dev),
                   slot=torch.empty(n, k, dtype=torch.int32, device=dev),
                   expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
                   expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                   lb_stats=torch.empty(2 * E + 1, dtype=torch.float32, device=dev),
                   router_losses=torch.empty(3, dtype=torch.float32, device=dev))
        demand = torch.empty(E, dtype=torch.int32, device=dev)
        partials = torch.empty(moe.moe_router_partials_count(E), dtype=torch.int64, device=dev)
        ws = moe.moe_layer_forward_shard_begin(args, w.T, demand, partials, aux=aux)
        shards.append(dict(args=args, aux=aux, demand=demand, partials=partials, ws=ws, n=n, x=x))
        t0 += n
    demand_all = torch.stack([s["demand"] for s in shards])
    totals = torch.stack([s["partials"] for s in shards]).sum(0)
    outs = []
    for r, s in enumerate(shards):
        out = torch.empty(s["n"], w.d_model, dtype=s["x"].dtype, device=s["x"].device)
        moe.moe_layer_forward_shard_end(s["args"], w.T, G, r, demand_all, totals, out, s["ws"],
                                        aux=s["aux"])
        assert moe.moe_get_device_error(s["ws"]) == 0
        outs.append(out)
    torch.cuda.synchronize()
    res = dict(out=np.concatenate([to_host(o) for o in outs]),
               demand_all=to_host(demand_all),
               lb=[to_host(s["aux"]["lb_stats"]) for s in shards],
               losses=[to_host(s["aux"]["router_losses"]) for s in shards])
    for name in ("expert_ids", "gates", "slot", "logits", "topk_probs"):
        res[name] = np.concatenate([to_host(s["aux"][name]) for s in shards])
    res["counts"] = [to_host(s["aux"]["expert_counts"]) for s in shards]
    res["offsets"] = [to_host(s["aux"]["expert_offsets"]) for s in shards]
    return res


def check_against_oracle(w, inp, sizes, sh, renormalize):
    """The shards' results against the oracle's layer over the whole batch."""
    ref = oracle_layer(inp, w, logits_in=sh["logits"], probs_in=sh["topk_probs"],
                       renormalize=renormalize)
    assert np.array_equal(sh["expert_ids"], ref["ids"])
    np.testing.assert_allclose(sh["gates"], ref["gates"], rtol=2e-6, atol=1e-12)
    assert np.array_equal(sh["demand_all"].sum(0), ref["counts"])
    base = np.concatenate([np.zeros((1, w.E), np.int64),
                           np.cumsum(sh["demand_all"], axis=0)[:-1]]).astype(np.int64)
    t0 = 0
    for r, n in enumerate(sizes):
        ids = sh["expert_ids"][t0:t0 + n]
        ls = sh["slot"][t0:t0 + n]
        rs = ref["slot"][t0:t0 + n]
        assert np.array_equal(ls < 0, rs < 0), r
        kept = ls >= 0
        assert np.array_equal(ls[kept] + base[r][ids[kept]], rs[kept]), r
        t0 += n
    E = w.E
    for r in range(len(sizes)):
        lb = sh["lb"][r]
        np.testing.assert_array_equal(lb[:E], ref["f"].astype(np.float32))
        np.testing.assert_allclose(lb[E:2 * E], ref["Q"], rtol=1e-5, atol=1e-9)
        assert abs(lb[2 * E] - ref["aux"]) <= 1e-5 * abs(ref["aux"]) + 1e-9
        z, ci, cl = sh["losses"][r]
        assert abs(z - ref["z_loss"]) <= 1e-5 * abs(ref["z_loss"]) + 1e-6
        assert abs(ci - ref["cov2_importance"]) <= 1e-5 * abs(ref["cov2_importance"]) + 1e-7
        assert abs(cl - ref["cov2_load"]) <= 1e-6 * abs(ref["cov2_load"]) + 1e-9
    bf16 = w.dtype == "bf16"
    check_out(sh["out"], ref["out_exact"], bf16, bf16, what=f"{w.name} shards {sizes}")
    return ref


def compare(w, sizes, renormalize=False, exact_stats=True):
    inp = synth.make_inputs(w)
    d_inp = dev_inputs(inp)
    whole = run_layer(w, d_inp, renormalize=renormalize, want_losses=True)
    sh = run_shards(w, d_inp, sizes, renormalize=renormalize)
    check_against_oracle(w, inp, sizes, sh, renormalize)
    assert np.array_equal(sh["expert_ids"], whole["expert_ids"])
    assert np.array_equal(sh["gates"], whole["gates"])
    # kept exactly where the whole batch keeps; local slot = global slot - earlier demand
    base = np.concatenate([np.zeros((1, w.E), np.int64),
                           np.cumsum(sh["demand_all"], axis=0)[:-1]]).astype(np.int64)
    t0 = 0
    for r, n in enumerate(sizes):
        ids = whole["expert_ids"][t0:t0 + n]
        gs = whole["slot"][t0:t0 + n]
        ls = sh["slot"][t0:t0 + n]
        assert np.array_equal(ls < 0, gs < 0)
        kept = gs >= 0
        assert np.array_equal(ls[kept], gs[kept] - base[r][ids[kept]])
        assert np.array_equal(sh["counts"][r], sh["demand_all"][r])
        t0 += n
    assert np.array_equal(sh["demand_all"].sum(0), whole["expert_counts"])
    assert np.array_equal(sh["out"].view(np.uint8), whole["out"].view(np.uint8))
    for r in range(len(sizes)):
        if exact_stats:
            assert np.array_equal(sh["lb"][r], whole["lb_stats"])
            assert np.array_equal(sh["losses"][r], whole["router_losses"])
        else:
            np.testing.assert_allclose(sh["lb"][r], whole["lb_stats"], rtol=1e-6, atol=1e-9)
            np.testing.assert_allclose(sh["losses"][r], whole["router_losses"], rtol=1e-5)
    return whole, sh


def test_shards_tiny_fp32_overflowing(cuda_ok):
    w = synth.WORKLOADS[1].with_(T=256)
    whole, _ = compare(w, [64, 128, 64])
    assert (whole["slot"] < 0).any()
    # shards of at most 64 tokens still take the whole batch's logits kernel
    compare(w, [64, 64, 64, 64])


@pytest.mark.parametrize("cfg,T,sizes", [
    (2, 4096, [1024, 1024, 1024, 1024]), (2, 2048, [1536, 512]), (3, 1024, [512, 512]),
    (4, 1024, [256, 768]), (5, 32, [32]),
])
def test_shards_match_whole_batch(cuda_ok, cfg, T, sizes):
    w = synth.WORKLOADS[cfg]
    shrink = dict(T=T)
    if cfg in (3, 4):
        shrink.update(d_model=1024, d_ff=2048)
    compare(w.with_(**shrink), sizes)


def test_shards_with_empty_and_ragged(cuda_ok):
    w = synth.WORKLOADS[2].with_(T=1000, d_model=512, d_ff=1024)
    compare(w, [0, 448, 0, 552])
    # shards that are not multiples of 64: statistics within fixed-point rounding
    compare(w, [333, 667], exact_stats=False)


def test_shards_renormalized_top2(cuda_ok):
    w = synth.WORKLOADS[4].with_(T=768, d_model=512, d_ff=1024)
    compare(w, [256, 256, 256], renormalize=True)
