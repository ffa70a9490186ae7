"""Shared helpers of the GPU parity tests: device copies of the synthetic inputs, one call of the
layer through the C ABI, and the output tolerances.

Tolerances (floating-point outputs; integer routing/dispatch results are compared bit-exactly):
  * fp32 layers: max |out - oracle| <= 1e-5 (absolute, outputs are O(1)).
  * bf16 layers, parity run with fp32 output: max-abs <= 2e-2 and relative L2 <= 1e-2.
  * bf16 layers, bf16 output: |out - oracle| <= 2e-2 + half a bf16 ulp of |oracle| per element,
    and relative L2 <= 1e-2 (rounding the output to bf16 alone costs up to half an ulp, which
    exceeds 2e-2 once |out| >= 4).
"""
from __future__ import annotations

import numpy as np
import torch

import synth
from mixture_experts_layer_57_b200 import moe

FP32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_REL_L2 = 1e-2


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """Host array (bf16 as uint16 bits, or f32/int32) -> device tensor of the same values."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> host array (bf16 as uint16 bits)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def as_f64(a: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def dev_inputs(inp: dict, device="cuda") -> dict:
    return {k: (to_dev(v, device) if isinstance(v, np.ndarray) else v) for k, v in inp.items()}


def run_layer(w: synth.Workload, d_inp: dict, out_dtype=None, add_input_residual=None,
              ws: torch.Tensor = None, overflow_priority: bool = False, renormalize: bool = False,
              want_losses: bool = False, w_router_prepared=None) -> dict:
    """One moe_layer_forward on device inputs; returns host copies of every output."""
    T, E, k = w.T, w.E, w.k
    x = d_inp["x"]
    dense = None
    if w.dense:
        dense = (d_inp["dense_w1"], d_inp["dense_b1"], d_inp["dense_w2"], d_inp["dense_b2"])
    res = w.add_input_residual if add_input_residual is None else add_input_residual
    args = moe.layer_args(x, d_inp["w_router"], d_inp["w1"], d_inp["b1"], d_inp["w2"], d_inp["b2"],
                          k=k, capacity_factor=w.capacity_factor, router_bias=d_inp.get("router_bias"),
                          dense=dense, add_input_residual=res, aux_alpha=w.aux_alpha,
                          out_dtype=out_dtype, overflow_priority=overflow_priority,
                          renormalize_gates=renormalize, w_router_prepared=w_router_prepared)
    dev = x.device
    aux = dict(logits=torch.empty(T, E, dtype=torch.float32, device=dev),
               expert_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               gates=torch.empty(T, k, dtype=torch.float32, device=dev),
               slot=torch.empty(T, k, dtype=torch.int32, device=dev),
               expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
               expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               lb_stats=torch.empty(2 * E + 1, dtype=torch.float32, device=dev),
               topk_probs=torch.empty(T, k, dtype=torch.float32, device=dev))
    if want_losses:
        aux["router_losses"] = torch.empty(3, dtype=torch.float32, device=dev)
    odt = x.dtype if out_dtype is None else out_dtype
    out = torch.empty(T, w.d_model, dtype=odt, device=dev)
    if ws is None:
        ws = moe.workspace(moe.moe_layer_workspace_bytes(args), dev)
    moe.moe_layer_forward(args, out, aux=aux, ws=ws)
    err = moe.moe_get_device_error(ws)
    r = {name: to_host(t) for name, t in aux.items()}
    r["out"] = to_host(out)
    r["device_error"] = err
    r["launches"] = moe.moe_last_launch_count()
    return r


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 values around |v| (8 significant bits)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def check_out(got: np.ndarray, ref: np.ndarray, layer_bf16: bool, out_bf16: bool, what=""):
    """Assert the output tolerances; returns (max_abs, rel_l2)."""
    g = as_f64(got)
    diff = np.abs(g - ref)
    max_abs = float(diff.max()) if diff.size else 0.0
    rel = float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)) if diff.size else 0.0
    if not layer_bf16:
        assert max_abs <= FP32_ATOL, f"{what}: fp32 max-abs {max_abs}"
    elif not out_bf16:
        assert max_abs <= BF16_ATOL, f"{what}: max-abs {max_abs}"
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel}"
    else:
        tol = BF16_ATOL + bf16_half_ulp(ref)
        bad = diff > tol
        assert not bad.any(), f"{what}: {bad.sum()} elements beyond 2e-2 + half ulp (max {max_abs})"
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel}"
    return max_abs, rel


def oracle_layer(inp: dict, w: synth.Workload, tokens=None, threads: int = 0, **kw) -> dict:
    """oracle.layer_forward of the workload, the output rows of `tokens` (None = all) computed by
    several independent oracle calls on chunks of the tokens in parallel threads (the oracle's C
    code runs outside the interpreter lock; each call routes the whole batch itself, so every
    chunk sees the same routing). Returns layer_forward's dict for the requested tokens."""
    import concurrent.futures as cf
    import os

    import oracle
    tok = np.arange(w.T, dtype=np.int64) if tokens is None else np.asarray(tokens, dtype=np.int64)
    n_thr = threads or max(1, min(16, (os.cpu_count() or 1), len(tok)))
    common = dict(add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha)
    common.update(kw)
    if n_thr == 1 or len(tok) < 2:
        return oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                                    tokens=tok, **common)
    chunks = [c for c in np.array_split(tok, n_thr) if len(c)]
    with cf.ThreadPoolExecutor(len(chunks)) as ex:
        parts = list(ex.map(lambda c: oracle.layer_forward(
            inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor, tokens=c, **common), chunks))
    r = dict(parts[0])
    r["out_exact"] = np.concatenate([p["out_exact"] for p in parts])
    r["out"] = np.concatenate([p["out"] for p in parts])
    r["tokens"] = tok
    return r


def spread_tokens(w: synth.Workload, ids: np.ndarray, slot: np.ndarray, n_min: int,
                  rng: np.random.Generator, tile: int = 128) -> np.ndarray:
    """Output rows to compare on a full-size workload: a kept token of every expert that keeps
    one, the first and last kept tokens of the largest segments and those on each side of a
    token-tile boundary inside them, dropped tokens and (k > 1) partially dropped ones, the first
    and last token, then random kept tokens up to n_min."""
    T, k = ids.shape
    pick = {0, T - 1}
    kept_pair = slot >= 0
    for e in np.unique(ids[kept_pair]):
        t_e = np.nonzero((ids == e) & kept_pair)[0]
        pick.add(int(rng.choice(t_e)))
    sizes = [(int(((ids == e) & kept_pair).sum()), e) for e in np.unique(ids)]
    for _, e in sorted(sizes, reverse=True)[:4]:
        # kept tokens of e in packed-row order (slot order)
        t_e, j_e = np.nonzero((ids == e) & kept_pair)
        order = t_e[np.argsort(slot[t_e, j_e], kind="stable")]
        pick.update(int(order[i]) for i in (0, len(order) - 1))
        for b in range(tile, len(order), tile):
            pick.update(int(order[i]) for i in (b - 1, b))
    dropped = np.nonzero((~kept_pair).all(1))[0]
    partial = np.nonzero((~kept_pair).any(1) & kept_pair.any(1))[0]
    for group in (dropped, partial):
        if len(group):
            pick.update(int(t) for t in rng.choice(group, min(len(group), 16), replace=False))
    kept = np.setdiff1d(np.nonzero(kept_pair.all(1))[0], np.array(sorted(pick), dtype=np.int64))
    need = n_min - len(pick)
    if need > 0 and len(kept):
        pick.update(int(t) for t in rng.choice(kept, min(len(kept), need), replace=False))
    return np.array(sorted(pick), dtype=np.int64)
