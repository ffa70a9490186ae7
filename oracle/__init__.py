"""CPU oracle of the MoE layer (forward pass, routing variants, backward pass) — TEST
INFRASTRUCTURE ONLY.

A plain, slow, single-threaded C++ reference (``moe_oracle.cpp``) with every
accumulation in double, plus this thin ctypes wrapper. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import it.
It shares no code with the CUDA library and never imports it.

Every function follows a passage of the pages (cited in ``moe_oracle.cpp``):
the MoE formula p(x)=softmax(W_r x), y=sum_{e in TopK} p_e E_e(x) of the
DeepSpeed MoE blog; the expert-capacity rule of the Switch/DeepSpeed comparison
article; the PR-MoE residual form of the DeepSpeed-MoE notes; the Switch
load-balance loss of the MoE survey notes; the comparison article's router z-loss
and capacity-by-probability example; the chain rule through all of them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle (g++, -O2, no FMA contraction, single-threaded)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
                    _SRC, "-o", tmp], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = dbl
        L.oracle_round_bf16.argtypes = [dbl]
        L.oracle_round_bf16.restype = ctypes.c_uint16
        L.oracle_gelu.argtypes = [dbl]
        L.oracle_gelu.restype = dbl
        L.oracle_router_logits.argtypes = [vp, i32, i64, i32, vp, vp, i32, vp]
        L.oracle_router_logits.restype = None
        L.oracle_route.argtypes = [vp, i64, i32, i32, vp, vp, vp]
        L.oracle_route.restype = None
        L.oracle_lb_stats.argtypes = [vp, vp, i64, i32, i32, dbl, vp, vp, vp]
        L.oracle_lb_stats.restype = None
        L.oracle_capacity.argtypes = [i64, i32, i32, dbl]
        L.oracle_capacity.restype = i64
        L.oracle_assign_slots.argtypes = [vp, i64, i32, i32, i64, vp, vp]
        L.oracle_assign_slots.restype = None
        L.oracle_ffn.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp]
        L.oracle_ffn.restype = None
        L.oracle_combine.argtypes = [i64, i32, i32, vp, i32, vp, vp, vp, vp, vp]
        L.oracle_combine.restype = None
        L.oracle_assign_slots_priority.argtypes = [vp, vp, i64, i32, i32, i64, vp, vp]
        L.oracle_assign_slots_priority.restype = None
        L.oracle_renormalize_gates.argtypes = [vp, i64, i32]
        L.oracle_renormalize_gates.restype = None
        L.oracle_router_losses.argtypes = [vp, vp, vp, i64, i32, i32, vp, vp, vp]
        L.oracle_router_losses.restype = None
        L.oracle_layer_forward.argtypes = (
            [i64, i32, i32, i32, i32, dbl, i32, i32] + [vp] * 11 + [dbl, vp, vp, i64] + [vp] * 8
            + [i32, i32, i32, vp, vp])
        L.oracle_layer_forward.restype = i64
        L.oracle_gelu_grad.argtypes = [dbl]
        L.oracle_gelu_grad.restype = dbl
        L.oracle_layer_backward.argtypes = (
            [i64, i32, i32, i32, i32, dbl, i32, i32] + [vp] * 11 + [dbl, i32, i32, vp, vp, vp, dbl, dbl]
            + [vp] * 13)
        L.oracle_layer_backward.restype = None
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _is_bf16(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return 1
    assert a.dtype == np.float32, a.dtype
    return 0


def bf16_to_float(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64 via the oracle."""
    f = lib().oracle_bf16_to_double
    return np.array([f(int(b)) for b in np.asarray(bits).ravel()]).reshape(np.shape(bits))


def round_bf16(v) -> np.ndarray:
    """Nearest bf16 (ties to even) of each double, as uint16 bits."""
    f = lib().oracle_round_bf16
    v = np.asarray(v, dtype=np.float64)
    return np.array([f(float(a)) for a in v.ravel()], dtype=np.uint16).reshape(v.shape)


def gelu(z: float) -> float:
    return lib().oracle_gelu(float(z))


def capacity(T: int, E: int, k: int, capacity_factor: float) -> int:
    return int(lib().oracle_capacity(T, E, k, capacity_factor))


def router_logits(x: np.ndarray, w_router: np.ndarray, router_bias: Optional[np.ndarray] = None) -> np.ndarray:
    T, d = x.shape
    E = w_router.shape[0]
    w_router = np.ascontiguousarray(w_router, dtype=np.float32)
    rb = None if router_bias is None else np.ascontiguousarray(router_bias, dtype=np.float32)
    out = np.empty((T, E), dtype=np.float32)
    lib().oracle_router_logits(_p(x), _is_bf16(x), T, d, _p(w_router), _p(rb), E, _p(out))
    return out


def route(logits: np.ndarray, k: int, want_probs: bool = False):
    """(ids [T,k] int32, gates [T,k] f32[, probs [T,E] f64]) from fp32 logits."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    gates = np.empty((T, k), dtype=np.float32)
    probs = np.empty((T, E), dtype=np.float64) if want_probs else None
    lib().oracle_route(_p(logits), T, E, k, _p(ids), _p(gates), _p(probs))
    return (ids, gates, probs) if want_probs else (ids, gates)


def lb_stats(logits: np.ndarray, ids: np.ndarray, alpha: float):
    """(f [E], Q [E], aux) in double."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, E = logits.shape
    k = ids.shape[1]
    f = np.empty(E)
    Q = np.empty(E)
    aux = np.empty(1)
    lib().oracle_lb_stats(_p(logits), _p(ids), T, E, k, alpha, _p(f), _p(Q), _p(aux))
    return f, Q, float(aux[0])


def assign_slots(ids: np.ndarray, E: int, C: int):
    """(slot [T,k] int32 (-1 = dropped), counts [E] int32 demand)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    slot = np.empty((T, k), dtype=np.int32)
    counts = np.empty(E, dtype=np.int32)
    lib().oracle_assign_slots(_p(ids), T, k, E, C, _p(slot), _p(counts))
    return slot, counts


def assign_slots_priority(ids: np.ndarray, probs: np.ndarray, E: int, C: int):
    """Priority overflow: (slot [T,k], counts [E]); ranks each expert's pairs by router
    probability (before any renormalisation) descending, then by pair index."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    probs = np.ascontiguousarray(probs, dtype=np.float32)
    T, k = ids.shape
    slot = np.empty((T, k), dtype=np.int32)
    counts = np.empty(E, dtype=np.int32)
    lib().oracle_assign_slots_priority(_p(ids), _p(probs), T, k, E, C, _p(slot), _p(counts))
    return slot, counts


def renormalize_gates(gates: np.ndarray) -> np.ndarray:
    g = np.array(gates, dtype=np.float32, copy=True, order="C")
    T, k = g.shape
    lib().oracle_renormalize_gates(_p(g), T, k)
    return g


def router_losses(logits: np.ndarray, ids: np.ndarray, gates: np.ndarray):
    """(z_loss, cov2_importance, cov2_load) in double."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    T, E = logits.shape
    k = ids.shape[1]
    out = np.empty(3)
    lib().oracle_router_losses(_p(logits), _p(ids), _p(gates), T, E, k, _p(out[0:1]), _p(out[1:2]),
                               _p(out[2:3]))
    return float(out[0]), float(out[1]), float(out[2])


def ffn(x_row: np.ndarray, w1, b1, w2, b2) -> np.ndarray:
    """One two-layer GeLU FFN on one token row; returns y [d] fp32."""
    d = x_row.shape[-1]
    d_ff = w1.shape[0]
    y = np.empty(d, dtype=np.float32)
    lib().oracle_ffn(_p(np.ascontiguousarray(x_row)), _is_bf16(x_row), d, d_ff, _p(w1), _p(b1),
                     _p(w2), _p(b2), _p(y))
    return y


def combine(gates, slot, y, residual=None, dense=None) -> np.ndarray:
    """out [T,d] double from per-pair expert outputs y [T,k,d] fp32."""
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    y = np.ascontiguousarray(y, dtype=np.float32)
    T, k, d = y.shape
    if dense is not None:
        dense = np.ascontiguousarray(dense, dtype=np.float32)
    out = np.empty((T, d), dtype=np.float64)
    lib().oracle_combine(T, d, k, _p(residual), 0 if residual is None else _is_bf16(residual),
                         _p(dense), _p(gates), _p(slot), _p(y), _p(out))
    return out


def layer_forward(inp: dict, T: int, d_model: int, d_ff: int, E: int, k: int,
                  capacity_factor: float, add_input_residual: bool = True, aux_alpha: float = 0.01,
                  logits_in: Optional[np.ndarray] = None, tokens: Optional[np.ndarray] = None,
                  out_bf16: Optional[bool] = None, overflow_priority: bool = False,
                  renormalize: bool = False, probs_in: Optional[np.ndarray] = None) -> dict:
    """The whole layer on host arrays (``synth.make_inputs`` layout).

    logits_in: [T,E] fp32 logits to route on instead of the oracle's own; probs_in: [T,k] fp32
    softmax probabilities of the chosen experts (before any renormalisation) to rank and gate
    with instead of the oracle's own.

    Returns dict: logits, ids, gates, slot, counts, C, f, Q, aux, out_exact [n,d] f64,
    out (rounded to the output type: uint16 bf16 bits or f32), tokens.
    """
    L = lib()
    x = inp["x"]
    bf16 = _is_bf16(x)
    if out_bf16 is None:
        out_bf16 = bool(bf16)
    n = T if tokens is None else len(tokens)
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    logits = np.empty((T, E), dtype=np.float32)
    ids = np.empty((T, k), dtype=np.int32)
    gates = np.empty((T, k), dtype=np.float32)
    slot = np.empty((T, k), dtype=np.int32)
    counts = np.empty(E, dtype=np.int32)
    stats = np.empty(2 * E + 1, dtype=np.float64)
    out_exact = np.empty((n, d_model), dtype=np.float64)
    out = np.empty((n, d_model), dtype=np.uint16 if out_bf16 else np.float32)
    losses = np.empty(3, dtype=np.float64)
    li = None if logits_in is None else np.ascontiguousarray(logits_in, dtype=np.float32)
    gi = None if probs_in is None else np.ascontiguousarray(probs_in, dtype=np.float32)
    g = inp.get
    C = L.oracle_layer_forward(
        T, d_model, d_ff, E, k, capacity_factor, bf16, int(bool(add_input_residual)),
        _p(x), _p(np.ascontiguousarray(inp["w_router"], dtype=np.float32)), _p(g("router_bias")),
        _p(inp["w1"]), _p(g("b1")), _p(inp["w2"]), _p(g("b2")),
        _p(g("dense_w1")), _p(g("dense_b1")), _p(g("dense_w2")), _p(g("dense_b2")),
        aux_alpha, _p(li), _p(tok), n,
        _p(logits), _p(ids), _p(gates), _p(slot), _p(counts), _p(stats), _p(out_exact), _p(out),
        int(bool(out_bf16)), int(bool(overflow_priority)), int(bool(renormalize)), _p(gi), _p(losses))
    return dict(logits=logits, ids=ids, gates=gates, slot=slot, counts=counts, C=int(C),
                f=stats[:E], Q=stats[E:2 * E], aux=float(stats[2 * E]), out_exact=out_exact,
                out=out, tokens=tok, z_loss=float(losses[0]), cov2_importance=float(losses[1]),
                cov2_load=float(losses[2]))


def gelu_grad(z: float) -> float:
    return lib().oracle_gelu_grad(float(z))


def layer_backward(inp: dict, T: int, d_model: int, d_ff: int, E: int, k: int,
                   capacity_factor: float, dout: np.ndarray, add_input_residual: bool = True,
                   aux_alpha: float = 0.01, aux_weight: float = 0.0, z_weight: float = 0.0,
                   logits_in: Optional[np.ndarray] = None, probs_in: Optional[np.ndarray] = None,
                   overflow_priority: bool = False, renormalize: bool = False) -> dict:
    """Gradients (float64) of L = sum(dout * out) + aux_weight * aux + z_weight * z_loss.

    Returns dict: dx, dw_router, db_router, dw1, db1, dw2, db2, dense_dw1, dense_db1,
    dense_dw2, dense_db2 (dense ones None without the dense MLP), dgates [T,k], dlogits [T,E].
    """
    L = lib()
    x = inp["x"]
    bf16 = _is_bf16(x)
    d, f = d_model, d_ff
    g = inp.get
    dense = g("dense_w1") is not None
    out = dict(dx=np.empty((T, d)), dw_router=np.empty((E, d)), db_router=np.empty(E),
               dw1=np.empty((E, f, d)), db1=np.empty((E, f)), dw2=np.empty((E, d, f)),
               db2=np.empty((E, d)), dgates=np.empty((T, k)), dlogits=np.empty((T, E)))
    out.update(dense_dw1=np.empty((f, d)) if dense else None,
               dense_db1=np.empty(f) if dense else None,
               dense_dw2=np.empty((d, f)) if dense else None,
               dense_db2=np.empty(d) if dense else None)
    li = None if logits_in is None else np.ascontiguousarray(logits_in, dtype=np.float32)
    gi = None if probs_in is None else np.ascontiguousarray(probs_in, dtype=np.float32)
    go = np.ascontiguousarray(dout, dtype=np.float64)
    L.oracle_layer_backward(
        T, d, f, E, k, capacity_factor, bf16, int(bool(add_input_residual)),
        _p(x), _p(np.ascontiguousarray(inp["w_router"], dtype=np.float32)), _p(g("router_bias")),
        _p(inp["w1"]), _p(g("b1")), _p(inp["w2"]), _p(g("b2")),
        _p(g("dense_w1")), _p(g("dense_b1")), _p(g("dense_w2")), _p(g("dense_b2")),
        aux_alpha, int(bool(overflow_priority)), int(bool(renormalize)), _p(li), _p(gi), _p(go),
        aux_weight, z_weight,
        _p(out["dx"]), _p(out["dw_router"]), _p(out["db_router"]), _p(out["dw1"]), _p(out["db1"]),
        _p(out["dw2"]), _p(out["db2"]), _p(out["dense_dw1"]), _p(out["dense_db1"]),
        _p(out["dense_dw2"]), _p(out["dense_db2"]), _p(out["dgates"]), _p(out["dlogits"]))
    return out


def layer_loss(inp: dict, T: int, d_model: int, d_ff: int, E: int, k: int, capacity_factor: float,
               dout: np.ndarray, add_input_residual: bool = True, aux_alpha: float = 0.01,
               aux_weight: float = 0.0, z_weight: float = 0.0, overflow_priority: bool = False,
               renormalize: bool = False) -> float:
    """L = sum(dout * out) + aux_weight * aux + z_weight * z_loss from the forward oracle (the
    objective layer_backward differentiates)."""
    r = layer_forward(inp, T, d_model, d_ff, E, k, capacity_factor,
                      add_input_residual=add_input_residual, aux_alpha=aux_alpha,
                      overflow_priority=overflow_priority, renormalize=renormalize)
    return (float(np.sum(np.asarray(dout, dtype=np.float64) * r["out_exact"]))
            + aux_weight * r["aux"] + z_weight * r["z_loss"])
