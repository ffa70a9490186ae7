"""Seeded synthetic inputs for the MoE layer: the workloads' shapes and value recipes.

This package is shared by the CUDA path's tests/bench and by the CPU oracle's tests.
It holds none of the method's arithmetic (no routing, capacity, FFN or combine):
only the tensors that go in. Everything is drawn on the host by ``moe_synth.c``
(counter-based splitmix64 + Box-Muller), so every element is a pure function of
(seed, stream, index) and any expert's slice can be regenerated on its own.

Workloads (shapes from the GPT+MoE models of the DeepSpeed-MoE notes, §2.1
"MoE based NLG Model Architecture", and the DeepSpeed MoE blog's top-k formula):

====  ==================  ======  =====  =====  ===  =  ====  =====
id    name                T       d      d_ff   E    k  cf    dtype
====  ==================  ======  =====  =====  ===  =  ====  =====
1     tiny-top1-fp32      64      32     64     4    1  1.0   f32
2     gpt350m-moe128      16384   1024   4096   128  1  1.0   bf16
3     gpt1.3b-prmoe128    16384   2048   8192   128  1  1.0   bf16 (+ dense MLP branch)
4     top2-e8-zipf        8192    4096   14336  8    2  1.25  bf16
5     decode-e128         32      2048   8192   128  1  2.0   bf16
====  ==================  ======  =====  =====  ===  =  ====  =====
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_synth.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_synth.so")

# Stream ids: one independent random stream per tensor.
STREAM = {
    "x": 1, "w_router": 2, "router_bias": 3,
    "w1": 4, "b1": 5, "w2": 6, "b2": 7,
    "dense_w1": 8, "dense_b1": 9, "dense_w2": 10, "dense_b2": 11,
    "zipf_perm": 12,
}


def build(force: bool = False) -> str:
    """Compile ``moe_synth.c`` into ``libmoe_synth.so`` (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                    "-ffp-contract=off", _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, i64, i32, dbl, vp = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32,
                                  ctypes.c_double, ctypes.c_void_p)
        L.synth_key.argtypes = [u64, u64]
        L.synth_key.restype = u64
        for name in ("synth_draw_u64", "synth_uniform_f64"):
            getattr(L, name).argtypes = [u64, u64, u64, i64, vp]
            getattr(L, name).restype = None
        for name in ("synth_normal_f64", "synth_normal_f32", "synth_normal_bf16"):
            getattr(L, name).argtypes = [u64, u64, u64, i64, dbl, dbl, vp]
            getattr(L, name).restype = None
        L.synth_permutation.argtypes = [u64, u64, i32, vp]
        L.synth_permutation.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def draw_u64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    lib().synth_draw_u64(seed, stream, offset, n, _ptr(out))
    return out


def uniform(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    lib().synth_uniform_f64(seed, stream, offset, n, _ptr(out))
    return out


def normal(seed: int, stream: int, shape, std: float = 1.0, mean: float = 0.0,
           dtype: str = "f32", offset: int = 0, out: Optional[np.ndarray] = None) -> np.ndarray:
    """N(mean, std^2) samples. dtype 'f64', 'f32' or 'bf16' (bf16 returned as uint16 bits)."""
    shape = tuple(np.atleast_1d(shape).tolist()) if not isinstance(shape, tuple) else shape
    n = int(np.prod(shape)) if len(shape) else 1
    np_dt = {"f64": np.float64, "f32": np.float32, "bf16": np.uint16}[dtype]
    if out is None:
        out = np.empty(shape, dtype=np_dt)
    assert out.dtype == np_dt and out.size == n
    fn = {"f64": lib().synth_normal_f64, "f32": lib().synth_normal_f32,
          "bf16": lib().synth_normal_bf16}[dtype]
    fn(seed, stream, offset, n, float(mean), float(std), _ptr(out))
    return out


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    """A seeded permutation of 1..n."""
    out = np.empty(n, dtype=np.int32)
    lib().synth_permutation(seed, stream, n, _ptr(out))
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic MoE-layer workload."""
    name: str
    T: int
    d_model: int
    d_ff: int
    E: int
    k: int
    capacity_factor: float
    dtype: str                      # "f32" or "bf16" (activations, expert weights, biases)
    x_std: float = 1.0
    w_router_std: float = 0.02
    router_bias: Optional[str] = None   # None | "normal" | "zipf"
    router_bias_std: float = 1.0        # std of the "normal" per-expert logit bias
    zipf_s: float = 1.2                 # exponent of the "zipf" logit bias
    w_std: float = 0.02
    b_std: float = 0.02
    dense: bool = False                 # PR-MoE fixed dense MLP branch
    add_input_residual: bool = True
    aux_alpha: float = 0.01
    seed: int = 5700
    description: str = ""

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    1: Workload("tiny-top1-fp32", T=64, d_model=32, d_ff=64, E=4, k=1, capacity_factor=1.0,
                dtype="f32", x_std=1.0, w_router_std=1.0, w_std=0.1, b_std=0.01, seed=5701,
                description="Tiny top-1 MoE layer, fp32: T=64, d_model=32, E=4, FFN 32->64->32 GeLU "
                            "with biases, capacity_factor=1.0 (capacity 16)"),
    2: Workload("gpt350m-moe128", T=16384, d_model=1024, d_ff=4096, E=128, k=1, capacity_factor=1.0,
                dtype="bf16", w_router_std=0.02, seed=5702,
                description="GPT-350M+MoE-128 shaped layer, bf16 with fp32 router: T=16384 (8x2048), "
                            "d_model=1024, E=128, top-1, FFN 1024->4096->1024 GeLU, capacity_factor=1.0"),
    3: Workload("gpt1.3b-prmoe128", T=16384, d_model=2048, d_ff=8192, E=128, k=1, capacity_factor=1.0,
                dtype="bf16", w_router_std=0.02, router_bias="normal", router_bias_std=1.0,
                dense=True, add_input_residual=False, seed=5703,
                description="GPT-1.3B+MoE-128 PR-MoE layer, bf16: T=16384, d_model=2048, E=128, top-1, "
                            "FFN 2048->8192->2048 GeLU, output = dense MLP + gate*expert, "
                            "per-expert logit bias N(0,1)"),
    4: Workload("top2-e8-zipf", T=8192, d_model=4096, d_ff=14336, E=8, k=2, capacity_factor=1.25,
                dtype="bf16", w_router_std=0.02, router_bias="zipf", zipf_s=1.2, seed=5704,
                description="Top-2 MoE layer, bf16: T=8192, d_model=4096, E=8, FFN 4096->14336->4096 "
                            "GeLU, unrenormalised gates, capacity_factor=1.25, Zipf(1.2) router bias"),
    5: Workload("decode-e128", T=32, d_model=2048, d_ff=8192, E=128, k=1, capacity_factor=2.0,
                dtype="bf16", w_router_std=0.02, seed=5705,
                description="Decode-shaped MoE layer, bf16: T=32 (32 sequences x 1 step), d_model=2048, "
                            "E=128, top-1, FFN 2048->8192->2048 GeLU, capacity_factor=2.0"),
}


def router_bias(w: Workload) -> Optional[np.ndarray]:
    """Per-expert logit bias b_r[E] (float32) or None.

    'normal': N(0, router_bias_std^2). 'zipf': b_e = -s * ln(r_e) with r a seeded
    permutation of 1..E, i.e. the log of a Zipf(s) pmf up to a constant.
    """
    if w.router_bias is None:
        return None
    if w.router_bias == "normal":
        return normal(w.seed, STREAM["router_bias"], (w.E,), std=w.router_bias_std, dtype="f32")
    if w.router_bias == "zipf":
        r = permutation(w.seed, STREAM["zipf_perm"], w.E).astype(np.float64)
        return (-w.zipf_s * np.log(r)).astype(np.float32)
    raise ValueError(w.router_bias)


def make_inputs(w: Workload, experts_only: bool = False) -> dict:
    """All host-side inputs of a workload as numpy arrays (bf16 as uint16 bits).

    Keys: x [T,d], w_router [E,d] f32, router_bias [E] f32|None, w1 [E,d_ff,d],
    b1 [E,d_ff], w2 [E,d,d_ff], b2 [E,d], and dense_w1 [d_ff,d], dense_b1 [d_ff],
    dense_w2 [d,d_ff], dense_b2 [d] when the workload has the dense branch.
    """
    dt = w.dtype
    T, d, f, E = w.T, w.d_model, w.d_ff, w.E
    out = {}
    if not experts_only:
        out["x"] = normal(w.seed, STREAM["x"], (T, d), std=w.x_std, dtype=dt)
        out["w_router"] = normal(w.seed, STREAM["w_router"], (E, d), std=w.w_router_std, dtype="f32")
        out["router_bias"] = router_bias(w)
    out["w1"] = normal(w.seed, STREAM["w1"], (E, f, d), std=w.w_std, dtype=dt)
    out["b1"] = normal(w.seed, STREAM["b1"], (E, f), std=w.b_std, dtype=dt)
    out["w2"] = normal(w.seed, STREAM["w2"], (E, d, f), std=w.w_std, dtype=dt)
    out["b2"] = normal(w.seed, STREAM["b2"], (E, d), std=w.b_std, dtype=dt)
    if w.dense:
        out["dense_w1"] = normal(w.seed, STREAM["dense_w1"], (f, d), std=w.w_std, dtype=dt)
        out["dense_b1"] = normal(w.seed, STREAM["dense_b1"], (f,), std=w.b_std, dtype=dt)
        out["dense_w2"] = normal(w.seed, STREAM["dense_w2"], (d, f), std=w.w_std, dtype=dt)
        out["dense_b2"] = normal(w.seed, STREAM["dense_b2"], (d,), std=w.b_std, dtype=dt)
    return out
