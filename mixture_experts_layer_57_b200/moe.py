"""Thin Python binding of the C ABI in ``include/moe.h`` (``libmoe.so``).

The functions carry the C entry points' names and only marshal arguments: torch tensors become
device pointers, missing outputs and workspaces are allocated with ``torch.empty``/``zeros`` on
the tensors' device, and the current CUDA stream is passed. Every step of the computation runs
in the library's kernels; there is no fallback: if ``libmoe.so`` is missing or no CUDA device is
present the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "moe.h")

MOE_F32, MOE_BF16 = 0, 1
MOE_EPILOGUE_BIAS_GELU, MOE_EPILOGUE_BIAS = 0, 1
MOE_OVERFLOW_FIRST_COME, MOE_OVERFLOW_PRIORITY = 0, 1
STATUS_BLOCK_BYTES = 256
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARGUMENT", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_FLAG",
                6: "MOE_ERR_MISALIGNED"}
DEVICE_ERRORS = {0: "MOE_DEVERR_NONE", 1: "MOE_DEVERR_TIMEOUT", 2: "MOE_DEVERR_BAD_EXPERT",
                 3: "MOE_DEVERR_BAD_OFFSETS", 4: "MOE_DEVERR_BAD_ROW"}


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")


class LayerArgs(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("capacity_factor", ctypes.c_double),
                ("dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("x", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p), ("dense_w1", ctypes.c_void_p),
                ("dense_b1", ctypes.c_void_p), ("dense_w2", ctypes.c_void_p),
                ("dense_b2", ctypes.c_void_p), ("add_input_residual", ctypes.c_int),
                ("aux_alpha", ctypes.c_float), ("overflow_policy", ctypes.c_int),
                ("renormalize_gates", ctypes.c_int), ("w_router_prepared", ctypes.c_void_p)]


class LayerAux(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("expert_ids", ctypes.c_void_p),
                ("gates", ctypes.c_void_p), ("slot", ctypes.c_void_p),
                ("expert_counts", ctypes.c_void_p), ("expert_offsets", ctypes.c_void_p),
                ("lb_stats", ctypes.c_void_p), ("router_losses", ctypes.c_void_p),
                ("topk_probs", ctypes.c_void_p)]


class LayerGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "dx", "dw_router", "db_router", "dw1", "db1", "dw2", "db2", "dense_dw1", "dense_db1",
        "dense_dw2", "dense_db2", "dgates", "dlogits")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load ``libmoe.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixture_experts_layer_57_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f32, f64, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                      ctypes.c_double, ctypes.c_size_t)
        P = ctypes.POINTER
        sig = {
            "moe_status_string": ([i32], ctypes.c_char_p),
            "moe_abi_version": ([], i32),
            "moe_last_launch_count": ([], i32),
            "moe_capacity": ([i64, i32, i32, f64, P(i64)], i32),
            "moe_packed_rows_max": ([i64, i32, i32, i64, P(i64)], i32),
            "moe_router_workspace_bytes": ([i64, i32, i32, P(sz)], i32),
            "moe_router_prepare_bytes": ([i32, i32, P(sz)], i32),
            "moe_router_prepare": ([vp, i32, i32, vp, sz, vp], i32),
            "moe_router_topk": ([vp, i32, i64, i32, vp, vp, i32, i32, vp, vp, vp, vp, f32, vp, sz, vp], i32),
            "moe_router_topk_ex": ([vp, i32, i64, i32, vp, vp, i32, i32, vp, vp, vp, vp, f32, i32, vp,
                                    vp, vp, sz, vp], i32),
            "moe_dispatch_workspace_bytes": ([i64, i32, i32, P(sz)], i32),
            "moe_dispatch": ([vp, i32, i64, i32, vp, i32, i32, i64, vp, vp, vp, vp, vp, i64, vp, sz, vp], i32),
            "moe_dispatch_priority": ([vp, i32, i64, i32, vp, vp, i32, i32, i64, vp, vp, vp, vp, vp, i64,
                                       vp, sz, vp], i32),
            "moe_dispatch_noalloc": ([vp, i32, i64, i32, vp, i32, i32, i64, vp, vp, vp, vp, vp, i64, vp], i32),
            "moe_expert_ffn_workspace_bytes": ([P(sz)], i32),
            "moe_expert_ffn": ([vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, vp, vp, vp, i64, vp, sz, vp], i32),
            "moe_grouped_gemm": ([vp, vp, i32, i64, i32, i32, i32, vp, vp, i32, vp, i64, vp, sz, vp], i32),
            "moe_combine_workspace_bytes": ([P(sz)], i32),
            "moe_combine": ([vp, vp, vp, vp, vp, i64, i32, i32, i32, i64, vp, i32, vp, vp, i32, vp, sz, vp], i32),
            "moe_layer_workspace_bytes": ([P(LayerArgs), P(sz)], i32),
            "moe_layer_forward": ([P(LayerArgs), vp, P(LayerAux), vp, sz, vp], i32),
            "moe_layer_forward_profiled": ([P(LayerArgs), vp, P(LayerAux), vp, sz, vp,
                                            P(vp), i32, P(i32), ctypes.c_char_p, sz], i32),
            "moe_layer_shard_workspace_bytes": ([P(LayerArgs), i64, P(sz)], i32),
            "moe_router_partials_count": ([i32], i64),
            "moe_layer_forward_shard_begin": ([P(LayerArgs), i64, P(LayerAux), vp, vp, vp, sz, vp], i32),
            "moe_layer_forward_shard_end": ([P(LayerArgs), i64, i32, i32, vp, vp, vp, P(LayerAux), vp,
                                             sz, vp], i32),
            "moe_layer_train_workspace_bytes": ([P(LayerArgs), P(sz)], i32),
            "moe_layer_forward_train": ([P(LayerArgs), vp, P(LayerAux), vp, sz, vp], i32),
            "moe_layer_backward": ([P(LayerArgs), vp, f32, f32, P(LayerGrads), vp, sz, vp], i32),
            "moe_workspace_reset": ([vp, sz, vp], i32),
            "moe_get_device_error": ([vp, P(i32), vp], i32),
            "moe_selftest_bounded_wait": ([vp, sz, ctypes.c_uint64, vp], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def header_symbols() -> list:
    """Names of the functions ``include/moe.h`` declares."""
    import re
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|int64_t|int|moe_status)\s+(moe_\w+)\s*\(", text, re.M)))


def _check(fn: str, status: int):
    if status != 0:
        raise MoEError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _torch_dt(code: int):
    return torch.bfloat16 if code == MOE_BF16 else torch.float32


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed workspace (status block cleared) of at least nbytes."""
    return torch.zeros(max(int(nbytes), STATUS_BLOCK_BYTES), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- sizes

def moe_capacity(T: int, E: int, k: int, capacity_factor: float) -> int:
    out = ctypes.c_int64()
    _check("moe_capacity", lib().moe_capacity(T, E, k, capacity_factor, ctypes.byref(out)))
    return out.value


def moe_packed_rows_max(T: int, E: int, k: int, C: int) -> int:
    out = ctypes.c_int64()
    _check("moe_packed_rows_max", lib().moe_packed_rows_max(T, E, k, C, ctypes.byref(out)))
    return out.value


def _ws_bytes(fn: str, *args) -> int:
    out = ctypes.c_size_t()
    _check(fn, getattr(lib(), fn)(*args, ctypes.byref(out)))
    return out.value


def moe_router_prepare(w_router: torch.Tensor, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """The router weight split for the tensor-core logits kernel (pass it to layer_args as
    w_router_prepared; prepare again whenever w_router changes)."""
    E, d = w_router.shape
    n = ctypes.c_size_t()
    _check("moe_router_prepare_bytes", lib().moe_router_prepare_bytes(E, d, ctypes.byref(n)))
    if out is None:
        out = torch.empty(n.value, dtype=torch.uint8, device=w_router.device)
    _check("moe_router_prepare", lib().moe_router_prepare(_ptr(w_router), E, d, _ptr(out),
                                                          out.numel(), _stream(stream)))
    return out


def moe_router_workspace_bytes(T, E, d_model):
    return _ws_bytes("moe_router_workspace_bytes", T, E, d_model)


def moe_dispatch_workspace_bytes(T, E, k):
    return _ws_bytes("moe_dispatch_workspace_bytes", T, E, k)


def moe_expert_ffn_workspace_bytes():
    return _ws_bytes("moe_expert_ffn_workspace_bytes")


def moe_combine_workspace_bytes():
    return _ws_bytes("moe_combine_workspace_bytes")


# ---------------------------------------------------------------- entry points

def moe_router_topk(x: torch.Tensor, w_router: torch.Tensor, k: int,
                    router_bias: Optional[torch.Tensor] = None, logits=None, expert_ids=None,
                    gates=None, lb_stats=None, aux_alpha: float = 0.01, want_stats: bool = True,
                    ws: Optional[torch.Tensor] = None, stream=None, renormalize: bool = False,
                    router_losses=None, probs=None) -> dict:
    """moe_router_topk, or moe_router_topk_ex when ``renormalize`` is set or ``router_losses``
    (a [3] fp32 tensor, or True to allocate one) or ``probs`` (a [T, k] fp32 tensor, or True:
    the probabilities before renormalisation) is given."""
    T, d = x.shape
    E = w_router.shape[0]
    dev = x.device
    if logits is None:
        logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    if expert_ids is None:
        expert_ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    if gates is None:
        gates = torch.empty(T, k, dtype=torch.float32, device=dev)
    if lb_stats is None and want_stats:
        lb_stats = torch.empty(2 * E + 1, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(moe_router_workspace_bytes(T, E, d), dev)
    if router_losses is True:
        router_losses = torch.empty(3, dtype=torch.float32, device=dev)
    if probs is True:
        probs = torch.empty(T, k, dtype=torch.float32, device=dev)
    if renormalize or router_losses is not None or probs is not None:
        _check("moe_router_topk_ex", lib().moe_router_topk_ex(
            _ptr(x), _dt(x), T, d, _ptr(w_router), _ptr(router_bias), E, k, _ptr(logits),
            _ptr(expert_ids), _ptr(gates), _ptr(lb_stats), aux_alpha, int(bool(renormalize)),
            _ptr(router_losses), _ptr(probs), _ptr(ws), ws.numel(), _stream(stream)))
    else:
        _check("moe_router_topk", lib().moe_router_topk(
            _ptr(x), _dt(x), T, d, _ptr(w_router), _ptr(router_bias), E, k, _ptr(logits),
            _ptr(expert_ids), _ptr(gates), _ptr(lb_stats), aux_alpha, _ptr(ws), ws.numel(),
            _stream(stream)))
    return dict(logits=logits, expert_ids=expert_ids, gates=gates, lb_stats=lb_stats, ws=ws,
                router_losses=router_losses, probs=probs)


def moe_dispatch(x: torch.Tensor, expert_ids: torch.Tensor, E: int, C: int, rows_max=None,
                 slot=None, expert_counts=None, expert_offsets=None, row_token=None, x_packed=None,
                 ws=None, stream=None, priority_probs: Optional[torch.Tensor] = None) -> dict:
    """moe_dispatch, or moe_dispatch_priority when ``priority_probs`` ([T, k] fp32 router
    probabilities before any renormalisation) is given."""
    T, d = x.shape
    k = expert_ids.shape[1]
    dev = x.device
    if rows_max is None:
        rows_max = moe_packed_rows_max(T, E, k, C)
    if slot is None:
        slot = torch.empty(T, k, dtype=torch.int32, device=dev)
    if expert_counts is None:
        expert_counts = torch.empty(E, dtype=torch.int32, device=dev)
    if expert_offsets is None:
        expert_offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty(max(rows_max, 1), dtype=torch.int32, device=dev)
    if x_packed is None:
        x_packed = torch.empty(max(rows_max, 1), d, dtype=x.dtype, device=dev)
    if ws is None:
        ws = workspace(moe_dispatch_workspace_bytes(T, E, k), dev)
    if priority_probs is not None:
        _check("moe_dispatch_priority", lib().moe_dispatch_priority(
            _ptr(x), _dt(x), T, d, _ptr(expert_ids), _ptr(priority_probs), E, k, C, _ptr(slot),
            _ptr(expert_counts), _ptr(expert_offsets), _ptr(row_token), _ptr(x_packed), rows_max,
            _ptr(ws), ws.numel(), _stream(stream)))
    else:
        _check("moe_dispatch", lib().moe_dispatch(
            _ptr(x), _dt(x), T, d, _ptr(expert_ids), E, k, C, _ptr(slot), _ptr(expert_counts),
            _ptr(expert_offsets), _ptr(row_token), _ptr(x_packed), rows_max, _ptr(ws), ws.numel(),
            _stream(stream)))
    return dict(slot=slot, expert_counts=expert_counts, expert_offsets=expert_offsets,
                row_token=row_token, x_packed=x_packed, rows_max=rows_max, ws=ws)


def moe_dispatch_noalloc(x: torch.Tensor, expert_ids: torch.Tensor, E: int, C: int, rows_max=None,
                         slot=None, expert_counts=None, expert_offsets=None, row_token=None,
                         x_packed=None, stream=None) -> dict:
    """moe_dispatch without a workspace: the library's built-in static scratch is used (for
    callers that cannot allocate; the outputs here are still allocated by torch when omitted)."""
    T, d = x.shape
    k = expert_ids.shape[1]
    dev = x.device
    if rows_max is None:
        rows_max = moe_packed_rows_max(T, E, k, C)
    if slot is None:
        slot = torch.empty(T, k, dtype=torch.int32, device=dev)
    if expert_counts is None:
        expert_counts = torch.empty(E, dtype=torch.int32, device=dev)
    if expert_offsets is None:
        expert_offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty(max(rows_max, 1), dtype=torch.int32, device=dev)
    if x_packed is None:
        x_packed = torch.empty(max(rows_max, 1), d, dtype=x.dtype, device=dev)
    _check("moe_dispatch_noalloc", lib().moe_dispatch_noalloc(
        _ptr(x), _dt(x), T, d, _ptr(expert_ids), E, k, C, _ptr(slot), _ptr(expert_counts),
        _ptr(expert_offsets), _ptr(row_token), _ptr(x_packed), rows_max, _stream(stream)))
    return dict(slot=slot, expert_counts=expert_counts, expert_offsets=expert_offsets,
                row_token=row_token, x_packed=x_packed, rows_max=rows_max)


def moe_expert_ffn(x_packed: torch.Tensor, expert_offsets: torch.Tensor, w1, b1, w2, b2,
                   rows_max=None, capacity_hint=None, h_packed=None, y_packed=None, ws=None,
                   stream=None) -> dict:
    E, d_ff, d = w1.shape
    dev = x_packed.device
    if rows_max is None:
        rows_max = x_packed.shape[0]
    if capacity_hint is None:
        capacity_hint = rows_max
    if h_packed is None:
        h_packed = torch.empty(max(rows_max, 1), d_ff, dtype=x_packed.dtype, device=dev)
    if y_packed is None:
        y_packed = torch.empty(max(rows_max, 1), d, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(moe_expert_ffn_workspace_bytes(), dev)
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        _ptr(x_packed), _ptr(expert_offsets), E, rows_max, d, d_ff, _dt(x_packed), _ptr(w1), _ptr(b1),
        _ptr(w2), _ptr(b2), _ptr(h_packed), _ptr(y_packed), capacity_hint, _ptr(ws), ws.numel(),
        _stream(stream)))
    return dict(h_packed=h_packed, y_packed=y_packed, ws=ws)


def moe_grouped_gemm(x_packed: torch.Tensor, expert_offsets: torch.Tensor, w: torch.Tensor, bias=None,
                     gelu: bool = True, rows_max=None, capacity_hint=None, out=None, ws=None,
                     stream=None) -> dict:
    """One grouped GEMM layer: out = GeLU(W[e] x + b[e]) (input dtype) or W[e] x + b[e] (fp32)."""
    E, N, K = w.shape
    dev = x_packed.device
    if rows_max is None:
        rows_max = x_packed.shape[0]
    if capacity_hint is None:
        capacity_hint = rows_max
    if out is None:
        out = torch.empty(max(rows_max, 1), N, dtype=x_packed.dtype if gelu else torch.float32,
                          device=dev)
    if ws is None:
        ws = workspace(moe_expert_ffn_workspace_bytes(), dev)
    _check("moe_grouped_gemm", lib().moe_grouped_gemm(
        _ptr(x_packed), _ptr(expert_offsets), E, rows_max, K, N, _dt(x_packed), _ptr(w), _ptr(bias),
        MOE_EPILOGUE_BIAS_GELU if gelu else MOE_EPILOGUE_BIAS, _ptr(out), capacity_hint, _ptr(ws),
        ws.numel(), _stream(stream)))
    return dict(out=out, ws=ws)


def moe_combine(y_packed: torch.Tensor, expert_offsets, expert_ids, slot, gates, residual=None,
                dense=None, out=None, out_dtype=None, rows_max=None, ws=None, stream=None) -> dict:
    T, k = expert_ids.shape
    d = y_packed.shape[1]
    E = expert_offsets.shape[0] - 1
    dev = y_packed.device
    if rows_max is None:
        rows_max = y_packed.shape[0]
    if out_dtype is None:
        out_dtype = residual.dtype if residual is not None else torch.float32
    if out is None:
        out = torch.empty(T, d, dtype=out_dtype, device=dev)
    if ws is None:
        ws = workspace(moe_combine_workspace_bytes(), dev)
    _check("moe_combine", lib().moe_combine(
        _ptr(y_packed), _ptr(expert_offsets), _ptr(expert_ids), _ptr(slot), _ptr(gates), T, d, E, k,
        rows_max, _ptr(residual), _dt(residual) if residual is not None else MOE_F32, _ptr(dense),
        _ptr(out), _dt(out), _ptr(ws), ws.numel(), _stream(stream)))
    return dict(out=out, ws=ws)


def layer_args(x, w_router, w1, b1, w2, b2, k: int, capacity_factor: float, router_bias=None,
               dense=None, add_input_residual: bool = True, aux_alpha: float = 0.01,
               out_dtype=None, overflow_priority: bool = False,
               renormalize_gates: bool = False, w_router_prepared=None) -> LayerArgs:
    """Fill a ``moe_layer_args`` struct from tensors (dense = (w1, b1, w2, b2) or None)."""
    T, d = x.shape
    E, d_ff, _ = w1.shape
    dw = dense if dense is not None else (None, None, None, None)
    return LayerArgs(T=T, d_model=d, d_ff=d_ff, E=E, k=k, capacity_factor=capacity_factor,
                     dtype=_dt(x), out_dtype=_dt(x) if out_dtype is None else
                     (MOE_BF16 if out_dtype == torch.bfloat16 else MOE_F32),
                     x=_ptr(x), w_router=_ptr(w_router), router_bias=_ptr(router_bias),
                     w1=_ptr(w1), b1=_ptr(b1), w2=_ptr(w2), b2=_ptr(b2),
                     dense_w1=_ptr(dw[0]), dense_b1=_ptr(dw[1]), dense_w2=_ptr(dw[2]),
                     dense_b2=_ptr(dw[3]), add_input_residual=int(bool(add_input_residual)),
                     aux_alpha=aux_alpha,
                     overflow_policy=MOE_OVERFLOW_PRIORITY if overflow_priority else
                     MOE_OVERFLOW_FIRST_COME,
                     renormalize_gates=int(bool(renormalize_gates)),
                     w_router_prepared=_ptr(w_router_prepared))


def moe_layer_workspace_bytes(args: LayerArgs) -> int:
    out = ctypes.c_size_t()
    _check("moe_layer_workspace_bytes", lib().moe_layer_workspace_bytes(ctypes.byref(args), ctypes.byref(out)))
    return out.value


def moe_layer_forward(args: LayerArgs, out: torch.Tensor, aux: Optional[dict] = None,
                      ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Run the whole layer into ``out``; ``aux`` may map LayerAux field names to tensors."""
    if ws is None:
        ws = workspace(moe_layer_workspace_bytes(args), out.device)
    a = LayerAux()
    if aux:
        for name, t in aux.items():
            setattr(a, name, _ptr(t))
    _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(args), _ptr(out), ctypes.byref(a), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def moe_layer_forward_profiled(args: LayerArgs, out: torch.Tensor, events: list, aux=None, ws=None,
                               stream=None):
    """moe_layer_forward recording ``events`` (torch.cuda.Event(enable_timing=True)) at stage
    boundaries; returns the list of stage labels, starting with "start"."""
    if ws is None:
        ws = workspace(moe_layer_workspace_bytes(args), out.device)
    for ev in events:
        if ev.cuda_event == 0:
            ev.record()   # create the underlying CUDA event
    a = LayerAux()
    if aux:
        for name, t in aux.items():
            setattr(a, name, _ptr(t))
    handles = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    n = ctypes.c_int()
    names = ctypes.create_string_buffer(512)
    _check("moe_layer_forward_profiled", lib().moe_layer_forward_profiled(
        ctypes.byref(args), _ptr(out), ctypes.byref(a), _ptr(ws), ws.numel(), _stream(stream),
        handles, len(events), ctypes.byref(n), names, 512))
    return names.value.decode().split(",")[: n.value]


def _aux_struct(aux: Optional[dict]) -> LayerAux:
    a = LayerAux()
    if aux:
        for name, t in aux.items():
            setattr(a, name, _ptr(t))
    return a


def moe_layer_shard_workspace_bytes(args: LayerArgs, T_global: int) -> int:
    out = ctypes.c_size_t()
    _check("moe_layer_shard_workspace_bytes",
           lib().moe_layer_shard_workspace_bytes(ctypes.byref(args), T_global, ctypes.byref(out)))
    return out.value


def moe_router_partials_count(E: int) -> int:
    return int(lib().moe_router_partials_count(E))


def moe_layer_forward_shard_begin(args: LayerArgs, T_global: int, demand: torch.Tensor,
                                  stat_partials: torch.Tensor, aux: Optional[dict] = None,
                                  ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """First half of a token shard's layer: writes ``demand`` [E] int32 and ``stat_partials``
    [4E+1] int64; returns the workspace, which the second half must get unchanged."""
    if ws is None:
        ws = workspace(moe_layer_shard_workspace_bytes(args, T_global), demand.device)
    _check("moe_layer_forward_shard_begin", lib().moe_layer_forward_shard_begin(
        ctypes.byref(args), T_global, ctypes.byref(_aux_struct(aux)), _ptr(demand),
        _ptr(stat_partials), _ptr(ws), ws.numel(), _stream(stream)))
    return ws


def moe_layer_forward_shard_end(args: LayerArgs, T_global: int, G: int, rank: int,
                                demand_all: torch.Tensor, stat_totals: torch.Tensor,
                                out: torch.Tensor, ws: torch.Tensor, aux: Optional[dict] = None,
                                stream=None) -> torch.Tensor:
    """Second half: dispatch with the global slot base, expert FFN and combine into ``out``."""
    _check("moe_layer_forward_shard_end", lib().moe_layer_forward_shard_end(
        ctypes.byref(args), T_global, G, rank, _ptr(demand_all), _ptr(stat_totals), _ptr(out),
        ctypes.byref(_aux_struct(aux)), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def exchange_shard_routing(demand: torch.Tensor, stat_partials: torch.Tensor, group=None):
    """The one exchange step of the token-sharded layer: every shard's demand gathered in rank
    order ([G, E] int32) and the statistics partials summed over shards (int64, exact)."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    demand_all = torch.empty(G, demand.numel(), dtype=demand.dtype, device=demand.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(demand_all, demand, group=group)
    else:
        dist.all_gather(list(demand_all.unbind(0)), demand, group=group)
    totals = stat_partials.clone()
    dist.all_reduce(totals, op=dist.ReduceOp.SUM, group=group)
    return demand_all, totals


def moe_layer_forward_sharded(args: LayerArgs, T_global: int, out: torch.Tensor, group=None,
                              aux: Optional[dict] = None, ws: Optional[torch.Tensor] = None,
                              stream=None) -> torch.Tensor:
    """The token-sharded layer on this rank (tokens of the ranks in rank order make the batch of
    ``T_global``): begin, the exchange over ``group``, end."""
    import torch.distributed as dist
    E = args.E
    dev = out.device
    demand = torch.empty(E, dtype=torch.int32, device=dev)
    partials = torch.empty(moe_router_partials_count(E), dtype=torch.int64, device=dev)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    with torch.cuda.stream(s):  # the collectives run on the same stream as the kernels
        ws = moe_layer_forward_shard_begin(args, T_global, demand, partials, aux=aux, ws=ws,
                                           stream=s)
        demand_all, totals = exchange_shard_routing(demand, partials, group)
        return moe_layer_forward_shard_end(args, T_global, dist.get_world_size(group),
                                           dist.get_rank(group), demand_all, totals, out, ws,
                                           aux=aux, stream=s)


def moe_layer_train_workspace_bytes(args: LayerArgs) -> int:
    out = ctypes.c_size_t()
    _check("moe_layer_train_workspace_bytes",
           lib().moe_layer_train_workspace_bytes(ctypes.byref(args), ctypes.byref(out)))
    return out.value


def moe_layer_forward_train(args: LayerArgs, out: torch.Tensor, aux: Optional[dict] = None,
                            ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Forward pass that keeps the backward pass's state in the returned workspace."""
    if ws is None:
        ws = workspace(moe_layer_train_workspace_bytes(args), out.device)
    _check("moe_layer_forward_train", lib().moe_layer_forward_train(
        ctypes.byref(args), _ptr(out), ctypes.byref(_aux_struct(aux)), _ptr(ws), ws.numel(),
        _stream(stream)))
    return ws


def moe_layer_backward(args: LayerArgs, d_out: torch.Tensor, grads: dict, ws: torch.Tensor,
                       aux_weight: float = 0.0, z_weight: float = 0.0, stream=None) -> dict:
    """Backward pass after moe_layer_forward_train with the same args and workspace. ``grads``
    maps moe_layer_grads field names to output tensors."""
    g = LayerGrads()
    for name, t in grads.items():
        setattr(g, name, _ptr(t))
    _check("moe_layer_backward", lib().moe_layer_backward(
        ctypes.byref(args), _ptr(d_out), aux_weight, z_weight, ctypes.byref(g), _ptr(ws),
        ws.numel(), _stream(stream)))
    return grads


def moe_workspace_reset(ws: torch.Tensor, stream=None):
    _check("moe_workspace_reset", lib().moe_workspace_reset(_ptr(ws), ws.numel(), _stream(stream)))


def moe_get_device_error(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the status word of the workspace (0 = no error)."""
    code = ctypes.c_int()
    st = lib().moe_get_device_error(_ptr(ws), ctypes.byref(code), _stream(stream))
    if st not in (0, 5):
        raise MoEError("moe_get_device_error", st)
    return code.value


def moe_last_launch_count() -> int:
    return lib().moe_last_launch_count()


MOE_SELFTEST_WS_BYTES = 256 + 32768


def moe_selftest_bounded_wait(wait_limit_ns: int, ws: Optional[torch.Tensor] = None,
                              device=None, stream=None) -> torch.Tensor:
    """Enqueue the failure-detection self-test (a grouped-GEMM launch whose wait can never
    complete and must give up after ``wait_limit_ns``); returns the workspace whose status
    block then holds MOE_DEVERR_TIMEOUT (read it with moe_get_device_error)."""
    if ws is None:
        ws = workspace(MOE_SELFTEST_WS_BYTES, device if device is not None else "cuda")
    _check("moe_selftest_bounded_wait", lib().moe_selftest_bounded_wait(
        _ptr(ws), ws.numel(), int(wait_limit_ns), _stream(stream)))
    return ws
