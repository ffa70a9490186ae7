"""The C-ABI library on the host: it loads, exports every function include/moe.h declares, and
rejects invalid arguments before any CUDA call (so these run without a GPU)."""
import ctypes
import subprocess

import pytest

from mixture_experts_layer_57_b200 import build as build_mod
from mixture_experts_layer_57_b200 import moe


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return moe.lib()


def test_exports_every_declared_symbol(L):
    names = moe.header_symbols()
    assert len(names) >= 17
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)


def test_abi_version_and_status_strings(L):
    assert L.moe_abi_version() == 3
    for code, name in moe.STATUS_NAMES.items():
        assert L.moe_status_string(code).decode() == name


def test_capacity_and_rows(L):
    assert moe.moe_capacity(16384, 128, 1, 1.0) == 128
    assert moe.moe_capacity(8192, 8, 2, 1.25) == 2560
    assert moe.moe_capacity(32, 128, 1, 2.0) == 1
    assert moe.moe_capacity(64, 4, 1, 1.0) == 16
    assert moe.moe_capacity(10, 4, 1, 0.0) == 0
    assert moe.moe_packed_rows_max(16384, 128, 1, 128) == 16384
    assert moe.moe_packed_rows_max(32, 128, 1, 1) == 32
    assert moe.moe_packed_rows_max(100, 4, 2, 10) == 40
    assert moe.moe_packed_rows_max(5, 2, 2, 5_000_000_000) == 10
    c = ctypes.c_int64()
    for args in [(-1, 4, 1, 1.0), (4, 0, 1, 1.0), (4, 4, 0, 1.0), (4, 4, 1, -1.0),
                 (4, 4, 1, float("nan")), (4, 4, 1, float("inf"))]:
        assert L.moe_capacity(*args, ctypes.byref(c)) == 1


def test_capacity_of_decimal_factor(L):
    # ceil(k T / E x cf) of the decimal factor: 100 tokens / 10 experts x 1.1 = 11, not 12
    assert moe.moe_capacity(100, 10, 1, 1.1) == 11
    assert moe.moe_capacity(1000, 100, 1, 1.1) == 11
    assert moe.moe_capacity(700, 10, 1, 0.7) == 49
    assert moe.moe_capacity(30, 10, 1, 1.1) == 4


def test_capacity_matches_oracle_formula(L):
    import oracle
    for T, E, k, cf in [(1000, 7, 2, 1.1), (3, 5, 1, 0.3), (16384, 128, 1, 1.0), (777, 13, 3, 2.5)]:
        assert moe.moe_capacity(T, E, k, cf) == oracle.capacity(T, E, k, cf)


def test_workspace_queries(L):
    # status block + statistics accumulators + split weight (3 bf16 parts) + logits scratch
    assert moe.moe_router_workspace_bytes(16384, 128, 1024) >= 256 + 128 * 12 + 128 * 3 * 1024 * 2 + 16384 * 128 * 4
    assert moe.moe_dispatch_workspace_bytes(16384, 128, 1) > 256
    assert moe.moe_expert_ffn_workspace_bytes() == 256
    assert moe.moe_combine_workspace_bytes() == 256


FAKE = 0x10000  # 16-byte aligned non-null address; never dereferenced: validation fails first


def _router(L, **kw):
    a = dict(x=FAKE, xdt=1, T=16, d=64, w=FAKE, b=None, E=8, k=2, logits=None, ids=FAKE,
             gates=FAKE, lb=None, alpha=0.01, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return L.moe_router_topk(a["x"], a["xdt"], a["T"], a["d"], a["w"], a["b"], a["E"], a["k"],
                             a["logits"], a["ids"], a["gates"], a["lb"], a["alpha"], a["ws"], a["wsb"], None)


def test_router_validation(L):
    assert _router(L, k=9, E=16) == 2           # k > 8 unsupported
    assert _router(L, k=3, E=2) == 1            # k > E
    assert _router(L, E=0) == 1
    assert _router(L, E=2000) == 2
    assert _router(L, T=-1) == 1
    assert _router(L, xdt=7) == 1
    assert _router(L, x=None) == 1
    assert _router(L, ids=None) == 1
    assert _router(L, ws=None) == 1
    assert _router(L, x=FAKE + 4) == 6          # misaligned
    assert _router(L, ws=FAKE + 16) == 6        # workspace must be 256-aligned
    assert _router(L, wsb=100) == 3             # workspace too small


def test_router_ex_validation(L, monkeypatch):
    def call(**kw):
        a = dict(x=FAKE, xdt=1, T=16, d=64, w=FAKE, b=None, E=8, k=2, logits=None, ids=FAKE,
                 gates=FAKE, lb=None, alpha=0.01, rn=1, losses=FAKE, probs=None, ws=FAKE,
                 wsb=1 << 30)
        a.update(kw)
        return L.moe_router_topk_ex(a["x"], a["xdt"], a["T"], a["d"], a["w"], a["b"], a["E"],
                                    a["k"], a["logits"], a["ids"], a["gates"], a["lb"], a["alpha"],
                                    a["rn"], a["losses"], a["probs"], a["ws"], a["wsb"], None)
    assert call(k=3, E=2) == 1
    assert call(losses=FAKE + 4) == 6           # misaligned router_losses
    assert call(probs=FAKE + 4) == 6            # misaligned probabilities output
    assert call(wsb=100) == 3
    monkeypatch.setenv("MOE_FAULT_INJECT", "moe_router_topk_ex")
    assert call() == 4
    assert _router(L, wsb=100) == 3             # the plain entry is a different name


def test_router_prepare_validation(L, monkeypatch):
    n = ctypes.c_size_t()
    assert L.moe_router_prepare_bytes(128, 1000, ctypes.byref(n)) == 0
    assert n.value == 128 * 3 * 1024 * 2                 # three bf16 parts, K padded to 64
    assert L.moe_router_prepare_bytes(0, 64, ctypes.byref(n)) == 1
    assert L.moe_router_prepare_bytes(2048, 64, ctypes.byref(n)) == 2
    big = 1 << 30
    assert L.moe_router_prepare(None, 8, 64, FAKE, big, None) == 1
    assert L.moe_router_prepare(FAKE, 8, 64, FAKE + 8, big, None) == 6
    assert L.moe_router_prepare(FAKE, 8, 64, FAKE, 100, None) == 3
    monkeypatch.setenv("MOE_FAULT_INJECT", "moe_router_prepare")
    assert L.moe_router_prepare(FAKE, 8, 64, FAKE, big, None) == 4


def test_dispatch_priority_validation(L):
    def call(**kw):
        a = dict(x=FAKE, dt=1, T=16, d=64, ids=FAKE, g=FAKE, E=4, k=1, C=4, slot=FAKE, cnt=FAKE,
                 off=FAKE, rt=FAKE, xp=FAKE, rows=16, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.moe_dispatch_priority(a["x"], a["dt"], a["T"], a["d"], a["ids"], a["g"], a["E"],
                                       a["k"], a["C"], a["slot"], a["cnt"], a["off"], a["rt"],
                                       a["xp"], a["rows"], a["ws"], a["wsb"], None)
    assert call(g=None) == 1                    # the probabilities are required
    assert call(g=FAKE + 4) == 6
    assert call(C=-1) == 1
    assert call(rows=15) == 1
    assert call(wsb=10) == 3


def test_dispatch_validation(L):
    def call(**kw):
        a = dict(x=FAKE, dt=1, T=16, d=64, ids=FAKE, E=4, k=1, C=4, slot=FAKE, cnt=FAKE, off=FAKE,
                 rt=FAKE, xp=FAKE, rows=16, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.moe_dispatch(a["x"], a["dt"], a["T"], a["d"], a["ids"], a["E"], a["k"], a["C"],
                              a["slot"], a["cnt"], a["off"], a["rt"], a["xp"], a["rows"], a["ws"],
                              a["wsb"], None)
    assert call(C=-1) == 1
    assert call(rows=15) == 1                   # packed buffers smaller than min(T k, E C)
    assert call(d=60) == 2                      # bf16 rows must be a multiple of 8 elements
    assert call(off=None) == 1
    assert call(slot=FAKE + 8) == 6
    assert call(wsb=10) == 3


def test_ffn_and_combine_validation(L):
    def ffn(**kw):
        a = dict(xp=FAKE, off=FAKE, E=4, rows=16, d=64, f=128, dt=1, w1=FAKE, b1=None, w2=FAKE,
                 b2=None, h=FAKE, y=FAKE, cap=16, ws=FAKE, wsb=256)
        a.update(kw)
        return L.moe_expert_ffn(a["xp"], a["off"], a["E"], a["rows"], a["d"], a["f"], a["dt"], a["w1"],
                                a["b1"], a["w2"], a["b2"], a["h"], a["y"], a["cap"], a["ws"], a["wsb"], None)
    assert ffn(f=100) == 2
    assert ffn(dt=0, d=20000) == 2
    assert ffn(w1=None) == 1
    assert ffn(cap=-1) == 1
    assert ffn(b1=FAKE + 2) == 6
    assert ffn(wsb=255) == 3

    def comb(**kw):
        a = dict(y=FAKE, off=FAKE, ids=FAKE, slot=FAKE, g=FAKE, T=8, d=64, E=4, k=2, rows=16,
                 res=None, rdt=1, dense=None, out=FAKE, odt=1, ws=FAKE, wsb=256)
        a.update(kw)
        return L.moe_combine(a["y"], a["off"], a["ids"], a["slot"], a["g"], a["T"], a["d"], a["E"],
                             a["k"], a["rows"], a["res"], a["rdt"], a["dense"], a["out"], a["odt"],
                             a["ws"], a["wsb"], None)
    assert comb(k=5, E=4) == 1
    assert comb(out=None) == 1
    assert comb(odt=3) == 1
    assert comb(dense=FAKE + 4) == 6


def test_layer_validation_and_workspace(L):
    args = moe.LayerArgs(T=16384, d_model=1024, d_ff=4096, E=128, k=1, capacity_factor=1.0,
                         dtype=1, out_dtype=1, x=FAKE, w_router=FAKE, w1=FAKE, w2=FAKE,
                         add_input_residual=1, aux_alpha=0.01)
    nbytes = moe.moe_layer_workspace_bytes(args)
    # packed x, h, y for 16384 rows plus routing buffers
    assert nbytes > 16384 * (1024 * 2 + 4096 * 2 + 1024 * 4)
    aux = moe.LayerAux()
    st = L.moe_layer_forward(ctypes.byref(args), FAKE, ctypes.byref(aux), FAKE, nbytes - 1, None)
    assert st == 3
    args.k = 0
    assert L.moe_layer_forward(ctypes.byref(args), FAKE, ctypes.byref(aux), FAKE, nbytes, None) == 1
    args.k = 1
    args.d_ff = 4100
    assert L.moe_layer_forward(ctypes.byref(args), FAKE, ctypes.byref(aux), FAKE, nbytes, None) == 2
    args.d_ff = 4096
    args.overflow_policy = 2                    # neither first-come nor priority
    assert L.moe_layer_forward(ctypes.byref(args), FAKE, ctypes.byref(aux), FAKE, nbytes, None) == 1
    args.overflow_policy = moe.MOE_OVERFLOW_PRIORITY
    assert moe.moe_layer_workspace_bytes(args) == nbytes
    aux.router_losses = FAKE + 4
    assert L.moe_layer_forward(ctypes.byref(args), FAKE, ctypes.byref(aux), FAKE, nbytes, None) == 6


def test_shard_entry_validation(L):
    args = moe.LayerArgs(T=4096, d_model=1024, d_ff=4096, E=128, k=1, capacity_factor=1.0,
                         dtype=1, out_dtype=1, x=FAKE, w_router=FAKE, w1=FAKE, w2=FAKE,
                         add_input_residual=1, aux_alpha=0.01)
    assert moe.moe_router_partials_count(128) == 513
    nb = moe.moe_layer_shard_workspace_bytes(args, 16384)
    # the capacity (and so nothing else in the layout) follows the whole batch
    assert nb >= moe.moe_layer_workspace_bytes(args)
    sz = ctypes.c_size_t()
    assert L.moe_layer_shard_workspace_bytes(ctypes.byref(args), 4095, ctypes.byref(sz)) == 1
    aux = moe.LayerAux()
    beg = lambda T_global=16384, dem=FAKE, par=FAKE, wsb=nb: L.moe_layer_forward_shard_begin(
        ctypes.byref(args), T_global, ctypes.byref(aux), dem, par, FAKE, wsb, None)
    end = lambda T_global=16384, G=4, r=1, da=FAKE, tot=FAKE, wsb=nb: L.moe_layer_forward_shard_end(
        ctypes.byref(args), T_global, G, r, da, tot, FAKE, ctypes.byref(aux), FAKE, wsb, None)
    assert beg(T_global=100) == 1               # the shard is part of the batch
    assert beg(dem=None) == 1 and beg(par=None) == 1
    assert beg(par=FAKE + 8) == 6
    assert beg(wsb=nb - 1) == 3
    assert end(G=0) == 1 and end(r=4) == 1 and end(r=-1) == 1
    assert end(da=None) == 1 and end(tot=None) == 1
    assert end(tot=FAKE + 4) == 6
    args.overflow_policy = moe.MOE_OVERFLOW_PRIORITY
    assert beg() == 2 and end() == 2            # a global priority order is not sharded


def test_training_entry_validation(L, monkeypatch):
    args = moe.LayerArgs(T=4096, d_model=1024, d_ff=4096, E=128, k=1, capacity_factor=1.0,
                         dtype=1, out_dtype=1, x=FAKE, w_router=FAKE, w1=FAKE, w2=FAKE,
                         add_input_residual=1, aux_alpha=0.01)
    nb = moe.moe_layer_train_workspace_bytes(args)
    # the training workspace holds the forward's plus h, GeLU'(z), dY, dZ, dX rows and more
    assert nb > moe.moe_layer_workspace_bytes(args) + 4096 * 4096 * 2 * 2
    aux = moe.LayerAux()
    fwd = lambda wsb=nb, out=FAKE: L.moe_layer_forward_train(ctypes.byref(args), out, ctypes.byref(aux),
                                                             FAKE, wsb, None)
    assert fwd(wsb=nb - 1) == 3
    assert fwd(out=None) == 1
    assert fwd(out=FAKE + 2) == 6
    g = moe.LayerGrads(dx=FAKE, dw_router=FAKE, dw1=FAKE, dw2=FAKE)
    bwd = lambda dout=FAKE, aw=0.0, zw=0.0, wsb=nb, grads=g: L.moe_layer_backward(
        ctypes.byref(args), dout, aw, zw, ctypes.byref(grads) if grads is not None else None,
        FAKE, wsb, None)
    assert bwd(grads=None) == 1
    assert bwd(dout=None) == 1
    assert bwd(aw=float("nan")) == 1
    assert bwd(wsb=nb - 1) == 3
    g2 = moe.LayerGrads(dx=FAKE, dw_router=FAKE, dw1=None, dw2=FAKE)
    assert bwd(grads=g2) == 1                   # expert weight gradients are required
    g3 = moe.LayerGrads(dx=FAKE, dw_router=FAKE, dw1=FAKE, dw2=FAKE, db1=FAKE + 4)
    assert bwd(grads=g3) == 6
    monkeypatch.setenv("MOE_FAULT_INJECT", "moe_layer_backward")
    assert bwd() == 4
    monkeypatch.setenv("MOE_FAULT_INJECT", "moe_layer_forward_train")
    assert fwd() == 4


def test_fault_injection_is_host_side(L, monkeypatch):
    # the injected failure is returned after validation and before any enqueue
    monkeypatch.setenv("MOE_FAULT_INJECT", "moe_router_topk")
    assert _router(L) == 4
    assert _router(L, k=3, E=2) == 1            # validation still comes first
    # naming another entry point leaves the router alone (it then fails on CUDA or the fake
    # pointers only after validation; no GPU is touched for the injected entry)
    monkeypatch.setenv("MOE_FAULT_INJECT", "moe_dispatch")
    assert _router(L, wsb=100) == 3


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        moe.lib()
