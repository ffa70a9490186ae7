"""GPU parity of moe_combine against the oracle's combine (double sum, one rounding)."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_57_b200 import moe
from tests.conftest import golden
from tests.helpers import as_f64, bf16_half_ulp, to_dev, to_host

pytestmark = pytest.mark.gpu


def case(rng, T, d, E, k, drop_p):
    counts = np.zeros(E, dtype=np.int64)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    slot = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            if rng.random() >= drop_p:
                slot[t, j] = counts[e]
                counts[e] += 1
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1])
    y = rng.normal(size=(max(rows, 1), d)).astype(np.float32)
    gates = rng.random((T, k)).astype(np.float32)
    y_pairs = np.zeros((T, k, d), dtype=np.float32)
    for t in range(T):
        for j in range(k):
            if slot[t, j] >= 0:
                y_pairs[t, j] = y[off[ids[t, j]] + slot[t, j]]
    return ids, slot, off, y, gates, y_pairs


@pytest.mark.parametrize("T,d,E,k,res,dense,out_bf16", [
    (500, 256, 8, 2, "bf16", False, True), (333, 64, 5, 1, "f32", True, False),
    (64, 30, 4, 3, None, True, False), (1, 8, 2, 2, "bf16", True, True),
    (2048, 1024, 128, 1, "bf16", False, True), (100, 72, 16, 8, "f32", False, True),
])
def test_combine(cuda_ok, T, d, E, k, res, dense, out_bf16):
    rng = np.random.default_rng(T + d)
    ids, slot, off, y, gates, y_pairs = case(rng, T, d, E, k, drop_p=0.2)
    resid = None
    if res == "bf16":
        resid = torch.randn(T, d).to(torch.bfloat16)
    elif res == "f32":
        resid = torch.randn(T, d)
    dns = rng.normal(size=(T, d)).astype(np.float32) if dense else None
    r = moe.moe_combine(to_dev(y), to_dev(off), to_dev(ids), to_dev(slot), to_dev(gates),
                        residual=None if resid is None else resid.cuda(),
                        dense=None if dns is None else to_dev(dns),
                        out_dtype=torch.bfloat16 if out_bf16 else torch.float32, rows_max=y.shape[0])
    assert moe.moe_get_device_error(r["ws"]) == 0
    got = as_f64(to_host(r["out"]))
    res_np = None if resid is None else to_host(resid)
    ref = oracle.combine(gates, slot, y_pairs, residual=res_np, dense=dns)
    diff = np.abs(got - ref)
    if out_bf16:
        assert (diff <= bf16_half_ulp(ref) + 1e-5 * (1 + np.abs(ref))).all()
    else:
        assert diff.max() <= 2e-6 * (1 + np.abs(ref).max())


def test_combine_prmoe_page_example(cuda_ok):
    g = golden("prmoe_residual.json")
    y = np.array([g["r_A"], g["r_B"]], dtype=np.float32)          # expert A row 0, expert B row 1
    off = np.array([0, 1, 2], dtype=np.int32)
    ids = np.array([[0]], dtype=np.int32)
    slot = np.array([[0]], dtype=np.int32)
    gates = np.array([[g["gate"]]], dtype=np.float32)
    dense = np.array([g["h_fixed"]], dtype=np.float32)
    r = moe.moe_combine(to_dev(y), to_dev(off), to_dev(ids), to_dev(slot), to_dev(gates),
                        dense=to_dev(dense), out_dtype=torch.float32, rows_max=2)
    np.testing.assert_allclose(to_host(r["out"])[0], g["output"], atol=1e-6)


def test_combine_flags_bad_row(cuda_ok):
    y = torch.randn(4, 16, device="cuda")
    off = torch.tensor([0, 2, 4], dtype=torch.int32, device="cuda")
    ids = torch.tensor([[0], [1]], dtype=torch.int32, device="cuda")
    slot = torch.tensor([[1], [7]], dtype=torch.int32, device="cuda")   # row 9 is beyond rows_max
    gates = torch.ones(2, 1, device="cuda")
    r = moe.moe_combine(y, off, ids, slot, gates, out_dtype=torch.float32, rows_max=4)
    assert moe.moe_get_device_error(r["ws"]) == 4   # MOE_DEVERR_BAD_ROW
    out = to_host(r["out"])
    np.testing.assert_array_equal(out[0], to_host(y)[1])
    np.testing.assert_array_equal(out[1], 0)
