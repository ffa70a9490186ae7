"""GPU parity of moe_dispatch: slots, demand counts, offsets, the token map and the packed rows
are compared bit-exactly with the oracle's first-come slot assignment and with the definition
offsets[e] = sum_{e' < e} min(counts[e'], C), x_packed[offsets[e] + slot] = x[t]."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_57_b200 import moe
from tests.helpers import to_dev, to_host

pytestmark = pytest.mark.gpu


def make_ids(rng, T, E, k, kind):
    if kind == "uniform":
        return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    if kind == "one_expert":
        ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        ids[:, 0] = E // 2
        for t in range(T):
            if k > 1 and (ids[t, 1:] == E // 2).any():
                others = [e for e in range(E) if e != E // 2]
                ids[t, 1:] = rng.choice(others, size=k - 1, replace=False)
        return ids
    if kind == "zipf":
        p = 1.0 / np.arange(1, E + 1) ** 1.2
        p /= p.sum()
        return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    raise ValueError(kind)


def check_dispatch(x_host, ids, E, C, dt):
    T, k = ids.shape
    x = to_dev(x_host)
    r = moe.moe_dispatch(x, to_dev(ids), E, C)
    assert moe.moe_get_device_error(r["ws"]) == 0
    slot, counts = oracle.assign_slots(ids, E, C)
    got_slot = to_host(r["slot"])
    assert np.array_equal(got_slot, slot)
    assert np.array_equal(to_host(r["expert_counts"]), counts)
    kept = np.minimum(counts, C)
    off = np.concatenate([[0], np.cumsum(kept)]).astype(np.int32)
    assert np.array_equal(to_host(r["expert_offsets"]), off)
    total = int(off[-1])
    assert total <= r["rows_max"]
    rt = to_host(r["row_token"])[:total]
    xp = to_host(r["x_packed"])[:total]
    for t in range(T):
        for j in range(k):
            if slot[t, j] >= 0:
                row = off[ids[t, j]] + slot[t, j]
                assert rt[row] == t
    assert np.array_equal(xp, x_host[rt])
    return total


@pytest.mark.parametrize("T,E,k,kind,cf", [
    (16384, 128, 1, "uniform", 1.0), (8192, 8, 2, "zipf", 1.25), (32, 128, 1, "uniform", 2.0),
    (1000, 37, 3, "zipf", 1.0), (777, 1024, 8, "uniform", 1.0), (513, 16, 4, "one_expert", 1.0),
    (1, 4, 1, "uniform", 1.0), (300, 5, 5, "uniform", 100.0), (300, 6, 2, "uniform", 0.0),
])
def test_dispatch_bit_exact(cuda_ok, T, E, k, kind, cf):
    rng = np.random.default_rng(T * 7 + E)
    ids = make_ids(rng, T, E, k, kind)
    C = moe.moe_capacity(T, E, k, cf)
    d = 64
    xbits = rng.integers(0, 1 << 16, size=(T, d), dtype=np.uint16)
    xbits[(xbits & 0x7f80) == 0x7f80] = 0   # keep the payload free of NaN/Inf bit patterns
    check_dispatch(xbits, ids, E, C, "bf16")


def test_dispatch_fp32_rows_and_odd_width(cuda_ok):
    rng = np.random.default_rng(5)
    T, E, k, d = 999, 9, 2, 13   # fp32 rows of 52 bytes: 4-byte copy path
    ids = make_ids(rng, T, E, k, "zipf")
    x = rng.normal(size=(T, d)).astype(np.float32)
    check_dispatch(x, ids, E, moe.moe_capacity(T, E, k, 1.0), "f32")


def test_dispatch_deterministic(cuda_ok):
    rng = np.random.default_rng(6)
    T, E, k = 4096, 64, 2
    ids = to_dev(make_ids(rng, T, E, k, "zipf"))
    x = torch.randn(T, 256, device="cuda").to(torch.bfloat16)
    C = moe.moe_capacity(T, E, k, 1.0)
    a = moe.moe_dispatch(x, ids, E, C)
    b = moe.moe_dispatch(x, ids, E, C)
    for n in ("slot", "expert_counts", "expert_offsets"):
        assert torch.equal(a[n], b[n])
    tot = int(a["expert_offsets"][-1])
    assert torch.equal(a["x_packed"][:tot].view(torch.int16), b["x_packed"][:tot].view(torch.int16))


def test_dispatch_flags_bad_expert_id(cuda_ok):
    T, E, k = 100, 4, 1
    ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    ids[17, 0] = 9
    x = torch.randn(T, 64, device="cuda").to(torch.bfloat16)
    r = moe.moe_dispatch(x, ids, E, 50)
    assert moe.moe_get_device_error(r["ws"]) == 2   # MOE_DEVERR_BAD_EXPERT
    slot = to_host(r["slot"])
    assert slot[17, 0] == -1 and slot[16, 0] == 16 and slot[18, 0] == 17
