"""GPU parity of moe_expert_ffn (tcgen05 grouped GEMM for bf16, fp32 FMA for fp32) against the
oracle's per-row two-layer GeLU FFN, over ragged segments that span several token tiles, empty
experts, feature counts that are not multiples of the 128-row tile and K tails."""
import numpy as np
import pytest
import torch

import oracle
import synth
from mixture_experts_layer_57_b200 import moe
from tests.helpers import as_f64, to_dev, to_host

pytestmark = pytest.mark.gpu


def run_ffn_case(E, d, d_ff, counts, dt, hint, seed=0, w_std=0.05, with_bias=True):
    rng = np.random.default_rng(seed)
    w = synth.Workload("t", T=1, d_model=d, d_ff=d_ff, E=E, k=1, capacity_factor=1.0, dtype=dt,
                       w_std=w_std, b_std=0.05, seed=seed + 100)
    ew = synth.make_inputs(w, experts_only=True)
    rows = int(sum(counts))
    rows_max = rows + 5   # slack rows beyond the last segment stay untouched
    xs = synth.normal(seed + 7, 1, (rows_max, d), std=1.0, dtype=dt)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    b1 = to_dev(ew["b1"]) if with_bias else None
    b2 = to_dev(ew["b2"]) if with_bias else None
    r = moe.moe_expert_ffn(to_dev(xs), to_dev(off), to_dev(ew["w1"]), b1, to_dev(ew["w2"]), b2,
                           rows_max=rows_max, capacity_hint=hint)
    assert moe.moe_get_device_error(r["ws"]) == 0
    y = to_host(r["y_packed"])[:rows]
    # oracle, row by row (sampled for large cases)
    idx = np.arange(rows)
    if rows > 600:
        idx = np.sort(rng.choice(rows, 600, replace=False))
    ref = np.empty((len(idx), d))
    for n, rr in enumerate(idx):
        e = int(np.searchsorted(off, rr, side="right") - 1)
        ref[n] = oracle.ffn(xs[rr], ew["w1"][e], ew["b1"][e] if with_bias else None, ew["w2"][e],
                            ew["b2"][e] if with_bias else None)
    diff = np.abs(y[idx].astype(np.float64) - ref)
    return diff, ref


@pytest.mark.parametrize("hint,counts", [
    (1, [1, 0, 1, 1, 0, 1]),                     # token tile 16, one row per expert (decode)
    (20, [20, 3, 0, 17, 20]),                    # token tile 32
    (50, [50, 64, 1, 0, 33]),                    # token tile 64
    (128, [128, 127, 0, 1, 100, 128]),           # token tile 128
    (300, [300, 257, 0, 5, 256, 513]),           # token tile 256, several tiles per expert
    (16, [40, 0, 33]),                           # segments longer than the hinted tile
])
def test_ffn_bf16_ragged(cuda_ok, hint, counts):
    diff, ref = run_ffn_case(len(counts), 256, 512, counts, "bf16", hint, seed=hint)
    assert diff.max() <= 2e-3, diff.max()
    assert np.linalg.norm(diff) <= 1e-3 * np.linalg.norm(ref)


@pytest.mark.parametrize("d,d_ff", [(136, 264), (64, 8), (8, 200), (1024, 4096)])
def test_ffn_bf16_feature_and_k_tails(cuda_ok, d, d_ff):
    diff, ref = run_ffn_case(3, d, d_ff, [70, 0, 129], "bf16", 128, seed=d + d_ff)
    assert diff.max() <= 2e-3 * max(1.0, np.abs(ref).max())
    assert np.linalg.norm(diff) <= 1e-3 * np.linalg.norm(ref)


def test_ffn_bf16_no_bias(cuda_ok):
    diff, ref = run_ffn_case(4, 128, 256, [5, 200, 0, 31], "bf16", 256, seed=3, with_bias=False)
    assert diff.max() <= 2e-3


@pytest.mark.parametrize("counts", [[16, 0, 7, 3], [1, 1, 1, 1, 1], [64]])
def test_ffn_fp32(cuda_ok, counts):
    diff, ref = run_ffn_case(len(counts), 32, 64, counts, "f32", 16, seed=9, w_std=0.1)
    assert diff.max() <= 1e-5


def test_ffn_fp32_odd_sizes(cuda_ok):
    diff, ref = run_ffn_case(2, 33, 130, [9, 4], "f32", 9, seed=10, w_std=0.1)
    assert diff.max() <= 1e-5


def test_ffn_hidden_is_gelu_rounded_to_bf16(cuda_ok):
    # one expert, identity-free check of h: compare the stored bf16 h with the oracle's rounding
    E, d, d_ff, n = 1, 64, 128, 40
    w = synth.Workload("t", T=1, d_model=d, d_ff=d_ff, E=E, k=1, capacity_factor=1.0, dtype="bf16",
                       w_std=0.1, b_std=0.1, seed=11)
    ew = synth.make_inputs(w, experts_only=True)
    xs = synth.normal(12, 1, (n, d), dtype="bf16")
    off = np.array([0, n], dtype=np.int32)
    r = moe.moe_expert_ffn(to_dev(xs), to_dev(off), to_dev(ew["w1"]), to_dev(ew["b1"]),
                           to_dev(ew["w2"]), to_dev(ew["b2"]), capacity_hint=n)
    h = as_f64(to_host(r["h_packed"]))
    z = as_f64(xs) @ as_f64(ew["w1"][0]).T + as_f64(ew["b1"][0])
    ref = np.vectorize(oracle.gelu)(z)
    ref_bf = as_f64(oracle.round_bf16(ref))
    # identical except where the pre-rounding values straddle a rounding boundary
    same = h == ref_bf
    assert same.mean() > 0.99
    assert np.all(np.abs(h - ref) <= 2 * (np.abs(ref) * 2.0 ** -8 + 1e-30) + 1e-6)


def test_ffn_flags_bad_offsets(cuda_ok):
    d, d_ff = 64, 128
    w1 = torch.randn(2, d_ff, d, device="cuda").to(torch.bfloat16)
    w2 = torch.randn(2, d, d_ff, device="cuda").to(torch.bfloat16)
    x = torch.randn(10, d, device="cuda").to(torch.bfloat16)
    off = torch.tensor([0, 8, 4], dtype=torch.int32, device="cuda")   # decreasing
    r = moe.moe_expert_ffn(x, off, w1, None, w2, None, rows_max=10, capacity_hint=8)
    assert moe.moe_get_device_error(r["ws"]) == 3   # MOE_DEVERR_BAD_OFFSETS
