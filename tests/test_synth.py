"""The seeded input generator: determinism, slicing, independence and moments."""
import numpy as np

import synth


def test_draws_are_counter_based_and_sliceable():
    a = synth.draw_u64(5702, 4, 1000)
    b = synth.draw_u64(5702, 4, 300, offset=700)
    assert np.array_equal(a[700:], b)
    assert len(np.unique(a)) == 1000
    assert not np.array_equal(a, synth.draw_u64(5702, 5, 1000))
    assert not np.array_equal(a, synth.draw_u64(5703, 4, 1000))


def test_splitmix64_finaliser_known_value():
    # The splitmix64 generator seeded with 0 first outputs 0xE220A8397B1DCDAF (its
    # published reference sequence); that output is mix64(G), which pins the finaliser.
    G = 0x9E3779B97F4A7C15
    M = (1 << 64) - 1

    def mix(z):
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        return z ^ (z >> 31)
    assert mix(G) == 0xE220A8397B1DCDAF
    L = synth.lib()
    out = np.empty(3, dtype=np.uint64)
    key = L.synth_key(1, 2)
    L.synth_draw_u64(1, 2, 0, 3, out.ctypes.data)
    assert [int(v) for v in out] == [mix((key + (i + 1) * G) & M) for i in range(3)]


def test_normal_moments_and_bf16():
    z = synth.normal(7, 1, (1 << 20,), std=1.0, dtype="f64")
    assert abs(z.mean()) < 4e-3 and abs(z.std() - 1) < 4e-3
    assert abs(np.mean(z ** 4) - 3) < 0.05
    f = synth.normal(7, 1, (1 << 20,), std=0.02, dtype="f32")
    assert np.allclose(f, (0.02 * z).astype(np.float32), rtol=1e-6, atol=0)
    bits = synth.normal(7, 1, (1 << 20,), std=0.02, dtype="bf16")
    back = synth.bf16_bits_to_f32(bits)
    assert np.max(np.abs(back - f) / np.maximum(np.abs(f), 1e-30)) <= 2 ** -8


def test_permutation_and_zipf_bias():
    p = synth.permutation(5704, synth.STREAM["zipf_perm"], 128)
    assert sorted(p.tolist()) == list(range(1, 129))
    w = synth.WORKLOADS[4]
    b = synth.router_bias(w)
    r = synth.permutation(w.seed, synth.STREAM["zipf_perm"], w.E)
    assert np.allclose(b, -1.2 * np.log(r.astype(np.float64)), atol=1e-6)


def test_workload_table():
    W = synth.WORKLOADS
    assert [W[i].T for i in range(1, 6)] == [64, 16384, 16384, 8192, 32]
    assert [W[i].E for i in range(1, 6)] == [4, 128, 128, 8, 128]
    assert [W[i].k for i in range(1, 6)] == [1, 1, 1, 2, 1]
    assert W[3].dense and not W[3].add_input_residual
    inp = synth.make_inputs(W[1])
    assert inp["x"].shape == (64, 32) and inp["w1"].shape == (4, 64, 32) and inp["w2"].shape == (4, 32, 64)
    again = synth.make_inputs(W[1])
    assert all(np.array_equal(inp[k], again[k]) for k in inp if inp[k] is not None)
