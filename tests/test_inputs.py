"""The synthetic-input generator: numpy definition vs its host C twin (the CUDA
twin is compared in tests/test_gpu_parity.py), and the shape of the draws."""
import numpy as np

import moe_inputs as mi
from moe_inputs import native


def test_splitmix64_reference_vector():
    # SplitMix64 with state 0: published first outputs of the generator
    # (Steele, Lea & Flood 2014; the reference implementation by S. Vigna)
    state = 0
    outs = []
    for _ in range(3):
        state = (state + mi.GOLDEN) & mi.MASK64
        outs.append(mi._mix_int(state))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_host_twin_matches_numpy():
    for bf16 in (False, True):
        for (tid, start, n, sigma) in [(3, 0, 1000, 1.0), (77, 123456789, 4097, 0.02), (5, 2**33 + 7, 300, 0.011)]:
            ref = mi.normal_f32(42, tid, start, n, sigma)
            got = native.fill_host(n, bf16, 42, tid, start, sigma)
            if bf16:
                assert np.array_equal(got, mi.f32_to_bf16_bits(ref))
            else:
                assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    ref = mi.uniform_f32(9, 3, 10, 999, -0.01, 0.01)
    got = native.fill_host(999, False, 9, 3, 10, uniform=(-0.01, 0.01))
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_normal_moments():
    x = mi.normal_f32(1, 1, 0, 1 << 20, 1.0).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.var() - 1.0) < 5e-3
    assert np.abs(x).max() <= 2 * np.sqrt(3) + 1e-6


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.005859375, 1.0 + 2**-8 + 2**-9, -3.3], np.float32)
    r = mi.round_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == np.float32(1.0078125)
    assert np.all(np.abs(r - x) <= np.abs(x) * 2.0**-8)


def test_workload_slices_regenerate():
    w = mi.WORKLOADS["finegrained_64x1408"].with_(T=16, d_model=64, d_ffn=32, d_ffn_shared=32, E_r=4)
    full = mi.gen_weight(w, "down")
    assert np.array_equal(full[2], mi.gen_weight(w, "down", 2))
    assert np.array_equal(full[3], native.weight_host(w, "down", 3))
    h = mi.gen_h(w, 0)
    assert np.array_equal(h[5:9], mi.gen_h(w, 0, slice(5, 9)))
