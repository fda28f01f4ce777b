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
        for (tid, start, n, sigma) in [(3, 0, 1000, 1.0), (77, 123456789, 4097, 0.02), (5, 2**33 + 7, 300, 0.011),
                                       (11, 0, 1 << 18, 1.0)]:
            ref = mi.normal_f32(42, tid, start, n, sigma)
            got = native.fill_host(n, bf16, 42, tid, start, sigma)
            if bf16:
                assert np.array_equal(got, mi.f32_to_bf16_bits(ref))
            else:
                assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    ref = mi.uniform_f32(9, 3, 10, 999, -0.01, 0.01)
    got = native.fill_host(999, False, 9, 3, 10, uniform=(-0.01, 0.01))
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_normal_draws_follow_the_normal_law():
    """Box-Muller draws: N(0, 1) moments, Gaussian tails (the +-6.76 sigma
    bound of u1 >= 2**-33), and a Kolmogorov-Smirnov distance to the normal
    CDF within what 2**20 samples allow."""
    from scipy import stats
    x = mi.normal_f32(1, 1, 0, 1 << 20, 1.0).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.var() - 1.0) < 5e-3
    kurt = ((x - x.mean()) ** 4).mean() / x.var() ** 2
    assert abs(kurt - 3.0) < 0.03
    assert 4.0 < np.abs(x).max() <= np.sqrt(-2.0 * np.log(2.0 ** -33)) + 1e-6
    assert abs(np.mean(np.abs(x) > 3.0) - 2 * stats.norm.sf(3.0)) < 4e-4
    assert stats.kstest(x, "norm").statistic < 2e-3
    y = mi.normal_f32(5, 9, 12345, 1 << 16, 0.02).astype(np.float64)
    assert abs(y.std() / 0.02 - 1.0) < 0.01


def test_ln_and_cos_series_against_the_library():
    """The generator's own ln and cos (fixed series in IEEE double) agree with
    the C library to within a few units in the last place, at the ends of both
    argument ranges, the sqrt(1/2) mantissa switch and the octant folds."""
    import math
    hi = np.array([0, 1, 2, 3, 4, 5, 181, 182, 1000, 2**20 + 3, 2**31 - 1, 2**31, 2**32 - 2, 2**32 - 1],
                  dtype=np.uint64)
    got = mi.ln_half_int(hi)
    for h, g in zip(hi, got):
        ref = math.log((int(h) + 0.5) * 2.0 ** -32)        # the scaling by 2**-32 is exact
        assert abs(g - ref) <= 4e-16 * abs(ref) + 1e-300, (int(h), g, ref)
    q = 1 << 30
    lo = np.array([0, 1, 2, q // 2 - 1, q // 2, q // 2 + 1, q - 1, q, q + 1, 2 * q - 1, 2 * q, 3 * q - 1, 3 * q,
                   4 * q - 1, 123456789, 3000000000], dtype=np.uint64)
    def cos_ref(l):
        # the library's cos / sin of the angle within the quadrant (reduced
        # exactly in integers, so the reference has no large-argument error)
        q, f = l >> 30, l & ((1 << 30) - 1)
        a = f * math.pi / 2.0 ** 31
        return (math.cos(a), -math.sin(a), -math.cos(a), math.sin(a))[q]

    gc = mi.cos_2pi_frac(lo)
    for l, g in zip(lo, gc):
        ref = cos_ref(int(l))
        assert abs(g - ref) <= 4e-16, (int(l), g, ref)
        assert abs(g - math.cos(2.0 * math.pi * int(l) / 2.0 ** 32)) <= 2e-15
    rng = np.random.default_rng(0)
    r = rng.integers(0, 2**32, size=4096, dtype=np.uint64)
    assert max(abs(g - cos_ref(int(l))) for l, g in zip(r, mi.cos_2pi_frac(r))) <= 4e-16
    ln_ref = np.log((r.astype(np.float64) + 0.5) * 2.0 ** -32)
    assert np.max(np.abs(mi.ln_half_int(r) - ln_ref) / np.abs(ln_ref)) <= 4e-16


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
