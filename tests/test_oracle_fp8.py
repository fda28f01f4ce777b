"""Pins of the oracle's e4m3 quantization (low-precision expert weights):
the e4m3 format's landmarks, torch's own float8_e4m3fn conversion, ties to
even at every midpoint, saturation, the closed form of the power-of-two row
scale, the per-element error bound, and the quantized expert against the
exact float64 one."""
import numpy as np
import torch

from oracle import moe_oracle as mo

F32 = np.float32


def test_e4m3_table_landmarks():
    t = mo.e4m3_table()
    assert t.shape == (127,) and np.all(np.diff(t) > 0)
    assert t[0] == 0.0 and t[1] == 2.0 ** -9 and t[7] == 7 * 2.0 ** -9      # subnormals
    assert t[8] == 2.0 ** -6                                                  # smallest normal
    assert t[0x38] == 1.0 and t[0x3C] == 1.5
    assert t[126] == 448.0 and t[125] == 416.0                                # largest finite


def test_encode_matches_torch_float8_cast():
    rng = np.random.default_rng(0)
    mags = rng.choice([1e-4, 3e-3, 0.1, 1.0, 30.0, 300.0], size=300000)
    x = np.clip(rng.normal(size=300000) * mags, -448, 448).astype(F32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mo.e4m3_encode(x), ref)
    # exact values map to their own codes, and decode inverts encode
    codes = np.arange(256, dtype=np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]                                     # drop NaN codes
    assert np.array_equal(mo.e4m3_encode(mo.e4m3_decode(codes).astype(F32)), codes)


def test_ties_go_to_the_even_code_and_saturation():
    t = mo.e4m3_table()
    mid = ((t[:-1] + t[1:]) / 2).astype(F32)
    assert np.all(mid.astype(np.float64) == (t[:-1] + t[1:]) / 2)              # exact in fp32
    c = mo.e4m3_encode(mid)
    assert np.all(c % 2 == 0)
    assert np.array_equal(c, torch.from_numpy(mid).to(torch.float8_e4m3fn).view(torch.uint8).numpy())
    big = np.array([448.0, 460.0, 1e6, 3e38, -449.0, -1e30], F32)
    assert list(mo.e4m3_encode(big)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert mo.e4m3_encode(np.array([-1e-6], F32))[0] == 0x80                  # -0


def test_pow2_scale_closed_form():
    rng = np.random.default_rng(1)
    a = (rng.uniform(0.5, 1.0, 50000) * 2.0 ** rng.integers(-40, 40, 50000)).astype(F32)
    s = mo.pow2_scale(a).astype(np.float64)
    m, _ = np.frexp(s)
    assert np.all(m == 0.5)                                                   # powers of two
    assert np.all(a / s <= 448.0) and np.all(a / (s / 2) > 448.0)             # smallest such
    edge = np.array([448.0, np.nextafter(F32(448.0), F32(1e9)), 0.0, 1.0, 1.75, 1.7500001, 224.0], F32)
    assert list(mo.pow2_scale(edge)) == [1.0, 2.0, 1.0, 2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 0.5]
    # the scale stays a normal fp32 number for tiny rows
    tiny = np.array([2.0 ** -120, 2.0 ** -140, np.finfo(F32).smallest_subnormal], F32)
    assert list(mo.pow2_scale(tiny)) == [2.0 ** -126] * 3


def test_quantize_rows_error_bound():
    rng = np.random.default_rng(2)
    x = (rng.normal(size=(64, 700)) * rng.choice([1e-3, 1.0, 50.0], size=(64, 1))).astype(F32)
    x[3] = 0.0
    codes, s = mo.quantize_rows(x)
    deq = mo.dequantize_rows(codes, s)
    rel = np.abs(deq - x) / np.maximum(np.abs(x), 1e-30)
    normal = np.abs(x) / s[:, None] >= 2.0 ** -6
    assert np.all(rel[normal] <= 2.0 ** -4)                                   # half of 3 mantissa bits
    assert np.all(np.abs(deq - x)[~normal] <= 2.0 ** -10 * np.broadcast_to(s[:, None], x.shape)[~normal])
    top = np.max(np.abs(mo.e4m3_decode(codes)), axis=1)
    assert np.all((top[np.arange(64) != 3] >= 224) & (top[np.arange(64) != 3] <= 448))
    assert s[3] == 1.0 and np.all(codes[3] == 0)


def test_quantized_expert_tracks_the_exact_one():
    """e4m3 weights and rows: the expert output stays within 10 % (RMS) of the
    float64 expert -- three roundings to 3 mantissa bits (rows, weights, A),
    each uniform within +-2^-4 relative, give about 6 % -- and the error is
    not zero (the quantization is applied)."""
    rng = np.random.default_rng(3)
    d, f, n = 256, 192, 40
    x = rng.normal(size=(n, d)).astype(F32)
    wg = (rng.normal(size=(f, d)) / np.sqrt(d)).astype(F32)
    wu = (rng.normal(size=(f, d)) / np.sqrt(d)).astype(F32)
    wd = (rng.normal(size=(d, f)) / np.sqrt(f)).astype(F32)
    exact = mo.swiglu(x, wg, wu, wd)
    q = mo.swiglu_q8(x, mo.quantize_rows(wg), mo.quantize_rows(wu), mo.quantize_rows(wd))
    err = np.sqrt(np.mean((q - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    assert 1e-3 < err < 0.10, err
    # zero down projection -> zero output; zero input -> zero output
    zero = mo.quantize_rows(np.zeros((d, f), F32))
    assert np.all(mo.swiglu_q8(x, mo.quantize_rows(wg), mo.quantize_rows(wu), zero) == 0)
    assert np.all(mo.swiglu_q8(np.zeros_like(x), mo.quantize_rows(wg), mo.quantize_rows(wu),
                               mo.quantize_rows(wd)) == 0)
