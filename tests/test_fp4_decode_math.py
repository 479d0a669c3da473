"""The arithmetic of the NVFP4 grouped GEMM's decode, checked exhaustively on
the host (no GPU): for every E2M1 code and every finite E4M3 scale byte,

  * the f16 encoding of the E2M1 value shifted right by three bits, sign bit
    kept in place, is the bf16 encoding of the same value times 2^-112;
  * bf16(scale x 2^112) is exact and finite;
  * the bf16 product of the two, rounded to nearest, is exactly
    value x scale (at most 6 significant bits), so the tensor cores see the
    exact weight up to the per-tensor scale.

The values come from the formats' definitions (E2M1: sign, 2 exponent bits
with bias 1, 1 mantissa bit; E4M3 through torch's float8_e4m3fn cast)."""
import numpy as np
import torch


def _e2m1(code: int) -> float:
    e, m = (code >> 1) & 3, code & 1
    v = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -v if code & 8 else v


def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_f16_shift_is_bf16_times_2_pow_minus_112():
    vals = np.array([_e2m1(c) for c in range(16)])
    h = vals.astype(np.float16).view(np.uint16).astype(np.uint32)
    r = ((h >> 3) & 0x0FFF) | (h & 0x8000)          # one half of the packed word
    got = _bf16_bits_to_f64(r.astype(np.uint16))
    np.testing.assert_array_equal(got, vals * 2.0 ** -112)
    # the packed form: the high half's low bits are zero, so a 32-bit shift
    # leaks nothing into the low half
    assert np.all((h & 0x7) == 0)


def test_scaled_products_are_exact_for_every_code_and_scale():
    finite = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)
    scale = torch.from_numpy(finite).view(torch.float8_e4m3fn).double().numpy()
    s_bits = _to_bf16_bits(scale * 2.0 ** 112)
    s_val = _bf16_bits_to_f64(s_bits)
    np.testing.assert_array_equal(s_val, scale * 2.0 ** 112)     # exact
    assert np.all(np.isfinite(s_val))
    vals = np.array([_e2m1(c) for c in range(16)])
    a = (vals * 2.0 ** -112)[:, None]                             # the re-encoded element
    prod = _bf16_bits_to_f64(_to_bf16_bits((a * s_val[None, :]).astype(np.float32)))
    np.testing.assert_array_equal(prod, vals[:, None] * scale[None, :])


def test_scale_zero_and_subnormals():
    # E4M3 0x00 (zero) and 0x01..0x07 (subnormal, 2^-9 .. 7 x 2^-9)
    b = np.arange(8, dtype=np.uint8)
    scale = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(scale, np.arange(8) * 2.0 ** -9)
    s_val = _bf16_bits_to_f64(_to_bf16_bits(scale * 2.0 ** 112))
    np.testing.assert_array_equal(s_val, scale * 2.0 ** 112)


# The GEMMs' f16 operands: the decoded weights and the token rows.

def test_f16_products_are_exact_for_every_code_and_scale():
    # every finite E4M3 scale is an f16 number, and so is every product with
    # an E2M1 value (at most 6 significant bits, 2^-10 .. 2688 in magnitude)
    finite = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)
    scale = torch.from_numpy(finite).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(scale.astype(np.float16).astype(np.float64), scale)
    vals = np.array([_e2m1(c) for c in range(16)])
    np.testing.assert_array_equal(vals.astype(np.float16).astype(np.float64), vals)
    prod16 = vals.astype(np.float16)[:, None] * scale.astype(np.float16)[None, :]   # f16 multiply
    np.testing.assert_array_equal(prod16.astype(np.float64), vals[:, None] * scale[None, :])
    nz = np.abs(vals[:, None] * scale[None, :])
    nz = nz[nz > 0]
    assert nz.min() == 2.0 ** -10 and nz.max() == 6 * 448      # normal f16 numbers


def _all_bf16() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32).astype(np.float64)
    return v[np.isfinite(v)]


def test_token_rows_as_f16_times_2_pow_minus_8():
    # bf16 -> f16(x * 2^-8), rounded to nearest: exact for 2^-9 <= |x| <=
    # 65504 * 2^8, within 2^-17 of x * 2^-8 * 2^8 below 2^-9, and beyond the
    # f16 range above 65504 * 2^8 (the kernels flag those)
    x = _all_bf16()
    y = (x * 2.0 ** -8).astype(np.float32).astype(np.float16).astype(np.float64) * 2.0 ** 8
    a = np.abs(x)
    inside = (a >= 2.0 ** -9) & (a <= 65504 * 2.0 ** 8)
    np.testing.assert_array_equal(y[inside], x[inside])
    small = a < 2.0 ** -9
    assert np.all(np.abs(y[small] - x[small]) <= 2.0 ** -17)
    big = a > 65504 * 2.0 ** 8
    assert big.any() and np.all(np.isinf(y[big]))
    # the bound is tight: something below 2^-9 does lose bits
    assert np.any(y[small] != x[small])
