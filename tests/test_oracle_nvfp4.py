"""Pins for the oracle's NVFP4 path (the 4-bit checkpoint format the Beam
pages name for Blackwell): the two small formats decoded from their
definitions against a closed form, the published E2M1 values and torch's
FP8 E4M3 cast; the NVFP4 expert against a numpy SwiGLU on independently
decoded weights; and its equality with the bf16 expert on the dequantized
weights, which are exact in bf16.  No GPU."""
import numpy as np
import torch
from scipy.special import expit

from group_limited_routing_sigmoid_b200 import workloads as W


def test_e2m1_values(oracle_lib):
    # sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal
    published = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for code in range(16):
        mag = published[code & 7]
        assert oracle_lib.e2m1_value(code) == (-mag if code & 8 else mag)
        e, m = (code >> 1) & 3, code & 1
        closed = (m * 0.5) if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
        assert abs(oracle_lib.e2m1_value(code)) == closed


def test_e4m3_values_match_torch(oracle_lib):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle_lib.e4m3_value(b) for b in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def _decode(codes, scales, gscale):
    """Independent NVFP4 decode with numpy and torch's E4M3 cast."""
    c = codes.astype(np.int64)
    nib = np.stack([c & 15, c >> 4], axis=-1).reshape(*codes.shape[:-1], -1)
    mag = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])[nib & 7]
    val = np.where(nib & 8, -mag, mag)
    sc = torch.from_numpy(scales).view(torch.float8_e4m3fn).double().numpy()
    return val * np.repeat(sc, 16, axis=-1) * gscale


def _silu(z):
    return z * expit(z)


def test_nvfp4_expert_matches_numpy_swiglu(oracle_lib):
    wl = W.WORKLOADS["tiny_nvfp4"]
    d = W.make_nvfp4_weights(wl, "cpu")
    x = W.bf16_bits(torch.randn(5, wl.hidden, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16))
    e = 3
    mats = [oracle_lib.Nvfp4Matrix(d[n + "_codes"][e].numpy(), d[n + "_scales"][e].numpy(), d[n + "_global"])
            for n in ("gate", "up", "down")]
    y, h = oracle_lib.expert_swiglu_nvfp4(x, *mats, want_h=True)
    wg, wu, wd = (_decode(m.codes, m.scales, m.global_scale) for m in mats)
    xf = oracle_lib.bf16_to_f64(x)
    g, u = xf @ wg.T, xf @ wu.T
    hb = W.bf16_bits(torch.from_numpy((_silu(g) * u).astype(np.float32)).to(torch.bfloat16))
    np.testing.assert_array_equal(h, hb)
    np.testing.assert_allclose(y, oracle_lib.bf16_to_f64(hb) @ wd.T, rtol=1e-10, atol=1e-14)


def test_nvfp4_expert_equals_bf16_expert_on_dequantized_weights(oracle_lib):
    """With per-tensor scales of 1, every NVFP4 weight (at most 6 significant
    bits) is a bf16 value, so the NVFP4 expert must equal the bf16 expert on
    those values exactly."""
    wl = W.WORKLOADS["tiny_nvfp4"]
    d = W.make_nvfp4_weights(wl, "cpu")
    x = W.bf16_bits(torch.randn(4, wl.hidden, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16))
    e = 7
    mats = [oracle_lib.Nvfp4Matrix(d[n + "_codes"][e].numpy(), d[n + "_scales"][e].numpy(), 1.0)
            for n in ("gate", "up", "down")]
    deq = [_decode(m.codes, m.scales, 1.0) for m in mats]
    bits = [W.bf16_bits(torch.from_numpy(w).to(torch.bfloat16)) for w in deq]
    for w, b in zip(deq, bits):                      # exactly representable
        np.testing.assert_array_equal(oracle_lib.bf16_to_f64(b), w)
    y4 = oracle_lib.expert_swiglu_nvfp4(x, *mats)
    y16 = oracle_lib.expert_swiglu(x, *bits)
    np.testing.assert_array_equal(y4, y16)


def test_quantizer_round_trip():
    """The input generator's encoding stays close to the weights it encodes."""
    w = torch.randn(64, 256, generator=torch.Generator().manual_seed(3)) * 0.02
    gs = W.nvfp4_global_scale(w)
    codes, scales = W.nvfp4_quantize(w, gs)
    deq = _decode(codes.numpy(), scales.numpy(), gs)
    rel = np.linalg.norm(deq - w.numpy()) / np.linalg.norm(w.numpy())
    assert rel < 0.15
