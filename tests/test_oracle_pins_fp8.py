"""Pins of the oracle's FP8 dispatch payload against facts outside the oracle.

The payload follows the reading stated in the oracle (OCP FP8 E4M3, one fp32
scale per token and 128-channel block, scale = amax / 448; the pages only say
that lower-precision activations cut dispatch bytes at a numerical price,
"DeepSeek 8.7 - communication", section 4).  Pinned by: torch's own
float8_e4m3fn type (decode of all 256 codes, nearest-even encode), the
format's closed forms (448 saturation, subnormal spacing), the quantizer's
error bound, and the layer composed from its steps.
"""
import numpy as np
import pytest
import torch

import synth


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _bf16_np(t):
    return t.float().numpy().astype(np.float64)


def _torch_e4m3(v):
    return int(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8))


def test_decode_matches_torch_for_all_codes(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([orc.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all() and nan.sum() == 2       # 0x7F and 0xFF only
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert orc.e4m3_decode(0x7E) == 448.0 and orc.e4m3_decode(0x01) == 2.0 ** -9
    assert orc.e4m3_decode(0x08) == 2.0 ** -6                    # smallest normal


def test_encode_matches_torch_nearest_even(orc):
    rng = np.random.default_rng(0)
    vals = list(rng.normal(0, 30, 400)) + list(rng.normal(0, 0.01, 200))
    codes = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (codes[:-1] + codes[1:]) / 2                           # exact ties
    vals += list(mids) + list(-mids) + [0.0, -0.0, 2.0 ** -10, 2.0 ** -11, 447.9, 463.9, -463.9]
    for v in vals:
        v32 = float(np.float32(v))
        assert orc.e4m3_encode(v32) == _torch_e4m3(v32), v32


def test_encode_saturates_at_448(orc):
    for v in (464.0, 470.0, 1e4, 3e38):
        assert orc.e4m3_encode(v) == 0x7E
        assert orc.e4m3_encode(-v) == 0xFE


def _rows(n, d, seed, sigma=1.0):
    return synth.normal(seed, 40, (n, d), sigma, torch.bfloat16)


def test_quantize_scale_and_amax_code(orc):
    x = _rows(6, 384, 1)
    q, sc = orc.fp8_quantize(x)
    xs = _bf16_np(x).reshape(6, 3, 128)
    amax = np.abs(xs).max(axis=2).astype(np.float32)
    np.testing.assert_array_equal(sc, amax / np.float32(448.0))
    # the element holding the block maximum encodes to +-448
    qb = q.reshape(6, 3, 128)
    for r in range(6):
        for b in range(3):
            i = int(np.abs(xs[r, b]).argmax())
            assert qb[r, b, i] & 0x7F == 0x7E


def test_quantize_error_bound(orc):
    """|x_hat - x| <= 2^-4 |x| (3 mantissa bits, nearest) in the normal range,
    <= 2^-10 s in the subnormal range, plus one bf16 rounding of x_hat."""
    x = _rows(8, 256, 2, sigma=3.0)
    q, sc = orc.fp8_quantize(x)
    xh = orc.fp8_dequantize(q, sc)
    xv = _bf16_np(x)
    xhv = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).double().numpy()
    s = np.repeat(sc, 128, axis=1).astype(np.float64)
    bound = np.maximum(2.0 ** -4 * np.abs(xv), 2.0 ** -10 * s) * (1 + 2.0 ** -8) + 2.0 ** -9 * np.abs(xhv)
    assert (np.abs(xhv - xv) <= bound + 1e-30).all()
    assert np.abs(xhv - xv).max() > 0                            # it does quantize


def test_quantize_zero_block_and_exact_values(orc):
    x = np.zeros((2, 256), np.float32)
    x[1, 128:] = np.tile([1.0, -2.0, 0.5, 448.0 / 56], 32)       # powers of two scale exactly
    xb = _bf16(x)
    q, sc = orc.fp8_quantize(xb)
    assert (q[0] == 0).all() and (sc[0] == 0).all() and (q[1, :128] == 0).all()
    xh = orc.fp8_dequantize(q, sc)
    back = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(back, xb.float().numpy())      # exactly representable values


def test_layer_with_fp8_payload_equals_composed_steps(orc):
    shape = synth.MoeShape("fp8mini", T=10, d=128, E=8, G=4, K=4, M=2, d_ff=16, n_shared=1,
                           d_ff_shared=8, x_sigma=1, e_sigma=1, bias_sigma=0.1)
    rng = np.random.default_rng(9)
    x = _bf16(rng.normal(size=(10, 128)))
    e = rng.normal(0, 0.1, size=(8, 128)).astype(np.float32)
    bias = rng.normal(0, 0.1, size=8).astype(np.float32)
    Wg = [_bf16(rng.normal(size=(16, 128)) / 11) for _ in range(8)]
    Wu = [_bf16(rng.normal(size=(16, 128)) / 11) for _ in range(8)]
    Wd = [_bf16(rng.normal(size=(128, 16)) / 4) for _ in range(8)]
    Sg, Su = _bf16(rng.normal(size=(1, 8, 128)) / 11), _bf16(rng.normal(size=(1, 8, 128)) / 11)
    Sd = _bf16(rng.normal(size=(1, 128, 8)) / 3)
    out, idx, w, _ = orc.layer_rows(range(10), shape, x, e, bias, Wg, Wu, Wd, Sg, Su, Sd,
                                    payload=1)
    out0, idx0, w0, _ = orc.layer_rows(range(10), shape, x, e, bias, Wg, Wu, Wd, Sg, Su, Sd)
    np.testing.assert_array_equal(idx, idx0)                     # the router keeps x
    np.testing.assert_array_equal(w, w0)
    q, sc = orc.fp8_quantize(x)
    xh = torch.from_numpy(orc.fp8_dequantize(q, sc).view(np.int16)).view(torch.bfloat16)
    want = np.stack([orc.shared_row(x[t], Sg, Su, Sd) + sum(
        float(w[t, j]) * orc.ffn_row(xh[t], Wg[idx[t, j]], Wu[idx[t, j]], Wd[idx[t, j]])
        for j in range(4)) for t in range(10)])
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)
    rel = np.linalg.norm(out - out0) / np.linalg.norm(out0)
    assert 1e-3 < rel < 0.1                                      # the price of the compression
