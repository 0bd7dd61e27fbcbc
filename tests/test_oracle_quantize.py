"""Pins of the oracle's 4-bit key quantiser against things other than itself:
a hand-worked example, a scalar re-derivation through IEEE conversions done by
the struct module, the error bound of round-to-nearest, and the memory figure
on the pages (about 1/8 of the KV cache)."""
import json
import math
import os
import struct

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def _f16(x: float) -> float:
    return struct.unpack("<e", struct.pack("<e", x))[0]


def _total_key(v: float):
    return (v, math.copysign(1.0, v))


def _scalar_group(vals):
    """Group quantisation by scalar IEEE steps: each fp32 op is done in fp64 and
    rounded once to fp32 (exact for +,-,/ of fp32 operands since 53 >= 2*24+2)."""
    mn = min(vals, key=_total_key)
    mx = max(vals, key=_total_key)
    d = _f32(mx - mn)
    scale = _f16(_f32(d / 15.0))
    codes = []
    for x in vals:
        if scale == 0.0:
            codes.append(0)
            continue
        r = _f32(_f32(x - mn) / scale)
        codes.append(min(15, max(0, int(round(r)))))   # round(): ties to even
    return codes, scale, mn


def test_worked_example_golden():
    g = json.load(open(os.path.join(GOLDEN, "quantize_worked_example.json")))
    x = np.array(sum(g["x_groups"], []), dtype=np.float16)
    codes, scales, zeros = O.quantize_keys(x[None])
    u = O.unpack_codes(codes)[0]
    assert u.tolist() == sum(g["expected_codes"], [])
    assert scales[0].astype(float).tolist() == g["expected_scales"]
    assert zeros[0].astype(float).tolist() == g["expected_zeros"]
    for i, b in g["expected_first_bytes"].items():
        assert int(codes[0, int(i)]) == b


def test_matches_scalar_ieee_rederivation():
    rng = np.random.default_rng(7)
    k = rng.standard_normal((40, 128)).astype(np.float32)
    k[3] *= 1e-6                       # tiny / subnormal fp16 range
    k[4] = 0.0
    k[4, 5] = -0.0
    k[5, 32:64] = 2.0 ** -24           # all-equal subnormal group
    k[6] *= 3000.0                     # large magnitudes
    k[7, :32] = np.linspace(-1, 1, 32)  # many exact halves
    k16 = k.astype(np.float16)
    codes, scales, zeros = O.quantize_keys(k16)
    u = O.unpack_codes(codes)
    for t in range(k16.shape[0]):
        for g in range(4):
            vals = [float(v) for v in k16[t, 32 * g:32 * (g + 1)]]
            c, s, mn = _scalar_group(vals)
            assert u[t, 32 * g:32 * (g + 1)].tolist() == c, (t, g)
            assert float(scales[t, g]) == s
            assert zeros[t, g].tobytes() == np.float16(mn).tobytes()


def test_group_extremes_and_error_bound():
    rng = np.random.default_rng(11)
    k16 = rng.standard_normal((500, 128)).astype(np.float16)
    codes, scales, zeros = O.quantize_keys(k16)
    u = O.unpack_codes(codes).reshape(500, 4, 32)
    x = k16.astype(np.float64).reshape(500, 4, 32)
    khat = O.dequantize_keys(codes, scales, zeros).reshape(500, 4, 32)
    s = scales.astype(np.float64)
    assert np.all(s > 0)
    # the group minimum maps to code 0 and the maximum to code 15
    assert np.all(u[np.arange(500)[:, None], np.arange(4)[None], x.argmin(-1)] == 0)
    assert np.all(u[np.arange(500)[:, None], np.arange(4)[None], x.argmax(-1)] == 15)
    # round-to-nearest error bound, widened by the fp16 rounding of the scale
    err = np.abs(x - khat)
    assert np.all(err <= s[..., None] * 0.5 * (1 + 2.0 ** -9) + 1e-12)
    assert np.all(zeros.astype(np.float64) == x.min(-1))


def test_all_equal_group_is_exact():
    k16 = np.full((3, 128), 0.3, dtype=np.float16)
    k16[1] = -7.0
    codes, scales, zeros = O.quantize_keys(k16)
    assert np.all(scales == 0) and np.all(codes == 0)
    np.testing.assert_array_equal(O.dequantize_keys(codes, scales, zeros), k16.astype(np.float64))


def test_negative_zero_total_order():
    x = np.zeros(128, np.float16)
    x[3] = np.float16(-0.0)
    x[40] = 1.0
    x[41] = np.float16(-0.0)
    x[42] = 0.0
    _, _, zeros = O.quantize_keys(x[None])
    # -0 is below +0 under totalOrder, so it is the stored zero point
    assert zeros[0, 0].view(np.uint16) == 0x8000
    assert zeros[0, 1].view(np.uint16) == 0x8000
    assert zeros[0, 2].view(np.uint16) == 0x0000


def test_numpy_fp16_rounding_is_ieee_rne():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, size=100000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) < 65504)]
    # exact halfway points between fp16 neighbours
    h = np.arange(0, 0x7BFF, 37, dtype=np.uint16).view(np.float16).astype(np.float32)
    mid = ((h.astype(np.float64) + np.nextafter(h.astype(np.float16), np.float16(np.inf))
            .astype(np.float64)) / 2).astype(np.float32)
    x = np.concatenate([x[:20000], mid])
    got = x.astype(np.float16).view(np.uint16)
    ref = np.array([struct.unpack("<H", struct.pack("<e", float(v)))[0] for v in x], np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_memory_overhead_is_one_eighth():
    # "about 1/8 extra KV cache" for the INT4 key cache (atlas.scime.ai, Limitations)
    codes_only = O.int4_cache_bytes_per_token(with_scale_zero=False)
    kv = O.kv_cache_bytes_per_token()
    assert codes_only * 8 == kv
    k16 = np.zeros((16, 128), np.float16)
    codes, scales, zeros = O.quantize_keys(k16)
    assert codes.nbytes == 16 * codes_only
    assert codes.nbytes + scales.nbytes + zeros.nbytes == 16 * O.int4_cache_bytes_per_token()
    assert (scales.nbytes + zeros.nbytes) * 32 == 16 * kv


def test_nibble_order_even_channel_low():
    x = np.zeros(128, np.float16)
    x[0:32] = np.arange(32) % 2 * 15     # odd channels = max -> 15, even -> 0
    codes, _, _ = O.quantize_keys(x[None])
    assert np.all(codes[0, :16] == 0xF0)
