"""Pins of the oracle's FP4 formats for the lightning indexer's QK path ("DeepSeek
V4 脱离 CUDA 全栈国产化 ..." §二 "闪电索引器" and "其他辅助设计"): E2M1 elements, E8M0
block scales, MX blocks of 32, two elements per byte."""
import numpy as np
import pytest
import torch

import oracle as O


def test_e2m1_decode_golden(golden):
    g = golden("e2m1_codes.txt")
    assert len(g) == 16
    for code, (val,) in g.items():
        got = O.e2m1_decode(int(code, 16))
        assert got == float(val) and np.signbit(got) == val.startswith("-"), code


def test_e8m0_decode_matches_torch():
    b = np.arange(255, dtype=np.uint8)
    ref = torch.from_numpy(b).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e8m0_decode(b), ref)
    assert np.isnan(O.e8m0_decode(255))


def test_e2m1_encode_is_nearest_with_ties_to_even():
    """Exhaustive search over the representable values decides every case."""
    vals = O.e2m1_decode(np.arange(16))
    rng = np.random.default_rng(0)
    mids = (np.unique(vals)[1:] + np.unique(vals)[:-1]) / 2        # every tie point
    x = np.concatenate([rng.uniform(-8, 8, 4000), mids, -mids, np.unique(vals), [6.5, -7.0, 1e9]])
    codes = O.e2m1_encode(x)
    got = O.e2m1_decode(codes)
    for xi, ci, gi in zip(x, codes, got):
        a = min(abs(xi), 6.0)
        d = np.abs(np.abs(vals[:8]) - a)
        best = np.flatnonzero(d == d.min())
        assert abs(abs(gi) - np.abs(vals[best[0]])) == 0 or len(best) > 1, xi
        assert (ci & 0x7) in best, xi
        if len(best) > 1:                        # a tie: the even code (mantissa bit 0) wins
            assert (ci & 0x1) == 0, xi
        assert gi == 0 or np.sign(gi) == np.sign(xi)
    # hand cases: ties 0.25 -> 0, 0.75 -> 1, 2.5 -> 2, 5 -> 4; saturation
    np.testing.assert_array_equal(O.e2m1_decode(O.e2m1_encode([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -100.0])),
                                  [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, -6.0])


def test_e2m1_roundtrip():
    c = np.arange(16, dtype=np.uint8)
    rt = O.e2m1_encode(O.e2m1_decode(c))
    np.testing.assert_array_equal(rt[c != 8], c[c != 8])
    assert rt[8] == 0                            # negative zero is not produced


def test_fp4_pack_layout_and_roundtrip():
    np.testing.assert_array_equal(O.fp4_pack([1, 2, 15, 0]), [0x21, 0x0F])   # even element in the low nibble
    rng = np.random.default_rng(1)
    c = rng.integers(0, 16, (5, 128)).astype(np.uint8)
    p = O.fp4_pack(c)
    assert p.shape == (5, 64)
    np.testing.assert_array_equal(O.fp4_unpack(p), c)


def test_mxfp4_block_scale_and_error_bound():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 128)) * np.exp2(rng.integers(-6, 7, (64, 1)))
    codes, sc = O.mxfp4_quantize(x)
    assert codes.shape == x.shape and sc.shape == (64, 4)
    scale = O.e8m0_decode(sc)
    amax = np.abs(x.reshape(64, 4, 32)).max(-1)
    r = amax / scale
    assert np.all((r >= 4) & (r < 8))            # the block maximum lands in [4, 8) before saturation
    deq = O.mxfp4_dequantize(codes, sc)
    y = x / np.repeat(scale, 32, axis=1)
    vals = np.unique(np.abs(O.e2m1_decode(np.arange(8))))
    # every element is its nearest grid value (saturating at 6), scaled back
    a = np.minimum(np.abs(y), 6.0)
    nearest = np.abs(a[..., None] - vals).min(-1)
    np.testing.assert_allclose(np.abs(np.abs(deq / np.repeat(scale, 32, axis=1)) - a), nearest, atol=1e-12)


def test_mxfp4_power_of_two_invariance_and_footprint():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 128))
    c0, s0 = O.mxfp4_quantize(x)
    c1, s1 = O.mxfp4_quantize(x * 8.0)
    np.testing.assert_array_equal(c1, c0)
    np.testing.assert_array_equal(s1.astype(int), s0.astype(int) + 3)
    x2 = x.copy()
    x2[:, 32:64] *= 100.0                         # only block 1 changes
    c2, s2 = O.mxfp4_quantize(x2)
    keep = np.ones(128, bool); keep[32:64] = False
    np.testing.assert_array_equal(c2[:, keep], c0[:, keep])
    np.testing.assert_array_equal(s2[:, [0, 2, 3]], s0[:, [0, 2, 3]])
    z, sz = O.mxfp4_quantize(np.zeros((1, 32)))
    assert sz[0, 0] == 0 and not z.any()
    with pytest.raises(ValueError):
        O.mxfp4_quantize(np.zeros((1, 33)))
