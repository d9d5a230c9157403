"""Pins of the oracle's KV compressor (CSA m=4 overlapping, HCA m'=128)."""
import math

import numpy as np
import pytest

import oracle as O


def _tiny():
    C = np.array([[1, 10], [2, 20], [3, 30], [4, 40], [5, 50]], float)
    Z = np.zeros((5, 2)); Z[:, 0] = [0, math.log(3), 0, math.log(3), 0]
    Bo = np.zeros((4, 2)); Bo[0, 1] = math.log(2)
    return C, Z, Bo


def test_golden_hand_example(golden):
    g = golden("compress_tiny.txt")
    C, Z, Bo = _tiny()
    kv = O.compress(C, Z, Bo, 2, True)
    assert kv.shape == (2, 2)                       # token 4 is a tail token
    np.testing.assert_allclose(kv.ravel(), np.array(g["overlap_joint"], float), rtol=1e-14)
    sep = O.compress(C, Z, Bo, 2, True, joint_softmax=False)
    np.testing.assert_allclose(sep[1], np.array(g["overlap_separate_entry1"], float), rtol=1e-14)
    kv2 = O.compress(C, Z, np.zeros((2, 2)), 2, False)
    np.testing.assert_allclose(kv2.ravel(), np.array(g["nonoverlap"], float), rtol=1e-14)


@pytest.mark.parametrize("S,m,ne", [(2048, 4, 512), (16384, 4, 4096), (131072, 128, 1024),
                                    (1 << 20, 4, 262144), (2050, 4, 512), (127, 128, 0)])
def test_entry_counts(S, m, ne):
    assert O.n_entries(S, m) == ne


def test_page_derived_counts():
    # 1M tokens at m'=128 gives about 7812 entries; top-k 1024 at m=4 reads
    # about 4096 token-equivalents (liduos.com, "1M Context 的结构与取舍").
    assert O.n_entries(10 ** 6, 128) == 7812
    assert 1024 * 4 == 4096


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 4), (False, 128), (True, 2)])
def test_constant_logits_give_block_mean(overlap, m):
    rng = np.random.default_rng(0)
    S, D = 6 * m + 3, 5
    C = rng.standard_normal((S, D))
    Z = np.full((S, D), 0.7)
    B = np.zeros((2 * m if overlap else m, D))
    kv = O.compress(C, Z, B, m, overlap)
    for i in range(S // m):
        lo = (i - 1) * m if (overlap and i > 0) else i * m
        np.testing.assert_allclose(kv[i], C[lo:(i + 1) * m].mean(axis=0), rtol=1e-13, atol=1e-14)


def test_dominant_logit_selects_one_token():
    rng = np.random.default_rng(1)
    m, S, D = 4, 40, 3
    C = rng.standard_normal((S, D)); Z = rng.standard_normal((S, D)); B = np.zeros((2 * m, D))
    for i in range(1, S // m):
        for j in range((i - 1) * m, (i + 1) * m):
            Zj = Z.copy(); Zj[j] += 1e4
            np.testing.assert_allclose(O.compress(Zj * 0 + C, Zj, B, m, True)[i], C[j], rtol=1e-12)


def test_bias_rows_belong_to_previous_then_current_block():
    m, D = 4, 1
    C = np.arange(12, dtype=float)[:, None]
    Z = np.zeros((12, 1))
    for r in range(2 * m):
        B = np.zeros((2 * m, D)); B[r] = 1e4
        kv = O.compress(C, Z, B, m, True)
        # entry 1 pools rows 0..7: bias row r picks row r (previous block first)
        assert kv[1, 0] == pytest.approx(float(r))
        # entry 0 has no previous block: only bias rows m..2m-1 act on rows 0..3
        if r >= m:
            assert kv[0, 0] == pytest.approx(float(r - m))


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 8)])
def test_overlap_footprint(overlap, m):
    rng = np.random.default_rng(2)
    S, D = 10 * m + 3, 4
    C = rng.standard_normal((S, D)); Z = rng.standard_normal((S, D))
    B = 0.1 * rng.standard_normal((2 * m if overlap else m, D))
    base = O.compress(C, Z, B, m, overlap)
    ne = S // m
    for j in range(S):
        C2 = C.copy(); C2[j] += 1.0
        changed = set(np.nonzero(np.any(O.compress(C2, Z, B, m, overlap) != base, axis=1))[0])
        expect = {j // m} | ({j // m + 1} if overlap else set())
        expect = {e for e in expect if e < ne}
        assert changed == expect, (j, changed, expect)


def test_convex_combination_bounds():
    rng = np.random.default_rng(3)
    m, S, D = 4, 64, 16
    C = rng.standard_normal((S, D)); Z = 3 * rng.standard_normal((S, D)); B = rng.standard_normal((2 * m, D))
    kv = O.compress(C, Z, B, m, True)
    for i in range(S // m):
        lo = max(0, (i - 1) * m)
        blk = C[lo:(i + 1) * m]
        assert np.all(kv[i] <= blk.max(axis=0) + 1e-12) and np.all(kv[i] >= blk.min(axis=0) - 1e-12)


def test_rmsnorm_and_rope_closed_forms():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((7, 512)) * 3
    y = O.rmsnorm(x)
    np.testing.assert_allclose((y * y).mean(axis=-1), 1.0 / (1.0 + 1e-6 / (x * x).mean(axis=-1)), rtol=1e-12)
    # RoPE: identity at position 0; norm-preserving; only the last 64 dims move
    np.testing.assert_array_equal(O.rope_partial(x, np.zeros(7)), x)
    r = O.rope_partial(x, np.arange(7) * 1000.0)
    np.testing.assert_array_equal(r[:, :448], x[:, :448])
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # inverse rotation undoes it
    np.testing.assert_allclose(O.rope_partial(r, np.arange(7) * 1000.0, inverse=True), x, atol=1e-12)
    # pair 0 has frequency 1: (1, 0) at position p -> (cos p, sin p); pair j has 10000^(-2j/64)
    e = np.zeros((1, 64)); e[0, 0] = 1.0; e[0, 5] = 1.0
    out = O.rope_partial(e, np.array([100.0]))
    assert out[0, 0] == pytest.approx(math.cos(100.0)) and out[0, 32] == pytest.approx(math.sin(100.0))
    f5 = 10000.0 ** (-10.0 / 64.0)
    assert out[0, 5] == pytest.approx(math.cos(100.0 * f5)) and out[0, 37] == pytest.approx(math.sin(100.0 * f5))
    # relative-position property on the rotated dims
    a = rng.standard_normal(64); b = rng.standard_normal(64)
    d1 = O.rope_partial(a[None], np.array([5.0]))[0] @ O.rope_partial(b[None], np.array([2.0]))[0]
    d2 = O.rope_partial(a[None], np.array([103.0]))[0] @ O.rope_partial(b[None], np.array([100.0]))[0]
    assert d1 == pytest.approx(d2, rel=1e-10)
