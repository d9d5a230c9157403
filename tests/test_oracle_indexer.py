"""Pins of the oracle's lightning indexer and top-k selection."""
import itertools

import numpy as np
import pytest

import oracle as O


def test_golden_scores(golden):
    g = golden("indexer_tiny.txt")
    qI = np.array([[[1, 0.5], [-1, 0]]], float)
    kI = np.array([[2, 2], [-1, 4], [1, -4]], float)
    w = np.array([[1, 0.5]])
    s = O.indexer_scores(qI, w, kI, [3])
    np.testing.assert_array_equal(s[0], np.array(g["scores"], float))
    s2 = O.indexer_scores(qI, w, kI, [2])
    assert s2[0, 2] == -np.inf and s2[0, 1] == 1.5


def test_golden_topk(golden):
    g = golden("indexer_tiny.txt")
    sc = np.array([g["tie_scores"]], float)
    assert O.topk_select(sc, [5], 2)[0].tolist() == [int(v) for v in g["tie_k2"]]
    assert O.topk_select(sc, [5], 4)[0].tolist() == [int(v) for v in g["tie_k4"]]
    assert O.topk_select(sc, [2], 3)[0].tolist() == [int(v) for v in g["short_nvis2_k3"]]


def _brute_topk(row, nv, k):
    """Exhaustive: the chosen set is the lexicographically smallest index set
    among all size-min(k,nv) subsets with the maximal score multiset."""
    best = None
    kk = min(k, nv)
    for comb in itertools.combinations(range(nv), kk):
        key = (sorted((-row[i] for i in comb)), comb)
        if best is None or key < best:
            best = key
    return list(best[1]) + [-1] * (k - kk)


def test_topk_brute_force_tiny():
    rng = np.random.default_rng(5)
    for trial in range(200):
        n = int(rng.integers(1, 8))
        k = int(rng.integers(1, 6))
        row = rng.integers(0, 4, n).astype(float)        # many ties
        nv = int(rng.integers(0, n + 1))
        got = O.topk_select(row[None], [nv], k)[0].tolist()
        assert got == (_brute_topk(row, nv, k) if nv > 0 else [-1] * k), (row, nv, k, got)


def test_relu_drops_negative_heads_and_w_is_linear():
    rng = np.random.default_rng(6)
    qI = rng.standard_normal((3, 4, 8)); kI = rng.standard_normal((10, 8)); w = rng.random((3, 4))
    s = O.indexer_scores(qI, w, kI, [10, 10, 10])
    assert np.all(s >= 0)
    np.testing.assert_allclose(O.indexer_scores(qI, 2 * w, kI, [10] * 3), 2 * s, rtol=1e-14)
    # a head whose dot products are all negative contributes nothing
    qI2 = qI.copy(); qI2[:, 0] = 0.0
    kneg = kI.copy()
    w0 = w.copy(); w0[:, 0] = 0
    np.testing.assert_allclose(O.indexer_scores(qI2, w, kneg, [10] * 3),
                               O.indexer_scores(qI, w0, kneg, [10] * 3), rtol=1e-14)
    # scaling a row of kI by a > 0 scales its scores by a (row scales factor out of the ReLU)
    k3 = kI.copy(); k3[4] *= 4.0
    np.testing.assert_allclose(O.indexer_scores(qI, w, k3, [10] * 3)[:, 4], 4 * s[:, 4], rtol=1e-14)


def test_single_head_unit_weight_is_relu_dot():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, 16)); k = rng.standard_normal((30, 16))
    s = O.indexer_scores(q, np.ones((1, 1)), k, [30])[0]
    for j in range(30):
        d = float(sum(q[0, 0, i] * k[j, i] for i in range(16)))
        assert s[j] == pytest.approx(max(d, 0.0), rel=1e-12, abs=1e-12)


def test_topk_k_at_least_nvis_returns_all_visible():
    rng = np.random.default_rng(8)
    sc = rng.random((5, 20))
    out = O.topk_select(sc, [0, 3, 7, 20, 20], 20)
    assert out[0].tolist() == [-1] * 20
    assert out[1].tolist() == [0, 1, 2] + [-1] * 17
    assert out[3].tolist() == list(range(20))


def test_grid_inputs_are_exact_in_fp32():
    """On the 1/8 grid (w on 1/16) every score is a multiple of 2^-10 below 2^13,
    so fp32 computes it exactly in any order; checked on the tiny workload."""
    from long_context_compressed_02_b200 import synth
    inp, cfg = synth.prefill_inputs("tiny_csa")
    qI = O.e4m3_decode(inp["qI_codes"]); kI = O.e4m3_decode(inp["kI_codes"])
    assert np.all(np.round(qI * 8) == qI * 8) and np.all(np.round(kI * 8) == kI * 8)
    nv = O.n_visible(np.arange(cfg["S"]), cfg["m"])
    s = O.indexer_scores(qI, inp["w"], kI, nv)
    fin = s[np.isfinite(s)]
    assert np.all(np.round(fin * 1024) == fin * 1024) and np.abs(fin).max() < 2 ** 13
    assert np.array_equal(fin.astype(np.float32).astype(np.float64), fin)
