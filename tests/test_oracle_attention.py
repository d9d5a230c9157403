"""Pins of the oracle's attention steps: shared K=V softmax attention, the
sliding window, the attention sink, and the whole-layer compositions checked
against a second (masked score matrix) formulation."""
import math

import numpy as np
import pytest

import oracle as O


def test_attend_rows_closed_forms():
    rows = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]])
    q0 = np.zeros((1, 2))
    Oh, l = O.attend_rows(q0, rows, 1 / math.sqrt(2))
    np.testing.assert_allclose(Oh[0], [3.0, 4.0], rtol=1e-15)          # equal logits: mean
    assert l[0] == pytest.approx(math.log(3.0))
    # with a sink s: O = sum(rows) / (n + e^s)
    m = O.merge_partials([(Oh, l)], sink=np.array([math.log(3.0)]))
    np.testing.assert_allclose(m[0], [9 / 6, 12 / 6], rtol=1e-14)
    # two rows with logits ln2 and 0 -> weights 2/3, 1/3
    q = np.array([[math.log(2.0) * math.sqrt(2.0), 0.0]])
    Oh, _ = O.attend_rows(q, np.array([[1.0, 0.0], [0.0, 0.0]]), 1 / math.sqrt(2))
    np.testing.assert_allclose(Oh[0], [2 / 3, 0.0], rtol=1e-14)
    # a single row is returned unchanged (K = V)
    Oh, l = O.attend_rows(np.ones((4, 2)), rows[1:2], 0.3)
    np.testing.assert_allclose(Oh, np.repeat(rows[1:2], 4, 0), rtol=1e-15)


def test_sink_limits():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((3, 16)); rows = rng.standard_normal((9, 16))
    Oh, l = O.attend_rows(q, rows, 0.25)
    np.testing.assert_allclose(O.merge_partials([(Oh, l)], sink=np.full(3, -1e300)), Oh, rtol=1e-14)
    np.testing.assert_allclose(O.merge_partials([(Oh, l)], sink=np.full(3, 1e300)), 0.0, atol=0)
    # merging a split of the rows equals attending over all of them
    a = O.attend_rows(q, rows[:4], 0.25); b = O.attend_rows(q, rows[4:], 0.25)
    np.testing.assert_allclose(O.merge_partials([a, b]), Oh, rtol=1e-13)


def _layer_inputs(S, H, D, m, HI=4, DI=16, seed=0, nb=None):
    rng = np.random.default_rng(seed)
    nb = 2 * m if nb is None else nb
    return dict(q=rng.standard_normal((S, H, D)), C=rng.standard_normal((S, D)),
                Z=rng.standard_normal((S, D)), B=0.1 * rng.standard_normal((nb, D)),
                qI=np.round(rng.standard_normal((S, HI, DI)) * 8) / 8,
                w=np.floor(rng.random((S, HI)) * 16) / 16,
                kI=np.round(rng.standard_normal((S // m, DI)) * 8) / 8,
                sink=rng.standard_normal(H))


@pytest.mark.parametrize("norm_rope,k", [(False, 5), (True, 7), (True, 1000)])
def test_csa_gather_matches_matrix_formulation(norm_rope, k):
    x = _layer_inputs(203, 3, 64, 4)
    kw = dict(k=k, m=4, W=16, norm_rope=norm_rope, inv_rope=norm_rope)
    Og, _ = O.csa_layer(x["q"], x["C"], x["Z"], x["B"], x["qI"], x["w"], x["kI"], x["sink"], **kw)
    Om = O.csa_layer_matrix(x["q"], x["C"], x["Z"], x["B"], x["qI"], x["w"], x["kI"], x["sink"], **kw)
    np.testing.assert_allclose(Og, Om, rtol=1e-11, atol=1e-12)


def test_hca_gather_matches_matrix_formulation():
    x = _layer_inputs(600, 2, 64, 32, nb=32)
    kw = dict(m=32, W=40, norm_rope=True, inv_rope=True)
    Og = O.hca_layer(x["q"], x["C"], x["Z"], x["B"], x["sink"], **kw)
    Om = O.hca_layer_matrix(x["q"], x["C"], x["Z"], x["B"], x["sink"], **kw)
    np.testing.assert_allclose(Og, Om, rtol=1e-11, atol=1e-12)


def test_topk_at_least_entries_is_dense_attention():
    x = _layer_inputs(160, 2, 32, 4)
    Og, idx = O.csa_layer(x["q"], x["C"], x["Z"], x["B"], x["qI"], x["w"], x["kI"], x["sink"],
                          k=40, m=4, W=8)
    kv = O.compress(x["C"], x["Z"], x["B"], 4, True)
    t = np.arange(160)
    Op, lp = O.dense_attention_partial(x["q"], kv, O.n_visible(t, 4))
    Od = O.window_sink_combine(x["q"], x["C"], t, 8, x["sink"], Op, lp)
    np.testing.assert_allclose(Og, Od, rtol=1e-12, atol=1e-13)
    assert np.all((idx >= 0).sum(axis=1) == O.n_visible(t, 4))


def test_no_visible_entry_is_window_plus_sink():
    x = _layer_inputs(40, 2, 16, 4)
    x["q"][:] = 0.0                                   # equal logits: closed form
    Og, idx = O.csa_layer(x["q"], x["C"], x["Z"], x["B"], x["qI"], x["w"], x["kI"], x["sink"],
                          k=4, m=4, W=128)
    for t in range(3):                                # t < m-1: nothing compressed yet
        assert np.all(idx[t] == -1)
        expect = x["C"][:t + 1].sum(axis=0)[None, :] / ((t + 1) + np.exp(x["sink"]))[:, None]
        np.testing.assert_allclose(Og[t], expect, rtol=1e-13)


def test_causality_bit_exact():
    x = _layer_inputs(120, 2, 96, 4, seed=3)
    kw = dict(k=6, m=4, W=10, norm_rope=True, inv_rope=True)
    base, _ = O.csa_layer(**{k: x[k] for k in ("q", "C", "Z", "B", "qI", "w", "kI", "sink")}, **kw)
    for t in (0, 3, 4, 57, 118):
        y = {k: v.copy() for k, v in x.items()}
        for key in ("q", "C", "Z", "qI", "w"):
            y[key][t + 1:] += 1.0
        y["kI"][(t + 1) // 4:] += 1.0                 # entries not yet complete at t
        out, _ = O.csa_layer(**{k: y[k] for k in ("q", "C", "Z", "B", "qI", "w", "kI", "sink")}, **kw)
        np.testing.assert_array_equal(out[:t + 1], base[:t + 1])


def test_tail_tokens_only_reach_the_window():
    x = _layer_inputs(2050, 1, 16, 4, seed=4)
    kw = dict(k=8, m=4, W=128)
    rows = np.array([2047, 2048, 2049])
    base, _ = O.csa_layer(**{k: x[k] for k in ("q", "C", "Z", "B", "qI", "w", "kI", "sink")}, rows=rows, **kw)
    assert O.n_entries(2050, 4) == 512 and x["kI"].shape[0] == 512
    y = {k: v.copy() for k, v in x.items()}
    y["C"][2049] += 1.0; y["Z"][2049] += 5.0
    out, _ = O.csa_layer(**{k: y[k] for k in ("q", "C", "Z", "B", "qI", "w", "kI", "sink")}, rows=rows, **kw)
    np.testing.assert_array_equal(out[:2], base[:2])      # t = 2047, 2048 unaffected
    assert not np.array_equal(out[2], base[2])             # t = 2049 sees it in its window


def test_inverse_rope_undoes_a_common_rotation():
    # If every key/value row carries the query's own rotation (all rows at
    # position t), the inverse RoPE of the output returns the unrotated average.
    rng = np.random.default_rng(5)
    rows = rng.standard_normal((6, 128)); t = 77
    rot = O.rope_partial(rows, np.full(6, t))
    q = np.zeros((1, 1, 128))
    Oh, l = O.attend_rows(q[0], rot, 0.1)
    back = O.rope_partial(Oh, np.array([[t]]), inverse=True)
    np.testing.assert_allclose(back[0], rows.mean(axis=0), atol=1e-13)


def test_decode_matches_prefill_last_row():
    """Decode at the newest position equals the prefill layer's last row when
    the caches hold the prefill's entries and the last W raw rows."""
    x = _layer_inputs(64, 2, 32, 4, seed=6)
    S = 64; t = S - 1
    Og, idx = O.csa_layer(x["q"], x["C"], x["Z"], x["B"], x["qI"], x["w"], x["kI"], x["sink"],
                          k=5, m=4, W=16)
    kv = O.compress(x["C"], x["Z"], x["B"], 4, True)
    Od, idd = O.csa_decode(x["q"][t], x["qI"][t], x["w"][t], x["kI"], kv, x["C"][t - 15:t + 1],
                           x["sink"], t, k=5, m=4, inv_rope=False)
    np.testing.assert_array_equal(idd, idx[t])
    np.testing.assert_allclose(Od, Og[t], rtol=1e-13)


def _decode_operands(x, t, m, overlap, W, norm_rope):
    """The decode functions' inputs at position t, built from the prefill
    definitions: the query row, every cache entry, and the raw window rows
    [max(0, t - W + 1), t], each normalised and rotated when norm_rope."""
    kv = O.compress(x["C"], x["Z"], x["B"], m, overlap)
    lo = max(0, t - W + 1)
    q, swa = x["q"][t], x["C"][lo:t + 1]
    if norm_rope:
        q = O.rope_partial(O.rmsnorm(q), np.full(q.shape[0], t))
        kv = O.rope_partial(O.rmsnorm(kv), np.arange(kv.shape[0]) * m)
        swa = O.rope_partial(O.rmsnorm(swa), np.arange(lo, t + 1))
    return q, kv, swa


@pytest.mark.parametrize("norm_rope", [False, True])
@pytest.mark.parametrize("t", [255, 128, 129, 20])
def test_hca_decode_matches_prefill_row(norm_rope, t):
    """[CS] "HCA": dense attention over every complete 128-token entry; [LD]:
    plus the 128-token raw window and the sink in one softmax, inverse RoPE on
    the output.  Decoding the token at position t against caches that hold the
    prefill's entries and the last W raw rows must reproduce row t of the
    prefill layer: at the last position, at the first token after a block
    boundary (a newly visible entry), one token later, and before any entry is
    complete (window only)."""
    m, W, S = 32, 40, 256
    x = _layer_inputs(S, 3, 128, m, nb=m, seed=7)
    Og = O.hca_layer(x["q"], x["C"], x["Z"], x["B"], x["sink"], m=m, W=W, norm_rope=norm_rope,
                     inv_rope=norm_rope)
    q, kv, swa = _decode_operands(x, t, m, False, W, norm_rope)
    Od = O.hca_decode(q, kv, swa, x["sink"], t, m=m, inv_rope=norm_rope)
    np.testing.assert_allclose(Od, Og[t], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("norm_rope", [False, True])
@pytest.mark.parametrize("t", [255, 128, 129])
def test_csa_decode_matches_prefill_row_with_rope(norm_rope, t):
    """As test_decode_matches_prefill_last_row, with the QK normalisation, the
    partial RoPE of queries, entries and window rows, and the inverse RoPE of
    the output ([CS] "其他辅助设计"; [LD]), at a block boundary as well."""
    m, W, S = 4, 40, 256
    x = _layer_inputs(S, 3, 128, m, seed=8)
    Og, idx = O.csa_layer(x["q"], x["C"], x["Z"], x["B"], x["qI"], x["w"], x["kI"], x["sink"], k=9, m=m, W=W,
                          norm_rope=norm_rope, inv_rope=norm_rope)
    q, kv, swa = _decode_operands(x, t, m, True, W, norm_rope)
    Od, idd = O.csa_decode(q, x["qI"][t], x["w"][t], x["kI"], kv, swa, x["sink"], t, k=9, m=m,
                           inv_rope=norm_rope)
    np.testing.assert_array_equal(idd, idx[t])
    np.testing.assert_allclose(Od, Og[t], rtol=1e-12, atol=1e-13)


def test_flop_counts_match_workload_table():
    a, i = O.flop_counts(16384, 64, 512, 4, k=512, HI=64, DI=128)
    assert abs(a / 1e12 - 1.305) < 0.01 and abs(i / 1e12 - 0.550) < 0.01
    a3, _ = O.flop_counts(131072, 64, 512, 128, dense=True)
    assert abs(a3 / 1e12 - 10.99) < 0.05
