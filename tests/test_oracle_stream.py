"""Oracle pins for the decode-time cache writer: the streaming compressor (one
token at a time, a ring of the last 2m tokens) must reproduce the batch
compressor entry by entry, and the FP8 row quantiser must meet the e4m3
definition (largest magnitude -> 448, per-element error within half an e4m3
step, zero rows, bf16 RoPE dims)."""
import numpy as np
import pytest

import oracle as O


def _batch(C, Z, B, m, overlap, norm_rope):
    kv = O.compress(C, Z, B, m, overlap)
    if norm_rope:
        kv = O.rope_partial(O.rmsnorm(kv), np.arange(kv.shape[0]) * m, 64)
    return kv


@pytest.mark.parametrize("m,overlap", [(4, True), (8, False), (4, False)])
@pytest.mark.parametrize("norm_rope", [True, False])
def test_stream_equals_batch(m, overlap, norm_rope):
    rng = np.random.default_rng(11)
    S, D = 6 * m + 3, 128
    C, Z = rng.standard_normal((S, D)), rng.standard_normal((S, D))
    B = 0.1 * rng.standard_normal((2 * m if overlap else m, D))
    ref = _batch(C, Z, B, m, overlap, norm_rope)
    ring_c, ring_z = np.zeros((2 * m, D)), np.zeros((2 * m, D))
    got = {}
    for t in range(S):
        r = O.stream_append(ring_c, ring_z, C[t], Z[t], t, B, m, overlap, norm_rope=norm_rope)
        assert (r is None) == ((t + 1) % m != 0)
        if r is not None:
            got[r[0]] = r[1]
    assert sorted(got) == list(range(S // m))                 # tail tokens emit nothing
    for i, row in got.items():
        assert np.array_equal(row, ref[i])


def test_stream_resumes_from_a_prefilled_ring():
    """A decode stream that starts after a prefill: the ring holds the last 2m
    prefill tokens, and the next entries equal the batch compressor's."""
    rng = np.random.default_rng(12)
    m, D, S0, S = 4, 128, 37, 53
    C, Z = rng.standard_normal((S, D)), rng.standard_normal((S, D))
    B = 0.1 * rng.standard_normal((2 * m, D))
    ref = _batch(C, Z, B, m, True, True)
    ring_c, ring_z = np.zeros((2 * m, D)), np.zeros((2 * m, D))
    for u in range(S0 - 2 * m, S0):
        ring_c[u % (2 * m)], ring_z[u % (2 * m)] = C[u], Z[u]
    for t in range(S0, S):
        r = O.stream_append(ring_c, ring_z, C[t], Z[t], t, B, m, True)
        if r is not None:
            assert np.array_equal(r[1], ref[r[0]])


def test_fp8_row_quantize_definition():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((5, 512)) * np.array([1e-3, 1.0, 30.0, 1.0, 7.0])[:, None]
    x[3, 100] = -9.0                                          # a negative row maximum
    codes, rope, scale = O.fp8_row_quantize(x, 64)
    nope = x[:, :448]
    amax = np.abs(nope).max(axis=1)
    assert np.allclose(scale, amax / 448.0, rtol=0, atol=0)
    # the largest magnitude maps to the largest finite code, with its sign
    for r in range(5):
        j = np.argmax(np.abs(nope[r]))
        assert codes[r, j] & 0x7F == 0x7E and (codes[r, j] >> 7) == (nope[r, j] < 0)
    # every element within half an e4m3 step: 2^-4 relative for normals,
    # 2^-10 of the scale below the smallest normal 2^-6
    deq = O.e4m3_decode(codes) * scale[:, None]
    bound = np.maximum(np.abs(nope) * 2.0 ** -4, scale[:, None] * 2.0 ** -10)
    assert np.all(np.abs(deq - nope) <= bound * (1 + 1e-12))
    assert np.array_equal(rope, O.bf16_round(x[:, 448:]))
    z_codes, _, z_scale = O.fp8_row_quantize(np.zeros((1, 512)), 64)
    assert z_scale[0] == 1.0 and not z_codes.any()


def test_index_key_stream_equals_batch_and_quantises_whole_row():
    """The indexer key of each block ([CS] "闪电索引器" scores compressed
    entries; reading taken: the key is pooled by the same per-channel softmax
    over its own (C_I, Z_I) stream, with no norm or RoPE) streamed one token at
    a time equals the batch compressor of that stream, and its e4m3 row has no
    bf16 part: every dim is a code under the row scale amax / 448."""
    rng = np.random.default_rng(14)
    m, DI, S = 4, 128, 45
    CI, ZI = rng.standard_normal((S, DI)), rng.standard_normal((S, DI))
    BI = 0.1 * rng.standard_normal((2 * m, DI))
    ref = O.compress(CI, ZI, BI, m, True)
    ring_c, ring_z = np.zeros((2 * m, DI)), np.zeros((2 * m, DI))
    for t in range(S):
        r = O.stream_append(ring_c, ring_z, CI[t], ZI[t], t, BI, m, True, norm_rope=False)
        if r is None:
            continue
        i, key = r
        assert np.array_equal(key, ref[i])
        codes, rope, scale = O.fp8_row_quantize(key, 0)
        assert codes.shape == (DI,) and rope.shape == (0,)
        assert scale == np.abs(key).max() / 448.0
        deq = O.e4m3_decode(codes) * scale
        assert np.all(np.abs(deq - key) <= np.maximum(np.abs(key) * 2.0 ** -4, scale * 2.0 ** -10) * (1 + 1e-12))
