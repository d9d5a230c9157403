"""GPU parity: the FP4 (MX) lightning indexer + top-k vs the float64 oracle on
the dequantised operands.

Grid inputs (E2M1 magnitudes 0, 0.5, 1; block scales 2^-1 .. 2^1; head weights
on the 1/16 grid) keep every score and partial sum exact in fp32, so the
selected sets must be bit-identical.  Rows whose block scales span 2^7 take the
converter's fp32 path; their sets may differ only within the fp32 rounding
bound of the k-th score."""
import numpy as np
import pytest

import oracle as O
from gpu_util import cuda, lib_loaded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lib_loaded()


_SMALL_CODES = np.array([0, 1, 2, 9, 10], np.uint8)     # 0, 0.5, 1, -0.5, -1


def _fp4_rows(rng, shape, scale_choices=(126, 127, 128)):
    """Packed codes [..., 64] and E8M0 bytes [..., 4] of 128-element rows."""
    codes = rng.choice(_SMALL_CODES, size=shape + (128,))
    scales = rng.choice(np.array(scale_choices, np.uint8), size=shape + (4,))
    return O.fp4_pack(codes), scales.astype(np.uint8)


def _deq(packed, scales):
    return O.mxfp4_dequantize(O.fp4_unpack(packed), scales)


def _run(q4, qs4, w, k4, ks4, q_pos, m, k):
    import long_context_compressed_02_b200 as csa
    idx = csa.csa_index_topk_fp4(cuda(q4), cuda(qs4), cuda(w), cuda(k4), cuda(ks4),
                                 cuda(np.asarray(q_pos, np.int64)), m, k)
    csa.check_device_error()
    return idx.cpu().numpy()


def _oracle_scores(q4, qs4, w, k4, ks4, q_pos, m, b):
    qI = _deq(q4[b], qs4[b])                    # [T, HI, 128]
    kI = _deq(k4[b], ks4[b])                    # [cap, 128]
    T = qI.shape[0]
    nv = np.minimum(kI.shape[0], O.n_visible(q_pos[b] + np.arange(T), m))
    return O.indexer_scores(qI, w[b], kI, nv), nv


@pytest.mark.parametrize("n_seq,T,cap,k,q_pos", [
    (3, 1, 40000, 512, [4 * 40000 - 1, 70001, 5]),    # decode: chunked rows, a short row
    (1, 300, 1200, 64, [0]),                          # prefill-shaped token blocks
])
def test_fp4_grid_bit_exact(n_seq, T, cap, k, q_pos):
    rng = np.random.default_rng(21)
    HI, m = 64, 4
    q4, qs4 = _fp4_rows(rng, (n_seq, T, HI))
    k4, ks4 = _fp4_rows(rng, (n_seq, cap))
    w = (np.floor(rng.random((n_seq, T, HI)) * 16) / 16).astype(np.float32)
    got = _run(q4, qs4, w, k4, ks4, q_pos, m, k)
    for b in range(n_seq):
        s, nv = _oracle_scores(q4, qs4, w, k4, ks4, q_pos, m, b)
        fin = s[np.isfinite(s)]
        assert np.array_equal(fin.astype(np.float32).astype(np.float64), fin)   # exact in fp32
        assert np.array_equal(got[b], O.topk_select(s, nv, k)), f"sequence {b}"


def test_fp4_wide_block_scale_span_within_rounding_bound():
    rng = np.random.default_rng(22)
    n_seq, T, HI, cap, m, k = 2, 1, 64, 8192, 4, 256
    q4, qs4 = _fp4_rows(rng, (n_seq, T, HI))
    k4, ks4 = _fp4_rows(rng, (n_seq, cap), scale_choices=(120, 127))   # d = -7: the fp32 path
    w = rng.random((n_seq, T, HI)).astype(np.float32)
    q_pos = [4 * cap - 1, 4 * cap - 1]
    got = _run(q4, qs4, w, k4, ks4, q_pos, m, k)
    for b in range(n_seq):
        s, nv = _oracle_scores(q4, qs4, w, k4, ks4, q_pos, m, b)
        ref = O.topk_select(s, nv, k)[0]
        a, r = set(got[b, 0][got[b, 0] >= 0].tolist()), set(ref[ref >= 0].tolist())
        assert len(a) == len(r) == min(k, nv[0])
        kth = np.sort(s[0, :nv[0]])[::-1][min(k, nv[0]) - 1]
        qI = _deq(q4[b], qs4[b])[0]; kI = _deq(k4[b], ks4[b])
        bound = 1e-5 * (np.abs(w[b, 0])[:, None] * np.abs(qI @ kI[:nv[0]].T)).sum(axis=0).max()
        for e in a ^ r:
            assert abs(s[0, e] - kth) <= bound, (b, e)
