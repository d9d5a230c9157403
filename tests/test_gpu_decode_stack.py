"""GPU parity of the mixed decode stack: four layers in the order CSA, HCA,
CSA, HCA, one new token per sequence, per-sequence context lengths, CSA top-k
1024 over an e4m3 indexer cache, HCA dense over m' = 128 entries, a 128-row
SWA cache and a sink on every layer; each layer against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close, host, lib_loaded
from long_context_compressed_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lib_loaded()


def _kv_rows(lay, b, rows, D):
    """Dequantised cache rows (e4m3 * row scale | bf16 RoPE part) of sequence b."""
    r = torch.from_numpy(np.asarray(rows, np.int64)).cuda()
    kv = np.zeros((len(rows), D))
    kv[:, :D - 64] = O.e4m3_decode(lay["kv_nope"][b][r].cpu().numpy()) * lay["kv_scale"][b][r].cpu().numpy()[:, None]
    kv[:, D - 64:] = lay["kv_rope"][b][r].float().cpu().numpy()
    return kv


def _run_stack(layers, q_pos, k, n_split_csa, n_split_hca):
    import long_context_compressed_02_b200 as csa
    res = []
    for lay in layers:
        out = torch.empty(lay["q"].shape, dtype=torch.float32, device="cuda")
        if lay["kind"] == "csa":
            out, idx = csa.csa_layer_decode(lay, q_pos, k=k, n_split=n_split_csa, out=out)
        else:
            out, idx = csa.hca_layer_decode(lay, q_pos, n_split=n_split_hca, out=out), None
        res.append((out, idx))
    csa.check_device_error()
    return res


def _check_layer(lay, res, b, t, k, W, D, what):
    out, idx = res
    q = lay["q"][b, 0].float().cpu().numpy()
    swa = lay["swa"][b].float().cpu().numpy()[:min(W, t + 1)]
    sink = lay["sink"].cpu().numpy()
    if lay["kind"] == "csa":
        nv = (t + 1) // 4
        kI = O.e4m3_decode(lay["kI"][b, :nv].cpu().numpy()) * lay["kI_scale"][b, :nv].cpu().numpy()[:, None]
        qI = O.e4m3_decode(lay["qI"][b, 0].cpu().numpy()) * lay["qI_scale"][b, 0].cpu().numpy()[:, None]
        w = lay["w"][b, 0].cpu().numpy()
        s = O.indexer_scores(qI[None], w[None], kI, [nv])
        ridx = O.topk_select(s, [nv], k)[0]
        assert np.array_equal(idx[b, 0].cpu().numpy(), ridx), f"{what}: top-k set"
        sel = ridx[ridx >= 0]
        kv = np.zeros((max(nv, 1), D))
        if len(sel):
            kv[sel] = _kv_rows(lay, b, sel, D)
        ref, _ = O.csa_decode(q, qI, w, kI, kv, swa, sink, t, k=k, m=4, inv_rope=True)
    else:
        nv = (t + 1) // 128
        kv = _kv_rows(lay, b, np.arange(nv), D) if nv else np.zeros((0, D))
        ref = O.hca_decode(q, kv, swa, sink, t, m=128, inv_rope=True)
    assert_close(host(out)[b, 0], ref, what=what)


@pytest.mark.parametrize("n_split", [(1, 1), (4, 16), (8, 8)])
def test_mixed_stack_small_contexts(n_split):
    """Four sequences with short, unequal contexts (one below top-k entries,
    one below a single HCA entry's worth of window): every sequence, every layer."""
    lengths = [3001, 9000, 20011, 700]
    layers, q_pos, cfg = synth.mixed_decode_inputs_device("cuda", seed=5, grid=True, lengths=lengths)
    res = _run_stack(layers, q_pos, cfg["k"], *n_split)
    for li, (lay, r) in enumerate(zip(layers, res)):
        for b, L in enumerate(lengths):
            _check_layer(lay, r, b, L - 1, cfg["k"], cfg["W"], cfg["D"], f"layer {li} ({lay['kind']}) b={b}")


def test_mixed_stack_full_size_sampled():
    """The full stack: 32 sequences with contexts U[64K, 1M]; the shortest and
    the longest sequence checked on every layer (top-k sets bit-exact on grid
    values)."""
    layers, q_pos, cfg = synth.mixed_decode_inputs_device("cuda", seed=0, grid=True)
    L = cfg["lengths"]
    res = _run_stack(layers, q_pos, cfg["k"], 4, 16)
    for b in (int(np.argmin(L)), int(np.argmax(L))):
        for li, (lay, r) in enumerate(zip(layers, res)):
            _check_layer(lay, r, b, int(L[b]) - 1, cfg["k"], cfg["W"], cfg["D"],
                         f"full-size layer {li} ({lay['kind']}) b={b} L={L[b]}")
