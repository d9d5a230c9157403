"""Pins of the oracle's remaining layer-stack pieces ("Deepseek-V4 技术报告里最值得
复现的三个改动", §3 config block and the note after it): the sliding-window-only
layer and the grouped output projection (8 groups, intermediate 1024 dims,
hidden size 4096)."""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O


def _proj_case(rng, T=5, H=8, D=6, G=4, d_mid=7, d_model=9):
    Ot = rng.standard_normal((T, H, D))
    w_grp = rng.standard_normal((G, d_mid, (H // G) * D))
    w_out = rng.standard_normal((d_model, G * d_mid))
    return Ot, w_grp, w_out


def test_grouped_proj_hand_example():
    """Heads 1, 2 | 3, 4 (D = 1) in two groups; group weights [1, 10] and
    [100, 1000], so each decimal digit of the result names one head's term and
    a wrong head order or group assignment changes the digits."""
    Ot = np.array([[[1.0], [2.0], [3.0], [4.0]]])
    w_grp = np.array([[[1.0, 10.0]], [[100.0, 1000.0]]])
    out, mid = O.grouped_out_proj(Ot, w_grp, np.array([[1.0, 1.0], [2.0, 0.0]]), return_mid=True)
    np.testing.assert_array_equal(mid, [[21.0, 4300.0]])
    np.testing.assert_array_equal(out, [[4321.0, 42.0]])


def test_grouped_proj_equals_block_diagonal_projection():
    """Grouped projection = one dense projection whose matrix is the block
    diagonal of the group matrices (an independent formulation)."""
    rng = np.random.default_rng(1)
    Ot, w_grp, w_out = _proj_case(rng)
    T, H, D = Ot.shape
    big = scipy.linalg.block_diag(*w_grp)                     # [G*d_mid, H*D]
    ref_mid = Ot.reshape(T, H * D) @ big.T
    out, mid = O.grouped_out_proj(Ot, w_grp, w_out, return_mid=True)
    np.testing.assert_allclose(mid, ref_mid, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(out, ref_mid @ w_out.T, rtol=1e-12, atol=1e-12)


def test_grouped_proj_one_group_is_two_linear_maps():
    rng = np.random.default_rng(2)
    Ot, w_grp, w_out = _proj_case(rng, G=1, d_mid=11)
    T, H, D = Ot.shape
    x = torch.from_numpy(Ot.reshape(T, H * D))
    ref = torch.nn.functional.linear(torch.nn.functional.linear(x, torch.from_numpy(w_grp[0])),
                                     torch.from_numpy(w_out)).numpy()
    np.testing.assert_allclose(O.grouped_out_proj(Ot, w_grp, w_out), ref, rtol=1e-12, atol=1e-12)


def test_grouped_proj_group_footprint():
    """Changing the heads of group g changes only intermediate columns
    [g*d_mid, (g+1)*d_mid)."""
    rng = np.random.default_rng(3)
    Ot, w_grp, w_out = _proj_case(rng)
    G, d_mid = w_grp.shape[:2]
    hg = Ot.shape[1] // G
    _, mid0 = O.grouped_out_proj(Ot, w_grp, w_out, return_mid=True)
    for g in range(G):
        O2 = Ot.copy()
        O2[:, g * hg:(g + 1) * hg] += rng.standard_normal(O2[:, g * hg:(g + 1) * hg].shape)
        _, mid = O.grouped_out_proj(O2, w_grp, w_out, return_mid=True)
        changed = np.any(mid != mid0, axis=0)
        expect = np.zeros(G * d_mid, bool)
        expect[g * d_mid:(g + 1) * d_mid] = True
        np.testing.assert_array_equal(changed, expect)


def test_grouped_proj_linear_and_rounded_intermediate():
    rng = np.random.default_rng(4)
    Ot, w_grp, w_out = _proj_case(rng)
    a = O.grouped_out_proj(Ot, w_grp, w_out)
    np.testing.assert_allclose(O.grouped_out_proj(2.5 * Ot, w_grp, w_out), 2.5 * a, rtol=1e-13)
    out, mid = O.grouped_out_proj(Ot, w_grp, w_out, mid_round=O.bf16_round, return_mid=True)
    # the stored intermediate is bf16-valued and the output is its exact product
    np.testing.assert_array_equal(mid, torch.from_numpy(mid).to(torch.bfloat16).double().numpy())
    np.testing.assert_allclose(out, mid @ w_out.T, rtol=1e-13)
    with pytest.raises(ValueError):
        O.grouped_out_proj(Ot, w_grp[:, :, :-1], w_out)


def _mqa_sdpa(q, kv, mask=None, causal=False):
    """torch's scaled-dot-product attention in float64 with K = V = kv shared by
    every head (q [T, H, D], kv [S, D])."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                 # [1, H, T, D]
    kt = torch.from_numpy(kv)[None, None].expand(1, q.shape[1], -1, -1)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=m, is_causal=causal)
    return o[0].permute(1, 0, 2).numpy()


def test_swa_layer_wide_window_is_causal_attention():
    """W >= S and a sink at -inf: plain causal softmax attention (torch SDPA)."""
    rng = np.random.default_rng(5)
    S, H, D = 40, 3, 8
    q = rng.standard_normal((S, H, D)); C = rng.standard_normal((S, D))
    out = O.swa_layer(q, C, np.full(H, -np.inf), W=S + 7)
    np.testing.assert_allclose(out, _mqa_sdpa(q, C, causal=True), rtol=1e-12, atol=1e-12)


def test_swa_layer_banded_window():
    """Window W < S: attention restricted to keys [t-W+1, t] (SDPA with a band mask)."""
    rng = np.random.default_rng(6)
    S, H, D, W = 50, 2, 8, 5
    q = rng.standard_normal((S, H, D)); C = rng.standard_normal((S, D))
    t = np.arange(S)
    band = (t[None, :] <= t[:, None]) & (t[None, :] > t[:, None] - W)
    rows = np.array([0, 3, 4, 5, 31, 49])
    out = O.swa_layer(q, C, np.full(H, -np.inf), W=W, rows=rows)
    np.testing.assert_allclose(out, _mqa_sdpa(q, C, mask=band)[rows], rtol=1e-12, atol=1e-12)


def test_swa_layer_window_of_one_with_sink():
    """W = 1: the token's own row, weighted by e^l / (e^l + e^s)."""
    rng = np.random.default_rng(7)
    S, H, D = 6, 4, 16
    q = rng.standard_normal((S, H, D)); C = rng.standard_normal((S, D)); sink = rng.standard_normal(H)
    out = O.swa_layer(q, C, sink, W=1)
    for t in range(S):
        for h in range(H):
            l = float(q[t, h] @ C[t]) / math.sqrt(D)
            np.testing.assert_allclose(out[t, h], C[t] / (1.0 + math.exp(sink[h] - l)), rtol=1e-13)


def test_swa_layer_is_csa_layer_before_the_first_entry():
    """Before any compressed entry is visible (t < m - 1) a CSA layer is a
    window-only layer."""
    rng = np.random.default_rng(8)
    S, H, D, m, HI, DI = 64, 2, 64, 4, 2, 8
    q = rng.standard_normal((S, H, D)); C = rng.standard_normal((S, D)); Z = rng.standard_normal((S, D))
    B = rng.standard_normal((2 * m, D)); sink = rng.standard_normal(H)
    qI = rng.standard_normal((S, HI, DI)); w = rng.random((S, HI)); kI = rng.standard_normal((S // m, DI))
    rows = np.arange(m - 1)
    ref, _ = O.csa_layer(q, C, Z, B, qI, w, kI, sink, k=4, m=m, norm_rope=True, inv_rope=True, rows=rows)
    out = O.swa_layer(q, C, sink, norm_rope=True, inv_rope=True, rows=rows)
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-13)
