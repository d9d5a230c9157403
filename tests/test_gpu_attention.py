"""GPU parity: tcgen05 shared-KV attention (sparse, dense, window + sink) vs
the float64 oracle on the same (bf16 / e4m3-valued) inputs."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import MAX_ABS_F32, REL_L2_F32, assert_close, cuda, host, lib_loaded
from long_context_compressed_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lib_loaded()


def _bf16(rng, shape, scale=1.0):
    return synth.to_bf16_values(rng.standard_normal(shape) * scale)


def _rand_idx(rng, T, k, ne, sizes):
    idx = np.full((T, k), -1, np.int32)
    for t in range(T):
        n = sizes[t % len(sizes)]
        n = min(n, ne, k)
        idx[t, :n] = np.sort(rng.choice(ne, n, replace=False))
    return idx


@pytest.mark.parametrize("H,D,dt", [(64, 512, "bf16"), (8, 128, "f32"), (64, 128, "bf16")])
def test_sparse_partial(H, D, dt):
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(1)
    T, ne, k = 70, 1000, 512
    q = O.rmsnorm(rng.standard_normal((T, H, D)))
    kv = O.rmsnorm(rng.standard_normal((ne, D)))
    if dt == "bf16":
        q, kv = synth.to_bf16_values(q), synth.to_bf16_values(kv)
        tq = cuda(q, torch.bfloat16); tkv = cuda(kv, torch.bfloat16)
    else:
        q, kv = q.astype(np.float32), kv.astype(np.float32)
        tq = cuda(q); tkv = cuda(kv)
    idx = _rand_idx(rng, T, k, ne, [512, 0, 1, 127, 128, 129, 300, 511, 256])
    Og, Lg = csa.csa_sparse_mqa(tq[None], tkv[None], cuda(idx)[None])
    csa.check_device_error()
    Or, Lr = O.sparse_attention_partial(q, kv, idx)
    has = (idx >= 0).any(axis=1)
    tol = dict(max_abs=MAX_ABS_F32, rel_l2=REL_L2_F32) if dt == "f32" else {}
    assert_close(host(Og)[0][has], Or[has], what="O_part", **tol)
    assert np.all(host(Og)[0][~has] == 0) and np.all(np.isneginf(host(Lg)[0][~has]))
    assert_close(host(Lg)[0][has], Lr[has], **(tol or dict(max_abs=1e-2, rel_l2=1e-3)), what="lse")


def test_sparse_partial_e4m3_store():
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(2)
    gen = torch.Generator(device="cuda").manual_seed(2)
    ne, D, H, T, k = 3000, 512, 64, 4, 512
    cache = synth.decode_csa_cache(ne, D, 128, 64, gen, "cuda")
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((T, H, D))) * 0.5)
    idx = _rand_idx(rng, T, k, ne, [512, 200, 1, 129])
    Og, Lg = csa.csa_sparse_mqa(cuda(q, torch.bfloat16)[None], cache["kv_nope"][None], cuda(idx)[None],
                                kv_rope=cache["kv_rope"][None], kv_scale=cache["kv_scale"][None])
    csa.check_device_error()
    kv = np.concatenate([O.e4m3_decode(cache["kv_nope"].cpu().numpy()) * cache["kv_scale"].cpu().numpy()[:, None],
                         cache["kv_rope"].float().cpu().numpy()], axis=1)
    Or, Lr = O.sparse_attention_partial(q, kv, idx, scale=1 / math.sqrt(D))
    assert_close(host(Og)[0], Or, what="e4m3 O_part")
    assert_close(host(Lg)[0], Lr, max_abs=2e-2, rel_l2=1e-3, what="e4m3 lse")


def test_dense_partial_multi_chunk():
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(3)
    T, cap, H, D, m = 40, 700, 64, 512, 128
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((T, H, D))))
    kv = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((cap, D))))
    pos0 = 128 * 520 - 20                         # n_vis crosses 520 -> 521 inside the block
    Og, Lg = csa.hca_dense_attn(cuda(q, torch.bfloat16)[None], cuda(kv, torch.bfloat16)[None],
                                cuda(np.array([pos0], np.int64)), m)
    csa.check_device_error()
    Or, Lr = O.dense_attention_partial(q, kv, O.n_visible(pos0 + np.arange(T), m))
    assert_close(host(Og)[0], Or, what="dense O_part")
    assert_close(host(Lg)[0], Lr, max_abs=1e-2, rel_l2=1e-3, what="dense lse")


@pytest.mark.parametrize("with_partial,inv_rope", [(True, True), (False, False), (True, False)])
def test_window_sink_combine_prefill(with_partial, inv_rope):
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(4)
    S, H, D, W = 300, 64, 512, 128
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((S, H, D))))
    kt = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((S, D))))
    sink = rng.standard_normal(H).astype(np.float32)
    Op = (0.3 * rng.standard_normal((S, H, D))).astype(np.float32)
    Lp = rng.standard_normal((S, H)).astype(np.float32)
    Lp[5] = -np.inf; Op[5] = 0                       # an empty compressed branch
    pos = np.array([0], np.int64)
    out = csa.swa_sink_combine(cuda(q, torch.bfloat16)[None], cuda(kt, torch.bfloat16)[None], cuda(pos), W,
                               cuda(sink), cuda(Op)[None] if with_partial else None,
                               cuda(Lp)[None] if with_partial else None, inv_rope=inv_rope,
                               rope_dim=64, out_dtype=torch.float32)
    csa.check_device_error()
    if not with_partial:
        Op2 = np.zeros_like(Op); Lp2 = np.full_like(Lp, -np.inf)
    else:
        Op2, Lp2 = Op, Lp
    ref = O.window_sink_combine(q, kt, np.arange(S), W, sink, Op2, Lp2, inv_rope=inv_rope)
    assert_close(host(out)[0], ref, what="combine")


def test_window_cache_decode_batch():
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(5)
    n_seq, H, D, W = 5, 64, 512, 128
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((n_seq, 1, H, D))))
    swa = synth.to_bf16_values(rng.standard_normal((n_seq, W, D)))
    sink = rng.standard_normal(H).astype(np.float32)
    pos = np.array([1 << 20, 3, 127, 128, 5000], np.int64)
    out = csa.swa_sink_combine(cuda(q, torch.bfloat16), cuda(swa, torch.bfloat16), cuda(pos), W, cuda(sink),
                               window_mode=1, inv_rope=True, out_dtype=torch.float32)
    csa.check_device_error()
    for b in range(n_seq):
        nrow = min(W, pos[b] + 1)
        ref = O.window_sink_combine(q[b], None, [pos[b]], W, sink, np.zeros((1, H, D)), np.full((1, H), -np.inf),
                                    inv_rope=True, window_rows=[swa[b][:nrow]])
        assert_close(host(out)[b], ref, what=f"decode window b={b}")


def test_batch_invariance_bit_exact():
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(6)
    n_seq, T, ne, H, D, k = 16, 3, 900, 64, 512, 512
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((n_seq, T, H, D))))
    kv = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((n_seq, ne, D))))
    idx = np.stack([_rand_idx(rng, T, k, ne, [512, 300, 77]) for _ in range(n_seq)])
    tq, tkv, ti = cuda(q, torch.bfloat16), cuda(kv, torch.bfloat16), cuda(idx)
    Ob, Lb = csa.csa_sparse_mqa(tq, tkv, ti)
    for b in (0, 7, 15):
        Oa, La = csa.csa_sparse_mqa(tq[b:b + 1].contiguous(), tkv[b:b + 1].contiguous(), ti[b:b + 1].contiguous())
        assert torch.equal(Oa[0], Ob[b]) and torch.equal(La[0], Lb[b])
    csa.check_device_error()


def _dequant(cache):
    return np.concatenate([O.e4m3_decode(cache["kv_nope"].cpu().numpy()) * cache["kv_scale"].cpu().numpy()[:, None],
                           cache["kv_rope"].float().cpu().numpy()], axis=1)


@pytest.mark.parametrize("n_split", [1, 2, 3, 8, 16])
def test_fused_csa_decode_e4m3_caches(n_split):
    """Decode: top-k entries from an e4m3 + bf16-RoPE cache, the 128-row SWA
    cache and the sink in one softmax, inverse RoPE at the query position."""
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(21)
    gen = torch.Generator(device="cuda").manual_seed(21)
    n_seq, cap, H, D, W, k = 4, 2500, 64, 512, 128, 512
    caches = [synth.decode_csa_cache(cap, D, 128, 64, gen, "cuda") for _ in range(n_seq)]
    kv_nope = torch.stack([c["kv_nope"] for c in caches]); kv_rope = torch.stack([c["kv_rope"] for c in caches])
    kv_scale = torch.stack([c["kv_scale"] for c in caches])
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((n_seq, 1, H, D))))
    swa = synth.to_bf16_values(rng.standard_normal((n_seq, W, D)))
    sink = rng.standard_normal(H).astype(np.float32)
    pos = np.array([4 * cap - 1, 3, 999, 4 * cap - 5], np.int64)
    idx = np.full((n_seq, 1, k), -1, np.int32)
    for b in range(n_seq):
        nv = min(cap, (pos[b] + 1) // 4)
        n = min(k, nv)
        idx[b, 0, :n] = np.sort(rng.choice(nv, n, replace=False)) if nv else []
    out = csa.csa_fused_attention(cuda(q, torch.bfloat16), kv_nope, cuda(swa, torch.bfloat16), cuda(pos), W,
                                  cuda(sink), idx=cuda(idx), kv_rope=kv_rope, kv_scale=kv_scale, window_mode=1,
                                  inv_rope=True, rope_dim=64, out_dtype=torch.float32, n_split=n_split)
    csa.check_device_error()
    for b in range(n_seq):
        kv = _dequant(caches[b])
        Op, Lp = O.sparse_attention_partial(q[b], kv, idx[b])
        nrow = min(W, pos[b] + 1)
        ref = O.window_sink_combine(q[b], None, [pos[b]], W, sink, Op, Lp, inv_rope=True, window_rows=[swa[b][:nrow]])
        assert_close(host(out)[b], ref, what=f"fused CSA decode b={b}")


@pytest.mark.parametrize("n_split", [1, 2, 4, 8])
def test_fused_hca_decode_e4m3_dense(n_split):
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(22)
    gen = torch.Generator(device="cuda").manual_seed(22)
    n_seq, cap, H, D, W, m = 3, 700, 64, 512, 128, 128
    caches = [synth.decode_csa_cache(cap, D, 128, 64, gen, "cuda") for _ in range(n_seq)]
    kv_nope = torch.stack([c["kv_nope"] for c in caches]); kv_rope = torch.stack([c["kv_rope"] for c in caches])
    kv_scale = torch.stack([c["kv_scale"] for c in caches])
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((n_seq, 1, H, D))))
    swa = synth.to_bf16_values(rng.standard_normal((n_seq, W, D)))
    sink = rng.standard_normal(H).astype(np.float32)
    pos = np.array([128 * 700 - 1, 130, 128 * 333 + 17], np.int64)
    out = csa.csa_fused_attention(cuda(q, torch.bfloat16), kv_nope, cuda(swa, torch.bfloat16), cuda(pos), W,
                                  cuda(sink), m=m, kv_rope=kv_rope, kv_scale=kv_scale, window_mode=1,
                                  inv_rope=True, rope_dim=64, out_dtype=torch.float32, n_split=n_split)
    csa.check_device_error()
    for b in range(n_seq):
        kv = _dequant(caches[b])
        ref = O.hca_decode(q[b][0], kv, swa[b][:min(W, pos[b] + 1)], sink, int(pos[b]), m=m)
        assert_close(host(out)[b][0], ref, what=f"fused HCA decode b={b}")


def test_fused_equals_separate_calls():
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(23)
    S, ne, H, D, k, W = 400, 100, 64, 512, 64, 128
    q = cuda(synth.to_bf16_values(O.rmsnorm(rng.standard_normal((1, S, H, D)))), torch.bfloat16)
    kv = cuda(synth.to_bf16_values(O.rmsnorm(rng.standard_normal((1, ne, D)))), torch.bfloat16)
    kt = cuda(synth.to_bf16_values(O.rmsnorm(rng.standard_normal((1, S, D)))), torch.bfloat16)
    idx = cuda(np.stack([_rand_idx(rng, S, k, ne, [64, 0, 5, 33])]))
    sink = cuda(rng.standard_normal(H).astype(np.float32))
    pos = cuda(np.array([0], np.int64))
    Op, Lp = csa.csa_sparse_mqa(q, kv, idx)
    sep = csa.swa_sink_combine(q, kt, pos, W, sink, Op, Lp, inv_rope=True, out_dtype=torch.float32)
    fus = csa.csa_fused_attention(q, kv, kt, pos, W, sink, idx=idx, inv_rope=True, out_dtype=torch.float32)
    csa.check_device_error()
    # both paths are bf16-probability approximations of the same softmax: the parity tolerance
    assert_close(host(fus), host(sep), what="fused vs separate")


@pytest.mark.parametrize("n_split", [3, 4, 8])
def test_split_kv_prefill_matches_oracle(n_split):
    """Split-KV over bf16 prefill rows (window first, then gathered entries);
    early tokens hold fewer half chunks than ranges, so some ranks are empty."""
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(24)
    S, ne, H, D, k, W = 300, 200, 64, 512, 160, 128
    q = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((S, H, D))))
    kv = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((ne, D))))
    kt = synth.to_bf16_values(O.rmsnorm(rng.standard_normal((S, D))))
    idx = _rand_idx(rng, S, k, ne, [160, 0, 1, 129, 70])
    sink = rng.standard_normal(H).astype(np.float32)
    out = csa.csa_fused_attention(cuda(q, torch.bfloat16)[None], cuda(kv, torch.bfloat16)[None],
                                  cuda(kt, torch.bfloat16)[None], cuda(np.array([0], np.int64)), W, cuda(sink),
                                  idx=cuda(idx)[None], inv_rope=True, rope_dim=64, out_dtype=torch.float32,
                                  n_split=n_split)
    csa.check_device_error()
    Op, Lp = O.sparse_attention_partial(q, kv, idx)
    ref = O.window_sink_combine(q, kt, np.arange(S), W, sink, Op, Lp, inv_rope=True)
    assert_close(host(out)[0], ref, what="split-KV prefill")


@pytest.mark.parametrize("H,D,n_split,dense", [(64, 512, 1, False), (8, 128, 1, True), (40, 512, 3, False),
                                               (8, 128, 2, True), (6, 128, 1, False), (3, 512, 2, True)])
def test_f32_path_fused_with_window_sink_and_inverse_rope(H, D, n_split, dense):
    """float32 queries, entries and window rows run in fp32 arithmetic: the
    fused call (selected or dense entries, window, sink, inverse RoPE) and its
    split-KV form match the oracle at the float32 tolerance."""
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(12)
    S, W, k, m = 300, 128, 64, 4
    ne = S // m
    q = O.rmsnorm(rng.standard_normal((S, H, D))).astype(np.float32)
    kv = O.rmsnorm(rng.standard_normal((ne, D))).astype(np.float32)
    kt = O.rmsnorm(rng.standard_normal((S, D))).astype(np.float32)
    sink = rng.standard_normal(H).astype(np.float32)
    pos = np.arange(S)
    nv = O.n_visible(pos, m)
    if dense:
        idx = None
        Op, Lp = O.dense_attention_partial(q, kv, nv)
    else:
        idx = np.full((S, k), -1, np.int32)
        for t in range(S):
            n = min(k, int(nv[t]), [64, 0, 5, 33][t % 4])
            idx[t, :n] = np.sort(rng.choice(int(nv[t]), n, replace=False)) if n else []
        Op, Lp = O.sparse_attention_partial(q, kv, idx)
    ref = O.window_sink_combine(q, kt, pos, W, sink, Op, Lp, inv_rope=True)
    out = csa.csa_fused_attention(cuda(q)[None], cuda(kv)[None], cuda(kt)[None], cuda(np.zeros(1, np.int64)), W,
                                  cuda(sink), idx=None if idx is None else cuda(idx)[None], m=m, inv_rope=True,
                                  rope_dim=64, out_dtype=torch.float32, n_split=n_split)
    csa.check_device_error()
    assert_close(host(out)[0], ref, max_abs=MAX_ABS_F32, rel_l2=REL_L2_F32, what="fp32 fused attention")


@pytest.mark.parametrize("fused", [False, True])
def test_growing_logits_lazy_rescale(fused):
    """Unit-RMS entries (and window rows) lean more and more on one direction u
    along the visit order, the heads lean on u by different amounts, and one
    head per token points at a late entry: the running maxima of later half
    chunks jump by more than the lazy-rescale threshold (a factor 2^8) for some
    columns and rise by less for others (these keep the old maximum, so their
    probabilities exceed 1).  Both branches run against the oracle."""
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(31)
    T, ne, H, D, k, W = 200, 1000, 64, 512, 512, 128
    u = rng.standard_normal(D)

    def leaning(n):
        a = 6.0 * (np.arange(n) / n) ** 2
        return O.rmsnorm(a[:, None] * u[None] + rng.standard_normal((n, D)))

    kv = synth.to_bf16_values(leaning(ne))
    kt = synth.to_bf16_values(leaning(T))
    idx = _rand_idx(rng, T, k, ne, [512, 300, 129, 64])
    beta = np.linspace(0, 3, H)
    q = O.rmsnorm(beta[None, :, None] * u[None, None] + rng.standard_normal((T, H, D)))
    for t in range(T):
        n = int((idx[t] >= 0).sum())
        q[t, t % H] = O.rmsnorm(kv[idx[t, n - 3]])       # one head locks onto a late entry
    q = synth.to_bf16_values(q)
    tq, tkv, ti = cuda(q, torch.bfloat16)[None], cuda(kv, torch.bfloat16)[None], cuda(idx)[None]
    Or, Lr = O.sparse_attention_partial(q, kv, idx)
    if not fused:
        Og, Lg = csa.csa_sparse_mqa(tq, tkv, ti)
        csa.check_device_error()
        assert_close(host(Og)[0], Or, what="growing-logit O_part")
        assert_close(host(Lg)[0], Lr, max_abs=1e-2, rel_l2=1e-3, what="growing-logit lse")
        return
    sink = rng.standard_normal(H).astype(np.float32)
    out = csa.csa_fused_attention(tq, tkv, cuda(kt, torch.bfloat16)[None], cuda(np.array([0], np.int64)), W,
                                  cuda(sink), idx=ti, inv_rope=True, rope_dim=64, out_dtype=torch.float32)
    csa.check_device_error()
    ref = O.window_sink_combine(q, kt, np.arange(T), W, sink, Or, Lr, inv_rope=True)
    assert_close(host(out)[0], ref, what="growing-logit fused")
