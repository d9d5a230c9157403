"""GPU parity: KV compressor and QK RMSNorm + RoPE vs the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close, cuda, host, lib_loaded
from long_context_compressed_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lib_loaded()


def test_tiny_csa_fp32():
    import long_context_compressed_02_b200 as csa
    inp, cfg = synth.prefill_inputs("tiny_csa")
    kv = csa.csa_compress(cuda(inp["C"]), cuda(inp["Z"]), cuda(inp["B"]), 4, True)
    torch.cuda.synchronize()
    ref = O.compress(inp["C"], inp["Z"], inp["B"], 4, True)
    assert kv.shape == (512, 128)
    assert_close(host(kv), ref, max_abs=1e-5, rel_l2=1e-6, what="tiny fp32 compress")


@pytest.mark.parametrize("S", [1, 3, 4, 5, 127, 2050])
def test_ragged_and_empty_lengths(S):
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(S)
    C = rng.standard_normal((S, 64)).astype(np.float32)
    Z = rng.standard_normal((S, 64)).astype(np.float32)
    B = (0.1 * rng.standard_normal((8, 64))).astype(np.float32)
    kv = csa.csa_compress(cuda(C), cuda(Z), cuda(B), 4, True)
    torch.cuda.synchronize()
    assert kv.shape == (S // 4, 64)
    if S >= 4:
        assert_close(host(kv), O.compress(C, Z, B, 4, True), max_abs=1e-5, rel_l2=1e-6)


@pytest.mark.parametrize("m,overlap,S", [(4, True, 2050), (128, False, 128 * 12 + 77), (128, False, 127)])
def test_bf16_norm_rope(m, overlap, S):
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(7)
    D = 512
    C = synth.to_bf16_values(rng.standard_normal((S, D)))
    Z = synth.to_bf16_values(rng.standard_normal((S, D)))
    B = (0.1 * rng.standard_normal((2 * m if overlap else m, D))).astype(np.float32)
    kv = csa.csa_compress(cuda(C, torch.bfloat16), cuda(Z, torch.bfloat16), cuda(B), m, overlap,
                          norm=True, rope_dim=64)
    torch.cuda.synchronize()
    ne = S // m
    assert kv.shape == (ne, D) and kv.dtype == torch.bfloat16
    if ne:
        ref = O.rope_partial(O.rmsnorm(O.compress(C, Z, B, m, overlap)), np.arange(ne) * m)
        assert_close(host(kv), ref, what=f"compress m={m}")


def test_separate_previous_block_stream():
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(3)
    S, D = 64, 128
    C, Z, Cb, Zb = (rng.standard_normal((S, D)).astype(np.float32) for _ in range(4))
    B = (0.1 * rng.standard_normal((8, D))).astype(np.float32)
    kv = csa.csa_compress(cuda(C), cuda(Z), cuda(B), 4, True, Cb=cuda(Cb), Zb=cuda(Zb))
    torch.cuda.synchronize()
    assert_close(host(kv), O.compress(C, Z, B, 4, True, Cb=Cb, Zb=Zb), max_abs=1e-5, rel_l2=1e-6)


@pytest.mark.parametrize("pos0", [0, (1 << 20) - 300])
def test_rmsnorm_rope_queries(pos0):
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(11)
    S, H, D = 300, 64, 512
    q = synth.to_bf16_values(rng.standard_normal((S, H, D)))
    out = csa.csa_rmsnorm_rope(cuda(q, torch.bfloat16), rows_per_pos=H, pos0=pos0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.rope_partial(O.rmsnorm(q), (pos0 + np.arange(S))[:, None])
    assert_close(host(out), ref, max_abs=1e-4, rel_l2=1e-5, what="q norm+rope")


def test_rmsnorm_rope_rows_bf16_out():
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(12)
    x = rng.standard_normal((1001, 512)).astype(np.float32)
    out = csa.csa_rmsnorm_rope(cuda(x), rows_per_pos=1, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ref = O.rope_partial(O.rmsnorm(x), np.arange(1001))
    assert_close(host(out), ref, what="row norm+rope")


@pytest.mark.parametrize("norm,out_dtype", [(True, torch.bfloat16), (False, torch.float32), (True, torch.float32)])
def test_rmsnorm_rope_bulk_path_ragged(norm, out_dtype):
    """bf16 rows sharing a position in groups of 32 (the chunked bulk-copy
    path), with a partial last chunk and a position near 2^20."""
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(13)
    rows, rpp, pos0 = 1000, 32, (1 << 20) - 17
    x = synth.to_bf16_values(rng.standard_normal((rows, 512)))
    out = csa.csa_rmsnorm_rope(cuda(x, torch.bfloat16), rows_per_pos=rpp, pos0=pos0, norm=norm, out_dtype=out_dtype)
    csa.check_device_error()
    y = O.rmsnorm(x) if norm else x.astype(np.float64)
    ref = O.rope_partial(y, pos0 + np.arange(rows) // rpp)
    tol = {} if out_dtype == torch.bfloat16 else dict(max_abs=1e-4, rel_l2=1e-5)
    assert_close(host(out), ref, what="bulk norm+rope", **tol)
