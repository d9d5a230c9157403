"""GPU parity of whole layers (compress -> index/top-k -> sparse MQA -> window
+ sink; compress -> dense -> window + sink) against the float64 oracle, plus
causality, and sampled rows at the full Flash-shaped prefill size."""
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


def _gpu_csa(inp, cfg, dt, fused=True):
    import long_context_compressed_02_b200 as csa
    out, idx = csa.csa_layer_prefill(
        cuda(inp["q"], dt), cuda(inp["C"], dt), cuda(inp["Z"], dt), cuda(inp["B"]), cuda(inp["qI_codes"]),
        cuda(inp["w"]), cuda(inp["kI_codes"]), cuda(inp["sink"]), k=cfg["k"], m=cfg["m"], W=cfg["W"],
        norm_rope=cfg["norm_rope"], inv_rope=cfg["inv_rope"], return_idx=True, fused=fused)
    csa.check_device_error()
    return out, idx


def _oracle_csa(inp, cfg, rows=None, store=None):
    return O.csa_layer(inp["q"], inp["C"], inp["Z"], inp["B"], O.e4m3_decode(inp["qI_codes"]), inp["w"],
                       O.e4m3_decode(inp["kI_codes"]), inp["sink"], k=cfg["k"], m=cfg["m"], W=cfg["W"],
                       norm_rope=cfg["norm_rope"], inv_rope=cfg["inv_rope"], store_round=store, rows=rows)


@pytest.mark.parametrize("fused", [True, False])
def test_tiny_csa_layer(fused):
    inp, cfg = synth.prefill_inputs("tiny_csa")
    out, idx = _gpu_csa(inp, cfg, torch.float32, fused)
    ref, ridx = _oracle_csa(inp, cfg)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert_close(host(out), ref, what="tiny CSA layer")


@pytest.mark.parametrize("S,fused", [(1534, True), (2048, True), (2048, False)])
def test_flash_shaped_csa_layer(S, fused):
    inp, cfg = synth.prefill_inputs("csa_prefill", S=S, grid=True)
    out, idx = _gpu_csa(inp, cfg, torch.bfloat16, fused)
    ref, ridx = _oracle_csa(inp, cfg, store=O.bf16_round)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert_close(host(out), ref, what="Flash-shaped CSA layer")


def test_csa_layer_causality_bit_exact():
    inp, cfg = synth.prefill_inputs("csa_prefill", S=700, grid=True)
    base, _ = _gpu_csa(inp, cfg, torch.bfloat16)
    t = 400
    pert = {k: v.copy() for k, v in inp.items()}
    rng = np.random.default_rng(9)
    for key in ("q", "C", "Z"):
        pert[key][t + 1:] = synth.to_bf16_values(rng.standard_normal(pert[key][t + 1:].shape))
    pert["qI_codes"][t + 1:] = synth.grid_codes(rng, pert["qI_codes"][t + 1:].shape)
    pert["kI_codes"][(t + 1) // 4:] = synth.grid_codes(rng, pert["kI_codes"][(t + 1) // 4:].shape)
    out, _ = _gpu_csa(pert, cfg, torch.bfloat16)
    assert torch.equal(out[:t + 1], base[:t + 1])
    assert not torch.equal(out[t + 1:], base[t + 1:])


@pytest.mark.parametrize("S,fused", [(128 * 6 + 37, True), (129, True), (128 * 6 + 37, False)])
def test_hca_layer(S, fused):
    import long_context_compressed_02_b200 as csa
    inp, cfg = synth.prefill_inputs("hca_prefill", S=S)
    out = csa.hca_layer_prefill(cuda(inp["q"], torch.bfloat16), cuda(inp["C"], torch.bfloat16),
                                cuda(inp["Z"], torch.bfloat16), cuda(inp["B"]), cuda(inp["sink"]),
                                m=128, W=128, norm_rope=True, inv_rope=True, fused=fused)
    csa.check_device_error()
    ref = O.hca_layer(inp["q"], inp["C"], inp["Z"], inp["B"], inp["sink"], m=128, W=128, norm_rope=True,
                      inv_rope=True, store_round=O.bf16_round)
    assert_close(host(out), ref, what="HCA layer")


def test_flash_prefill_full_size_sampled_rows():
    """The benchmark workload (S 16384, 64 x 512, top-k 512) with grid indexer
    values: top-k sets of sampled rows bit-exact, outputs within tolerance."""
    inp, cfg = synth.prefill_inputs("csa_prefill", grid=True)
    out, idx = _gpu_csa(inp, cfg, torch.bfloat16)
    rows = np.array([0, 3, 4, 127, 128, 2047, 2048, 4095, 8191, 12000, 16383])
    ref, ridx = _oracle_csa(inp, cfg, rows=rows, store=O.bf16_round)
    assert np.array_equal(idx.cpu().numpy()[rows], ridx)
    assert_close(host(out[torch.from_numpy(rows).cuda()]), ref, what="full-size sampled rows")
