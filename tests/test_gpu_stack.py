"""GPU parity of the rest of the layer stack against the float64 oracle: the
grouped output projection (tcgen05 GEMMs, both stages) and the sliding-window-
only layer, prefill and decode."""
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


def _oracle_proj(x, rows=None):
    o = host(x["o"]) if rows is None else host(x["o"][rows])
    return O.grouped_out_proj(o, host(x["w_grp"]), host(x["w_out"]), mid_round=O.bf16_round, return_mid=True)


@pytest.mark.parametrize("S,H,D,G,d_mid,d_model,out_dtype", [
    (300, 64, 512, 8, 1024, 4096, torch.float32),    # the model's shape, 3 row tiles with a ragged tail
    (300, 64, 512, 8, 1024, 4096, torch.bfloat16),
    (130, 16, 128, 2, 256, 512, torch.float32),      # other group count, one row past a tile
    (7, 8, 64, 1, 256, 256, torch.bfloat16),         # fewer rows than one tile, a single group
])
def test_grouped_out_proj(S, H, D, G, d_mid, d_model, out_dtype):
    import long_context_compressed_02_b200 as csa
    x, _ = synth.out_proj_inputs_device("cuda", seed=S + G, S=S, H=H, D=D, G=G, d_mid=d_mid, d_model=d_model)
    out, mid = csa.csa_grouped_out_proj(x["o"], x["w_grp"], x["w_out"], out_dtype=out_dtype, return_mid=True)
    csa.check_device_error()
    ref_out, ref_mid = _oracle_proj(x)
    assert_close(host(mid), ref_mid, what="grouped projection intermediate")
    assert_close(host(out), ref_out, what="grouped projection output")


def test_grouped_out_proj_full_size_sampled_rows():
    """The full workload (16384 tokens, 64 x 512 -> 8 x 1024 -> 4096); sampled
    rows at tile edges and the last row against the oracle."""
    import long_context_compressed_02_b200 as csa
    x, cfg = synth.out_proj_inputs_device("cuda", seed=0)
    out, mid = csa.csa_grouped_out_proj(x["o"], x["w_grp"], x["w_out"], return_mid=True)
    csa.check_device_error()
    rows = [0, 1, 127, 128, 4095, 8191, 16383]
    ref_out, ref_mid = _oracle_proj(x, rows)
    assert_close(host(mid[rows]), ref_mid, what="full-size intermediate")
    assert_close(host(out[rows]), ref_out, what="full-size output")


def test_grouped_out_proj_zero_rows_and_linearity():
    """M = 0 is a no-op; doubling the input doubles the output exactly (powers
    of two commute with bf16 rounding and fp32 accumulation)."""
    import long_context_compressed_02_b200 as csa
    x, _ = synth.out_proj_inputs_device("cuda", seed=3, S=200, H=16, D=128, G=2, d_mid=256, d_model=256)
    empty = torch.empty((0, 16, 128), dtype=torch.bfloat16, device="cuda")
    assert csa.csa_grouped_out_proj(empty, x["w_grp"], x["w_out"]).shape == (0, 256)
    a = csa.csa_grouped_out_proj(x["o"], x["w_grp"], x["w_out"], out_dtype=torch.float32)
    b = csa.csa_grouped_out_proj(x["o"] * 2, x["w_grp"], x["w_out"], out_dtype=torch.float32)
    csa.check_device_error()
    assert torch.equal(b, 2 * a)


def test_swa_layer_prefill():
    import long_context_compressed_02_b200 as csa
    inp, cfg = synth.prefill_inputs("csa_prefill", S=700)
    dt = torch.bfloat16
    out = csa.swa_layer_prefill(cuda(inp["q"], dt), cuda(inp["C"], dt), cuda(inp["sink"]), W=cfg["W"],
                                norm_rope=True, inv_rope=True)
    csa.check_device_error()
    ref = O.swa_layer(inp["q"], inp["C"], inp["sink"], W=cfg["W"], norm_rope=True, inv_rope=True,
                      store_round=O.bf16_round)
    assert_close(host(out), ref, what="window-only layer (prefill)")


def test_swa_layer_decode():
    import long_context_compressed_02_b200 as csa
    g = torch.Generator(device="cuda").manual_seed(11)
    n_seq, H, D, W = 6, 64, 512, 128
    lay = {"q": torch.randn(n_seq, 1, H, D, generator=g, device="cuda").to(torch.bfloat16),
           "swa": torch.randn(n_seq, W, D, generator=g, device="cuda").to(torch.bfloat16),
           "sink": torch.randn(H, generator=g, device="cuda")}
    pos = torch.tensor([0, 5, 126, 127, 128, (1 << 20) - 1], dtype=torch.int64, device="cuda")
    out = csa.swa_layer_decode(lay, pos, W=W)
    csa.check_device_error()
    q, swa, sink = host(lay["q"]), host(lay["swa"]), host(lay["sink"])
    for b, t in enumerate(pos.tolist()):
        n = min(W, t + 1)
        ref = O.window_sink_combine(q[b], None, [t], W, sink, np.zeros((1, H, D)), np.full((1, H), -np.inf),
                                    inv_rope=True, window_rows=[swa[b][:n]])
        assert_close(host(out[b]), ref, what=f"window-only layer (decode) b={b}")
