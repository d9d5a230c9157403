"""GPU parity of the decode-time cache writer (csa_compress_append): tokens are
streamed one launch at a time through the per-sequence ring, and every cache
row the writer emits is compared with the oracle's batch compressor entry
(RMSNorm + RoPE) quantised to e4m3 with the row scale amax / 448."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import cuda, lib_loaded
from long_context_compressed_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lib_loaded()


@pytest.mark.parametrize("D,m,overlap,dt", [(512, 4, True, "bf16"), (128, 8, False, "f32")])
def test_streamed_cache_rows_match_batch_entries(D, m, overlap, dt):
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(31)
    n_seq, S, steps, r = 2, 72, 40, 64
    C = rng.standard_normal((n_seq, S, D))
    Z = rng.standard_normal((n_seq, S, D))
    B = (0.1 * rng.standard_normal((2 * m if overlap else m, D))).astype(np.float32)
    if dt == "bf16":
        C, Z = synth.to_bf16_values(C), synth.to_bf16_values(Z)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    p0 = np.array([0, 20], np.int64)                 # sequence 1 resumes after a 20-token prefill
    L = 2 * m
    ring_C = torch.zeros(n_seq, L, D, dtype=tdt, device="cuda")
    ring_Z = torch.zeros(n_seq, L, D, dtype=tdt, device="cuda")
    for u in range(max(0, p0[1] - L), p0[1]):
        ring_C[1, u % L] = cuda(C[1, u], tdt)
        ring_Z[1, u % L] = cuda(Z[1, u], tdt)
    cap = S // m
    kv_nope = torch.zeros(n_seq, cap, D - r, dtype=torch.uint8, device="cuda")
    kv_rope = torch.zeros(n_seq, cap, r, dtype=torch.bfloat16, device="cuda")
    kv_scale = torch.full((n_seq, cap), -1.0, device="cuda")
    Bd = cuda(B)
    for s in range(steps):
        pos = p0 + s
        c_tok = cuda(np.stack([C[b, pos[b]] for b in range(n_seq)]), tdt)
        z_tok = cuda(np.stack([Z[b, pos[b]] for b in range(n_seq)]), tdt)
        csa.csa_compress_append(c_tok, z_tok, Bd, m, overlap, cuda(pos), ring_C, ring_Z, kv_nope, kv_rope,
                                kv_scale)
    csa.check_device_error()
    nope_g = kv_nope.cpu().numpy()
    rope_g = kv_rope.float().cpu().numpy()
    scale_g = kv_scale.cpu().numpy()
    same = total = 0
    for b in range(n_seq):
        last = p0[b] + steps - 1
        ref = O.compress(C[b, :last + 1], Z[b, :last + 1], B, m, overlap)
        ref = O.rope_partial(O.rmsnorm(ref), np.arange(ref.shape[0]) * m, r)
        written = [i for i in range(cap) if p0[b] <= (i + 1) * m - 1 <= last]
        for i in range(cap):
            if i not in written:
                assert scale_g[b, i] == -1.0, f"row {i} of sequence {b} should be untouched"
        for i in written:
            v = ref[i]
            codes, rope_ref, s_ref = O.fp8_row_quantize(v, r)
            assert abs(scale_g[b, i] - s_ref) <= 1e-4 * s_ref
            deq = O.e4m3_decode(nope_g[b, i]) * scale_g[b, i]
            # within one e4m3 step of the exact entry (half a step of rounding plus a
            # possible flip at a rounding boundary under fp32 arithmetic)
            bound = np.maximum(np.abs(v[:D - r]) * 2.0 ** -3, s_ref * 2.0 ** -9) * 1.01 + 1e-6
            assert np.all(np.abs(deq - v[:D - r]) <= bound)
            same += int((nope_g[b, i] == codes).sum())
            total += codes.size
            assert np.all(np.abs(rope_g[b, i] - v[D - r:]) <= np.abs(v[D - r:]) * 2.0 ** -8 + 1e-5)
    assert same >= 0.99 * total, f"{same} of {total} codes equal the oracle's"


def test_cache_append_writes_kv_rows_and_indexer_keys():
    """csa_cache_append: in one launch per token, the KV row (RMSNorm + RoPE,
    e4m3 + bf16) and the indexer key of the same block (pooled from its own
    stream, no norm or RoPE, all dims e4m3 under amax / 448) match the oracle's
    batch compressor of each stream."""
    import long_context_compressed_02_b200 as csa
    rng = np.random.default_rng(41)
    n_seq, S, steps, D, DI, m, r = 2, 64, 36, 512, 128, 4, 64
    C = synth.to_bf16_values(rng.standard_normal((n_seq, S, D)))
    Z = synth.to_bf16_values(rng.standard_normal((n_seq, S, D)))
    CI = synth.to_bf16_values(rng.standard_normal((n_seq, S, DI)))
    ZI = synth.to_bf16_values(rng.standard_normal((n_seq, S, DI)))
    B = (0.1 * rng.standard_normal((2 * m, D))).astype(np.float32)
    BI = (0.1 * rng.standard_normal((2 * m, DI))).astype(np.float32)
    bf = torch.bfloat16
    p0 = np.array([0, 13], np.int64)
    L, cap = 2 * m, S // m
    rings = {key: torch.zeros(n_seq, L, d, dtype=bf, device="cuda")
             for key, d in (("C", D), ("Z", D), ("CI", DI), ("ZI", DI))}
    for u in range(max(0, p0[1] - L), p0[1]):
        for key, src in (("C", C), ("Z", Z), ("CI", CI), ("ZI", ZI)):
            rings[key][1, u % L] = cuda(src[1, u], bf)
    kv_nope = torch.zeros(n_seq, cap, D - r, dtype=torch.uint8, device="cuda")
    kv_rope = torch.zeros(n_seq, cap, r, dtype=bf, device="cuda")
    kv_scale = torch.full((n_seq, cap), -1.0, device="cuda")
    kI = torch.zeros(n_seq, cap, DI, dtype=torch.uint8, device="cuda")
    kI_scale = torch.full((n_seq, cap), -1.0, device="cuda")
    for s in range(steps):
        pos = p0 + s
        tok = {key: cuda(np.stack([src[b, pos[b]] for b in range(n_seq)]), bf)
               for key, src in (("C", C), ("Z", Z), ("CI", CI), ("ZI", ZI))}
        csa.csa_cache_append(tok["C"], tok["Z"], cuda(B), m, True, cuda(pos), rings["C"], rings["Z"], kv_nope,
                             kv_rope, kv_scale, tok["CI"], tok["ZI"], cuda(BI), rings["CI"], rings["ZI"], kI,
                             kI_scale)
    csa.check_device_error()
    nope_g, kI_g = kv_nope.cpu().numpy(), kI.cpu().numpy()
    scale_g, kIs_g = kv_scale.cpu().numpy(), kI_scale.cpu().numpy()
    same = total = 0
    for b in range(n_seq):
        last = p0[b] + steps - 1
        ref = O.rope_partial(O.rmsnorm(O.compress(C[b, :last + 1], Z[b, :last + 1], B, m, True)),
                             np.arange((last + 1) // m) * m, r)
        keys = O.compress(CI[b, :last + 1], ZI[b, :last + 1], BI, m, True)
        written = [i for i in range(cap) if p0[b] <= (i + 1) * m - 1 <= last]
        for i in range(cap):
            if i not in written:
                assert scale_g[b, i] == -1.0 and kIs_g[b, i] == -1.0
        for i in written:
            for got_codes, got_scale, v in ((nope_g[b, i], scale_g[b, i], ref[i][:D - r]),
                                            (kI_g[b, i], kIs_g[b, i], keys[i])):
                codes, _, s_ref = O.fp8_row_quantize(v, 0)
                assert abs(got_scale - s_ref) <= 1e-4 * s_ref
                deq = O.e4m3_decode(got_codes) * got_scale
                bound = np.maximum(np.abs(v) * 2.0 ** -3, s_ref * 2.0 ** -9) * 1.01 + 1e-6
                assert np.all(np.abs(deq - v) <= bound)
                same += int((got_codes == codes).sum())
                total += codes.size
    assert same >= 0.99 * total, f"{same} of {total} codes equal the oracle's"
