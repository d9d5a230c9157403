"""The allocation-free indexer entry point (csa_index_topk_noalloc), called
through the C ABI, returns exactly what csa_index_topk returns with a caller
workspace, on two calls in a row.  It serves callers that cannot allocate
device memory; its scratch is a fixed 32 MiB array inside libcsa.so, shared
by every call, so the second call, whose rows are shorter than the first
call's (fewer visible entries, more -1 padding), also checks that scores left
in the array by the first call do not leak into the result.  Collected last on
purpose."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import cuda, lib_loaded
from long_context_compressed_02_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(L):
    fn = L.csa_index_topk_noalloc
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    fn.argtypes = [P, P, P, P, P, P, I, I, I, I, I64, I, I, P, P]
    fn.restype = I
    return fn


def _case(seed, n_seq, T, cap, HI, DI, k, q_pos, grid):
    rng = np.random.default_rng(seed)
    if grid:
        qI = synth.grid_codes(rng, (n_seq, T, HI, DI))
        kI = synth.grid_codes(rng, (n_seq, cap, DI))
        w = (np.floor(rng.random((n_seq, T, HI)) * 16) / 16).astype(np.float32)
    else:
        qI = synth.to_e4m3_codes(rng.standard_normal((n_seq, T, HI, DI)))
        kI = synth.to_e4m3_codes(rng.standard_normal((n_seq, cap, DI)))
        w = rng.random((n_seq, T, HI)).astype(np.float32)
    ks = np.exp2(rng.integers(-2, 3, (n_seq, cap))).astype(np.float32)
    return cuda(qI), cuda(w), cuda(kI), cuda(ks), cuda(np.asarray(q_pos, np.int64))


# q_pos per call: the second call's rows are shorter than the first call's
@pytest.mark.parametrize("shape", [
    dict(n_seq=1, T=600, cap=150, HI=64, DI=128, k=64, q_pos=([0], [0]), grid=True),          # prefill-like
    dict(n_seq=3, T=1, cap=40000, HI=64, DI=128, k=512, q_pos=([159999, 70001, 5], [159999, 70001, 5]),
         grid=False),                                                                             # chunked decode
    dict(n_seq=3, T=1, cap=40000, HI=64, DI=128, k=512, q_pos=([159999, 70001, 4000], [60003, 1000, 2]),
         grid=False),                                                                             # rows shrink
    dict(n_seq=1, T=300, cap=150, HI=64, DI=128, k=64, q_pos=([300], [0]), grid=True),        # prefill, shorter
])
def test_noalloc_matches_workspace_entry_point_on_two_calls(shape):
    import long_context_compressed_02_b200 as csa
    L = lib_loaded()
    fn = _noalloc(L)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    n_seq, T, k = shape["n_seq"], shape["T"], shape["k"]
    for call in range(2):
        qI, w, kI, ks, pos = _case(100 + call, shape["n_seq"], shape["T"], shape["cap"], shape["HI"],
                                   shape["DI"], shape["k"], shape["q_pos"][call], shape["grid"])
        ref = csa.csa_index_topk(qI, w, kI, pos, 4, k, kI_scale=ks)
        got = torch.full((n_seq, T, k), -7, dtype=torch.int32, device="cuda")
        st = fn(ctypes.c_void_p(qI.data_ptr()), None, ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(kI.data_ptr()),
                ctypes.c_void_p(ks.data_ptr()), ctypes.c_void_p(pos.data_ptr()), n_seq, T, shape["HI"], shape["DI"],
                shape["cap"], 4, k, ctypes.c_void_p(got.data_ptr()), stream)
        assert st == 0, L.csa_last_error()
        assert L.csa_check_device_error(stream) == 0
        assert torch.equal(got, ref), f"call {call}: index sets differ"


def test_noalloc_rejects_sizes_beyond_its_array():
    L = lib_loaded()
    fn = _noalloc(L)
    d = ctypes.c_void_p(256)
    # 1 x 16384 queries x 4096 entries of fp32 scores = 256 MiB > 32 MiB
    st = fn(d, None, d, d, None, d, 1, 16384, 64, 128, 4096, 4, 512, d, None)
    assert st == 2 and b"scratch" in L.csa_last_error()
