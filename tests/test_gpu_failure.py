"""Failure path of the bounded on-chip waits, without faulting the GPU: a wait
on a barrier phase that nothing completes expires after its limit, the kernel
records the expiry in the device error word and returns, csa_check_device_error
reports CSA_ERR_TIMEOUT once (the word is cleared), and the context keeps
running kernels."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close, cuda, host, lib_loaded

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_once_and_the_context_survives():
    import long_context_compressed_02_b200 as csa
    lib_loaded()
    csa.check_device_error()                         # start from a clean error word
    csa.selftest_wait_timeout(2_000_000)             # a 2 ms limit
    with pytest.raises(csa.CsaError, match="CSA_ERR_TIMEOUT"):
        csa.check_device_error()
    csa.check_device_error()                         # reported once, then cleared
    # the context still runs the library's kernels correctly
    rng = np.random.default_rng(5)
    C, Z = rng.standard_normal((64, 128)).astype(np.float32), rng.standard_normal((64, 128)).astype(np.float32)
    B = (0.1 * rng.standard_normal((8, 128))).astype(np.float32)
    kv = csa.csa_compress(cuda(C), cuda(Z), cuda(B), 4, True)
    csa.check_device_error()
    assert_close(host(kv), O.compress(C, Z, B, 4, True), max_abs=1e-5, rel_l2=1e-6, what="compress after expiry")


def test_selftest_rejects_limits_outside_its_range():
    import long_context_compressed_02_b200 as csa
    lib_loaded()
    for bad in (10, 10 ** 9):
        with pytest.raises(csa.CsaError, match="CSA_ERR_INVALID_ARG"):
            csa.selftest_wait_timeout(bad)
