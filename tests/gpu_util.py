"""Helpers for the GPU parity tests (no test functions here)."""
import numpy as np
import torch

# Output tolerance for BF16 / FP8 inputs (max-abs and relative L2 error).
MAX_ABS = 2e-2
REL_L2 = 5e-3
# Output tolerance of the float32 path (fp32 arithmetic throughout): a float32
# evaluation of the tiny layer in numpy differs from the float64 oracle by
# 8e-7 max-abs and 4e-7 relative L2; these bounds leave a margin of about 25x
# and 12x for other summation orders and the device's expf.
MAX_ABS_F32 = 2e-5
REL_L2_F32 = 5e-6


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    return float(np.abs(diff).max(initial=0.0)), float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30))


def assert_close(got, ref, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    ma, rl = errors(got, ref)
    assert np.all(np.isfinite(np.asarray(got, np.float64))), f"{what}: non-finite output"
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs {ma:.3e} (<= {max_abs}), rel_l2 {rl:.3e} (<= {rel_l2})"


def cuda(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.int32 else t.cpu().numpy()


def lib_loaded():
    """Builds (if needed) and loads libcsa.so; raises if it cannot."""
    from long_context_compressed_02_b200 import build, lib
    build.build()
    return lib()
