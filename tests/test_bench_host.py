"""Host-side arithmetic of bench.py: its FLOP accounting agrees with the
oracle's count of the same workloads."""
import importlib.util
import os

import oracle as O
from conftest import ROOT


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_prefill_flops_match_oracle_count():
    b = _bench()
    for S, m, k in ((16384, 4, 512), (2048, 4, 64), (777, 4, 100)):
        sparse, window, indexer = b._flops(S, 64, 512, m, k, 128, 64, 128)
        attn, idx = O.flop_counts(S, 64, 512, m, k=k, HI=64, DI=128)
        assert sparse + window == attn and indexer == idx
    # the headline workload's figures
    sparse, window, indexer = b._flops(16384, 64, 512, 4, 512, 128, 64, 128)
    assert abs((sparse + window) / 1e12 - 1.305) < 1e-3 and abs(indexer / 1e12 - 0.550) < 1e-3



def test_bench_calls_only_bound_entry_points():
    """Every `csa.<name>` that bench.py calls exists in the binding, so a leg
    cannot fail on a missing wrapper after the GPU work has started."""
    import re

    import long_context_compressed_02_b200 as csa
    src = open(os.path.join(ROOT, "bench.py")).read()
    names = set(re.findall(r"\bcsa\.([A-Za-z_][A-Za-z0-9_]*)\s*\(", src))
    assert names, "no binding calls found"
    missing = sorted(n for n in names if not hasattr(csa, n))
    assert not missing, missing


def test_oracle_samples_are_shared_by_both_cpu_legs():
    b = _bench()
    rows = b.oracle_rows(16384)
    assert len(rows) == b.ORACLE_ROWS and rows[0] == 0 and rows[-1] == 16383
    shifted = b.oracle_rows(16384, shift=3)
    assert len(shifted) <= b.ORACLE_ROWS and shifted.max() <= 16383
