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

