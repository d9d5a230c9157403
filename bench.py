#!/usr/bin/env python
"""Benchmark of the CSA layer forward on B200 (Flash-shaped prefill:
S 16384, 64 heads x 512, m 4 with overlap -> 4096 entries, e4m3 indexer
64 x 128, top-k 512, window 128, sink).

One step = the whole hot path of the layer, in the library's kernels:
  Q RMSNorm+RoPE, window-row RMSNorm+RoPE, compressor (+ K norm/RoPE),
  lightning indexer + top-k, and the fused attention (selected entries +
  128-token window + sink in one softmax, inverse RoPE, bf16 output).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent
replica of the workload (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA decode tokens/s @1M ctx and prefill TFLOP/s, % of HBM/TC roofline"
WORKLOAD = "csa_prefill"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# dominant kernels, from ncu captures of smaller cases of the same kernels scaled
# by the units processed: the fused attention at S 4096 (507.5 MB) x 4 for
# S 16384; the indexer scores kernel at decode batch 4 (142.9 MB) x 4 for
# batch 16.  Reset to None whenever one of these kernels changes.
PROFILED_TRAFFIC = {"fused_attention": 4 * 507.55e6, "index_topk": 4 * 142.95e6}


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def fp8_peak_tflops(torch, dev, n=8192, reps=10):
    """Dense e4m3 tensor throughput of this GPU, measured here with the library
    FP8 GEMM (torch._scaled_mm, cuBLASLt) on n^3, best of `reps` by CUDA events:
    the roofline denominator of the FP8 indexer (no FP8 figure is recorded with
    the measured HBM and BF16 peaks).  None if the library call is unavailable."""
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev)
        best = None
        for _ in range(reps + 2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) * 1e-3
            best = t if best is None else min(best, t)
        return 2.0 * n ** 3 / best / 1e12
    except Exception:
        return None


def _flops(S, H, D, m, k, W, HI, DI):
    t = np.arange(S, dtype=np.int64)
    nv = (t + 1) // m
    sparse = 4 * D * H * int(np.minimum(k, nv).sum())
    window = 4 * D * H * int(np.minimum(W, t + 1).sum())
    indexer = 2 * HI * DI * int(nv.sum())
    return sparse, window, indexer


class Clocks:
    """Samples the GPU's SM clock, power and clock-event reasons every 10 ms
    from a background thread (NVML, read-only queries) while the benchmark
    runs; summary() reports the samples taken between mark_start() and
    mark_end().  Falls back to nothing if NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, torch, device):
        import threading
        self.samples, self.t0, self.t1 = [], None, None
        self.stop_ev = threading.Event()
        self.h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.h = None
            return
        self.th = threading.Thread(target=self._run, daemon=True)
        self.th.start()

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self.h),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
            except Exception:
                pass
            self.stop_ev.wait(0.01)

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self.h is None:
            return None
        self.stop_ev.set()
        self.th.join(timeout=2)
        rows = [r for r in self.samples if self.t0 is not None and self.t0 <= r[0] <= (self.t1 or r[0])]
        if not rows:
            return None
        reasons = sorted({n for r in rows for n, bit in self.REASONS if r[2] & bit})
        return {"sm_mhz": float(np.median([r[1] for r in rows])), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[3] for r in rows),
                "source": "NVML every 10 ms during the timed region"}


# Query rows per oracle sample: the reference arm times one such sample per
# step and the cpu_baseline leg one sample, so both rates are the same
# measurement (each sample also runs the oracle's full-sequence compressor
# and window-row passes, whose cost is spread over these rows).
ORACLE_ROWS = 2048


def oracle_rows(S, shift=0):
    """ORACLE_ROWS evenly spaced query rows of an S-token layer, moved by
    `shift` (different samples for different reference-arm steps)."""
    base = np.linspace(0, S - 1, min(S, ORACLE_ROWS)).astype(np.int64)
    return np.unique(np.minimum(S - 1, base + shift))


def cpu_oracle_sample(inp_host, cfg, rows):
    """Times the float64 oracle on the given query rows of the workload."""
    import oracle as O
    cores = _blas_threads()
    t0 = time.perf_counter()
    O.csa_layer(inp_host["q"][rows], inp_host["C"], inp_host["Z"], inp_host["B"],
                O.e4m3_decode(inp_host["qI_codes"][rows]), inp_host["w"][rows],
                O.e4m3_decode(inp_host["kI_codes"]), inp_host["sink"], k=cfg["k"], m=cfg["m"], W=cfg["W"],
                norm_rope=True, inv_rope=True, rows=rows, row_inputs=True)
    dt = time.perf_counter() - t0
    t = np.asarray(rows, np.int64)
    nv = (t + 1) // cfg["m"]
    fl = (4 * cfg["D"] * cfg["H"] * (np.minimum(cfg["k"], nv) + np.minimum(cfg["W"], t + 1)).sum()
          + 2 * cfg["HI"] * cfg["DI"] * nv.sum())
    return float(fl), dt, cores


def host_inputs(dev_inp):
    """float32 / uint8 numpy copies of the workload tensors."""
    import torch
    return {k: (v.cpu().numpy() if v.dtype == torch.uint8 else v.float().cpu().numpy()) for k, v in dev_inp.items()}


def run_reference(args, rank, world):
    """Reference arm: the float64 CPU oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import torch
    from long_context_compressed_02_b200 import synth
    inp, cfg = synth.prefill_inputs_device(WORKLOAD, "cpu", seed=0)
    host = host_inputs(inp)
    times, flops = [], []
    cores = 1
    for step in range(args.warmup + args.steps):
        rows = oracle_rows(cfg["S"], shift=step)
        fl, dt, cores = cpu_oracle_sample(host, cfg, rows)
        if step >= args.warmup:
            times.append(dt)
            flops.append(fl)
    value = sum(flops) / sum(times) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "S": cfg["S"], "H": cfg["H"], "D": cfg["D"], "m": cfg["m"],
                       "top_k": cfg["k"], "window": cfg["W"],
                       "sample": f"{ORACLE_ROWS} evenly spaced query rows per step (shifted by the step index)"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{ORACLE_ROWS} evenly spaced query rows of the S=16384 layer per step, "
                                       "including the oracle's full-sequence compressor and window-row passes "
                                       "(the same sample as the native arm's cpu_baseline)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        return len(os.sched_getaffinity(0))


def decode_oracle_sample(inp, cfg, b=0):
    """Times the float64 oracle's whole decode step (indexer over every visible
    entry, top-k, attention over the selected entries + SWA cache + sink) for
    sequence b of the batch.  Its inputs, the caches decoded exactly to float64
    through the e4m3 code table, are prepared before the clock starts."""
    import oracle as O
    tab = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    D, ne = cfg["D"], cfg["n_e"]
    kI = tab[inp["kI"][b].cpu().numpy()] * inp["kI_scale"][b].double().cpu().numpy()[:, None]
    qI = tab[inp["qI"][b, 0].cpu().numpy()] * inp["qI_scale"][b, 0].double().cpu().numpy()[:, None]
    kv = np.empty((ne, D))
    kv[:, :D - 64] = tab[inp["kv_nope"][b].cpu().numpy()]
    kv[:, :D - 64] *= inp["kv_scale"][b].double().cpu().numpy()[:, None]
    kv[:, D - 64:] = inp["kv_rope"][b].double().cpu().numpy()
    q = inp["q"][b, 0].double().cpu().numpy()
    w = inp["w"][b, 0].double().cpu().numpy()
    swa = inp["swa"][b].double().cpu().numpy()
    sink = inp["sink"].double().cpu().numpy()
    t = int(inp["q_pos"][b].item())
    t0 = time.perf_counter()
    O.csa_decode(q, qI, w, kI, kv, swa, sink, t, k=cfg["k"], m=4, inv_rope=True)
    dt = time.perf_counter() - t0
    return {"value": 1.0 / dt, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"one whole decode step of sequence {b} ({ne} entries, top-k {cfg['k']}), {dt:.2f} s; "
                      "caches decoded to float64 beforehand"}


def decode_leg(dev, steps, warmup, csa, synth, torch, batch=None, seed=1, n_split=None, cpu_baseline=False):
    """CSA decode at 2^20 context, batch 16 (one new token per sequence): indexer
    scan over the e4m3 key cache + top-k, then the fused attention over the 512
    selected e4m3 entries, the 128-row bf16 SWA cache and the sink."""
    inp, cfg = synth.decode_inputs_device("csa_decode_1m", dev, seed=seed, batch=batch)
    Bn, ne, k, W, H, D, HI, DI = (cfg[x] for x in ("batch", "n_e", "k", "W", "H", "D", "HI", "DI"))
    ws = torch.empty(csa.csa_index_topk_workspace(Bn, 1, ne, k), dtype=torch.uint8, device=dev)
    idx = torch.empty(Bn, 1, k, dtype=torch.int32, device=dev)
    out = torch.empty(Bn, 1, H, D, dtype=torch.bfloat16, device=dev)
    # split each token's 10 half chunks (8 x 64 selected entries + the window)
    # into ranges of about two (more splits cost more in partials than they gain)
    if n_split is None:
        n_split = max(1, min(5, csa.num_sms() // Bn))
    aws = torch.empty(csa.csa_fused_attention_workspace(Bn, 1, H, D, n_split), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        csa.csa_index_topk(inp["qI"], inp["w"], inp["kI"], inp["q_pos"], 4, k, qI_scale=inp["qI_scale"],
                           kI_scale=inp["kI_scale"], workspace=ws, idx=idx)
        if ev is not None:
            ev[1].record(stream)
        csa.csa_fused_attention(inp["q"], inp["kv_nope"], inp["swa"], inp["q_pos"], W, inp["sink"], idx=idx,
                                kv_rope=inp["kv_rope"], kv_scale=inp["kv_scale"], window_mode=1, inv_rope=True,
                                rope_dim=64, out=out, n_split=n_split, workspace=aws)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(3, warmup)):
        step()
    csa.check_device_error()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    csa.check_device_error()
    # the decode-time cache writer for the same batch: append one token per
    # sequence (at a block boundary, so every call emits an e4m3 KV row and the
    # block's e4m3 indexer key)
    m_c = 4
    ring_C = torch.zeros(Bn, 2 * m_c, D, dtype=torch.bfloat16, device=dev)
    ring_Z = torch.zeros_like(ring_C)
    ring_CI = torch.zeros(Bn, 2 * m_c, DI, dtype=torch.bfloat16, device=dev)
    ring_ZI = torch.zeros_like(ring_CI)
    c_tok = torch.randn(Bn, D, device=dev).to(torch.bfloat16)
    z_tok = torch.randn(Bn, D, device=dev).to(torch.bfloat16)
    ci_tok = torch.randn(Bn, DI, device=dev).to(torch.bfloat16)
    zi_tok = torch.randn(Bn, DI, device=dev).to(torch.bfloat16)
    B_c = torch.zeros(2 * m_c, D, device=dev)
    B_i = torch.zeros(2 * m_c, DI, device=dev)
    pos_c = torch.full((Bn,), 4 * 1000 - 1, dtype=torch.int64, device=dev)
    row_nope = torch.empty(Bn, 1024, D - 64, dtype=torch.uint8, device=dev)
    row_rope = torch.empty(Bn, 1024, 64, dtype=torch.bfloat16, device=dev)
    row_scale = torch.empty(Bn, 1024, device=dev)
    key_codes = torch.empty(Bn, 1024, DI, dtype=torch.uint8, device=dev)
    key_scale = torch.empty(Bn, 1024, device=dev)

    def append():
        csa.csa_cache_append(c_tok, z_tok, B_c, m_c, True, pos_c, ring_C, ring_Z, row_nope, row_rope, row_scale,
                             ci_tok, zi_tok, B_i, ring_CI, ring_ZI, key_codes, key_scale)
    for _ in range(3):
        append()
    wa, wb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wa.record(stream)
    for _ in range(steps):
        append()
    wb.record(stream)
    torch.cuda.synchronize()
    csa.check_device_error()
    t_app = wa.elapsed_time(wb) / steps
    t_idx = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_att = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms = float(np.mean([e[0].elapsed_time(e[2]) for e in evs]))
    # algorithmic bytes: every visible indexer key + scale, the selected e4m3 rows
    # (448 + 128 + 4 bytes), the SWA rows, the queries; plus the fp32 score row
    # written and read once by the selection
    scan = Bn * ne * (DI + 4)
    gather = Bn * k * (D - 64 + 128 + 4)
    swa = Bn * W * D * 2
    qbytes = Bn * (H * D * 2 + HI * DI + HI * 8)
    algo = scan + gather + swa + qbytes
    hbm, _, _, src = _peaks()
    ach_idx = scan / (t_idx * 1e-3) / 1e9
    cpu = decode_oracle_sample(inp, cfg) if cpu_baseline else None
    return {"workload": "csa_decode_1m", "batch": Bn, "cpu_baseline": cpu, "attention_splits": n_split, "context": cfg["ctx"], "entries": ne, "top_k": k,
            "tokens_per_s": Bn / (ms * 1e-3), "ms_per_step": ms, "kernels_ms": {"index_topk": t_idx,
                                                                                 "fused_attention": t_att},
            "algorithmic_bytes_per_step": algo,
            "cache_append": {"ms": t_app, "rows_per_call": Bn,
                             "note": "new token appended to the 2m-token rings, the block's KV entry pooled, "
                                     "normalised, rotated and written as an e4m3 cache row, and its indexer key "
                                     "pooled and written as an e4m3 key row, one launch (not part of ms_per_step)"},
            "hbm_frac_step": algo / (ms * 1e-3) / 1e9 / hbm,
            "roofline": {"kernel": "index_topk", "bound": "hbm", "achieved": ach_idx, "peak": hbm, "unit": "GB/s",
                         "frac": ach_idx / hbm,
                         "traffic": PROFILED_TRAFFIC["index_topk"] if Bn == 16 else None,
                         "peak_source": f"{src} copy bandwidth"}}


def decode_fp4_leg(dev, steps, warmup, csa, synth, torch, seed=1, n_split=None):
    """The 2^20-context decode step of decode_leg with the indexer's QK path in
    MX FP4: packed E2M1 keys (64 B) + E8M0 block scales (4 B) per entry, 68 B
    scanned per entry instead of 132 B."""
    inp, cfg = synth.decode_inputs_device("csa_decode_1m", dev, seed=seed)
    Bn, ne, k, W, H, D, HI, DI = (cfg[x] for x in ("batch", "n_e", "k", "W", "H", "D", "HI", "DI"))
    g = torch.Generator(device=dev).manual_seed(seed + 100)
    kI4 = torch.randint(0, 256, (Bn, ne, 64), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
    kI4s = torch.randint(125, 130, (Bn, ne, 4), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
    qI4 = torch.randint(0, 256, (Bn, 1, HI, 64), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
    qI4s = torch.randint(125, 130, (Bn, 1, HI, 4), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
    ws = torch.empty(csa.csa_index_topk_fp4_workspace(Bn, 1, HI, ne, k), dtype=torch.uint8, device=dev)
    idx = torch.empty(Bn, 1, k, dtype=torch.int32, device=dev)
    out = torch.empty(Bn, 1, H, D, dtype=torch.bfloat16, device=dev)
    if n_split is None:
        n_split = max(1, min(5, csa.num_sms() // Bn))
    aws = torch.empty(csa.csa_fused_attention_workspace(Bn, 1, H, D, n_split), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        csa.csa_index_topk_fp4(qI4, qI4s, inp["w"], kI4, kI4s, inp["q_pos"], 4, k, workspace=ws, idx=idx)
        if ev is not None:
            ev[1].record(stream)
        csa.csa_fused_attention(inp["q"], inp["kv_nope"], inp["swa"], inp["q_pos"], W, inp["sink"], idx=idx,
                                kv_rope=inp["kv_rope"], kv_scale=inp["kv_scale"], window_mode=1, inv_rope=True,
                                rope_dim=64, out=out, n_split=n_split, workspace=aws)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(3, warmup)):
        step()
    csa.check_device_error()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    csa.check_device_error()
    t_idx = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_att = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms = float(np.mean([e[0].elapsed_time(e[2]) for e in evs]))
    scan = Bn * ne * (64 + 4)
    gather = Bn * k * (D - 64 + 128 + 4)
    algo = scan + gather + Bn * W * D * 2 + Bn * (H * D * 2 + HI * 68 + HI * 4)
    hbm, _, _, src = _peaks()
    ach_idx = scan / (t_idx * 1e-3) / 1e9
    return {"workload": "csa_decode_1m_fp4_indexer", "batch": Bn, "entries": ne, "top_k": k,
            "tokens_per_s": Bn / (ms * 1e-3), "ms_per_step": ms,
            "kernels_ms": {"index_topk_fp4": t_idx, "fused_attention": t_att},
            "algorithmic_bytes_per_step": algo, "hbm_frac_step": algo / (ms * 1e-3) / 1e9 / hbm,
            "roofline": {"kernel": "index_topk_fp4", "bound": "hbm", "achieved": ach_idx, "peak": hbm,
                         "unit": "GB/s", "frac": ach_idx / hbm, "traffic": None,
                         "peak_source": f"{src} copy bandwidth"}}


def mixed_decode_leg(dev, steps, warmup, csa, synth, torch, seed=0, split=None):
    """The 4-layer decode stack (CSA, HCA, CSA, HCA), batch 32, per-sequence
    contexts U[64K, 1M]: one new token per sequence through all four layers."""
    layers, q_pos, cfg = synth.mixed_decode_inputs_device(dev, seed=seed)
    Bn, k, W, H, D, HI, DI = (cfg[x] for x in ("batch", "k", "W", "H", "D", "HI", "DI"))
    L = cfg["lengths"]
    sms = csa.num_sms()
    # split-KV ranges per sequence (items are claimed dynamically, so unequal
    # sequence lengths balance across CTAs)
    if split is None:
        split = {"csa": max(1, min(9, sms // Bn)), "hca": 12}
    bufs = []
    for lay in layers:
        b = {"out": torch.empty(Bn, 1, H, D, dtype=torch.bfloat16, device=dev)}
        cap = lay["kv_nope"].shape[1]
        ns = split[lay["kind"]]
        b["aws"] = torch.empty(csa.csa_fused_attention_workspace(Bn, 1, H, D, ns), dtype=torch.uint8, device=dev)
        if lay["kind"] == "csa":
            b["idx"] = torch.empty(Bn, 1, k, dtype=torch.int32, device=dev)
            b["iws"] = torch.empty(csa.csa_index_topk_workspace(Bn, 1, cap, k), dtype=torch.uint8, device=dev)
        bufs.append(b)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        for i, (lay, b) in enumerate(zip(layers, bufs)):
            if ev is not None:
                ev[i].record(stream)
            if lay["kind"] == "csa":
                csa.csa_layer_decode(lay, q_pos, k=k, n_split=split["csa"], idx=b["idx"], out=b["out"],
                                     index_workspace=b["iws"], attn_workspace=b["aws"])
            else:
                csa.hca_layer_decode(lay, q_pos, n_split=split["hca"], out=b["out"], attn_workspace=b["aws"])
        if ev is not None:
            ev[len(layers)].record(stream)

    for _ in range(max(3, warmup)):
        step()
    csa.check_device_error()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(layers) + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    csa.check_device_error()
    per_layer = [float(np.mean([e[i].elapsed_time(e[i + 1]) for e in evs])) for i in range(len(layers))]
    ms = float(np.mean([e[0].elapsed_time(e[len(layers)]) for e in evs]))
    # algorithmic bytes per step: CSA = every visible indexer key + scale, the
    # selected e4m3 rows (448 + 128 + 4 bytes); HCA = every complete entry;
    # both = the SWA rows and the query side
    row = D - 64 + 128 + 4
    qside = H * D * 2
    algo = 0
    for lay in layers:
        if lay["kind"] == "csa":
            nv = (L // 4)
            algo += int((nv * (DI + 4)).sum() + (np.minimum(k, nv) * row).sum()) + Bn * (HI * DI + HI * 8)
        else:
            algo += int(((L // 128) * row).sum())
        algo += Bn * (W * D * 2 + qside)
    hbm, _, _, src = _peaks()
    return {"workload": "mixed_decode", "layers": [l["kind"] for l in layers], "batch": Bn,
            "context_min": int(L.min()), "context_max": int(L.max()), "top_k": k,
            "attention_splits": split, "tokens_per_s": Bn / (ms * 1e-3), "ms_per_step": ms,
            "layers_ms": per_layer, "algorithmic_bytes_per_step": algo,
            "hbm_frac_step": algo / (ms * 1e-3) / 1e9 / hbm, "peak_source": f"{src} copy bandwidth"}


def hca_prefill_leg(dev, steps, warmup, csa, synth, torch, seed=0):
    """HCA layer prefill, S 131072, 64 x 512 bf16, m' 128 (1024 entries):
    Q and window-row RMSNorm + RoPE, compressor (+ K norm / RoPE), and the fused
    dense attention over complete entries + 128-token window + sink."""
    inp, cfg = synth.prefill_inputs_device("hca_prefill", dev, seed=seed)
    S, H, D, m, W = (cfg[x] for x in ("S", "H", "D", "m", "W"))
    ne = S // m
    bf = torch.bfloat16
    pos = torch.zeros(1, dtype=torch.int64, device=dev)
    qn = torch.empty(S, H, D, dtype=bf, device=dev)
    kt = torch.empty(S, D, dtype=bf, device=dev)
    kv = torch.empty(ne, D, dtype=bf, device=dev)
    out = torch.empty(1, S, H, D, dtype=bf, device=dev)
    stream = torch.cuda.current_stream()
    names = ["q_norm_rope", "kv_tok_norm_rope", "compress", "fused_attention"]

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        csa.csa_rmsnorm_rope(inp["q"], rows_per_pos=H, out=qn)
        mark(1)
        csa.csa_rmsnorm_rope(inp["C"], rows_per_pos=1, out=kt)
        mark(2)
        csa.csa_compress(inp["C"], inp["Z"], inp["B"], m, False, norm=True, rope_dim=64, out=kv)
        mark(3)
        csa.csa_fused_attention(qn[None], kv[None], kt[None], pos, W, inp["sink"], m=m, inv_rope=True,
                                rope_dim=64, out=out)
        mark(4)

    for _ in range(max(3, warmup)):
        step()
    csa.check_device_error()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    csa.check_device_error()
    per = {n: float(np.mean([e[j].elapsed_time(e[j + 1]) for e in evs])) for j, n in enumerate(names)}
    ms = float(np.mean([e[0].elapsed_time(e[len(names)]) for e in evs]))
    t = np.arange(S, dtype=np.int64)
    fl_dense = 4 * D * H * int(((t + 1) // m).sum())
    fl_window = 4 * D * H * int(np.minimum(W, t + 1).sum())
    _, bf16_burst, _, src = _peaks()
    ach = (fl_dense + fl_window) / (per["fused_attention"] * 1e-3) / 1e12
    return {"workload": "hca_prefill", "S": S, "H": H, "D": D, "m": m, "entries": ne, "window": W,
            "tflops": (fl_dense + fl_window) / (ms * 1e-3) / 1e12, "ms_per_step": ms,
            "prefill_tokens_per_s": S / (ms * 1e-3), "kernels_ms": per,
            "flops_per_step": {"hca_dense": fl_dense, "swa_window": fl_window},
            "roofline": {"kernel": "fused_attention", "bound": "tensor", "achieved": ach, "peak": bf16_burst,
                         "unit": "TFLOP/s", "frac": ach / bf16_burst, "traffic": None,
                         "peak_source": f"{src} bf16 burst (timed region well under a second)"}}


def out_proj_leg(dev, steps, warmup, csa, synth, torch, seed=0, S=None):
    """Grouped output projection of one prefill layer's attention output:
    16384 tokens, 64 heads x 512 in 8 groups -> 8 x 1024 (bf16 intermediate)
    -> 4096; two launches of the tcgen05 GEMM kernel per step.  The input
    (1 GiB) is larger than L2."""
    x, cfg = synth.out_proj_inputs_device(dev, seed=seed, S=S)
    S, H, D, G, dm, dmod = (cfg[k] for k in ("S", "H", "D", "G", "d_mid", "d_model"))
    bf = torch.bfloat16
    mid = torch.empty(S, G * dm, dtype=bf, device=dev)
    out = torch.empty(S, dmod, dtype=bf, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        csa.csa_grouped_out_proj(x["o"], x["w_grp"], x["w_out"], mid=mid, out=out)

    for _ in range(max(3, warmup)):
        step()
    csa.check_device_error()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in evs:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    csa.check_device_error()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    fl_group = 2 * S * H * D * dm
    fl_out = 2 * S * G * dm * dmod
    _, bf16_burst, _, src = _peaks()
    ach = (fl_group + fl_out) / (ms * 1e-3) / 1e12
    return {"workload": "out_proj", "S": S, "H": H, "D": D, "groups": G, "d_mid": dm, "d_model": dmod,
            "ms_per_step": ms, "tflops": ach, "tokens_per_s": S / (ms * 1e-3),
            "flops_per_step": {"group_stage": fl_group, "output_stage": fl_out},
            "roofline": {"kernel": "proj_gemm", "bound": "tensor", "achieved": ach, "peak": bf16_burst,
                         "unit": "TFLOP/s", "frac": ach / bf16_burst, "traffic": None,
                         "peak_source": f"{src} bf16 burst (the leg runs alone, a few ms)"}}


def tiny_leg(dev, steps, warmup, csa, synth, torch):
    """The tiny fp32 CSA layer (S 2048, 8 heads x 128, indexer 4 x 32, top-k 64):
    launch-latency bound; reported in microseconds per layer step (4 kernels)."""
    inp, cfg = synth.prefill_inputs("tiny_csa")
    S, H, D, m, k, W, HI, DI = (cfg[x] for x in ("S", "H", "D", "m", "k", "W", "HI", "DI"))

    def dv(x):
        return torch.from_numpy(np.ascontiguousarray(x)).to(dev)

    q, C, Z, B, qI, w, kI, sink = (dv(inp[x]) for x in ("q", "C", "Z", "B", "qI_codes", "w", "kI_codes", "sink"))
    ws = torch.empty(csa.csa_index_topk_workspace(1, S, S // m, k), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        csa.csa_layer_prefill(q, C, Z, B, qI, w, kI, sink, k=k, m=m, W=W, workspace=ws)

    for _ in range(max(3, warmup)):
        step()
    csa.check_device_error()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in evs:
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    csa.check_device_error()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    sparse, window, indexer = _flops(S, H, D, m, k, W, HI, DI)
    return {"workload": "tiny_csa", "S": S, "H": H, "D": D, "dtype": "f32 storage and fp32 attention arithmetic",
            "us_per_step": ms * 1e3, "kernels_per_step": 4,
            "flops_per_step": {"attention": sparse + window, "indexer_fp8": indexer},
            "bound": "launch latency"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--S", type=int, default=None, help="shorter sequence (profiling cases only)")
    ap.add_argument("--no-decode", action="store_true", help="skip the 1M-context decode leg")
    ap.add_argument("--decode-batch", type=int, default=None, help="fewer decode sequences (profiling cases only)")
    ap.add_argument("--no-prefill", action="store_true", help="run only the decode legs (profiling cases only)")
    ap.add_argument("--no-hca", action="store_true", help="skip the HCA prefill leg (S 131072)")
    ap.add_argument("--no-mixed", action="store_true", help="skip the 4-layer mixed decode leg")
    ap.add_argument("--no-out-proj", action="store_true", help="skip the grouped output projection leg")
    ap.add_argument("--no-tiny", action="store_true", help="skip the tiny fp32 layer leg")
    ap.add_argument("--out-proj-only", action="store_true", help="run only the output projection leg (profiling)")
    args = ap.parse_args()
    from long_context_compressed_02_b200 import replicas
    rank, world, local = replicas.rank_world()

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    import long_context_compressed_02_b200 as csa
    from long_context_compressed_02_b200 import build, synth
    build.build()
    csa.lib()

    if args.out_proj_only:
        leg = out_proj_leg(dev, args.steps, args.warmup, csa, synth, torch, seed=replicas.replica_seed(rank), S=args.S)
        if rank == 0:
            print(json.dumps({"out_proj": leg}), flush=True)
        return
    if args.no_prefill:
        out = {}
        if not args.no_decode:
            out["decode_1m"] = decode_leg(dev, args.steps, args.warmup, csa, synth, torch, batch=args.decode_batch,
                                        seed=replicas.replica_seed(rank, base=1))
        if not args.no_mixed:
            out["decode_mixed"] = mixed_decode_leg(dev, args.steps, args.warmup, csa, synth, torch, seed=replicas.replica_seed(rank))
        if rank == 0:
            print(json.dumps(out), flush=True)
        return
    inp, cfg = synth.prefill_inputs_device(WORKLOAD, dev, seed=replicas.replica_seed(rank), S=args.S)
    S, H, D, m, k, W, HI, DI = (cfg[x] for x in ("S", "H", "D", "m", "k", "W", "HI", "DI"))
    ne = S // m
    bf = torch.bfloat16
    pos = torch.zeros(1, dtype=torch.int64, device=dev)
    # persistent buffers (the library allocates nothing)
    qn = torch.empty(S, H, D, dtype=bf, device=dev)
    kt = torch.empty(S, D, dtype=bf, device=dev)
    kv = torch.empty(ne, D, dtype=bf, device=dev)
    idx = torch.empty(1, S, k, dtype=torch.int32, device=dev)
    ws = torch.empty(csa.csa_index_topk_workspace(1, S, ne, k), dtype=torch.uint8, device=dev)
    out = torch.empty(1, S, H, D, dtype=bf, device=dev)
    stream = torch.cuda.current_stream()
    # The query RMSNorm/RoPE (memory-bound) runs on a second stream, beside the
    # key side (window rows, compressor, indexer + top-k, which is compute-bound);
    # the attention waits for both.  Each step's query pass waits for the
    # previous step's attention, which reads the same buffer.
    side = torch.cuda.Stream(device=dev)
    fork, join = torch.cuda.Event(), torch.cuda.Event()
    names = ["q_norm_rope", "kv_tok_norm_rope", "compress", "index_topk", "fused_attention"]

    def step(ev=None, x=None, o=None):
        x = inp if x is None else x            # this step's inputs and output buffer
        o = out if o is None else o

        def mark(i, s=stream):
            if ev is not None:
                ev[i].record(s)
        fork.record(stream)
        side.wait_event(fork)
        mark(0, side)
        csa.csa_rmsnorm_rope(x["q"], rows_per_pos=H, out=qn, stream=side)
        mark(6, side)
        join.record(side)
        mark(1)
        csa.csa_rmsnorm_rope(x["C"], rows_per_pos=1, out=kt)
        mark(2)
        csa.csa_compress(x["C"], x["Z"], x["B"], m, True, norm=True, rope_dim=64, out=kv)
        mark(3)
        csa.csa_index_topk(x["qI_codes"][None], x["w"][None], x["kI_codes"][None], pos, m, k,
                           workspace=ws, idx=idx)
        mark(7)
        stream.wait_event(join)
        mark(4)
        csa.csa_fused_attention(qn[None], kv[None], kt[None], pos, W, x["sink"], idx=idx, inv_rope=True,
                                rope_dim=64, out=o)
        mark(5)

    launches_per_step = 6      # 2 norm/rope, compress, indexer scores, top-k, fused attention
    clocks = Clocks(torch, dev) if rank == 0 else None
    for _ in range(max(3, args.warmup)):
        step()
    csa.check_device_error()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 3)] for _ in range(args.steps)]
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if clocks:
        clocks.mark_start()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    barrier()
    if clocks:
        clocks.mark_end()
    clk = clocks.stop() if clocks else None
    csa.check_device_error()
    ms = t_start.elapsed_time(t_end) / args.steps
    # events: 0 / 6 around the query pass (second stream), 1, 2, 3, 7 around the key-side
    # calls, 4 / 5 around the attention (after its wait for the query pass)
    spans = {"q_norm_rope": (0, 6), "kv_tok_norm_rope": (1, 2), "compress": (2, 3), "index_topk": (3, 7),
             "fused_attention": (4, 5)}
    per = {n: float(np.mean([evs[i][a].elapsed_time(evs[i][b]) for i in range(args.steps)]))
           for n, (a, b) in spans.items()}
    ms = replicas.max_over_ranks(ms, device=dev)      # the slowest replica's step time

    fl_sparse, fl_window, fl_index = _flops(S, H, D, m, k, W, HI, DI)
    fl_total = fl_sparse + fl_window + fl_index
    value = replicas.job_rate(fl_total, world, ms * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers (every rank its own
    # replica; the job's time is the slowest rank's).  Each step uploads its
    # inputs from pinned host memory and downloads its output; uploads, compute
    # and downloads of consecutive steps overlap on three streams with
    # double-buffered device inputs and outputs (a serving pipeline's shape).
    e2e = None
    if not args.no_e2e:
        keys = ["q", "C", "Z", "B", "qI_codes", "w", "kI_codes", "sink"]
        pinned = {kk: torch.empty(inp[kk].shape, dtype=inp[kk].dtype, pin_memory=True) for kk in keys}
        for kk in keys:
            pinned[kk].copy_(inp[kk])
        dev_in = [inp, {kk: torch.empty_like(inp[kk]) for kk in keys}]
        dev_out = [out, torch.empty_like(out)]
        out_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        h2d = sum(pinned[kk].numel() * pinned[kk].element_size() for kk in keys)
        d2h = out_host[0].numel() * out_host[0].element_size()
        n_e2e = max(4, min(args.steps, 8))
        s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in_ready", "in_free", "out_ready", "out_free")}
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_up.wait_event(a)
        s_down.wait_event(a)
        for i in range(n_e2e):
            j = i % 2
            if i >= 2:
                s_up.wait_event(ev["in_free"][j])          # step i - 2 has consumed this input set
            with torch.cuda.stream(s_up):
                for kk in keys:
                    dev_in[j][kk].copy_(pinned[kk], non_blocking=True)
                ev["in_ready"][j].record(s_up)
            stream.wait_event(ev["in_ready"][j])
            if i >= 2:
                stream.wait_event(ev["out_free"][j])        # step i - 2's output has been downloaded
            step(x=dev_in[j], o=dev_out[j])
            ev["in_free"][j].record(stream)
            ev["out_ready"][j].record(stream)
            s_down.wait_event(ev["out_ready"][j])
            with torch.cuda.stream(s_down):
                out_host[j].copy_(dev_out[j], non_blocking=True)
                ev["out_free"][j].record(s_down)
        for j in range(2):
            stream.wait_event(ev["out_free"][j])
        b.record(stream)
        barrier()
        e2e_ms = replicas.max_over_ranks(a.elapsed_time(b) / n_e2e, device=dev)
        e2e = {"value": replicas.job_rate(fl_total, world, e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e, "pipelined": "uploads / compute / downloads of consecutive steps overlap"}
        del dev_in, dev_out

    # ---- roofline of the dominant call.  The timed region lasts a fraction of
    # a second at the maximum SM clock, so the BF16 denominator is the measured
    # burst figure; the FP8 one is measured in this run (fp8_peak_tflops).
    hbm, bf16_burst, bf16_sus, src = _peaks()
    fp8_peak = fp8_peak_tflops(torch, dev)
    algo = {"fused_attention": (fl_sparse + fl_window, "tensor", bf16_burst, f"{src} bf16 burst"),
            "index_topk": (fl_index, "tensor", fp8_peak,
                           "e4m3 GEMM measured in this run (torch._scaled_mm 8192^3, best of 10)")}
    dom = max(per, key=per.get)
    if dom in algo and algo[dom][2]:
        fl, bound, peak, psrc = algo[dom]
        ach = fl / (per[dom] * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": bound, "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak,
                "traffic": PROFILED_TRAFFIC.get(dom) if args.S is None else None,
                "peak_source": psrc}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": hbm, "unit": "GB/s", "frac": None,
                "traffic": None}
    idx_ach = fl_index / (per["index_topk"] * 1e-3) / 1e12
    indexer_roof = {"kernel": "index_topk", "bound": "tensor", "achieved": idx_ach, "peak": fp8_peak,
                    "unit": "TFLOP/s", "frac": idx_ach / fp8_peak if fp8_peak else None,
                    "peak_source": algo["index_topk"][3]}

    decode = decode_fp4 = None
    if not args.no_decode and args.S is None:
        decode = decode_leg(dev, args.steps, args.warmup, csa, synth, torch, batch=args.decode_batch,
                            seed=replicas.replica_seed(rank, base=1),
                            cpu_baseline=rank == 0 and world == 1 and not args.no_cpu_baseline)
        if args.decode_batch is None:
            decode_fp4 = decode_fp4_leg(dev, args.steps, args.warmup, csa, synth, torch,
                                        seed=replicas.replica_seed(rank, base=1))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_inputs(inp)
        rows = oracle_rows(S)
        fl, dt, cores = cpu_oracle_sample(host, cfg, rows)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{len(rows)} evenly spaced query rows of the same S={S} layer (float64 numpy oracle, "
                         f"{dt:.1f} s including its full-sequence compressor and window-row passes; the "
                         f"reference arm times the same sample per step)"}

    hca = mixed = proj = tiny = None
    if args.S is None:
        del inp, qn, kt, kv, idx, ws, out
        torch.cuda.empty_cache()
        if not args.no_hca:
            hca = hca_prefill_leg(dev, args.steps, args.warmup, csa, synth, torch, seed=replicas.replica_seed(rank))
            torch.cuda.empty_cache()
        if not args.no_mixed:
            mixed = mixed_decode_leg(dev, args.steps, args.warmup, csa, synth, torch, seed=replicas.replica_seed(rank))
            torch.cuda.empty_cache()
        if not args.no_out_proj:
            proj = out_proj_leg(dev, args.steps, args.warmup, csa, synth, torch, seed=replicas.replica_seed(rank))
            torch.cuda.empty_cache()
        if not args.no_tiny:
            tiny = tiny_leg(dev, args.steps, args.warmup, csa, synth, torch)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": WORKLOAD if args.S is None else f"{WORKLOAD}_S{S}", "S": S, "H": H, "D": D, "m": m, "entries": ne, "top_k": k,
                           "window": W, "indexer": f"e4m3 {HI}x{DI}", "batch_per_gpu": 1,
                           "parallelism": f"replicas x{world}",
                           "l2": "inputs larger than L2 (q alone is 1 GiB)",
                           "streams": "query RMSNorm/RoPE on a second stream beside the key side; kernels_ms of "
                                      "concurrent calls overlap",
                           "flops_per_step": {"sparse_mqa": fl_sparse, "swa_window": fl_window,
                                              "indexer_fp8": fl_index}},
                "prefill_tokens_per_s": replicas.job_rate(S, world, ms * 1e-3),
                "kernels_ms": per, "roofline": roof, "indexer_roofline": indexer_roof, "cpu_baseline": cpu, "e2e": e2e, "decode_1m": decode, "decode_1m_fp4": decode_fp4,
                "hca_prefill": hca, "decode_mixed": mixed, "out_proj": proj, "tiny_csa": tiny,
                "gpu_launches": launches_per_step * args.steps, "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
