"""Seeded synthetic inputs with the shapes and value distributions of the
CSA / HCA workloads.  This module only draws random numbers and converts them
to the storage formats (bf16, e4m3 codes); it holds none of the layer's
arithmetic, so both the CUDA path and the float64 oracle can consume it.

Workloads (names used across tests and the benchmark):
  tiny_csa      single CSA layer, S 2048, 8 heads x 128, fp32, m 4, indexer 4 x 32,
                top-k 64, window 128, sink 0, indexer values on the 1/8 grid.
  csa_prefill   S 16384, 64 heads x 512 bf16, QK RMSNorm + RoPE(64), m 4 with
                overlap (4096 entries), e4m3 indexer 64 x 128, top-k 512.
  hca_prefill   S 131072, 64 x 512 bf16, m' 128 (1024 entries), window 128.
  csa_decode_1m batch 16, context 2^20, caches: e4m3 KV [2^18, 448] + bf16 RoPE
                [2^18, 64] + fp32 row scale; e4m3 indexer keys [2^18, 128] + scale.
  mixed_decode  batch 32, context U[64K, 1M], layers CSA, HCA, CSA, HCA, top-k 1024.
  out_proj      grouped output projection of a prefill layer's attention output:
                S 16384 tokens, 64 heads x 512 in 8 groups -> 8 x 1024 -> 4096.
"""
from __future__ import annotations

import numpy as np
import torch

WORKLOADS = {
    "tiny_csa": dict(S=2048, H=8, D=128, m=4, HI=4, DI=32, k=64, W=128, dtype="f32",
                     norm_rope=False, inv_rope=False, sink="zero"),
    "csa_prefill": dict(S=16384, H=64, D=512, m=4, HI=64, DI=128, k=512, W=128, dtype="bf16",
                        norm_rope=True, inv_rope=True, sink="normal"),
    "hca_prefill": dict(S=131072, H=64, D=512, m=128, W=128, dtype="bf16",
                        norm_rope=True, inv_rope=True, sink="normal"),
    "csa_decode_1m": dict(batch=16, ctx=1 << 20, H=64, D=512, m=4, HI=64, DI=128, k=512, W=128,
                          rope_dim=64),
    "out_proj": dict(S=16384, H=64, D=512, G=8, d_mid=1024, d_model=4096),
    "mixed_decode": dict(batch=32, ctx_lo=65536, ctx_hi=1 << 20, H=64, D=512, HI=64, DI=128,
                         k=1024, W=128, rope_dim=64, layers=("csa", "hca", "csa", "hca")),
}


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """float32 array holding the nearest bf16 values (storage format conversion)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.to(torch.float32).numpy()


def to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """uint8 E4M3 codes of x (storage format conversion, round to nearest)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def grid_codes(rng, shape, step=0.125):
    """N(0,1) rounded to a multiple of `step`, then to E4M3.  With step 1/8
    every resulting value is a multiple of 1/8, so products and sums of them
    stay exact in fp32 while their magnitude is below 2^13."""
    return to_e4m3_codes(np.round(rng.standard_normal(shape) / step) * step)


def prefill_inputs(name: str, S: int | None = None, seed: int = 0, grid: bool | None = None):
    """Inputs of one prefill layer.  S overrides the sequence length (tests).

    Returns a dict of numpy arrays:
      q [S,H,D], C [S,D], Z [S,D], B [2m or m, D] (float32, bf16-valued for bf16
      workloads), sink [H] float32, and for CSA: qI_codes [S,HI,DI] uint8,
      kI_codes [n_e,DI] uint8, w [S,HI] float32.
    grid: indexer values on the 1/8 grid and w on the 1/16 grid (default for
    tiny_csa; bit-exact top-k runs use it everywhere).
    """
    cfg = dict(WORKLOADS[name])
    S = cfg["S"] if S is None else S
    rng = np.random.default_rng(seed)
    H, D, m = cfg["H"], cfg["D"], cfg["m"]
    csa = "HI" in cfg
    nb = 2 * m if csa else m
    out = {}
    out["C"] = rng.standard_normal((S, D)).astype(np.float32)
    out["Z"] = rng.standard_normal((S, D)).astype(np.float32)
    out["B"] = (0.1 * rng.standard_normal((nb, D))).astype(np.float32)
    out["q"] = rng.standard_normal((S, H, D)).astype(np.float32)
    if cfg["sink"] == "zero":
        out["sink"] = np.zeros(H, np.float32)
    else:
        out["sink"] = rng.standard_normal(H).astype(np.float32)
    if cfg["dtype"] == "bf16":
        for key in ("C", "Z", "B", "q"):
            out[key] = to_bf16_values(out[key])
    if csa:
        grid = (name == "tiny_csa") if grid is None else grid
        HI, DI, ne = cfg["HI"], cfg["DI"], S // m
        if grid:
            out["qI_codes"] = grid_codes(rng, (S, HI, DI))
            out["kI_codes"] = grid_codes(rng, (ne, DI))
            out["w"] = (np.floor(rng.random((S, HI)) * 16.0) / 16.0).astype(np.float32)
        else:
            out["qI_codes"] = to_e4m3_codes(rng.standard_normal((S, HI, DI)))
            out["kI_codes"] = to_e4m3_codes(rng.standard_normal((ne, DI)))
            out["w"] = rng.random((S, HI)).astype(np.float32)
    return out, dict(cfg, S=S)


def decode_lengths(name: str, seed: int = 0):
    """Per-sequence context lengths of a decode workload (int64 [batch])."""
    cfg = WORKLOADS[name]
    if "ctx" in cfg:
        return np.full(cfg["batch"], cfg["ctx"], dtype=np.int64)
    rng = np.random.default_rng(seed)
    return rng.integers(cfg["ctx_lo"], cfg["ctx_hi"] + 1, size=cfg["batch"]).astype(np.int64)


def decode_csa_cache(n_e: int, D: int, DI: int, rope_dim: int, gen: torch.Generator,
                     device, grid: bool = False):
    """One sequence's CSA caches on `device` (drawn with torch's seeded generator):
      kv_nope [n_e, D-rope] e4m3 codes, kv_rope [n_e, rope] bf16, kv_scale [n_e] fp32,
      kI [n_e, DI] e4m3 codes, kI_scale [n_e] fp32.
    Row scales are powers of two (2^-2 .. 2^2) and the codes hold N(0,1)/scale,
    so dequantised values are ~N(0,1).  grid=True puts the indexer keys on the
    1/8 grid with unit scales, for bit-exact selection runs."""
    nope = D - rope_dim
    sc = torch.pow(2.0, torch.randint(-2, 3, (n_e,), generator=gen, device=device).float())
    x = torch.randn(n_e, nope, generator=gen, device=device) / sc[:, None]
    kv_nope = x.to(torch.float8_e4m3fn).view(torch.uint8)
    kv_rope = torch.randn(n_e, rope_dim, generator=gen, device=device).to(torch.bfloat16)
    ks = torch.pow(2.0, torch.randint(-2, 3, (n_e,), generator=gen, device=device).float())
    y = torch.randn(n_e, DI, generator=gen, device=device)
    if grid:
        y = torch.round(y * 8.0) / 8.0
        ks = torch.ones_like(ks)
    else:
        y = y / ks[:, None]
    kI = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return dict(kv_nope=kv_nope, kv_rope=kv_rope, kv_scale=sc, kI=kI, kI_scale=ks)


def decode_query(H: int, D: int, HI: int, DI: int, W: int, gen: torch.Generator, device,
                 grid: bool = False):
    """One sequence's decode-step query side: q [H,D] bf16, qI [HI,DI] e4m3 codes,
    qI_scale [HI] fp32 (powers of two), w [HI] fp32, swa [W,D] bf16, sink [H] fp32."""
    q = torch.randn(H, D, generator=gen, device=device).to(torch.bfloat16)
    qs = torch.pow(2.0, torch.randint(-2, 3, (HI,), generator=gen, device=device).float())
    y = torch.randn(HI, DI, generator=gen, device=device)
    if grid:
        y = torch.round(y * 8.0) / 8.0
        qs = torch.ones_like(qs)
        w = torch.floor(torch.rand(HI, generator=gen, device=device) * 16.0) / 16.0
    else:
        y = y / qs[:, None]
        w = torch.rand(HI, generator=gen, device=device)
    qI = y.to(torch.float8_e4m3fn).view(torch.uint8)
    swa = torch.randn(W, D, generator=gen, device=device).to(torch.bfloat16)
    sink = torch.randn(H, generator=gen, device=device)
    return dict(q=q, qI=qI, qI_scale=qs, w=w, swa=swa, sink=sink)


def prefill_inputs_device(name: str, device, seed: int = 0, S: int | None = None, grid: bool = False):
    """The same recipe as prefill_inputs, drawn on `device` with torch's seeded
    generator (for benchmark-sized inputs).  Returns torch tensors: q [S,H,D],
    C, Z [S,D] in the workload dtype, B [2m or m, D] f32, sink [H] f32 and, for
    CSA, qI_codes [S,HI,DI] u8, kI_codes [n_e,DI] u8, w [S,HI] f32."""
    cfg = dict(WORKLOADS[name])
    S = cfg["S"] if S is None else S
    g = torch.Generator(device=device).manual_seed(seed)
    H, D, m = cfg["H"], cfg["D"], cfg["m"]
    dt = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
    csa = "HI" in cfg
    out = {
        "C": torch.randn(S, D, generator=g, device=device).to(dt),
        "Z": torch.randn(S, D, generator=g, device=device).to(dt),
        "B": (0.1 * torch.randn(2 * m if csa else m, D, generator=g, device=device)).to(dt).float(),
        "q": torch.randn(S, H, D, generator=g, device=device).to(dt),
        "sink": (torch.zeros(H, device=device) if cfg["sink"] == "zero"
                 else torch.randn(H, generator=g, device=device)),
    }
    if csa:
        HI, DI, ne = cfg["HI"], cfg["DI"], S // m
        qI = torch.randn(S, HI, DI, generator=g, device=device)
        kI = torch.randn(ne, DI, generator=g, device=device)
        if grid:
            qI, kI = torch.round(qI * 8) / 8, torch.round(kI * 8) / 8
            w = torch.floor(torch.rand(S, HI, generator=g, device=device) * 16) / 16
        else:
            w = torch.rand(S, HI, generator=g, device=device)
        out["qI_codes"] = qI.to(torch.float8_e4m3fn).view(torch.uint8)
        out["kI_codes"] = kI.to(torch.float8_e4m3fn).view(torch.uint8)
        out["w"] = w.contiguous()
    return out, dict(cfg, S=S)


def _decode_layer(g, B, ne, H, D, HI, DI, W, r, grid, indexer):
    """One layer's batched decode caches and query side, drawn from generator g.
    Row scales are powers of two 2^U{-2..2} and codes hold N(0,1)/scale."""
    device = g.device

    def pow2(*shape):
        return torch.pow(2.0, torch.randint(-2, 3, shape, generator=g, device=device).float())

    out = {}
    sc = pow2(B, ne)
    out["kv_nope"] = (torch.randn(B, ne, D - r, generator=g, device=device) / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
    out["kv_rope"] = torch.randn(B, ne, r, generator=g, device=device).to(torch.bfloat16)
    out["kv_scale"] = sc
    if indexer:
        ks = pow2(B, ne)
        y = torch.randn(B, ne, DI, generator=g, device=device)
        qs = pow2(B, 1, HI)
        x = torch.randn(B, 1, HI, DI, generator=g, device=device)
        if grid:
            y, x = torch.round(y * 8) / 8, torch.round(x * 8) / 8
            ks, qs = torch.ones_like(ks), torch.ones_like(qs)
            w = torch.floor(torch.rand(B, 1, HI, generator=g, device=device) * 16) / 16
        else:
            y, x = y / ks[..., None], x / qs[..., None]
            w = torch.rand(B, 1, HI, generator=g, device=device)
        out["kI"] = y.to(torch.float8_e4m3fn).view(torch.uint8)
        out["kI_scale"] = ks
        out["qI"] = x.to(torch.float8_e4m3fn).view(torch.uint8)
        out["qI_scale"] = qs
        out["w"] = w.contiguous()
    out["q"] = torch.randn(B, 1, H, D, generator=g, device=device).to(torch.bfloat16)
    out["swa"] = torch.randn(B, W, D, generator=g, device=device).to(torch.bfloat16)
    out["sink"] = torch.randn(H, generator=g, device=device)
    return out


def decode_inputs_device(name: str, device, seed: int = 0, grid: bool = False, batch: int | None = None,
                         ctx: int | None = None):
    """Batched decode-step inputs for `csa_decode_1m` on `device` (torch's seeded
    generator), stacked over the batch:
      kv_nope [B, n_e, D-64] e4m3, kv_rope [B, n_e, 64] bf16, kv_scale [B, n_e] f32,
      kI [B, n_e, DI] e4m3, kI_scale [B, n_e] f32 (row scales 2^U{-2..2}, codes N(0,1)/scale),
      q [B, 1, H, D] bf16, qI [B, 1, HI, DI] e4m3, qI_scale [B, 1, HI], w [B, 1, HI] f32,
      swa [B, W, D] bf16, sink [H] f32, q_pos [B] int64 (= context - 1).
    grid=True puts the indexer values on the 1/8 grid (w on 1/16) with unit scales."""
    cfg = dict(WORKLOADS[name])
    B = cfg["batch"] if batch is None else batch
    L = cfg["ctx"] if ctx is None else ctx
    H, D, HI, DI, W, r = cfg["H"], cfg["D"], cfg["HI"], cfg["DI"], cfg["W"], cfg["rope_dim"]
    m = cfg["m"]
    ne = L // m
    g = torch.Generator(device=device).manual_seed(seed)
    out = _decode_layer(g, B, ne, H, D, HI, DI, W, r, grid, True)
    out["q_pos"] = torch.full((B,), L - 1, dtype=torch.int64, device=device)
    return out, dict(cfg, batch=B, ctx=L, n_e=ne)


def mixed_decode_inputs_device(device, seed: int = 0, grid: bool = False, batch: int | None = None,
                               lengths=None):
    """Inputs of one decode step of the 4-layer stack `mixed_decode` (CSA, HCA,
    CSA, HCA), each layer with its own independently drawn caches and query:
    per-sequence contexts L_b (decode_lengths, or `lengths`), caches padded to
    the longest sequence (CSA: max L / 4 entries, HCA: max L / 128), new token
    at position L_b - 1.  Returns (layers, q_pos [B] int64, cfg); each layer is a
    dict like decode_inputs_device's plus "kind" and "m"."""
    cfg = dict(WORKLOADS["mixed_decode"])
    L = decode_lengths("mixed_decode", seed) if lengths is None else np.asarray(lengths, np.int64)
    if batch is not None:
        L = L[:batch]
    B = len(L)
    H, D, HI, DI, W, r = cfg["H"], cfg["D"], cfg["HI"], cfg["DI"], cfg["W"], cfg["rope_dim"]
    g = torch.Generator(device=device).manual_seed(seed)
    layers = []
    for kind in cfg["layers"]:
        m = 4 if kind == "csa" else 128
        lay = _decode_layer(g, B, int(L.max()) // m, H, D, HI, DI, W, r, grid, kind == "csa")
        lay["kind"], lay["m"] = kind, m
        layers.append(lay)
    q_pos = torch.as_tensor(L - 1, dtype=torch.int64).to(device)
    return layers, q_pos, dict(cfg, batch=B, lengths=L)


def out_proj_inputs_device(device, seed: int = 0, S: int | None = None, H: int | None = None,
                           D: int | None = None, G: int | None = None, d_mid: int | None = None,
                           d_model: int | None = None):
    """Inputs of the grouped output projection, drawn on `device`: an attention
    output o [S, H, D] bf16 ~ N(0, 1/4) (the scale of a softmax-weighted mix of
    unit rows) and random-init weights w_grp [G, d_mid, (H/G)*D], w_out
    [d_model, G*d_mid], bf16 ~ N(0, 1/fan_in) (no trained weights exist here)."""
    cfg = dict(WORKLOADS["out_proj"])
    for k, v in (("S", S), ("H", H), ("D", D), ("G", G), ("d_mid", d_mid), ("d_model", d_model)):
        if v is not None:
            cfg[k] = v
    g = torch.Generator(device=device).manual_seed(seed)
    S, H, D, G, dm, dmod = cfg["S"], cfg["H"], cfg["D"], cfg["G"], cfg["d_mid"], cfg["d_model"]
    d_in = (H // G) * D
    o = (0.5 * torch.randn(S, H, D, generator=g, device=device)).to(torch.bfloat16)
    w_grp = (torch.randn(G, dm, d_in, generator=g, device=device) / d_in ** 0.5).to(torch.bfloat16)
    w_out = (torch.randn(dmod, G * dm, generator=g, device=device) / (G * dm) ** 0.5).to(torch.bfloat16)
    return dict(o=o, w_grp=w_grp, w_out=w_out), cfg
