"""Float64 reference ("oracle") for the CSA / HCA hybrid attention forward pass.

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the library.  It is the
plain, slow definition of each step, in numpy float64, with no blocking, fusion
or reordering beyond what the definition states.

Sources (web write-ups of the DeepSeek-V4 technical report):
  [LQ]  "Deepseek-V4 技术报告里最值得复现的三个改动" (m.lqnn.cn), §3 config
        block (m=4, top-k 512, m'=128, 64 heads x 512, window 128, indexer
        64 x 128) and §5 (tail tokens are dropped).
  [YH]  "DeepSeek V4 技术深度：1.6T 参数 + 32T tokens + CSA/HCA + mHC + Muon",
        "5 大架构 / 1. CSA + HCA 混合注意力" (4 -> 1 sparse, 128 -> 1 dense).
  [LD]  liduos.com "deepseek-v4-engineering-tradeoffs", section
        "1M Context 的结构与取舍" (HCA / CSA / SWA channels, top-k, 128-token
        raw window, attention sink, partial RoPE with inverse RoPE on output).
  [CS]  "DeepSeek V4 脱离 CUDA 全栈国产化：1.6T MoE 逐层拆解 + 昇腾迁移数据",
        §二 "CSA + HCA 混合注意力": "KV 压缩" (compressor formula),
        "闪电索引器" (indexer), "共享 KV MQA", "HCA（重压缩注意力）",
        "其他辅助设计" (QK RMSNorm, partial RoPE on the last 64 dims, BF16 RoPE
        dims / FP8 rest).

Readings taken where the pages are silent or garbled (each is a keyword
argument whose default is the reading):
  * compressor: one joint per-channel softmax over the previous and the current
    block (2m logits) [CS "KV 压缩"]; the first entry has no previous block;
    bias rows 0..m-1 weight the previous block, rows m..2m-1 the current one;
  * tail tokens that do not fill a block form no entry [LQ §5];
  * entry i is visible to query t iff its block is complete: (i+1)*m - 1 <= t;
  * indexer: I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s]) with no extra scale
    [CS "闪电索引器"]; FP8 operands are dequantised by their row scales;
  * top-k: largest scores, ties to the lower entry index, min(k, n_vis) kept,
    returned in ascending index order and padded with -1;
  * attention: softmax scale 1/sqrt(D); selected entries, window tokens and the
    sink share one softmax; the sink adds exp(s_h) to the denominator and has
    a zero value [LD "Attention Sink"];
  * window = raw tokens [max(0, t-W+1), t], W = 128 [LD "SWA"];
  * RMSNorm over all D dims, eps 1e-6, unit gain [CS "其他辅助设计"];
  * partial RoPE on dims [D-64, D), pairs (d, d+32), theta_j = 10000^(-2j/64);
    positions: query t, CSA/HCA entry i -> i*m, window token u -> u;
  * inverse RoPE (rotation by -t) on the last 64 dims of the output [LD];
  * the first layers of the stack are window-only: window + sink, no
    compressed branch [LQ §3, note after the config block];
  * grouped output projection [LQ §3 config: output_proj_groups 8,
    intermediate_attn_dim 1024, hidden_size 4096]: consecutive heads form a
    group, each group has its own [d_mid, (H/G)*D] matrix, the concatenated
    group outputs go through one [d_model, G*d_mid] matrix, no bias; the
    intermediate is stored as bf16 like every other activation of the layer;
  * FP4 indexer operands [CS "闪电索引器"]: OCP MX FP4 (E2M1 elements, blocks of
    32 sharing an E8M0 power-of-two scale), two elements per byte.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "e4m3_decode", "e4m3_encode", "bf16_round",
    "n_entries", "n_visible",
    "compress", "rmsnorm", "rope_partial",
    "indexer_scores", "topk_select",
    "attend_rows", "sparse_attention_partial", "dense_attention_partial",
    "window_sink_combine", "merge_partials",
    "csa_layer", "hca_layer", "csa_layer_matrix", "hca_layer_matrix",
    "csa_decode", "hca_decode", "flop_counts",
    "fp8_row_quantize", "stream_append",
    "swa_layer", "grouped_out_proj",
    "e2m1_decode", "e2m1_encode", "e8m0_decode", "fp4_pack", "fp4_unpack",
    "mxfp4_quantize", "mxfp4_dequantize",
]

# ----------------------------------------------------------------------------
# Number formats.  OCP 8-bit floating point, E4M3 ("fn" variant): 1 sign bit,
# 4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is
# NaN, largest finite magnitude 448.  Stated in [LD] (FP8 caches) and [CS
# "其他辅助设计"] (non-RoPE dims in FP8); the bit layout is the OCP definition.
# ----------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Exact float64 value of each E4M3 byte."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    mant = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, mant / 8.0 * 2.0 ** (1 - 7),
                   (1.0 + mant / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, val)
    return sign * val


_E4M3_POS = None


def _e4m3_table():
    global _E4M3_POS
    if _E4M3_POS is None:
        _E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # codes 0..126, ascending
    return _E4M3_POS


def e4m3_encode(x) -> np.ndarray:
    """Round-to-nearest-even to E4M3, saturating at +-448 (NaN is not produced)."""
    x = np.asarray(x, dtype=np.float64)
    tab = _e4m3_table()
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(tab, a, side="left"), 0, len(tab) - 1)
    lo = np.clip(hi - 1, 0, len(tab) - 1)
    dlo = a - tab[lo]
    dhi = tab[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a == tab[hi], hi, code).astype(np.uint8)
    neg = (x < 0) & (code != 0)
    return np.where(neg, code | 0x80, code).astype(np.uint8)


# ----------------------------------------------------------------------------
# FP4 for the lightning indexer's QK path ([CS] "闪电索引器": the QK path runs in
# FP4; "其他辅助设计": the indexer is stored in FP4).  The pages name no block
# format; the reading taken is the OCP Microscaling (MX) FP4 format: E2M1
# elements (1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit, subnormal
# at exponent 0, no infinities or NaN, largest magnitude 6) in blocks of 32
# consecutive elements sharing one E8M0 scale (an unsigned power of two
# 2^(byte - 127), byte 0xFF = NaN).  Storage: two elements per byte, the even
# element in the low nibble.
# ----------------------------------------------------------------------------

def e2m1_decode(codes) -> np.ndarray:
    """Exact value of each 4-bit E2M1 code (0..15)."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 0x1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e.astype(np.float64) - 1.0))
    return sign * mag


_E2M1_POS = None


def _e2m1_table():
    global _E2M1_POS
    if _E2M1_POS is None:
        _E2M1_POS = e2m1_decode(np.arange(8))          # 0, 0.5, 1, 1.5, 2, 3, 4, 6
    return _E2M1_POS


def e2m1_encode(x) -> np.ndarray:
    """Round to the nearest E2M1 value, ties to the even code (mantissa bit 0),
    saturating at +-6; returns codes 0..15 (no negative zero)."""
    x = np.asarray(x, dtype=np.float64)
    tab = _e2m1_table()
    a = np.minimum(np.abs(x), 6.0)
    hi = np.clip(np.searchsorted(tab, a, side="left"), 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    dlo = a - tab[lo]
    dhi = tab[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a == tab[hi], hi, code)
    neg = (x < 0) & (code != 0)
    return np.where(neg, code | 0x8, code).astype(np.uint8)


def e8m0_decode(b) -> np.ndarray:
    """Value of each E8M0 scale byte: 2^(b - 127); 0xFF is NaN."""
    b = np.asarray(b).astype(np.int64)
    return np.where(b == 0xFF, np.nan, np.exp2((b - 127).astype(np.float64)))


def fp4_pack(codes) -> np.ndarray:
    """[..., 2n] codes 0..15 -> [..., n] bytes, element 2j in the low nibble."""
    c = np.asarray(codes).astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def fp4_unpack(packed) -> np.ndarray:
    """Inverse of fp4_pack: [..., n] bytes -> [..., 2n] codes."""
    p = np.asarray(packed).astype(np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def mxfp4_quantize(x, block: int = 32):
    """MX FP4 quantisation of the last axis: for each block of `block`
    elements the shared scale is 2^(floor(log2(amax)) - 2) (2 = the largest
    E2M1 exponent), clamped to the E8M0 range, and each element is
    e2m1_encode(v / scale) (saturating).  An all-zero block gets scale 2^-127.
    Returns (codes [..., n] 0..15, scale bytes [..., n / block])."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    if n % block:
        raise ValueError("the last axis must be a multiple of the block size")
    xb = x.reshape(x.shape[:-1] + (n // block, block))
    amax = np.abs(xb).max(axis=-1)
    with np.errstate(divide="ignore"):
        e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2.0, -127.0)
    e = np.clip(e, -127.0, 127.0)
    codes = e2m1_encode(xb / np.exp2(e)[..., None]).reshape(x.shape)
    return codes, (e + 127.0).astype(np.uint8)


def mxfp4_dequantize(codes, scales, block: int = 32) -> np.ndarray:
    """Values of MX FP4 data: e2m1_decode(code) * e8m0_decode(block scale)."""
    v = e2m1_decode(codes)
    s = np.repeat(e8m0_decode(scales), block, axis=-1)
    return v * s


def bf16_round(x) -> np.ndarray:
    """Round float64 to the nearest bfloat16 value (8 significant bits, ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


# ----------------------------------------------------------------------------
# Entry counting and causal visibility.
# ----------------------------------------------------------------------------

def n_entries(S: int, m: int) -> int:
    """Compressed entries of a length-S sequence: one per complete block of m
    tokens; a tail shorter than m forms none ([LQ §5], [YH 1.], [CS "KV 压缩"])."""
    return S // m


def n_visible(t, m: int):
    """Entries visible to query position t: those whose block ends at or before t."""
    return (np.asarray(t) + 1) // m


# ----------------------------------------------------------------------------
# (a1, a2) KV compressor  [CS §二 "KV 压缩"; "HCA（重压缩注意力）"].
# ----------------------------------------------------------------------------

def compress(C, Z, B, m: int, overlap: bool, Cb=None, Zb=None, joint_softmax: bool = True):
    """Softmax-gated pooling of m-token blocks, per channel.

    C, Z: [S, D] content and gate logits; B: [2m, D] (overlap) or [m, D] bias.
    Overlapping (CSA): entry i pools positions [(i-1)m, (i+1)m): the previous
    block with bias rows 0..m-1 (stream b: Cb, Zb, default C, Z) and the current
    block with bias rows m..2m-1 (stream a: C, Z).  Entry 0 has only its own
    block.  Non-overlapping (HCA): entry i pools block i with bias rows 0..m-1.
    joint_softmax=False takes the other reading of the garbled formula: the two
    blocks are normalised separately and summed.
    Returns KV [S // m, D] float64.
    """
    C = np.asarray(C, np.float64); Z = np.asarray(Z, np.float64); B = np.asarray(B, np.float64)
    Cb = C if Cb is None else np.asarray(Cb, np.float64)
    Zb = Z if Zb is None else np.asarray(Zb, np.float64)
    S, D = C.shape
    ne = n_entries(S, m)
    out = np.zeros((ne, D))
    for i in range(ne):
        cur = slice(i * m, (i + 1) * m)
        if not overlap:
            logit = Z[cur] + B[:m]
            p = np.exp(logit - logit.max(axis=0))
            p /= p.sum(axis=0)
            out[i] = (p * C[cur]).sum(axis=0)
            continue
        la = Z[cur] + B[m:2 * m]
        if i == 0:
            p = np.exp(la - la.max(axis=0)); p /= p.sum(axis=0)
            out[i] = (p * C[cur]).sum(axis=0)
            continue
        prev = slice((i - 1) * m, i * m)
        lb = Zb[prev] + B[:m]
        if joint_softmax:
            mx = np.maximum(la.max(axis=0), lb.max(axis=0))
            pa = np.exp(la - mx); pb = np.exp(lb - mx)
            den = pa.sum(axis=0) + pb.sum(axis=0)
            out[i] = ((pa * C[cur]).sum(axis=0) + (pb * Cb[prev]).sum(axis=0)) / den
        else:
            pa = np.exp(la - la.max(axis=0)); pa /= pa.sum(axis=0)
            pb = np.exp(lb - lb.max(axis=0)); pb /= pb.sum(axis=0)
            out[i] = (pa * C[cur]).sum(axis=0) + (pb * Cb[prev]).sum(axis=0)
    return out


# ----------------------------------------------------------------------------
# QK normalisation and partial RoPE  [CS "其他辅助设计"; LD].
# ----------------------------------------------------------------------------

def rmsnorm(x, eps: float = 1e-6):
    """x / sqrt(mean(x^2) + eps) over the last axis (unit gain)."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)


def rope_partial(x, pos, rope_dim: int = 64, base: float = 10000.0, inverse: bool = False):
    """Rotate the last rope_dim dims of x by position pos (half-split pairs).

    x: [..., D]; pos broadcastable to x.shape[:-1].  Pair j (< rope_dim/2) is
    (x[D-r+j], x[D-r+j+r/2]) rotated by angle pos * base^(-2j/r).
    """
    x = np.array(x, np.float64, copy=True)
    D = x.shape[-1]
    h = rope_dim // 2
    j = np.arange(h, dtype=np.float64)
    inv_freq = base ** (-2.0 * j / rope_dim)
    ang = np.asarray(pos, np.float64)[..., None] * inv_freq
    if inverse:
        ang = -ang
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., D - rope_dim:D - h].copy()
    b = x[..., D - h:].copy()
    x[..., D - rope_dim:D - h] = a * c - b * s
    x[..., D - h:] = a * s + b * c
    return x


# ----------------------------------------------------------------------------
# (a3) Lightning indexer and (a4) top-k  [CS "闪电索引器"; LD "CSA"].
# ----------------------------------------------------------------------------

def indexer_scores(qI, w, kI, n_vis):
    """I[t, s] = sum_h w[t,h] * max(0, qI[t,h,:] . kI[s,:]) for s < n_vis[t].

    qI: [T, HI, DI] dequantised queries; w: [T, HI]; kI: [n_e, DI].
    Returns [T, n_e] float64 with -inf at invisible entries.
    """
    qI = np.asarray(qI, np.float64); w = np.asarray(w, np.float64); kI = np.asarray(kI, np.float64)
    n_vis = np.broadcast_to(np.asarray(n_vis), (qI.shape[0],))
    T, ne = qI.shape[0], kI.shape[0]
    out = np.full((T, ne), -np.inf)
    for t in range(T):
        nv = int(min(n_vis[t], ne))
        if nv <= 0:
            continue
        dots = qI[t] @ kI[:nv].T              # [HI, nv]
        out[t, :nv] = (w[t][:, None] * np.maximum(dots, 0.0)).sum(axis=0)
    return out


def topk_select(scores, n_vis, k: int):
    """Per row: the min(k, n_vis) visible entries with the largest score; equal
    scores go to the lower index.  Returned ascending, padded with -1: [T, k] int32."""
    scores = np.asarray(scores, np.float64)
    T = scores.shape[0]
    n_vis = np.broadcast_to(np.asarray(n_vis), (T,))
    out = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        nv = int(min(n_vis[t], scores.shape[1]))
        if nv <= 0:
            continue
        s = scores[t, :nv]
        order = np.lexsort((np.arange(nv), -s))   # primary -score, then index
        keep = np.sort(order[:min(k, nv)])
        out[t, :len(keep)] = keep
    return out


# ----------------------------------------------------------------------------
# (a5, a6) attention over a row set with K = V  [CS "共享 KV MQA", "HCA"].
# ----------------------------------------------------------------------------

def attend_rows(q, rows, scale):
    """One query position, H heads: logits l = scale * q @ rows.T, softmax over
    the rows, O = P @ rows (values are the same rows as keys).
    Returns (O [H, D] normalised, lse [H]); with no rows O = 0 and lse = -inf."""
    q = np.asarray(q, np.float64)
    if rows.shape[0] == 0:
        return np.zeros_like(q), np.full(q.shape[0], -np.inf)
    l = scale * (q @ rows.T)
    mx = l.max(axis=1, keepdims=True)
    p = np.exp(l - mx)
    den = p.sum(axis=1, keepdims=True)
    return (p @ rows) / den, (mx + np.log(den))[:, 0]


def sparse_attention_partial(q, kv, idx, scale=None):
    """CSA main branch: for each t, attend over kv[idx[t, j]] for idx >= 0.
    q: [T, H, D]; kv: [n_e, D]; idx: [T, k].  Returns (O [T,H,D], lse [T,H])."""
    q = np.asarray(q, np.float64); kv = np.asarray(kv, np.float64)
    T, H, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    O = np.zeros((T, H, D)); L = np.zeros((T, H))
    for t in range(T):
        sel = idx[t][idx[t] >= 0]
        O[t], L[t] = attend_rows(q[t], kv[sel], scale)
    return O, L


def dense_attention_partial(q, kv, n_vis, scale=None):
    """HCA main branch: for each t, attend over kv[0:n_vis[t]]."""
    q = np.asarray(q, np.float64); kv = np.asarray(kv, np.float64)
    T, H, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    n_vis = np.broadcast_to(np.asarray(n_vis), (T,))
    O = np.zeros((T, H, D)); L = np.zeros((T, H))
    for t in range(T):
        O[t], L[t] = attend_rows(q[t], kv[:int(min(n_vis[t], kv.shape[0]))], scale)
    return O, L


def merge_partials(parts, sink=None):
    """Joint softmax of several normalised partials (O_i, lse_i) plus an optional
    per-head sink logit with zero value: O = sum_i e^{lse_i - M} O_i /
    (sum_i e^{lse_i - M} + e^{s - M})."""
    lses = [np.asarray(l, np.float64) for _, l in parts]
    if sink is not None:
        lses_all = lses + [np.broadcast_to(np.asarray(sink, np.float64), lses[0].shape)]
    else:
        lses_all = lses
    M = np.max(np.stack(lses_all), axis=0)
    M = np.where(np.isfinite(M), M, 0.0)
    num = 0.0
    den = 0.0
    for (O, _), l in zip(parts, lses):
        wgt = np.exp(l - M)
        num = num + wgt[..., None] * np.asarray(O, np.float64)
        den = den + wgt
    if sink is not None:
        den = den + np.exp(np.broadcast_to(np.asarray(sink, np.float64), M.shape) - M)
    return num / den[..., None]


def window_sink_combine(q, kv_tok, positions, W, sink, O_part, lse_part, scale=None,
                        inv_rope: bool = False, rope_dim: int = 64, rope_base: float = 10000.0,
                        window_rows=None):
    """(a7) Attend over the raw window rows, merge with the compressed-branch
    partial and the sink in one softmax, then optionally un-rotate the output.

    Prefill: window of query t = kv_tok[max(0, t-W+1) : t+1].  Decode: pass
    window_rows[b] = the SWA cache rows (already the window, newest included).
    """
    q = np.asarray(q, np.float64)
    T, H, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    O = np.zeros((T, H, D))
    for i in range(T):
        if window_rows is not None:
            rows = np.asarray(window_rows[i], np.float64)
        else:
            t = int(positions[i])
            rows = np.asarray(kv_tok[max(0, t - W + 1):t + 1], np.float64)
        Ow, lw = attend_rows(q[i], rows, scale)
        O[i] = merge_partials([(O_part[i], lse_part[i]), (Ow, lw)], sink)
    if inv_rope:
        O = rope_partial(O, np.asarray(positions)[:, None], rope_dim, rope_base, inverse=True)
    return O


# ----------------------------------------------------------------------------
# Whole layers (prefill), gather formulation.
# ----------------------------------------------------------------------------

def _prep(q, C, pos_q, norm_rope, rope_dim, rope_base):
    if not norm_rope:
        return np.asarray(q, np.float64), np.asarray(C, np.float64)
    qn = rope_partial(rmsnorm(q), np.asarray(pos_q)[:, None], rope_dim, rope_base)
    kt = rope_partial(rmsnorm(C), np.arange(C.shape[0]), rope_dim, rope_base)
    return qn, kt


def _entries(C, Z, B, m, overlap, norm_rope, rope_dim, rope_base, store_round):
    kv = compress(C, Z, B, m, overlap)
    if norm_rope:
        kv = rope_partial(rmsnorm(kv), np.arange(kv.shape[0]) * m, rope_dim, rope_base)
    return store_round(kv) if store_round else kv


def csa_layer(q, C, Z, B, qI, w, kI, sink, *, k: int, m: int = 4, W: int = 128,
              norm_rope: bool = False, inv_rope: bool = False, rope_dim: int = 64,
              rope_base: float = 10000.0, store_round=None, rows=None, row_inputs: bool = False):
    """CSA layer forward for query rows `rows` (default all): compress (a1),
    indexer + top-k (a3, a4), sparse MQA (a5), window + sink (a7).
    store_round rounds tensors the method stores (entries, normalised q, window
    rows) to their storage type, e.g. bf16_round.  row_inputs: q, qI and w hold
    only the selected rows (in the order of `rows`).  Returns (O, idx)."""
    S = np.asarray(C).shape[0]
    rows = np.arange(S) if rows is None else np.asarray(rows)
    sel = slice(None) if row_inputs else rows
    qr = np.asarray(q)[sel].astype(np.float64)
    qn, kt = _prep(qr, C, rows, norm_rope, rope_dim, rope_base)
    if store_round:
        qn, kt = store_round(qn), store_round(kt)
    kv = _entries(C, Z, B, m, True, norm_rope, rope_dim, rope_base, store_round)
    nv = n_visible(rows, m)
    idx = topk_select(indexer_scores(np.asarray(qI)[sel].astype(np.float64), np.asarray(w)[sel], kI, nv), nv, k)
    Op, lp = sparse_attention_partial(qn, kv, idx)
    O = window_sink_combine(qn, kt, rows, W, sink, Op, lp, inv_rope=inv_rope,
                            rope_dim=rope_dim, rope_base=rope_base)
    return O, idx


def hca_layer(q, C, Z, B, sink, *, m: int = 128, W: int = 128, norm_rope: bool = False,
              inv_rope: bool = False, rope_dim: int = 64, rope_base: float = 10000.0,
              store_round=None, rows=None):
    """HCA layer forward: non-overlapping m'-compression (a2), dense causal
    attention over complete entries (a6), window + sink (a7)."""
    S = np.asarray(C).shape[0]
    rows = np.arange(S) if rows is None else np.asarray(rows)
    qr = np.asarray(q, np.float64)[rows]
    qn, kt = _prep(qr, C, rows, norm_rope, rope_dim, rope_base)
    if store_round:
        qn, kt = store_round(qn), store_round(kt)
    kv = _entries(C, Z, B, m, False, norm_rope, rope_dim, rope_base, store_round)
    Op, lp = dense_attention_partial(qn, kv, n_visible(rows, m))
    return window_sink_combine(qn, kt, rows, W, sink, Op, lp, inv_rope=inv_rope,
                               rope_dim=rope_dim, rope_base=rope_base)


# ----------------------------------------------------------------------------
# Second, independent formulation: one masked score matrix per query block over
# [all entries | all raw tokens | sink].  Used to cross-check the gather path.
# ----------------------------------------------------------------------------

def _matrix_attention(qn, keys, mask, sink):
    T, H, D = qn.shape
    scale = 1.0 / math.sqrt(D)
    logits = scale * np.einsum("thd,nd->thn", qn, keys)
    logits = np.where(mask[:, None, :], logits, -np.inf)
    s = np.broadcast_to(np.asarray(sink, np.float64), (H,))
    full = np.concatenate([logits, np.broadcast_to(s[None, :, None], (T, H, 1))], axis=2)
    mx = full.max(axis=2, keepdims=True)
    p = np.exp(full - mx)
    p /= p.sum(axis=2, keepdims=True)
    return np.einsum("thn,nd->thd", p[:, :, :-1], keys)


def csa_layer_matrix(q, C, Z, B, qI, w, kI, sink, *, k, m=4, W=128, norm_rope=False,
                     inv_rope=False, rope_dim=64, rope_base=10000.0, store_round=None, rows=None):
    """Same result as csa_layer, written as one masked softmax over the
    concatenation [entries; raw tokens] with a selection mask built from the
    full score matrix (argsort of the whole row, not the gather path)."""
    S = np.asarray(C).shape[0]
    rows = np.arange(S) if rows is None else np.asarray(rows)
    qr = np.asarray(q, np.float64)[rows]
    qn, kt = _prep(qr, C, rows, norm_rope, rope_dim, rope_base)
    if store_round:
        qn, kt = store_round(qn), store_round(kt)
    kv = _entries(C, Z, B, m, True, norm_rope, rope_dim, rope_base, store_round)
    ne = kv.shape[0]
    qI = np.asarray(qI, np.float64)[rows]; w = np.asarray(w, np.float64)[rows]
    dots = np.einsum("thd,nd->thn", qI, np.asarray(kI, np.float64))
    I = np.einsum("th,thn->tn", w, np.maximum(dots, 0.0))
    vis = np.arange(ne)[None, :] < n_visible(rows, m)[:, None]
    I = np.where(vis, I, -np.inf)
    # rank of each entry under (-score, index); selected iff rank < k and visible
    order = np.argsort(-I, axis=1, kind="stable")
    rank = np.empty_like(order)
    np.put_along_axis(rank, order, np.arange(ne)[None, :].repeat(len(rows), 0), axis=1)
    sel = vis & (rank < k)
    tok = np.arange(S)[None, :]
    win = (tok <= rows[:, None]) & (tok > rows[:, None] - W)
    mask = np.concatenate([sel, win], axis=1)
    O = _matrix_attention(qn, np.concatenate([kv, kt], axis=0), mask, sink)
    if inv_rope:
        O = rope_partial(O, rows[:, None], rope_dim, rope_base, inverse=True)
    return O


def hca_layer_matrix(q, C, Z, B, sink, *, m=128, W=128, norm_rope=False, inv_rope=False,
                     rope_dim=64, rope_base=10000.0, store_round=None, rows=None):
    S = np.asarray(C).shape[0]
    rows = np.arange(S) if rows is None else np.asarray(rows)
    qr = np.asarray(q, np.float64)[rows]
    qn, kt = _prep(qr, C, rows, norm_rope, rope_dim, rope_base)
    if store_round:
        qn, kt = store_round(qn), store_round(kt)
    kv = _entries(C, Z, B, m, False, norm_rope, rope_dim, rope_base, store_round)
    vis = np.arange(kv.shape[0])[None, :] < n_visible(rows, m)[:, None]
    tok = np.arange(S)[None, :]
    win = (tok <= rows[:, None]) & (tok > rows[:, None] - W)
    O = _matrix_attention(qn, np.concatenate([kv, kt], axis=0), np.concatenate([vis, win], 1), sink)
    if inv_rope:
        O = rope_partial(O, rows[:, None], rope_dim, rope_base, inverse=True)
    return O


# ----------------------------------------------------------------------------
# Decode (one new query per sequence, caches precomputed).
# ----------------------------------------------------------------------------

def csa_decode(q, qI, w, kI, kv, swa, sink, t, *, k, m=4, inv_rope=True, rope_dim=64,
               rope_base=10000.0):
    """One sequence, one query at position t (the newest token).
    q [H, D] (already normalised and rotated), qI [HI, DI], w [HI], kI [n_e, DI],
    kv [n_e, D] dequantised cache, swa [W, D] raw window rows (newest included).
    Returns (O [H, D], idx [k])."""
    nv = int(n_visible(t, m))
    I = indexer_scores(np.asarray(qI, np.float64)[None], np.asarray(w, np.float64)[None], kI, [nv])
    idx = topk_select(I, [nv], k)
    Op, lp = sparse_attention_partial(np.asarray(q, np.float64)[None], kv, idx)
    O = window_sink_combine(np.asarray(q, np.float64)[None], None, [t], None, sink, Op, lp,
                            inv_rope=inv_rope, rope_dim=rope_dim, rope_base=rope_base,
                            window_rows=[swa])
    return O[0], idx[0]


def hca_decode(q, kv, swa, sink, t, *, m=128, inv_rope=True, rope_dim=64, rope_base=10000.0):
    nv = int(n_visible(t, m))
    Op, lp = dense_attention_partial(np.asarray(q, np.float64)[None], kv, [nv])
    O = window_sink_combine(np.asarray(q, np.float64)[None], None, [t], None, sink, Op, lp,
                            inv_rope=inv_rope, rope_dim=rope_dim, rope_base=rope_base,
                            window_rows=[swa])
    return O[0]


# ----------------------------------------------------------------------------
# The rest of the layer stack [LQ §3, config block and the note after it]: the
# first layers attend through the sliding window only, and every layer's
# attention output goes through a grouped output projection
# (output_proj_groups 8, intermediate_attn_dim 1024, hidden_size 4096).
# ----------------------------------------------------------------------------

def swa_layer(q, C, sink, *, W: int = 128, norm_rope: bool = False, inv_rope: bool = False,
              rope_dim: int = 64, rope_base: float = 10000.0, store_round=None, rows=None):
    """Sliding-window-only layer: each query attends to the raw tokens
    [max(0, t-W+1), t] and the sink in one softmax; no compressed branch.
    Same normalisation, RoPE and window rows as csa_layer / hca_layer."""
    S = np.asarray(C).shape[0]
    rows = np.arange(S) if rows is None else np.asarray(rows)
    qr = np.asarray(q, np.float64)[rows]
    qn, kt = _prep(qr, C, rows, norm_rope, rope_dim, rope_base)
    if store_round:
        qn, kt = store_round(qn), store_round(kt)
    T, H, _ = qn.shape
    empty_O, empty_lse = np.zeros(qn.shape), np.full((T, H), -np.inf)
    return window_sink_combine(qn, kt, rows, W, sink, empty_O, empty_lse, inv_rope=inv_rope,
                               rope_dim=rope_dim, rope_base=rope_base)


def grouped_out_proj(O, w_grp, w_out, *, mid_round=None, return_mid: bool = False):
    """Grouped output projection of an attention output O [T, H, D].

    The H heads form G = w_grp.shape[0] groups of H/G consecutive heads.  Group
    g's heads, concatenated in head order ([T, (H/G)*D]), are mapped by its own
    matrix w_grp[g] ([d_mid, (H/G)*D], laid out [out, in]) to d_mid dims; the
    G results, concatenated in group order ([T, G*d_mid]), are mapped by
    w_out ([d_model, G*d_mid]) to the model width.  No bias.  mid_round rounds
    the intermediate to its storage type (e.g. bf16_round).
    Returns out [T, d_model] (and the intermediate if return_mid)."""
    O = np.asarray(O, np.float64)
    w_grp = np.asarray(w_grp, np.float64)
    T, H, D = O.shape
    G, d_mid, d_in = w_grp.shape
    if H % G or d_in != (H // G) * D:
        raise ValueError("w_grp must be [G, d_mid, (H/G)*D] with G dividing H")
    hg = H // G
    parts = []
    for g in range(G):
        X = O[:, g * hg:(g + 1) * hg, :].reshape(T, hg * D)
        parts.append(X @ w_grp[g].T)
    mid = np.concatenate(parts, axis=1)
    if mid_round is not None:
        mid = mid_round(mid)
    out = mid @ np.asarray(w_out, np.float64).T
    return (out, mid) if return_mid else out


# ----------------------------------------------------------------------------
# Decode-time cache writer: the compressor applied to a token stream, one token
# at a time, emitting a cache row when a block completes  [CS "KV 压缩" (entries
# are produced block by block), "其他辅助设计" (non-RoPE dims in FP8, RoPE dims
# in BF16); LD (FP8 caches)].
# ----------------------------------------------------------------------------

def fp8_row_quantize(x, rope_dim: int = 64):
    """One cache row: the first D - rope_dim dims as e4m3 codes under the row
    scale amax / 448 (value = decode(code) * scale; scale 1 for an all-zero
    row), the last rope_dim dims rounded to bf16.  Returns (codes [D - r] uint8,
    rope [r] float64 bf16-valued, scale float64)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    nope = x[..., :D - rope_dim]
    amax = np.abs(nope).max(axis=-1)
    scale = np.where(amax > 0, amax / 448.0, 1.0)
    codes = e4m3_encode(nope / scale[..., None])
    return codes, bf16_round(x[..., D - rope_dim:]), scale


def stream_append(ring_C, ring_Z, c, z, pos: int, B, m: int, overlap: bool, *, norm_rope: bool = True,
                  rope_dim: int = 64, rope_base: float = 10000.0):
    """Store token `pos` (rows c, z) in the sequence's ring of the last 2m
    tokens (slot pos % 2m) and, when its block is complete ((pos + 1) % m == 0),
    return (i, entry) for entry i = (pos + 1) / m - 1: the compressor over the
    current block (and, overlapping, the previous one) read from the ring, then
    RMSNorm and RoPE at position i * m.  Otherwise returns None."""
    L = 2 * m
    ring_C[pos % L] = c
    ring_Z[pos % L] = z
    if (pos + 1) % m:
        return None
    i = (pos + 1) // m - 1
    first = (i - 1) * m if (overlap and i > 0) else i * m
    rows = [(first + j) % L for j in range((i + 1) * m - first)]
    entry = compress(np.asarray(ring_C)[rows], np.asarray(ring_Z)[rows], B, m, overlap)[-1]
    if norm_rope:
        entry = rope_partial(rmsnorm(entry), i * m, rope_dim, rope_base)
    return i, entry


def flop_counts(S, H, D, m, k=None, W=128, HI=0, DI=0, dense=False):
    """Algorithmic FLOPs of one prefill layer: attention 4*D*H per (query, row)
    over min(k, n_vis) (or n_vis if dense) entries plus min(W, t+1) window rows;
    indexer 2*HI*DI per (query, visible entry)."""
    t = np.arange(S, dtype=np.int64)
    nv = (t + 1) // m
    rows_c = nv if dense else np.minimum(k, nv)
    attn = 4 * D * H * int((rows_c + np.minimum(W, t + 1)).sum())
    idx = 0 if dense else 2 * HI * DI * int(nv.sum())
    return attn, idx
