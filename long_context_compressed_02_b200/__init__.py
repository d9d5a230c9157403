"""Python binding of libcsa.so (CSA / HCA hybrid compressed attention on B200).

Argument marshalling only: every step of the layer runs in the CUDA kernels
behind the C ABI declared in include/csa.h.  torch supplies device memory and
the current stream.  There is no fallback: if libcsa.so is missing or a call
fails, an exception is raised.

Entry points (same names as the C ABI):
  csa_compress, csa_compress_append, csa_rmsnorm_rope, csa_index_topk,
  csa_sparse_mqa, hca_dense_attn, swa_sink_combine, csa_fused_attention,
  csa_fused_attention_splitkv (n_split > 1), csa_index_topk_fp4, csa_cache_append,
  csa_grouped_out_proj
and compositions of them: csa_layer_prefill, hca_layer_prefill,
swa_layer_prefill, csa_layer_decode, hca_layer_decode, swa_layer_decode.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

F32, BF16, E4M3 = 0, 1, 2
_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.uint8: E4M3}

_lib = None


class CsaError(RuntimeError):
    pass


def lib():
    """Loads libcsa.so once and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise CsaError(f"{LIB_PATH} is not built; run `python -m long_context_compressed_02_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "csa_abi_version": ([], I),
        "csa_status_string": ([I], ctypes.c_char_p),
        "csa_last_error": ([], ctypes.c_char_p),
        "csa_check_device_error": ([P], I),
        "csa_compress": ([P, P, P, P, P, I64, I, I, I, I, I, I, F, F, P, I, P], I),
        "csa_rmsnorm_rope": ([P, I, I64, I, I, I64, I, I, F, F, P, I, P], I),
        "csa_index_topk_workspace": ([I, I, I64, I], SZ),
        "csa_index_topk": ([P, P, P, P, P, P, I, I, I, I, I64, I, I, P, P, SZ, P], I),
        "csa_sparse_mqa": ([P, I, P, I, P, P, I64, P, I, I, I, I, I, I, F, P, P, P], I),
        "hca_dense_attn": ([P, I, P, I, P, P, I64, P, I, I, I, I, I, I, F, P, P, P], I),
        "swa_sink_combine": ([P, I, P, I, I64, P, I, I, P, P, P, I, I, I, I, I, F, I, F, P, I, P], I),
        "csa_fused_attention": ([P, I, P, I, P, P, I64, P, I, I, P, I, I64, I, I, P, P, I, I, I, I, I, F, I, F,
                                 P, I, P], I),
        "csa_index_topk_noalloc": ([P, P, P, P, P, P, I, I, I, I, I64, I, I, P, P], I),
        "csa_fused_attention_workspace": ([I, I, I, I, I], SZ),
        "csa_fused_attention_splitkv": ([P, I, P, I, P, P, I64, P, I, I, P, I, I64, I, I, P, P, I, I, I, I, I, F, I, F,
                                         I, P, SZ, P, I, P], I),
        "csa_compress_append": ([P, P, I, P, I, I, I, I, P, P, P, P, P, P, I64, I, I, F, F, P], I),
        "csa_grouped_out_proj": ([P, P, P, I, I, I, I, I, I, P, P, I, P], I),
        "csa_get_last_error_string": ([], ctypes.c_char_p),
        "csa_workspace_size": ([I, I, I64, I, I, I, I], SZ),
        "csa_selftest_wait_timeout": ([ctypes.c_uint64, P], I),
        "csa_cache_append": ([P, P, I, P, I, I, I, I, P, P, P, P, P, P, I64, I, F, F, P, P, P, I, P, P, P, P, P], I),
        "csa_index_topk_fp4_workspace": ([I, I, I, I64, I], SZ),
        "csa_index_topk_fp4": ([P, P, P, P, P, P, I, I, I, I64, I, I, P, P, SZ, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(status, what):
    if status != 0:
        L = lib()
        raise CsaError(f"{what}: {L.csa_status_string(status).decode()}: {L.csa_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name):
    if t is None:
        return
    if not t.is_cuda:
        raise CsaError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise CsaError(f"{name} must be contiguous")


def num_sms(device=None):
    """Streaming multiprocessors of the current (or given) CUDA device."""
    return torch.cuda.get_device_properties(torch.cuda.current_device() if device is None else device).multi_processor_count


def csa_fused_attention_workspace(n_seq, T, H, D, n_split):
    return int(lib().csa_fused_attention_workspace(n_seq, T, H, D, n_split))


def selftest_wait_timeout(limit_ns=1_000_000, stream=None):
    """Launches the bounded-wait self-test (a wait that nothing completes,
    limit limit_ns); the next check_device_error reports the expiry."""
    _check(lib().csa_selftest_wait_timeout(int(limit_ns), _stream(stream)), "csa_selftest_wait_timeout")


def check_device_error(stream=None):
    """Synchronises the stream and raises if a kernel recorded an error."""
    _check(lib().csa_check_device_error(_stream(stream)), "csa_check_device_error")


# ---------------------------------------------------------------- steps

def csa_compress(C, Z, B, m, overlap, *, Cb=None, Zb=None, norm=False, rope_dim=0, rope_base=10000.0,
                 eps=1e-6, out_dtype=None, out=None, stream=None):
    """Softmax-gated block compressor: [S, D] -> [S // m, D]."""
    for t, n in ((C, "C"), (Z, "Z"), (B, "B"), (Cb, "Cb"), (Zb, "Zb")):
        _dev(t, n)
    S, D = C.shape
    out_dtype = C.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((S // m, D), dtype=out_dtype, device=C.device)
    _check(lib().csa_compress(_ptr(C), _ptr(Z), _ptr(Cb), _ptr(Zb), _ptr(B), S, D, m, int(overlap),
                              _DT[C.dtype], int(norm), rope_dim, rope_base, eps, _ptr(out), _DT[out.dtype],
                              _stream(stream)), "csa_compress")
    return out


def csa_compress_append(c_tok, z_tok, B, m, overlap, q_pos, ring_C, ring_Z, kv_nope, kv_rope, kv_scale, *,
                        norm=True, rope_dim=64, rope_base=10000.0, eps=1e-6, stream=None):
    """Decode-time cache writer: appends each sequence's new token (c_tok, z_tok
    [n_seq, D]) at position q_pos[b] to its ring of the last 2m tokens
    (ring_C, ring_Z [n_seq, 2m, D], same dtype) and, when the token completes a
    block, writes the block's entry into the e4m3 cache row (kv_nope
    [n_seq, cap, D-64] uint8, kv_rope [n_seq, cap, 64] bf16, kv_scale [n_seq, cap])."""
    for t, n in ((c_tok, "c_tok"), (z_tok, "z_tok"), (B, "B"), (q_pos, "q_pos"), (ring_C, "ring_C"),
                 (ring_Z, "ring_Z"), (kv_nope, "kv_nope"), (kv_rope, "kv_rope"), (kv_scale, "kv_scale")):
        _dev(t, n)
    n_seq, D = c_tok.shape
    if z_tok.shape != c_tok.shape or ring_C.dtype != c_tok.dtype or ring_Z.dtype != c_tok.dtype or \
            tuple(ring_C.shape) != (n_seq, 2 * m, D) or tuple(ring_Z.shape) != (n_seq, 2 * m, D):
        raise CsaError("csa_compress_append: c_tok/z_tok [n_seq, D] and rings [n_seq, 2m, D] of one dtype expected")
    if kv_nope.shape[:2] != kv_rope.shape[:2] or tuple(kv_scale.shape) != tuple(kv_nope.shape[:2]) or \
            kv_nope.shape[0] != n_seq or kv_nope.shape[2] + rope_dim != D:
        raise CsaError("csa_compress_append: cache rows [n_seq, cap, D - rope_dim] / [n_seq, cap, rope_dim] / "
                       "[n_seq, cap] expected")
    _check(lib().csa_compress_append(_ptr(c_tok), _ptr(z_tok), _DT[c_tok.dtype], _ptr(B), n_seq, D, m, int(overlap),
                                     _ptr(q_pos), _ptr(ring_C), _ptr(ring_Z), _ptr(kv_nope), _ptr(kv_rope),
                                     _ptr(kv_scale), kv_nope.shape[1], int(norm), rope_dim, rope_base, eps,
                                     _stream(stream)), "csa_compress_append")


def csa_cache_append(c_tok, z_tok, B, m, overlap, q_pos, ring_C, ring_Z, kv_nope, kv_rope, kv_scale,
                     ci_tok, zi_tok, B_I, ring_CI, ring_ZI, kI, kI_scale, *, rope_dim=64, rope_base=10000.0,
                     eps=1e-6, stream=None):
    """Decode-time cache write of a CSA layer in one launch: the KV row (as
    csa_compress_append with norm on) and the indexer key of the same block,
    pooled from its own stream (ci_tok, zi_tok [n_seq, DI], B_I, rings
    [n_seq, 2m, DI]) and stored as e4m3 kI [n_seq, cap, DI] + kI_scale [n_seq, cap]."""
    for t, n in ((c_tok, "c_tok"), (z_tok, "z_tok"), (B, "B"), (q_pos, "q_pos"), (ring_C, "ring_C"),
                 (ring_Z, "ring_Z"), (kv_nope, "kv_nope"), (kv_rope, "kv_rope"), (kv_scale, "kv_scale"),
                 (ci_tok, "ci_tok"), (zi_tok, "zi_tok"), (B_I, "B_I"), (ring_CI, "ring_CI"), (ring_ZI, "ring_ZI"),
                 (kI, "kI"), (kI_scale, "kI_scale")):
        _dev(t, n)
    n_seq, D = c_tok.shape
    DI = ci_tok.shape[1]
    cap = kv_nope.shape[1]
    if tuple(ring_C.shape) != (n_seq, 2 * m, D) or tuple(ring_CI.shape) != (n_seq, 2 * m, DI) or \
            tuple(kI.shape) != (n_seq, cap, DI) or tuple(kI_scale.shape) != (n_seq, cap) or \
            ci_tok.dtype != c_tok.dtype or ring_CI.dtype != c_tok.dtype or ring_C.dtype != c_tok.dtype:
        raise CsaError("csa_cache_append: rings [n_seq, 2m, D|DI], kI [n_seq, cap, DI], kI_scale [n_seq, cap] of "
                       "the token dtype expected")
    _check(lib().csa_cache_append(_ptr(c_tok), _ptr(z_tok), _DT[c_tok.dtype], _ptr(B), n_seq, D, m, int(overlap),
                                  _ptr(q_pos), _ptr(ring_C), _ptr(ring_Z), _ptr(kv_nope), _ptr(kv_rope),
                                  _ptr(kv_scale), cap, rope_dim, rope_base, eps, _ptr(ci_tok), _ptr(zi_tok),
                                  _ptr(B_I), DI, _ptr(ring_CI), _ptr(ring_ZI), _ptr(kI), _ptr(kI_scale),
                                  _stream(stream)), "csa_cache_append")


def csa_rmsnorm_rope(x, rows_per_pos=1, pos0=0, *, norm=True, rope_dim=64, rope_base=10000.0, eps=1e-6,
                     out_dtype=None, out=None, stream=None):
    """RMSNorm + partial RoPE of rows; x [..., D], rows_per_pos rows share a position."""
    _dev(x, "x")
    D = x.shape[-1]
    rows = x.numel() // D
    out_dtype = x.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype, device=x.device)
    _check(lib().csa_rmsnorm_rope(_ptr(x), _DT[x.dtype], rows, D, rows_per_pos, pos0, int(norm), rope_dim,
                                  rope_base, eps, _ptr(out), _DT[out.dtype], _stream(stream)), "csa_rmsnorm_rope")
    return out


def csa_index_topk_workspace(n_seq, T, cap, k):
    return int(lib().csa_index_topk_workspace(n_seq, T, cap, k))


def csa_index_topk(qI, w, kI, q_pos, m, k, *, qI_scale=None, kI_scale=None, workspace=None, idx=None,
                   stream=None):
    """Lightning indexer + top-k.  qI [n_seq, T, HI, DI] uint8 (e4m3 codes),
    w [n_seq, T, HI] f32, kI [n_seq, cap, DI] uint8, q_pos [n_seq] int64.
    Returns idx [n_seq, T, k] int32 (ascending, -1 padded)."""
    for t, n in ((qI, "qI"), (w, "w"), (kI, "kI"), (q_pos, "q_pos"), (qI_scale, "qI_scale"), (kI_scale, "kI_scale")):
        _dev(t, n)
    n_seq, T, HI, DI = qI.shape
    cap = kI.shape[1]
    need = csa_index_topk_workspace(n_seq, T, cap, k)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=qI.device)
    if idx is None:
        idx = torch.empty((n_seq, T, k), dtype=torch.int32, device=qI.device)
    _check(lib().csa_index_topk(_ptr(qI), _ptr(qI_scale), _ptr(w), _ptr(kI), _ptr(kI_scale), _ptr(q_pos),
                                n_seq, T, HI, DI, cap, m, k, _ptr(idx), _ptr(workspace), workspace.numel(),
                                _stream(stream)), "csa_index_topk")
    return idx


def csa_index_topk_fp4_workspace(n_seq, T, HI, cap, k):
    return int(lib().csa_index_topk_fp4_workspace(n_seq, T, HI, cap, k))


def csa_index_topk_fp4(qI4, qI4_scale, w, kI4, kI4_scale, q_pos, m, k, *, workspace=None, idx=None, stream=None):
    """Lightning indexer + top-k on MX FP4 operands: qI4 [n_seq, T, HI, 64] and
    kI4 [n_seq, cap, 64] uint8 (packed E2M1, the even element in the low
    nibble), qI4_scale [n_seq, T, HI, 4] and kI4_scale [n_seq, cap, 4] uint8
    (E8M0 per 32-element block), w [n_seq, T, HI] f32, q_pos [n_seq] int64.
    Returns idx [n_seq, T, k] int32 (ascending, -1 padded)."""
    for t, n in ((qI4, "qI4"), (qI4_scale, "qI4_scale"), (w, "w"), (kI4, "kI4"), (kI4_scale, "kI4_scale"),
                 (q_pos, "q_pos")):
        _dev(t, n)
    n_seq, T, HI, _ = qI4.shape
    cap = kI4.shape[1]
    if qI4.shape[-1] != 64 or kI4.shape[-1] != 64 or qI4_scale.shape[-1] != 4 or kI4_scale.shape[-1] != 4:
        raise CsaError("csa_index_topk_fp4: 64 code bytes and 4 scale bytes per 128-element row expected")
    need = int(lib().csa_index_topk_fp4_workspace(n_seq, T, HI, cap, k))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=qI4.device)
    if idx is None:
        idx = torch.empty((n_seq, T, k), dtype=torch.int32, device=qI4.device)
    _check(lib().csa_index_topk_fp4(_ptr(qI4), _ptr(qI4_scale), _ptr(w), _ptr(kI4), _ptr(kI4_scale), _ptr(q_pos),
                                    n_seq, T, HI, cap, m, k, _ptr(idx), _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "csa_index_topk_fp4")
    return idx


def _kv_args(kv, kv_rope, kv_scale):
    return _DT[kv.dtype], _ptr(kv), _ptr(kv_rope), _ptr(kv_scale)


def csa_sparse_mqa(q, kv, idx, *, kv_rope=None, kv_scale=None, scale=None, rope_dim=None, out=None,
                   stream=None):
    """Sparse shared-KV MQA over kv[b, idx[b, t, :]].  q [n_seq, T, H, D];
    kv [n_seq, cap, D] (bf16/f32) or e4m3 [n_seq, cap, D-64] + kv_rope + kv_scale.
    Returns (O_part [n_seq, T, H, D] f32, lse_part [n_seq, T, H] f32)."""
    for t, n in ((q, "q"), (kv, "kv"), (idx, "idx"), (kv_rope, "kv_rope"), (kv_scale, "kv_scale")):
        _dev(t, n)
    n_seq, T, H, D = q.shape
    cap = kv.shape[1]
    k = idx.shape[-1]
    rope_dim = (64 if kv.dtype == torch.uint8 else 0) if rope_dim is None else rope_dim
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    O = torch.empty((n_seq, T, H, D), dtype=torch.float32, device=q.device) if out is None else out[0]
    L = torch.empty((n_seq, T, H), dtype=torch.float32, device=q.device) if out is None else out[1]
    kvd, kvp, kvr, kvs = _kv_args(kv, kv_rope, kv_scale)
    _check(lib().csa_sparse_mqa(_ptr(q), _DT[q.dtype], kvp, kvd, kvr, kvs, cap, _ptr(idx), k, n_seq, T, H, D,
                                rope_dim, scale, _ptr(O), _ptr(L), _stream(stream)), "csa_sparse_mqa")
    return O, L


def hca_dense_attn(q, kv, q_pos, m, *, kv_rope=None, kv_scale=None, scale=None, rope_dim=None, out=None,
                   stream=None):
    """Dense causal attention over the complete m-entries kv[b, :n_vis]."""
    for t, n in ((q, "q"), (kv, "kv"), (q_pos, "q_pos"), (kv_rope, "kv_rope"), (kv_scale, "kv_scale")):
        _dev(t, n)
    n_seq, T, H, D = q.shape
    cap = kv.shape[1]
    rope_dim = (64 if kv.dtype == torch.uint8 else 0) if rope_dim is None else rope_dim
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    O = torch.empty((n_seq, T, H, D), dtype=torch.float32, device=q.device) if out is None else out[0]
    L = torch.empty((n_seq, T, H), dtype=torch.float32, device=q.device) if out is None else out[1]
    kvd, kvp, kvr, kvs = _kv_args(kv, kv_rope, kv_scale)
    _check(lib().hca_dense_attn(_ptr(q), _DT[q.dtype], kvp, kvd, kvr, kvs, cap, _ptr(q_pos), m, n_seq, T, H, D,
                                rope_dim, scale, _ptr(O), _ptr(L), _stream(stream)), "hca_dense_attn")
    return O, L


def swa_sink_combine(q, kv_tok, q_pos, W, sink, O_part=None, lse_part=None, *, window_mode=0, inv_rope=False,
                     rope_dim=64, rope_base=10000.0, scale=None, out_dtype=None, out=None, stream=None):
    """Window attention + sink + merge with the compressed-branch partial."""
    for t, n in ((q, "q"), (kv_tok, "kv_tok"), (q_pos, "q_pos"), (sink, "sink"), (O_part, "O_part"),
                 (lse_part, "lse_part")):
        _dev(t, n)
    n_seq, T, H, D = q.shape
    cap = kv_tok.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((n_seq, T, H, D), dtype=out_dtype, device=q.device)
    _check(lib().swa_sink_combine(_ptr(q), _DT[q.dtype], _ptr(kv_tok), _DT[kv_tok.dtype], cap, _ptr(q_pos), W,
                                  window_mode, _ptr(sink), _ptr(O_part), _ptr(lse_part), n_seq, T, H, D,
                                  rope_dim, rope_base, int(inv_rope), scale,
                                  _ptr(out), _DT[out.dtype], _stream(stream)), "swa_sink_combine")
    return out


def csa_fused_attention(q, kv, kv_tok, q_pos, W, sink, *, idx=None, m=1, kv_rope=None, kv_scale=None,
                        window_mode=0, inv_rope=False, rope_dim=None, rope_base=10000.0, scale=None,
                        out_dtype=None, out=None, n_split=1, workspace=None, stream=None):
    """Compressed rows (idx given: gathered top-k entries; else the dense prefix
    of complete m-entries) + raw window rows + sink in one softmax, then the
    optional inverse RoPE.  q [n_seq, T, H, D]; kv [n_seq, cap, D] (or e4m3 +
    kv_rope + kv_scale); kv_tok [n_seq, tok_cap, D]."""
    for t, n in ((q, "q"), (kv, "kv"), (kv_tok, "kv_tok"), (q_pos, "q_pos"), (sink, "sink"), (idx, "idx"),
                 (kv_rope, "kv_rope"), (kv_scale, "kv_scale")):
        _dev(t, n)
    n_seq, T, H, D = q.shape
    rope_dim = (64 if (kv.dtype == torch.uint8 or inv_rope) else 0) if rope_dim is None else rope_dim
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((n_seq, T, H, D), dtype=out_dtype, device=q.device)
    k = 0 if idx is None else idx.shape[-1]
    kvd, kvp, kvr, kvs = _kv_args(kv, kv_rope, kv_scale)
    if n_split > 1:
        need = int(lib().csa_fused_attention_workspace(n_seq, T, H, D, n_split))
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _check(lib().csa_fused_attention_splitkv(
            _ptr(q), _DT[q.dtype], kvp, kvd, kvr, kvs, kv.shape[1], _ptr(idx), k, m, _ptr(kv_tok), _DT[kv_tok.dtype],
            kv_tok.shape[1], W, window_mode, _ptr(q_pos), _ptr(sink), n_seq, T, H, D, rope_dim, rope_base,
            int(inv_rope), scale, n_split, _ptr(workspace), workspace.numel(), _ptr(out), _DT[out.dtype],
            _stream(stream)), "csa_fused_attention_splitkv")
        return out
    _check(lib().csa_fused_attention(_ptr(q), _DT[q.dtype], kvp, kvd, kvr, kvs, kv.shape[1], _ptr(idx), k, m,
                                     _ptr(kv_tok), _DT[kv_tok.dtype], kv_tok.shape[1], W, window_mode, _ptr(q_pos),
                                     _ptr(sink), n_seq, T, H, D, rope_dim, rope_base, int(inv_rope), scale,
                                     _ptr(out), _DT[out.dtype], _stream(stream)), "csa_fused_attention")
    return out


def csa_grouped_out_proj(o, w_grp, w_out, *, mid=None, out=None, out_dtype=torch.bfloat16, return_mid=False,
                         stream=None):
    """Grouped output projection: o [M, H, D] bf16; w_grp [G, d_mid, (H/G)*D]
    bf16 (group g = heads g*H/G ..); w_out [d_model, G*d_mid] bf16.  Returns
    out [M, d_model] (and the bf16 intermediate [M, G*d_mid] if return_mid)."""
    for t, n in ((o, "o"), (w_grp, "w_grp"), (w_out, "w_out"), (mid, "mid"), (out, "out")):
        _dev(t, n)
    M, H, D = o.shape
    G, d_mid, d_in = w_grp.shape
    d_model = w_out.shape[0]
    if o.dtype != torch.bfloat16 or w_grp.dtype != torch.bfloat16 or w_out.dtype != torch.bfloat16:
        raise CsaError("csa_grouped_out_proj: o, w_grp and w_out must be bf16")
    if H % G or d_in != (H // G) * D or tuple(w_out.shape) != (d_model, G * d_mid):
        raise CsaError("csa_grouped_out_proj: w_grp [G, d_mid, (H/G)*D] and w_out [d_model, G*d_mid] expected")
    if mid is None:
        mid = torch.empty((M, G * d_mid), dtype=torch.bfloat16, device=o.device)
    if out is None:
        out = torch.empty((M, d_model), dtype=out_dtype, device=o.device)
    if mid.dtype != torch.bfloat16 or tuple(mid.shape) != (M, G * d_mid) or tuple(out.shape) != (M, d_model):
        raise CsaError("csa_grouped_out_proj: mid [M, G*d_mid] bf16 and out [M, d_model] expected")
    _check(lib().csa_grouped_out_proj(_ptr(o), _ptr(w_grp), _ptr(w_out), M, H, D, G, d_mid, d_model, _ptr(mid),
                                      _ptr(out), _DT[out.dtype], _stream(stream)), "csa_grouped_out_proj")
    return (out, mid) if return_mid else out


# ---------------------------------------------------------------- layers

def csa_layer_prefill(q, C, Z, B, qI, w, kI, sink, *, k, m=4, W=128, norm_rope=False, inv_rope=False,
                      rope_dim=64, rope_base=10000.0, kv_dtype=None, workspace=None, return_idx=False,
                      fused=True):
    """One CSA layer (batch 1): compress -> index/top-k -> sparse MQA -> window + sink.
    q [S, H, D], C/Z [S, D], B [2m, D] f32, qI [S, HI, DI] u8, w [S, HI], kI [S//m, DI] u8, sink [H]."""
    S, H, D = q.shape
    dev = q.device
    kv_dtype = q.dtype if kv_dtype is None else kv_dtype
    pos = torch.zeros(1, dtype=torch.int64, device=dev)
    if norm_rope:
        qn = csa_rmsnorm_rope(q, rows_per_pos=H, rope_dim=rope_dim, rope_base=rope_base)
        kt = csa_rmsnorm_rope(C, rows_per_pos=1, rope_dim=rope_dim, rope_base=rope_base, out_dtype=kv_dtype)
        kv = csa_compress(C, Z, B, m, True, norm=True, rope_dim=rope_dim, rope_base=rope_base, out_dtype=kv_dtype)
    else:
        qn, kt = q, C
        kv = csa_compress(C, Z, B, m, True, out_dtype=kv_dtype)
    idx = csa_index_topk(qI[None], w[None], kI[None], pos, m, k, workspace=workspace)
    if fused:
        out = csa_fused_attention(qn[None], kv[None], kt[None], pos, W, sink, idx=idx, inv_rope=inv_rope,
                                  rope_dim=rope_dim if norm_rope else 0, rope_base=rope_base)
    else:
        Op, Lp = csa_sparse_mqa(qn[None], kv[None], idx)
        out = swa_sink_combine(qn[None], kt[None], pos, W, sink, Op, Lp, window_mode=0, inv_rope=inv_rope,
                               rope_dim=rope_dim if norm_rope else 0, rope_base=rope_base)
    return (out[0], idx[0]) if return_idx else out[0]


def hca_layer_prefill(q, C, Z, B, sink, *, m=128, W=128, norm_rope=False, inv_rope=False, rope_dim=64,
                      rope_base=10000.0, kv_dtype=None, fused=True):
    """One HCA layer (batch 1): compress (m' = 128) -> dense attention -> window + sink."""
    S, H, D = q.shape
    dev = q.device
    kv_dtype = q.dtype if kv_dtype is None else kv_dtype
    pos = torch.zeros(1, dtype=torch.int64, device=dev)
    if norm_rope:
        qn = csa_rmsnorm_rope(q, rows_per_pos=H, rope_dim=rope_dim, rope_base=rope_base)
        kt = csa_rmsnorm_rope(C, rows_per_pos=1, rope_dim=rope_dim, rope_base=rope_base, out_dtype=kv_dtype)
        kv = csa_compress(C, Z, B, m, False, norm=True, rope_dim=rope_dim, rope_base=rope_base, out_dtype=kv_dtype)
    else:
        qn, kt = q, C
        kv = csa_compress(C, Z, B, m, False, out_dtype=kv_dtype)
    if fused:
        out = csa_fused_attention(qn[None], kv[None], kt[None], pos, W, sink, m=m, inv_rope=inv_rope,
                                  rope_dim=rope_dim if norm_rope else 0, rope_base=rope_base)
    else:
        Op, Lp = hca_dense_attn(qn[None], kv[None], pos, m)
        out = swa_sink_combine(qn[None], kt[None], pos, W, sink, Op, Lp, window_mode=0, inv_rope=inv_rope,
                               rope_dim=rope_dim if norm_rope else 0, rope_base=rope_base)
    return out[0]


def swa_layer_prefill(q, C, sink, *, W=128, norm_rope=False, inv_rope=False, rope_dim=64, rope_base=10000.0,
                      kv_dtype=None):
    """One sliding-window-only layer (batch 1): window + sink attention over the
    raw tokens, no compressed branch.  q [S, H, D], C [S, D], sink [H]."""
    S, H, D = q.shape
    kv_dtype = q.dtype if kv_dtype is None else kv_dtype
    pos = torch.zeros(1, dtype=torch.int64, device=q.device)
    if norm_rope:
        qn = csa_rmsnorm_rope(q, rows_per_pos=H, rope_dim=rope_dim, rope_base=rope_base)
        kt = csa_rmsnorm_rope(C, rows_per_pos=1, rope_dim=rope_dim, rope_base=rope_base, out_dtype=kv_dtype)
    else:
        qn, kt = q, C
    out = swa_sink_combine(qn[None], kt[None], pos, W, sink, window_mode=0, inv_rope=inv_rope,
                           rope_dim=rope_dim if norm_rope else 0, rope_base=rope_base)
    return out[0]


def swa_layer_decode(lay, q_pos, *, W=128, out=None, stream=None):
    """One sliding-window-only layer, one decode step per sequence: the SWA
    cache and the sink in one softmax, inverse RoPE at q_pos.  `lay` holds q,
    swa and sink (the layout of synth's decode inputs)."""
    return swa_sink_combine(lay["q"], lay["swa"], q_pos, W, lay["sink"], window_mode=1, inv_rope=True,
                            rope_dim=64, out=out, stream=stream)


def csa_layer_decode(lay, q_pos, *, k, m=4, W=128, n_split=1, idx=None, out=None, index_workspace=None,
                     attn_workspace=None, stream=None):
    """One CSA layer, one decode step per sequence over its caches: lightning
    indexer + top-k over the e4m3 key cache, then the selected e4m3 entries,
    the SWA cache and the sink in one softmax, inverse RoPE at q_pos.
    `lay` holds q, qI, qI_scale, w, kI, kI_scale, kv_nope, kv_rope, kv_scale,
    swa, sink (the layout of synth's decode inputs).  Returns (out, idx)."""
    idx = csa_index_topk(lay["qI"], lay["w"], lay["kI"], q_pos, m, k, qI_scale=lay["qI_scale"],
                         kI_scale=lay["kI_scale"], workspace=index_workspace, idx=idx, stream=stream)
    out = csa_fused_attention(lay["q"], lay["kv_nope"], lay["swa"], q_pos, W, lay["sink"], idx=idx,
                              kv_rope=lay["kv_rope"], kv_scale=lay["kv_scale"], window_mode=1, inv_rope=True,
                              rope_dim=lay["kv_rope"].shape[-1], out=out, n_split=n_split,
                              workspace=attn_workspace, stream=stream)
    return out, idx


def hca_layer_decode(lay, q_pos, *, m=128, W=128, n_split=1, out=None, attn_workspace=None, stream=None):
    """One HCA layer, one decode step per sequence: dense attention over every
    complete m'-entry of the e4m3 cache, the SWA cache and the sink in one
    softmax, inverse RoPE at q_pos."""
    return csa_fused_attention(lay["q"], lay["kv_nope"], lay["swa"], q_pos, W, lay["sink"], m=m,
                               kv_rope=lay["kv_rope"], kv_scale=lay["kv_scale"], window_mode=1, inv_rope=True,
                               rope_dim=lay["kv_rope"].shape[-1], out=out, n_split=n_split,
                               workspace=attn_workspace, stream=stream)
