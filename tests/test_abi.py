"""The C-ABI library loads on a machine without a GPU, exports every entry
point declared in include/csa.h, and rejects bad arguments on the host before
touching the device."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "csa.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(csa_\w+|hca_\w+|swa_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from long_context_compressed_02_b200 import build, lib
    build.build()
    return lib()


def test_header_declares_the_five_layer_entry_points():
    d = _declared()
    for n in ("csa_compress", "csa_index_topk", "csa_sparse_mqa", "hca_dense_attn", "swa_sink_combine"):
        assert n in d


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_abi_version_and_status_strings(L):
    assert L.csa_abi_version() == 1
    assert L.csa_status_string(0) == b"CSA_OK"
    assert L.csa_status_string(3) == b"CSA_ERR_WORKSPACE"


def test_workspace_size_is_host_arithmetic(L):
    # prefill: one chunk, the score matrix and the item counter (one 256-byte
    # block); decode: chunked candidates and key histograms too
    assert L.csa_index_topk_workspace(1, 16384, 4096, 512) == 16384 * 4096 * 4 + 256
    dec = L.csa_index_topk_workspace(16, 1, 262144, 512)
    assert dec >= 16 * 262144 * 4 + 2 * 16 * 16 * 512 * 4
    assert L.csa_index_topk_workspace(0, 1, 1, 1) == 0


def test_host_argument_validation(L):
    null = None
    # D not a multiple of 8
    st = L.csa_compress(ctypes.c_void_p(16), ctypes.c_void_p(16), null, null, null, 64, 7, 4, 1, 0, 0, 0,
                        10000.0, 1e-6, ctypes.c_void_p(16), 0, null)
    assert st == 1 and b"multiple of 8" in L.csa_last_error()
    # misaligned pointer
    st = L.csa_compress(ctypes.c_void_p(17), ctypes.c_void_p(16), null, null, null, 64, 8, 4, 1, 0, 0, 0,
                        10000.0, 1e-6, ctypes.c_void_p(16), 0, null)
    assert st == 1 and b"aligned" in L.csa_last_error()
    # indexer: DI unsupported
    st = L.csa_index_topk(ctypes.c_void_p(16), null, ctypes.c_void_p(16), ctypes.c_void_p(16), null,
                          ctypes.c_void_p(16), 1, 1, 4, 48, 8, 4, 4, ctypes.c_void_p(16), ctypes.c_void_p(16), 1 << 20,
                          null)
    assert st == 1 and b"DI" in L.csa_last_error()
    # indexer: workspace too small
    st = L.csa_index_topk(ctypes.c_void_p(16), null, ctypes.c_void_p(16), ctypes.c_void_p(16), null,
                          ctypes.c_void_p(16), 1, 8, 4, 32, 64, 4, 4, ctypes.c_void_p(16), ctypes.c_void_p(16), 8,
                          null)
    assert st == 3
    # attention: unsupported head dim
    st = L.csa_sparse_mqa(ctypes.c_void_p(16), 1, ctypes.c_void_p(16), 1, null, null, 16, ctypes.c_void_p(16), 4,
                          1, 1, 8, 96, 0, 0.1, ctypes.c_void_p(16), ctypes.c_void_p(16), null)
    assert st == 1 and b"D must be" in L.csa_last_error()
    # e4m3 store without its RoPE part
    st = L.hca_dense_attn(ctypes.c_void_p(16), 1, ctypes.c_void_p(16), 2, null, null, 16, ctypes.c_void_p(16), 128,
                          1, 1, 8, 512, 64, 0.1, ctypes.c_void_p(16), ctypes.c_void_p(16), null)
    assert st == 1 and b"e4m3" in L.csa_last_error()
    # combine: inverse RoPE without RoPE dims
    st = L.swa_sink_combine(ctypes.c_void_p(16), 1, ctypes.c_void_p(16), 1, 16, ctypes.c_void_p(16), 128, 0, null,
                            null, null, 1, 1, 8, 512, 0, 10000.0, 1, 0.1, ctypes.c_void_p(16), 1, null)
    assert st == 1 and b"inv_rope" in L.csa_last_error()


def test_cache_writer_host_validation(L):
    """csa_compress_append rejects bad shapes and pointers before any device work."""
    v = ctypes.c_void_p(16)
    args = dict(c=v, z=v, dt=1, B=v, n=2, D=512, m=4, ov=1, pos=v, rc=v, rz=v, kn=v, kr=v, ks=v, cap=16, norm=1,
                rope=64, base=10000.0, eps=1e-6)

    def call(**kw):
        a = dict(args, **kw)
        return L.csa_compress_append(a["c"], a["z"], a["dt"], a["B"], a["n"], a["D"], a["m"], a["ov"], a["pos"],
                                     a["rc"], a["rz"], a["kn"], a["kr"], a["ks"], a["cap"], a["norm"], a["rope"],
                                     a["base"], a["eps"], None)
    assert call(D=500) == 1 and b"multiple of 8" in L.csa_last_error()
    assert call(m=0) == 1 and b"m must be" in L.csa_last_error()
    assert call(rope=32) == 1 and b"rope_dim" in L.csa_last_error()
    assert call(dt=2) == 1 and b"in_dtype" in L.csa_last_error()
    assert call(cap=0) == 1
    assert call(rz=None) == 1 and b"null" in L.csa_last_error()
    assert call(kn=ctypes.c_void_p(24)) == 1 and b"aligned" in L.csa_last_error()
    assert call(n=0) == 0                                    # nothing to do


def test_python_binding_refuses_cpu_tensors():
    import torch
    import long_context_compressed_02_b200 as csa
    with pytest.raises(csa.CsaError):
        csa.csa_compress(torch.zeros(8, 8), torch.zeros(8, 8), torch.zeros(8, 8), 4, True)


def test_grouped_out_proj_host_validation(L):
    null = None
    p = ctypes.c_void_p(16)
    # group count must divide the head count
    assert L.csa_grouped_out_proj(p, p, p, 4, 64, 512, 7, 1024, 4096, p, p, 0, null) == 1
    assert b"divide" in L.csa_last_error()
    # widths that are not whole 256-column tiles
    assert L.csa_grouped_out_proj(p, p, p, 4, 64, 512, 8, 1000, 4096, p, p, 0, null) == 2
    # misaligned pointer
    assert L.csa_grouped_out_proj(ctypes.c_void_p(8), p, p, 4, 64, 512, 8, 1024, 4096, p, p, 0, null) == 1
    # bad output dtype
    assert L.csa_grouped_out_proj(p, p, p, 4, 64, 512, 8, 1024, 4096, p, p, 2, null) == 1
    # no rows: nothing to do, null pointers accepted, no device call
    assert L.csa_grouped_out_proj(null, null, null, 0, 64, 512, 8, 1024, 4096, null, null, 1, null) == 0


def test_plain_c_client(L, tmp_path):
    """The header is C (not only C++): a C99 program includes it, links
    libcsa.so and runs the host-side checks (no GPU needed)."""
    import shutil
    import subprocess
    from long_context_compressed_02_b200 import LIB_PATH
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cuda_inc = "/usr/local/cuda/include"
    src = os.path.join(ROOT, "tests", "abi_c", "check_abi.c")
    exe = str(tmp_path / "check_abi")
    lib_dir = os.path.dirname(LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                        src, "-o", exe, LIB_PATH, f"-Wl,-rpath,{lib_dir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and "check_abi: ok" in r.stdout, r.stdout + r.stderr


def test_layer_workspace_is_the_larger_of_the_two(L):
    a = L.csa_index_topk_workspace(16, 1, 262144, 512)
    b = L.csa_fused_attention_workspace(16, 1, 64, 512, 5)
    assert L.csa_workspace_size(16, 1, 262144, 512, 64, 512, 5) == max(a, b)
    assert L.csa_workspace_size(1, 16384, 4096, 512, 64, 512, 1) == L.csa_index_topk_workspace(1, 16384, 4096, 512)
    L.csa_compress(None, None, None, None, None, 64, 7, 4, 1, 0, 0, 0, 10000.0, 1e-6, None, 0, None)
    assert L.csa_get_last_error_string() == L.csa_last_error() != b""


def test_fp4_indexer_host_validation(L):
    p = ctypes.c_void_p(16)
    base = L.csa_index_topk_workspace(2, 1, 4096, 512)
    assert L.csa_index_topk_fp4_workspace(2, 1, 64, 4096, 512) == base + 2 * 64 * 128 + 512
    # cap not a multiple of 4
    st = L.csa_index_topk_fp4(p, p, p, p, p, p, 2, 1, 64, 4095, 4, 512, p, p, 1 << 30, None)
    assert st == 1 and b"multiple of 4" in L.csa_last_error()
    # workspace too small
    st = L.csa_index_topk_fp4(p, p, p, p, p, p, 2, 1, 64, 4096, 4, 512, p, p, 16, None)
    assert st == 3
