"""The C-ABI library loads without a GPU, exports every symbol ``include/*.h``
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

from paged_kv_cache_454_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")


def declared_symbols():
    names = set()
    for f in sorted(os.listdir(INCLUDE)):
        if f.endswith(".h"):
            text = open(os.path.join(INCLUDE, f)).read()
            names |= set(re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    return _abi.load()


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("pa_reshape_and_cache", "pa_copy_blocks", "pa_decode", "pa_decode_workspace_size",
              "pa_chunked_prefill", "pa_gather_kv", "pa_get_device_error", "pa_kvm_create",
              "pa_kvm_add_sequence", "pa_kvm_append_tokens", "pa_kvm_batch"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in _abi.SIGNATURES, f"binding lacks a signature for {name}"
    # and nothing else is bound that the header does not declare
    assert set(_abi.SIGNATURES) == set(declared_symbols())


def test_status_strings_and_version(lib):
    assert lib.pa_abi_version() == 1
    assert lib.pa_status_string(0) == b"PA_OK"
    assert b"WORKSPACE" in lib.pa_status_string(_abi.PA_ERR_WORKSPACE)


def pool(nb=8, hkv=2, bs=16, d=128):
    return _abi.PoolDesc(nb, hkv, bs, d)


def test_workspace_size_is_monotone(lib):
    a = lib.pa_decode_workspace_size(4, 8, pool(), 16)
    b = lib.pa_decode_workspace_size(4, 8, pool(), 64)
    c = lib.pa_decode_workspace_size(8, 8, pool(), 64)
    assert 0 < a < b < c
    # partitions of 128 tokens need more room than 1024-token ones
    assert (lib.pa_decode_workspace_size_ex(4, 8, pool(), 64, 128) >
            lib.pa_decode_workspace_size_ex(4, 8, pool(), 64, 1024))
    assert lib.pa_decode_workspace_size(4, 8, pool(), 0) == 0


def test_host_argument_checks(lib):
    fake = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: calls fail first
    # unsupported block size / head dim
    assert lib.pa_reshape_and_cache(fake, fake, 256, fake, fake, pool(bs=32), fake, 4,
                                    None) == _abi.PA_ERR_UNSUPPORTED
    assert lib.pa_reshape_and_cache(fake, fake, 256, fake, fake, pool(d=96), fake, 4,
                                    None) == _abi.PA_ERR_UNSUPPORTED
    # null pointers, negative counts, misaligned strides
    assert lib.pa_reshape_and_cache(None, fake, 256, fake, fake, pool(), fake, 4,
                                    None) == _abi.PA_ERR_ARG
    assert lib.pa_reshape_and_cache(fake, fake, 256, fake, fake, pool(), fake, -1,
                                    None) == _abi.PA_ERR_ARG
    assert lib.pa_reshape_and_cache(fake, fake, 250, fake, fake, pool(), fake, 4,
                                    None) == _abi.PA_ERR_ARG
    # zero tokens is a no-op
    assert lib.pa_reshape_and_cache(None, None, 0, None, None, pool(), None, 0, None) == 0
    # group size not a whole number
    assert lib.pa_decode(fake, 384, fake, fake, pool(hkv=2), fake, 4, fake, 1, 3, 1.0, fake, None,
                         fake, 1 << 20, None) == _abi.PA_ERR_SHAPE
    # group size above 16
    assert lib.pa_decode(fake, 34 * 128, fake, fake, pool(hkv=2), fake, 4, fake, 1, 34, 1.0, fake,
                         None, fake, 1 << 20, None) == _abi.PA_ERR_UNSUPPORTED
    # workspace too small
    assert lib.pa_decode(fake, 4 * 128, fake, fake, pool(hkv=2), fake, 4, fake, 1, 4, 1.0, fake,
                         None, fake, 16, None) == _abi.PA_ERR_WORKSPACE
    # partition length not a multiple of 128
    assert lib.pa_decode_ex(fake, 4 * 128, fake, fake, pool(hkv=2), fake, 4, fake, 1, 4, 1.0, fake,
                            None, fake, 1 << 20, 100, 0, None) == _abi.PA_ERR_ARG
    # misaligned q
    assert lib.pa_decode(ctypes.c_void_p(0x10002), 4 * 128, fake, fake, pool(hkv=2), fake, 4, fake,
                         1, 4, 1.0, fake, None, fake, 1 << 20, None) == _abi.PA_ERR_ARG


def _pairs(lst):
    a = np.ascontiguousarray(np.asarray(lst, np.int64).reshape(-1, 2))
    return a, a.ctypes.data_as(ctypes.c_void_p)


def test_copy_blocks_rules_checked_on_host(lib):
    fake = ctypes.c_void_p(0x10000)
    for bad in ([[1, 4], [2, 4]],      # repeated destination
                [[1, 4], [4, 5]],      # destination is also a source
                [[1, 8]],              # outside the 8-block pool
                [[-1, 3]]):
        arr, ptr = _pairs(bad)
        assert lib.pa_copy_blocks(fake, fake, pool(), ptr, arr.shape[0], None) == _abi.PA_ERR_ARG
    assert lib.pa_copy_blocks(fake, fake, pool(), None, 0, None) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    import paged_kv_cache_454_b200 as pa
    kp = torch.zeros((4, 1, 16, 64), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        pa.pa_decode(torch.zeros((1, 1, 64), dtype=torch.bfloat16), kp, kp,
                     torch.zeros((1, 1), dtype=torch.int32), torch.ones(1, dtype=torch.int32), 1.0)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        _abi.load(str(tmp_path / "libpa.so"))


def test_read_probe_host_argument_checks(lib):
    fake = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: calls fail first
    odd = ctypes.c_void_p(0x10004)
    call = lambda **kw: lib.pa_read_probe(
        kw.get("k", fake), kw.get("v", fake), kw.get("pool", pool()), kw.get("tables", fake),
        kw.get("max_blocks", 4), kw.get("lens", fake), kw.get("seqs", 3), kw.get("out", fake),
        kw.get("ctas", 8), None)
    assert call(pool=pool(bs=32)) == _abi.PA_ERR_UNSUPPORTED
    assert call(pool=pool(d=96)) == _abi.PA_ERR_UNSUPPORTED
    assert call(ctas=0) == _abi.PA_ERR_ARG
    assert call(ctas=65536) == _abi.PA_ERR_ARG
    assert call(seqs=-1) == _abi.PA_ERR_ARG
    assert call(seqs=4097) == _abi.PA_ERR_ARG
    assert call(max_blocks=-1) == _abi.PA_ERR_ARG
    assert call(k=None) == _abi.PA_ERR_ARG
    assert call(out=None) == _abi.PA_ERR_ARG
    assert call(tables=None) == _abi.PA_ERR_ARG
    assert call(lens=None) == _abi.PA_ERR_ARG
    assert call(v=odd) == _abi.PA_ERR_ARG
    assert call(out=odd) == _abi.PA_ERR_ARG


@pytest.mark.parametrize("flags", [[], ["-DPA_NO_NVTX"]], ids=["nvtx", "no_nvtx"])
def test_nvtx_range_compiles_in_and_out(tmp_path, flags):
    # the range guard every entry point opens, built with and without NVTX
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no host compiler")
    src = tmp_path / "r.cpp"
    src.write_text('#include "internal.h"\n'
                   'int f() { PA_NVTX_RANGE("pa_test"); return 7; }\n'
                   'int main() { return f() == 7 ? 0 : 1; }\n')
    csrc = os.path.join(ROOT, "paged_kv_cache_454_b200", "csrc")
    exe = tmp_path / "r"
    r = subprocess.run([gxx, "-std=c++17", "-I", csrc, "-I", "/usr/local/cuda/include", *flags,
                        str(src), "-o", str(exe), "-ldl"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0
