"""The C-ABI library loads and exports every symbol its headers declare (CPU only).

No compute call is made here: only argument combinations that the library
rejects on the host, before any CUDA call, are passed.
"""
import ctypes
import glob
import os
import re

import pytest

import gated_delta_rule_131_b200 as gdn2
from gated_delta_rule_131_b200 import build as gbuild

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdn2.lib()


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        names += re.findall(r"GDN2_API\s+[\w\s\*]+?\b(gdn2_\w+)\s*\(", txt)
    return sorted(set(names))


def test_headers_declare_the_entry_points():
    names = declared_symbols()
    assert "gdn2_chunk_fwd" in names and "gdn2_decode_step" in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_symbols():
        assert hasattr(L, name), f"{name} declared in include/ but not exported"


def test_library_is_built_for_sm100a():
    assert "arch=compute_100a,code=sm_100a" in " ".join(gbuild.NVCC_FLAGS)


def test_status_strings(L):
    for s in range(5):
        assert L.gdn2_status_string(s).decode().startswith("GDN2")
    assert L.gdn2_status_string(99).decode()


# A plausible, 16-byte aligned address; never dereferenced because every call below is rejected first.
FAKE = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10004)


def chunk(L, ptrs=None, B=1, T=64, H=1, dk=64, dv=64, chunk=64, cu=None, dtype=gdn2.GDN2_BF16):
    p = ptrs or [FAKE] * 9
    return L.gdn2_chunk_fwd(*p, B, T, H, dk, dv, chunk, cu, dtype, None)


def test_chunk_null_token_pointers_allowed_without_tokens(L):
    p = [None] * 7 + [None, None]
    assert chunk(L, p, B=0, T=0) == gdn2.GDN2_OK


def test_chunk_rejects_null_pointers(L):
    for i in range(6):
        p = [FAKE] * 9
        p[i] = None
        assert chunk(L, p) == gdn2.GDN2_ERR_INVALID_ARG
    p = [FAKE] * 9
    p[7] = None  # o
    assert chunk(L, p) == gdn2.GDN2_ERR_INVALID_ARG


def test_chunk_rejects_misaligned(L):
    for i in range(9):
        p = [FAKE] * 9
        p[i] = MIS
        assert chunk(L, p) == gdn2.GDN2_ERR_INVALID_ARG


def test_chunk_rejects_bad_sizes(L):
    assert chunk(L, B=-1) == gdn2.GDN2_ERR_INVALID_ARG
    assert chunk(L, T=-5) == gdn2.GDN2_ERR_INVALID_ARG
    assert chunk(L, H=0) == gdn2.GDN2_ERR_INVALID_ARG
    assert chunk(L, dtype=7) == gdn2.GDN2_ERR_INVALID_ARG
    assert chunk(L, B=1 << 30, T=1 << 30, H=1 << 20) == gdn2.GDN2_ERR_INVALID_ARG


def test_chunk_unsupported_shapes(L):
    assert chunk(L, dk=96) == gdn2.GDN2_ERR_UNSUPPORTED
    assert chunk(L, dv=32) == gdn2.GDN2_ERR_UNSUPPORTED
    assert chunk(L, chunk=32) == gdn2.GDN2_ERR_UNSUPPORTED


def test_chunk_empty_batch_is_a_no_op(L):
    before = L.gdn2_launch_count()
    assert chunk(L, B=0) == gdn2.GDN2_OK
    assert L.gdn2_launch_count() == before


def decode(L, ptrs=None, B=1, H=1, dk=64, dv=64, dtype=gdn2.GDN2_BF16):
    p = ptrs or [FAKE] * 8
    return L.gdn2_decode_step(*p, B, H, dk, dv, dtype, None)


def test_decode_validation(L):
    for i in range(8):
        p = [FAKE] * 8
        p[i] = None
        assert decode(L, p) == gdn2.GDN2_ERR_INVALID_ARG
        p[i] = MIS
        assert decode(L, p) == gdn2.GDN2_ERR_INVALID_ARG
    assert decode(L, B=-1) == gdn2.GDN2_ERR_INVALID_ARG
    assert decode(L, H=0) == gdn2.GDN2_ERR_INVALID_ARG
    assert decode(L, dk=32) == gdn2.GDN2_ERR_UNSUPPORTED
    assert decode(L, dv=512) == gdn2.GDN2_ERR_UNSUPPORTED
    assert decode(L, B=0) == gdn2.GDN2_OK


def test_python_binding_has_no_cpu_path():
    import torch
    x = torch.zeros(1, 64, 1, 64)
    with pytest.raises((ValueError, RuntimeError)):
        gdn2.chunk_fwd(x, x, x, x, x, x)
