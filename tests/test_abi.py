"""The C-ABI library loads and exports every symbol its headers declare (CPU only).

No compute call is made here: only argument combinations that the library
rejects on the host, before any launch or allocation, are passed.
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


def bwd(L, ptrs=None, B=1, T=64, H=1, dk=64, dv=64, cu=None, dtype=gdn2.GDN2_BF16):
    p = ptrs or [FAKE] * 16
    return L.gdn2_chunk_bwd(*p, B, T, H, dk, dv, cu, dtype, None)


# argument order: q k v alpha b w S0 dO dS_T | dq dk dv dalpha db dw dS0
BWD_REQUIRED = [0, 1, 2, 3, 4, 5, 7, 9, 10, 11, 12, 13, 14]
BWD_OPTIONAL = [6, 8, 15]


def test_bwd_validation(L):
    before = L.gdn2_launch_count()
    for i in BWD_REQUIRED:
        p = [FAKE] * 16
        p[i] = None
        assert bwd(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
        p[i] = MIS
        assert bwd(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    for i in BWD_OPTIONAL:  # S0, dS_T and dS0 may be NULL, but not misaligned
        p = [FAKE] * 16
        p[i] = MIS
        assert bwd(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    assert bwd(L, B=-1) == gdn2.GDN2_ERR_INVALID_ARG
    assert bwd(L, T=-1) == gdn2.GDN2_ERR_INVALID_ARG
    assert bwd(L, H=0) == gdn2.GDN2_ERR_INVALID_ARG
    assert bwd(L, dtype=3) == gdn2.GDN2_ERR_INVALID_ARG
    assert bwd(L, dk=96) == gdn2.GDN2_ERR_UNSUPPORTED
    assert bwd(L, dv=32) == gdn2.GDN2_ERR_UNSUPPORTED
    assert bwd(L, B=1 << 30, T=1 << 30, H=1 << 20) == gdn2.GDN2_ERR_INVALID_ARG
    assert bwd(L, B=0) == gdn2.GDN2_OK
    assert L.gdn2_launch_count() == before


def test_bwd_workspace_bytes(L):
    # the key-side accumulator (4 fp32 per token, head and key row), d_t (fp32), checkpoints of every
    # tile's state every 64 tokens, and per (sequence, head) a scratch of the 16 states before the
    # 4-token segments of one 64-token group: 0.54 GB on the 1.3B layer
    n = L.gdn2_chunk_bwd_workspace_bytes(4, 2048, 16, 128, 128, 0)
    slots = 4 * 2048 // 64 + 4 + 1
    expect = 4 * 2048 * 16 * 128 * 16 + 4 * 2048 * 16 * 128 * 4 + slots * 16 * 128 * 128 * 4 + 4 * 16 * 16 * 128 * 128 * 4
    assert expect <= n < expect + 3 * 256
    assert n < 0.6e9
    assert L.gdn2_chunk_bwd_workspace_bytes(4, 2048, 16, 96, 128, 0) == 0
    assert L.gdn2_chunk_bwd_workspace_bytes(0, 2048, 16, 128, 128, 0) == 0


def prologue(L, ptrs=None, B=1, T=64, H=1, dk=64, dv=64, K=4, cu=None, dtype=gdn2.GDN2_BF16):
    p = ptrs or [FAKE] * 15
    return L.gdn2_block_prologue(*p, B, T, H, dk, dv, K, cu, dtype, None)


def test_block_prologue_validation(L):
    before = L.gdn2_launch_count()
    for i in range(15):
        p = [FAKE] * 15
        p[i] = None
        assert prologue(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    for i in list(range(6)) + list(range(9, 15)):  # token tensors: 16-byte alignment
        p = [FAKE] * 15
        p[i] = MIS
        assert prologue(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    for i in range(6, 9):  # convolution weights: 4-byte alignment is enough
        p = [FAKE] * 15
        p[i] = ctypes.c_void_p(0x10002)
        assert prologue(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    assert prologue(L, K=0) == gdn2.GDN2_ERR_UNSUPPORTED
    assert prologue(L, K=5) == gdn2.GDN2_ERR_UNSUPPORTED
    assert prologue(L, dk=256) == gdn2.GDN2_ERR_UNSUPPORTED
    assert prologue(L, H=0) == gdn2.GDN2_ERR_INVALID_ARG
    assert prologue(L, dtype=9) == gdn2.GDN2_ERR_INVALID_ARG
    assert prologue(L, B=0) == gdn2.GDN2_OK
    assert L.gdn2_launch_count() == before


def epilogue(L, ptrs=None, tokens=64, H=1, dv=64, dtype=gdn2.GDN2_BF16):
    p = ptrs or [FAKE] * 4
    return L.gdn2_block_epilogue(*p, tokens, H, dv, dtype, None)


def test_block_epilogue_validation(L):
    before = L.gdn2_launch_count()
    for i in range(4):
        p = [FAKE] * 4
        p[i] = None
        assert epilogue(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    for i in (0, 1, 3):
        p = [FAKE] * 4
        p[i] = MIS
        assert epilogue(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    assert epilogue(L, tokens=-1) == gdn2.GDN2_ERR_INVALID_ARG
    assert epilogue(L, dv=32) == gdn2.GDN2_ERR_UNSUPPORTED
    assert epilogue(L, tokens=0) == gdn2.GDN2_OK
    assert L.gdn2_launch_count() == before


def test_chunk_workspace_layout(L):
    """The tensor-core path's workspace (host arithmetic only; 148 SMs when no GPU is present)."""
    record = 32768 + 16384 + 16384 + 8192 + 512  # M, N, Q, P tiles in bf16 and e^{g_C} in fp32

    def counters(records):  # the WY kernel's 256 bytes of counters and one int32 ready flag per record
        return (256 + 4 * records + 255) // 256 * 256

    # 1.3B layer: 2048 (chunk, head) records; one walk per head, no scan buffers (the state pass forms
    # U = w * v itself)
    assert L.gdn2_chunk_fwd_workspace_bytes(4, 2048, 16, 128, 128, 64, 0, gdn2.GDN2_BF16) == 2048 * record + counters(2048)
    # long context (1 x 65536 tokens, 16 heads): the two-level scan adds, per head, S - 1 segment maps
    # A_j (128 x 128) and B_j (128 x d_v) and S entry states, all fp32: 64 KiB x (3 S - 2)
    n = L.gdn2_chunk_fwd_workspace_bytes(1, 65536, 16, 128, 128, 64, 0, gdn2.GDN2_BF16)
    extra = n - 16384 * record - counters(16384)
    assert extra > 0 and extra % (16 * 65536) == 0 and (extra // (16 * 65536) + 2) % 3 == 0
    assert (extra // (16 * 65536) + 2) // 3 >= 2
    # fp32 runs the SIMT kernel, which needs no workspace; bf16 with d_k = 64 runs the tensor-core
    # path with the same 128-channel records
    assert L.gdn2_chunk_fwd_workspace_bytes(4, 2048, 16, 128, 128, 64, 0, gdn2.GDN2_F32) == 0
    assert L.gdn2_chunk_fwd_workspace_bytes(4, 2048, 16, 64, 128, 64, 0, gdn2.GDN2_BF16) == 2048 * record + counters(2048)


def recurrent(L, ptrs=None, B=1, T=64, H=1, dk=64, dv=64, cu=None, erase=gdn2.GDN2_ERASE_R2, dtype=gdn2.GDN2_BF16):
    p = ptrs or [FAKE] * 9
    return L.gdn2_recurrent_fwd(*p, B, T, H, dk, dv, cu, erase, dtype, None)


def test_recurrent_validation(L):
    before = L.gdn2_launch_count()
    assert recurrent(L, erase=2) == gdn2.GDN2_ERR_INVALID_ARG
    assert recurrent(L, erase=-1) == gdn2.GDN2_ERR_INVALID_ARG
    assert recurrent(L, dk=96) == gdn2.GDN2_ERR_UNSUPPORTED
    assert recurrent(L, dv=32) == gdn2.GDN2_ERR_UNSUPPORTED
    assert recurrent(L, dtype=7) == gdn2.GDN2_ERR_INVALID_ARG
    assert recurrent(L, B=-1) == gdn2.GDN2_ERR_INVALID_ARG
    for i in range(9):
        if i in (6, 8):  # S0, S_T may be NULL
            continue
        p = [FAKE] * 9
        p[i] = None
        assert recurrent(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
        p[i] = MIS
        assert recurrent(L, p) == gdn2.GDN2_ERR_INVALID_ARG, i
    assert recurrent(L, [None] * 9, B=0, T=0) == gdn2.GDN2_OK
    assert L.gdn2_launch_count() == before



def plan(L, B, T, H, dk=128, dv=128, packed=0, sms=148, dtype=gdn2.GDN2_BF16):
    p = gdn2.ChunkPlan()
    st = L.gdn2_chunk_fwd_plan(B, T, H, dk, dv, 64, packed, dtype, sms, ctypes.byref(p))
    return st, {name: getattr(p, name) for name, _ in gdn2.ChunkPlan._fields_}


def test_chunk_fwd_plan(L):
    """The launch plan of the tensor-core path (host arithmetic only; nothing is launched)."""
    before = L.gdn2_launch_count()
    # 1.3B layer on 148 SMs: 2048 records over 296 persistent WY CTAs; 64 whole-sequence walks leave
    # 84 SMs, so the CTAs on 64 SMs stop claiming at records - floor(2 (148 - 64) 32 x 1.9 / 9)
    st, p = plan(L, 4, 2048, 16)
    assert st == gdn2.GDN2_OK
    assert (p["records"], p["wy_ctas"], p["state_ctas"], p["segments"], p["launches"]) == (2048, 296, 64, 1, 2)
    assert p["handover_sms"] == 64 and p["order"] == 2
    assert p["handover_at"] == 2048 - int(2 * 84 * 32 * 1.9 / 9)
    assert p["workspace_bytes"] == L.gdn2_chunk_fwd_workspace_bytes(4, 2048, 16, 128, 128, 64, 0, gdn2.GDN2_BF16)
    # fewer SMs leave fewer for the rest of the factorisation: the hand-over comes later
    st, p100 = plan(L, 4, 2048, 16, sms=100)
    assert p100["wy_ctas"] == 200 and p100["handover_at"] == 2048 - int(2 * 36 * 32 * 1.9 / 9)
    # walks that fill the GPU: no hand-over, last chunk first
    st, p = plan(L, 64, 2048, 16)
    assert (p["state_ctas"], p["handover_sms"], p["handover_at"], p["order"]) == (1024, 0, 32768, 1)
    # d_v = 256: two 128-column walks per (sequence, head)
    st, p = plan(L, 4, 2048, 16, dv=256)
    assert p["state_ctas"] == 128 and p["handover_sms"] == 128
    # one long sequence: the two-level scan (summaries, chain, walks), no hand-over
    st, p = plan(L, 1, 65536, 16)
    assert p["segments"] > 1 and p["segments"] * p["segment_chunks"] >= 1024 > (p["segments"] - 1) * p["segment_chunks"]
    assert p["segment_chunks"] >= 16 and p["launches"] == 4 and p["handover_sms"] == 0 and p["order"] == 1
    assert p["state_ctas"] == 16 * (p["segments"] - 1) * 2
    # a packed batch: chunk offsets first, records in record order, no hand-over
    st, p = plan(L, 32, 156118, 32, dv=256, packed=1)
    assert (p["launches"], p["order"], p["handover_sms"]) == (3, 0, 0)
    assert p["records"] == ((156118 + 63 * 32) // 64) * 32 and p["state_ctas"] == 32 * 32 * 2
    # a single record: a hand-over from the start
    st, p = plan(L, 1, 64, 1)
    assert (p["records"], p["wy_ctas"], p["handover_sms"], p["handover_at"]) == (1, 1, 1, 0)
    # no token: no WY launch
    st, p = plan(L, 2, 0, 4)
    assert (p["wy_ctas"], p["launches"]) == (0, 1)
    # not the tensor-core path, or bad arguments
    assert plan(L, 4, 2048, 16, dtype=gdn2.GDN2_F32)[0] == gdn2.GDN2_ERR_UNSUPPORTED
    st, p = plan(L, 4, 2048, 16, dv=64)  # d_v = 64: one 128-column walk per (sequence, head), half of it zero
    assert st == gdn2.GDN2_OK and p["state_ctas"] == 64
    assert plan(L, 4, 2048, 16, dk=96)[0] == gdn2.GDN2_ERR_UNSUPPORTED
    assert plan(L, -1, 2048, 16)[0] == gdn2.GDN2_ERR_INVALID_ARG
    assert plan(L, 4, 2048, 16, sms=-1)[0] == gdn2.GDN2_ERR_INVALID_ARG
    assert L.gdn2_chunk_fwd_plan(4, 2048, 16, 128, 128, 64, 0, gdn2.GDN2_BF16, 148, None) == gdn2.GDN2_ERR_INVALID_ARG
    # the binding returns the same numbers
    assert gdn2.chunk_fwd_plan(4, 2048, 16, 128, 128, sms=148)["handover_at"] == 2048 - int(2 * 84 * 32 * 1.9 / 9)
    assert L.gdn2_launch_count() == before
