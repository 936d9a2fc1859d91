"""gdn2_chunk_fwd_noalloc: the chunk forward for callers that cannot allocate device memory.

Some callers reserve all of their device memory up front, or run this library under a memory
manager of their own, and so cannot let it call cudaMalloc or a stream-ordered allocator.  This
entry point runs the same kernels over one fixed device array compiled into the library.  The
tests check, through the C ABI, that it gives bit for bit the output of gdn2_chunk_fwd on two calls
in a row, for a dense batch, a packed batch and a long sequence that takes the two-level state
scan (whose segment maps and entry states then also live in the fixed array).

Collected last on purpose: it must pass alone and after every other test (the fixed workspace
then still holds whatever earlier calls left in it, which must not matter).
"""
import ctypes
import re
import os

import pytest
import torch

import gated_delta_rule_131_b200 as gdn2
import gdn2_workloads as W
from gated_delta_rule_131_b200 import build as gbuild

TOK = ("q", "k", "v", "alpha", "b", "w")
ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def test_limit_matches_header():
    txt = open(os.path.join(ROOT, "include", "gdn2.h")).read()
    m = re.search(r"#define GDN2_NOALLOC_WORKSPACE_BYTES \((\d+)u << (\d+)\)", txt)
    assert m and int(m.group(1)) << int(m.group(2)) == gdn2.NOALLOC_WORKSPACE_BYTES


def test_oversized_shape_is_rejected_before_any_launch_or_allocation():
    gbuild.build()
    L = gdn2.lib()
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    B, T, H = 64, 2048, 16
    assert gdn2.chunk_fwd_workspace_bytes(B, T, H, 128, 128) > gdn2.NOALLOC_WORKSPACE_BYTES
    st = L.gdn2_chunk_fwd_noalloc(*[fake] * 9, B, T, H, 128, 128, 64, None, gdn2.GDN2_BF16, None)
    assert st == gdn2.GDN2_ERR_UNSUPPORTED


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gdn2.lib()
    return gdn2


def _both_entries_twice(g, wl, seeds, lengths=None):
    ds = [W.chunk_inputs(wl, device="cuda", seed=s, lengths=lengths) for s in seeds]
    fixed = [g.chunk_fwd_noalloc(*[d[n] for n in TOK], S0=d["S0"], cu_seqlens=d["cu_seqlens"]) for d in ds]
    pooled = [g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"], cu_seqlens=d["cu_seqlens"]) for d in ds]
    torch.cuda.synchronize()
    for (on, sn), (op, sp) in zip(fixed, pooled):  # same kernels on the same inputs: identical bits
        assert torch.equal(on, op)
        assert torch.equal(sn, sp)


@pytest.mark.gpu
def test_noalloc_matches_pooled_entry_two_calls_in_a_row(g):
    wl = W.Workload("noalloc", B=2, T=700, H=8, dk=128, dv=128)
    assert g.chunk_fwd_workspace_bytes(wl.B, wl.T, wl.H, wl.dk, wl.dv) <= g.NOALLOC_WORKSPACE_BYTES
    _both_entries_twice(g, wl, (31, 32))


@pytest.mark.gpu
def test_noalloc_matches_pooled_entry_packed(g):
    lengths = [300, 1, 64, 0, 129]
    wl = W.Workload("noalloc_packed", B=len(lengths), T=512, H=4, dk=128, dv=256, varlen=True)
    assert g.chunk_fwd_workspace_bytes(len(lengths), sum(lengths), wl.H, wl.dk, wl.dv,
                                       packed=True) <= g.NOALLOC_WORKSPACE_BYTES
    _both_entries_twice(g, wl, (33, 34), lengths=lengths)


@pytest.mark.gpu
def test_noalloc_matches_pooled_entry_two_level_scan(g):
    """One long sequence and one head: the state walk is cut into segments (two-level scan)."""
    wl = W.Workload("noalloc_scan", B=1, T=4096, H=1, dk=128, dv=128)
    dense = g.chunk_fwd_workspace_bytes(wl.B, wl.T, wl.H, wl.dk, wl.dv)
    packed = g.chunk_fwd_workspace_bytes(wl.B, wl.T, wl.H, wl.dk, wl.dv, packed=True)
    # the same chunk records either way; only a dense batch can take the scan, whose segment maps
    # and entry states (about 0.6 MB here) make its workspace the larger one
    assert dense > packed + 500_000
    assert dense <= g.NOALLOC_WORKSPACE_BYTES
    _both_entries_twice(g, wl, (35, 36))
