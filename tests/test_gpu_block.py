"""Block prologue and epilogue around the mixer on the GPU vs the fp64 oracle (needs a GPU).

Tolerances as for the chunk forward: fp32 normwise max-relative <= 1e-4; bf16 elementwise
|gpu - oracle| <= 1e-2 + 2e-2 |oracle|.  Every call goes through the C ABI.
"""
import ctypes

import numpy as np
import pytest
import torch

import gdn2_workloads as W
import oracle

pytestmark = pytest.mark.gpu

PRE = ("xq", "xk", "xv", "xa", "xb", "xw")
CONV = ("conv_q", "conv_k", "conv_v")
TOK = ("q", "k", "v", "alpha", "b", "w")


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_131_b200 as gdn2
    gdn2.lib()
    return gdn2


def np64(t):
    return t.double().cpu().numpy()


def check(gpu, ref, dtype, what):
    if dtype == "f32":
        err = np.max(np.abs(gpu - ref)) / max(np.max(np.abs(ref)), 1e-30)
        assert err <= 1e-4, f"{what}: normwise max-relative error {err:.3e}"
    else:
        bad = np.abs(gpu - ref) > 1e-2 + 2e-2 * np.abs(ref)
        assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} out of tolerance"


def prologue_case(g, wl, K, seed, lengths=None):
    d = W.block_inputs(wl, device="cuda", seed=seed, conv_len=K, lengths=lengths)
    outs = g.block_prologue(*[d[n] for n in PRE], *[d[n] for n in CONV], cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    cu = None if d["cu_seqlens"] is None else d["cu_seqlens"].cpu().numpy()
    refs = oracle.block_prologue(*[np64(d[n]) for n in PRE], *[np64(d[n]) for n in CONV], cu_seqlens=cu)
    for name, out, ref in zip(TOK, outs, refs):
        check(np64(out), ref, wl.dtype, f"prologue {name}")
    return d, outs


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [1, 3, 4])
def test_prologue_dense(g, dtype, K):
    wl = W.Workload("block_dense", B=2, T=150, H=3, dk=128, dv=256, dtype=dtype)
    prologue_case(g, wl, K, seed=51)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 256)])
def test_prologue_packed_sequences_restart_the_convolution(g, dk, dv):
    lengths = [1, 70, 64, 0, 131, 2]
    wl = W.Workload("block_packed", B=len(lengths), T=256, H=2, dk=dk, dv=dv, varlen=True)
    prologue_case(g, wl, 4, seed=52, lengths=lengths)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dv", [64, 128, 256])
def test_epilogue(g, dtype, dv):
    wl = W.Workload("block_out", B=3, T=77, H=4, dk=128, dv=dv, dtype=dtype)
    d = W.block_inputs(wl, device="cuda", seed=53)
    o = d["xv"].clone()  # any [.., H, d_v] tensor serves as the mixer output here
    y = g.block_epilogue(o, d["z"], d["norm_weight"])
    o2 = o.clone()
    g.block_epilogue(o2, d["z"], d["norm_weight"], y=o2)  # y may alias o
    torch.cuda.synchronize()
    ref = oracle.block_epilogue(np64(o), np64(d["z"]), np64(d["norm_weight"]))
    check(np64(y), ref, dtype, "epilogue")
    assert torch.equal(y, o2)


def test_block_chain_matches_oracle_chain(g):
    """prologue -> chunk_fwd -> epilogue on the GPU against the same chain of oracle functions."""
    wl = W.Workload("block_chain", B=2, T=200, H=2, dk=128, dv=128)
    d = W.block_inputs(wl, device="cuda", seed=54)
    q, k, v, alpha, b, w = g.block_prologue(*[d[n] for n in PRE], *[d[n] for n in CONV])
    o, ST = g.chunk_fwd(q, k, v, alpha, b, w, S0=d["S0"])
    y = g.block_epilogue(o, d["z"], d["norm_weight"])
    torch.cuda.synchronize()
    # the oracle chain starts from the GPU prologue's rounded outputs, as the chunk oracle does
    o_ref, S_ref = oracle.recurrent(*[np64(t) for t in (q, k, v, alpha, b, w)], S0=np64(d["S0"]))
    check(np64(o), o_ref, "bf16", "chain o")
    check(ST.cpu().double().numpy(), S_ref, "bf16", "chain S_T")
    y_ref = oracle.block_epilogue(np64(o), np64(d["z"]), np64(d["norm_weight"]))
    check(np64(y), y_ref, "bf16", "chain y")


def test_prologue_guard_bands_untouched(g):
    wl = W.Workload("block_guard", B=1, T=90, H=2, dk=128, dv=128)
    d = W.block_inputs(wl, device="cuda", seed=55)
    pad, canary = 4096, -777.0
    n = 90 * 2 * 128
    bufs = [torch.full((2 * pad + n,), canary, device="cuda", dtype=torch.bfloat16) for _ in range(6)]
    outs = [buf[pad:pad + n].view(1, 90, 2, 128) for buf in bufs]
    L = g.lib()
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.gdn2_block_prologue(*[ptr(d[x]) for x in PRE], *[ptr(d[x]) for x in CONV], *[ptr(t) for t in outs],
                               1, 90, 2, 128, 128, 4, None, g.GDN2_BF16, stream)
    torch.cuda.synchronize()
    assert st == g.GDN2_OK
    for buf in bufs:
        assert torch.all(buf[:pad] == canary) and torch.all(buf[-pad:] == canary)


def test_full_layer_shape_in_the_benchmark_launch(g):
    """The 1.3B-layer shape (4 x 2048 tokens, 16 heads, d = 128, 4 taps), launched as the benchmark
    launches it (one wave of long token runs), against the oracle on every output element."""
    wl = W.WORKLOADS["layer_1p3b"]
    d, outs = prologue_case(g, wl, 4, seed=0)
    y = g.block_epilogue(d["xv"], d["z"], d["norm_weight"])
    torch.cuda.synchronize()
    ref = oracle.block_epilogue(np64(d["xv"]), np64(d["z"]), np64(d["norm_weight"]))
    check(np64(y), ref, wl.dtype, "epilogue")
