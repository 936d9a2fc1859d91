"""Backward of the recurrence on the GPU vs the fp64 oracle's gradient (needs a GPU).

Every call goes through the C ABI (``gdn2_chunk_bwd``).  Tolerances, per gradient tensor y
(oracle) and x (GPU):

* fp32: normwise max|x - y| / max|y| <= 1e-4, as for the forward;
* bf16: |x - y| <= 2^-7 |y| + 1e-3 max|y|.  The first term is two roundings to bf16 (the
  inputs the oracle reads are the rounded ones, so only the result's rounding and the fp32
  arithmetic remain); the second bounds the fp32 accumulation along the sequence relative to the
  tensor's scale, where elements near zero carry the cancellation of much larger terms.
"""
import numpy as np
import pytest
import torch

import gdn2_workloads as W
import oracle

pytestmark = pytest.mark.gpu

TOK = ("q", "k", "v", "alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dalpha", "db", "dw", "dS0")


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
    scale = max(np.max(np.abs(ref)), 1e-30)
    if dtype == "f32":
        err = np.max(np.abs(gpu - ref)) / scale
        assert err <= 1e-4, f"{what}: normwise max-relative error {err:.3e}"
    else:
        bad = np.abs(gpu - ref) > 2.0 ** -7 * np.abs(ref) + 1e-3 * scale
        assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} out of tolerance"


def upstream(shape_o, shape_S, device, seed):
    gen = torch.Generator(device="cpu").manual_seed(seed)
    dO = torch.randn(shape_o, generator=gen)
    dST = torch.randn(shape_S, generator=gen) * 0.1
    return dO.to(device), dST.to(device)


def run_case(g, wl, seed, lengths=None, with_S0=True, with_dST=True):
    d = W.chunk_inputs(wl, device="cuda", seed=seed, lengths=lengths) if lengths is not None else \
        W.chunk_inputs(wl, device="cuda", seed=seed)
    N = d["S0"].shape[0]
    dO, dST = upstream(d["q"].shape[:-1] + (wl.dv,), (N, wl.H, wl.dk, wl.dv), "cuda", seed + 1000)
    dO = dO.to(d["q"].dtype)
    S0 = d["S0"] if with_S0 else None
    dS_T = dST if with_dST else None
    out = g.chunk_bwd(*[d[n] for n in TOK], dO, S0=S0, dS_T=dS_T, cu_seqlens=d.get("cu_seqlens"))
    torch.cuda.synchronize()
    cu = d.get("cu_seqlens")
    refs = oracle.recurrent_bwd(*[np64(d[n]) for n in TOK], np64(dO), S0=None if S0 is None else np64(S0),
                                dST=None if dS_T is None else np64(dS_T),
                                cu_seqlens=None if cu is None else cu.cpu().numpy())
    for name, x, y in zip(GRADS, out, refs):
        check(np64(x), y, wl.dtype, name)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 256), (128, 128), (128, 256)])
def test_fp32_dense(g, dk, dv):
    wl = W.Workload("bwd_f32", B=2, T=37, H=2, dk=dk, dv=dv, dtype="f32")
    run_case(g, wl, seed=61)


def test_bf16_dense(g):
    wl = W.Workload("bwd_bf16", B=2, T=200, H=3, dk=128, dv=128)
    run_case(g, wl, seed=62)


def test_packed_sequences(g):
    lengths = [1, 17, 0, 40, 8]
    wl = W.Workload("bwd_packed", B=len(lengths), T=64, H=2, dk=128, dv=128, dtype="f32", varlen=True)
    run_case(g, wl, seed=63, lengths=lengths)


def test_without_initial_state_or_state_gradient(g):
    wl = W.Workload("bwd_plain", B=1, T=24, H=2, dk=64, dv=128, dtype="f32")
    run_case(g, wl, seed=64, with_S0=False, with_dST=False)


def test_full_layer_shape_sampled_heads(g):
    """The 1.3B-layer shape (4 x 2048 tokens, 16 heads, d = 128, bf16) in the benchmark's launch;
    the oracle checks three (sequence, head) pairs in full."""
    wl = W.WORKLOADS["layer_1p3b"]
    d = W.chunk_inputs(wl, device="cuda", seed=0)
    dO, dST = upstream(d["q"].shape[:-1] + (wl.dv,), (wl.B, wl.H, wl.dk, wl.dv), "cuda", 1000)
    dO = dO.to(torch.bfloat16)
    out = g.chunk_bwd(*[d[n] for n in TOK], dO, S0=d["S0"], dS_T=dST)
    torch.cuda.synchronize()
    for n, h in ((0, 0), (1, 9), (3, 15)):
        sl = lambda t: np64(t[n:n + 1, :, h:h + 1])
        refs = oracle.recurrent_bwd(*[sl(d[x]) for x in TOK], sl(dO), S0=np64(d["S0"][n:n + 1, h:h + 1]),
                                    dST=np64(dST[n:n + 1, h:h + 1]))
        for name, x, y in zip(GRADS, out, refs):
            xs = np64(x[n:n + 1, h:h + 1]) if name == "dS0" else sl(x)
            check(xs, y, "bf16", f"{name} (sequence {n}, head {h})")


def test_empty_batch_and_zero_length(g):
    wl = W.Workload("bwd_zero", B=2, T=0, H=2, dk=128, dv=128, dtype="f32")
    z = lambda *s: torch.zeros(*s, device="cuda")
    q = z(2, 0, 2, 128)
    dST = torch.randn(2, 2, 128, 128, device="cuda")
    out = g.chunk_bwd(q, q, q, q, q, q, q, S0=None, dS_T=dST)
    torch.cuda.synchronize()
    assert torch.equal(out[-1], dST)  # no tokens: dS0 = dS_T
