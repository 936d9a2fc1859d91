"""The five workloads at full size, in the launch configuration the benchmark times (needs a GPU).

The GPU always runs the whole workload.  The fp64 oracle checks every output
where it finishes in seconds (the 1.3B layer shape), otherwise a seeded sample
of (sequence, head) pairs, all tokens of each; the sample is named in each test.
Tolerance: elementwise |gpu - oracle| <= 1e-2 + 2e-2 |oracle| (bf16 inputs,
fp32 state) on o and the final state.
"""
import numpy as np
import pytest
import torch

import gdn2_workloads as W
import oracle
from test_gpu_parity import check_bf16, np64, TOK, g  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu


def oracle_heads(d, heads, seq_slices, S0):
    """Oracle on selected heads of selected sequences; returns {(n, h): (o [len, dv], S [dk, dv])}."""
    out = {}
    for n, sl in seq_slices:
        x = [np64(d[name][sl][:, heads]) for name in TOK]     # [len, nh, d]
        o, S = oracle.recurrent(*[t[None] for t in x], S0=np64(S0[n][heads])[None])
        for i, h in enumerate(heads):
            out[(n, h)] = (o[0, :, i], S[0, i])
    return out


def test_layer_1p3b_full(g):
    wl = W.WORKLOADS["layer_1p3b"]
    d = W.chunk_inputs(wl, device="cuda", seed=0)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=np64(d["S0"]))
    check_bf16(np64(o), o_ref, "layer_1p3b o")
    check_bf16(np64(ST), S_ref, "layer_1p3b S_T")


def test_long_context_sampled_heads(g):
    """All 16 heads run on the GPU; the oracle checks heads 0, 9 and 15 over all 65536 tokens."""
    wl = W.WORKLOADS["long_context"]
    d = W.chunk_inputs(wl, device="cuda", seed=0)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"])
    torch.cuda.synchronize()
    heads = [0, 9, 15]
    dd = {n: d[n][0] for n in TOK}
    ref = oracle_heads(dd, heads, [(0, slice(0, wl.T))], d["S0"])
    for (n, h), (o_r, S_r) in ref.items():
        check_bf16(np64(o[0, :, h]), o_r, f"long_context o head {h}")
        check_bf16(np64(ST[0, h]), S_r, f"long_context S_T head {h}")


@pytest.mark.parametrize("name", ["varlen", "varlen_kda", "varlen_gdn"])
def test_varlen_sampled(g, name):
    """32 packed sequences x 32 heads on the GPU; the oracle checks the shortest, the longest and
    sequence 5, on heads 0 and 31 (every token of each)."""
    wl = W.WORKLOADS[name]
    d = W.chunk_inputs(wl, device="cuda", seed=0)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"], cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    lens = d["lengths"]
    cu = np.concatenate([[0], np.cumsum(lens)])
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 5})
    heads = [0, 31]
    ref = oracle_heads(d, heads, [(n, slice(int(cu[n]), int(cu[n + 1]))) for n in seqs], d["S0"])
    for (n, h), (o_r, S_r) in ref.items():
        check_bf16(np64(o[int(cu[n]):int(cu[n + 1]), h]), o_r, f"{name} o seq {n} head {h}")
        check_bf16(np64(ST[n, h]), S_r, f"{name} S_T seq {n} head {h}")


def test_decode_1024_steps_sampled(g):
    """256 x 16 heads for 1024 steps on the GPU; the oracle follows 24 seeded (batch, head) pairs."""
    wl = W.WORKLOADS["decode"]
    S = W.decode_state(wl, device="cuda", seed=0)
    rng = np.random.default_rng(0)
    picks = [(int(b), int(h)) for b, h in zip(rng.integers(0, wl.B, 24), rng.integers(0, wl.H, 24))]
    S_ref = np.stack([np64(S[b, h]) for b, h in picks])[:, None]            # [24, 1, dk, dv]
    xs = {n: [] for n in TOK}
    outs = []
    for step in range(wl.decode_steps):
        t = W.decode_token_inputs(wl, step, device="cuda", seed=0)
        o = g.decode_step(*[t[n] for n in TOK], S=S)
        for n in TOK:
            xs[n].append(torch.stack([t[n][b, h] for b, h in picks]))
        outs.append(torch.stack([o[b, h] for b, h in picks]))
    torch.cuda.synchronize()
    seq = {n: np64(torch.stack(xs[n], 1))[:, :, None] for n in TOK}   # [24, steps, 1, d]
    o_ref, S_fin = oracle.recurrent(*[seq[n] for n in TOK], S0=S_ref)
    check_bf16(np64(torch.stack(outs, 1)), o_ref[:, :, 0], "decode o")
    check_bf16(np.stack([np64(S[b, h]) for b, h in picks]), S_fin[:, 0], "decode S")
