"""The five workloads at full size, in the launch configuration the benchmark times (needs a GPU).

The GPU always runs the whole workload in one call, and the fp64 oracle checks every output of it:
every head of the long-context sequence, every (sequence, head) pair of the three packed
workloads, and every (batch entry, head) pair of the decode workload at every one of its 1024
steps.  The oracle runs in groups of heads (or of decode steps) so that its fp64 copies of the
inputs stay within a few GB of host memory.
Tolerance: elementwise |gpu - oracle| <= 1e-2 + 2e-2 |oracle| (bf16 inputs, fp32 state) on o and
the final state.
"""
import numpy as np
import pytest
import torch

import gdn2_workloads as W
import oracle
from test_gpu_parity import check_bf16, np64, TOK, g  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu


def check_heads_in_groups(d, o, ST, heads_per_group, what, cu=None):
    """Every head of every sequence against the oracle, ``heads_per_group`` heads per oracle call.

    Dense: d[name] is [N, T, H, dim]; packed (``cu`` given): [T_total, H, dim]."""
    H = d["q"].shape[-2]
    S0 = d["S0"]
    for h0 in range(0, H, heads_per_group):
        hs = slice(h0, min(H, h0 + heads_per_group))
        x = [np64(d[name][..., hs, :]) for name in TOK]
        o_ref, S_ref = oracle.recurrent(*x, S0=np64(S0[:, hs]), cu_seqlens=cu)
        check_bf16(np64(o[..., hs, :]), o_ref, f"{what} o, heads {h0}..{hs.stop - 1}")
        check_bf16(np64(ST[:, hs]), S_ref, f"{what} S_T, heads {h0}..{hs.stop - 1}")


def test_layer_1p3b_full(g):
    wl = W.WORKLOADS["layer_1p3b"]
    d = W.chunk_inputs(wl, device="cuda", seed=0)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=np64(d["S0"]))
    check_bf16(np64(o), o_ref, "layer_1p3b o")
    check_bf16(np64(ST), S_ref, "layer_1p3b S_T")


def test_long_context_all_heads(g):
    """B=1, H=16, T=65536: all 16 heads of the one sequence over all tokens, 4 heads per oracle call."""
    wl = W.WORKLOADS["long_context"]
    d = W.chunk_inputs(wl, device="cuda", seed=0)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"])
    torch.cuda.synchronize()
    check_heads_in_groups(d, o, ST, 4, "long_context")


@pytest.mark.parametrize("name", ["varlen", "varlen_kda", "varlen_gdn"])
def test_varlen_all_pairs(g, name):
    """32 packed sequences x 32 heads (d_v = 256): every (sequence, head) pair, 2 heads per oracle call."""
    wl = W.WORKLOADS[name]
    d = W.chunk_inputs(wl, device="cuda", seed=0)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"], cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    cu = d["cu_seqlens"].cpu().numpy().astype(np.int64)
    check_heads_in_groups(d, o, ST, 2, name, cu=cu)


def test_decode_1024_steps_all_pairs(g):
    """256 x 16 heads for 1024 steps on the GPU; the oracle follows every (batch, head) pair through
    every step, 32 steps per oracle call, and checks o at every step and the final state."""
    wl = W.WORKLOADS["decode"]
    S = W.decode_state(wl, device="cuda", seed=0)
    S_ref = np64(S)                                                      # [B, H, dk, dv]
    block = 32
    for s0 in range(0, wl.decode_steps, block):
        steps = range(s0, min(wl.decode_steps, s0 + block))
        xs = {n: [] for n in TOK}
        outs = []
        for step in steps:
            t = W.decode_token_inputs(wl, step, device="cuda", seed=0)
            outs.append(g.decode_step(*[t[n] for n in TOK], S=S))
            for n in TOK:
                xs[n].append(t[n])
        torch.cuda.synchronize()
        # the steps of this block as sequences of len(steps) tokens: [B, steps, H, d]
        seq = {n: np64(torch.stack(xs[n], 1)) for n in TOK}
        o_ref, S_ref = oracle.recurrent(*[seq[n] for n in TOK], S0=S_ref)
        check_bf16(np64(torch.stack(outs, 1)), o_ref, f"decode o, steps {s0}..{steps[-1]}")
    check_bf16(np64(S), S_ref, "decode final S")
