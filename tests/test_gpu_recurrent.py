"""gdn2_recurrent_fwd: the token loop on the GPU in both erase orientations, against the fp64 oracle
(needs a GPU).

The pages leave open on which side of the rank-1 erase the key-side gate b sits.  The oracle
implements both readings behind one switch (pinned on the CPU: both reduce to the textbook KDA and
Gated DeltaNet loops, and both equal a brute-force product of per-token transitions); this kernel
implements both, and is compared here element by element with the oracle on the same inputs.
Tolerances as everywhere: fp32 normwise 1e-4; bf16 |gpu - oracle| <= 1e-2 + 2e-2 |oracle|.
"""
import numpy as np
import pytest
import torch

import gdn2_workloads as W
import oracle
from test_gpu_parity import check_bf16, check_f32, np64, TOK, g  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu

ERASE = {"R1": (0, oracle.ERASE_R1), "R2": (1, oracle.ERASE_R2)}


def run(g, wl, erase, seed=0, lengths=None, s0=True):
    d = W.chunk_inputs(wl, device="cuda", seed=seed, lengths=lengths)
    S0 = d["S0"] if s0 else None
    o, ST = g.recurrent_fwd(*[d[n] for n in TOK], S0=S0, cu_seqlens=d["cu_seqlens"], erase=ERASE[erase][0])
    torch.cuda.synchronize()
    cu = None if d["cu_seqlens"] is None else d["cu_seqlens"].cpu().numpy().astype(np.int64)
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=None if S0 is None else np64(S0),
                                    cu_seqlens=cu, orientation=ERASE[erase][1])
    check = check_f32 if wl.dtype == "f32" else check_bf16
    check(np64(o), o_ref, f"{wl.name} {erase} o")
    check(np64(ST), S_ref, f"{wl.name} {erase} S_T")
    return d, o, ST


@pytest.mark.parametrize("erase", ["R1", "R2"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 256), (128, 64)])
def test_fp32_dense(g, erase, dk, dv):
    run(g, W.Workload("rec_f32", B=2, T=150, H=3, dk=dk, dv=dv, dtype="f32"), erase, seed=11)


@pytest.mark.parametrize("erase", ["R1", "R2"])
@pytest.mark.parametrize("variant", ["full", "kda", "gdn"])
def test_bf16_packed_with_empty_sequence(g, erase, variant):
    lengths = [90, 1, 0, 64, 200]
    wl = W.Workload("rec_bf16", B=len(lengths), T=256, H=2, dk=128, dv=128, varlen=True, variant=variant)
    run(g, wl, erase, seed=12, lengths=lengths, s0=False)


def test_orientations_differ_and_r1_matches_chunk_fwd(g):
    """The two readings give different results on the same inputs (so each test above pins its
    own); the R1 token loop and the chunkwise forward agree within the bf16 tolerance."""
    wl = W.Workload("rec_cmp", B=2, T=300, H=2, dk=128, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=13)
    o1, S1 = g.recurrent_fwd(*[d[n] for n in TOK], S0=d["S0"], erase=g.GDN2_ERASE_R1)
    o2, S2 = g.recurrent_fwd(*[d[n] for n in TOK], S0=d["S0"], erase=g.GDN2_ERASE_R2)
    oc, Sc = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"])
    torch.cuda.synchronize()
    assert np.max(np.abs(np64(o1) - np64(o2))) > 1e-2
    check_bf16(np64(oc), np64(o1), "chunk_fwd vs recurrent R1 o")
    check_bf16(np64(Sc), np64(S1), "chunk_fwd vs recurrent R1 S_T")


def test_empty_batch_keeps_initial_state(g):
    wl = W.Workload("rec_empty", B=2, T=0, H=2, dk=64, dv=64, dtype="f32")
    d = W.chunk_inputs(wl, device="cuda", seed=14)
    o, ST = g.recurrent_fwd(*[d[n] for n in TOK], S0=d["S0"], erase=g.GDN2_ERASE_R2)
    torch.cuda.synchronize()
    assert torch.equal(ST, d["S0"])
