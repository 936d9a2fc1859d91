"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a GPU).

Tolerances (written here, applied to o and S_T):
* fp32 inputs:  max|gpu - oracle| / max|oracle| <= 1e-4   (normwise max-relative)
* bf16 inputs, fp32 state: elementwise |gpu - oracle| <= 1e-2 + 2e-2 |oracle|
Every call goes through the C ABI (the ctypes binding in the package).
"""
import numpy as np
import pytest
import torch

import gdn2_workloads as W
import oracle

pytestmark = pytest.mark.gpu

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


def check_f32(gpu, ref, what):
    err = np.max(np.abs(gpu - ref)) / max(np.max(np.abs(ref)), 1e-30)
    assert err <= 1e-4, f"{what}: normwise max-relative error {err:.3e} > 1e-4"


def check_bf16(gpu, ref, what):
    bad = np.abs(gpu - ref) > 1e-2 + 2e-2 * np.abs(ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                             f"first at {tuple(i)}: gpu {gpu[tuple(i)]:.6g} oracle {ref[tuple(i)]:.6g}")


def run_case(g, wl, seed=0, lengths=None, s0=True, check=None):
    d = W.chunk_inputs(wl, device="cuda", seed=seed, lengths=lengths)
    S0 = d["S0"] if s0 else None
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=S0, cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    cu = None if d["cu_seqlens"] is None else d["cu_seqlens"].cpu().numpy().astype(np.int64)
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=None if S0 is None else np64(S0), cu_seqlens=cu)
    check = check or (check_f32 if wl.dtype == "f32" else check_bf16)
    check(np64(o), o_ref, f"{wl.name} o")
    check(ST.cpu().numpy().astype(np.float64), S_ref, f"{wl.name} S_T")
    return d, o, ST


# ------------------------------------------------------------------ the small fp32 workload

def test_oracle_small_fp32(g):
    run_case(g, W.WORKLOADS["oracle_small"])


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 256), (128, 64)])
def test_fp32_ragged_tail(g, dk, dv):
    wl = W.Workload("f32_ragged", B=2, T=200, H=3, dk=dk, dv=dv, dtype="f32")
    run_case(g, wl, seed=3)


# ------------------------------------------------------------------ bf16, several tiles + ragged tail

@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 256), (64, 128)])
def test_bf16_ragged_tail(g, dk, dv):
    wl = W.Workload("bf16_ragged", B=2, T=333, H=4, dk=dk, dv=dv)
    run_case(g, wl, seed=5)


@pytest.mark.parametrize("variant", ["full", "kda", "gdn"])
def test_bf16_varlen_edge_lengths(g, variant):
    lengths = [1, 63, 64, 65, 0, 128, 129, 7, 200]
    wl = W.Workload("varlen_edges", B=len(lengths), T=256, H=2, dk=128, dv=256, varlen=True, variant=variant)
    run_case(g, wl, seed=7, lengths=lengths)


def test_zero_initial_state_and_no_final_state(g):
    wl = W.Workload("nos0", B=1, T=130, H=2, dk=128, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=9)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=None, output_final_state=False)
    assert ST is None
    o_ref, _ = oracle.recurrent(*[np64(d[n]) for n in TOK])
    check_bf16(np64(o), o_ref, "o")


def test_final_state_may_alias_initial_state(g):
    wl = W.Workload("alias", B=2, T=100, H=2, dk=64, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=10)
    S = d["S0"].clone()
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=np64(S))
    g.chunk_fwd(*[d[n] for n in TOK], S0=S, S_T=S)
    torch.cuda.synchronize()
    check_bf16(S.cpu().double().numpy(), S_ref, "aliased S_T")


def test_zero_length(g):
    wl = W.Workload("empty", B=2, T=0, H=2, dk=128, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=11)
    o, ST = g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"])
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(ST, d["S0"])


def test_guard_bands_untouched(g):
    wl = W.Workload("guard", B=1, T=77, H=2, dk=128, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=12)
    pad = 4096
    canary = -12345.0
    o_buf = torch.full((pad * 2 + 77 * 2 * 128,), canary, device="cuda", dtype=torch.bfloat16)
    s_buf = torch.full((pad * 2 + 2 * 128 * 128,), canary, device="cuda", dtype=torch.float32)
    o = o_buf[pad:pad + 77 * 2 * 128].view(1, 77, 2, 128)
    ST = s_buf[pad:pad + 2 * 128 * 128].view(1, 2, 128, 128)
    g.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"], o=o, S_T=ST)
    torch.cuda.synchronize()
    for buf in (o_buf, s_buf):
        assert torch.all(buf[:pad] == canary) and torch.all(buf[-pad:] == canary)
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=np64(d["S0"]))
    check_bf16(np64(o), o_ref, "o")


def test_resume_split_mid_chunk(g):
    wl = W.Workload("resume", B=1, T=300, H=2, dk=128, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=13)
    split = 100
    first = {n: d[n][:, :split].contiguous() for n in TOK}
    second = {n: d[n][:, split:].contiguous() for n in TOK}
    o1, S1 = g.chunk_fwd(*[first[n] for n in TOK], S0=d["S0"])
    o2, S2 = g.chunk_fwd(*[second[n] for n in TOK], S0=S1)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=np64(d["S0"]))
    check_bf16(np64(torch.cat([o1, o2], 1)), o_ref, "o")
    check_bf16(np64(S2), S_ref, "S_T")


def test_invalid_arguments_return_status(g):
    x = torch.zeros(1, 64, 1, 96, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(g.Gdn2Error) as e:
        g.chunk_fwd(x, x, x, x, x, x)
    assert e.value.status == g.GDN2_ERR_UNSUPPORTED


# ------------------------------------------------------------------ decode

def test_decode_small(g):
    wl = W.Workload("dec_small", B=3, T=1, H=2, dk=128, dv=128)
    S = W.decode_state(wl, device="cuda", seed=1)
    S_ref = np64(S)
    for step in range(5):
        t = W.decode_token_inputs(wl, step, device="cuda", seed=1)
        o = g.decode_step(*[t[n] for n in TOK], S=S)
        o_ref, S_ref = oracle.decode_step(*[np64(t[n]) for n in TOK], S=S_ref)
        torch.cuda.synchronize()
        check_bf16(np64(o), o_ref, f"o step {step}")
    check_bf16(np64(S), S_ref, "S")


@pytest.mark.parametrize("dk,dv,dtype", [(64, 64, "f32"), (128, 256, "bf16"), (64, 128, "bf16")])
def test_decode_shapes(g, dk, dv, dtype):
    wl = W.Workload("dec_shapes", B=4, T=1, H=3, dk=dk, dv=dv, dtype=dtype)
    S = W.decode_state(wl, device="cuda", seed=2)
    t = W.decode_token_inputs(wl, 0, device="cuda", seed=2)
    o_ref, S_ref = oracle.decode_step(*[np64(t[n]) for n in TOK], S=np64(S))
    o = g.decode_step(*[t[n] for n in TOK], S=S)
    torch.cuda.synchronize()
    chk = check_f32 if dtype == "f32" else check_bf16
    chk(np64(o), o_ref, "o")
    chk(np64(S), S_ref, "S")


def test_decode_continues_chunk_fwd(g):
    wl = W.Workload("prefill_then_decode", B=2, T=150, H=2, dk=128, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=14)
    pre = 120
    o1, S = g.chunk_fwd(*[d[n][:, :pre].contiguous() for n in TOK], S0=d["S0"])
    outs = [o1]
    for t in range(pre, 150):
        o = g.decode_step(*[d[n][:, t].contiguous() for n in TOK], S=S)
        outs.append(o[:, None])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=np64(d["S0"]))
    check_bf16(np64(torch.cat(outs, 1)), o_ref, "o")
    check_bf16(np64(S), S_ref, "S")


# ------------------------------------------------------------------ failure path of the bounded waits

def test_bounded_wait_timeout_is_reported_and_context_survives(g):
    """A device wait that nothing completes gives up after its limit and records GDN2_ERR_TIMEOUT;
    no fault, and the context keeps working (a chunk_fwd afterwards still matches the oracle)."""
    torch.cuda.synchronize()
    assert g.device_status(reset=True) == g.GDN2_OK
    g.selftest_bounded_wait(limit_us=20000)
    torch.cuda.synchronize()
    assert g.device_status(reset=True) == g.GDN2_ERR_TIMEOUT
    assert g.device_status() == g.GDN2_OK
    wl = W.Workload("after_timeout", B=1, T=100, H=2, dk=128, dv=128)
    run_case(g, wl, seed=21)
    assert g.device_status() == g.GDN2_OK


# ------------------------------------------------------------------ two-level (segment) state scan
# Long dense sequences over few (sequence, head) pairs take the segmented path: segment maps,
# their chain into entry states, then every segment from its entry state.

@pytest.mark.parametrize("B,T,H,dv", [(1, 2500, 2, 128), (1, 4100, 1, 256), (1, 3000, 2, 64)])
def test_two_level_scan_matches_oracle(g, B, T, H, dv):
    wl = W.Workload("segmented", B=B, T=T, H=H, dk=128, dv=dv)
    run_case(g, wl, seed=41)


def test_two_level_scan_zero_state_and_aliased_final_state(g):
    wl = W.Workload("segmented_alias", B=1, T=2600, H=2, dk=128, dv=128)
    d = W.chunk_inputs(wl, device="cuda", seed=42)
    o, _ = g.chunk_fwd(*[d[n] for n in TOK], S0=None, output_final_state=False)
    S = d["S0"].clone()
    o2, _ = g.chunk_fwd(*[d[n] for n in TOK], S0=S, S_T=S)
    torch.cuda.synchronize()
    o_ref, _ = oracle.recurrent(*[np64(d[n]) for n in TOK])
    check_bf16(np64(o), o_ref, "o, zero initial state")
    o_ref2, S_ref2 = oracle.recurrent(*[np64(d[n]) for n in TOK], S0=np64(d["S0"]))
    check_bf16(np64(o2), o_ref2, "o")
    check_bf16(S.cpu().double().numpy(), S_ref2, "aliased S_T")


# ------------------------------------------------------------------ d_k = 64 on the tensor-core path
# bf16 with d_k = 64 runs the same two tensor-core kernels as d_k = 128 (its second 64-channel block
# arrives as zeros and the state rows it would carry stay zero); the workspace size and the launch
# count show that the tensor-core path ran, not the SIMT kernel.

@pytest.mark.parametrize("dv", [64, 128, 256])
def test_dk64_bf16_tensor_core_path(g, dv):
    wl = W.Workload("dk64_tc", B=2, T=333, H=3, dk=64, dv=dv)
    assert g.chunk_fwd_workspace_bytes(wl.B, wl.T, wl.H, wl.dk, wl.dv) > 0
    c0 = g.launch_count()
    run_case(g, wl, seed=51)
    assert g.launch_count() - c0 == 2  # the WY kernel and the state pass


def test_dk64_bf16_packed_and_two_level_scan(g):
    lengths = [1, 63, 64, 65, 0, 128, 129, 200]
    wl = W.Workload("dk64_packed", B=len(lengths), T=256, H=2, dk=64, dv=128, varlen=True)
    assert g.chunk_fwd_workspace_bytes(len(lengths), sum(lengths), wl.H, wl.dk, wl.dv, packed=True) > 0
    run_case(g, wl, seed=52, lengths=lengths)
    wl = W.Workload("dk64_scan", B=1, T=2600, H=2, dk=64, dv=128)
    c0 = g.launch_count()
    run_case(g, wl, seed=53)
    assert g.launch_count() - c0 == 4  # WY, segment maps, their chain, the segments' walks
