"""Pins of the fp64 oracle to things other than itself (CPU only).

Each pin comes from what the pages fix, or from mathematics:
* exact-rational fixtures (tests/golden, transition-matrix brute force);
* the special cases the pages name: KDA when b_t = w_t = beta_t, Gated
  DeltaNet when alpha_t is also a scalar, DeltaNet when ungated
  ("Jerarquía de Generalización", needhelp.icu; "Gated DeltaNet-2の核心",
  ai.warp-studio.com) -- checked against textbook loops written here in numpy;
* the chunkwise WY form ("Algoritmo WY por Bloques", needhelp.icu) equals the
  token loop;
* closed forms (no erase => gated linear attention), the delta rule's exact
  write (fast-weight view, "Vista de Actualización de Pesos Rápidos"),
  channel-permutation symmetries, linearity in (S0, v), resume by splitting.
A final test plants each plausible mistake in the oracle and checks that at
least one pin fails.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import make_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOK = ("q", "k", "v", "alpha", "b", "w")


def _rel(x, y):
    return float(np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300))


def _load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        doc = json.load(f)
    cv = lambda a: np.array([[float(Fraction(x)) for x in r] for r in a]) if isinstance(a[0], list) \
        else np.array([float(Fraction(x)) for x in a])  # noqa: E731
    return {k: cv(v) for k, v in doc["inputs"].items()}, cv(doc["o"]), cv(doc["S_T"])


def _as_batch(x):
    """[T, d] -> [N=1, T, H=1, d]"""
    return x[None, :, None, :]


# ---------------------------------------------------------------- numpy textbook loops (independent)

def np_kda(q, k, v, alpha, beta, S0):
    """KDA: S = (I - beta k k^T) Diag(alpha) S + beta k v^T, o = S^T q.  q..: [T, d], beta [T]."""
    S = S0.copy()
    dk = q.shape[1]
    o = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        M = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(alpha[t])
        S = M @ S + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def np_gdn(q, k, v, alpha, beta, S0):
    """Gated DeltaNet: S = alpha (I - beta k k^T) S + beta k v^T; alpha, beta [T]."""
    S = S0.copy()
    dk = q.shape[1]
    o = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        S = alpha[t] * (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ S + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def np_deltanet(q, k, v, beta, S0):
    """DeltaNet: S = (I - beta k k^T) S + beta k v^T."""
    S = S0.copy()
    dk = q.shape[1]
    o = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        S = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ S + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def np_transition_products(q, k, v, alpha, b, w, S0, orientation):
    """Brute force: explicit per-token transitions multiplied out from S0 for every t."""
    T, dk = q.shape
    Ms, Ws = [], []
    for t in range(T):
        a = b[t] * k[t]
        E = np.eye(dk) - (np.outer(k[t], a) if orientation == oracle.ERASE_R1 else np.outer(a, k[t]))
        Ms.append(E @ np.diag(alpha[t]))
        Ws.append(np.outer(k[t], w[t] * v[t]))
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        P = np.eye(dk)
        for s in range(t, -1, -1):
            P = P @ Ms[s]
        S = P @ S0
        for s in range(t + 1):
            R = np.eye(dk)
            for r in range(t, s, -1):
                R = R @ Ms[r]
            S = S + R @ Ws[s]
        o[t] = S.T @ q[t]
    return o, S


# ---------------------------------------------------------------- golden fixtures

def test_golden_gdn2_exact():
    inp, o_ref, S_ref = _load_golden("gdn2_tiny_exact.json")
    o, S = oracle.recurrent(*[_as_batch(inp[n]) for n in TOK], S0=inp["S0"][None, None])
    assert np.max(np.abs(o[0, :, 0] - o_ref)) < 1e-14
    assert np.max(np.abs(S[0, 0] - S_ref)) < 1e-14


@pytest.mark.parametrize("orientation", [oracle.ERASE_R1, oracle.ERASE_R2])
def test_golden_kda_exact(orientation):
    inp, o_ref, S_ref = _load_golden("kda_tiny_exact.json")
    T, dk = inp["q"].shape
    dv = inp["v"].shape[1]
    b = np.repeat(inp["beta"][:, None], dk, 1)
    w = np.repeat(inp["beta"][:, None], dv, 1)
    o, S = oracle.recurrent(*[_as_batch(x) for x in (inp["q"], inp["k"], inp["v"], inp["alpha"], b, w)],
                            S0=inp["S0"][None, None], orientation=orientation)
    assert np.max(np.abs(o[0, :, 0] - o_ref)) < 1e-14
    assert np.max(np.abs(S[0, 0] - S_ref)) < 1e-14


def test_golden_gdn_exact():
    inp, o_ref, S_ref = _load_golden("gdn_tiny_exact.json")
    T, dk = inp["q"].shape
    dv = inp["v"].shape[1]
    al = np.repeat(inp["alpha_scalar"][:, None], dk, 1)
    b = np.repeat(inp["beta"][:, None], dk, 1)
    w = np.repeat(inp["beta"][:, None], dv, 1)
    o, S = oracle.recurrent(*[_as_batch(x) for x in (inp["q"], inp["k"], inp["v"], al, b, w)],
                            S0=inp["S0"][None, None])
    assert np.max(np.abs(o[0, :, 0] - o_ref)) < 1e-14
    assert np.max(np.abs(S[0, 0] - S_ref)) < 1e-14


# ---------------------------------------------------------------- reductions named by the pages

@pytest.mark.parametrize("orientation", [oracle.ERASE_R1, oracle.ERASE_R2])
def test_kda_reduction(orientation):
    _, c = make_case(T=48, dk=16, dv=12, H=2, N=2, seed=1, variant="kda")
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"], orientation=orientation)
    for n in range(2):
        for h in range(2):
            beta = c["b"][n, :, h, 0]
            o_ref, S_ref = np_kda(c["q"][n, :, h], c["k"][n, :, h], c["v"][n, :, h], c["alpha"][n, :, h],
                                  beta, c["S0"][n, h])
            assert _rel(o[n, :, h], o_ref) < 1e-12
            assert _rel(S[n, h], S_ref) < 1e-12


def test_gdn_reduction():
    _, c = make_case(T=48, dk=16, dv=12, H=2, N=1, seed=2, variant="gdn")
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"])
    for h in range(2):
        o_ref, S_ref = np_gdn(c["q"][0, :, h], c["k"][0, :, h], c["v"][0, :, h], c["alpha"][0, :, h, 0],
                              c["b"][0, :, h, 0], c["S0"][0, h])
        assert _rel(o[0, :, h], o_ref) < 1e-12
        assert _rel(S[0, h], S_ref) < 1e-12


def test_deltanet_reduction():
    _, c = make_case(T=40, dk=8, dv=8, seed=3, variant="kda")
    ones = np.ones_like(c["alpha"])
    o, S = oracle.recurrent(c["q"], c["k"], c["v"], ones, c["b"], c["w"], S0=c["S0"])
    o_ref, S_ref = np_deltanet(c["q"][0, :, 0], c["k"][0, :, 0], c["v"][0, :, 0], c["b"][0, :, 0, 0], c["S0"][0, 0])
    assert _rel(o[0, :, 0], o_ref) < 1e-12
    assert _rel(S[0, 0], S_ref) < 1e-12


# ---------------------------------------------------------------- brute force on tiny inputs

@pytest.mark.parametrize("orientation", [oracle.ERASE_R1, oracle.ERASE_R2])
def test_bruteforce_transition_product(orientation):
    _, c = make_case(T=7, dk=5, dv=4, seed=4, s0="normal")
    S0 = c["S0"] * 20.0  # O(1) initial state so every term is visible
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=S0, orientation=orientation)
    o_ref, S_ref = np_transition_products(*[c[n][0, :, 0] for n in TOK], S0[0, 0], orientation)
    assert _rel(o[0, :, 0], o_ref) < 1e-12
    assert _rel(S[0, 0], S_ref) < 1e-12


def test_orientations_differ_off_the_reductions():
    _, c = make_case(T=10, dk=6, dv=6, seed=5)
    o1, S1 = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"], orientation=oracle.ERASE_R1)
    o2, S2 = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"], orientation=oracle.ERASE_R2)
    assert _rel(S1, S2) > 1e-3


# ---------------------------------------------------------------- chunkwise WY form == token loop

@pytest.mark.parametrize("chunk", [1, 2, 16, 64])
def test_chunkwise_equals_recurrent(chunk):
    _, c = make_case(T=150, dk=16, dv=24, H=2, N=2, seed=6)
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"])
    oc, Sc = oracle.chunkwise(*[c[n] for n in TOK], S0=c["S0"], chunk=chunk)
    assert _rel(oc, o) < 1e-12
    assert _rel(Sc, S) < 1e-12


def test_chunkwise_equals_recurrent_varlen_strong_decay():
    lengths = [1, 63, 64, 65, 130, 7]
    _, c = make_case(T=0, dk=16, dv=16, H=2, N=len(lengths), seed=7, lengths=lengths, shift=-1.0)
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"], cu_seqlens=c["cu_seqlens"])
    oc, Sc = oracle.chunkwise(*[c[n] for n in TOK], S0=c["S0"], cu_seqlens=c["cu_seqlens"], chunk=64)
    assert _rel(oc, o) < 1e-11
    assert _rel(Sc, S) < 1e-11


# ---------------------------------------------------------------- closed forms

def test_no_erase_is_gated_linear_attention():
    """b = 0: S_T = Diag(prod alpha) S0 + sum_t Diag(prod_{s>t} alpha_s) k_t (w_t*v_t)^T."""
    _, c = make_case(T=30, dk=8, dv=6, seed=8)
    zeros = np.zeros_like(c["b"])
    o, S = oracle.recurrent(c["q"], c["k"], c["v"], c["alpha"], zeros, c["w"], S0=c["S0"])
    q, k, v, al, w = (c[n][0, :, 0] for n in ("q", "k", "v", "alpha", "w"))
    T = q.shape[0]
    for t in range(T):
        St = np.prod(al[: t + 1], axis=0)[:, None] * c["S0"][0, 0]
        for s in range(t + 1):
            St = St + np.prod(al[s + 1: t + 1], axis=0)[:, None] * np.outer(k[s], w[s] * v[s])
        assert np.max(np.abs(o[0, t, 0] - St.T @ q[t])) < 1e-13
    assert np.max(np.abs(S[0, 0] - St)) < 1e-13


def test_no_decay_no_erase_is_sum_of_outer_products():
    _, c = make_case(T=25, dk=7, dv=5, seed=9)
    o, S = oracle.recurrent(c["q"], c["k"], c["v"], np.ones_like(c["alpha"]), np.zeros_like(c["b"]), c["w"],
                            S0=c["S0"])
    k, v, w = (c[n][0, :, 0] for n in ("k", "v", "w"))
    assert np.max(np.abs(S[0, 0] - (c["S0"][0, 0] + k.T @ (w * v)))) < 1e-13


def test_delta_rule_exact_write():
    """b = 1 and |k| = 1: the erase removes exactly what k reads, so S_t^T k_t = w_t * v_t."""
    _, c = make_case(T=40, dk=16, dv=8, seed=10)
    k = c["k"] / np.linalg.norm(c["k"], axis=-1, keepdims=True)  # unit norm in fp64
    ones = np.ones_like(c["b"])
    o, _ = oracle.recurrent(k, k, c["v"], c["alpha"], ones, c["w"], S0=c["S0"])
    assert np.max(np.abs(o - c["w"] * c["v"])) < 1e-13


# ---------------------------------------------------------------- symmetries and linearity

def test_value_channel_permutation():
    _, c = make_case(T=33, dk=8, dv=10, seed=11)
    perm = np.random.default_rng(0).permutation(10)
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"])
    op, Sp = oracle.recurrent(c["q"], c["k"], c["v"][..., perm], c["alpha"], c["b"], c["w"][..., perm],
                              S0=c["S0"][..., perm])
    assert np.max(np.abs(op - o[..., perm])) < 1e-13
    assert np.max(np.abs(Sp - S[..., perm])) < 1e-13


def test_key_channel_permutation():
    _, c = make_case(T=33, dk=9, dv=6, seed=12)
    perm = np.random.default_rng(1).permutation(9)
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"])
    pk = lambda x: x[..., perm]  # noqa: E731
    op, Sp = oracle.recurrent(pk(c["q"]), pk(c["k"]), c["v"], pk(c["alpha"]), pk(c["b"]), c["w"],
                              S0=c["S0"][:, :, perm, :])
    assert np.max(np.abs(op - o)) < 1e-13
    assert np.max(np.abs(Sp - S[:, :, perm, :])) < 1e-13


def test_linear_in_initial_state_and_values():
    _, c1 = make_case(T=20, dk=6, dv=5, seed=13)
    _, c2 = make_case(T=20, dk=6, dv=5, seed=14)
    base = [c1[n] for n in ("q", "k")]
    run = lambda v, S0: oracle.recurrent(*base, v, c1["alpha"], c1["b"], c1["w"], S0=S0)  # noqa: E731
    oa, Sa = run(c1["v"], c1["S0"])
    ob, Sb = run(c2["v"], c2["S0"] * 7)
    os_, Ss = run(c1["v"] + c2["v"], c1["S0"] + c2["S0"] * 7)
    assert np.max(np.abs(os_ - (oa + ob))) < 1e-12
    assert np.max(np.abs(Ss - (Sa + Sb))) < 1e-12


# ---------------------------------------------------------------- state as checkpoint, layouts

@pytest.mark.parametrize("split", [1, 37, 64, 100])
def test_resume_split_equals_one_call(split):
    _, c = make_case(T=130, dk=8, dv=8, H=2, seed=15)
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"])
    o1, S1 = oracle.recurrent(*[c[n][:, :split] for n in TOK], S0=c["S0"])
    o2, S2 = oracle.recurrent(*[c[n][:, split:] for n in TOK], S0=S1)
    assert np.max(np.abs(np.concatenate([o1, o2], 1) - o)) < 1e-13
    assert np.max(np.abs(S2 - S)) < 1e-13


def test_packed_equals_per_sequence():
    lengths = [5, 0, 17, 64, 1]
    _, c = make_case(T=0, dk=8, dv=6, H=3, N=len(lengths), seed=16, lengths=lengths)
    o, S = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"], cu_seqlens=c["cu_seqlens"])
    cu = c["cu_seqlens"]
    for n, L in enumerate(lengths):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = oracle.recurrent(*[c[x][sl][None] for x in TOK], S0=c["S0"][n:n + 1])
        assert np.array_equal(on[0], o[sl])
        assert np.array_equal(Sn[0], S[n])
    # an empty sequence passes its state through unchanged
    assert np.array_equal(S[1], c["S0"][1])


def test_decode_step_is_one_token_of_the_recurrence():
    _, c = make_case(T=1, dk=8, dv=6, H=2, N=3, seed=17)
    sq = lambda x: x[:, 0]  # noqa: E731
    o, S = oracle.decode_step(*[sq(c[n]) for n in TOK], S=c["S0"])
    o_ref, S_ref = oracle.recurrent(*[c[n] for n in TOK], S0=c["S0"])
    assert np.array_equal(o, o_ref[:, 0])
    assert np.array_equal(S, S_ref)


def test_zero_length_returns_initial_state():
    _, c = make_case(T=4, dk=4, dv=4, seed=18)
    o, S = oracle.recurrent(*[c[n][:, :0] for n in TOK], S0=c["S0"])
    assert o.shape[1] == 0 and np.array_equal(S, c["S0"])


# ---------------------------------------------------------------- the pins catch planted mistakes

def _pin_failures(rec):
    """Run the pins with ``rec`` in place of the oracle; return the names of the pins that fail."""
    failed = []
    inp, o_ref, S_ref = _load_golden("gdn2_tiny_exact.json")
    inp_sq = inp  # d_k != d_v: plants that need a square state skip this pin
    try:
        o, S = rec(*[_as_batch(inp_sq[n]) for n in TOK], S0=inp_sq["S0"][None, None])
        if np.max(np.abs(o[0, :, 0] - o_ref)) > 1e-12 or np.max(np.abs(S[0, 0] - S_ref)) > 1e-12:
            failed.append("golden")
    except RuntimeError:
        pass
    _, c = make_case(T=24, dk=8, dv=8, seed=19, variant="kda")
    o, S = rec(*[c[n] for n in TOK], S0=c["S0"] * 20)
    o_ref, S_ref = np_kda(*[c[n][0, :, 0] for n in ("q", "k", "v", "alpha")], c["b"][0, :, 0, 0], c["S0"][0, 0] * 20)
    if _rel(o[0, :, 0], o_ref) > 1e-10 or _rel(S[0, 0], S_ref) > 1e-10:
        failed.append("kda")
    _, c = make_case(T=24, dk=8, dv=8, seed=20)
    k = c["k"] / np.linalg.norm(c["k"], axis=-1, keepdims=True)
    o, _ = rec(k, k, c["v"], c["alpha"], np.ones_like(c["b"]), c["w"], S0=c["S0"] * 20)
    if np.max(np.abs(o - c["w"] * c["v"])) > 1e-10:
        failed.append("exact_write")
    _, c = make_case(T=24, dk=8, dv=8, seed=21)
    S0 = c["S0"] * 20
    o, S = rec(*[c[n] for n in TOK], S0=S0)
    o_ref, S_ref = np_transition_products(*[c[n][0, :, 0] for n in TOK], S0[0, 0], oracle.ERASE_R1)
    if _rel(o[0, :, 0], o_ref) > 1e-10 or _rel(S[0, 0], S_ref) > 1e-10:
        failed.append("bruteforce")
    oc, Sc = oracle.chunkwise(*[c[n] for n in TOK], S0=S0, chunk=8)
    if _rel(o, oc) > 1e-10 or _rel(S, Sc) > 1e-10:
        failed.append("chunkwise")
    return failed


def test_pins_pass_on_the_oracle():
    assert _pin_failures(oracle.recurrent) == []


@pytest.mark.parametrize("plant", sorted(oracle.PLANTS))
def test_each_planted_mistake_is_caught(plant):
    rec = lambda *a, **kw: oracle.recurrent_planted(*a, plant=plant, **kw)  # noqa: E731
    assert _pin_failures(rec), f"no pin caught planted mistake: {oracle.PLANTS[plant]}"
