"""The chunk records of the tensor-core forward, and their transpose for a chunked backward,
checked in fp64 against the oracle (CPU only).

The tensor-core forward does not run the WY form of "Gated DeltaNet-2: Separando Borrado y
Escritura en la Atención Lineal" (needhelp.icu), "Innovaciones Técnicas", item 1, as two
dependent passes per chunk. It regroups it into one record per (chunk, head), so that the state
chain is one product per chunk. With m the running log-decay at the chunk's token 31, g_C the
chunk's total, A_m = (b (.) k) e^{g-m}, Q_m = q e^{g-m}, K_m = k e^{m-g},
L = strict_lower(A_m K_m^T), P = lower(Q_m K_m^T), T = (I + L)^-1, W = -T A_m:

    S_next = Diag(e^{g_C}) S + Mt S + Nt U,      O = Qt S + Pt U,
    Mt = Diag(e^{g_C-m}) K_m^T W Diag(e^m),      Nt = Diag(e^{g_C-m}) K_m^T T,
    Qt = (Q_m + P W) Diag(e^m),                  Pt = P T,                        U = w (.) v.

The chain is affine in (S, U), so its transpose gives the entering state's gradient and U's
gradient chunk by chunk, backwards, from the next chunk's dS and the chunk's dO:

    dS = (Diag(e^{g_C}) + Mt)^T dS_next + Qt^T dO,   dU = Nt^T dS_next + Pt^T dO,
    dv = dU (.) w,  dw = dU (.) v.

These are this library's regrouping, not the pages' formulas. They are checked here against the
token-loop oracle (``oracle.recurrent``) and its hand-derived gradient (``oracle.recurrent_bwd``),
which share none of this code.
"""
import numpy as np
import pytest

import oracle

rng = np.random.default_rng(11)
C = 64


def _records(q, k, b, alpha):
    """Mt, Nt, Qt, Pt and e^{g_C} of one chunk (tokens on the first axis, Cc <= 64 of them)."""
    Cc, dk = q.shape
    g = np.cumsum(np.log(alpha), axis=0)
    m = g[min(31, Cc - 1)]
    f = np.exp(g - m)
    A, Q, K = b * k * f, q * f, k / f
    L = np.tril(A @ K.T, -1)
    P = np.tril(Q @ K.T)
    T = np.linalg.inv(np.eye(Cc) + L)
    W = -T @ A
    gc = np.exp(g[-1] - m)
    em = np.exp(m)
    Mt = (gc[:, None] * (K.T @ W)) * em[None, :]
    Nt = gc[:, None] * (K.T @ T)
    Qt = (Q + P @ W) * em[None, :]
    Pt = P @ T
    return Mt, Nt, Qt, Pt, np.exp(g[-1])


def _problem(T, dk, dv):
    x = {n: rng.standard_normal((1, T, 1, dk)) for n in ("q", "k", "b")}
    x["k"] /= np.sqrt(dk)
    x["alpha"] = rng.uniform(0.6, 1.0, (1, T, 1, dk))
    x["v"], x["w"], x["dO"] = (rng.standard_normal((1, T, 1, dv)) for _ in range(3))
    x["S0"] = rng.standard_normal((1, 1, dk, dv))
    x["dST"] = rng.standard_normal((1, 1, dk, dv))
    return x


def _chunks(x, T):
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        yield sl, {n: x[n][0, sl, 0] for n in ("q", "k", "b", "alpha", "v", "w", "dO")}


@pytest.mark.parametrize("T,dk,dv", [(64, 16, 8), (200, 32, 24), (37, 8, 8)])
def test_records_reproduce_the_forward(T, dk, dv):
    """Walking the records chunk by chunk gives the oracle's outputs and final state."""
    x = _problem(T, dk, dv)
    o_ref, S_ref = oracle.recurrent(*[x[n] for n in ("q", "k", "v", "alpha", "b", "w")], S0=x["S0"])
    S = x["S0"][0, 0].copy()
    o = np.zeros((T, dv))
    for sl, ch in _chunks(x, T):
        Mt, Nt, Qt, Pt, G = _records(ch["q"], ch["k"], ch["b"], ch["alpha"])
        U = ch["w"] * ch["v"]
        o[sl] = Qt @ S + Pt @ U
        S = G[:, None] * S + Mt @ S + Nt @ U
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("T,dk,dv", [(64, 16, 8), (200, 32, 24), (37, 8, 8)])
def test_transposed_records_give_dv_dw_and_dS0(T, dk, dv):
    """The records' transpose, walked backwards, gives the oracle's dv, dw and dS0."""
    x = _problem(T, dk, dv)
    grads = oracle.recurrent_bwd(*[x[n] for n in ("q", "k", "v", "alpha", "b", "w", "dO")], S0=x["S0"], dST=x["dST"])
    dv_ref, dw_ref, dS0_ref = grads[2], grads[5], grads[6]
    chunks = list(_chunks(x, T))
    dS = x["dST"][0, 0].copy()
    dv_ = np.zeros((T, dv))
    dw_ = np.zeros((T, dv))
    for sl, ch in reversed(chunks):
        Mt, Nt, Qt, Pt, G = _records(ch["q"], ch["k"], ch["b"], ch["alpha"])
        dU = Nt.T @ dS + Pt.T @ ch["dO"]
        dv_[sl] = dU * ch["w"]
        dw_[sl] = dU * ch["v"]
        dS = G[:, None] * dS + Mt.T @ dS + Qt.T @ ch["dO"]
    np.testing.assert_allclose(dv_, dv_ref[0, :, 0], rtol=1e-8, atol=1e-9)
    np.testing.assert_allclose(dw_, dw_ref[0, :, 0], rtol=1e-8, atol=1e-9)
    np.testing.assert_allclose(dS, dS0_ref[0, 0], rtol=1e-8, atol=1e-9)


def test_a_wrong_record_is_caught():
    """Dropping the Diag(e^m) scale of Mt (a plausible slip) breaks the forward check."""
    x = _problem(128, 16, 8)
    _, S_ref = oracle.recurrent(*[x[n] for n in ("q", "k", "v", "alpha", "b", "w")], S0=x["S0"])
    S = x["S0"][0, 0].copy()
    for sl, ch in _chunks(x, 128):
        Mt, Nt, Qt, Pt, G = _records(ch["q"], ch["k"], ch["b"], ch["alpha"])
        g = np.cumsum(np.log(ch["alpha"]), axis=0)
        Mt_wrong = Mt / np.exp(g[31])[None, :]
        S = G[:, None] * S + Mt_wrong @ S + Nt @ (ch["w"] * ch["v"])
    assert np.max(np.abs(S - S_ref[0, 0])) > 1e-3
