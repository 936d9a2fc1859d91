"""Pins of the backward oracle (the gradient of the token loop; CPU only).

The gradient in ``oracle/bwd_oracle.c`` is derived by hand from the recurrence of
"[논문] 게이트형 DeltaNet-2" (euno.news), section "방법론", and
"NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section "Gated DeltaNet-2の核心".
It is pinned against three things that do not share its derivation:

* central finite differences of the forward oracle, element by element, on tiny
  dense and packed problems (every term of the chain rule moves some element);
* torch autograd through a token loop written here from the same definition;
* closed forms at alpha = 1, b = 0 (plain linear attention), where every gradient
  is a sum over later tokens rather than a reverse recurrence.

The chunk-form companion (``oracle.chunkwise_bwd``) is pinned against the token-loop
gradient at several chunk sizes, ragged and packed.
"""
import numpy as np
import pytest
import torch

import oracle

rng = np.random.default_rng(7)


def _problem(N, T, H, dk, dv, packed=None):
    lead = (int(sum(packed)), H) if packed else (N, T, H)
    x = {n: rng.standard_normal(lead + (dk,)) for n in ("q", "k", "b")}
    x["alpha"] = rng.uniform(0.4, 1.0, lead + (dk,))
    x["v"], x["w"], x["dO"] = (rng.standard_normal(lead + (dv,)) for _ in range(3))
    nseq = len(packed) if packed else N
    x["S0"] = rng.standard_normal((nseq, H, dk, dv)) * 0.3
    x["dST"] = rng.standard_normal((nseq, H, dk, dv))
    cu = None if not packed else np.concatenate([[0], np.cumsum(packed)]).astype(np.int64)
    return x, cu


def _loss(x, cu):
    o, ST = oracle.recurrent(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], S0=x["S0"], cu_seqlens=cu)
    return float(np.sum(o * x["dO"]) + np.sum(ST * x["dST"]))


NAMES = ("q", "k", "v", "alpha", "b", "w", "S0")


def _grads(x, cu):
    return dict(zip(NAMES, oracle.recurrent_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["dO"],
                                                S0=x["S0"], dST=x["dST"], cu_seqlens=cu)))


@pytest.mark.parametrize("packed", [None, [3, 1, 0, 4]])
def test_every_element_matches_central_differences(packed):
    x, cu = _problem(2, 5, 2, 3, 2, packed)
    g = _grads(x, cu)
    eps = 1e-6
    for name in NAMES:
        flat = x[name].reshape(-1)
        fd = np.empty_like(flat)
        for e in range(flat.size):
            keep = flat[e]
            flat[e] = keep + eps
            up = _loss(x, cu)
            flat[e] = keep - eps
            dn = _loss(x, cu)
            flat[e] = keep
            fd[e] = (up - dn) / (2 * eps)
        np.testing.assert_allclose(g[name].reshape(-1), fd, rtol=1e-6, atol=1e-7, err_msg=name)


def _torch_loop(q, k, v, alpha, b, w, S0):
    """Token loop for one (sequence, head), [T, d] tensors; returns o [T, d_v] and S_T."""
    S = S0
    outs = []
    for t in range(q.shape[0]):
        Sp = alpha[t][:, None] * S
        delta = w[t] * v[t] - Sp.T @ (b[t] * k[t])
        S = Sp + torch.outer(k[t], delta)
        outs.append(S.T @ q[t])
    return torch.stack(outs), S


def test_matches_autograd_of_an_independent_loop():
    N, T, H, dk, dv = 2, 17, 2, 6, 5
    x, _ = _problem(N, T, H, dk, dv)
    g = _grads(x, None)
    for n in range(N):
        for h in range(H):
            leaves = {nm: torch.tensor(x[nm][n, :, h], requires_grad=True)
                      for nm in ("q", "k", "v", "alpha", "b", "w")}
            S0 = torch.tensor(x["S0"][n, h], requires_grad=True)
            o, ST = _torch_loop(*[leaves[nm] for nm in ("q", "k", "v", "alpha", "b", "w")], S0)
            L = (o * torch.tensor(x["dO"][n, :, h])).sum() + (ST * torch.tensor(x["dST"][n, h])).sum()
            L.backward()
            for nm, leaf in leaves.items():
                np.testing.assert_allclose(g[nm][n, :, h], leaf.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=nm)
            np.testing.assert_allclose(g["S0"][n, h], S0.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_empty_sequence_passes_the_state_gradient_through():
    x, cu = _problem(1, 0, 2, 3, 4, packed=[2, 0, 3])
    g = _grads(x, cu)
    # the empty sequence 1 has S_T = S0, so dS0 = dST
    np.testing.assert_array_equal(g["S0"][1], x["dST"][1])


def test_zero_upstream_gives_zero_gradients():
    x, cu = _problem(1, 6, 1, 4, 3)
    x["dO"][:] = 0.0
    x["dST"][:] = 0.0
    for name, gr in _grads(x, cu).items():
        assert not gr.any(), name


def test_linearity_in_the_upstream_gradients():
    # L is linear in (dO, dST), so the gradients are too: g(dO, dST) = g(dO, 0) + g(0, dST)
    x, cu = _problem(2, 7, 2, 3, 3)
    both = _grads(x, cu)
    keep = x["dST"].copy()
    x["dST"][:] = 0.0
    only_o = _grads(x, cu)
    x["dST"] = keep
    x["dO"] = np.zeros_like(x["dO"])
    only_s = _grads(x, cu)
    for name in NAMES:
        np.testing.assert_allclose(both[name], only_o[name] + only_s[name], rtol=1e-12, atol=1e-13)


def test_linear_attention_closed_forms():
    """alpha = 1, b = 0: S_t = S0 + sum_{s<=t} k_s u_s^T (u = w (.) v) and o_t = S_t^T q_t.  Every
    gradient is then a sum over later tokens, written here without the reverse recurrence:
      dq_t = S_t dO_t,   G_s = sum_{t>=s} q_t dO_t^T + dST,   du_s = G_s^T k_s,
      dk_s = G_s u_s,    dS0 = G_1,   dalpha_s[i] = sum_j G_s[i, j] S_{s-1}[i, j],
      db_s = -k_s (.) (S_{s-1} (G_s^T k_s))   (the erase probe's derivative at b = 0)."""
    N, T, H, dk, dv = 1, 9, 1, 4, 3
    x, cu = _problem(N, T, H, dk, dv)
    x["alpha"][:] = 1.0
    x["b"][:] = 0.0
    g = _grads(x, cu)
    q, k, v, w, dO = (x[n][0, :, 0] for n in ("q", "k", "v", "w", "dO"))
    S0, dST = x["S0"][0, 0], x["dST"][0, 0]
    u = w * v
    S = [S0]
    for t in range(T):
        S.append(S[-1] + np.outer(k[t], u[t]))
    G = [sum((np.outer(q[t], dO[t]) for t in range(s, T)), np.zeros((dk, dv))) + dST for s in range(T)]
    for s in range(T):
        np.testing.assert_allclose(g["q"][0, s, 0], S[s + 1] @ dO[s], rtol=1e-12, atol=1e-12)
        du = G[s].T @ k[s]
        np.testing.assert_allclose(g["v"][0, s, 0], du * w[s], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g["w"][0, s, 0], du * v[s], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g["k"][0, s, 0], G[s] @ u[s], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g["alpha"][0, s, 0], (G[s] * S[s]).sum(1), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g["b"][0, s, 0], -k[s] * (S[s] @ du), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["S0"][0, 0], G[0], rtol=1e-12, atol=1e-12)


def _contractive(x):
    """The path's input regime: unit q and k, gates in (0, 1).  Each step's erase then shrinks
    the state (1 - b.k^2 in (0, 1)), so long sequences stay well conditioned."""
    for n in ("q", "k"):
        x[n] /= np.linalg.norm(x[n], axis=-1, keepdims=True)
    for n in ("b", "w"):
        x[n] = 1.0 / (1.0 + np.exp(-x[n]))
    return x


@pytest.mark.parametrize("chunk", [1, 2, 16, 64])
@pytest.mark.parametrize("T", [37, 70])
def test_chunk_form_gradient_equals_the_token_loop(chunk, T):
    """The companion that takes the gradient through the chunkwise WY form (one triangular system
    per chunk) equals the token loop's gradient up to rounding, with a ragged last chunk."""
    x, cu = _problem(2, T, 2, 5, 4)
    x = _contractive(x)
    ref = _grads(x, cu)
    got = oracle.chunkwise_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["dO"], S0=x["S0"],
                               dST=x["dST"], chunk=chunk)
    for name, y in zip(NAMES, got):
        np.testing.assert_allclose(y, ref[name], rtol=1e-9, atol=1e-11 * np.max(np.abs(ref[name])), err_msg=name)


def test_chunk_form_gradient_packed():
    x, cu = _problem(1, 0, 2, 4, 3, packed=[9, 0, 1, 70, 33])
    x = _contractive(x)
    ref = _grads(x, cu)
    got = oracle.chunkwise_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["dO"], S0=x["S0"],
                               dST=x["dST"], cu_seqlens=cu, chunk=16)
    for name, y in zip(NAMES, got):
        np.testing.assert_allclose(y, ref[name], rtol=1e-9, atol=1e-11 * np.max(np.abs(ref[name])), err_msg=name)
