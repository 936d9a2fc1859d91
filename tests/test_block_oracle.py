"""Pins of the block oracle (the work around the mixer; CPU only).

The oracle's block functions follow "NVIDIA AIがGated DeltaNet-2を発表"
(ai.warp-studio.com), section "アーキテクチャとパフォーマンスベンチマーク".  Each
pin checks them against something other than their own formula: numpy's
convolution, closed forms at points where sigmoid and SiLU are exact
fractions, invariants of the two normalisations, and the independence of
packed sequences.
"""
import math

import numpy as np
import pytest
from scipy.special import expit

import oracle

rng = np.random.default_rng(2026)


def _inputs(N, T, H, dk, dv, K, positive=False):
    draw = (lambda *s: rng.uniform(0.05, 1.0, s)) if positive else (lambda *s: rng.standard_normal(s))
    x = [draw(N, T, H, d) for d in (dk, dk, dv, dk, dk, dv)]
    W = [draw(H * d, K) for d in (dk, dk, dv)]
    return x, W


def _silu_inverse(s):
    """y >= 0 with y sigmoid(y) = s, by Newton's method (SiLU is increasing there)."""
    y = np.maximum(s, 0.0) + 0.5
    for _ in range(60):
        sg = expit(y)
        y = y - (y * sg - s) / (sg + y * sg * (1.0 - sg))
    return y


@pytest.mark.parametrize("K", [1, 2, 4])
def test_value_path_is_numpy_causal_convolution(K):
    # positive inputs and weights keep the pre-activation >= 0, where SiLU can be inverted exactly
    N, T, H, dk, dv = 2, 11, 2, 3, 4
    x, W = _inputs(N, T, H, dk, dv, K, positive=True)
    v = oracle.block_prologue(*x, *W)[2]
    y = _silu_inverse(v)
    for n in range(N):
        for h in range(H):
            for c in range(dv):
                ref = np.convolve(x[2][n, :, h, c], W[2][h * dv + c][::-1])[:T]  # last tap = current token
                np.testing.assert_allclose(y[n, :, h, c], ref, rtol=1e-10, atol=1e-12)


def test_shift_kernel_delays_by_its_tap():
    N, T, H, dk, dv, K = 1, 9, 1, 2, 2, 4
    x, W = _inputs(N, T, H, dk, dv, K, positive=True)
    for lag in range(K):
        Wv = np.zeros_like(W[2])
        Wv[:, K - 1 - lag] = 1.0
        v = oracle.block_prologue(*x, W[0], W[1], Wv)[2]
        y = _silu_inverse(v)
        shifted = np.zeros_like(x[2])
        shifted[:, lag:] = x[2][:, : T - lag]
        np.testing.assert_allclose(y, shifted, atol=1e-12)


def test_query_and_key_have_unit_norm():
    N, T, H, dk, dv, K = 2, 7, 3, 8, 4, 4
    x, W = _inputs(N, T, H, dk, dv, K)
    q, k = oracle.block_prologue(*x, *W)[:2]
    for out in (q, k):
        assert np.all(np.abs(np.linalg.norm(out, axis=-1) - 1.0) < 1e-4)  # eps = 1e-6 under the root


def test_query_direction_with_equal_head_sizes():
    N, T, H, d, K = 1, 6, 2, 5, 3
    x, W = _inputs(N, T, H, d, d, K)
    q = oracle.block_prologue(*x, *W)[0]
    raw = oracle.block_prologue(x[0], x[1], x[0], x[3], x[4], x[5], W[0], W[1], W[0])[2]
    np.testing.assert_allclose(q, raw / np.sqrt((raw ** 2).sum(-1, keepdims=True) + 1e-6), rtol=1e-12)


def test_gates_and_decay_closed_forms():
    N, T, H, dk, dv, K = 1, 3, 1, 3, 3, 1
    x, W = _inputs(N, T, H, dk, dv, K)
    ln3 = math.log(3.0)
    pts = np.array([0.0, ln3, -ln3])
    xa = np.broadcast_to(pts, (N, T, H, dk)).copy()
    xb = xa.copy()
    xw = np.broadcast_to(pts, (N, T, H, dv)).copy()
    _, _, _, alpha, b, w = oracle.block_prologue(x[0], x[1], x[2], xa, xb, xw, *W)
    np.testing.assert_allclose(alpha[0, 0, 0], [0.5, 0.25, 0.75], rtol=1e-14)  # exp(-softplus(x)) = 1/(1+e^x)
    np.testing.assert_allclose(b[0, 0, 0], [0.5, 0.75, 0.25], rtol=1e-14)
    np.testing.assert_allclose(w[0, 0, 0], [0.5, 0.75, 0.25], rtol=1e-14)
    xr = rng.standard_normal((N, T, H, dk))
    a2, b2 = oracle.block_prologue(x[0], x[1], x[2], xr, xr, np.zeros((N, T, H, dv)), *W)[3:5]
    np.testing.assert_allclose(a2, expit(-xr), rtol=1e-13)
    np.testing.assert_allclose(b2, expit(xr), rtol=1e-13)


def test_packed_sequences_restart_the_convolution():
    lengths = [5, 1, 8, 3]
    H, dk, dv, K = 2, 4, 3, 4
    cu = np.concatenate([[0], np.cumsum(lengths)])
    Tt = int(cu[-1])
    xs = [rng.standard_normal((Tt, H, d)) for d in (dk, dk, dv, dk, dk, dv)]
    W = [rng.standard_normal((H * d, K)) for d in (dk, dk, dv)]
    packed = oracle.block_prologue(*xs, *W, cu_seqlens=cu)
    for n, L in enumerate(lengths):
        sl = slice(cu[n], cu[n + 1])
        alone = oracle.block_prologue(*[x[None, sl] for x in xs], *W)
        for a, b in zip(packed, alone):
            np.testing.assert_array_equal(a[sl], b[0])


def test_epilogue_invariants_and_closed_form():
    T, H, dv = 5, 3, 16
    o = rng.standard_normal((T, H, dv))
    z = rng.standard_normal((T, H, dv))
    g = rng.uniform(0.5, 1.5, dv)
    y = oracle.block_epilogue(o, z, g)
    # scale invariance of the RMS normalisation (up to eps = 1e-5 against mean(o^2) ~ 1)
    np.testing.assert_allclose(oracle.block_epilogue(2.0 * o, z, g), y, rtol=1e-4, atol=1e-6)
    # the normalised part has unit RMS: y / (g SiLU(z)) = o / rms(o)
    unit = y / (g * z * expit(z))
    ms = (o ** 2).mean(-1)
    np.testing.assert_allclose((unit ** 2).mean(-1), ms / (ms + 1e-5), rtol=1e-10)
    # constant o and z = ln 3, where SiLU(ln 3) = (3/4) ln 3 exactly
    c, ln3 = 0.8, math.log(3.0)
    yc = oracle.block_epilogue(np.full((1, 1, dv), c), np.full((1, 1, dv), ln3), g)
    np.testing.assert_allclose(yc[0, 0], c / math.sqrt(c * c + 1e-5) * g * 0.75 * ln3, rtol=1e-13)
