"""Exact rational brute force of the Gated Delta Rule-2 recurrence -- TEST INFRASTRUCTURE.

Tiny inputs only (pure-Python ``fractions.Fraction``).  This formulation is
deliberately different from the token loop in ``gdn2_oracle.c``: every token
becomes an explicit d_k x d_k transition matrix

    M_t = (I - k_t a_t^T) Diag(alpha_t),   a_t = b_t (.) k_t,

and the state is the affine product

    S_t = M_t ... M_1 S_0 + sum_{s<=t} M_t ... M_{s+1} k_s u_s^T,   u_s = w_s (.) v_s,

read out as o_t = S_t^T q_t.  This is the per-token update of
"NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section
"Gated DeltaNet-2の核心" (decay before the edit; key-side erase gate b_t;
value-side write gate w_t), under the erase reading k_t (b_t (.) k_t)^T.

Also the textbook recurrences of the special cases named in
"Jerarquía de Generalización" (needhelp.icu page): KDA
S = (I - beta k k^T) Diag(alpha) S + beta k v^T and Gated DeltaNet
S = alpha (I - beta k k^T) S + beta k v^T, DeltaNet S = (I - beta k k^T) S + beta k v^T.
"""
from fractions import Fraction


def _zeros(r, c):
    return [[Fraction(0)] * c for _ in range(r)]


def _eye(n):
    m = _zeros(n, n)
    for i in range(n):
        m[i][i] = Fraction(1)
    return m


def _mm(A, B):
    return [[sum((A[i][l] * B[l][j] for l in range(len(B))), Fraction(0)) for j in range(len(B[0]))]
            for i in range(len(A))]


def _add(A, B):
    return [[A[i][j] + B[i][j] for j in range(len(A[0]))] for i in range(len(A))]


def _outer(x, y):
    return [[xi * yj for yj in y] for xi in x]


def _readout(S, q):
    return [sum((S[i][j] * q[i] for i in range(len(q))), Fraction(0)) for j in range(len(S[0]))]


def gdn2_transition_products(q, k, v, alpha, b, w, S0):
    """Exact o (list of T vectors) and S_T for one head; inputs are nested lists of Fractions."""
    T, dk, dv = len(q), len(q[0]), len(v[0])
    Ms, writes = [], []
    for t in range(T):
        a = [b[t][i] * k[t][i] for i in range(dk)]
        u = [w[t][j] * v[t][j] for j in range(dv)]
        D = _zeros(dk, dk)
        for i in range(dk):
            D[i][i] = alpha[t][i]
        E = _eye(dk)
        ka = _outer(k[t], a)
        E = [[E[i][j] - ka[i][j] for j in range(dk)] for i in range(dk)]
        Ms.append(_mm(E, D))
        writes.append(_outer(k[t], u))
    outs = []
    S_t = None
    for t in range(T):
        prod = _eye(dk)
        for s in range(t, -1, -1):       # M_t ... M_1 applied to S0
            prod = _mm(prod, Ms[s])
        S_t = _mm(prod, S0)
        for s in range(t + 1):           # sum_s M_t ... M_{s+1} k_s u_s^T
            P = _eye(dk)
            for r in range(t, s, -1):
                P = _mm(P, Ms[r])
            S_t = _add(S_t, _mm(P, writes[s]))
        outs.append(_readout(S_t, q[t]))
    return outs, S_t


def kda_textbook(q, k, v, alpha, beta, S0):
    """KDA: S = (I - beta k k^T) Diag(alpha) S + beta k v^T; beta one scalar per token."""
    T, dk = len(q), len(q[0])
    S = [row[:] for row in S0]
    outs = []
    for t in range(T):
        D = _zeros(dk, dk)
        for i in range(dk):
            D[i][i] = alpha[t][i]
        E = _eye(dk)
        kk = _outer(k[t], k[t])
        E = [[E[i][j] - beta[t] * kk[i][j] for j in range(dk)] for i in range(dk)]
        S = _add(_mm(_mm(E, D), S), [[beta[t] * x for x in row] for row in _outer(k[t], v[t])])
        outs.append(_readout(S, q[t]))
    return outs, S


def gdn_textbook(q, k, v, alpha, beta, S0):
    """Gated DeltaNet: S = alpha (I - beta k k^T) S + beta k v^T; alpha, beta scalars per token."""
    T, dk = len(q), len(q[0])
    S = [row[:] for row in S0]
    outs = []
    for t in range(T):
        E = _eye(dk)
        kk = _outer(k[t], k[t])
        E = [[alpha[t] * (E[i][j] - beta[t] * kk[i][j]) for j in range(dk)] for i in range(dk)]
        S = _add(_mm(E, S), [[beta[t] * x for x in row] for row in _outer(k[t], v[t])])
        outs.append(_readout(S, q[t]))
    return outs, S
