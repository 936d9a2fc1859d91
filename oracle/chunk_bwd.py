"""fp64 chunkwise form of the backward -- TEST INFRASTRUCTURE ONLY (a companion of the oracle).

The gradient of the Gated Delta Rule-2 recurrence (erase reading R1) taken through the chunkwise
WY form instead of the token loop: per chunk of C tokens, matrix products replace the per-token
chain.  The forward chunk form follows "Gated DeltaNet-2: Separando Borrado y Escritura en la
Atención Lineal" (needhelp.icu), "Innovaciones Técnicas", item 1 (the decay folded into erase
factors, one unit-lower-triangular system per chunk), and "[논문] 게이트형 DeltaNet-2"
(euno.news), "주요 기여"; the pages give no formula for the backward, which is the chain rule
through that form.  It is pinned against the token-loop gradient (``oracle.recurrent_bwd``).

For one chunk with entering state S (tokens r, i = 0..C-1, per key channel c):

    g_r = sum_{s<=r} log alpha_s,  F[r,i,c] = exp(g_rc - g_ic) (i <= r),  Gam = exp(g)
    a = b (.) k,  U = w (.) v,  A = Gam (.) a,  Qh = Gam (.) q,  Kh_i = exp(g_{C-1} - g_i) (.) k_i
    L[r,i] = sum_c a_rc k_ic F[r,i,c] (i < r),  P[r,i] = sum_c q_rc k_ic F[r,i,c] (i <= r)
    Y = U - A S,  Delta = (I + L)^{-1} Y,  O = Qh S + P Delta,  S' = Diag(Gam_{C-1}) S + Kh^T Delta

and backwards, given dO and dS' (the entering state's gradient of the next chunk):

    dDelta = P^T dO + Kh dS',   dY = (I + L)^{-T} dDelta,   dU = dY
    dS     = Qh^T dO + Diag(Gam_{C-1}) dS' - A^T dY
    dA = -dY S^T,  dQh = dO S^T,  dKh = Delta dS'^T,
    dL = -strict_lower(dY Delta^T),  dP = lower(dO Delta^T)

then through the factors to a, q, k and g (dg_r collects every exp(g_r ...) factor), and
dalpha_s = (sum_{r>=s} dg_r) / alpha_s inside the chunk.
"""
import numpy as np


def _chunk_forward(q, k, b, alpha, u, S):
    """One chunk's forward quantities (see the module docstring).  q, k, b, alpha: [C, dk];
    u: [C, dv]; S: [dk, dv] entering state."""
    C = q.shape[0]
    g = np.cumsum(np.log(alpha), axis=0)
    a = b * k
    low_strict = np.tril(np.ones((C, C)), -1)
    low_incl = np.tril(np.ones((C, C)))
    # F[r, i, c] = exp(g_rc - g_ic); only i <= r is used (above the diagonal the factors would grow)
    F = np.exp(g[:, None, :] - g[None, :, :]) * low_incl[:, :, None]
    L = np.einsum("rc,ic,ric->ri", a, k, F) * low_strict
    P = np.einsum("rc,ic,ric->ri", q, k, F) * low_incl
    Gam = np.exp(g)
    A, Qh = Gam * a, Gam * q
    EC = np.exp(g[-1][None, :] - g)  # [i, c]
    Kh = EC * k
    IL = np.eye(C) + L
    Delta = np.linalg.solve(IL, u - A @ S)
    S_next = Gam[-1][:, None] * S + Kh.T @ Delta
    return dict(g=g, a=a, F=F, L=L, P=P, Gam=Gam, A=A, Qh=Qh, EC=EC, Kh=Kh, IL=IL, Delta=Delta,
                S_next=S_next, low_strict=low_strict, low_incl=low_incl)


def _chunk_grads(q, k, b, alpha, u, S, dO, dSn):
    """One chunk backwards: returns (dq, dk, db, dalpha, dU, dS) with dS the entering state's
    gradient.  dO: [C, dv]; dSn: [dk, dv] gradient of the state the chunk hands on."""
    f = _chunk_forward(q, k, b, alpha, u, S)
    a, F, P, Gam, A, Qh, EC, Kh, IL, Delta = (f[x] for x in ("a", "F", "P", "Gam", "A", "Qh", "EC", "Kh",
                                                              "IL", "Delta"))
    low_strict, low_incl = f["low_strict"], f["low_incl"]
    # backward
    dDelta = P.T @ dO + Kh @ dSn
    dY = np.linalg.solve(IL.T, dDelta)
    dU = dY
    dS = Qh.T @ dO + Gam[-1][:, None] * dSn - A.T @ dY
    dA = -dY @ S.T
    dQh = dO @ S.T
    dKh = Delta @ dSn.T
    dL = -(dY @ Delta.T) * low_strict
    dP = (dO @ Delta.T) * low_incl
    # through L and P: every pair term a_rc k_ic F[r,i,c] (or q_rc k_ic F[r,i,c])
    WL = dL[:, :, None] * F  # [r, i, c]
    WP = dP[:, :, None] * F
    da = np.einsum("ric,ic->rc", WL, k)
    dq = np.einsum("ric,ic->rc", WP, k)
    dk = np.einsum("ric,rc->ic", WL, a) + np.einsum("ric,rc->ic", WP, q)
    tL = WL * a[:, None, :] * k[None, :, :]  # d/dg_r of each term is the term, d/dg_i its negative
    tP = WP * q[:, None, :] * k[None, :, :]
    dg = tL.sum(1) - tL.sum(0) + tP.sum(1) - tP.sum(0)
    # through A = Gam a, Qh = Gam q, Kh = exp(g_{C-1} - g) k and the carried Diag(Gam_{C-1}) S
    da += Gam * dA
    dg += dA * A
    dq += Gam * dQh
    dg += dQh * Qh
    dk += EC * dKh
    dg -= dKh * Kh
    dg[-1] += (dKh * Kh).sum(0)
    dg[-1] += Gam[-1] * (dSn * S).sum(1)
    # a = b (.) k; g = cumsum(log alpha)
    db = da * k
    dk += da * b
    dlog = np.cumsum(dg[::-1], axis=0)[::-1]
    dalpha = dlog / alpha
    return dq, dk, db, dalpha, dU, dS


def chunkwise_bwd(q, k, v, alpha, b, w, dO, S0=None, dST=None, cu_seqlens=None, chunk=64):
    """Gradients ``(dq, dk, dv, dalpha, db, dw, dS0)`` of ``L = <o, dO> + <S_T, dST>`` through the
    chunk form, chunk by chunk; same layouts as :func:`oracle.recurrent_bwd`."""
    arrs = [np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, b, w, dO)]
    q, k, v, alpha, b, w, dO = arrs
    if cu_seqlens is None:
        N, T, H, dk_ = q.shape
        spans = [(n, None, None) for n in range(N)]
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        N = len(cu) - 1
        H, dk_ = q.shape[1], q.shape[2]
        spans = [(n, int(cu[n]), int(cu[n + 1])) for n in range(N)]
    dv_ = v.shape[-1]
    grads = [np.zeros_like(x) for x in (q, k, v, alpha, b, w)]
    dS0 = np.zeros((N, H, dk_, dv_))
    for n, lo, hi in spans:
        for h in range(H):
            sel = (lambda x: x[n, :, h]) if lo is None else (lambda x: x[lo:hi, h])
            qs, ks, vs, als, bs, ws, dOs = (sel(x) for x in (q, k, v, alpha, b, w, dO))
            T_ = qs.shape[0]
            S = np.zeros((dk_, dv_)) if S0 is None else np.array(S0[n, h], dtype=np.float64)
            # forward over the chunks: the state entering each one
            enter = []
            for c0 in range(0, T_, chunk):
                c1 = min(c0 + chunk, T_)
                enter.append(S)
                S = _chunk_forward(qs[c0:c1], ks[c0:c1], bs[c0:c1], als[c0:c1], (ws * vs)[c0:c1], S)["S_next"]
            dS = np.zeros((dk_, dv_)) if dST is None else np.array(dST[n, h], dtype=np.float64)
            out = [sel(gr) for gr in grads]  # views into the gradient arrays
            for m in reversed(range(len(enter))):
                c0 = m * chunk
                c1 = min(c0 + chunk, T_)
                dq, dk, db, dal, dU, dS = _chunk_grads(qs[c0:c1], ks[c0:c1], bs[c0:c1], als[c0:c1],
                                                          (ws * vs)[c0:c1], enter[m], dOs[c0:c1], dS)
                out[0][c0:c1] = dq
                out[1][c0:c1] = dk
                out[2][c0:c1] = dU * ws[c0:c1]
                out[3][c0:c1] = dal
                out[4][c0:c1] = db
                out[5][c0:c1] = dU * vs[c0:c1]
            dS0[n, h] = dS
    return (*grads, dS0)
