"""fp64 CPU oracle for the Gated Delta Rule-2 recurrence -- TEST INFRASTRUCTURE.

Only tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  It is independent of the CUDA library: it shares no
code with it and never calls it.

The arithmetic lives in ``gdn2_oracle.c`` (plain loops, fp64, OpenMP over
(sequence, head)); this module only marshals numpy arrays through ctypes.

Functions and the passages they follow:

* :func:`recurrent` -- the token-by-token recurrence (decay on the key axis
  first, erase gated per key channel by ``b``, write ``k (w*v)^T`` gated per
  value channel by ``w``, readout ``o_t = S_t^T q_t``), from
  "NVIDIA AIがGated DeltaNet-2を発表" (ai.warp-studio.com), section
  "Gated DeltaNet-2の核心", and "[논문] 게이트형 DeltaNet-2" (euno.news),
  section "방법론".  This is the oracle.
* :func:`chunkwise` -- the chunkwise WY form of the same recurrence in fp64,
  from "Gated DeltaNet-2: Separando Borrado y Escritura en la Atención Lineal"
  (needhelp.icu), "Innovaciones Técnicas", item 1; pinned against
  :func:`recurrent`.
* :func:`recurrent_planted` -- the recurrence with one planted mistake, used
  only to show that the pins catch each mistake.
* :func:`block_prologue`, :func:`block_epilogue` -- the elementwise and
  short-convolution work around the mixer in its block (short causal
  convolution, SiLU, L2 normalisation of q and k; decay and gates; RMS
  normalisation times a SiLU output gate), from "NVIDIA AIがGated DeltaNet-2を発表"
  (ai.warp-studio.com), section "アーキテクチャとパフォーマンスベンチマーク";
  the code is in ``block_oracle.c``.
* :func:`recurrent_bwd` -- the reverse-mode gradient of :func:`recurrent`
  (erase reading R1) with respect to q, k, v, alpha, b, w and S0, taken step by
  step backwards through the same token loop; the code is in ``bwd_oracle.c``.
* :func:`chunkwise_bwd` -- the same gradient taken through the chunkwise WY form
  (a companion, in numpy, ``chunk_bwd.py``); pinned against :func:`recurrent_bwd`.
"""
import ctypes
import os

import numpy as np

from . import build as _build
from .chunk_bwd import chunkwise_bwd  # noqa: F401

ERASE_R1 = 0  # S_t = (I - k (b*k)^T) Diag(alpha) S + k (w*v)^T   (adopted reading)
ERASE_R2 = 1  # S_t = (I - (b*k) k^T) Diag(alpha) S + k (w*v)^T

PLANTS = {
    1: "no decay",
    2: "erase sign flipped",
    3: "readout before the edit",
    4: "decay after the edit",
    5: "write gate ignored",
    6: "erase gate ignored",
    7: "readout transposed",
    8: "erase probe reads the undecayed state",
    9: "erase and write gates swapped",
}

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        ci = ctypes.c_int
        common = [dp] * 6 + [dp, dp, dp] + [ci] * 5 + [i64p]
        lib.oracle_gdn2_recurrent.argtypes = common + [ci, ci]
        lib.oracle_gdn2_recurrent.restype = ci
        lib.oracle_gdn2_recurrent_planted.argtypes = common + [ci]
        lib.oracle_gdn2_recurrent_planted.restype = ci
        lib.oracle_gdn2_chunkwise.argtypes = common + [ci, ci]
        lib.oracle_gdn2_chunkwise.restype = ci
        lib.oracle_plant_count.restype = ci
        lib.oracle_block_prologue.argtypes = [dp] * 15 + [ci] * 6 + [i64p]
        lib.oracle_block_prologue.restype = ci
        lib.oracle_block_epilogue.argtypes = [dp] * 4 + [ctypes.c_int64, ci, ci]
        lib.oracle_block_epilogue.restype = ci
        lib.oracle_gdn2_recurrent_bwd.argtypes = [dp] * 16 + [ci] * 5 + [i64p, ci]
        lib.oracle_gdn2_recurrent_bwd.restype = ci
        lib.oracle_max_threads.restype = ci
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the oracle's OpenMP loops use by default."""
    return int(_load().oracle_max_threads())


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shapes(q, v, cu_seqlens):
    if cu_seqlens is None:
        N, T, H, dk = q.shape
    else:
        N = len(cu_seqlens) - 1
        T = int(cu_seqlens[-1])
        _, H, dk = q.shape
    dv = v.shape[-1]
    return N, T, H, dk, dv


def _prep(q, k, v, alpha, b, w, S0, cu_seqlens):
    q, k, v, alpha, b, w = (_f64(x) for x in (q, k, v, alpha, b, w))
    cu = None if cu_seqlens is None else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N, T, H, dk, dv = _shapes(q, v, cu)
    for x, d in ((k, dk), (alpha, dk), (b, dk), (w, dv)):
        if x.shape[:-1] != q.shape[:-1] or x.shape[-1] != d:
            raise ValueError("token tensors disagree in shape")
    S0 = None if S0 is None else _f64(S0).reshape(N, H, dk, dv)
    o = np.zeros(q.shape[:-1] + (dv,), dtype=np.float64)
    ST = np.zeros((N, H, dk, dv), dtype=np.float64)
    cup = None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    return (q, k, v, alpha, b, w, S0, o, ST, N, T, H, dk, dv, cu, cup)


def recurrent(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, orientation=ERASE_R1, nthreads=0):
    """Token-by-token fp64 recurrence.  Returns ``(o, S_T)`` as float64 arrays.

    Dense layout: q, k, alpha, b ``[N, T, H, d_k]``; v, w ``[N, T, H, d_v]``.
    Packed layout (``cu_seqlens`` given, ``N+1`` offsets): ``[T_total, H, d]``.
    ``S0`` is ``[N, H, d_k, d_v]`` or ``None`` (zeros).
    """
    (q, k, v, alpha, b, w, S0, o, ST, N, T, H, dk, dv, cu, cup) = _prep(q, k, v, alpha, b, w, S0, cu_seqlens)
    rc = _load().oracle_gdn2_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                                       _ptr(S0), _ptr(o), _ptr(ST), N, T, H, dk, dv, cup,
                                       int(orientation), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gdn2_recurrent failed with {rc}")
    return o, ST


def recurrent_bwd(q, k, v, alpha, b, w, dO, S0=None, dST=None, cu_seqlens=None, nthreads=0):
    """Gradients of a loss L through the token loop, given ``dO = dL/do`` (the layout of o) and
    ``dST = dL/dS_T`` (``[N, H, d_k, d_v]`` or ``None``: zero).

    Returns ``(dq, dk, dv, dalpha, db, dw, dS0)`` as float64 arrays in the layouts of their inputs.
    """
    (q, k, v, alpha, b, w, S0, o, ST, N, T, H, dk_, dv_, cu, cup) = _prep(q, k, v, alpha, b, w, S0, cu_seqlens)
    dO = _f64(dO)
    if dO.shape != o.shape:
        raise ValueError("dO must have the layout of o")
    dST = None if dST is None else _f64(dST).reshape(N, H, dk_, dv_)
    grads = [np.zeros_like(x) for x in (q, k, v, alpha, b, w)]
    dS0 = np.zeros((N, H, dk_, dv_), dtype=np.float64)
    rc = _load().oracle_gdn2_recurrent_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                                           _ptr(S0), _ptr(dO), _ptr(dST), *[_ptr(g) for g in grads],
                                           _ptr(dS0), N, T, H, dk_, dv_, cup, int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gdn2_recurrent_bwd failed with {rc}")
    return (*grads, dS0)


def recurrent_planted(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, plant=0):
    """The recurrence with planted mistake ``plant`` (see :data:`PLANTS`)."""
    (q, k, v, alpha, b, w, S0, o, ST, N, T, H, dk, dv, cu, cup) = _prep(q, k, v, alpha, b, w, S0, cu_seqlens)
    rc = _load().oracle_gdn2_recurrent_planted(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                                               _ptr(S0), _ptr(o), _ptr(ST), N, T, H, dk, dv, cup, int(plant))
    if rc != 0:
        raise RuntimeError(f"oracle_gdn2_recurrent_planted failed with {rc}")
    return o, ST


def chunkwise(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, chunk=64, nthreads=0):
    """fp64 chunkwise WY form (erase reading R1).  Returns ``(o, S_T)``."""
    (q, k, v, alpha, b, w, S0, o, ST, N, T, H, dk, dv, cu, cup) = _prep(q, k, v, alpha, b, w, S0, cu_seqlens)
    rc = _load().oracle_gdn2_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                                       _ptr(S0), _ptr(o), _ptr(ST), N, T, H, dk, dv, cup,
                                       int(chunk), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gdn2_chunkwise failed with {rc}")
    return o, ST


def decode_step(q, k, v, alpha, b, w, S):
    """One recurrent step for a batch of single tokens.

    q, k, alpha, b ``[B, H, d_k]``; v, w ``[B, H, d_v]``; S ``[B, H, d_k, d_v]``.
    Returns ``(o [B, H, d_v], S_new)``.
    """
    ex = lambda x: _f64(x)[:, None]  # noqa: E731  -- a length-1 sequence per batch entry
    o, ST = recurrent(ex(q), ex(k), ex(v), ex(alpha), ex(b), ex(w), S0=S)
    return o[:, 0], ST


def block_prologue(xq, xk, xv, xa, xb, xw, Wq, Wk, Wv, cu_seqlens=None):
    """q, k, v, alpha, b, w from the projections' outputs (see ``block_oracle.c``).

    Dense: token tensors ``[N, T, H, d]``; packed: ``[T_total, H, d]`` with ``cu_seqlens`` (N+1).
    Convolution weights ``[H*d, K]``.  Returns six fp64 arrays shaped like the inputs.
    """
    xq, xk, xv, xa, xb, xw, Wq, Wk, Wv = (_f64(x) for x in (xq, xk, xv, xa, xb, xw, Wq, Wk, Wv))
    if cu_seqlens is None:
        N, T, H, dk = xq.shape
        cu = None
    else:
        T, H, dk = xq.shape
        N = len(cu_seqlens) - 1
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    dv = xv.shape[-1]
    K = Wq.shape[1]
    outs = [np.zeros_like(x) for x in (xq, xk, xv, xa, xb, xw)]
    i64p = ctypes.POINTER(ctypes.c_int64)
    rc = _load().oracle_block_prologue(*[_ptr(x) for x in (xq, xk, xv, xa, xb, xw, Wq, Wk, Wv)],
                                       *[_ptr(x) for x in outs], N, T, H, dk, dv, K,
                                       None if cu is None else cu.ctypes.data_as(i64p))
    if rc != 0:
        raise ValueError(f"oracle_block_prologue failed ({rc})")
    return tuple(outs)


def block_epilogue(o, z, g):
    """y = RMSNorm(o) * g * SiLU(z) per (token, head) over d_v (see ``block_oracle.c``)."""
    o, z, g = _f64(o), _f64(z), _f64(g)
    H, dv = o.shape[-2], o.shape[-1]
    tokens = o.size // (H * dv)
    y = np.zeros_like(o)
    rc = _load().oracle_block_epilogue(_ptr(o), _ptr(z), _ptr(g), _ptr(y), tokens, H, dv)
    if rc != 0:
        raise ValueError(f"oracle_block_epilogue failed ({rc})")
    return y
