"""gdn2 -- Gated Delta Rule-2 kernels for NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in ``include/gdn2.h``: argument marshalling
only.  Every step of the computation runs in the CUDA library
``_build/libgdn2.so``; PyTorch provides device memory and streams.  There is
no CPU fallback: if the library is missing or no GPU is present the calls
raise.

Entry points (same names as the C ABI):

* :func:`chunk_fwd` -- chunkwise parallel forward over whole sequences
  (``gdn2_chunk_fwd``);
* :func:`chunk_bwd` -- gradients through the chunkwise forward
  (``gdn2_chunk_bwd``);
* :func:`decode_step` -- one recurrent step for a batch of single tokens
  (``gdn2_decode_step``);
* :func:`recurrent_fwd` -- the token loop over whole sequences in either erase orientation
  (``gdn2_recurrent_fwd``);
* :func:`block_prologue`, :func:`block_epilogue` -- the work around the mixer
  in its block (``gdn2_block_prologue``, ``gdn2_block_epilogue``).
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_build", "libgdn2.so")

GDN2_OK, GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_CUDA, GDN2_ERR_TIMEOUT = range(5)
GDN2_F32, GDN2_BF16 = 0, 1
GDN2_ERASE_R1, GDN2_ERASE_R2 = 0, 1
_DTYPES = {torch.float32: GDN2_F32, torch.bfloat16: GDN2_BF16}

_lib = None


class Gdn2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib().gdn2_status_string(status).decode()}")


def lib():
    """The loaded ctypes library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"gdn2 CUDA library not built ({LIB_PATH} missing); "
                               "run `python -m gated_delta_rule_131_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci = ctypes.c_void_p, ctypes.c_int
        L.gdn2_chunk_fwd.argtypes = [vp] * 9 + [ci] * 6 + [vp, ci, vp]
        L.gdn2_chunk_fwd.restype = ci
        L.gdn2_chunk_fwd_noalloc.argtypes = [vp] * 9 + [ci] * 6 + [vp, ci, vp]
        L.gdn2_chunk_fwd_noalloc.restype = ci
        L.gdn2_block_prologue.argtypes = [vp] * 15 + [ci] * 6 + [vp, ci, vp]
        L.gdn2_block_prologue.restype = ci
        L.gdn2_block_epilogue.argtypes = [vp] * 4 + [ctypes.c_longlong, ci, ci, ci, vp]
        L.gdn2_block_epilogue.restype = ci
        L.gdn2_decode_step.argtypes = [vp] * 8 + [ci] * 5 + [vp]
        L.gdn2_decode_step.restype = ci
        L.gdn2_status_string.argtypes = [ci]
        L.gdn2_status_string.restype = ctypes.c_char_p
        L.gdn2_device_status.argtypes = [ci]
        L.gdn2_device_status.restype = ci
        L.gdn2_selftest_bounded_wait.argtypes = [ci, vp]
        L.gdn2_selftest_bounded_wait.restype = ci
        L.gdn2_launch_count.argtypes = []
        L.gdn2_chunk_fwd_workspace_bytes.argtypes = [ci] * 7 + [ci]
        L.gdn2_chunk_fwd_workspace_bytes.restype = ctypes.c_size_t
        L.gdn2_launch_count.restype = ctypes.c_uint64
        L.gdn2_recurrent_fwd.argtypes = [vp] * 9 + [ci] * 5 + [vp, ci, ci, vp]
        L.gdn2_recurrent_fwd.restype = ci
        L.gdn2_chunk_bwd.argtypes = [vp] * 16 + [ci] * 5 + [vp, ci, vp]
        L.gdn2_chunk_bwd.restype = ci
        L.gdn2_chunk_bwd_workspace_bytes.argtypes = [ci] * 6
        L.gdn2_chunk_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.gdn2_chunk_fwd_plan.argtypes = [ci] * 9 + [ctypes.POINTER(ChunkPlan)]
        L.gdn2_chunk_fwd_plan.restype = ci
        _lib = L
    return _lib


class ChunkPlan(ctypes.Structure):
    """``gdn2_chunk_plan`` of include/gdn2.h."""
    _fields_ = [("records", ctypes.c_longlong), ("wy_ctas", ctypes.c_longlong), ("state_ctas", ctypes.c_longlong),
                ("segments", ctypes.c_int), ("segment_chunks", ctypes.c_int), ("handover_sms", ctypes.c_int),
                ("handover_at", ctypes.c_longlong), ("order", ctypes.c_int), ("launches", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t)]


def chunk_fwd_plan(B, T, H, dk, dv, packed=False, sms=0, dtype=torch.bfloat16, chunk=64) -> dict:
    """What a tensor-core ``chunk_fwd`` call of this shape decides before it launches, for a device
    of ``sms`` SMs (0: the current one): records, grids, segments, the SM hand-over, the walking
    order, launches and workspace bytes.  Host only; raises ``Gdn2Error`` when the shape does not
    take the tensor-core path."""
    plan = ChunkPlan()
    st = lib().gdn2_chunk_fwd_plan(B, T, H, dk, dv, chunk, 1 if packed else 0, _DTYPES[dtype], sms, ctypes.byref(plan))
    if st != GDN2_OK:
        raise Gdn2Error(st, "chunk_fwd_plan")
    return {name: int(getattr(plan, name)) for name, _ in ChunkPlan._fields_}


def chunk_fwd_workspace_bytes(B, T, H, dk, dv, packed=False, dtype=torch.bfloat16, chunk=64) -> int:
    """Device bytes ``chunk_fwd`` takes from the library's pool for this shape (0: none)."""
    return int(lib().gdn2_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, 1 if packed else 0, _DTYPES[dtype]))


def launch_count() -> int:
    """Kernel launches issued by the library so far in this process."""
    return int(lib().gdn2_launch_count())


def device_status(reset=False) -> int:
    """Sticky device-side status (GDN2_OK or GDN2_ERR_TIMEOUT); synchronises with the device."""
    return int(lib().gdn2_device_status(1 if reset else 0))


def selftest_bounded_wait(limit_us=20000, stream=None):
    """Run the bounded-wait self-test (a wait that nothing completes gives up after limit_us)."""
    st = lib().gdn2_selftest_bounded_wait(int(limit_us), _stream(stream))
    if st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_selftest_bounded_wait")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_tensors(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("gdn2: all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("gdn2: all tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("gdn2: tensors on different devices")


def _chunk(entry, q, k, v, alpha, b, w, S0, cu_seqlens, chunk, o, S_T, output_final_state, stream):
    if cu_seqlens is None:
        B, T, H, dk = q.shape
    else:
        if cu_seqlens.dtype != torch.int32:
            raise ValueError("gdn2: cu_seqlens must be int32")
        B = cu_seqlens.numel() - 1
        T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DTYPES or any(x.dtype != q.dtype for x in (k, v, alpha, b, w)):
        raise ValueError("gdn2: q, k, v, alpha, b, w must share dtype float32 or bfloat16")
    if o is None:
        o = torch.empty(q.shape[:-1] + (dv,), dtype=q.dtype, device=q.device)
    if S_T is None and output_final_state:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if S0 is not None and S0.dtype != torch.float32:
        raise ValueError("gdn2: S0 must be float32")
    _check_tensors(q, k, v, alpha, b, w, S0, o, S_T, cu_seqlens)
    fn = getattr(lib(), entry)
    with torch.cuda.device(q.device):  # the library's pool and fixed workspace follow the current device
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o), _ptr(S_T),
                B, T, H, dk, dv, chunk, _ptr(cu_seqlens), _DTYPES[q.dtype], _stream(stream, q.device))
    if st != GDN2_OK:
        raise Gdn2Error(st, entry)
    return o, S_T


def chunk_fwd(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, chunk=64, o=None, S_T=None,
              output_final_state=True, stream=None):
    """Chunkwise forward.  Returns ``(o, S_T)`` (``S_T`` None if not requested).

    Dense: q, k, alpha, b ``[B, T, H, d_k]``; v, w ``[B, T, H, d_v]``.
    Packed (``cu_seqlens`` int32 ``[N+1]`` on the device): ``[T_total, H, d]``.
    ``S0`` / ``S_T``: ``[N, H, d_k, d_v]`` float32.
    """
    return _chunk("gdn2_chunk_fwd", q, k, v, alpha, b, w, S0, cu_seqlens, chunk, o, S_T,
                  output_final_state, stream)


def chunk_fwd_noalloc(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, chunk=64, o=None, S_T=None,
                      output_final_state=True, stream=None):
    """``chunk_fwd`` through the library's fixed workspace: the library allocates nothing.

    For callers that cannot let the library allocate device memory (all memory reserved up front,
    or owned by the caller's own memory manager).  The first call on a device looks the fixed
    array's address up; make it before any stream capture.  Shapes whose workspace exceeds
    ``NOALLOC_WORKSPACE_BYTES`` raise ``Gdn2Error`` (``GDN2_ERR_UNSUPPORTED``).  Calls that overlap
    in time on one device race on the shared workspace; calls on one stream are ordered.
    """
    return _chunk("gdn2_chunk_fwd_noalloc", q, k, v, alpha, b, w, S0, cu_seqlens, chunk, o, S_T,
                  output_final_state, stream)


NOALLOC_WORKSPACE_BYTES = 64 << 20  # GDN2_NOALLOC_WORKSPACE_BYTES in include/gdn2.h


def recurrent_fwd(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, erase=GDN2_ERASE_R1, o=None, S_T=None,
                  output_final_state=True, stream=None):
    """Token-by-token forward in either erase orientation (``GDN2_ERASE_R1`` or ``GDN2_ERASE_R2``).

    Same layouts and returns as :func:`chunk_fwd`; see ``gdn2_recurrent_fwd`` in ``include/gdn2.h``.
    """
    if cu_seqlens is None:
        B, T, H, dk = q.shape
    else:
        if cu_seqlens.dtype != torch.int32:
            raise ValueError("gdn2: cu_seqlens must be int32")
        B = cu_seqlens.numel() - 1
        T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DTYPES or any(x.dtype != q.dtype for x in (k, v, alpha, b, w)):
        raise ValueError("gdn2: q, k, v, alpha, b, w must share dtype float32 or bfloat16")
    if o is None:
        o = torch.empty(q.shape[:-1] + (dv,), dtype=q.dtype, device=q.device)
    if S_T is None and output_final_state:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    if S0 is not None and S0.dtype != torch.float32:
        raise ValueError("gdn2: S0 must be float32")
    _check_tensors(q, k, v, alpha, b, w, S0, o, S_T, cu_seqlens)
    with torch.cuda.device(q.device):
        st = lib().gdn2_recurrent_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                                      _ptr(S_T), B, T, H, dk, dv, _ptr(cu_seqlens), int(erase), _DTYPES[q.dtype],
                                      _stream(stream, q.device))
    if st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_recurrent_fwd")
    return o, S_T


def chunk_bwd(q, k, v, alpha, b, w, dO, S0=None, dS_T=None, cu_seqlens=None, want_dS0=True, stream=None):
    """Gradients of a loss through ``chunk_fwd`` given ``dO = dL/do`` and ``dS_T = dL/dS_T`` (or None).

    Returns ``(dq, dk, dv, dalpha, db, dw, dS0)`` in the layouts and dtype of the inputs (``dS0``
    float32 ``[N, H, d_k, d_v]``, None unless ``want_dS0``).  See ``gdn2_chunk_bwd`` in ``include/gdn2.h``.
    """
    if cu_seqlens is None:
        B, T, H, dk = q.shape
    else:
        if cu_seqlens.dtype != torch.int32:
            raise ValueError("gdn2: cu_seqlens must be int32")
        B = cu_seqlens.numel() - 1
        T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DTYPES or any(x.dtype != q.dtype for x in (k, v, alpha, b, w, dO)):
        raise ValueError("gdn2: q, k, v, alpha, b, w, dO must share dtype float32 or bfloat16")
    if any(x is not None and x.dtype != torch.float32 for x in (S0, dS_T)):
        raise ValueError("gdn2: S0 and dS_T must be float32")
    grads = [torch.empty_like(x) for x in (q, k, v, alpha, b, w)]
    dS0 = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device) if want_dS0 else None
    _check_tensors(q, k, v, alpha, b, w, dO, S0, dS_T, *grads, dS0, cu_seqlens)
    with torch.cuda.device(q.device):
        st = lib().gdn2_chunk_bwd(*[_ptr(x) for x in (q, k, v, alpha, b, w, S0, dO, dS_T)],
                                  *[_ptr(x) for x in grads], _ptr(dS0), B, T, H, dk, dv, _ptr(cu_seqlens),
                                  _DTYPES[q.dtype], _stream(stream, q.device))
    if st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_chunk_bwd")
    dq, dk_, dv_, dalpha, db, dw = grads
    return dq, dk_, dv_, dalpha, db, dw, dS0


def chunk_bwd_workspace_bytes(B, T, H, d_k, d_v, packed=False):
    """Device bytes ``chunk_bwd`` takes from the library's pool for this shape."""
    return int(lib().gdn2_chunk_bwd_workspace_bytes(B, T, H, d_k, d_v, int(bool(packed))))


def block_prologue(xq, xk, xv, xa, xb, xw, conv_q, conv_k, conv_v, cu_seqlens=None, stream=None):
    """The mixer's inputs from the projections' outputs: returns ``(q, k, v, alpha, b, w)``.

    Token tensors ``[B, T, H, d]`` (dense) or ``[T_total, H, d]`` with ``cu_seqlens``; convolution
    weights ``[H*d, K]`` float32 with K in 1..4.  See ``gdn2_block_prologue`` in ``include/gdn2.h``.
    """
    if cu_seqlens is None:
        B, T, H, dk = xq.shape
    else:
        if cu_seqlens.dtype != torch.int32:
            raise ValueError("gdn2: cu_seqlens must be int32")
        B = cu_seqlens.numel() - 1
        T, H, dk = xq.shape
    dv = xv.shape[-1]
    if xq.dtype not in _DTYPES or any(x.dtype != xq.dtype for x in (xk, xv, xa, xb, xw)):
        raise ValueError("gdn2: the pre-activations must share dtype float32 or bfloat16")
    if any(W.dtype != torch.float32 for W in (conv_q, conv_k, conv_v)):
        raise ValueError("gdn2: convolution weights must be float32")
    outs = [torch.empty_like(x) for x in (xq, xk, xv, xa, xb, xw)]
    _check_tensors(xq, xk, xv, xa, xb, xw, conv_q, conv_k, conv_v, *outs, cu_seqlens)
    with torch.cuda.device(xq.device):
        st = lib().gdn2_block_prologue(*[_ptr(x) for x in (xq, xk, xv, xa, xb, xw, conv_q, conv_k, conv_v)],
                                       *[_ptr(x) for x in outs], B, T, H, dk, dv, conv_q.shape[1],
                                       _ptr(cu_seqlens), _DTYPES[xq.dtype], _stream(stream, xq.device))
    if st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_block_prologue")
    return tuple(outs)


def block_epilogue(o, gate, norm_weight, y=None, stream=None):
    """``y = RMSNorm(o) * norm_weight * SiLU(gate)`` per (token, head) over d_v; ``y`` may be ``o``."""
    H, dv = o.shape[-2], o.shape[-1]
    tokens = o.numel() // (H * dv)
    if o.dtype not in _DTYPES or gate.dtype != o.dtype:
        raise ValueError("gdn2: o and gate must share dtype float32 or bfloat16")
    if norm_weight.dtype != torch.float32:
        raise ValueError("gdn2: norm_weight must be float32")
    if y is None:
        y = torch.empty_like(o)
    _check_tensors(o, gate, norm_weight, y)
    with torch.cuda.device(o.device):
        st = lib().gdn2_block_epilogue(_ptr(o), _ptr(gate), _ptr(norm_weight), _ptr(y), tokens, H, dv,
                                       _DTYPES[o.dtype], _stream(stream, o.device))
    if st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_block_epilogue")
    return y


def decode_step(q, k, v, alpha, b, w, S, o=None, stream=None):
    """One decode step: updates ``S`` ``[B, H, d_k, d_v]`` in place, returns ``o`` ``[B, H, d_v]``."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DTYPES or any(x.dtype != q.dtype for x in (k, v, alpha, b, w)):
        raise ValueError("gdn2: q, k, v, alpha, b, w must share dtype float32 or bfloat16")
    if S.dtype != torch.float32:
        raise ValueError("gdn2: S must be float32")
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    _check_tensors(q, k, v, alpha, b, w, S, o)
    with torch.cuda.device(q.device):
        st = lib().gdn2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S),
                                    _ptr(o), B, H, dk, dv, _DTYPES[q.dtype], _stream(stream, q.device))
    if st != GDN2_OK:
        raise Gdn2Error(st, "gdn2_decode_step")
    return o
