"""Seeded synthetic inputs for the Gated Delta Rule-2 kernels and the oracle.

This module holds no arithmetic of the recurrence.  It only draws the inputs
that both the CUDA path and the fp64 oracle consume, with the shapes and value
distributions of the workloads the pages' 1.3B-parameter model implies
(16 heads x 128 channels), since the pages' own data (FineWeb-Edu, RULER,
LAMBADA) and trained weights are not available:

* q, k ~ N(0, 1), then L2-normalised over d_k per (token, head);
* v ~ N(0, 1);
* alpha = exp(-softplus(x - shift)), x ~ N(0, 1), per key channel
  (shift 2, or 4 for the retention-biased long-context workload);
* b = sigmoid(x) per key channel, w = sigmoid(x) per value channel;
* S0 ~ N(0, 0.02^2) fp32, or zeros;
* gate variants: "full" (per-channel b, w), "kda" (b = w = one scalar beta
  per token-head), "gdn" (also one scalar alpha per token-head).

Every sequence (and, for decode, every step) draws from its own generator,
seeded by a hash of (seed, tag, index), so any subset of sequences can be
regenerated alone -- on the same device -- with values identical to the full
batch.  Values are drawn in fp32 and then cast to the workload dtype; the
oracle consumes the cast values.
"""
from dataclasses import dataclass, replace
from typing import List, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int                 # batch size (dense) or number of sequences (packed)
    T: int                 # sequence length (dense); max length (packed)
    H: int
    dk: int
    dv: int
    chunk: int = 64
    dtype: str = "bf16"    # "f32" or "bf16": dtype of q, k, v, alpha, b, w, o
    s0: str = "normal"     # "normal" (N(0, 0.02^2)) or "zeros"
    alpha_shift: float = 2.0
    varlen: bool = False   # lengths uniform in [1, T], packed with cu_seqlens
    decode_steps: int = 0  # > 0: a decode workload of that many single-token steps
    variant: str = "full"  # "full" | "kda" | "gdn"


WORKLOADS = {
    # small case the oracle finishes in seconds; all fp32
    "oracle_small": Workload("oracle_small", B=1, H=2, T=256, dk=64, dv=64, dtype="f32", s0="zeros"),
    # one layer of the 1.3B model, forward
    "layer_1p3b": Workload("layer_1p3b", B=4, H=16, T=2048, dk=128, dv=128),
    # long-context forward with retention-biased decay
    "long_context": Workload("long_context", B=1, H=16, T=65536, dk=128, dv=128, alpha_shift=4.0),
    # recurrent decode: 256 sequences x 16 heads, 1024 single-token steps
    "decode": Workload("decode", B=256, H=16, T=1, dk=128, dv=128, decode_steps=1024),
    # packed varlen stress, three gate variants
    "varlen": Workload("varlen", B=32, H=32, T=8192, dk=128, dv=256, varlen=True),
    "varlen_kda": Workload("varlen_kda", B=32, H=32, T=8192, dk=128, dv=256, varlen=True, variant="kda"),
    "varlen_gdn": Workload("varlen_gdn", B=32, H=32, T=8192, dk=128, dv=256, varlen=True, variant="gdn"),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _mix(*key) -> int:
    """Deterministic 63-bit seed from a tuple of ints/strings (splitmix64 finaliser)."""
    h = 0x9E3779B97F4A7C15
    for part in key:
        if isinstance(part, str):
            for ch in part.encode():
                h = ((h ^ ch) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
        else:
            h = (h ^ (int(part) & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
        h = (h + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
        z = h
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        h = z ^ (z >> 31)
    return h & 0x7FFFFFFFFFFFFFFF


def _gen(device, *key) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(_mix(*key))
    return g


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-6)


def token_inputs(wl: Workload, length: int, device, seed: int, tag: str, index: int,
                 H: Optional[int] = None) -> dict:
    """Draw q, k, v, alpha, b, w of shape [length, H, d] for one sequence (or one decode step)."""
    H = wl.H if H is None else H
    g = _gen(device, seed, tag, index)
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    q = torch.randn(length, H, wl.dk, **f32)
    k = torch.randn(length, H, wl.dk, **f32)
    v = torch.randn(length, H, wl.dv, **f32)
    xa = torch.randn(length, H, wl.dk, **f32)
    xb = torch.randn(length, H, wl.dk, **f32)
    xw = torch.randn(length, H, wl.dv, **f32)
    q, k = _l2n(q), _l2n(k)
    alpha = torch.exp(-torch.nn.functional.softplus(xa - wl.alpha_shift))
    b = torch.sigmoid(xb)
    w = torch.sigmoid(xw)
    if wl.variant in ("kda", "gdn"):
        beta = torch.sigmoid(xb[..., :1])
        b = beta.expand(length, H, wl.dk)
        w = beta.expand(length, H, wl.dv)
    if wl.variant == "gdn":
        alpha = torch.exp(-torch.nn.functional.softplus(xa[..., :1] - wl.alpha_shift)).expand(length, H, wl.dk)
    dt = TORCH_DTYPE[wl.dtype]
    return {n: t.to(dt).contiguous() for n, t in
            dict(q=q, k=k, v=v, alpha=alpha, b=b, w=w).items()}


def initial_state(wl: Workload, n_seq: int, device, seed: int, index0: int = 0,
                  indices: Optional[List[int]] = None) -> torch.Tensor:
    """S0 [n_seq, H, d_k, d_v] fp32; sequence i (global index) draws from its own generator."""
    idx = list(range(index0, index0 + n_seq)) if indices is None else list(indices)
    out = torch.zeros(len(idx), wl.H, wl.dk, wl.dv, device=device, dtype=torch.float32)
    if wl.s0 == "normal":
        for j, i in enumerate(idx):
            g = _gen(device, seed, "S0", i)
            out[j] = torch.randn(wl.H, wl.dk, wl.dv, device=device, dtype=torch.float32,
                                 generator=g) * 0.02
    return out


def shard(n_global: int, world_size: int, rank: int) -> List[int]:
    """Global sequence indices owned by ``rank``: contiguous blocks, sizes differing by at most one."""
    per, extra = divmod(n_global, world_size)
    start = rank * per + min(rank, extra)
    return list(range(start, start + per + (1 if rank < extra else 0)))


def seq_lengths(wl: Workload, seed: int) -> List[int]:
    """Per-sequence lengths: T for dense workloads, uniform in [1, T] for packed ones."""
    if not wl.varlen:
        return [wl.T] * wl.B
    g = _gen("cpu", seed, "lengths")
    return [int(x) for x in torch.randint(1, wl.T + 1, (wl.B,), generator=g)]


def chunk_inputs(wl: Workload, device="cpu", seed: int = 0, lengths: Optional[List[int]] = None,
                 indices: Optional[List[int]] = None) -> dict:
    """All inputs of a chunk_fwd workload (or of the sequences ``indices`` of it, e.g. one rank's shard).

    Dense: q, k, alpha, b [B, T, H, d_k]; v, w [B, T, H, d_v]; cu_seqlens None.
    Packed: the same tensors are [T_total, H, d]; cu_seqlens int32 [N+1] on ``device``.
    Also returns S0 [N, H, d_k, d_v] fp32 and the list of lengths.
    """
    all_lens = seq_lengths(wl, seed) if lengths is None else list(lengths)
    idx = list(range(len(all_lens))) if indices is None else list(indices)
    if lengths is None and not wl.varlen and indices is not None:
        all_lens = [wl.T] * (max(idx) + 1 if idx else 0)
    lens = [all_lens[i] for i in idx]
    per = [token_inputs(wl, all_lens[i], device, seed, "seq", i) for i in idx]
    names = ("q", "k", "v", "alpha", "b", "w")
    if wl.varlen:
        out = {n: torch.cat([p[n] for p in per], 0) for n in names}
        cu = [0]
        for L in lens:
            cu.append(cu[-1] + L)
        out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    else:
        out = {n: torch.stack([p[n] for p in per], 0) for n in names}
        out["cu_seqlens"] = None
    out["S0"] = initial_state(wl, len(lens), device, seed, indices=idx)
    out["lengths"] = lens
    return out


def block_inputs(wl: Workload, device="cpu", seed: int = 0, conv_len: int = 4,
                 lengths: Optional[List[int]] = None) -> dict:
    """Inputs of the block prologue and epilogue around the mixer (the projections' outputs).

    Token tensors xq, xk, xa, xb [.., H, d_k] and xv, xw, z [.., H, d_v] ~ N(0, 1) (xa shifted by
    -alpha_shift, the bias of the decay branch), cast to the workload dtype; dense [B, T, H, d] or
    packed [T_total, H, d] with cu_seqlens.  Convolution weights conv_q, conv_k [H*d_k, K] and
    conv_v [H*d_v, K] ~ N(0, 1/K) fp32; norm_weight [d_v] ~ U(0.5, 1.5) fp32.
    """
    lens = seq_lengths(wl, seed) if lengths is None else list(lengths)
    dt = TORCH_DTYPE[wl.dtype]
    per = []
    for i, L in enumerate(lens):
        g = _gen(device, seed, "block_seq", i)
        f32 = dict(device=device, dtype=torch.float32, generator=g)
        d = {n: torch.randn(L, wl.H, wl.dk if n in ("xq", "xk", "xa", "xb") else wl.dv, **f32)
             for n in ("xq", "xk", "xv", "xa", "xb", "xw", "z")}
        d["xa"] = d["xa"] - wl.alpha_shift
        per.append({n: t.to(dt) for n, t in d.items()})
    names = ("xq", "xk", "xv", "xa", "xb", "xw", "z")
    if wl.varlen:
        out = {n: torch.cat([p[n] for p in per], 0).contiguous() for n in names}
        cu = [0]
        for L in lens:
            cu.append(cu[-1] + L)
        out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    else:
        out = {n: torch.stack([p[n] for p in per], 0).contiguous() for n in names}
        out["cu_seqlens"] = None
    g = _gen(device, seed, "block_weights")
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    out["conv_q"] = torch.randn(wl.H * wl.dk, conv_len, **f32) / conv_len ** 0.5
    out["conv_k"] = torch.randn(wl.H * wl.dk, conv_len, **f32) / conv_len ** 0.5
    out["conv_v"] = torch.randn(wl.H * wl.dv, conv_len, **f32) / conv_len ** 0.5
    out["norm_weight"] = torch.rand(wl.dv, **f32) + 0.5
    out["S0"] = initial_state(wl, len(lens), device, seed)
    out["lengths"] = lens
    return out


def sequence_inputs(wl: Workload, index: int, device="cpu", seed: int = 0) -> dict:
    """The inputs of one sequence of ``chunk_inputs`` alone: [len, H, d] tensors and S0 [H, d_k, d_v]."""
    L = seq_lengths(wl, seed)[index]
    d = token_inputs(wl, L, device, seed, "seq", index)
    d["S0"] = initial_state(wl, 1, device, seed, index0=index)[0]
    return d


def decode_state(wl: Workload, device="cpu", seed: int = 0) -> torch.Tensor:
    """Decode state S [B, H, d_k, d_v] fp32 ~ N(0, 0.02^2)."""
    g = _gen(device, seed, "decode_S")
    return torch.randn(wl.B, wl.H, wl.dk, wl.dv, device=device, dtype=torch.float32, generator=g) * 0.02


def decode_token_inputs(wl: Workload, step: int, device="cpu", seed: int = 0) -> dict:
    """Single-token inputs of decode step ``step``: [B, H, d] tensors."""
    return token_inputs(wl, wl.B, device, seed, "decode_step", step)


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return replace(wl, **kw)
