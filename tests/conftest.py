import os
import sys

import numpy as np
import pytest

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (runs the sm_100a kernels)")


def make_case(T, dk, dv, H=1, N=1, seed=0, variant="full", s0="normal", shift=2.0, lengths=None,
              dtype="f32", device="cpu"):
    """Seeded small inputs through the shared generator; returns (torch dict, float64 numpy dict)."""
    import gdn2_workloads as W
    wl = W.Workload("case", B=N, T=T, H=H, dk=dk, dv=dv, dtype=dtype, s0=s0, alpha_shift=shift,
                    varlen=lengths is not None, variant=variant)
    d = W.chunk_inputs(wl, device=device, seed=seed, lengths=lengths)
    npd = {n: d[n].double().cpu().numpy() for n in ("q", "k", "v", "alpha", "b", "w", "S0")}
    npd["cu_seqlens"] = None if d["cu_seqlens"] is None else d["cu_seqlens"].cpu().numpy().astype(np.int64)
    return d, npd
