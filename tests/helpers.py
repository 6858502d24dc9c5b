"""Shared test plumbing: conversions, the error metric, and moving seeded inputs onto
the GPU.  Holds no TPA arithmetic."""
from __future__ import annotations

import os

import numpy as np
import torch

# Tolerances: max|gpu - oracle| / max|oracle| per output tensor.  1e-5 for fp32
# layers, 1e-2 for bf16 inputs with fp32 accumulation.
TOL = {"f32": 1e-5, "bf16": 1e-2}


def f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


# Every error rel_err measures during a test session, with the test that measured it
# (pytest's PYTEST_CURRENT_TEST); conftest.py writes them out at the end of the session.
RECORDED: list = []


def rel_err(gpu, ref) -> float:
    g, r = f64(gpu), f64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), "non-finite GPU output"
    err = float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300))
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").rsplit(" ", 1)[0]
    RECORDED.append({"test": test, "err": err, "elements": int(g.size)})
    return err


def dims_of(wl, binding):
    return binding.Dims(wl.d_model, wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v,
                        binding.BF16 if wl.dtype == "bf16" else binding.F32, int(wl.shared_basis))


def fill_cache(cache, b, seq: dict, start: int = 0):
    """Copy one sequence's seeded factors into cache slot b at [start, start+L) (plumbing)."""
    n = seq["a_k"].shape[0]
    for name in ("a_k", "a_v") if "b_k" not in seq else ("a_k", "a_v", "b_k", "b_v"):
        getattr(cache, name)[b, start:start + n].copy_(seq[name], non_blocking=False)


def oracle_dims(wl):
    import oracle
    return oracle.Dims(wl.d_model, wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v,
                       shared_basis=wl.shared_basis)
