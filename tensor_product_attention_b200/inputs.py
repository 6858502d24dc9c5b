"""Seeded synthetic inputs for the TPA hot path.

This module draws random numbers and rounds them to the storage dtype; it holds none
of TPA's arithmetic (no projection, RoPE, attention or softmax).  It is the one piece
shared by the CUDA path's callers (tests, bench) and the oracle checks.

Every draw comes from numpy's PCG64, seeded by (workload seed, stream tag, sequence
index), so any one sequence of a large workload can be regenerated on its own.
Values are drawn in fp32 and rounded to bf16 (round-to-nearest-even) for bf16
workloads; fp32 workloads keep the fp32 draw.

Decode workloads draw the cached B_K and the query's B_Q (or q) directly as already
rotated values: a RoPE rotation maps a pair of independent N(0, s^2) values to a pair
of independent N(0, s^2) values, so "b ~ N(0, 1/d_h), rotated at its position" has
the same distribution as a plain N(0, 1/d_h) draw.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

# stream tags, so that each tensor of a workload has its own random stream
_TAG = {"x": 1, "w": 2, "len": 3, "a_k": 4, "a_v": 5, "b_k": 6, "b_v": 7,
        "a_q": 8, "b_q": 9, "q": 10, "misc": 11, "wo": 12, "o": 13,
        "basis_k": 14, "basis_v": 15}


@dataclass(frozen=True)
class Workload:
    """One benchmark workload.  Sizes follow the TPA layer shapes it is named for."""

    name: str
    kind: str            # "prefill" (project + append + causal prefill) or "decode"
    dtype: str           # "f32" or "bf16"
    batch: int
    n_heads: int
    head_dim: int
    rank_q: int          # 0: TPA-KVonly (plain per-head query)
    rank_k: int
    rank_v: int
    rope_base: float
    seed: int
    seqlen: int = 0      # prefill: tokens per sequence
    d_model: int = 0     # prefill: model width
    context: tuple = field(default=(0, 0))   # decode: (min, max) context length
    shared_basis: bool = False   # B_K, B_V are layer parameters shared by all tokens

    def dims(self):
        return dict(d_model=self.d_model, n_heads=self.n_heads, head_dim=self.head_dim,
                    rank_q=self.rank_q, rank_k=self.rank_k, rank_v=self.rank_v,
                    shared_basis=self.shared_basis)


WORKLOADS = {
    w.name: w for w in (
        Workload("prefill_tiny_f32", "prefill", "f32", batch=1, seqlen=64, d_model=64,
                 n_heads=4, head_dim=16, rank_q=2, rank_k=1, rank_v=1,
                 rope_base=1e4, seed=1001),
        Workload("prefill_b8_s2048_d1024", "prefill", "bf16", batch=8, seqlen=2048,
                 d_model=1024, n_heads=16, head_dim=64, rank_q=6, rank_k=2, rank_v=2,
                 rope_base=1e4, seed=1002),
        Workload("decode_b64_ctx32k", "decode", "bf16", batch=64, context=(32768, 32768),
                 n_heads=16, head_dim=128, rank_q=6, rank_k=2, rank_v=2,
                 rope_base=1e4, seed=1003),
        Workload("kvonly_decode_b16_ctx64k_128k", "decode", "bf16", batch=16,
                 context=(65536, 131072), n_heads=32, head_dim=128, rank_q=0,
                 rank_k=2, rank_v=2, rope_base=5e5, seed=1004),
        Workload("layer_prefill_b4_s8192_d2048", "prefill", "bf16", batch=4, seqlen=8192,
                 d_model=2048, n_heads=16, head_dim=128, rank_q=6, rank_k=2, rank_v=2,
                 rope_base=1e4, seed=1005),
        # TPA-KVonly layer prefill: the KV-only decode shape (h 32, d_h 128, R 2, base
        # 5e5) with d_model = h * d_h; a measurement case for the KV-only prefill path
        Workload("kvonly_layer_prefill_b4_s8192_d4096", "prefill", "bf16", batch=4, seqlen=8192,
                 d_model=4096, n_heads=32, head_dim=128, rank_q=0, rank_k=2, rank_v=2,
                 rope_base=5e5, seed=1006),
        # shared-basis variant (B_K, B_V shared across tokens): the decode shape of
        # decode_b64_ctx32k with only A_K, A_V cached per token
        Workload("shared_basis_decode_b64_ctx32k", "decode", "bf16", batch=64,
                 context=(32768, 32768), n_heads=16, head_dim=128, rank_q=6, rank_k=2,
                 rank_v=2, rope_base=1e4, seed=1007, shared_basis=True),
    )
}


def rng(seed: int, tag: str, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, _TAG[tag], index]))


def normal(gen: np.random.Generator, shape, std: float) -> np.ndarray:
    out = gen.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def to_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    """fp32 numpy -> CPU torch tensor in the storage dtype (bf16 by RNE, or fp32)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def torch_dtype(dtype: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def factor_widths(n_heads, head_dim, rank_q, rank_k, rank_v, shared_basis=False):
    """Rows of the stacked projection weight: W_A_q, W_A_k, W_A_v, W_B_q, W_B_k, W_B_v.
    TPA-KVonly (rank_q = 0): no W_A_q rows, and the W_B_q block is the plain query
    projection with n_heads * head_dim rows.  Shared basis: no W_B_k, W_B_v rows."""
    kb = 0 if shared_basis else rank_k * head_dim
    vb = 0 if shared_basis else rank_v * head_dim
    return [n_heads * rank_q, n_heads * rank_k, n_heads * rank_v,
            (rank_q if rank_q > 0 else n_heads) * head_dim, kb, vb]


# ------------------------------------------------------------------- prefill inputs

def prefill_x(wl: Workload, b: int, seqlen: int | None = None, seed: int | None = None) -> torch.Tensor:
    """Hidden states of sequence ``b``: [seqlen, d_model] ~ N(0, 1)."""
    s = wl.seqlen if seqlen is None else seqlen
    return to_storage(normal(rng(wl.seed if seed is None else seed, "x", b), (s, wl.d_model), 1.0), wl.dtype)


def prefill_w(wl: Workload, seed: int | None = None) -> torch.Tensor:
    """The six stacked projection weights: [sum of widths, d_model] ~ N(0, 1/d_model)."""
    n = sum(factor_widths(wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v, wl.shared_basis))
    g = rng(wl.seed if seed is None else seed, "w")
    return to_storage(normal(g, (n, wl.d_model), 1.0 / np.sqrt(wl.d_model)), wl.dtype)


def output_w(wl: Workload, seed: int | None = None) -> torch.Tensor:
    """The output projection weight: [d_model, n_heads * head_dim] ~ N(0, 1/(h d_h))."""
    n = wl.n_heads * wl.head_dim
    g = rng(wl.seed if seed is None else seed, "wo")
    return to_storage(normal(g, (wl.d_model, n), 1.0 / np.sqrt(n)), wl.dtype)


def attn_out(wl: Workload, T: int, seed: int | None = None) -> torch.Tensor:
    """A stand-in attention output [T, h, d_h] ~ N(0, 1/d_h) (output-projection checks)."""
    g = rng(wl.seed if seed is None else seed, "o")
    return to_storage(normal(g, (T, wl.n_heads, wl.head_dim), 1.0 / np.sqrt(wl.head_dim)), wl.dtype)


def shared_basis(wl: Workload, seed: int | None = None) -> dict:
    """The layer's shared key and value basis (shared-basis variant), un-rotated:
    b_k [R_K, d_h], b_v [R_V, d_h] ~ N(0, 1/d_h), like the per-token B factors."""
    s = wl.seed if seed is None else seed
    sd = 1.0 / np.sqrt(wl.head_dim)
    return {"b_k": to_storage(normal(rng(s, "basis_k"), (wl.rank_k, wl.head_dim), sd), wl.dtype),
            "b_v": to_storage(normal(rng(s, "basis_v"), (wl.rank_v, wl.head_dim), sd), wl.dtype)}


# -------------------------------------------------------------------- decode inputs

def decode_lengths(wl: Workload) -> np.ndarray:
    lo, hi = wl.context
    if lo == hi:
        return np.full(wl.batch, lo, dtype=np.int64)
    return rng(wl.seed, "len").integers(lo, hi, size=wl.batch, endpoint=True).astype(np.int64)


def decode_sequence(wl: Workload, b: int, length: int, a_scale: float = 1.0) -> dict:
    """Cached factors of sequence ``b`` (B_K already rotated) and its one query.

    a_k, a_v: [length, h, R] ~ N(0, a_scale^2); b_k, b_v: [length, R, d] ~ N(0, 1/d);
    query a_q: [h, R_Q] ~ N(0, a_scale^2) and b_q: [R_Q, d] ~ N(0, 1/d), or, for
    TPA-KVonly, q: [h, d] ~ N(0, 1/d).  ``a_scale`` > 1 sharpens the softmax (the
    configured scales give a nearly uniform one).  Shared-basis workloads have no
    per-token b_k, b_v (see ``shared_basis``).
    """
    h, d, s = wl.n_heads, wl.head_dim, wl.seed
    sd = 1.0 / np.sqrt(d)
    out = {
        "a_k": to_storage(normal(rng(s, "a_k", b), (length, h, wl.rank_k), a_scale), wl.dtype),
        "a_v": to_storage(normal(rng(s, "a_v", b), (length, h, wl.rank_v), a_scale), wl.dtype),
    }
    if not wl.shared_basis:
        out["b_k"] = to_storage(normal(rng(s, "b_k", b), (length, wl.rank_k, d), sd), wl.dtype)
        out["b_v"] = to_storage(normal(rng(s, "b_v", b), (length, wl.rank_v, d), sd), wl.dtype)
    if wl.rank_q == 0:
        out["q"] = to_storage(normal(rng(s, "q", b), (h, d), sd), wl.dtype)
    else:
        out["a_q"] = to_storage(normal(rng(s, "a_q", b), (h, wl.rank_q), a_scale), wl.dtype)
        out["b_q"] = to_storage(normal(rng(s, "b_q", b), (wl.rank_q, d), sd), wl.dtype)
    return out


def prefill_factors(wl: Workload, b: int, n_query: int, n_keys: int, a_scale: float = 1.0) -> dict:
    """Factors for attention-only prefill checks of sequence ``b``: cached K/V factors
    for ``n_keys`` tokens (B_K already rotated) and query factors for ``n_query``
    tokens (B_Q already rotated), same distributions as ``decode_sequence``; for
    TPA-KVonly the query is ``q`` [n_query, h, d] ~ N(0, 1/d).  Shared-basis workloads
    have no per-token b_k, b_v."""
    h, d, s = wl.n_heads, wl.head_dim, wl.seed
    sd = 1.0 / np.sqrt(d)
    out = {
        "a_k": to_storage(normal(rng(s, "a_k", b), (n_keys, h, wl.rank_k), a_scale), wl.dtype),
        "a_v": to_storage(normal(rng(s, "a_v", b), (n_keys, h, wl.rank_v), a_scale), wl.dtype),
    }
    if not wl.shared_basis:
        out["b_k"] = to_storage(normal(rng(s, "b_k", b), (n_keys, wl.rank_k, d), sd), wl.dtype)
        out["b_v"] = to_storage(normal(rng(s, "b_v", b), (n_keys, wl.rank_v, d), sd), wl.dtype)
    if wl.rank_q == 0:
        out["q"] = to_storage(normal(rng(s, "q", b), (n_query, h, d), sd), wl.dtype)
    else:
        out["a_q"] = to_storage(normal(rng(s, "a_q", b), (n_query, h, wl.rank_q), a_scale), wl.dtype)
        out["b_q"] = to_storage(normal(rng(s, "b_q", b), (n_query, wl.rank_q, d), sd), wl.dtype)
    return out


def custom(name: str, base: Workload, **changes) -> Workload:
    """A copy of ``base`` with some fields changed (edge-case and reduced-size tests)."""
    from dataclasses import replace
    return replace(base, name=name, **changes)
