"""Plain, slow, fp64 CPU oracle for the Tensor Product Attention (TPA) hot path.

TEST INFRASTRUCTURE ONLY.  This module exists to check the CUDA path, never to stand
in for it: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and ``--impl reference``) may import it.  The product path (the
CUDA library under ``tensor_product_attention_b200/`` and its Python binding) never
imports it, and this module imports nothing from the product.  It takes plain numpy
arrays and returns fp64 numpy arrays.

Sources, cited by page title and section (formulas on these pages were flattened
from HTML; where they are silent or garbled the reading taken is stated inline):

  [review]  "【拜读】Tensor Product Attention Is All You Need 姚期智团队开源兼容RoPE位置编码"
            (coreui.cn): 核心机制总结 §3 公式描述 (the Q/K/V factor formulas),
            关键问题及回答 问题2 (RoPE pre-rotation of B_K), 代码 类定义与初始化
            (projection and cache shapes), 代码 前向传播 (the forward pass).
  [popsci]  "张量积注意力（TPA）：让注意力机制飞得更高、跑得更快的秘密武器" (jieyibu.net):
            Ⅱ.1 从传统注意力机制说起 (softmax(QK^T/sqrt(d_k))V).
  [explain] "TPA Paper Explained" (gyanendradas.substack.com): "Rotary Position
            Embedding (RoPE)" and "RoPE Compatibility and Acceleration".

Every function is pinned by ``tests/test_oracle_pins.py`` against something other than
itself: closed forms, library routines (torch's scaled_dot_product_attention and
F.linear in fp64), the MHA/MQA/GQA special cases, and invariants the pages state.
Nothing here is blocked, fused or reordered beyond what the definitions say, except
that ``decode_attention`` walks the keys in chunks so that a 131072-token context does
not need 4 GB of fp64 keys at once; each chunk computes the same per-key values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

FACTOR_NAMES = ("a_q", "a_k", "a_v", "b_q", "b_k", "b_v")


@dataclass(frozen=True)
class Dims:
    """The shape parameters of one TPA layer ([review] 代码 类定义与初始化).

    d_model = ``dim``, n_heads = ``n_heads``, head_dim = ``head_dim``, rank_q =
    ``q_rank``; the page uses one ``rank`` for K and V, kept here as rank_k = rank_v.
    rank_q = 0 marks the TPA-KVonly variant, whose query is a plain per-head vector.
    shared_basis marks the variant whose key and value B factors are shared across
    tokens ([review] 优点与创新 5, "跨标记共享基向量"): the pages name it in one clause.
    Reading taken: B_K and B_V are layer parameters, b_r^K(x_t) = b_r^K for every token
    (the non-contextual B of 优点与创新 4 applied to B), A_K and A_V stay contextual, the
    query keeps its own factors, and RoPE acts on the key at its position as in
    contextual TPA.  The per-token projections W_B_k, W_B_v then do not exist.
    """

    d_model: int
    n_heads: int
    head_dim: int
    rank_q: int
    rank_k: int
    rank_v: int
    shared_basis: bool = False


def factor_widths(dims: Dims) -> dict:
    """Output width of each of the six bias-free projections ([review] 类定义与初始化):
    W_A_* map d_model -> n_heads*rank, W_B_* map d_model -> rank*head_dim.

    TPA-KVonly (rank_q = 0) keeps the standard query projection ([review] 实验/结果
    names the variant; its projection is not printed).  Reading taken: it takes the
    b_q slot as W_Q with n_heads*head_dim outputs, viewed (n_heads, head_dim), and the
    a_q slot is empty.  With a shared basis the b_k and b_v slots are empty (their
    factors are parameters, not projections of x_t)."""
    h, d = dims.n_heads, dims.head_dim
    return {
        "a_q": h * dims.rank_q,
        "a_k": h * dims.rank_k,
        "a_v": h * dims.rank_v,
        "b_q": (dims.rank_q if dims.rank_q > 0 else h) * d,
        "b_k": 0 if dims.shared_basis else dims.rank_k * d,
        "b_v": 0 if dims.shared_basis else dims.rank_v * d,
    }


def cache_elements_per_token(dims: Dims) -> int:
    """Factor-cache elements stored per token: cache_kA/cache_vA are [.., n_heads, rank]
    and cache_kB/cache_vB are [.., rank, head_dim] ([review] 类定义与初始化), i.e.
    (R_K + R_V) * (h + d_h).  With a shared basis only the A factors are per token:
    (R_K + R_V) * h."""
    h, d = dims.n_heads, dims.head_dim
    if dims.shared_basis:
        return dims.rank_k * h + dims.rank_v * h
    return dims.rank_k * h + dims.rank_v * h + dims.rank_k * d + dims.rank_v * d


# --------------------------------------------------------------------------- RoPE

def rope_inv_freq(head_dim: int, base: float) -> np.ndarray:
    """theta_k = base^(-2k/d) for k = 0 .. d/2-1.

    The pages name RoPE (``apply_rotary_emb(q, k, freqs_cis)`` in [review] 前向传播,
    and [explain] "Rotary Position Embedding (RoPE)") but do not print its formula.
    Reading taken: the LLaMA convention the page's ``freqs_cis`` name comes from —
    interleaved pairs (2k, 2k+1), frequencies base^(-2k/d), the whole head rotated,
    0-based absolute positions.
    """
    if head_dim % 2:
        raise ValueError("RoPE needs an even head_dim")
    k = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * k / head_dim)


def rope_rotate(x: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotate every interleaved pair of the last axis of ``x`` by position * theta_k.

    ``x`` has shape [T, ..., d]; ``positions`` has shape [T] and gives the absolute
    position of each leading index.  Pair (x_{2k}, x_{2k+1}) becomes
    (x_{2k} cos a - x_{2k+1} sin a, x_{2k} sin a + x_{2k+1} cos a), a = p * theta_k.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    pos = np.asarray(positions, dtype=np.float64).reshape(-1)
    if pos.shape[0] != x.shape[0]:
        raise ValueError("one position per leading index")
    angle = pos[:, None] * rope_inv_freq(d, base)[None, :]          # [T, d/2]
    shape = (x.shape[0],) + (1,) * (x.ndim - 2) + (d // 2,)
    c = np.cos(angle).reshape(shape)
    s = np.sin(angle).reshape(shape)
    even = x[..., 0::2]
    odd = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = even * s + odd * c
    return out


# --------------------------------------------------------------------- projection

def split_factors(y: np.ndarray, dims: Dims) -> dict:
    """Cut the concatenated projection output into the six factors, with the views of
    [review] 前向传播: A_* is viewed (.., n_heads, rank) and B_* (.., rank, head_dim),
    so column h*R + r of W_A_* is (head h, rank r) and column r*d + k of W_B_* is
    (rank r, dim k).  The concatenation order is FACTOR_NAMES.  For TPA-KVonly the
    result holds the query ``q`` (.., n_heads, head_dim) in place of a_q and b_q."""
    widths = factor_widths(dims)
    h, d = dims.n_heads, dims.head_dim
    ranks = {"q": dims.rank_q, "k": dims.rank_k, "v": dims.rank_v}
    out = {}
    col = 0
    lead = y.shape[:-1]
    for name in FACTOR_NAMES:
        w = widths[name]
        part = y[..., col:col + w]
        r = ranks[name[-1]]
        if dims.rank_q == 0 and name in ("a_q", "b_q"):
            if name == "b_q":
                out["q"] = part.reshape(lead + (h, d))     # TPA-KVonly: the plain query
        elif w == 0 and name in ("b_k", "b_v"):
            pass                                           # shared basis: not projected
        elif name.startswith("a_"):
            out[name] = part.reshape(lead + (h, r))
        else:
            out[name] = part.reshape(lead + (r, d))
        col += w
    if col != y.shape[-1]:
        raise ValueError("projection width does not match dims")
    return out


def project(x: np.ndarray, w_cat: np.ndarray, dims: Dims) -> dict:
    """The six bias-free projections W_A_q/k/v, W_B_q/k/v of [review] 类定义与初始化,
    applied as in 前向传播.  ``w_cat`` stacks the six nn.Linear weights ([out, d_model]
    each) row-wise in FACTOR_NAMES order; the result is x @ w_cat^T in fp64, cut into
    un-rotated factors."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_cat, dtype=np.float64)
    return split_factors(x @ w.T, dims)


def materialize(a: np.ndarray, b: np.ndarray, rank: int) -> np.ndarray:
    """Q_t = (1/R) sum_r a_r(x_t) (outer) b_r(x_t)  ([review] §3 公式描述).

    a: [T, h, R], b: [T, R, d] -> [T, h, d]; the page computes it as
    ``torch.bmm(A, B).div_(rank)`` ([review] 前向传播)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.einsum("thr,trd->thd", a, b) / rank


# ---------------------------------------------------------------------- attention

def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                     q_positions: np.ndarray, return_probs: bool = False):
    """softmax(q k^T / sqrt(d_h) + causal mask) v for one sequence.

    q: [S, h, d] at absolute positions ``q_positions`` [S]; k, v: [L, h, d] at
    positions 0..L-1.  Key j is visible to the query at position p iff j <= p — the
    additive mask of [review] 前向传播, read as causal over absolute positions.  The
    scale is 1/sqrt(head_dim) ([popsci] Ⅱ.1, [review] 前向传播).  The softmax is
    taken in fp64 after subtracting the row maximum.  Returns out [S, h, d] (and the
    probabilities [h, S, L] when asked).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = q.shape[-1]
    pos = np.asarray(q_positions).reshape(-1)
    L = k.shape[0]
    scores = np.einsum("shd,lhd->hsl", q, k) / math.sqrt(d)          # [h, S, L]
    visible = np.arange(L)[None, :] <= pos[:, None]                   # [S, L]
    if not visible.any(axis=1).all():
        raise ValueError("a query row sees no key")
    scores = np.where(visible[None, :, :], scores, -np.inf)
    m = scores.max(axis=-1, keepdims=True)
    e = np.exp(scores - m)
    p = e / e.sum(axis=-1, keepdims=True)
    out = np.einsum("hsl,lhd->shd", p, v)
    if return_probs:
        return out, p
    return out


def broadcast_basis(basis: dict, n_tokens: int, dims: Dims) -> dict:
    """The shared-basis variant's B_K and B_V for ``n_tokens`` tokens: every token's
    factor is the layer's basis, b_r(x_t) = b_r ([review] 优点与创新 5, reading in
    ``Dims``).  basis["b_k"]: [R_K, d], basis["b_v"]: [R_V, d] -> [n_tokens, R, d]."""
    out = {}
    for n, r in (("b_k", dims.rank_k), ("b_v", dims.rank_v)):
        b = np.asarray(basis[n], dtype=np.float64).reshape(r, dims.head_dim)
        out[n] = np.broadcast_to(b, (n_tokens, r, dims.head_dim))
    return out


def shared_basis_tables(basis: dict, dims: Dims, capacity: int, rope_base: float) -> dict:
    """The shared-basis cache's B side for positions 0..capacity-1, pre-rotated as
    contextual TPA caches B_K ([review] 关键问题及回答 问题2): row p of b_k is the key
    basis rotated at position p, row p of b_v is the value basis (no rotation).  Every
    sequence's key at position p uses row p, so these are per layer, not per sequence.
    Returns {"b_k": [capacity, R_K, d], "b_v": [capacity, R_V, d]}."""
    b = broadcast_basis(basis, capacity, dims)
    return {"b_k": rope_rotate(b["b_k"], np.arange(capacity), rope_base),
            "b_v": np.array(b["b_v"])}


def tpa_forward(x: np.ndarray, w_cat: np.ndarray, dims: Dims, rope_base: float,
                start_pos: int = 0, prior: dict | None = None, basis: dict | None = None):
    """The pages' TPA forward for one batch, without the output projection.

    Follows [review] 前向传播 in the page's own order: project x into the six
    factors; write the new A_k/A_v/B_k/B_v at [start_pos, start_pos+S) of the cache
    (``prior`` holds the un-rotated factors of positions [0, start_pos)); read the
    cache back over [0, start_pos+S); materialise q, k, v with bmm and 1/R; apply
    RoPE to the materialised q (positions start_pos+i) and k (positions j); causal
    softmax attention.  ``self.wo`` is not applied: the page uses it without defining
    it in __init__.  With a shared basis (``dims.shared_basis``) ``basis`` holds the
    layer's b_k [R_K, d] and b_v [R_V, d], used as every token's B_K and B_V.

    x: [B, S, d_model].  Returns (out [B, S, h, d], new) where ``new`` holds the
    un-rotated factors of the S new tokens ([B, S, ...] each).
    """
    x = np.asarray(x, dtype=np.float64)
    B, S, _ = x.shape
    new = project(x.reshape(B * S, -1), w_cat, dims)
    new = {n: t.reshape((B, S) + t.shape[1:]) for n, t in new.items()}
    cached = ("a_k", "a_v") if dims.shared_basis else ("a_k", "a_v", "b_k", "b_v")
    outs = []
    for b in range(B):
        cache = {}
        for n in cached:
            head = prior[n][b][:start_pos] if (prior is not None and start_pos) else \
                np.zeros((0,) + new[n].shape[2:])
            cache[n] = np.concatenate([np.asarray(head, np.float64), new[n][b]], axis=0)
        if dims.shared_basis:
            cache.update(broadcast_basis(basis, cache["a_k"].shape[0], dims))
        if dims.rank_q == 0:
            q = new["q"][b]                               # TPA-KVonly: plain query
        else:
            q = materialize(new["a_q"][b], new["b_q"][b], dims.rank_q)
        k = materialize(cache["a_k"], cache["b_k"], dims.rank_k)
        v = materialize(cache["a_v"], cache["b_v"], dims.rank_v)
        q_pos = start_pos + np.arange(S)
        q = rope_rotate(q, q_pos, rope_base)
        k = rope_rotate(k, np.arange(k.shape[0]), rope_base)
        outs.append(causal_attention(q, k, v, q_pos))
    return np.stack(outs), new


def attend_from_factors(q_factors: dict, kv: dict, dims: Dims,
                        q_positions: np.ndarray) -> np.ndarray:
    """Attention for one sequence from a factor cache whose B_K is already rotated.

    This is the pre-rotated form of [review] 关键问题及回答 问题2 (B_K rotated at
    its position before it is cached) and [explain] "RoPE Compatibility and
    Acceleration": the cached factors are used as they are, with no rotation at
    attention time.  ``q_factors`` holds a_q [S, h, R_Q] and b_q [S, R_Q, d] with b_q
    already rotated at ``q_positions``; for TPA-KVonly (rank_q == 0) it holds the
    rotated per-head query ``q`` [S, h, d] instead.  ``kv`` holds a_k, a_v [L, h, R]
    and b_k (rotated), b_v [L, R, d].  Returns out [S, h, d].
    """
    if dims.rank_q == 0:
        q = np.asarray(q_factors["q"], dtype=np.float64)
    else:
        q = materialize(q_factors["a_q"], q_factors["b_q"], dims.rank_q)
    k = materialize(kv["a_k"], kv["b_k"], dims.rank_k)
    v = materialize(kv["a_v"], kv["b_v"], dims.rank_v)
    return causal_attention(q, k, v, q_positions)


def decode_query(q_factors: dict, dims: Dims) -> np.ndarray:
    """The one decode query of a sequence, [h, d]: (1/R_Q) sum_r a_r (outer) b_r with
    b already rotated at its position, or the given per-head query for TPA-KVonly."""
    if dims.rank_q == 0:
        return np.asarray(q_factors["q"], dtype=np.float64).reshape(dims.n_heads, dims.head_dim)
    a = np.asarray(q_factors["a_q"], dtype=np.float64).reshape(1, dims.n_heads, dims.rank_q)
    b = np.asarray(q_factors["b_q"], dtype=np.float64).reshape(1, dims.rank_q, dims.head_dim)
    return materialize(a, b, dims.rank_q)[0]


def decode_attention(q_factors: dict, kv: dict, dims: Dims, length: int,
                     chunk: int = 4096) -> np.ndarray:
    """Decode for one sequence: the query at position length-1 attends to all cached
    keys 0..length-1 (the cache is written before it is read in [review] 前向传播, so
    the new token attends to itself).  Same value as ``attend_from_factors`` with one
    query; the keys are visited in chunks of ``chunk`` tokens in two passes (scores,
    then the softmax-weighted sum of values) so that long contexts fit in memory.
    Returns out [h, d].
    """
    q = decode_query(q_factors, dims)                                   # [h, d]
    d = dims.head_dim
    scores = np.empty((dims.n_heads, length), dtype=np.float64)
    for j0 in range(0, length, chunk):
        j1 = min(length, j0 + chunk)
        k = materialize(np.asarray(kv["a_k"][j0:j1]), np.asarray(kv["b_k"][j0:j1]), dims.rank_k)
        scores[:, j0:j1] = np.einsum("hd,lhd->hl", q, k) / math.sqrt(d)
    m = scores.max(axis=1, keepdims=True)
    e = np.exp(scores - m)
    p = e / e.sum(axis=1, keepdims=True)
    out = np.zeros((dims.n_heads, d), dtype=np.float64)
    for j0 in range(0, length, chunk):
        j1 = min(length, j0 + chunk)
        v = materialize(np.asarray(kv["a_v"][j0:j1]), np.asarray(kv["b_v"][j0:j1]), dims.rank_v)
        out += np.einsum("hl,lhd->hd", p[:, j0:j1], v)
    return out


def output_projection(out: np.ndarray, w_o: np.ndarray) -> np.ndarray:
    """The layer's closing ``self.wo(output)`` ([review] 前向传播): the attention output
    [T, h, d] is flattened per token to h*d features (``transpose(1,2).view(bsz,
    seqlen, -1)``) and mapped to d_model by a bias-free linear map.  The page uses
    ``wo`` without defining it; reading taken: nn.Linear(h*d, d_model, bias=False),
    w_o of shape [d_model, h*d].  The T6GroupNorm the page constructs is not applied
    in its forward and is left out."""
    o = np.asarray(out, dtype=np.float64)
    return o.reshape(o.shape[0], -1) @ np.asarray(w_o, dtype=np.float64).T


def tpa_forward_rows(x: np.ndarray, w_cat: np.ndarray, dims: Dims, rope_base: float,
                     rows, basis: dict | None = None) -> np.ndarray:
    """``tpa_forward`` for one sequence that starts at position 0, evaluated only for
    the query rows ``rows`` (the keys and values still cover the whole sequence), so
    that long sequences can be checked on a sample of their outputs.

    x: [S, d_model].  Returns out [len(rows), h, d].  Same steps, same order as
    ``tpa_forward``: project, materialise, rotate the materialised q and k, attend
    (``basis`` as in ``tpa_forward``).
    """
    x = np.asarray(x, dtype=np.float64)
    rows = np.asarray(rows).reshape(-1)
    f = project(x, w_cat, dims)
    if dims.shared_basis:
        f.update(broadcast_basis(basis, x.shape[0], dims))
    if dims.rank_q == 0:
        q = f["q"][rows]                                  # TPA-KVonly: plain query
    else:
        q = materialize(f["a_q"][rows], f["b_q"][rows], dims.rank_q)
    k = materialize(f["a_k"], f["b_k"], dims.rank_k)
    v = materialize(f["a_v"], f["b_v"], dims.rank_v)
    q = rope_rotate(q, rows, rope_base)
    k = rope_rotate(k, np.arange(x.shape[0]), rope_base)
    return causal_attention(q, k, v, rows)
