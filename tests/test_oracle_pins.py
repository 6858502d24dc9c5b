"""Pins for the fp64 oracle, checked against what the pages and the mathematics fix.

Every check compares the oracle with something other than itself: closed forms,
torch library routines in fp64 (scaled_dot_product_attention, F.linear, bmm),
MHA/MQA/GQA as special cases of TPA, and invariants the pages state.  Each is chosen
so that a plausible slip in the oracle (a dropped 1/R, a wrong sign or pairing in
RoPE, a transposed view, a wrong softmax scale or mask) fails at least one of them;
``test_planted_mistakes_are_caught`` plants such slips and checks that they do.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import Dims

HERE = os.path.dirname(os.path.abspath(__file__))
TOL = 1e-12


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def gen(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- RoPE

def test_rope_closed_form_first_pair():
    # theta_0 = base^0 = 1 for any base: the first pair turns by exactly `p` radians.
    pos = np.arange(6)
    e0 = np.zeros((6, 2)); e0[:, 0] = 1.0
    e1 = np.zeros((6, 2)); e1[:, 1] = 1.0
    r0 = oracle.rope_rotate(e0, pos, 10000.0)
    r1 = oracle.rope_rotate(e1, pos, 10000.0)
    for p in range(6):
        assert r0[p, 0] == pytest.approx(math.cos(p), abs=TOL)
        assert r0[p, 1] == pytest.approx(math.sin(p), abs=TOL)
        assert r1[p, 0] == pytest.approx(-math.sin(p), abs=TOL)
        assert r1[p, 1] == pytest.approx(math.cos(p), abs=TOL)


def test_rope_frequencies_closed_form():
    # d = 8, base = 10000: theta = 1, 10^-1, 10^-2, 10^-3.
    th = oracle.rope_inv_freq(8, 10000.0)
    np.testing.assert_allclose(th, [1.0, 0.1, 0.01, 0.001], rtol=0, atol=1e-15)


def test_rope_is_complex_multiplication_of_interleaved_pairs():
    # The LLaMA form the page's `freqs_cis` comes from: view (x_2k, x_2k+1) as one
    # complex number and multiply by exp(i * p * theta_k).
    g = gen(1)
    T, R, d, base = 7, 3, 16, 500000.0
    x = g.standard_normal((T, R, d))
    pos = g.integers(0, 131072, size=T)
    xc = x[..., 0::2] + 1j * x[..., 1::2]
    theta = base ** (-(np.arange(0, d, 2) / d))
    rot = np.exp(1j * pos[:, None, None] * theta[None, None, :])
    want = np.empty_like(x)
    want[..., 0::2] = (xc * rot).real
    want[..., 1::2] = (xc * rot).imag
    assert rel(oracle.rope_rotate(x, pos, base), want) < 1e-10


def test_rope_invariants():
    g = gen(2)
    x = g.standard_normal((5, 2, 32))
    pos0 = np.zeros(5, dtype=int)
    assert rel(oracle.rope_rotate(x, pos0, 1e4), x) == 0.0                     # p = 0
    pm, pn = g.integers(0, 5000, 5), g.integers(0, 5000, 5)
    two = oracle.rope_rotate(oracle.rope_rotate(x, pm, 1e4), pn, 1e4)
    assert rel(two, oracle.rope_rotate(x, pm + pn, 1e4)) < 1e-9                 # R_m R_n = R_{m+n}
    np.testing.assert_allclose(np.linalg.norm(oracle.rope_rotate(x, pm, 1e4), axis=-1),
                               np.linalg.norm(x, axis=-1), rtol=1e-12)          # a rotation


def test_rope_relative_position():
    # "TPA Paper Explained", RoPE section: scores depend only on relative position.
    g = gen(3)
    q, k = g.standard_normal((1, 64)), g.standard_normal((1, 64))
    for m, n in [(5, 2), (1000, 997), (70000, 69997)]:
        a = np.dot(oracle.rope_rotate(q, [m], 1e4)[0], oracle.rope_rotate(k, [n], 1e4)[0])
        b = np.dot(oracle.rope_rotate(q, [m - n], 1e4)[0], k[0])
        assert a == pytest.approx(b, rel=1e-9, abs=1e-12)


# ----------------------------------------------------------------------- projection

def test_projection_matches_six_separate_linears():
    # [review] 类定义与初始化 / 前向传播: six bias-free nn.Linear, then .view().
    g = gen(4)
    dims = Dims(d_model=24, n_heads=3, head_dim=8, rank_q=4, rank_k=2, rank_v=3)
    T = 9
    x = g.standard_normal((T, dims.d_model))
    widths = oracle.factor_widths(dims)
    ws = {n: g.standard_normal((widths[n], dims.d_model)) for n in oracle.FACTOR_NAMES}
    w_cat = np.concatenate([ws[n] for n in oracle.FACTOR_NAMES], axis=0)
    got = oracle.project(x, w_cat, dims)
    xt = torch.from_numpy(x)
    h, d = dims.n_heads, dims.head_dim
    views = {"a_q": (T, h, dims.rank_q), "a_k": (T, h, dims.rank_k), "a_v": (T, h, dims.rank_v),
             "b_q": (T, dims.rank_q, d), "b_k": (T, dims.rank_k, d), "b_v": (T, dims.rank_v, d)}
    for n in oracle.FACTOR_NAMES:
        want = F.linear(xt, torch.from_numpy(ws[n])).view(*views[n]).numpy()
        assert got[n].shape == want.shape
        assert rel(got[n], want) < TOL, n


def test_materialize_hand_example():
    # h = 2, R = 2, d = 4: Q = (1/2) * [[1, 2, 0, 0], [3, 4, 0, 0]].
    a = np.array([[[1.0, 2.0], [3.0, 4.0]]])               # [T=1, h=2, R=2]
    b = np.array([[[1.0, 0, 0, 0], [0, 1.0, 0, 0]]])       # [T=1, R=2, d=4]
    want = 0.5 * np.array([[[1.0, 2.0, 0, 0], [3.0, 4.0, 0, 0]]])
    assert rel(oracle.materialize(a, b, 2), want) == 0.0


def test_materialize_matches_bmm():
    g = gen(5)
    a, b = g.standard_normal((11, 5, 3)), g.standard_normal((11, 3, 16))
    want = torch.bmm(torch.from_numpy(a), torch.from_numpy(b)).div_(3).numpy()
    assert rel(oracle.materialize(a, b, 3), want) < TOL


def test_cache_size_formula_golden():
    with open(os.path.join(HERE, "golden", "cache_bytes_per_token.json")) as f:
        gold = json.load(f)
    for row in gold["rows"]:
        dims = Dims(0, row["n_heads"], row["head_dim"], 0, row["rank_k"], row["rank_v"])
        assert oracle.cache_elements_per_token(dims) * row["elem_bytes"] == row["bytes_per_token"]
        mha = 2 * row["n_heads"] * row["head_dim"]
        assert mha / oracle.cache_elements_per_token(dims) == pytest.approx(row["mha_ratio"], rel=1e-3)


# ------------------------------------------------------------------------ attention

def sdpa(q, k, v, mask):
    """torch's fp64 scaled_dot_product_attention; q [S,h,d], k/v [L,h,d], mask [S,L]."""
    t = lambda z: torch.from_numpy(np.ascontiguousarray(z)).permute(1, 0, 2)[None]
    out = F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=torch.from_numpy(mask))
    return out[0].permute(1, 0, 2).numpy()


def test_causal_attention_matches_sdpa():
    g = gen(6)
    S, L, h, d = 7, 19, 3, 16
    q, k, v = g.standard_normal((S, h, d)), g.standard_normal((L, h, d)), g.standard_normal((L, h, d))
    pos = np.arange(L - S, L)                                   # the last S positions
    mask = np.arange(L)[None, :] <= pos[:, None]
    assert rel(oracle.causal_attention(q, k, v, pos), sdpa(q, k, v, mask)) < 1e-12
    # and the plain is_causal form when queries start at 0
    pos = np.arange(S)
    want = F.scaled_dot_product_attention(
        *(torch.from_numpy(z).permute(1, 0, 2)[None] for z in (q, k[:S], v[:S])), is_causal=True)
    assert rel(oracle.causal_attention(q, k[:S], v[:S], pos), want[0].permute(1, 0, 2).numpy()) < 1e-12


def test_softmax_rows_sum_to_one_and_constant_values():
    g = gen(7)
    S, L, h, d = 5, 12, 2, 8
    q, k = 3 * g.standard_normal((S, h, d)), 3 * g.standard_normal((L, h, d))
    c = g.standard_normal((h, d))
    v = np.broadcast_to(c, (L, h, d)).copy()
    pos = np.arange(L - S, L)
    out, p = oracle.causal_attention(q, k, v, pos, return_probs=True)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-13)
    assert rel(out, np.broadcast_to(c, (S, h, d))) < 1e-13


def test_single_key_returns_its_value():
    g = gen(8)
    q, k, v = g.standard_normal((1, 4, 8)), g.standard_normal((1, 4, 8)), g.standard_normal((1, 4, 8))
    assert rel(oracle.causal_attention(q, k, v, [0]), v) < 1e-15


def _factor_case(g, L, S, h, d, rq, rk, rv):
    kv = {"a_k": g.standard_normal((L, h, rk)), "a_v": g.standard_normal((L, h, rv)),
          "b_k": g.standard_normal((L, rk, d)), "b_v": g.standard_normal((L, rv, d))}
    qf = {"a_q": g.standard_normal((S, h, rq)), "b_q": g.standard_normal((S, rq, d))}
    return qf, kv


def test_mha_is_tpa_with_one_hot_heads():
    # "MHA, MQA, GQA are non-contextual TPA" ([review] summary): R = h, a_r = R e_r.
    g = gen(9)
    L, S, h, d = 10, 4, 3, 8
    Wq, Wk, Wv = (g.standard_normal((L, h, d)) for _ in range(3))
    onehot = np.broadcast_to(h * np.eye(h), (L, h, h)).copy()
    dims = Dims(0, h, d, h, h, h)
    qf = {"a_q": onehot[:S], "b_q": Wq[:S]}
    kv = {"a_k": onehot, "b_k": Wk, "a_v": onehot, "b_v": Wv}
    pos = np.arange(L - S, L)
    got = oracle.attend_from_factors(qf, kv, dims, pos)
    mask = np.arange(L)[None, :] <= pos[:, None]
    assert rel(got, sdpa(Wq[:S], Wk, Wv, mask)) < 1e-12


def test_mqa_is_tpa_with_rank_one_constant_heads():
    # MQA (the bbzoh.cn MQA/GQA blog, 第二部分): one K/V head broadcast to all query heads.
    g = gen(10)
    L, S, h, d = 9, 3, 4, 8
    k1, v1 = g.standard_normal((L, 1, d)), g.standard_normal((L, 1, d))
    qf = {"a_q": g.standard_normal((S, h, 2)), "b_q": g.standard_normal((S, 2, d))}
    kv = {"a_k": np.ones((L, h, 1)), "b_k": k1, "a_v": np.ones((L, h, 1)), "b_v": v1}
    dims = Dims(0, h, d, 2, 1, 1)
    pos = np.arange(L - S, L)
    got = oracle.attend_from_factors(qf, kv, dims, pos)
    q = oracle.materialize(qf["a_q"], qf["b_q"], 2)
    mask = np.arange(L)[None, :] <= pos[:, None]
    want = sdpa(q, np.repeat(k1, h, axis=1), np.repeat(v1, h, axis=1), mask)
    assert rel(got, want) < 1e-12


def test_gqa_is_tpa_with_group_indicator_heads():
    # GQA (the bbzoh.cn blog, 第三部分): n_heads query heads share n_kv_heads K/V heads.
    g = gen(11)
    L, S, h, G, d = 11, 5, 8, 4, 16
    kg, vg = g.standard_normal((L, G, d)), g.standard_normal((L, G, d))
    a = np.zeros((L, h, G))
    for head in range(h):
        a[:, head, head // (h // G)] = G
    qf = {"a_q": g.standard_normal((S, h, 3)), "b_q": g.standard_normal((S, 3, d))}
    kv = {"a_k": a, "b_k": kg, "a_v": a, "b_v": vg}
    dims = Dims(0, h, d, 3, G, G)
    pos = np.arange(L - S, L)
    got = oracle.attend_from_factors(qf, kv, dims, pos)
    q = oracle.materialize(qf["a_q"], qf["b_q"], 3)
    mask = np.arange(L)[None, :] <= pos[:, None]
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(kg).permute(1, 0, 2)[None]
    tv = torch.from_numpy(vg).permute(1, 0, 2)[None]
    want = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(mask), enable_gqa=True)
    assert rel(got, want[0].permute(1, 0, 2).numpy()) < 1e-12


def test_pre_rotated_cache_equals_rotating_materialised_keys():
    # [review] 问题2: caching RoPE_t(B_K) gives the same attention as rotating the
    # materialised k (the page's code order); likewise for the query.
    g = gen(12)
    dims = Dims(d_model=32, n_heads=4, head_dim=16, rank_q=3, rank_k=2, rank_v=2)
    B, S, base = 2, 13, 1e4
    x = g.standard_normal((B, S, dims.d_model))
    w = g.standard_normal((sum(oracle.factor_widths(dims).values()), dims.d_model)) / math.sqrt(dims.d_model)
    out, new = oracle.tpa_forward(x, w, dims, base)
    for b in range(B):
        pos = np.arange(S)
        qf = {"a_q": new["a_q"][b], "b_q": oracle.rope_rotate(new["b_q"][b], pos, base)}
        kv = {"a_k": new["a_k"][b], "a_v": new["a_v"][b], "b_v": new["b_v"][b],
              "b_k": oracle.rope_rotate(new["b_k"][b], pos, base)}
        assert rel(oracle.attend_from_factors(qf, kv, dims, pos), out[b]) < 1e-12


def test_chunked_prefill_equals_one_shot_and_is_causal():
    g = gen(13)
    dims = Dims(d_model=16, n_heads=2, head_dim=8, rank_q=2, rank_k=1, rank_v=2)
    S0, S1, base = 6, 5, 1e4
    x = g.standard_normal((1, S0 + S1, dims.d_model))
    w = g.standard_normal((sum(oracle.factor_widths(dims).values()), dims.d_model)) / 4.0
    full, _ = oracle.tpa_forward(x, w, dims, base)
    first, new0 = oracle.tpa_forward(x[:, :S0], w, dims, base)
    second, _ = oracle.tpa_forward(x[:, S0:], w, dims, base, start_pos=S0, prior=new0)
    assert rel(first, full[:, :S0]) < 1e-12
    assert rel(second, full[:, S0:]) < 1e-12
    # changing a later token leaves every earlier output unchanged
    x2 = x.copy(); x2[0, 8] += 3.0
    alt, _ = oracle.tpa_forward(x2, w, dims, base)
    assert rel(alt[:, :8], full[:, :8]) == 0.0 and rel(alt[:, 8:], full[:, 8:]) > 1e-3


def test_shifting_all_positions_leaves_attention_unchanged():
    g = gen(14)
    dims = Dims(0, 3, 16, 2, 2, 2)
    L, S = 12, 4
    qf, kv = _factor_case(g, L, S, 3, 16, 2, 2, 2)
    pos = np.arange(L - S, L)
    outs = []
    for shift in (0, 37, 100000):
        q2 = dict(qf, b_q=oracle.rope_rotate(qf["b_q"], pos + shift, 1e4))
        kv2 = dict(kv, b_k=oracle.rope_rotate(kv["b_k"], np.arange(L) + shift, 1e4))
        outs.append(oracle.attend_from_factors(q2, kv2, dims, pos))
    assert rel(outs[1], outs[0]) < 1e-9 and rel(outs[2], outs[0]) < 1e-9


def test_decode_equals_last_row_of_causal_attention():
    g = gen(15)
    for rq in (3, 0):
        dims = Dims(0, 4, 8, rq, 2, 1)
        L = 23
        kv = {"a_k": g.standard_normal((L, 4, 2)), "a_v": g.standard_normal((L, 4, 1)),
              "b_k": g.standard_normal((L, 2, 8)), "b_v": g.standard_normal((L, 1, 8))}
        if rq:
            qf = {"a_q": g.standard_normal((4, rq)), "b_q": g.standard_normal((rq, 8))}
            qf1 = {"a_q": qf["a_q"][None], "b_q": qf["b_q"][None]}
        else:
            qf = {"q": g.standard_normal((4, 8))}
            qf1 = {"q": qf["q"][None]}
        dense = oracle.attend_from_factors(qf1, kv, dims, [L - 1])[0]
        for chunk in (1, 5, 4096):
            assert rel(oracle.decode_attention(qf, kv, dims, L, chunk=chunk), dense) < 1e-13


def test_kvonly_decode_is_plain_attention_on_materialised_kv():
    g = gen(16)
    dims = Dims(0, 4, 16, 0, 2, 2)
    L = 17
    kv = {"a_k": g.standard_normal((L, 4, 2)), "a_v": g.standard_normal((L, 4, 2)),
          "b_k": g.standard_normal((L, 2, 16)), "b_v": g.standard_normal((L, 2, 16))}
    q = g.standard_normal((4, 16))
    k = np.einsum("lhr,lrd->lhd", kv["a_k"], kv["b_k"]) / 2
    v = np.einsum("lhr,lrd->lhd", kv["a_v"], kv["b_v"]) / 2
    want = F.scaled_dot_product_attention(torch.from_numpy(q)[:, None], torch.from_numpy(k).permute(1, 0, 2),
                                          torch.from_numpy(v).permute(1, 0, 2))[:, 0].numpy()
    assert rel(oracle.decode_attention({"q": q}, kv, dims, L), want) < 1e-12


# ------------------------------------------------------------- planted mistakes

def _pins_fail(monkeypatch, target, replacement, tests):
    monkeypatch.setattr(oracle.tpa_oracle, target, replacement)
    monkeypatch.setattr(oracle, target, replacement, raising=False)
    failed = 0
    for t in tests:
        try:
            t()
        except AssertionError:
            failed += 1
    return failed


def test_planted_mistakes_are_caught(monkeypatch):
    real_mat = oracle.tpa_oracle.materialize
    real_rot = oracle.tpa_oracle.rope_rotate
    real_att = oracle.tpa_oracle.causal_attention
    # 1. the 1/R of the factor formula dropped
    assert _pins_fail(monkeypatch, "materialize", lambda a, b, r: real_mat(a, b, 1),
                      [test_materialize_hand_example, test_mha_is_tpa_with_one_hot_heads]) == 2
    monkeypatch.setattr(oracle.tpa_oracle, "materialize", real_mat)
    monkeypatch.setattr(oracle, "materialize", real_mat)

    # 2. RoPE turning the wrong way
    def wrong_sign(x, p, base):
        return real_rot(x, -np.asarray(p), base)
    assert _pins_fail(monkeypatch, "rope_rotate", wrong_sign,
                      [test_rope_closed_form_first_pair, test_rope_is_complex_multiplication_of_interleaved_pairs]) == 2
    monkeypatch.setattr(oracle.tpa_oracle, "rope_rotate", real_rot)
    monkeypatch.setattr(oracle, "rope_rotate", real_rot)

    # 3. RoPE pairing the two halves instead of neighbours
    def half_split(x, p, base):
        x = np.asarray(x, np.float64)
        d = x.shape[-1]
        perm = np.empty(d, dtype=int)
        perm[0::2] = np.arange(d // 2)
        perm[1::2] = np.arange(d // 2, d)
        inv = np.argsort(perm)
        return real_rot(x[..., perm], p, base)[..., inv]
    assert _pins_fail(monkeypatch, "rope_rotate", half_split,
                      [test_rope_is_complex_multiplication_of_interleaved_pairs]) == 1
    monkeypatch.setattr(oracle.tpa_oracle, "rope_rotate", real_rot)
    monkeypatch.setattr(oracle, "rope_rotate", real_rot)

    # 4. softmax scaled by 1/d instead of 1/sqrt(d), and 5. the mask off by one
    def wrong_scale(q, k, v, pos, return_probs=False):
        return real_att(np.asarray(q) / math.sqrt(np.asarray(q).shape[-1]), k, v, pos, return_probs)
    assert _pins_fail(monkeypatch, "causal_attention", wrong_scale,
                      [test_causal_attention_matches_sdpa, test_mha_is_tpa_with_one_hot_heads]) == 2

    def off_by_one(q, k, v, pos, return_probs=False):
        return real_att(q, k, v, np.asarray(pos) - 1 + (np.asarray(pos) == 0), return_probs)
    assert _pins_fail(monkeypatch, "causal_attention", off_by_one,
                      [test_causal_attention_matches_sdpa]) == 1
    monkeypatch.setattr(oracle.tpa_oracle, "causal_attention", real_att)
    monkeypatch.setattr(oracle, "causal_attention", real_att)

    # 6. A factors viewed (R, h) instead of (h, R)
    real_split = oracle.tpa_oracle.split_factors

    def transposed_view(y, dims):
        out = real_split(y, dims)
        for n in ("a_q", "a_k", "a_v"):
            t = out[n]
            out[n] = t.reshape(t.shape[:-2] + (t.shape[-1], t.shape[-2])).swapaxes(-1, -2)
        return out
    assert _pins_fail(monkeypatch, "split_factors", transposed_view,
                      [test_projection_matches_six_separate_linears]) == 1


def test_forward_rows_equals_forward():
    g = gen(17)
    dims = Dims(d_model=16, n_heads=2, head_dim=8, rank_q=2, rank_k=2, rank_v=1)
    x = g.standard_normal((1, 21, 16))
    w = g.standard_normal((sum(oracle.factor_widths(dims).values()), 16)) / 4
    full, _ = oracle.tpa_forward(x, w, dims, 1e4)
    rows = [0, 5, 20]
    assert rel(oracle.tpa_forward_rows(x[0], w, dims, 1e4, rows), full[0, rows]) < 1e-13


# ------------------------------------------------------------------- TPA-KVonly

def _kvonly_weights(g, dims):
    widths = oracle.factor_widths(dims)
    assert widths["a_q"] == 0 and widths["b_q"] == dims.n_heads * dims.head_dim
    ws = {n: g.standard_normal((widths[n], dims.d_model)) / math.sqrt(dims.d_model) for n in oracle.FACTOR_NAMES}
    return ws, np.concatenate([ws[n] for n in oracle.FACTOR_NAMES], axis=0)


def test_kvonly_projection_is_a_plain_query_linear_plus_kv_factors():
    # TPA-KVonly ([review] 实验/结果): the query is a standard per-head linear map.
    g = gen(21)
    dims = Dims(d_model=24, n_heads=3, head_dim=8, rank_q=0, rank_k=2, rank_v=3)
    T = 7
    x = g.standard_normal((T, dims.d_model))
    ws, w_cat = _kvonly_weights(g, dims)
    got = oracle.project(x, w_cat, dims)
    assert set(got) == {"q", "a_k", "a_v", "b_k", "b_v"}
    xt = torch.from_numpy(x)
    want_q = F.linear(xt, torch.from_numpy(ws["b_q"])).view(T, dims.n_heads, dims.head_dim).numpy()
    assert rel(got["q"], want_q) < TOL
    want_bv = F.linear(xt, torch.from_numpy(ws["b_v"])).view(T, dims.rank_v, dims.head_dim).numpy()
    assert rel(got["b_v"], want_bv) < TOL


def test_kvonly_forward_is_textbook_attention_on_rotated_q_and_materialised_kv():
    # Independent route in torch: F.linear for the projections, bmm/R for K and V,
    # RoPE as complex multiplication, causal fp64 scaled_dot_product_attention.
    g = gen(22)
    dims = Dims(d_model=20, n_heads=4, head_dim=8, rank_q=0, rank_k=2, rank_v=2)
    B, S, base = 2, 11, 1e4
    x = g.standard_normal((B, S, dims.d_model))
    ws, w_cat = _kvonly_weights(g, dims)
    out, new = oracle.tpa_forward(x, w_cat, dims, base)
    h, d, R = dims.n_heads, dims.head_dim, dims.rank_k
    theta = torch.tensor(base, dtype=torch.float64) ** (-(torch.arange(0, d, 2, dtype=torch.float64) / d))
    pos = torch.arange(S, dtype=torch.float64)
    rot = torch.polar(torch.ones(S, d // 2, dtype=torch.float64), pos[:, None] * theta[None, :])

    def rope(t):                                   # t [S, h, d]
        c = torch.view_as_complex(t.reshape(S, h, d // 2, 2).contiguous())
        return torch.view_as_real(c * rot[:, None, :]).reshape(S, h, d)

    for b in range(B):
        xt = torch.from_numpy(x[b])
        lin = {n: F.linear(xt, torch.from_numpy(ws[n])) for n in oracle.FACTOR_NAMES if ws[n].shape[0]}
        q = lin["b_q"].view(S, h, d)
        k = torch.bmm(lin["a_k"].view(S, h, R), lin["b_k"].view(S, R, d)) / R
        v = torch.bmm(lin["a_v"].view(S, h, R), lin["b_v"].view(S, R, d)) / R
        q, k = rope(q), rope(k)
        want = F.scaled_dot_product_attention(q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2),
                                              is_causal=True).permute(1, 0, 2)
        assert rel(out[b], want.numpy()) < 1e-12
        # the pre-rotated form the kernels use: rotate q and B_K, then attend from factors
        qf = {"q": oracle.rope_rotate(new["q"][b], np.arange(S), base)}
        kv = {"a_k": new["a_k"][b], "a_v": new["a_v"][b], "b_v": new["b_v"][b],
              "b_k": oracle.rope_rotate(new["b_k"][b], np.arange(S), base)}
        assert rel(oracle.attend_from_factors(qf, kv, dims, np.arange(S)), out[b]) < 1e-12
    rows = [0, 6, 10]
    assert rel(oracle.tpa_forward_rows(x[1], w_cat, dims, base, rows), out[1, rows]) < 1e-12


def test_output_projection_is_a_bias_free_linear_on_flattened_heads():
    # [review] 前向传播: output.transpose(1, 2).contiguous().view(bsz, seqlen, -1), then wo
    g = gen(23)
    T, h, d, D = 6, 3, 4, 10
    out = g.standard_normal((T, h, d))
    w_o = g.standard_normal((D, h * d))
    want = F.linear(torch.from_numpy(out).reshape(T, h * d), torch.from_numpy(w_o)).numpy()
    assert rel(oracle.output_projection(out, w_o), want) < TOL
    # head-major flattening: feature h*d + k of the input is head h, dim k
    e = np.zeros((1, h, d)); e[0, 2, 1] = 1.0
    assert rel(oracle.output_projection(e, w_o)[0], w_o[:, 2 * d + 1]) < TOL


# ------------------------------------------------------- shared-basis variant

def _shared_case(g, dims, B, S):
    widths = oracle.factor_widths(dims)
    assert widths["b_k"] == 0 and widths["b_v"] == 0
    ws = {n: g.standard_normal((widths[n], dims.d_model)) / math.sqrt(dims.d_model) for n in oracle.FACTOR_NAMES}
    basis = {"b_k": g.standard_normal((dims.rank_k, dims.head_dim)),
             "b_v": g.standard_normal((dims.rank_v, dims.head_dim))}
    x = g.standard_normal((B, S, dims.d_model))
    return ws, np.concatenate([ws[n] for n in oracle.FACTOR_NAMES], axis=0), basis, x


def _torch_rope(t, positions, base):
    """RoPE as complex multiplication of interleaved pairs; t [S, n, d] (fp64 torch)."""
    S, n, d = t.shape
    theta = torch.tensor(base, dtype=torch.float64) ** (-(torch.arange(0, d, 2, dtype=torch.float64) / d))
    pos = torch.as_tensor(np.asarray(positions), dtype=torch.float64)
    rot = torch.polar(torch.ones(S, d // 2, dtype=torch.float64), pos[:, None] * theta[None, :])
    c = torch.view_as_complex(t.reshape(S, n, d // 2, 2).contiguous())
    return torch.view_as_real(c * rot[:, None, :]).reshape(S, n, d)


def test_shared_basis_projection_has_no_per_token_key_value_basis():
    # [review] 优点与创新 5: basis vectors shared across tokens.  Reading: W_B_k and
    # W_B_v are gone; the cache keeps (R_K + R_V) h elements per token.
    g = gen(31)
    dims = Dims(d_model=24, n_heads=3, head_dim=8, rank_q=2, rank_k=2, rank_v=3, shared_basis=True)
    ws, w_cat, _, x = _shared_case(g, dims, 1, 5)
    assert w_cat.shape[0] == 3 * (2 + 2 + 3) + 2 * 8
    got = oracle.project(x[0], w_cat, dims)
    assert set(got) == {"a_q", "b_q", "a_k", "a_v"}
    want_av = F.linear(torch.from_numpy(x[0]), torch.from_numpy(ws["a_v"])).view(5, 3, 3).numpy()
    assert rel(got["a_v"], want_av) < TOL
    assert oracle.cache_elements_per_token(dims) == (2 + 3) * 3
    # same layer with a contextual basis: the per-token B side is what the variant drops
    ctx = Dims(24, 3, 8, 2, 2, 3)
    assert oracle.cache_elements_per_token(ctx) - oracle.cache_elements_per_token(dims) == (2 + 3) * 8


def test_shared_basis_forward_is_textbook_attention_on_materialised_kv():
    # Independent route in torch: F.linear for the A projections and the query, K and V
    # as (1/R) a . basis with matmul, RoPE as complex multiplication on q and k,
    # causal fp64 scaled_dot_product_attention.
    g = gen(32)
    dims = Dims(d_model=20, n_heads=4, head_dim=8, rank_q=3, rank_k=2, rank_v=3, shared_basis=True)
    B, S, base = 2, 13, 1e4
    ws, w_cat, basis, x = _shared_case(g, dims, B, S)
    out, new = oracle.tpa_forward(x, w_cat, dims, base, basis=basis)
    h, d = dims.n_heads, dims.head_dim
    bk, bv = torch.from_numpy(basis["b_k"]), torch.from_numpy(basis["b_v"])
    tables = oracle.shared_basis_tables(basis, dims, S + 3, base)
    for b in range(B):
        xt = torch.from_numpy(x[b])
        lin = {n: F.linear(xt, torch.from_numpy(ws[n])) for n in oracle.FACTOR_NAMES if ws[n].shape[0]}
        q = torch.bmm(lin["a_q"].view(S, h, 3), lin["b_q"].view(S, 3, d)) / 3
        k = torch.matmul(lin["a_k"].view(S, h, 2), bk) / 2
        v = torch.matmul(lin["a_v"].view(S, h, 3), bv) / 3
        q, k = _torch_rope(q, np.arange(S), base), _torch_rope(k, np.arange(S), base)
        want = F.scaled_dot_product_attention(q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2),
                                              is_causal=True).permute(1, 0, 2)
        assert rel(out[b], want.numpy()) < 1e-12
        # the pre-rotated form the kernels use: query factors rotated at their positions,
        # keys read against the per-position tables (row j = basis rotated at j)
        qf = {"a_q": new["a_q"][b], "b_q": oracle.rope_rotate(new["b_q"][b], np.arange(S), base)}
        kv = {"a_k": new["a_k"][b], "a_v": new["a_v"][b],
              "b_k": tables["b_k"][:S], "b_v": tables["b_v"][:S]}
        assert rel(oracle.attend_from_factors(qf, kv, dims, np.arange(S)), out[b]) < 1e-12
        dec = oracle.decode_attention({"a_q": qf["a_q"][S - 1], "b_q": qf["b_q"][S - 1]}, kv, dims, S)
        assert rel(dec, out[b, S - 1]) < 1e-12
    rows = [0, 7, 12]
    assert rel(oracle.tpa_forward_rows(x[1], w_cat, dims, base, rows, basis=basis), out[1, rows]) < 1e-12
    # a second chunk after a cached prefix gives the rows of the one-shot pass
    head, new_h = oracle.tpa_forward(x[:, :8], w_cat, dims, base, basis=basis)
    tail, _ = oracle.tpa_forward(x[:, 8:], w_cat, dims, base, start_pos=8, prior=new_h, basis=basis)
    assert rel(np.concatenate([head, tail], axis=1), out) < 1e-12


def test_shared_basis_with_identity_basis_is_mha():
    # With R_K = R_V = d_h and the identity as the shared basis, the key of head h is
    # its own contextual d_h-vector a^K_{t,h,:} / d_h: plain MHA with key and value
    # projections W_A_k / R_K and W_A_v / R_V (the per-head view of 类定义与初始化).
    g = gen(33)
    h, d, D, S, base = 3, 8, 16, 9, 1e4
    dims = Dims(d_model=D, n_heads=h, head_dim=d, rank_q=0, rank_k=d, rank_v=d, shared_basis=True)
    ws, w_cat, _, x = _shared_case(g, dims, 1, S)
    basis = {"b_k": np.eye(d), "b_v": np.eye(d)}
    out, _ = oracle.tpa_forward(x, w_cat, dims, base, basis=basis)
    xt = torch.from_numpy(x[0])
    q = F.linear(xt, torch.from_numpy(ws["b_q"])).view(S, h, d)
    k = F.linear(xt, torch.from_numpy(ws["a_k"] / d)).view(S, h, d)
    v = F.linear(xt, torch.from_numpy(ws["a_v"] / d)).view(S, h, d)
    q, k = _torch_rope(q, np.arange(S), base), _torch_rope(k, np.arange(S), base)
    want = F.scaled_dot_product_attention(q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2),
                                          is_causal=True).permute(1, 0, 2)
    assert rel(out[0], want.numpy()) < 1e-12


def test_shared_basis_tables_closed_form():
    # Row p of the key table is the basis turned by p * theta_k per pair; for the unit
    # vector e_0 (theta_0 = 1) that is (cos p, sin p, 0, ...).  The value table is the
    # basis itself on every row.
    dims = Dims(0, 1, 4, 0, 2, 1, shared_basis=True)
    e = np.zeros((2, 4)); e[0, 0] = 1.0; e[1, 3] = 1.0
    bv = np.array([[0.5, -1.0, 2.0, 0.25]])
    t = oracle.shared_basis_tables({"b_k": e, "b_v": bv}, dims, 5, 100.0)
    assert t["b_k"].shape == (5, 2, 4) and t["b_v"].shape == (5, 1, 4)
    for p in range(5):
        np.testing.assert_allclose(t["b_k"][p, 0], [math.cos(p), math.sin(p), 0, 0], atol=TOL)
        a = p * 100.0 ** (-2 / 4)                  # pair 1 turns by p * base^(-1/2)
        np.testing.assert_allclose(t["b_k"][p, 1], [0, 0, -math.sin(a), math.cos(a)], atol=TOL)
        np.testing.assert_array_equal(t["b_v"][p], bv)


def test_shared_basis_planted_mistakes_are_caught(monkeypatch):
    real = oracle.tpa_oracle.shared_basis_tables
    real_bb = oracle.tpa_oracle.broadcast_basis

    # 1. tables rotated one position late
    def late(basis, dims, capacity, base):
        t = real(basis, dims, capacity + 1, base)
        return {"b_k": t["b_k"][1:], "b_v": t["b_v"][1:]}
    assert _pins_fail(monkeypatch, "shared_basis_tables", late,
                      [test_shared_basis_tables_closed_form,
                       test_shared_basis_forward_is_textbook_attention_on_materialised_kv]) == 2
    monkeypatch.setattr(oracle.tpa_oracle, "shared_basis_tables", real)
    monkeypatch.setattr(oracle, "shared_basis_tables", real)

    # 2. the basis vectors read back to front along d_h
    def reversed_d(basis, n_tokens, dims):
        out = real_bb(basis, n_tokens, dims)
        return {n: np.ascontiguousarray(t[..., ::-1]) for n, t in out.items()}
    assert _pins_fail(monkeypatch, "broadcast_basis", reversed_d,
                      [test_shared_basis_forward_is_textbook_attention_on_materialised_kv]) == 1


# -------------------------------------------------------------- brute force (scalar)

def _brute_layer(x, w_cat, h, d, rq, rk, rv, base, basis=None):
    """The TPA layer for one sequence as plain scalar loops, written from the definitions
    (no array code): y = W x per token; factors cut in the order A_q, A_k, A_v, B_q,
    B_k, B_v with the (head, rank) and (rank, dim) views; Q/K/V as (1/R) sums of outer
    products (KV-only: the plain query; shared basis: B_K, B_V from ``basis``); RoPE on
    interleaved pairs of q and k at positions 0.. ; causal softmax(q.k / sqrt(d)) v."""
    S, D = len(x), len(x[0])
    N = len(w_cat)
    y = [[sum(w_cat[n][c] * x[t][c] for c in range(D)) for n in range(N)] for t in range(S)]
    widths = [h * rq, h * rk, h * rv, (rq if rq else h) * d,
              0 if basis else rk * d, 0 if basis else rv * d]
    offs = [sum(widths[:i]) for i in range(6)]

    def A(t, seg, hh, r, R):
        return y[t][offs[seg] + hh * R + r]

    def Bf(t, seg, r, k):
        return y[t][offs[seg] + r * d + k]

    def rot(v, p):
        out = list(v)
        for k in range(d // 2):
            ang = p * base ** (-2.0 * k / d)
            c, s = math.cos(ang), math.sin(ang)
            out[2 * k] = v[2 * k] * c - v[2 * k + 1] * s
            out[2 * k + 1] = v[2 * k] * s + v[2 * k + 1] * c
        return out

    Q = [[None] * h for _ in range(S)]
    K = [[None] * h for _ in range(S)]
    V = [[None] * h for _ in range(S)]
    for t in range(S):
        for hh in range(h):
            if rq:
                q = [sum(A(t, 0, hh, r, rq) * Bf(t, 3, r, k) for r in range(rq)) / rq for k in range(d)]
            else:
                q = [y[t][offs[3] + hh * d + k] for k in range(d)]
            if basis:
                kk = [sum(A(t, 1, hh, s, rk) * basis["b_k"][s][k] for s in range(rk)) / rk for k in range(d)]
                vv = [sum(A(t, 2, hh, s, rv) * basis["b_v"][s][k] for s in range(rv)) / rv for k in range(d)]
            else:
                kk = [sum(A(t, 1, hh, s, rk) * Bf(t, 4, s, k) for s in range(rk)) / rk for k in range(d)]
                vv = [sum(A(t, 2, hh, s, rv) * Bf(t, 5, s, k) for s in range(rv)) / rv for k in range(d)]
            Q[t][hh], K[t][hh], V[t][hh] = rot(q, t), rot(kk, t), vv
    out = [[[0.0] * d for _ in range(h)] for _ in range(S)]
    for i in range(S):
        for hh in range(h):
            sc = [sum(Q[i][hh][k] * K[j][hh][k] for k in range(d)) / math.sqrt(d) for j in range(i + 1)]
            mx = max(sc)
            e = [math.exp(v - mx) for v in sc]
            z = sum(e)
            for k in range(d):
                out[i][hh][k] = sum(e[j] / z * V[j][hh][k] for j in range(i + 1))
    return out


@pytest.mark.parametrize("rq,rk,rv,shared", [(2, 1, 2, False), (0, 2, 1, False), (3, 2, 2, True), (0, 1, 2, True)],
                         ids=["tpa", "kvonly", "shared", "kvonly-shared"])
def test_forward_equals_scalar_brute_force(rq, rk, rv, shared):
    g = gen(41)
    h, d, D, S, base = 2, 4, 6, 5, 100.0
    dims = Dims(D, h, d, rq, rk, rv, shared_basis=shared)
    n = sum(oracle.factor_widths(dims).values())
    w = g.standard_normal((n, D)) / 2
    x = g.standard_normal((1, S, D))
    basis = {"b_k": g.standard_normal((rk, d)), "b_v": g.standard_normal((rv, d))} if shared else None
    got, _ = oracle.tpa_forward(x, w, dims, base, basis=basis)
    want = _brute_layer(x[0].tolist(), w.tolist(), h, d, rq, rk, rv, base,
                        basis={k: v.tolist() for k, v in basis.items()} if shared else None)
    assert rel(got[0], np.array(want)) < 1e-12
