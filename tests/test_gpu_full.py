"""GPU parity at the benchmark workloads' full sizes, in the launch configuration the
bench times, checked on sampled outputs the oracle computes one by one (whole
sequences for decode, sampled query rows for prefill)."""
import numpy as np
import pytest
import torch

import oracle
from tensor_product_attention_b200 import inputs as I
from helpers import TOL, dims_of, f64, fill_cache, oracle_dims, rel_err

pytestmark = pytest.mark.gpu


def _full_prefill(tpa, wl, sample_seqs, rows):
    dims = dims_of(wl, tpa)
    B, S = wl.batch, wl.seqlen
    cs = torch.empty((S, wl.head_dim // 2, 2), dtype=torch.float32, device="cuda")
    tpa.tpa_rope_table(dims, wl.rope_base, S, cs)
    x = torch.cat([I.prefill_x(wl, b) for b in range(B)]).cuda()
    w = I.prefill_w(wl)
    fac = tpa.alloc_factors(dims, B * S)
    cache = tpa.alloc_cache(dims, B, S)
    out = torch.empty((B * S, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    start = [0] * B
    tpa.tpa_project(dims, x, w.cuda(), B, S, start, cs, S, fac)
    tpa.tpa_cache_append(dims, cache, fac, B, S, start)
    tpa.tpa_prefill(dims, fac, cache, B, S, start, out)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    assert cache.lengths.cpu().tolist() == [S] * B
    out = out.view(B, S, wl.n_heads, wl.head_dim)
    od = oracle_dims(wl)
    for b in sample_seqs:
        ref = oracle.tpa_forward_rows(f64(x[b * S:(b + 1) * S].cpu()), f64(w), od, wl.rope_base, rows)
        err = rel_err(out[b, rows], ref)
        assert err < TOL["bf16"], (b, err)


def _rows(S, n, seed):
    g = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, 1, S // 2, S - 1], g.integers(0, S, n)]))


def test_full_prefill_b8_s2048_d1024(tpa):
    wl = I.WORKLOADS["prefill_b8_s2048_d1024"]
    _full_prefill(tpa, wl, [0, wl.batch - 1], _rows(wl.seqlen, 120, 1))


def test_full_layer_prefill_b4_s8192_d2048(tpa):
    wl = I.WORKLOADS["layer_prefill_b4_s8192_d2048"]
    _full_prefill(tpa, wl, [wl.batch - 1], _rows(wl.seqlen, 40, 2))


def test_full_layer_prefill_rows_sharp(tpa):
    """The 8192-token layer shape at the factor level with a x 8 (a sharp softmax over up
    to 8192 keys), on two of its sequences: sampled query rows against the oracle on the
    same bf16 factors, so the check isolates the attention kernel."""
    wl = I.WORKLOADS["layer_prefill_b4_s8192_d2048"]
    B, S = 2, wl.seqlen
    dims = dims_of(wl, tpa)
    cache = tpa.alloc_cache(dims, B, S, fill=float("nan"))
    q = tpa.alloc_factors(dims, B * S, kv=False)
    seqs = []
    for b in range(B):
        seq = I.prefill_factors(wl, b, S, S, a_scale=8.0)
        fill_cache(cache, b, seq)
        q.a_q[b * S:(b + 1) * S].copy_(seq["a_q"])
        q.b_q[b * S:(b + 1) * S].copy_(seq["b_q"])
        seqs.append(seq)
    out = torch.empty((B * S, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    tpa.tpa_prefill(dims, q, cache, B, S, [0] * B, out)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    out = out.view(B, S, wl.n_heads, wl.head_dim)
    od = oracle_dims(wl)
    rows = _rows(S, 40, 11)
    for b in range(B):
        seq = {k: f64(v) for k, v in seqs[b].items()}
        qf = {"a_q": seq["a_q"][rows], "b_q": seq["b_q"][rows]}
        ref = oracle.attend_from_factors(qf, seq, od, rows)
        err = rel_err(out[b, rows], ref)
        assert err < TOL["bf16"], (b, err)


def test_full_kvonly_layer_prefill_b4_s8192_d4096(tpa):
    wl = I.WORKLOADS["kvonly_layer_prefill_b4_s8192_d4096"]
    _full_prefill(tpa, wl, [wl.batch - 1], _rows(wl.seqlen, 24, 3))


def _full_decode(tpa, wl, sample, a_scale=1.0):
    dims = dims_of(wl, tpa)
    lengths = [int(v) for v in I.decode_lengths(wl)]
    B = wl.batch
    cache = tpa.alloc_cache(dims, B, max(lengths))
    basis = None
    if wl.shared_basis:
        basis = I.shared_basis(wl)
        cs = torch.empty((max(lengths), wl.head_dim // 2, 2), dtype=torch.float32, device="cuda")
        tpa.tpa_rope_table(dims, wl.rope_base, max(lengths), cs)
        tpa.tpa_shared_basis_tables(dims, basis["b_k"].cuda(), basis["b_v"].cuda(), cs, max(lengths),
                                    cache.b_k, cache.b_v)
        del cs
    q_parts = {}
    for b, L in enumerate(lengths):
        seq = I.decode_sequence(wl, b, L, a_scale=a_scale)
        fill_cache(cache, b, seq)
        for k in ("a_q", "b_q", "q"):
            if k in seq:
                q_parts.setdefault(k, []).append(seq[k])
        del seq
    if wl.rank_q:
        q_a = torch.stack(q_parts["a_q"]).cuda()
        q_b = torch.stack(q_parts["b_q"]).cuda()
    else:
        q_a, q_b = None, torch.stack(q_parts["q"]).cuda()
    out = torch.empty((B, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    tpa.tpa_decode(dims, q_a, q_b, cache, lengths, out, tpa.alloc_workspace(dims, lengths))
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    od = oracle_dims(wl)
    tab = None
    if basis is not None:
        tab = oracle.shared_basis_tables({n: f64(t) for n, t in basis.items()}, od, max(lengths), wl.rope_base)
    for b in sample:
        seq = {k: f64(v) for k, v in I.decode_sequence(wl, b, lengths[b], a_scale=a_scale).items()}
        kv = seq if tab is None else {"a_k": seq["a_k"], "a_v": seq["a_v"], **tab}
        err = rel_err(out[b], oracle.decode_attention(seq, kv, od, lengths[b]))
        assert err < TOL["bf16"], (b, lengths[b], err)


def test_full_decode_b64_ctx32k(tpa):
    wl = I.WORKLOADS["decode_b64_ctx32k"]
    _full_decode(tpa, wl, [0, 37, wl.batch - 1])


def test_full_kvonly_decode_b16_ctx64k_128k(tpa):
    wl = I.WORKLOADS["kvonly_decode_b16_ctx64k_128k"]
    lengths = I.decode_lengths(wl)
    _full_decode(tpa, wl, [int(np.argmin(lengths)), int(np.argmax(lengths))])


# The workload scales give a nearly uniform softmax; a x 8 sharpens it at full size.
def test_full_decode_b64_ctx32k_sharp(tpa):
    wl = I.WORKLOADS["decode_b64_ctx32k"]
    _full_decode(tpa, wl, [5, wl.batch - 2], a_scale=8.0)


def test_full_kvonly_decode_b16_ctx64k_128k_sharp(tpa):
    wl = I.WORKLOADS["kvonly_decode_b16_ctx64k_128k"]
    lengths = I.decode_lengths(wl)
    _full_decode(tpa, wl, [int(np.argmax(lengths))], a_scale=8.0)


def test_full_shared_basis_decode_b64_ctx32k(tpa):
    wl = I.WORKLOADS["shared_basis_decode_b64_ctx32k"]
    _full_decode(tpa, wl, [0, 41, wl.batch - 1])
