"""GPU parity: every call of the C ABI against the fp64 oracle on the same seeded
inputs, at sizes that span several kernel tiles and a ragged tail.

Tolerance: max|gpu - oracle| / max|oracle| per output tensor, 1e-5 for fp32 layers
and 1e-2 for bf16 layers (bf16 inputs, fp32 accumulation); cache bytes and lengths
must match bit for bit.  Inputs come from tensor_product_attention_b200.inputs only;
nothing the GPU computes is fed to the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from tensor_product_attention_b200 import inputs as I
from helpers import TOL, dims_of, f64, fill_cache, oracle_dims, rel_err

pytestmark = pytest.mark.gpu

TINY = I.WORKLOADS["prefill_tiny_f32"]
C2 = I.WORKLOADS["prefill_b8_s2048_d1024"]
C3 = I.WORKLOADS["decode_b64_ctx32k"]
C4 = I.WORKLOADS["kvonly_decode_b16_ctx64k_128k"]
C5 = I.WORKLOADS["layer_prefill_b4_s8192_d2048"]


def rope_table(tpa, dims, base, max_pos):
    cs = torch.empty((max_pos, dims.head_dim // 2, 2), dtype=torch.float32, device="cuda")
    tpa.tpa_rope_table(dims, base, max_pos, cs)
    return cs


# --------------------------------------------------------------------------- RoPE

@pytest.mark.parametrize("head_dim,base", [(16, 1e4), (128, 5e5)])
def test_rope_table_matches_oracle_rotation(tpa, head_dim, base):
    dims = tpa.Dims(64, 4, head_dim, 2, 1, 1, tpa.F32)
    max_pos = 131072
    cs = rope_table(tpa, dims, base, max_pos).cpu().numpy().astype(np.float64)
    pos = np.array([0, 1, 2, 17, 1000, 65535, 99991, 131071])
    # rotating the unit vector e_{2k} at position p gives (cos, sin)(p theta_k)
    unit = np.zeros((len(pos), head_dim // 2, head_dim))
    for k in range(head_dim // 2):
        unit[:, k, 2 * k] = 1.0
    rot = oracle.rope_rotate(unit, pos, base)
    want_c = np.stack([rot[:, k, 2 * k] for k in range(head_dim // 2)], axis=1)
    want_s = np.stack([rot[:, k, 2 * k + 1] for k in range(head_dim // 2)], axis=1)
    assert np.max(np.abs(cs[pos, :, 0] - want_c)) < 1.2e-7
    assert np.max(np.abs(cs[pos, :, 1] - want_s)) < 1.2e-7


# --------------------------------------------------------------------- projection

def _project_case(tpa, wl, batch, seqlen, start):
    dims = dims_of(wl, tpa)
    max_pos = max(start) + seqlen
    cs = rope_table(tpa, dims, wl.rope_base, max_pos)
    x = torch.cat([I.prefill_x(wl, b, seqlen) for b in range(batch)]).cuda()
    w = I.prefill_w(wl).cuda()
    out = tpa.alloc_factors(dims, batch * seqlen)
    tpa.tpa_project(dims, x, w, batch, seqlen, start, cs, max_pos, out)
    torch.cuda.synchronize()
    od = oracle_dims(wl)
    ref = oracle.project(f64(x), f64(w), od)
    pos = np.concatenate([np.arange(s, s + seqlen) for s in start])
    if wl.rank_q == 0:
        # TPA-KVonly: the rotated plain query lands in the b_q slot
        ref["b_q"] = ref.pop("q")
    names = [n for n in oracle.FACTOR_NAMES if n in ref]
    ref["b_q"] = oracle.rope_rotate(ref["b_q"], pos, wl.rope_base)
    ref["b_k"] = oracle.rope_rotate(ref["b_k"], pos, wl.rope_base)
    return {n: rel_err(getattr(out, n), ref[n]) for n in names}


def test_project_tiny_f32(tpa):
    errs = _project_case(tpa, TINY, 1, 64, [0])
    assert max(errs.values()) < TOL["f32"], errs
    errs = _project_case(tpa, TINY, 3, 21, [0, 40, 7])
    assert max(errs.values()) < TOL["f32"], errs


@pytest.mark.parametrize("wl", [C2, C5], ids=["d64", "d128"])
def test_project_bf16_ragged(tpa, wl):
    small = I.custom("proj_small", wl, d_model=256 if wl is C2 else 384)
    errs = _project_case(tpa, small, 3, 173, [0, 5, 1000])
    assert max(errs.values()) < TOL["bf16"], errs


@pytest.mark.parametrize("wl", [C2, C5], ids=["d64", "d128"])
def test_project_bf16_many_tiles(tpa, wl):
    """4100 tokens (more tiles than SMs, so persistent CTAs take several tiles and both
    TMEM accumulators), a ragged last tile and two sequences at different start
    positions: every element of all six factors against the oracle."""
    errs = _project_case(tpa, wl, 2, 2050, [0, 3])
    assert max(errs.values()) < TOL["bf16"], errs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_project_kvonly(tpa, dtype):
    """TPA-KVonly: W_Q (h*d_h rows) in the W_B_q slot, rotated per head into b_q."""
    wl = I.custom("proj_kvonly", C4, dtype=dtype, d_model=256, seed=1011)
    errs = _project_case(tpa, wl, 2, 150, [0, 700])
    assert set(errs) == {"b_q", "a_k", "a_v", "b_k", "b_v"}
    assert max(errs.values()) < TOL[dtype], errs


# ------------------------------------------------------------------ cache append

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_cache_append_bit_exact(tpa, dtype):
    wl = I.custom("append", C3, dtype=dtype, n_heads=8, head_dim=64)
    dims = dims_of(wl, tpa)
    batch, n, cap = 3, 37, 128
    start = [0, 5, 91]
    fac = tpa.alloc_factors(dims, batch * n, queries=False)
    g = torch.Generator().manual_seed(7)
    for name in ("a_k", "a_v", "b_k", "b_v"):
        t = getattr(fac, name)
        t.copy_(torch.randn(t.shape, generator=g).to(t.dtype))
    cache = tpa.alloc_cache(dims, batch + 1, cap, fill=-7.0)
    tpa.tpa_cache_append(dims, cache, fac, batch, n, start)
    torch.cuda.synchronize()
    ibits = torch.int16 if dtype == "bf16" else torch.int32
    for name in ("a_k", "a_v", "b_k", "b_v"):
        src = getattr(fac, name).view(batch, n, *getattr(fac, name).shape[1:])
        dst = getattr(cache, name)
        for b in range(batch):
            assert torch.equal(dst[b, start[b]:start[b] + n].view(ibits), src[b].view(ibits))
            untouched = torch.cat([dst[b, :start[b]], dst[b, start[b] + n:]])
            assert bool((untouched == -7.0).all())
        assert bool((dst[batch] == -7.0).all())
    assert cache.lengths.cpu().tolist() == [s + n for s in start] + [0]


# ------------------------------------------------------------------------ prefill

PREFILL_CASES = [
    # (workload, batch, seqlen, starts, a_scale)
    (TINY, 1, 64, [0], 1.0),
    (TINY, 2, 37, [0, 50], 8.0),
    (I.custom("p_d64", C2), 2, 200, [0, 13], 1.0),
    (I.custom("p_d64", C2), 2, 131, [7, 0], 8.0),
    (I.custom("p_d128", C5), 2, 150, [0, 90], 1.0),
    (I.custom("p_d128", C5), 1, 1, [300], 8.0),
    (I.custom("p_d128", C5), 1, 256, [0], 8.0),
    # the tensor-core kernel's generic paths: ranks 1 and 4, head counts other than 16
    (I.custom("p_r1", C2, n_heads=8, rank_k=1, rank_v=1, rank_q=3), 2, 150, [0, 40], 8.0),
    (I.custom("p_r4", C2, rank_k=4, rank_v=4), 2, 97, [5, 0], 8.0),
    (I.custom("p_h32", C5, n_heads=32), 1, 160, [30], 8.0),
    (I.custom("p_h4", C2, n_heads=4, rank_k=2, rank_v=2), 1, 300, [0], 1.0),
    # TPA-KVonly: plain per-head query (rank_q = 0)
    (I.custom("p_kv_f32", C4, dtype="f32", n_heads=4, head_dim=32), 2, 45, [0, 20], 8.0),
    (I.custom("p_kv_d128", C4, n_heads=16), 2, 170, [0, 33], 1.0),
    (I.custom("p_kv_d128", C4, n_heads=16), 1, 150, [64], 8.0),
    (I.custom("p_kv_d64", C4, n_heads=16, head_dim=64), 2, 131, [7, 0], 8.0),
]


@pytest.mark.parametrize("case", PREFILL_CASES,
                         ids=[f"{c[0].dtype}-d{c[0].head_dim}-S{c[2]}-st{max(c[3])}-a{c[4]:g}" for c in PREFILL_CASES])
def test_prefill_from_factors(tpa, case):
    wl, batch, S, start, a_scale = case
    dims = dims_of(wl, tpa)
    od = oracle_dims(wl)
    cap = max(start) + S + 5
    cache = tpa.alloc_cache(dims, batch, cap, fill=float("nan"))
    q = tpa.alloc_factors(dims, batch * S, kv=False)
    seqs = []
    for b in range(batch):
        seq = I.prefill_factors(wl, b, S, start[b] + S, a_scale)
        seqs.append(seq)
        fill_cache(cache, b, seq)
        if wl.rank_q == 0:
            q.b_q[b * S:(b + 1) * S].copy_(seq["q"])     # TPA-KVonly query in the b_q slot
        else:
            q.a_q[b * S:(b + 1) * S].copy_(seq["a_q"])
            q.b_q[b * S:(b + 1) * S].copy_(seq["b_q"])
    out = torch.empty((batch * S, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    tpa.tpa_prefill(dims, q, cache, batch, S, start, out)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    for b in range(batch):
        seq = {k: f64(v) for k, v in seqs[b].items()}
        ref = oracle.attend_from_factors(seq, seq, od, np.arange(start[b], start[b] + S))
        err = rel_err(out[b * S:(b + 1) * S], ref)
        assert err < TOL[wl.dtype], (b, err)


# ------------------------------------------------------------------------- decode

DECODE_CASES = [
    (I.custom("d_f32", C3, dtype="f32", n_heads=4, head_dim=16, rank_q=2, rank_k=1, rank_v=1), [1, 64, 300], 1.0),
    (I.custom("d_small", C3), [1, 129, 1000], 1.0),
    (I.custom("d_small", C3), [4099, 77, 2048], 8.0),
    (I.custom("d_kvonly", C4), [77, 5000], 1.0),
    (I.custom("d_kvonly", C4), [1, 3001], 8.0),
    # more key tiles than SMs: every CTA walks several tiles, parts cross sequences
    (I.custom("d_multi", C3), [12000, 9001, 1, 14500], 1.0),
    (I.custom("d_multi", C3), [12000, 9001, 1, 14501], 8.0),
    (I.custom("d_multi", C3), [700] * 29 + [33], 8.0),
    (I.custom("d_kvmulti", C4), [20000, 13001], 8.0),
    # head_dim 64 (the value MMA repeats the 64-wide tile to fill its 128 rows)
    (I.custom("d_d64", C3, head_dim=64), [2049, 1, 700], 8.0),
    (I.custom("d_d64", C3, head_dim=64), [9000] * 8, 1.0),
]


@pytest.mark.parametrize("case", DECODE_CASES,
                         ids=[f"{c[0].name}-{c[0].dtype}-L{max(c[1])}-a{c[2]:g}" for c in DECODE_CASES])
def test_decode_from_factors(tpa, case):
    wl, lengths, a_scale = case
    dims = dims_of(wl, tpa)
    od = oracle_dims(wl)
    batch = len(lengths)
    cache = tpa.alloc_cache(dims, batch, max(lengths) + 3, fill=float("nan"))
    seqs = []
    for b, L in enumerate(lengths):
        seq = I.decode_sequence(wl, b, L, a_scale)
        seqs.append(seq)
        fill_cache(cache, b, seq)
    if wl.rank_q:
        q_a = torch.stack([s["a_q"] for s in seqs]).cuda()
        q_b = torch.stack([s["b_q"] for s in seqs]).cuda()
    else:
        q_a, q_b = None, torch.stack([s["q"] for s in seqs]).cuda()
    out = torch.empty((batch, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    ws = tpa.alloc_workspace(dims, lengths)
    tpa.tpa_decode(dims, q_a, q_b, cache, lengths, out, ws)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    for b, L in enumerate(lengths):
        seq = {k: f64(v) for k, v in seqs[b].items()}
        ref = oracle.decode_attention(seq, seq, od, L)
        err = rel_err(out[b], ref)
        assert err < TOL[wl.dtype], (b, L, err)


def test_decode_is_deterministic(tpa):
    wl = I.custom("d_small", C3)
    dims = dims_of(wl, tpa)
    lengths = [3000, 777]
    cache = tpa.alloc_cache(dims, 2, 3000)
    seqs = [I.decode_sequence(wl, b, L) for b, L in enumerate(lengths)]
    for b, s in enumerate(seqs):
        fill_cache(cache, b, s)
    q_a = torch.stack([s["a_q"] for s in seqs]).cuda()
    q_b = torch.stack([s["b_q"] for s in seqs]).cuda()
    ws = tpa.alloc_workspace(dims, lengths)
    outs = []
    for _ in range(3):
        out = torch.empty((2, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
        tpa.tpa_decode(dims, q_a, q_b, cache, lengths, out, ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))


# ------------------------------------------------------------ end to end from x

def _layer_prefill(tpa, wl, x, w, dims, cache, cs, max_pos, start, seqlen, batch):
    fac = tpa.alloc_factors(dims, batch * seqlen)
    tpa.tpa_project(dims, x, w, batch, seqlen, start, cs, max_pos, fac)
    tpa.tpa_cache_append(dims, cache, fac, batch, seqlen, start)
    out = torch.empty((batch * seqlen, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    tpa.tpa_prefill(dims, fac, cache, batch, seqlen, start, out)
    return out


E2E_CASES = [
    (TINY, 1, [64]),
    (TINY, 2, [40, 24]),
    (I.custom("e_d64", C2, d_model=256), 2, [150, 58]),
    (I.custom("e_d128", C5, d_model=256), 2, [130]),
    (I.custom("e_kv_f32", C4, dtype="f32", d_model=64, n_heads=4, head_dim=16, seed=1012), 2, [33, 20]),
    (I.custom("e_kv_d128", C4, d_model=256, n_heads=16, seed=1013), 2, [100, 41]),
]


@pytest.mark.parametrize("case", E2E_CASES,
                         ids=[f"{c[0].dtype}-d{c[0].head_dim}-rq{c[0].rank_q}-chunks{len(c[2])}" for c in E2E_CASES])
def test_layer_prefill_end_to_end(tpa, case):
    """project -> append -> prefill from x, in one or two chunks (second chunk at
    start_pos > 0), against the pages' forward evaluated in fp64."""
    wl, batch, chunks = case
    dims = dims_of(wl, tpa)
    S = sum(chunks)
    cs = rope_table(tpa, dims, wl.rope_base, S)
    xs = [I.prefill_x(wl, b, S) for b in range(batch)]
    w = I.prefill_w(wl)
    wd = w.cuda()
    cache = tpa.alloc_cache(dims, batch, S, fill=float("nan"))
    outs, s0 = [], 0
    for n in chunks:
        x = torch.cat([xb[s0:s0 + n] for xb in xs]).cuda()
        outs.append(_layer_prefill(tpa, wl, x, wd, dims, cache, cs, S, [s0] * batch, n, batch)
                    .view(batch, n, wl.n_heads, wl.head_dim))
        s0 += n
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=1)
    ref, _ = oracle.tpa_forward(np.stack([f64(xb) for xb in xs]), f64(w), oracle_dims(wl), wl.rope_base)
    assert rel_err(got, ref) < TOL[wl.dtype]
    assert cache.lengths.cpu().tolist() == [S] * batch


def test_decode_step_after_prefill_end_to_end(tpa):
    """Prefill S tokens, then one decode step: project the new token at position S,
    append it, decode; against the pages' forward over all S+1 tokens."""
    wl = I.custom("e_dec", C5, d_model=256)
    dims = dims_of(wl, tpa)
    batch, S = 2, 97
    cs = rope_table(tpa, dims, wl.rope_base, S + 1)
    xs = [I.prefill_x(wl, b, S + 1) for b in range(batch)]
    w = I.prefill_w(wl)
    wd = w.cuda()
    cache = tpa.alloc_cache(dims, batch, S + 1)
    x = torch.cat([xb[:S] for xb in xs]).cuda()
    _layer_prefill(tpa, wl, x, wd, dims, cache, cs, S + 1, [0] * batch, S, batch)
    xn = torch.stack([xb[S] for xb in xs]).cuda()
    fac = tpa.alloc_factors(dims, batch)
    tpa.tpa_project(dims, xn, wd, batch, 1, [S] * batch, cs, S + 1, fac)
    tpa.tpa_cache_append(dims, cache, fac, batch, 1, [S] * batch)
    out = torch.empty((batch, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    lengths = [S + 1] * batch
    tpa.tpa_decode(dims, fac.a_q, fac.b_q, cache, lengths, out, tpa.alloc_workspace(dims, lengths))
    torch.cuda.synchronize()
    ref, _ = oracle.tpa_forward(np.stack([f64(xb) for xb in xs]), f64(w), oracle_dims(wl), wl.rope_base)
    assert rel_err(out, ref[:, S]) < TOL["bf16"]


# ------------------------------------------------------------ fused decode step

STEP_CASES = [
    # (workload, pre-step lengths)
    (I.custom("s_d128", C5, d_model=256), [97, 40, 1]),
    (I.custom("s_kv", C4, d_model=256, n_heads=16, seed=1014), [64, 133]),
    (I.custom("s_f32", TINY), [30, 0]),
]


@pytest.mark.parametrize("case", STEP_CASES,
                         ids=[f"{c[0].dtype}-d{c[0].head_dim}-rq{c[0].rank_q}" for c in STEP_CASES])
def test_decode_step_fused(tpa, case):
    """tpa_decode_step (project the new token straight into the cache, then decode)
    against the pages' forward over lengths[b] + 1 tokens, and against the separate
    project -> append path for the cache rows it writes (bit for bit)."""
    wl, lengths = case
    dims = dims_of(wl, tpa)
    B, cap = len(lengths), max(lengths) + 3
    max_pos = cap
    cs = rope_table(tpa, dims, wl.rope_base, max_pos)
    xs = [I.prefill_x(wl, b, L + 1) for b, L in enumerate(lengths)]
    w = I.prefill_w(wl)
    wd = w.cuda()
    cache = tpa.alloc_cache(dims, B, cap, fill=float("nan"))
    twin = tpa.alloc_cache(dims, B, cap, fill=float("nan"))
    for b, L in enumerate(lengths):
        if L == 0:
            continue
        fac = tpa.alloc_factors(dims, L)
        tpa.tpa_project(dims, xs[b][:L].cuda(), wd, 1, L, [0], cs, max_pos, fac)
        one = tpa.Cache(*(getattr(cache, n)[b:b + 1] for n in ("a_k", "a_v", "b_k", "b_v")), cache.lengths[b:b + 1])
        tpa.tpa_cache_append(dims, one, fac, 1, L, [0])
        for n in ("a_k", "a_v", "b_k", "b_v"):
            getattr(twin, n)[b].copy_(getattr(cache, n)[b])
    xn = torch.stack([xs[b][L] for b, L in enumerate(lengths)]).cuda()
    out = torch.empty((B, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    tpa.tpa_decode_step(dims, xn, wd, cs, max_pos, cache, lengths, out, tpa.alloc_step_workspace(dims, lengths))
    # the same token through the separate calls, into the twin cache
    fac1 = tpa.alloc_factors(dims, B)
    tpa.tpa_project(dims, xn, wd, B, 1, lengths, cs, max_pos, fac1)
    tpa.tpa_cache_append(dims, twin, fac1, B, 1, lengths)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    assert cache.lengths.cpu().tolist() == [L + 1 for L in lengths]
    ibits = torch.int16 if wl.dtype == "bf16" else torch.int32
    for n in ("a_k", "a_v", "b_k", "b_v"):
        for b, L in enumerate(lengths):
            assert torch.equal(getattr(cache, n)[b, L].view(ibits), getattr(twin, n)[b, L].view(ibits)), (n, b)
    od = oracle_dims(wl)
    for b, L in enumerate(lengths):
        ref = oracle.tpa_forward_rows(f64(xs[b]), f64(w), od, wl.rope_base, [L])
        assert rel_err(out[b:b + 1], ref) < TOL[wl.dtype], b


# ------------------------------------------------------------ output projection

@pytest.mark.parametrize("wl,T", [(TINY, 64), (I.custom("wo_d64", C2, d_model=512), 301),
                                  (I.custom("wo_d128", C5, d_model=384), 77), (C2, 5000)],
                         ids=["f32", "bf16-d64", "bf16-d128", "bf16-many-tiles"])
def test_output_project(tpa, wl, T):
    dims = dims_of(wl, tpa)
    attn = I.attn_out(wl, T).cuda()
    w_o = I.output_w(wl).cuda()
    out = torch.empty((T, wl.d_model), dtype=dims.torch_dtype, device="cuda")
    tpa.tpa_output_project(dims, attn, w_o, out)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    assert rel_err(out, oracle.output_projection(f64(attn), f64(w_o))) < TOL[wl.dtype]


def test_full_layer_with_output_projection(tpa):
    """x -> project -> append -> prefill -> wo, against the pages' forward followed by wo."""
    wl = I.custom("e_wo", C5, d_model=256)
    dims = dims_of(wl, tpa)
    B, S = 2, 90
    cs = rope_table(tpa, dims, wl.rope_base, S)
    xs = [I.prefill_x(wl, b, S) for b in range(B)]
    w, w_o = I.prefill_w(wl), I.output_w(wl)
    cache = tpa.alloc_cache(dims, B, S)
    attn = _layer_prefill(tpa, wl, torch.cat(xs).cuda(), w.cuda(), dims, cache, cs, S, [0] * B, S, B)
    y = torch.empty((B * S, wl.d_model), dtype=torch.bfloat16, device="cuda")
    tpa.tpa_output_project(dims, attn, w_o.cuda(), y)
    torch.cuda.synchronize()
    ref, _ = oracle.tpa_forward(np.stack([f64(xb) for xb in xs]), f64(w), oracle_dims(wl), wl.rope_base)
    want = oracle.output_projection(ref.reshape(B * S, wl.n_heads, wl.head_dim), f64(w_o))
    assert rel_err(y, want) < TOL["bf16"]
