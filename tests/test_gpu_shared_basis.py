"""GPU parity for the shared-basis variant (B_K, B_V shared across tokens): every call
that changes with it, against the fp64 oracle on the same seeded inputs.

The oracle builds its own per-position tables from the basis in fp64
(``oracle.shared_basis_tables``); nothing the GPU computes is fed to it.  Tolerances
as in test_gpu_parity: 1e-5 (fp32 layers), 1e-2 (bf16 layers); cache rows and lengths
bit for bit.
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
C4 = I.WORKLOADS["kvonly_decode_b16_ctx64k_128k"]
C5 = I.WORKLOADS["layer_prefill_b4_s8192_d2048"]
SB = I.WORKLOADS["shared_basis_decode_b64_ctx32k"]


def shared(name, base, **changes):
    return I.custom(name, base, shared_basis=True, **changes)


def rope_table(tpa, dims, base, max_pos):
    cs = torch.empty((max_pos, dims.head_dim // 2, 2), dtype=torch.float32, device="cuda")
    tpa.tpa_rope_table(dims, base, max_pos, cs)
    return cs


def gpu_tables(tpa, wl, dims, cache, basis, max_pos=None):
    """Fill the cache's b_k, b_v tables from the basis on the GPU (product call)."""
    cap = cache.b_k.shape[0]
    max_pos = cap if max_pos is None else max_pos
    cs = rope_table(tpa, dims, wl.rope_base, max_pos)
    tpa.tpa_shared_basis_tables(dims, basis["b_k"].cuda(), basis["b_v"].cuda(), cs, max_pos,
                                cache.b_k, cache.b_v)
    return cs


def oracle_tables(wl, basis, capacity):
    return oracle.shared_basis_tables({n: f64(t) for n, t in basis.items()}, oracle_dims(wl),
                                      capacity, wl.rope_base)


# ------------------------------------------------------------------------- tables

@pytest.mark.parametrize("wl", [shared("t_f32", TINY), shared("t_d128", C5), shared("t_d64_r4", C2, rank_k=4, rank_v=3)],
                         ids=["f32", "bf16-d128", "bf16-d64-r4"])
def test_shared_basis_tables(tpa, wl):
    dims = dims_of(wl, tpa)
    cap = 4099
    cache = tpa.alloc_cache(dims, 1, cap, fill=float("nan"))
    basis = I.shared_basis(wl)
    gpu_tables(tpa, wl, dims, cache, basis, max_pos=cap + 10)
    torch.cuda.synchronize()
    ref = oracle_tables(wl, basis, cap)
    # one rounding of a rotation of dtype inputs: within the dtype's tolerance
    assert rel_err(cache.b_k, ref["b_k"]) < TOL[wl.dtype]
    # row 0 is the basis itself; the value table repeats the basis bit for bit
    ibits = torch.int16 if wl.dtype == "bf16" else torch.int32
    assert torch.equal(cache.b_k[0].cpu().view(ibits), basis["b_k"].view(ibits))
    want_v = basis["b_v"].view(ibits).unsqueeze(0).expand(cap, -1, -1)
    assert torch.equal(cache.b_v.cpu().view(ibits), want_v)


# --------------------------------------------------------------------- projection

@pytest.mark.parametrize("wl", [shared("pj_f32", TINY), shared("pj_bf16", C2, d_model=256),
                                shared("pj_kv", C4, d_model=256, n_heads=16, seed=1021)],
                         ids=["f32", "bf16", "bf16-kvonly"])
def test_project_shared_basis(tpa, wl):
    """No W_B_k / W_B_v blocks: the projection writes a_q, b_q (rotated), a_k, a_v."""
    dims = dims_of(wl, tpa)
    batch, seqlen, start = 2, 133, [0, 500]
    max_pos = max(start) + seqlen
    cs = rope_table(tpa, dims, wl.rope_base, max_pos)
    x = torch.cat([I.prefill_x(wl, b, seqlen) for b in range(batch)]).cuda()
    w = I.prefill_w(wl)
    assert w.shape[0] == dims.n_proj
    out = tpa.alloc_factors(dims, batch * seqlen)
    assert out.b_k is None and out.b_v is None
    tpa.tpa_project(dims, x, w.cuda(), batch, seqlen, start, cs, max_pos, out)
    torch.cuda.synchronize()
    ref = oracle.project(f64(x), f64(w), oracle_dims(wl))
    if wl.rank_q == 0:
        ref["b_q"] = ref.pop("q")
    assert "b_k" not in ref and "b_v" not in ref
    pos = np.concatenate([np.arange(s, s + seqlen) for s in start])
    ref["b_q"] = oracle.rope_rotate(ref["b_q"], pos, wl.rope_base)
    for n, r in ref.items():
        assert rel_err(getattr(out, n), r) < TOL[wl.dtype], n


def test_cache_append_shared_basis_copies_a_only(tpa):
    wl = shared("ap", SB, n_heads=8, head_dim=64)
    dims = dims_of(wl, tpa)
    batch, n, cap = 3, 37, 128
    start = [0, 5, 91]
    fac = tpa.alloc_factors(dims, batch * n, queries=False)
    g = torch.Generator().manual_seed(9)
    for name in ("a_k", "a_v"):
        t = getattr(fac, name)
        t.copy_(torch.randn(t.shape, generator=g).to(t.dtype))
    cache = tpa.alloc_cache(dims, batch, cap, fill=-7.0)
    tpa.tpa_cache_append(dims, cache, fac, batch, n, start)
    torch.cuda.synchronize()
    for name in ("a_k", "a_v"):
        src = getattr(fac, name).view(batch, n, *getattr(fac, name).shape[1:])
        for b in range(batch):
            assert torch.equal(getattr(cache, name)[b, start[b]:start[b] + n].view(torch.int16),
                               src[b].view(torch.int16))
    # the per-layer tables are not per-token state: append leaves them alone
    assert bool((cache.b_k == -7.0).all()) and bool((cache.b_v == -7.0).all())
    assert cache.lengths.cpu().tolist() == [s + n for s in start]


# ------------------------------------------------------------------------ prefill

PREFILL_CASES = [
    # (workload, batch, seqlen, starts, a_scale)
    (shared("sp_f32", TINY), 2, 37, [0, 50], 8.0),
    (shared("sp_d64", C2), 2, 200, [0, 13], 1.0),           # packed path (h 16, R 2)
    (shared("sp_d64", C2), 2, 131, [7, 0], 8.0),
    (shared("sp_d128", C5), 2, 150, [0, 90], 8.0),
    (shared("sp_r1", C2, n_heads=8, rank_k=1, rank_v=1, rank_q=3), 2, 150, [0, 40], 8.0),
    (shared("sp_r4", C2, rank_k=4, rank_v=4), 1, 97, [5], 8.0),
    (shared("sp_kv", C4, n_heads=16), 2, 170, [0, 33], 1.0),
]


@pytest.mark.parametrize("case", PREFILL_CASES,
                         ids=[f"{c[0].name}-S{c[2]}-st{max(c[3])}-a{c[4]:g}" for c in PREFILL_CASES])
def test_prefill_shared_basis(tpa, case):
    wl, batch, S, start, a_scale = case
    dims = dims_of(wl, tpa)
    od = oracle_dims(wl)
    cap = max(start) + S + 5
    cache = tpa.alloc_cache(dims, batch, cap, fill=float("nan"))
    basis = I.shared_basis(wl)
    gpu_tables(tpa, wl, dims, cache, basis)
    q = tpa.alloc_factors(dims, batch * S, kv=False)
    seqs = []
    for b in range(batch):
        seq = I.prefill_factors(wl, b, S, start[b] + S, a_scale)
        seqs.append(seq)
        fill_cache(cache, b, seq)
        if wl.rank_q == 0:
            q.b_q[b * S:(b + 1) * S].copy_(seq["q"])
        else:
            q.a_q[b * S:(b + 1) * S].copy_(seq["a_q"])
            q.b_q[b * S:(b + 1) * S].copy_(seq["b_q"])
    out = torch.empty((batch * S, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    tpa.tpa_prefill(dims, q, cache, batch, S, start, out)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    tab = oracle_tables(wl, basis, cap)
    for b in range(batch):
        seq = {k: f64(v) for k, v in seqs[b].items()}
        L = start[b] + S
        kv = {"a_k": seq["a_k"], "a_v": seq["a_v"], "b_k": tab["b_k"][:L], "b_v": tab["b_v"][:L]}
        ref = oracle.attend_from_factors(seq, kv, od, np.arange(start[b], L))
        assert rel_err(out[b * S:(b + 1) * S], ref) < TOL[wl.dtype], b


# ------------------------------------------------------------------------- decode

DECODE_CASES = [
    (shared("sd_f32", SB, dtype="f32", n_heads=4, head_dim=16, rank_q=2, rank_k=1, rank_v=1), [1, 64, 300], 1.0, 3),
    (shared("sd", SB), [1, 129, 1000], 1.0, 3),
    (shared("sd", SB), [4099, 77, 2048], 8.0, 3),
    # capacity below one key tile: the kept value stage is part zero fill
    (shared("sd", SB), [1, 5, 30], 8.0, 0),
    # more key tiles than SMs: CTAs start mid-sequence and parts cross sequences
    (shared("sd_multi", SB), [12000, 9001, 1, 14501], 8.0, 3),
    (shared("sd_multi", SB), [700] * 29 + [33], 8.0, 3),
    (shared("sd_kv", C4), [77, 5000], 1.0, 3),
    (shared("sd_kvmulti", C4), [20000, 13001], 8.0, 3),
    (shared("sd_d64", SB, head_dim=64), [2049, 1, 700], 8.0, 3),
    # pairs with an odd capacity (a-factor tiles by bulk copies) and the KV-only query
    (shared("sd_kv16", SB, rank_q=0, seed=1032), [333, 4000, 17], 8.0, 3),
    (shared("sd_odd", SB), [2049, 77, 1, 5000, 3], 1.0, 2),
]


@pytest.mark.parametrize("case", DECODE_CASES,
                         ids=[f"{c[0].name}-{c[0].dtype}-L{max(c[1])}-a{c[2]:g}-pad{c[3]}" for c in DECODE_CASES])
def test_decode_shared_basis(tpa, case):
    wl, lengths, a_scale, pad = case
    dims = dims_of(wl, tpa)
    od = oracle_dims(wl)
    batch = len(lengths)
    cap = max(lengths) + pad
    cache = tpa.alloc_cache(dims, batch, cap, fill=float("nan"))
    basis = I.shared_basis(wl)
    gpu_tables(tpa, wl, dims, cache, basis)
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
    tpa.tpa_decode(dims, q_a, q_b, cache, lengths, out, tpa.alloc_workspace(dims, lengths))
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    tab = oracle_tables(wl, basis, cap)
    for b, L in enumerate(lengths):
        seq = {k: f64(v) for k, v in seqs[b].items()}
        kv = {"a_k": seq["a_k"], "a_v": seq["a_v"], "b_k": tab["b_k"], "b_v": tab["b_v"]}
        ref = oracle.decode_attention(seq, kv, od, L)
        assert rel_err(out[b], ref) < TOL[wl.dtype], (b, L)


# ------------------------------------------------------------ end to end from x

E2E_CASES = [
    (shared("se_f32", TINY), 2, [40, 24]),
    (shared("se_d64", C2, d_model=256), 2, [150, 58]),
    (shared("se_d128", C5, d_model=256), 1, [130]),
    (shared("se_kv", C4, d_model=256, n_heads=16, seed=1022), 2, [100, 41]),
]


@pytest.mark.parametrize("case", E2E_CASES, ids=[c[0].name for c in E2E_CASES])
def test_shared_basis_layer_end_to_end(tpa, case):
    """tables -> project -> append -> prefill from x in one or two chunks, then a fused
    decode step for one more token, against the pages' forward (shared-basis reading)."""
    wl, batch, chunks = case
    dims = dims_of(wl, tpa)
    S = sum(chunks)
    basis = I.shared_basis(wl)
    xs = [I.prefill_x(wl, b, S + 1) for b in range(batch)]
    w = I.prefill_w(wl)
    wd = w.cuda()
    cache = tpa.alloc_cache(dims, batch, S + 1, fill=float("nan"))
    cs = gpu_tables(tpa, wl, dims, cache, basis)
    outs, s0 = [], 0
    for n in chunks:
        x = torch.cat([xb[s0:s0 + n] for xb in xs]).cuda()
        fac = tpa.alloc_factors(dims, batch * n)
        tpa.tpa_project(dims, x, wd, batch, n, [s0] * batch, cs, S + 1, fac)
        tpa.tpa_cache_append(dims, cache, fac, batch, n, [s0] * batch)
        out = torch.empty((batch * n, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
        tpa.tpa_prefill(dims, fac, cache, batch, n, [s0] * batch, out)
        outs.append(out.view(batch, n, wl.n_heads, wl.head_dim))
        s0 += n
    lengths = [S] * batch
    xn = torch.stack([xb[S] for xb in xs]).cuda()
    dec = torch.empty((batch, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    tpa.tpa_decode_step(dims, xn, wd, cs, S + 1, cache, lengths, dec, tpa.alloc_step_workspace(dims, lengths))
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    assert cache.lengths.cpu().tolist() == [S + 1] * batch
    ref, _ = oracle.tpa_forward(np.stack([f64(xb) for xb in xs]), f64(w), oracle_dims(wl), wl.rope_base,
                                basis={n: f64(t) for n, t in basis.items()})
    assert rel_err(torch.cat(outs, dim=1), ref[:, :S]) < TOL[wl.dtype]
    assert rel_err(dec, ref[:, S]) < TOL[wl.dtype]


def test_shared_basis_decode_step_writes_a_rows_like_append(tpa):
    """The fused step's cache rows equal project -> append's, bit for bit."""
    wl = shared("ss", C5, d_model=256)
    dims = dims_of(wl, tpa)
    lengths = [40, 1, 0]
    B, cap = len(lengths), max(lengths) + 2
    cache = tpa.alloc_cache(dims, B, cap, fill=float("nan"))
    twin = tpa.alloc_cache(dims, B, cap, fill=float("nan"))
    basis = I.shared_basis(wl)
    cs = gpu_tables(tpa, wl, dims, cache, basis)
    twin.b_k.copy_(cache.b_k)
    twin.b_v.copy_(cache.b_v)
    w = I.prefill_w(wl).cuda()
    xn = torch.stack([I.prefill_x(wl, b, L + 1)[L] for b, L in enumerate(lengths)]).cuda()
    out = torch.empty((B, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    # sequences start empty except for the rows the step reads: fill them from seeded A
    for b, L in enumerate(lengths):
        if L:
            seq = I.decode_sequence(wl, b, L)
            fill_cache(cache, b, {"a_k": seq["a_k"], "a_v": seq["a_v"]})
            fill_cache(twin, b, {"a_k": seq["a_k"], "a_v": seq["a_v"]})
    tpa.tpa_decode_step(dims, xn, w, cs, cap, cache, lengths, out, tpa.alloc_step_workspace(dims, lengths))
    fac = tpa.alloc_factors(dims, B)
    tpa.tpa_project(dims, xn, w, B, 1, lengths, cs, cap, fac)
    tpa.tpa_cache_append(dims, twin, fac, B, 1, lengths)
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    for n in ("a_k", "a_v"):
        for b, L in enumerate(lengths):
            assert torch.equal(getattr(cache, n)[b, L].view(torch.int16), getattr(twin, n)[b, L].view(torch.int16))
    assert cache.lengths.cpu().tolist() == [L + 1 for L in lengths]
