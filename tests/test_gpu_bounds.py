"""The bounds-checked build (libtpa_debug.so, -DTPA_DEBUG_BOUNDS) on the edge cases of
every call: no kernel may record TPA_DEVERR_BOUNDS (an index outside its buffer's
extent) or any other device error, and every bf16 output and all integer state must
equal the release library's bit for bit (the checks only guard accesses); fp32 outputs
agree to 1e-6 (the compiler may contract multiply-adds differently around the guards).

This stands in for a memory checker, which cannot run on these machines: a failed
check skips the access and leaves an error code, so a bad index is reported without a
fault.
"""
import numpy as np
import pytest
import torch

from tensor_product_attention_b200 import inputs as I
from helpers import dims_of, fill_cache

pytestmark = pytest.mark.gpu

TINY = I.WORKLOADS["prefill_tiny_f32"]
C2 = I.WORKLOADS["prefill_b8_s2048_d1024"]
C3 = I.WORKLOADS["decode_b64_ctx32k"]
C4 = I.WORKLOADS["kvonly_decode_b16_ctx64k_128k"]
C5 = I.WORKLOADS["layer_prefill_b4_s8192_d2048"]


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _layer_case(tpa, wl, batch, chunks, decode_steps):
    """project -> append -> prefill in chunks (the last chunk ends exactly at the cache
    capacity minus the decode steps), then fused decode steps up to the capacity, then
    a plain decode and the output projection; returns every output tensor."""
    dims = dims_of(wl, tpa)
    S = sum(chunks)
    cap = S + decode_steps
    cs = torch.empty((cap, wl.head_dim // 2, 2), dtype=torch.float32, device="cuda")
    tpa.tpa_rope_table(dims, wl.rope_base, cap, cs)
    xs = [I.prefill_x(wl, b, cap) for b in range(batch)]
    w = I.prefill_w(wl).cuda()
    cache = tpa.alloc_cache(dims, batch, cap, fill=0.0)
    if wl.shared_basis:
        basis = I.shared_basis(wl)
        tpa.tpa_shared_basis_tables(dims, basis["b_k"].cuda(), basis["b_v"].cuda(), cs, cap, cache.b_k, cache.b_v)
    outs, s0 = [], 0
    for n in chunks:
        x = torch.cat([xb[s0:s0 + n] for xb in xs]).cuda()
        fac = tpa.alloc_factors(dims, batch * n)
        tpa.tpa_project(dims, x, w, batch, n, [s0] * batch, cs, cap, fac)
        tpa.tpa_cache_append(dims, cache, fac, batch, n, [s0] * batch)
        out = torch.zeros((batch * n, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
        tpa.tpa_prefill(dims, fac, cache, batch, n, [s0] * batch, out)
        outs.append(out)
        s0 += n
    for k in range(decode_steps):
        L = [S + k] * batch
        xn = torch.stack([xb[S + k] for xb in xs]).cuda()
        out = torch.zeros((batch, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
        tpa.tpa_decode_step(dims, xn, w, cs, cap, cache, L, out, tpa.alloc_step_workspace(dims, L))
        outs.append(out)
    if wl.d_model:
        attn = outs[0]
        wo = I.output_w(wl).cuda()
        y = torch.zeros((attn.shape[0], wl.d_model), dtype=dims.torch_dtype, device="cuda")
        tpa.tpa_output_project(dims, attn, wo, y)
        outs.append(y)
    outs += [cache.a_k, cache.a_v, cache.b_k, cache.b_v, cache.lengths]
    return outs


def _decode_case(tpa, wl, lengths, cap):
    dims = dims_of(wl, tpa)
    batch = len(lengths)
    cache = tpa.alloc_cache(dims, batch + 1, cap, fill=0.0)     # one sequence more than used
    if wl.shared_basis:
        cs = torch.empty((cap, wl.head_dim // 2, 2), dtype=torch.float32, device="cuda")
        tpa.tpa_rope_table(dims, wl.rope_base, cap, cs)
        basis = I.shared_basis(wl)
        tpa.tpa_shared_basis_tables(dims, basis["b_k"].cuda(), basis["b_v"].cuda(), cs, cap, cache.b_k, cache.b_v)
    seqs = [I.decode_sequence(wl, b, L) for b, L in enumerate(lengths)]
    for b, seq in enumerate(seqs):
        fill_cache(cache, b, seq)
    if wl.rank_q:
        q_a = torch.stack([s["a_q"] for s in seqs]).cuda()
        q_b = torch.stack([s["b_q"] for s in seqs]).cuda()
    else:
        q_a, q_b = None, torch.stack([s["q"] for s in seqs]).cuda()
    out = torch.zeros((batch, wl.n_heads, wl.head_dim), dtype=dims.torch_dtype, device="cuda")
    tpa.tpa_decode(dims, q_a, q_b, cache, lengths, out, tpa.alloc_workspace(dims, lengths))
    out2 = torch.zeros_like(out)
    tpa.tpa_decode_static(dims, q_a, q_b, cache, lengths, out2)
    return [out, out2]


LAYER_CASES = [
    (TINY, 2, [1, 30], 2),                                           # fp32 CUDA-core kernels
    (I.custom("bd_d64", C2, d_model=256), 2, [37, 64], 2),           # packed prefill path
    (I.custom("bd_d128", C5, d_model=128), 1, [1, 129], 1),
    (I.custom("bd_kv", C4, d_model=256, n_heads=16, seed=1031), 2, [70], 2),
    (I.custom("bd_r1", C2, d_model=128, n_heads=8, rank_q=3, rank_k=1, rank_v=1), 2, [50], 1),
    (I.custom("bd_sb", C5, d_model=128, shared_basis=True), 2, [33, 31], 2),
    (I.custom("bd_sb_f32", TINY, shared_basis=True), 1, [20], 1),
]

DECODE_CASES = [
    (I.custom("bd_dec", C3), [1, 64, 129, 700], 700),                # length = capacity
    (I.custom("bd_dec", C3), [3001, 1], 3001),
    (I.custom("bd_dec_d64", C3, head_dim=64), [65, 2], 66),
    (I.custom("bd_dec_kv", C4), [5, 2049], 2050),
    (I.custom("bd_dec_f32", C3, dtype="f32", n_heads=4, head_dim=16, rank_q=2, rank_k=1, rank_v=1), [1, 40], 40),
    (I.custom("bd_dec_sb", C3, shared_basis=True), [1, 30], 30),     # capacity below one key tile
    (I.custom("bd_dec_sb", C3, shared_basis=True), [12000, 9001], 12000),
]


def _run_both(tpa, fn):
    with tpa.use_library(tpa.DEBUG_LIB_PATH):
        assert "bounds-checked" in tpa.tpa_build_info()
        got = fn()
        torch.cuda.synchronize()
        code = tpa.tpa_get_device_error()
    assert code == 0, f"device error {code} (2 = an index outside its buffer)"
    want = fn()
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    assert len(got) == len(want)
    for i, (g, w) in enumerate(zip(got, want)):
        if g.dtype == torch.float32:
            # fp32 kernels: the guards change the code around some multiply-adds, so
            # the compiler may contract them into FMAs differently (last-bit changes)
            den = max(float(w.abs().max()), 1e-30)
            assert float((g - w).abs().max()) / den < 1e-6, f"output {i} differs from the release build"
        else:
            assert torch.equal(_bits(g), _bits(w)), f"output {i} differs from the release build"


@pytest.mark.parametrize("case", LAYER_CASES, ids=[c[0].name + "-" + c[0].dtype for c in LAYER_CASES])
def test_bounds_checked_layer(tpa, case):
    wl, batch, chunks, steps = case
    _run_both(tpa, lambda: _layer_case(tpa, wl, batch, chunks, steps))


@pytest.mark.parametrize("case", DECODE_CASES, ids=[f"{c[0].name}-L{max(c[1])}" for c in DECODE_CASES])
def test_bounds_checked_decode(tpa, case):
    wl, lengths, cap = case
    _run_both(tpa, lambda: _decode_case(tpa, wl, lengths, cap))
