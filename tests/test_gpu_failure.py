"""Failure detection without a GPU fault: every wait in the tcgen05 kernels is bounded.

With the wait limit lowered to a single poll, the waits of each kernel run out.  The
kernel must record TPA_DEVERR_TIMEOUT in the device error word and return.  Before it
exits it drains its own copies and MMAs, under a separate fixed bound.  The CUDA
context must stay usable: the same call, after the limit is restored, gives exactly
the result it gave before.  No trap, no assert, no bad address is used.
"""
import pytest
import torch

from tensor_product_attention_b200 import inputs as I
from helpers import dims_of, fill_cache

pytestmark = pytest.mark.gpu

TIMEOUT = 1   # TPA_DEVERR_TIMEOUT


def _expire_then_recover(tpa, run, out):
    run()
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    ref = out.clone()
    tpa.tpa_set_wait_limit(1)
    try:
        out.zero_()
        run()
        code = tpa.tpa_get_device_error()
    finally:
        tpa.tpa_set_wait_limit(0)
    assert code == TIMEOUT
    out.zero_()
    run()
    torch.cuda.synchronize()
    assert tpa.tpa_get_device_error() == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_decode_wait_expiry(tpa):
    wl = I.custom("fail_dec", I.WORKLOADS["decode_b64_ctx32k"])
    dims = dims_of(wl, tpa)
    lengths = [9000, 7000, 12000, 5000]
    cache = tpa.alloc_cache(dims, len(lengths), max(lengths))
    seqs = [I.decode_sequence(wl, b, L) for b, L in enumerate(lengths)]
    for b, sq in enumerate(seqs):
        fill_cache(cache, b, sq)
    q_a = torch.stack([sq["a_q"] for sq in seqs]).cuda()
    q_b = torch.stack([sq["b_q"] for sq in seqs]).cuda()
    out = torch.empty((len(lengths), wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    ws = tpa.alloc_workspace(dims, lengths)
    _expire_then_recover(tpa, lambda: tpa.tpa_decode(dims, q_a, q_b, cache, lengths, out, ws), out)


def test_prefill_wait_expiry(tpa):
    wl = I.custom("fail_pre", I.WORKLOADS["prefill_b8_s2048_d1024"])
    dims = dims_of(wl, tpa)
    B, S = 2, 700
    cache = tpa.alloc_cache(dims, B, S)
    q = tpa.alloc_factors(dims, B * S, kv=False)
    for b in range(B):
        sq = I.prefill_factors(wl, b, S, S)
        fill_cache(cache, b, sq)
        q.a_q[b * S:(b + 1) * S].copy_(sq["a_q"])
        q.b_q[b * S:(b + 1) * S].copy_(sq["b_q"])
    out = torch.empty((B * S, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    _expire_then_recover(tpa, lambda: tpa.tpa_prefill(dims, q, cache, B, S, [0] * B, out), out)


def test_projection_wait_expiry(tpa):
    wl = I.custom("fail_proj", I.WORKLOADS["prefill_b8_s2048_d1024"], d_model=512)
    dims = dims_of(wl, tpa)
    B, S = 2, 1000
    cs = torch.empty((S, wl.head_dim // 2, 2), dtype=torch.float32, device="cuda")
    tpa.tpa_rope_table(dims, wl.rope_base, S, cs)
    x = torch.cat([I.prefill_x(wl, b, S) for b in range(B)]).cuda()
    w = I.prefill_w(wl).cuda()
    fac = tpa.alloc_factors(dims, B * S)
    _expire_then_recover(tpa, lambda: tpa.tpa_project(dims, x, w, B, S, [0] * B, cs, S, fac), fac.b_k)
