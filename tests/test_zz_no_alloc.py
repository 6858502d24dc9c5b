"""tpa_decode_static: decode for callers that cannot allocate device memory.

Such callers (a plug-in whose host application owns every allocation, a server that
must not call cudaMalloc while it serves) pass only inputs and outputs; the split-K
scratch is the library's own fixed device array.  These checks call it through the
C ABI and compare it with tpa_decode on a caller-allocated workspace, twice in a
row, so that the scratch left by one call is shown not to disturb the next.  Both
calls plan the same parts and run the same kernels in the same order, so the
results must agree bit for bit, not only within the bf16 parity tolerance.

The file is named to be collected last, so that a failure here cannot hide an
earlier test's result in a run that stops at the first failure.
"""
import ctypes

import pytest
import torch

from tensor_product_attention_b200 import inputs as I
from helpers import TOL, dims_of, fill_cache, rel_err

pytestmark = pytest.mark.gpu


def _decode_inputs(tpa, wl, lengths):
    dims = dims_of(wl, tpa)
    cache = tpa.alloc_cache(dims, len(lengths), max(lengths), fill=float("nan"))
    qa, qb = [], []
    for b, L in enumerate(lengths):
        seq = I.decode_sequence(wl, b, L, a_scale=4.0)
        fill_cache(cache, b, seq)
        if wl.rank_q:
            qa.append(seq["a_q"]); qb.append(seq["b_q"])
        else:
            qb.append(seq["q"])
    q_a = torch.stack(qa).cuda() if qa else None
    return dims, cache, q_a, torch.stack(qb).cuda()


@pytest.mark.parametrize("name,lengths", [
    ("decode_b64_ctx32k", [1, 300, 4099, 2048]),
    ("kvonly_decode_b16_ctx64k_128k", [77, 9000]),
])
def test_static_scratch_decode_matches_workspace_decode(tpa, name, lengths):
    wl = I.custom("no_alloc", I.WORKLOADS[name])
    dims, cache, q_a, q_b = _decode_inputs(tpa, wl, lengths)
    shape = (len(lengths), wl.n_heads, wl.head_dim)
    ref = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    tpa.tpa_decode(dims, q_a, q_b, cache, lengths, ref, tpa.alloc_workspace(dims, lengths))
    for _ in range(2):                       # two calls in a row share the scratch
        out = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        tpa.tpa_decode_static(dims, q_a, q_b, cache, lengths, out)
        torch.cuda.synchronize()
        assert tpa.tpa_get_device_error() == 0
        assert rel_err(out, ref) < TOL["bf16"]
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_static_scratch_decode_rejects_more_than_its_array(tpa):
    # 1024 sequences x 32 heads x (128 + 2) fp32 partials need 17 MB > 16 MiB
    dims = tpa.Dims(0, 32, 128, 0, 2, 2)
    lengths = [128] * 1024
    assert tpa.tpa_decode_workspace_bytes(dims, lengths) > tpa.TPA_DECODE_STATIC_SCRATCH_BYTES
    fake = 0x10000          # never dereferenced: the size check comes first
    c = tpa.tpa_cache(fake, fake, fake, fake, fake, 1024, 128)
    st = tpa._lib.tpa_decode_static(ctypes.byref(dims.c()), None, fake, ctypes.byref(c),
                                    tpa._ints(lengths), 1024, fake, None)
    assert st == 5          # TPA_ERR_WORKSPACE
