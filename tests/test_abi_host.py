"""Host-only checks of the C ABI: the library loads, exports every symbol tpa.h
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import json
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tpa.h")


@pytest.fixture(scope="module")
def bnd():
    from tensor_product_attention_b200 import build
    build.build()
    from tensor_product_attention_b200 import binding
    return binding


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tpa_[a-z_]+)\s*\(", text)))


def test_header_declares_what_binding_wraps(bnd):
    assert declared_functions() == sorted(bnd.EXPORTS)


def test_library_exports_every_declared_symbol(bnd):
    lib = ctypes.CDLL(bnd.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings(bnd):
    assert bnd.tpa_abi_version() == 2
    assert "sm_100a" in bnd.tpa_build_info()
    for code in range(7):
        assert bnd._lib.tpa_status_string(code)


def test_cache_bytes_per_token_matches_golden(bnd):
    gold = json.load(open(os.path.join(ROOT, "tests", "golden", "cache_bytes_per_token.json")))
    for row in gold["rows"]:
        dt = bnd.F32 if row["elem_bytes"] == 4 else bnd.BF16
        dims = bnd.Dims(64, row["n_heads"], row["head_dim"], 2, row["rank_k"], row["rank_v"], dt)
        assert bnd.tpa_cache_bytes_per_token(dims) == row["bytes_per_token"]
    assert bnd.tpa_cache_bytes_per_token(bnd.Dims(64, 4, 15, 2, 1, 1)) == 0   # odd head_dim


def _call(bnd, name, *args):
    return getattr(bnd._lib, name)(*args)


def test_host_validation_rejects_bad_arguments(bnd):
    d = bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32).c()
    by = ctypes.byref
    fake = 0x10000                       # aligned, never dereferenced: validation fails first
    f = bnd.tpa_factors(fake, fake, fake, fake, fake, fake)
    c = bnd.tpa_cache(fake, fake, fake, fake, fake, 2, 8)
    sp = bnd._ints([0, 0])
    # null pointers
    assert _call(bnd, "tpa_project", by(d), None, fake, 2, 4, sp, fake, 8, by(f), None) == 1
    assert _call(bnd, "tpa_prefill", by(d), None, by(c), 2, 4, sp, fake, None) == 1
    assert _call(bnd, "tpa_decode", by(d), fake, None, by(c), bnd._ints([1, 1]), 2, fake, fake, 1 << 20, None) == 1
    # misaligned pointer
    assert _call(bnd, "tpa_project", by(d), fake + 2, fake, 2, 4, sp, fake, 8, by(f), None) == 1
    # positions past the RoPE table / the cache
    assert _call(bnd, "tpa_project", by(d), fake, fake, 2, 4, bnd._ints([0, 5]), fake, 8, by(f), None) == 3
    assert _call(bnd, "tpa_cache_append", by(d), by(c), by(f), 2, 4, bnd._ints([0, 5]), None) == 3
    assert _call(bnd, "tpa_prefill", by(d), by(f), by(c), 2, 4, bnd._ints([5, 0]), fake, None) == 3
    assert _call(bnd, "tpa_decode", by(d), fake, fake, by(c), bnd._ints([9, 1]), 2, fake, fake, 1 << 20, None) == 3
    # batch larger than the cache, zero-length decode, negative start
    assert _call(bnd, "tpa_cache_append", by(d), by(c), by(f), 3, 1, bnd._ints([0, 0, 0]), None) == 1
    assert _call(bnd, "tpa_decode", by(d), fake, fake, by(c), bnd._ints([0, 1]), 2, fake, fake, 1 << 20, None) == 1
    assert _call(bnd, "tpa_cache_append", by(d), by(c), by(f), 2, 1, bnd._ints([-1, 0]), None) == 1
    # workspace too small
    need = bnd.tpa_decode_workspace_bytes(bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32), [3, 5])
    assert need > 0
    assert _call(bnd, "tpa_decode", by(d), fake, fake, by(c), bnd._ints([3, 5]), 2, fake, fake, need - 4, None) == 5
    # bad dims: odd head_dim, zero rank, factorised-query call with rank_q = 0
    bad = bnd.Dims(64, 4, 15, 2, 1, 1, bnd.F32).c()
    assert _call(bnd, "tpa_cache_append", by(bad), by(c), by(f), 2, 1, sp, None) == 1
    # TPA-KVonly takes its query from b_q (a_q may be NULL); a missing b_q is invalid
    kvonly = bnd.Dims(64, 4, 16, 0, 1, 1, bnd.F32).c()
    no_q = bnd.tpa_factors(None, None, fake, fake, fake, fake)
    assert _call(bnd, "tpa_prefill", by(kvonly), by(no_q), by(c), 2, 1, sp, fake, None) == 1
    assert _call(bnd, "tpa_project", by(kvonly), fake, fake, 2, 4, sp, fake, 8, by(no_q), None) == 1
    assert _call(bnd, "tpa_prefill", by(kvonly), by(f), by(c), 2, 1, bnd._ints([8, 0]), fake, None) == 3
    negq = bnd.Dims(64, 4, 16, -1, 1, 1, bnd.F32).c()
    assert _call(bnd, "tpa_prefill", by(negq), by(f), by(c), 2, 1, sp, fake, None) == 1
    assert _call(bnd, "tpa_rope_table", by(d), 0.5, 8, fake, None) == 1


def test_static_decode_returns_the_same_status_as_decode(bnd):
    """tpa_decode_static checks its arguments as tpa_decode does, before any CUDA call,
    so an unsupported shape, a null query or a length past the cache gives the same
    code from both (and the scratch array is never looked up)."""
    by = ctypes.byref
    fake = 0x10000
    c = bnd.tpa_cache(fake, fake, fake, fake, fake, 2, 8)
    cases = [
        (bnd.Dims(64, 5000, 16, 2, 1, 1, bnd.F32), fake, [1, 1], 2),     # h > 4096: unsupported
        (bnd.Dims(64, 4, 16, 2, 300, 1, bnd.F32), fake, [1, 1], 2),      # rank > 256: unsupported
        (bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32), None, [1, 1], 1),        # null query: invalid
        (bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32), fake, [9, 1], 3),        # past the capacity
        (bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32), fake, [0, 1], 1),        # empty context
    ]
    for dims, q_b, lengths, want in cases:
        d = dims.c()
        got_ws = _call(bnd, "tpa_decode", by(d), fake, q_b, by(c), bnd._ints(lengths), 2, fake, fake,
                       1 << 20, None)
        got_static = _call(bnd, "tpa_decode_static", by(d), fake, q_b, by(c), bnd._ints(lengths), 2,
                           fake, None)
        assert got_ws == got_static == want, (dims, got_ws, got_static)


def test_kernel_family_names_the_path_each_shape_takes(bnd):
    # the configured bf16 layers take the tensor-core kernels for every call
    for h, d, rq in ((16, 64, 6), (16, 128, 6), (32, 128, 0)):
        dims = bnd.Dims(1024, h, d, rq, 2, 2, bnd.BF16)
        for call in (bnd.CALL_PROJECT, bnd.CALL_PREFILL, bnd.CALL_DECODE):
            assert bnd.tpa_kernel_family(dims, call) == "tensor_core", (h, d, rq, call)
    # fp32 layers and bf16 shapes outside the tensor-core limits use the CUDA cores
    f32 = bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32)
    for call in (bnd.CALL_PROJECT, bnd.CALL_PREFILL, bnd.CALL_DECODE):
        assert bnd.tpa_kernel_family(f32, call) == "cuda_core"
    assert bnd.tpa_kernel_family(bnd.Dims(64, 8, 32, 2, 3, 3, bnd.BF16), bnd.CALL_DECODE) == "cuda_core"
    # invalid dims or an unknown call
    assert bnd.tpa_kernel_family(bnd.Dims(64, 4, 15, 2, 1, 1, bnd.F32), bnd.CALL_DECODE) == "none"
    assert bnd.tpa_kernel_family(f32, 7) == "none"


def test_decode_step_host_validation(bnd):
    d = bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32).c()
    by = ctypes.byref
    fake = 0x10000
    c = bnd.tpa_cache(fake, fake, fake, fake, fake, 2, 8)
    need = bnd.tpa_decode_step_workspace_bytes(bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32), [3, 5])
    assert need > bnd.tpa_decode_workspace_bytes(bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32), [4, 6])
    step = lambda *a: _call(bnd, "tpa_decode_step", *a)
    ok = (fake, fake, fake, 16, by(c), bnd._ints([3, 5]), 2, fake, fake, need, None)
    # null input, misaligned workspace, workspace too small
    assert step(by(d), None, *ok[1:]) == 1
    assert step(by(d), *ok[:8], fake + 16, need, None) == 1
    assert step(by(d), *ok[:9], need - 4, None) == 5
    # no room in the cache (capacity 8), position past the RoPE table (max_pos 6)
    assert step(by(d), fake, fake, fake, 16, by(c), bnd._ints([3, 8]), 2, fake, fake, need, None) == 3
    assert step(by(d), fake, fake, fake, 6, by(c), bnd._ints([3, 6]), 2, fake, fake, need, None) == 3
    # negative length, batch larger than the cache
    assert step(by(d), fake, fake, fake, 16, by(c), bnd._ints([-1, 5]), 2, fake, fake, need, None) == 1
    assert step(by(d), fake, fake, fake, 16, by(c), bnd._ints([1, 1, 1]), 3, fake, fake, need, None) == 1
    assert bnd.tpa_decode_step_workspace_bytes(bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32), [-1]) == 0


def test_output_project_host_validation(bnd):
    d = bnd.Dims(64, 4, 16, 2, 1, 1, bnd.F32).c()
    by = ctypes.byref
    fake = 0x10000
    op = lambda *a: _call(bnd, "tpa_output_project", *a)
    assert op(by(d), None, fake, 8, fake, None) == 1
    assert op(by(d), fake, fake, 0, fake, None) == 1
    assert op(by(d), fake, fake + 4, 8, fake, None) == 1
    no_model = bnd.Dims(0, 4, 16, 2, 1, 1, bnd.F32).c()
    assert op(by(no_model), fake, fake, 8, fake, None) == 1


def test_workspace_size_formula(bnd):
    dims = bnd.Dims(0, 16, 128, 6, 2, 2)
    lengths = [32768] * 64
    n = bnd.tpa_decode_workspace_bytes(dims, lengths)
    # one (m, l) pair and one d_h-vector of fp32 per (part, head); every sequence has at
    # least one part, and a persistent grid of G CTAs adds at most G more
    per_part = 16 * (128 + 2) * 4
    assert n % per_part == 0
    assert 64 * per_part <= n <= (64 + 1024) * per_part


def test_shared_basis_host_validation(bnd):
    # shared basis: only A_K, A_V per token, (R_K + R_V) h elements
    sh = bnd.Dims(64, 16, 128, 6, 2, 2, bnd.BF16, 1)
    assert bnd.tpa_cache_bytes_per_token(sh) == (2 + 2) * 16 * 2
    assert bnd.tpa_cache_bytes_per_token(bnd.Dims(64, 16, 128, 6, 2, 2, bnd.BF16, 2)) == 0
    assert sh.n_proj == 16 * (6 + 2 + 2) + 6 * 128
    by = ctypes.byref
    fake = 0x10000                      # aligned, never dereferenced: validation fails first
    d = sh.c()
    tables = bnd._lib.tpa_shared_basis_tables
    ctx = bnd.Dims(64, 16, 128, 6, 2, 2, bnd.BF16, 0).c()
    assert tables(by(ctx), fake, fake, fake, 64, 64, fake, fake, None) == 1      # not shared
    assert tables(by(d), None, fake, fake, 64, 64, fake, fake, None) == 1
    assert tables(by(d), fake, fake, fake, 64, 64, fake + 8, fake, None) == 1   # misaligned
    assert tables(by(d), fake, fake, fake, 64, 0, fake, fake, None) == 1        # no capacity
    assert tables(by(d), fake, fake, fake, 64, 65, fake, fake, None) == 3       # past RoPE table
    # projection: shared layers need no B_K / B_V outputs, but still the A factors
    f = bnd.tpa_factors(fake, fake, None, None, None, None)
    assert bnd._lib.tpa_project(by(d), fake, fake, 1, 1, bnd._ints([0]), fake, 8, by(f), None) == 1
    # append: A factors are still required
    cache = bnd.tpa_cache(fake, fake, fake, fake, fake, 1, 8)
    assert bnd._lib.tpa_cache_append(by(d), by(cache), by(f), 1, 1, bnd._ints([0]), None) == 1
    assert bnd._lib.tpa_cache_append(by(d), by(cache), by(f), 1, 1, bnd._ints([8]), None) == 1


def test_bounds_checked_library_has_the_same_abi(bnd):
    """libtpa_debug.so (TPA_DEBUG_BOUNDS) exports every declared symbol and says so."""
    lib = ctypes.CDLL(bnd.DEBUG_LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    with bnd.use_library(bnd.DEBUG_LIB_PATH):
        assert "bounds-checked" in bnd.tpa_build_info()
        assert bnd.tpa_abi_version() == 2
    assert "bounds-checked" not in bnd.tpa_build_info()


def _parts_by_overlap(unit_tiles, members, sms=148):
    """Independent count of the tensor-core decode's parts: a persistent grid of
    min(sms, N) CTAs splits the N concatenated unit tiles evenly (CTA c takes
    [c*N/G, (c+1)*N/G)); every (CTA, unit) overlap gives each member sequence a part."""
    n = sum(unit_tiles)
    G = min(sms, n)
    starts = np.cumsum([0] + list(unit_tiles))
    parts = 0
    for c in range(G):
        lo, hi = c * n // G, (c + 1) * n // G
        for u in range(len(unit_tiles)):
            if starts[u] < hi and starts[u + 1] > lo:
                parts += members[u]
    return parts


@pytest.mark.parametrize("lengths", [[32768] * 64, [1, 5, 30], [12000, 9001, 1, 14501], [700] * 29 + [33],
                                     [3001], [5, 2049, 3], [65536, 1, 131072, 7, 2]])
def test_decode_plan_parts_match_an_independent_count(bnd, lengths):
    # The workspace holds one (m, l, o) state per (part, head); the part count of the
    # plan built inside the library must match the overlap count above.  This runs on
    # the host only (without a GPU the library assumes 148 SMs, as on a B200).
    h, d, kt = 16, 128, 64
    per_part = h * (2 + d) * 4
    tiles = [(L + kt - 1) // kt for L in lengths]
    ctx = bnd.Dims(0, h, d, 6, 2, 2, bnd.BF16, 0)
    assert bnd.tpa_decode_workspace_bytes(ctx, lengths) == _parts_by_overlap(tiles, [1] * len(tiles)) * per_part
    # shared basis at h 16: units of two sequences sharing each key tile
    U = (len(lengths) + 1) // 2
    unit_tiles = [max(tiles[2 * u], tiles[2 * u + 1] if 2 * u + 1 < len(tiles) else 0) for u in range(U)]
    members = [min(2, len(lengths) - 2 * u) for u in range(U)]
    sb = bnd.Dims(0, h, d, 6, 2, 2, bnd.BF16, 1)
    assert bnd.tpa_decode_workspace_bytes(sb, lengths) == _parts_by_overlap(unit_tiles, members) * per_part


def test_product_and_oracle_stay_apart():
    """The product (the package, its CUDA sources and binding) never imports or reads the
    oracle, and the oracle never imports the product; bench.py and smoke() import the
    oracle only inside the functions that time or check it."""
    import ast
    pkg = os.path.join(ROOT, "tensor_product_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in text.lower() or f == "inputs.py", f
    # inputs.py may name the oracle in prose only (it serves both sides)
    tree = ast.parse(open(os.path.join(pkg, "inputs.py"), encoding="utf-8").read())
    for node in ast.walk(tree):
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] + ([node.module] if isinstance(node, ast.ImportFrom) else [])
            assert not any(n and n.split(".")[0] == "oracle" for n in names)
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith(".py"):
            tree = ast.parse(open(os.path.join(ROOT, "oracle", f), encoding="utf-8").read())
            for node in ast.walk(tree):
                if isinstance(node, (ast.Import, ast.ImportFrom)):
                    names = [a.name for a in node.names] + ([node.module] if isinstance(node, ast.ImportFrom) else [])
                    assert not any(n and n.split(".")[0] == "tensor_product_attention_b200" for n in names), f
    for f in ("bench.py", "__graft_entry__.py"):
        tree = ast.parse(open(os.path.join(ROOT, f), encoding="utf-8").read())
        for node in tree.body:                       # module level: no oracle import
            if isinstance(node, (ast.Import, ast.ImportFrom)):
                names = [a.name for a in node.names] + ([node.module] if isinstance(node, ast.ImportFrom) else [])
                assert not any(n and n.split(".")[0] == "oracle" for n in names), f
