"""Python binding of libtpa.so (include/tpa.h), with the C call names.

Argument marshalling only: every function turns torch tensors into device pointers,
host lists into int32 arrays and the current torch stream into a cudaStream_t, calls
the C entry point of the same name and raises ``TPAError`` on a non-zero status.
All arithmetic runs in the library's CUDA kernels.  Importing this module fails loudly
(``ImportError``) when the library has not been built; there is no other code path.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtpa.so")
# The bounds-checked build of the same sources (python -m tensor_product_attention_b200.build
# --debug): a bad index records TPA_DEVERR_BOUNDS (2) in the device error word.
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtpa_debug.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: run `python -m tensor_product_attention_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

F32, BF16 = 0, 1
STATUS = {0: "TPA_OK", 1: "TPA_ERR_INVALID", 2: "TPA_ERR_UNSUPPORTED", 3: "TPA_ERR_CAPACITY",
          4: "TPA_ERR_CUDA", 5: "TPA_ERR_WORKSPACE", 6: "TPA_ERR_DEVICE"}
TPA_MAX_BATCH = 1024

# Every symbol include/tpa.h declares (checked by tests/test_abi_host.py).
EXPORTS = ("tpa_abi_version", "tpa_build_info", "tpa_status_string", "tpa_cache_bytes_per_token",
           "tpa_rope_table", "tpa_project", "tpa_cache_append", "tpa_prefill", "tpa_decode",
           "tpa_decode_workspace_bytes", "tpa_decode_static", "tpa_decode_step",
           "tpa_decode_step_workspace_bytes", "tpa_output_project", "tpa_shared_basis_tables",
           "tpa_get_device_error", "tpa_set_wait_limit", "tpa_kernel_family")
TPA_DECODE_STATIC_SCRATCH_BYTES = 16 << 20


class tpa_dims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("rank_q", ctypes.c_int32),
                ("rank_k", ctypes.c_int32), ("rank_v", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("shared_basis", ctypes.c_int32)]


class tpa_factors(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("a_q", "b_q", "a_k", "b_k", "a_v", "b_v")]


class tpa_cache(ctypes.Structure):
    _fields_ = [("a_k", ctypes.c_void_p), ("a_v", ctypes.c_void_p), ("b_k", ctypes.c_void_p),
                ("b_v", ctypes.c_void_p), ("lengths", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("capacity", ctypes.c_int32)]


_P = ctypes.POINTER
_i32p = _P(ctypes.c_int32)
_sig = {
    "tpa_abi_version": (ctypes.c_int32, []),
    "tpa_build_info": (ctypes.c_char_p, []),
    "tpa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tpa_cache_bytes_per_token": (ctypes.c_size_t, [_P(tpa_dims)]),
    "tpa_rope_table": (ctypes.c_int, [_P(tpa_dims), ctypes.c_double, ctypes.c_int32,
                                      ctypes.c_void_p, ctypes.c_void_p]),
    "tpa_project": (ctypes.c_int, [_P(tpa_dims), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                   ctypes.c_int32, _i32p, ctypes.c_void_p, ctypes.c_int32,
                                   _P(tpa_factors), ctypes.c_void_p]),
    "tpa_cache_append": (ctypes.c_int, [_P(tpa_dims), _P(tpa_cache), _P(tpa_factors),
                                        ctypes.c_int32, ctypes.c_int32, _i32p, ctypes.c_void_p]),
    "tpa_prefill": (ctypes.c_int, [_P(tpa_dims), _P(tpa_factors), _P(tpa_cache), ctypes.c_int32,
                                   ctypes.c_int32, _i32p, ctypes.c_void_p, ctypes.c_void_p]),
    "tpa_decode": (ctypes.c_int, [_P(tpa_dims), ctypes.c_void_p, ctypes.c_void_p, _P(tpa_cache),
                                  _i32p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_size_t, ctypes.c_void_p]),
    "tpa_decode_workspace_bytes": (ctypes.c_size_t, [_P(tpa_dims), _i32p, ctypes.c_int32]),
    "tpa_decode_static": (ctypes.c_int, [_P(tpa_dims), ctypes.c_void_p, ctypes.c_void_p, _P(tpa_cache),
                                         _i32p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "tpa_decode_step": (ctypes.c_int, [_P(tpa_dims), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_int32, _P(tpa_cache), _i32p, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tpa_decode_step_workspace_bytes": (ctypes.c_size_t, [_P(tpa_dims), _i32p, ctypes.c_int32]),
    "tpa_output_project": (ctypes.c_int, [_P(tpa_dims), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                          ctypes.c_void_p, ctypes.c_void_p]),
    "tpa_shared_basis_tables": (ctypes.c_int, [_P(tpa_dims), ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "tpa_get_device_error": (ctypes.c_int, [ctypes.c_void_p, _i32p]),
    "tpa_set_wait_limit": (None, [ctypes.c_uint32]),
    "tpa_kernel_family": (ctypes.c_int32, [_P(tpa_dims), ctypes.c_int32]),
}
def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    for name, (res, args) in _sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_declare(_lib)


@contextlib.contextmanager
def use_library(path: str):
    """Route every call of this module to the library at ``path`` (same ABI) for the
    duration of the block, e.g. DEBUG_LIB_PATH.  Not thread-safe."""
    global _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing")
    prev, _lib = _lib, _declare(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = prev


class TPAError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        msg = _lib.tpa_status_string(status).decode()
        super().__init__(f"{call}: {STATUS.get(status, status)} ({msg})")


def _check(call: str, status: int) -> None:
    if status != 0:
        raise TPAError(call, status)


# ----------------------------------------------------------------- value types

@dataclass(frozen=True)
class Dims:
    d_model: int
    n_heads: int
    head_dim: int
    rank_q: int
    rank_k: int
    rank_v: int
    dtype: int = BF16
    shared_basis: int = 0      # 1: B_K, B_V shared across tokens (per-position tables)

    def c(self) -> tpa_dims:
        return tpa_dims(self.d_model, self.n_heads, self.head_dim, self.rank_q, self.rank_k,
                        self.rank_v, self.dtype, int(self.shared_basis))

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == BF16 else torch.float32

    @property
    def n_proj(self) -> int:
        """Rows of the stacked projection weight w_cat (tpa_project)."""
        h, d = self.n_heads, self.head_dim
        q_rows = self.rank_q if self.rank_q > 0 else h
        kv_b = 0 if self.shared_basis else (self.rank_k + self.rank_v) * d
        return h * (self.rank_q + self.rank_k + self.rank_v) + q_rows * d + kv_b


@dataclass
class Factors:
    """Device tensors of the six factors for T tokens (any may be None when unused)."""
    a_q: torch.Tensor | None = None
    b_q: torch.Tensor | None = None
    a_k: torch.Tensor | None = None
    b_k: torch.Tensor | None = None
    a_v: torch.Tensor | None = None
    b_v: torch.Tensor | None = None

    def c(self) -> tpa_factors:
        p = lambda t: None if t is None else t.data_ptr()
        return tpa_factors(p(self.a_q), p(self.b_q), p(self.a_k), p(self.b_k), p(self.a_v), p(self.b_v))


@dataclass
class Cache:
    """Device tensors of the factor cache (caller-owned, see tpa.h)."""
    a_k: torch.Tensor
    a_v: torch.Tensor
    b_k: torch.Tensor
    b_v: torch.Tensor
    lengths: torch.Tensor

    @property
    def batch(self) -> int:
        return self.a_k.shape[0]

    @property
    def capacity(self) -> int:
        return self.a_k.shape[1]

    def c(self) -> tpa_cache:
        return tpa_cache(self.a_k.data_ptr(), self.a_v.data_ptr(), self.b_k.data_ptr(),
                         self.b_v.data_ptr(), self.lengths.data_ptr(), self.batch, self.capacity)


def alloc_factors(dims: Dims, T: int, device="cuda", queries=True, kv=True) -> Factors:
    h, d, dt = dims.n_heads, dims.head_dim, dims.torch_dtype
    f = Factors()
    if queries and dims.rank_q > 0:
        f.a_q = torch.empty((T, h, dims.rank_q), dtype=dt, device=device)
        f.b_q = torch.empty((T, dims.rank_q, d), dtype=dt, device=device)
    elif queries:
        # TPA-KVonly: the plain per-head query sits in the b_q slot, [T][h][d_h]
        f.b_q = torch.empty((T, h, d), dtype=dt, device=device)
    if kv:
        f.a_k = torch.empty((T, h, dims.rank_k), dtype=dt, device=device)
        f.a_v = torch.empty((T, h, dims.rank_v), dtype=dt, device=device)
        if not dims.shared_basis:
            f.b_k = torch.empty((T, dims.rank_k, d), dtype=dt, device=device)
            f.b_v = torch.empty((T, dims.rank_v, d), dtype=dt, device=device)
    return f


def alloc_cache(dims: Dims, batch: int, capacity: int, device="cuda", fill=None) -> Cache:
    """Cache tensors; with a shared basis b_k, b_v are the per-position tables
    [capacity][R][d_h] (fill them with tpa_shared_basis_tables)."""
    h, d, dt = dims.n_heads, dims.head_dim, dims.torch_dtype
    mk = (lambda s: torch.full(s, fill, dtype=dt, device=device)) if fill is not None else \
        (lambda s: torch.empty(s, dtype=dt, device=device))
    lead = (capacity,) if dims.shared_basis else (batch, capacity)
    return Cache(mk((batch, capacity, h, dims.rank_k)), mk((batch, capacity, h, dims.rank_v)),
                 mk(lead + (dims.rank_k, d)), mk(lead + (dims.rank_v, d)),
                 torch.zeros(batch, dtype=torch.int32, device=device))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ints(vals) -> ctypes.Array:
    vals = [int(v) for v in vals]
    return (ctypes.c_int32 * max(1, len(vals)))(*vals)


def _ptr(t):
    return None if t is None else t.data_ptr()


# ----------------------------------------------------------------- the calls

def tpa_abi_version() -> int:
    return _lib.tpa_abi_version()


def tpa_build_info() -> str:
    return _lib.tpa_build_info().decode()


def tpa_cache_bytes_per_token(dims: Dims) -> int:
    return _lib.tpa_cache_bytes_per_token(ctypes.byref(dims.c()))


def tpa_rope_table(dims: Dims, base: float, max_pos: int, cs: torch.Tensor, stream=None) -> None:
    _check("tpa_rope_table", _lib.tpa_rope_table(ctypes.byref(dims.c()), float(base), int(max_pos),
                                                 _ptr(cs), _stream(stream)))


def tpa_project(dims: Dims, x, w_cat, batch: int, seqlen: int, start_pos, rope_cs, max_pos: int,
                out: Factors, stream=None) -> None:
    _check("tpa_project", _lib.tpa_project(ctypes.byref(dims.c()), _ptr(x), _ptr(w_cat), int(batch),
                                           int(seqlen), _ints(start_pos), _ptr(rope_cs), int(max_pos),
                                           ctypes.byref(out.c()), _stream(stream)))


def tpa_cache_append(dims: Dims, cache: Cache, kv: Factors, batch: int, n_tokens: int, start_pos,
                     stream=None) -> None:
    _check("tpa_cache_append", _lib.tpa_cache_append(ctypes.byref(dims.c()), ctypes.byref(cache.c()),
                                                     ctypes.byref(kv.c()), int(batch), int(n_tokens),
                                                     _ints(start_pos), _stream(stream)))


def tpa_shared_basis_tables(dims: Dims, basis_k, basis_v, rope_cs, max_pos: int, table_k, table_v,
                            stream=None) -> None:
    """Shared basis: table_k[p] = basis_k rotated at position p, table_v[p] = basis_v,
    for p < table_k.shape[0] (the cache capacity)."""
    _check("tpa_shared_basis_tables", _lib.tpa_shared_basis_tables(
        ctypes.byref(dims.c()), _ptr(basis_k), _ptr(basis_v), _ptr(rope_cs), int(max_pos),
        int(table_k.shape[0]), _ptr(table_k), _ptr(table_v), _stream(stream)))


def tpa_prefill(dims: Dims, q: Factors, cache: Cache, batch: int, seqlen: int, start_pos, out,
                stream=None) -> None:
    _check("tpa_prefill", _lib.tpa_prefill(ctypes.byref(dims.c()), ctypes.byref(q.c()),
                                           ctypes.byref(cache.c()), int(batch), int(seqlen),
                                           _ints(start_pos), _ptr(out), _stream(stream)))


def tpa_decode_workspace_bytes(dims: Dims, lengths) -> int:
    lengths = list(lengths)
    return _lib.tpa_decode_workspace_bytes(ctypes.byref(dims.c()), _ints(lengths), len(lengths))


def tpa_decode(dims: Dims, q_a, q_b, cache: Cache, lengths, out, workspace, stream=None) -> None:
    lengths = list(lengths)
    _check("tpa_decode", _lib.tpa_decode(ctypes.byref(dims.c()), _ptr(q_a), _ptr(q_b),
                                         ctypes.byref(cache.c()), _ints(lengths), len(lengths),
                                         _ptr(out), _ptr(workspace),
                                         0 if workspace is None else workspace.numel() * workspace.element_size(),
                                         _stream(stream)))


def tpa_decode_static(dims: Dims, q_a, q_b, cache: Cache, lengths, out, stream=None) -> None:
    """tpa_decode without a workspace argument, for callers that cannot allocate device
    memory: the scratch is the library's own fixed device array
    (TPA_DECODE_STATIC_SCRATCH_BYTES per GPU).  Calls that overlap on the GPU race."""
    lengths = list(lengths)
    _check("tpa_decode_static", _lib.tpa_decode_static(ctypes.byref(dims.c()), _ptr(q_a), _ptr(q_b),
                                                       ctypes.byref(cache.c()), _ints(lengths), len(lengths),
                                                       _ptr(out), _stream(stream)))


def tpa_decode_step_workspace_bytes(dims: Dims, lengths) -> int:
    lengths = list(lengths)
    return _lib.tpa_decode_step_workspace_bytes(ctypes.byref(dims.c()), _ints(lengths), len(lengths))


def tpa_decode_step(dims: Dims, x, w_cat, rope_cs, max_pos: int, cache: Cache, lengths, out,
                    workspace, stream=None) -> None:
    """Project the new token of every sequence, append its K/V factors at lengths[b]
    (advancing cache.lengths) and decode it; ``lengths`` are the pre-step lengths."""
    lengths = list(lengths)
    _check("tpa_decode_step", _lib.tpa_decode_step(
        ctypes.byref(dims.c()), _ptr(x), _ptr(w_cat), _ptr(rope_cs), int(max_pos),
        ctypes.byref(cache.c()), _ints(lengths), len(lengths), _ptr(out), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))


def alloc_step_workspace(dims: Dims, lengths, device="cuda") -> torch.Tensor:
    n = tpa_decode_step_workspace_bytes(dims, lengths)
    if n == 0:
        raise ValueError("invalid decode-step arguments")
    return torch.empty(n, dtype=torch.uint8, device=device)


def tpa_output_project(dims: Dims, attn, w_o, out, stream=None) -> None:
    """out [T][d_model] = attn [T][h][d_h] (flattened per token) @ w_o[d_model][h*d_h]^T."""
    T = attn.shape[0]
    _check("tpa_output_project", _lib.tpa_output_project(ctypes.byref(dims.c()), _ptr(attn), _ptr(w_o),
                                                         int(T), _ptr(out), _stream(stream)))


def tpa_get_device_error(stream=None) -> int:
    code = ctypes.c_int32(0)
    st = _lib.tpa_get_device_error(_stream(stream), ctypes.byref(code))
    if st not in (0, 6):
        _check("tpa_get_device_error", st)
    return code.value


def tpa_set_wait_limit(polls: int) -> None:
    _lib.tpa_set_wait_limit(int(polls))


CALL_PROJECT, CALL_PREFILL, CALL_DECODE = 0, 1, 2
FAMILY = {-1: "none", 0: "cuda_core", 1: "tensor_core"}


def tpa_kernel_family(dims: Dims, call: int) -> str:
    """'tensor_core', 'cuda_core' or 'none': the kernel family the call takes."""
    return FAMILY[_lib.tpa_kernel_family(ctypes.byref(dims.c()), int(call))]


def alloc_workspace(dims: Dims, lengths, device="cuda") -> torch.Tensor:
    n = tpa_decode_workspace_bytes(dims, lengths)
    if n == 0:
        raise ValueError("invalid decode arguments")
    return torch.empty(n, dtype=torch.uint8, device=device)
