"""Python binding of libtq (TurboQuant KV-cache quantization + packed decode
attention for B200).  Argument marshalling only: every step of the path runs
in the CUDA kernels of libtq.so; PyTorch supplies device memory and streams.

The functions keep the names of the C ABI in include/tq.h.  There is no CPU
fallback: importing this package fails loudly when libtq.so is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtq.so")

TQ_F32, TQ_BF16 = 0, 1
TQ_MODE_MSE, TQ_MODE_PROD = 0, 1
TQ_ROT_HAAR, TQ_ROT_HADAMARD = 0, 1
TQ_K, TQ_V = 0, 1
STATUS_NAMES = {0: "TQ_OK", 1: "TQ_ERR_ARG", 2: "TQ_ERR_UNSUPPORTED", 3: "TQ_ERR_ALIGN",
                4: "TQ_ERR_CAPACITY", 5: "TQ_ERR_CUDA", 6: "TQ_ERR_NOMEM"}


class TqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtq.so is not built ({LIB_PATH}); run python online_vector_quantization_b200/build.py")
_lib = ctypes.CDLL(LIB_PATH)

c_int, c_void_p, c_size_t, c_float, c_uint64, c_int64 = (
    ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float, ctypes.c_uint64, ctypes.c_int64)
_dp = ctypes.POINTER(ctypes.c_double)


class TqConfig(ctypes.Structure):
    _fields_ = [("d", c_int), ("bits_k", c_int), ("bits_v", c_int), ("mode_k", c_int),
                ("mode_v", c_int), ("mixed_k", c_int), ("mixed_v", c_int), ("m", c_int),
                ("seed", c_uint64), ("rotation", c_int)]


class TqPacked(ctypes.Structure):
    _fields_ = [("codes", c_void_p), ("norms", c_void_p), ("qjl", c_void_p), ("res_norms", c_void_p)]


class TqCache(ctypes.Structure):
    _fields_ = [("n_seq", c_int), ("n_kv_heads", c_int), ("capacity", c_int), ("n_sink", c_int),
                ("k_codes", c_void_p), ("k_norms", c_void_p), ("k_qjl", c_void_p), ("k_res_norms", c_void_p),
                ("v_codes", c_void_p), ("v_norms", c_void_p), ("v_qjl", c_void_p), ("v_res_norms", c_void_p),
                ("k_sink", c_void_p), ("v_sink", c_void_p), ("lens", c_void_p), ("status", c_void_p)]


class TqAttnFlags(ctypes.Structure):
    _fields_ = [("sparse_v_threshold", c_float), ("reserved", c_int), ("sparse_v_stats", c_void_p)]


_SIGS = {
    "tq_codebook": (c_int, [c_int, c_int, _dp, _dp]),
    "tq_rotation": (c_int, [c_uint64, c_int, _dp]),
    "tq_hadamard_rotation": (c_int, [c_uint64, c_int, _dp]),
    "tq_qjl_matrix": (c_int, [c_uint64, c_int, c_int, _dp]),
    "tq_params_create": (c_int, [ctypes.POINTER(TqConfig), ctypes.POINTER(c_void_p)]),
    "tq_params_destroy": (None, [c_void_p]),
    "tq_params_status": (c_int, [c_void_p, ctypes.POINTER(ctypes.c_int32), c_int]),
    "tq_row_bytes": (c_int, [c_void_p, c_int, ctypes.POINTER(c_int), ctypes.POINTER(c_int)]),
    "tq_quantize": (c_int, [c_void_p, c_void_p, c_int, c_int64, c_int, ctypes.POINTER(TqPacked), c_void_p]),
    "tq_dequantize": (c_int, [c_void_p, ctypes.POINTER(TqPacked), c_int64, c_int, c_void_p, c_void_p]),
    "tq_cache_bytes": (c_size_t, [c_void_p, c_int, c_int, c_int, c_int]),
    "tq_cache_bind": (c_int, [c_void_p, c_void_p, c_size_t, c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                              ctypes.POINTER(TqCache)]),
    "tq_append": (c_int, [c_void_p, ctypes.POINTER(TqCache), c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                          c_void_p]),
    "tq_cache_write_rows": (c_int, [c_void_p, ctypes.POINTER(TqCache), c_int, c_int, c_int, c_int, c_int64,
                                    ctypes.POINTER(TqPacked), c_void_p]),
    "tq_cache_read_rows": (c_int, [c_void_p, ctypes.POINTER(TqCache), c_int, c_int, c_int, c_int, c_int64,
                                   ctypes.POINTER(TqPacked), c_void_p]),
    "tq_decode_workspace_bytes": (c_size_t, [c_void_p, c_int, c_int, c_int, c_int]),
    "tq_decode_workspace_init": (c_int, [c_void_p, c_size_t, c_void_p]),
    "tq_decode_attn": (c_int, [c_void_p, c_void_p, c_int, ctypes.POINTER(TqCache), c_int, c_int, c_int, c_void_p,
                               c_int, c_void_p, c_size_t, ctypes.POINTER(TqAttnFlags), c_void_p]),
    "tq_decode_attn_noalloc": (c_int, [c_void_p, c_void_p, c_int, ctypes.POINTER(TqCache), c_int, c_int, c_int,
                                       c_void_p, c_int, ctypes.POINTER(TqAttnFlags), c_void_p]),
    "tq_search_workspace_bytes": (c_size_t, []),
    "tq_search": (c_int, [c_void_p, c_int, ctypes.POINTER(TqPacked), c_int64, c_void_p, c_int, c_int, c_int,
                          c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "tq_last_error": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def _check(status: int):
    if status != 0:
        raise TqError(status, _lib.tq_last_error().decode())


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---- host tables -----------------------------------------------------------

def tq_codebook(d: int, bits: int):
    c = np.zeros(1 << bits)
    b = np.zeros((1 << bits) - 1)
    _check(_lib.tq_codebook(d, bits, c.ctypes.data_as(_dp), b.ctypes.data_as(_dp)))
    return c, b


def tq_rotation(seed: int, d: int) -> np.ndarray:
    out = np.zeros((d, d))
    _check(_lib.tq_rotation(seed, d, out.ctypes.data_as(_dp)))
    return out


def tq_hadamard_rotation(seed: int, d: int) -> np.ndarray:
    out = np.zeros((d, d))
    _check(_lib.tq_hadamard_rotation(seed, d, out.ctypes.data_as(_dp)))
    return out


def tq_qjl_matrix(seed: int, m: int, d: int) -> np.ndarray:
    out = np.zeros((m, d))
    _check(_lib.tq_qjl_matrix(seed, m, d, out.ctypes.data_as(_dp)))
    return out


# ---- parameters ------------------------------------------------------------

class Params:
    """Owner of a tq_params handle (device tables on the current device)."""

    def __init__(self, bits_k: int, bits_v: int, mode_k: int = TQ_MODE_MSE, mode_v: int = TQ_MODE_MSE,
                 mixed_k: int = 0, mixed_v: int = 0, seed: int = 0, d: int = 128, m: int = 128,
                 rotation: int = 0):
        self.config = TqConfig(d, bits_k, bits_v, mode_k, mode_v, mixed_k, mixed_v, m, seed, rotation)
        h = c_void_p()
        _check(_lib.tq_params_create(ctypes.byref(self.config), ctypes.byref(h)))
        self.handle = h.value
        self.d, self.m = d, m

    def status(self, clear: bool = False) -> int:
        """Error bits recorded by quantize kernels for these parameters (see tq.h)."""
        out = ctypes.c_int32()
        _check(_lib.tq_params_status(self.handle, ctypes.byref(out), int(clear)))
        return out.value

    def row_bytes(self, which: int):
        cb, qb = c_int(), c_int()
        _check(_lib.tq_row_bytes(self.handle, which, ctypes.byref(cb), ctypes.byref(qb)))
        return cb.value, qb.value

    def close(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.tq_params_destroy(self.handle)
        self.handle = None

    def __del__(self):
        self.close()


def tq_params_create(**kw) -> Params:
    return Params(**kw)


@dataclass
class Packed:
    """Device planes of n packed rows (torch tensors)."""
    codes: object
    norms: object
    qjl: object = None
    res_norms: object = None

    @staticmethod
    def empty(params: Params, n: int, which: int, device="cuda") -> "Packed":
        import torch
        cb, qb = params.row_bytes(which)
        return Packed(torch.zeros(n, cb, dtype=torch.uint8, device=device) if cb else None,
                      torch.zeros(n, dtype=torch.float32, device=device),
                      torch.zeros(n, qb, dtype=torch.uint8, device=device) if qb else None,
                      torch.zeros(n, dtype=torch.float32, device=device) if qb else None)

    def struct(self) -> TqPacked:
        return TqPacked(_ptr(self.codes), _ptr(self.norms), _ptr(self.qjl), _ptr(self.res_norms))


def tq_quantize(params: Params, x, which: int, out: Packed, stream=None):
    """x: (n, d) fp32/bf16 CUDA tensor, contiguous."""
    assert x.is_contiguous()
    st = out.struct()
    _check(_lib.tq_quantize(params.handle, _ptr(x), _dtype_code(x), x.shape[0], which, ctypes.byref(st),
                            _stream(stream)))


def tq_dequantize(params: Params, packed: Packed, n: int, which: int, out, stream=None):
    st = packed.struct()
    _check(_lib.tq_dequantize(params.handle, ctypes.byref(st), n, which, _ptr(out), _stream(stream)))


# ---- cache -----------------------------------------------------------------

class Cache:
    """A packed KV cache in one device buffer (planes carved by tq_cache_bind)."""

    def __init__(self, params: Params, n_seq: int, n_kv_heads: int, capacity: int, n_sink: int = 0,
                 device="cuda"):
        import torch
        nbytes = _lib.tq_cache_bytes(params.handle, n_seq, n_kv_heads, capacity, n_sink)
        if nbytes == 0:
            raise TqError(1, "tq_cache_bytes: bad cache sizes")
        self.buffer = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.lens = torch.zeros(n_seq, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.struct = TqCache()
        _check(_lib.tq_cache_bind(params.handle, _ptr(self.buffer), nbytes, n_seq, n_kv_heads, capacity, n_sink,
                                  _ptr(self.lens), _ptr(self.status), ctypes.byref(self.struct)))
        self.params = params
        self.n_seq, self.n_kv_heads, self.capacity, self.n_sink = n_seq, n_kv_heads, capacity, n_sink

    def plane(self, name: str, dtype, row_elems: int):
        """View of one row-ordered plane (norms, qjl, res_norms, sink) as a
        tensor [n_seq][n_kv_heads][rows][row_elems].  The code planes are
        tiled: use read_rows / write_rows for them."""
        import torch
        if name.endswith("_codes"):
            raise ValueError("code planes are tiled; use Cache.read_rows / Cache.write_rows")
        ptr = getattr(self.struct, name)
        if not ptr:
            return None
        rows = self.n_sink if name.endswith("sink") else self.capacity
        itemsize = torch.tensor([], dtype=dtype).element_size()
        count = self.n_seq * self.n_kv_heads * rows * row_elems
        off = ptr - self.buffer.data_ptr()
        flat = self.buffer[off: off + count * itemsize].view(dtype)
        return flat.view(self.n_seq, self.n_kv_heads, rows, row_elems)


def tq_cache_write_rows(params: Params, cache: Cache, which: int, seq: int, kv_head: int, row0: int,
                        rows: Packed, n: int, stream=None):
    """Copy n packed rows into quantized rows row0.. of unit (seq, kv_head)."""
    st = rows.struct()
    _check(_lib.tq_cache_write_rows(params.handle, ctypes.byref(cache.struct), which, seq, kv_head, row0, n,
                                    ctypes.byref(st), _stream(stream)))


def tq_cache_read_rows(params: Params, cache: Cache, which: int, seq: int, kv_head: int, row0: int,
                       rows: Packed, n: int, stream=None):
    """Copy quantized rows row0 .. row0 + n - 1 of unit (seq, kv_head) out as packed rows."""
    st = rows.struct()
    _check(_lib.tq_cache_read_rows(params.handle, ctypes.byref(cache.struct), which, seq, kv_head, row0, n,
                                   ctypes.byref(st), _stream(stream)))


def tq_append(params: Params, cache: Cache, seq_ids, k, v, stream=None):
    """k, v: (n_seq, n_tok, n_kv_heads, d) CUDA tensors; seq_ids: int32 CUDA (n_seq,)."""
    assert k.is_contiguous() and v.is_contiguous() and k.dtype == v.dtype
    n_seq, n_tok = k.shape[0], k.shape[1]
    _check(_lib.tq_append(params.handle, ctypes.byref(cache.struct), _ptr(seq_ids), _ptr(k), _ptr(v),
                          _dtype_code(k), n_tok, n_seq, _stream(stream)))


def tq_decode_workspace_bytes(params: Params, B: int, hq: int, n_kv_heads: int, max_len: int) -> int:
    return _lib.tq_decode_workspace_bytes(params.handle, B, hq, n_kv_heads, max_len)


def tq_decode_workspace_init(workspace, stream=None):
    _check(_lib.tq_decode_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream)))


def decode_workspace(params: Params, B: int, hq: int, n_kv_heads: int, max_len: int, device="cuda"):
    """Allocate and zero a workspace for tq_decode_attn."""
    import torch
    nbytes = tq_decode_workspace_bytes(params, B, hq, n_kv_heads, max_len)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def tq_decode_attn(params: Params, q, cache: Cache, max_len: int, out, workspace,
                   sparse_v_threshold: float = 0.0, stream=None, sparse_v_stats=None):
    """q, out: (B, hq, d) CUDA tensors (fp32 or bf16).  sparse_v_stats: None
    or a (4,) int64 CUDA tensor the call adds its sparse-V tallies to."""
    B, hq = q.shape[0], q.shape[1]
    flags = TqAttnFlags(sparse_v_threshold, 0, _ptr(sparse_v_stats))
    _check(_lib.tq_decode_attn(params.handle, _ptr(q), _dtype_code(q), ctypes.byref(cache.struct), B, hq,
                               max_len, _ptr(out), _dtype_code(out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), ctypes.byref(flags),
                               _stream(stream)))


def tq_decode_attn_noalloc(params: Params, q, cache: Cache, max_len: int, out, sparse_v_threshold: float = 0.0,
                           stream=None, sparse_v_stats=None):
    """tq_decode_attn with the library's fixed device scratch instead of a
    caller workspace (see include/tq.h)."""
    B, hq = q.shape[0], q.shape[1]
    flags = TqAttnFlags(sparse_v_threshold, 0, _ptr(sparse_v_stats))
    _check(_lib.tq_decode_attn_noalloc(params.handle, _ptr(q), _dtype_code(q), ctypes.byref(cache.struct), B, hq,
                                       max_len, _ptr(out), _dtype_code(out), ctypes.byref(flags), _stream(stream)))


# ---- inner-product search ----------------------------------------------------

def tq_search_workspace_bytes() -> int:
    return _lib.tq_search_workspace_bytes()


def search_workspace(device="cuda"):
    """Allocate a workspace for tq_search."""
    import torch
    return torch.empty(tq_search_workspace_bytes(), dtype=torch.uint8, device=device)


def tq_search(params: Params, which: int, db: Packed, n: int, q, k: int, scores, rows, workspace, stream=None):
    """q: (n_queries, d) CUDA tensor (fp32 or bf16); scores: (n_queries, k)
    fp32 and rows: (n_queries, k) int64 CUDA tensors."""
    assert q.is_contiguous() and scores.is_contiguous() and rows.is_contiguous()
    st = db.struct()
    _check(_lib.tq_search(params.handle, which, ctypes.byref(st), n, _ptr(q), _dtype_code(q), q.shape[0], k,
                          _ptr(scores), _ptr(rows), _ptr(workspace), workspace.numel() * workspace.element_size(),
                          _stream(stream)))
