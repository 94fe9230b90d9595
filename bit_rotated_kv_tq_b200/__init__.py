"""Python binding of the TQ4/4 C-ABI library (include/tq.h) for B200.

Argument marshalling only: every step of the append / decode / dequantise
path runs in the CUDA kernels of ``libtq_b200.so``.  PyTorch supplies device
memory and the current stream.  There is no fallback: if the shared library
is missing, every call raises.

Method: "TurboQuant 在 AMD GPU 上把長上下文延遲壓下來" (TQ4/4: Walsh-Hadamard-
rotated keys with a 16-entry table, uniform 4-bit values) and
"UltraQuant：4-bit KV 快取加速長代理" (Lloyd-Max or re-fitted centroid table).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq_b200.so")

BLOCK = 16
VALUE_GROUP = 32
TQ_CACHE_UNROTATED = 1  # cache flag: keys quantised without the rotation
TQ_CACHE_BF16 = 2       # cache flag: full-precision bf16 rows (layers kept unquantised)

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_ALIGNMENT, TQ_ERR_CUDA, TQ_ERR_WORKSPACE = range(6)
STATUS_BAD_SLOT, STATUS_BAD_BLOCK, STATUS_RANGE, STATUS_BAD_LEN, STATUS_TIMEOUT, STATUS_INTERNAL = \
    1, 2, 4, 8, 16, 32


class TQError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"tq error {code}: {msg}")
        self.code = code


class _Cache(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("data", ctypes.c_void_p)]


_lib = None
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def load(path: str | None = None):
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: run `python bit_rotated_kv_tq_b200/build.py`")
    L = ctypes.CDLL(p)
    L.tq_record_bytes.restype = _Z
    L.tq_record_bytes.argtypes = [_I]
    L.tq_cache_bytes.restype = _Z
    L.tq_cache_bytes.argtypes = [_I, _I, _I]
    L.tq_cache_record_bytes.restype = _Z
    L.tq_cache_record_bytes.argtypes = [_I, _I]
    L.tq_lloyd_max_table.argtypes = [_I, _P]
    L.tq_fit_k_table.argtypes = [_P, _I, _I, _P, _I, _P]
    L.tq_quantize_append.argtypes = [_P, _P, _P, _I, _I, _P, _I, ctypes.POINTER(_Cache), _P, _P, _P]
    L.tq_decode_default_splits.argtypes = [_I, _I, _I]
    L.tq_decode_workspace_bytes.restype = _Z
    L.tq_decode_workspace_bytes.argtypes = [_I, _I, _I, _I]
    L.tq_decode_attention.argtypes = [_P, ctypes.POINTER(_Cache), _P, _P, _I, _P, _I, _I, _I, _F,
                                      _P, _P, _Z, _I, _P, _P]
    L.tq_dequantize.argtypes = [ctypes.POINTER(_Cache), _P, _P, _I, _P, _I, _I, _P, _P, _P, _P]
    L.tq_decode_attention_static.argtypes = [_P, ctypes.POINTER(_Cache), _P, _P, _I, _P, _I, _I, _I, _F,
                                             _P, _I, _P, _P]
    L.tq_decode_static_scratch_bytes.restype = _Z
    L.tq_decode_static_scratch_bytes.argtypes = []
    L.tq_prefill_attention.argtypes = [_P, ctypes.POINTER(_Cache), _P, _P, _I, _P, _P, _I, _I, _I, _I, _F, _P,
                                       _P, _P]
    L.tq_last_error.restype = ctypes.c_char_p
    L.tq_last_error.argtypes = []
    _lib = L
    return L


def _check(rc: int):
    if rc != TQ_OK:
        raise TQError(rc, load().tq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    """A contiguous CUDA tensor of `dtype` on the current device (the one the
    library launches on), or None."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}; the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    return t


def _shape(t, shape, name):
    """The library sees bare pointers: every extent it will read or write is
    checked here.  None in `shape` matches any size."""
    if t is None:
        return
    if t.dim() != len(shape) or any(w is not None and int(g) != w for g, w in zip(t.shape, shape)):
        want = "[" + "][".join("*" if w is None else str(w) for w in shape) + "]"
        raise ValueError(f"{name} has shape {list(t.shape)}, expected {want}")


def _tables(k_tables, cache):
    """k_tables: [H_kv][16] values (any shape holding exactly that many)."""
    if k_tables is not None and k_tables.numel() != cache.num_kv_heads * 16:
        raise ValueError(f"k_tables holds {k_tables.numel()} values, expected "
                         f"{cache.num_kv_heads} x 16")


def _status(status):
    """The library writes status[0] only."""
    if status is not None and status.numel() < 1:
        raise ValueError("status must hold at least one int32")


# ------------------------------------------------------------------ sizes, tables
def record_bytes(head_dim: int) -> int:
    return int(load().tq_record_bytes(head_dim))


def lloyd_max_table(head_dim: int) -> np.ndarray:
    """The default fp16 key table (numpy float16 [16])."""
    out = np.zeros(16, np.uint16)
    _check(load().tq_lloyd_max_table(head_dim, out.ctypes.data_as(_P)))
    return out.view(np.float16)


def fit_k_table(keys: torch.Tensor, init: np.ndarray, max_iter: int = 100):
    """keys: bf16 [n][d] (host), init: float16 [16]; returns (float16 [16] table, iterations)."""
    k = keys.detach().to("cpu").contiguous()
    if k.dtype != torch.bfloat16 or k.dim() != 2:
        raise ValueError("keys must be a 2-D bf16 tensor")
    bits = k.view(torch.int16).numpy().view(np.uint16)
    init = np.ascontiguousarray(init)
    if init.dtype != np.float16:
        raise ValueError("init must be a float16 table")
    init = init.view(np.uint16)
    out = np.zeros(16, np.uint16)
    rc = load().tq_fit_k_table(bits.ctypes.data_as(_P), k.shape[0], k.shape[1],
                               init.ctypes.data_as(_P), max_iter, out.ctypes.data_as(_P))
    if rc < 0:
        _check(-rc)
    return out.view(np.float16), rc


# ------------------------------------------------------------------ cache
class Cache:
    """A paged TQ4/4 cache: uint8 [num_blocks][num_kv_heads][record] in device memory.

    rotate=False makes an unrotated cache (TQ_CACHE_UNROTATED: keys quantised without
    the Walsh-Hadamard rotation, the baseline the rotation is measured against);
    bf16=True a full-precision cache (TQ_CACHE_BF16: bf16 rows, for the layers a
    model keeps unquantised).
    """

    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int, device="cuda", data=None,
                 rotate: bool = True, bf16: bool = False):
        flags = (0 if rotate else TQ_CACHE_UNROTATED) | (TQ_CACHE_BF16 if bf16 else 0)
        nbytes = int(load().tq_cache_bytes(num_blocks, num_kv_heads, head_dim))
        rec = int(load().tq_cache_record_bytes(head_dim, flags))
        if nbytes == 0 or rec == 0:
            raise TQError(TQ_ERR_UNSUPPORTED,
                          f"cache shape ({num_blocks}, {num_kv_heads}, {head_dim}), flags {flags}")
        if data is None:
            data = torch.zeros((num_blocks, num_kv_heads, rec), dtype=torch.uint8, device=device)
        if tuple(data.shape) != (num_blocks, num_kv_heads, rec) or data.dtype != torch.uint8:
            raise ValueError("cache data has the wrong shape or dtype")
        self.data = data
        self.num_blocks, self.num_kv_heads, self.head_dim = num_blocks, num_kv_heads, head_dim
        self.rotate, self.bf16, self.flags = bool(rotate), bool(bf16), flags
        self._c = _Cache(num_blocks, num_kv_heads, head_dim, flags, data.data_ptr())

    @property
    def c(self):
        self._c.data = self.data.data_ptr()
        return ctypes.byref(self._c)


# ------------------------------------------------------------------ hot calls
def quantize_append(K, V, slot_mapping, cache: Cache, block_table=None, k_tables=None,
                    status=None, stream=None):
    """Quantise K, V (bf16 [T][H_kv][d], CUDA) into `cache` at `slot_mapping` (int32 [T]).

    With block_table (int32 [num_seqs][max_blocks]) the slots are logical:
    seq * max_blocks * 16 + position.
    """
    T = K.shape[0] if K.dim() == 3 else -1
    _shape(K, (T, cache.num_kv_heads, cache.head_dim), "K")
    _shape(V, (T, cache.num_kv_heads, cache.head_dim), "V")
    _shape(slot_mapping, (T,), "slot_mapping")
    _shape(block_table, (None, None), "block_table")
    _tables(k_tables, cache)
    _status(status)
    _dev(K, torch.bfloat16, "K")
    _dev(V, torch.bfloat16, "V")
    _dev(slot_mapping, torch.int32, "slot_mapping")
    _dev(block_table, torch.int32, "block_table")
    _dev(k_tables, torch.float16, "k_tables")
    _dev(status, torch.int32, "status")
    _dev(cache.data, torch.uint8, "cache.data")
    ns, mb = (0, 0) if block_table is None else (block_table.shape[0], block_table.shape[1])
    _check(load().tq_quantize_append(_ptr(K), _ptr(V), _ptr(block_table), ns, mb, _ptr(slot_mapping),
                                     T, cache.c, _ptr(k_tables), _ptr(status), _stream(stream)))


def default_splits(B: int, H_kv: int, max_seq_len: int) -> int:
    return int(load().tq_decode_default_splits(B, H_kv, max_seq_len))


def workspace_bytes(B: int, H_q: int, head_dim: int, num_splits: int) -> int:
    return int(load().tq_decode_workspace_bytes(B, H_q, head_dim, num_splits))


def decode_attention(q, cache: Cache, block_tables, seq_lens, max_seq_len: int, scale: float,
                     out=None, workspace=None, num_splits: int = 0, k_tables=None, status=None,
                     stream=None):
    """Split-K decode attention over the compressed cache; returns fp32 [B][H_q][d]."""
    B, Hq, d = _decode_checks(q, cache, block_tables, seq_lens, out, k_tables, status)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    S = num_splits or default_splits(B, cache.num_kv_heads, max_seq_len)
    if workspace is None:
        nb = workspace_bytes(B, Hq, d, S)
        workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=q.device)
    _dev(workspace, workspace.dtype, "workspace")
    _check(load().tq_decode_attention(_ptr(q), cache.c, _ptr(k_tables), _ptr(block_tables),
                                      block_tables.shape[1], _ptr(seq_lens), B, Hq, int(max_seq_len),
                                      float(scale), _ptr(out), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      int(num_splits), _ptr(status), _stream(stream)))
    return out


def _decode_checks(q, cache, block_tables, seq_lens, out, k_tables, status):
    """Shapes first (any device), then placement; returns (B, H_q, d)."""
    if q.dim() != 3:
        raise ValueError(f"q has shape {list(q.shape)}, expected [B][H_q][d]")
    B, Hq, d = (int(x) for x in q.shape)
    _shape(q, (B, Hq, cache.head_dim), "q")
    _shape(block_tables, (B, None), "block_tables")
    _shape(seq_lens, (B,), "seq_lens")
    _shape(out, (B, Hq, d), "out")
    _tables(k_tables, cache)
    _status(status)
    _dev(q, torch.bfloat16, "q")
    _dev(block_tables, torch.int32, "block_tables")
    _dev(seq_lens, torch.int32, "seq_lens")
    _dev(out, torch.float32, "out")
    _dev(k_tables, torch.float16, "k_tables")
    _dev(status, torch.int32, "status")
    _dev(cache.data, torch.uint8, "cache.data")
    return B, Hq, d


def decode_attention_static(q, cache: Cache, block_tables, seq_lens, max_seq_len: int, scale: float,
                            out=None, num_splits: int = 0, k_tables=None, status=None, stream=None):
    """decode_attention for callers that cannot allocate: no workspace argument; the split
    partials use the library's fixed device array (see tq_decode_attention_static)."""
    B, Hq, d = _decode_checks(q, cache, block_tables, seq_lens, out, k_tables, status)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _check(load().tq_decode_attention_static(_ptr(q), cache.c, _ptr(k_tables), _ptr(block_tables),
                                             block_tables.shape[1], _ptr(seq_lens), B, Hq,
                                             int(max_seq_len), float(scale), _ptr(out), int(num_splits),
                                             _ptr(status), _stream(stream)))
    return out


def prefill_attention(q, cache: Cache, block_tables, seq_lens, q_start, max_q_len: int, scale: float,
                      out=None, k_tables=None, status=None, stream=None):
    """Chunked-prefill attention over the compressed cache (the chunk appended first):
    chunk token i of sequence b attends to cached positions 0 .. seq_lens[b] - q_len + i.
    q bf16 [T][H_q][d]; chunk b is rows q_start[b] .. q_start[b+1]-1; returns fp32
    [T][H_q][d].  max_q_len bounds the chunks (it sizes the grid)."""
    if q.dim() != 3:
        raise ValueError(f"q has shape {list(q.shape)}, expected [T][H_q][d]")
    T, Hq, d = (int(x) for x in q.shape)
    B = int(seq_lens.shape[0]) if seq_lens.dim() == 1 else -1
    _shape(q, (T, Hq, cache.head_dim), "q")
    _shape(seq_lens, (B,), "seq_lens")
    _shape(block_tables, (B, None), "block_tables")
    _shape(q_start, (B + 1,), "q_start")
    _shape(out, (T, Hq, d), "out")
    _tables(k_tables, cache)
    _status(status)
    for t, dt, name in ((q, torch.bfloat16, "q"), (block_tables, torch.int32, "block_tables"),
                        (seq_lens, torch.int32, "seq_lens"), (q_start, torch.int32, "q_start"),
                        (out, torch.float32, "out"), (k_tables, torch.float16, "k_tables"),
                        (status, torch.int32, "status"), (cache.data, torch.uint8, "cache.data")):
        _dev(t, dt, name)
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.float32, device=q.device)
    _check(load().tq_prefill_attention(_ptr(q), cache.c, _ptr(k_tables), _ptr(block_tables),
                                       block_tables.shape[1], _ptr(seq_lens), _ptr(q_start), B, Hq, T,
                                       int(max_q_len), float(scale), _ptr(out), _ptr(status),
                                       _stream(stream)))
    return out


def dequantize(cache: Cache, block_tables, seq_lens, max_len: int, k_tables=None, status=None,
               stream=None):
    """(K_hat, V_hat) fp32 [B][max_len][H_kv][d] in the original domain (checks only)."""
    _shape(block_tables, (None, None), "block_tables")
    _shape(seq_lens, (block_tables.shape[0],), "seq_lens")
    _tables(k_tables, cache)
    _status(status)
    _dev(cache.data, torch.uint8, "cache.data")
    _dev(block_tables, torch.int32, "block_tables")
    _dev(seq_lens, torch.int32, "seq_lens")
    _dev(k_tables, torch.float16, "k_tables")
    _dev(status, torch.int32, "status")
    B = block_tables.shape[0]
    shape = (B, max_len, cache.num_kv_heads, cache.head_dim)
    Kh = torch.empty(shape, dtype=torch.float32, device=block_tables.device)
    Vh = torch.empty(shape, dtype=torch.float32, device=block_tables.device)
    _check(load().tq_dequantize(cache.c, _ptr(k_tables), _ptr(block_tables), block_tables.shape[1],
                                _ptr(seq_lens), B, max_len, _ptr(Kh), _ptr(Vh), _ptr(status),
                                _stream(stream)))
    return Kh, Vh
