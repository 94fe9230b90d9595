"""Plain fp64 CPU oracle for TQ4/4 KV-cache compression (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The product path never does: it shares no
code with the CUDA kernels.  The arithmetic lives in ``tq_oracle.c`` (plain C
loops in binary64); this module only marshals numpy arrays through ctypes.

Functions follow "TurboQuant 在 AMD GPU 上把長上下文延遲壓下來" sections 2 and 4
(keys: Walsh-Hadamard rotation then a 16-entry look-up table; values: uniform
quantisation) and "UltraQuant：4-bit KV 快取加速長代理" section
「方法怎麼做，白話講」 (Lloyd-Max or re-fitted 16-entry table, no QJL).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "libtq_oracle.so")

BLOCK = 16
VGROUP = 32


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math) into oracle/."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "tq_oracle.h"))
    ):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-fPIC", "-shared",
             "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double


def _declare(L):
    L.orc_bf16_to_double.restype = _D
    L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
    L.orc_fp16_to_double.restype = _D
    L.orc_fp16_to_double.argtypes = [ctypes.c_uint16]
    L.orc_fp16_from_double.restype = ctypes.c_uint16
    L.orc_fp16_from_double.argtypes = [_D, _I]
    L.orc_lloyd_max_gaussian16.argtypes = [_P, _D, _I, _P]
    L.orc_default_table.argtypes = [_I, _P]
    L.orc_hadamard.argtypes = [_I, _P]
    L.orc_encode_k.argtypes = [_P, _I, _P, _P, _P, _P]
    L.orc_decode_k.argtypes = [_P, ctypes.c_uint16, _I, _P, _P]
    L.orc_encode_v.argtypes = [_P, _I, _P, _P, _P, _P]
    L.orc_decode_v.argtypes = [_P, _P, _P, _I, _P]
    L.orc_record_bytes.restype = ctypes.c_size_t
    L.orc_record_bytes.argtypes = [_I]
    L.orc_pack_token.argtypes = [_P, _I, _I, _P, ctypes.c_uint16, _P, _P, _P]
    L.orc_unpack_token.argtypes = [_P, _I, _I, _P, _P, _P, _P, _P]
    L.orc_quantize_append.argtypes = [_P, _P, _I, _I, _I, _P, _I, _I, _P, _P, _P, _I, _P, _P]
    L.orc_quantize_append_ex.argtypes = [_P, _P, _I, _I, _I, _P, _I, _I, _P, _P, _P, _I, _P, _P, _I]
    L.orc_dequantize.argtypes = [_P, _I, _I, _I, _P, _P, _I, _P, _I, _I, _P, _P]
    L.orc_dequantize_ex.argtypes = [_P, _I, _I, _I, _P, _P, _I, _P, _I, _I, _P, _P, _I]
    L.orc_encode_k_unrotated.argtypes = [_P, _I, _P, _P, _P, _P]
    L.orc_decode_k_unrotated.argtypes = [_P, ctypes.c_uint16, _I, _P, _P]
    L.orc_attention.argtypes = [_P, _I, _I, _I, _I, _P, _P, _I, _P, _D, _P]
    L.orc_prefill_attention.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _D, _P]
    L.orc_kmeans_table.argtypes = [_P, _I, _P, _I, _P]
    L.orc_rotated_unit_samples.argtypes = [_P, _I, _I, _P]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _h(table):
    """fp16 table(s) as contiguous uint16 bit patterns."""
    t = np.ascontiguousarray(table)
    if t.dtype != np.float16:
        raise TypeError("key tables are fp16 arrays")
    return t.view(np.uint16)


def _check(rc, what):
    if rc < 0:
        raise ValueError(f"oracle {what} failed with code {rc}")
    return rc


# ---------------------------------------------------------------- scalars
def bf16_to_double(bits: int) -> float:
    return lib().orc_bf16_to_double(int(bits))


def fp16_to_double(bits: int) -> float:
    return lib().orc_fp16_to_double(int(bits))


def fp16_from_double(x: float, mode: int = 0) -> int:
    """mode 0: nearest-even, -1: toward -inf, +1: toward +inf; returns the bit pattern."""
    return int(lib().orc_fp16_from_double(float(x), int(mode)))


# ---------------------------------------------------------------- tables
def lloyd_max_gaussian16(tol: float = 1e-15, max_iter: int = 10_000_000):
    c = np.zeros(16, np.float64)
    it = ctypes.c_int(0)
    _check(lib().orc_lloyd_max_gaussian16(_ptr(c), tol, max_iter, ctypes.byref(it)), "lloyd_max")
    return c, it.value


def default_table(d: int) -> np.ndarray:
    """fp16 [16] default key table (as a numpy float16 array)."""
    out = np.zeros(16, np.uint16)
    _check(lib().orc_default_table(d, _ptr(out)), "default_table")
    return out.view(np.float16)


def hadamard(d: int) -> np.ndarray:
    H = np.zeros((d, d), np.float64)
    _check(lib().orc_hadamard(d, _ptr(H)), "hadamard")
    return H


# ---------------------------------------------------------------- codecs
def encode_k(k_bits: np.ndarray, table: np.ndarray):
    """k_bits: uint16 bf16 bit patterns [d].  Returns (idx uint8[d], norm16 bits, y fp64[d])."""
    k = _c(k_bits, np.uint16)
    d = k.shape[-1]
    idx = np.zeros(d, np.uint8)
    n16 = np.zeros(1, np.uint16)
    y = np.zeros(d, np.float64)
    _check(lib().orc_encode_k(_ptr(k), d, _ptr(_h(table)), _ptr(idx), _ptr(n16), _ptr(y)),
           "encode_k")
    return idx, int(n16[0]), y


def decode_k(idx: np.ndarray, norm16: int, table: np.ndarray) -> np.ndarray:
    idx = _c(idx, np.uint8)
    d = idx.shape[-1]
    out = np.zeros(d, np.float64)
    _check(lib().orc_decode_k(_ptr(idx), int(norm16), d, _ptr(_h(table)), _ptr(out)),
           "decode_k")
    return out


def encode_k_unrotated(k_bits: np.ndarray, table: np.ndarray):
    """The unrotated baseline: (idx, norm16 bits, y = k / n)."""
    k = _c(k_bits, np.uint16)
    d = k.shape[-1]
    idx = np.zeros(d, np.uint8)
    n16 = np.zeros(1, np.uint16)
    y = np.zeros(d, np.float64)
    _check(lib().orc_encode_k_unrotated(_ptr(k), d, _ptr(_h(table)), _ptr(idx), _ptr(n16), _ptr(y)),
           "encode_k_unrotated")
    return idx, int(n16[0]), y


def decode_k_unrotated(idx: np.ndarray, norm16: int, table: np.ndarray) -> np.ndarray:
    idx = _c(idx, np.uint8)
    d = idx.shape[-1]
    out = np.zeros(d, np.float64)
    _check(lib().orc_decode_k_unrotated(_ptr(idx), int(norm16), d, _ptr(_h(table)), _ptr(out)),
           "decode_k_unrotated")
    return out


def encode_v(v_bits: np.ndarray):
    v = _c(v_bits, np.uint16)
    d = v.shape[-1]
    q = np.zeros(d, np.uint8)
    s = np.zeros(d // VGROUP, np.uint16)
    z = np.zeros(d // VGROUP, np.uint16)
    r = np.zeros(d, np.float64)
    _check(lib().orc_encode_v(_ptr(v), d, _ptr(q), _ptr(s), _ptr(z), _ptr(r)), "encode_v")
    return q, s, z, r


def decode_v(q, s, z) -> np.ndarray:
    q = _c(q, np.uint8)
    d = q.shape[-1]
    out = np.zeros(d, np.float64)
    _check(lib().orc_decode_v(_ptr(q), _ptr(_c(s, np.uint16)), _ptr(_c(z, np.uint16)), d, _ptr(out)),
           "decode_v")
    return out


def record_bytes(d: int) -> int:
    return int(lib().orc_record_bytes(d))


def pack_token(record: np.ndarray, d: int, offset: int, kidx, knorm: int, vq, vscale, vzero):
    """Write one token's fields into a record (uint8 numpy array, modified in place)."""
    if record.dtype != np.uint8 or not record.flags.c_contiguous:
        raise ValueError("record must be a contiguous uint8 array")
    _check(lib().orc_pack_token(_ptr(record), d, offset, _ptr(_c(kidx, np.uint8)), int(knorm),
                                _ptr(_c(vq, np.uint8)), _ptr(_c(vscale, np.uint16)),
                                _ptr(_c(vzero, np.uint16))), "pack_token")


def unpack_token(record: np.ndarray, d: int, offset: int):
    rec = _c(record, np.uint8)
    kidx = np.zeros(d, np.uint8)
    vq = np.zeros(d, np.uint8)
    kn = np.zeros(1, np.uint16)
    vs = np.zeros(d // VGROUP, np.uint16)
    vz = np.zeros(d // VGROUP, np.uint16)
    _check(lib().orc_unpack_token(_ptr(rec), d, offset, _ptr(kidx), _ptr(kn), _ptr(vq), _ptr(vs), _ptr(vz)),
           "unpack_token")
    return kidx, int(kn[0]), vq, vs, vz


# ---------------------------------------------------------------- paged cache
def quantize_append(K_bits, V_bits, slots, cache, tables=None, block_table=None, want_aux=False,
                    rotate=True):
    """K_bits/V_bits: uint16 [T][Hkv][d]; cache: uint8 [num_blocks][Hkv][record] (updated in place).

    Returns (rc, ky, vr): the (rotated, unless rotate=False) unit key coordinates and
    (v-z)/s, fp64 [T][Hkv][d] when want_aux, else None.
    """
    K = _c(K_bits, np.uint16)
    V = _c(V_bits, np.uint16)
    T, Hkv, d = K.shape
    sl = _c(slots, np.int32)
    assert cache.dtype == np.uint8 and cache.flags.c_contiguous
    num_blocks = cache.shape[0]
    tb = None if tables is None else _h(tables)
    bt = None if block_table is None else _c(block_table, np.int32)
    num_seqs = 0 if bt is None else bt.shape[0]
    max_blocks = 0 if bt is None else bt.shape[1]
    ky = np.zeros((T, Hkv, d), np.float64) if want_aux else None
    vr = np.zeros((T, Hkv, d), np.float64) if want_aux else None
    rc = lib().orc_quantize_append_ex(_ptr(K), _ptr(V), T, Hkv, d, _ptr(bt), num_seqs, max_blocks,
                                      _ptr(sl), _ptr(tb), _ptr(cache), num_blocks, _ptr(ky), _ptr(vr),
                                      1 if rotate else 0)
    return rc, ky, vr


def dequantize(cache, Hkv, d, block_tables, seq_lens, max_len, tables=None, rotate=True):
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    B, max_blocks = bt.shape
    # filled with NaN so that the oracle's own clearing of rows past each length is
    # what a caller sees (a missed row would show as NaN, not as a lucky 0)
    Kh = np.full((B, max_len, Hkv, d), np.nan, np.float64)
    Vh = np.full((B, max_len, Hkv, d), np.nan, np.float64)
    tb = None if tables is None else _h(tables)
    rc = lib().orc_dequantize_ex(_ptr(cache), cache.shape[0], Hkv, d, _ptr(tb), _ptr(bt), max_blocks,
                                 _ptr(sl), B, max_len, _ptr(Kh), _ptr(Vh), 1 if rotate else 0)
    _check(rc, "dequantize")
    return Kh, Vh


def attention(q_bits, Khat, Vhat, seq_lens, scale):
    q = _c(q_bits, np.uint16)
    B, Hq, d = q.shape
    _, max_len, Hkv, _ = Khat.shape
    out = np.zeros((B, Hq, d), np.float64)
    _check(lib().orc_attention(_ptr(q), B, Hq, Hkv, d, _ptr(_c(Khat, np.float64)), _ptr(_c(Vhat, np.float64)),
                               max_len, _ptr(_c(seq_lens, np.int32)), float(scale), _ptr(out)), "attention")
    return out


def prefill_attention(q_bits, q_start, Khat, Vhat, seq_lens, scale):
    """Chunked prefill: q_bits uint16 [T][Hq][d] (bf16), q_start int32 [B+1]; the chunk of
    sequence b is its last q_start[b+1] - q_start[b] cached tokens, each attending causally.
    Returns fp64 [T][Hq][d]."""
    q = _c(q_bits, np.uint16)
    T, Hq, d = q.shape
    qs = _c(q_start, np.int32)
    B = qs.shape[0] - 1
    _, max_len, Hkv, _ = Khat.shape
    out = np.zeros((T, Hq, d), np.float64)
    _check(lib().orc_prefill_attention(_ptr(q), _ptr(qs), B, Hq, Hkv, d, _ptr(_c(Khat, np.float64)),
                                       _ptr(_c(Vhat, np.float64)), max_len,
                                       _ptr(_c(seq_lens, np.int32)), float(scale), _ptr(out)),
           "prefill_attention")
    return out


# ---------------------------------------------------------------- calibration
def rotated_unit_samples(k_bits) -> np.ndarray:
    k = _c(k_bits, np.uint16)
    n, d = k.shape
    out = np.zeros((n, d), np.float64)
    _check(lib().orc_rotated_unit_samples(_ptr(k), n, d, _ptr(out)), "rotated_unit_samples")
    return out


def kmeans_table(samples, init, max_iter: int = 100):
    """Re-fit a 16-entry fp16 table on scalar samples; returns (float16 [16], iterations)."""
    s = _c(samples, np.float64).ravel()
    out = np.zeros(16, np.uint16)
    it = _check(lib().orc_kmeans_table(_ptr(s), s.size, _ptr(_h(init)), max_iter, _ptr(out)),
                "kmeans_table")
    return out.view(np.float16), it
