"""Host-side checks of the C-ABI library: it loads, exports every symbol that
include/tq.h declares, and its host-only routines (tables, sizes, argument
validation) behave as documented.  No call here launches GPU work."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import bit_rotated_kv_tq_b200 as tq
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "tq.h")


@pytest.fixture(scope="module")
def lib():
    from bit_rotated_kv_tq_b200 import build

    build.build()
    return tq.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for want in ("tq_quantize_append", "tq_decode_attention", "tq_dequantize", "tq_last_error"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_record_and_cache_sizes(lib, orc):
    for d in (64, 128):
        assert tq.record_bytes(d) == orc.record_bytes(d)
        assert lib.tq_cache_bytes(10, 3, d) == 30 * orc.record_bytes(d)
    assert tq.record_bytes(96) == 0 and lib.tq_cache_bytes(0, 1, 64) == 0


@pytest.mark.parametrize("d", [64, 128])
def test_default_table_equals_oracle(lib, orc, d):
    assert np.array_equal(tq.lloyd_max_table(d), orc.default_table(d))


def test_default_table_other_power_of_two(lib, orc):
    assert np.array_equal(tq.lloyd_max_table(256), orc.default_table(256))
    with pytest.raises(tq.TQError):
        tq.lloyd_max_table(96)


def test_fit_k_table_equals_oracle(lib, orc):
    rng = np.random.default_rng(7)
    for d in (64, 128):
        keys = torch.from_numpy((rng.standard_t(4, (20, d)) * rng.lognormal(0, 1, d)).astype(np.float32))
        keys = keys.to(torch.bfloat16)
        init = orc.default_table(d)
        assert init.dtype == np.float16
        got, it = tq.fit_k_table(keys, init, 100)
        bits = keys.view(torch.int16).numpy().view(np.uint16)
        want, it2 = orc.kmeans_table(orc.rotated_unit_samples(bits), init, 100)
        assert np.array_equal(got, want) and it == it2
    # degenerate calibration sets: no vector keeps the initial table; zero keys put every
    # sample at 0, which moves the level that takes 0 (the lower of the two middle ones)
    init = orc.default_table(128)
    got, it = tq.fit_k_table(torch.zeros((0, 128), dtype=torch.bfloat16), init, 10)
    assert it == 0 and np.array_equal(got.view(np.uint16), init.view(np.uint16))
    zeros = torch.zeros((3, 128), dtype=torch.bfloat16)
    got, it = tq.fit_k_table(zeros, init, 10)
    want, it2 = orc.kmeans_table(orc.rotated_unit_samples(np.zeros((3, 128), np.uint16)), init, 10)
    assert np.array_equal(got, want) and it == it2
    assert float(got[7]) == 0.0 and np.array_equal(np.delete(got, 7), np.delete(init, 7))


def _cache_struct(num_blocks=4, heads=2, d=128, data=0x1000):
    return tq._Cache(num_blocks, heads, d, 0, data)


def test_argument_validation_without_launch(lib):
    """Every case is rejected by host validation before anything is enqueued."""
    P = ctypes.c_void_p
    c = _cache_struct(d=96)
    rc = lib.tq_quantize_append(P(16), P(16), None, 0, 0, P(16), 4, ctypes.byref(c), None, None, None)
    assert rc == tq.TQ_ERR_UNSUPPORTED and b"head_dim" in lib.tq_last_error()
    c = _cache_struct(data=0)
    rc = lib.tq_quantize_append(P(16), P(16), None, 0, 0, P(16), 4, ctypes.byref(c), None, None, None)
    assert rc == tq.TQ_ERR_INVALID_ARG
    c = _cache_struct(data=0x1008)
    rc = lib.tq_quantize_append(P(16), P(16), None, 0, 0, P(16), 4, ctypes.byref(c), None, None, None)
    assert rc == tq.TQ_ERR_ALIGNMENT
    c = _cache_struct()
    rc = lib.tq_quantize_append(P(24), P(16), None, 0, 0, P(16), 4, ctypes.byref(c), None, None, None)
    assert rc == tq.TQ_ERR_ALIGNMENT
    rc = lib.tq_quantize_append(None, P(16), None, 0, 0, P(16), 4, ctypes.byref(c), None, None, None)
    assert rc == tq.TQ_ERR_INVALID_ARG
    rc = lib.tq_quantize_append(None, None, None, 0, 0, None, 0, ctypes.byref(c), None, None, None)
    assert rc == tq.TQ_OK  # T == 0 is a no-op
    # cache flags: TQ_CACHE_UNROTATED and TQ_CACHE_BF16 are the defined bits, never both;
    # every call checks them
    for bad in (2, 4, 1 << 30):
        c = tq._Cache(4, 2, 128, bad | tq.TQ_CACHE_UNROTATED, 0x1000)
        rc = lib.tq_quantize_append(None, None, None, 0, 0, None, 0, ctypes.byref(c), None, None, None)
        assert rc == tq.TQ_ERR_INVALID_ARG and b"flags" in lib.tq_last_error()
        rc = lib.tq_dequantize(ctypes.byref(c), None, P(16), 1, P(16), 1, 16, P(16), P(16), None, None)
        assert rc == tq.TQ_ERR_INVALID_ARG and b"flags" in lib.tq_last_error()
    c = tq._Cache(4, 2, 128, tq.TQ_CACHE_UNROTATED, 0x1000)
    rc = lib.tq_quantize_append(None, None, None, 0, 0, None, 0, ctypes.byref(c), None, None, None)
    assert rc == tq.TQ_OK
    # decode: H_q not a multiple of H_kv, or a GQA group above 64, unsupported; workspace
    # too small; bad split count
    c = _cache_struct(heads=2)
    args = dict(q=P(16), k=None, bt=P(16), mb=4, sl=P(16), B=1, Hq=6, L=64, scale=0.1, out=P(16),
                ws=None, wsb=0, S=0)

    def dec(**kw):
        a = {**args, **kw}
        return lib.tq_decode_attention(a["q"], ctypes.byref(c), a["k"], a["bt"], a["mb"], a["sl"], a["B"],
                                       a["Hq"], a["L"], ctypes.c_float(a["scale"]), a["out"], a["ws"],
                                       a["wsb"], a["S"], None, None)

    assert dec(Hq=5) == tq.TQ_ERR_UNSUPPORTED
    assert dec(Hq=2 * 65) == tq.TQ_ERR_UNSUPPORTED
    assert dec(Hq=4, S=4) == tq.TQ_ERR_WORKSPACE
    assert dec(Hq=4, S=2000) == tq.TQ_ERR_UNSUPPORTED
    assert dec(Hq=4, L=65) == tq.TQ_ERR_INVALID_ARG  # max_seq_len beyond max_blocks * 16
    assert dec(Hq=4, scale=float("nan")) == tq.TQ_ERR_INVALID_ARG
    assert dec(Hq=4, B=0) == tq.TQ_OK
    # out takes 8-byte pair stores; q and the int32 arrays need 4 bytes
    for mis in (dict(out=P(20)), dict(out=P(18)), dict(q=P(18)), dict(bt=P(2)), dict(sl=P(6)), dict(k=P(2))):
        assert dec(Hq=4, **mis) == tq.TQ_ERR_ALIGNMENT, mis
    assert dec(Hq=4, B=0, out=P(20)) == tq.TQ_OK  # an empty batch checks no pointer
    # explicit splits: at most B * H_q * S + 1 ranges, two partial slots of four heads each
    assert lib.tq_decode_workspace_bytes(2, 8, 128, 4) == (2 * 8 * 4 + 1) * 2 * 4 * (128 * 4 + 8)
    assert lib.tq_decode_workspace_bytes(2, 8, 64, 3) == (2 * 8 * 3 + 1) * 2 * 4 * (64 * 4 + 8)
    assert lib.tq_decode_workspace_bytes(2, 8, 128, 1) == 0
    assert lib.tq_decode_default_splits(32, 8, 8192) == 0  # the even cut, no fixed count
    # the fixed-scratch entry runs the same checks first, with the same codes
    def dec_static(**kw):
        a = {**args, **kw}
        return lib.tq_decode_attention_static(a["q"], ctypes.byref(c), a["k"], a["bt"], a["mb"],
                                              a["sl"], a["B"], a["Hq"], a["L"],
                                              ctypes.c_float(a["scale"]), a["out"], a["S"], None, None)

    assert dec_static(Hq=4, S=1025) == tq.TQ_ERR_UNSUPPORTED
    assert dec_static(Hq=4, S=1025, B=4096) == tq.TQ_ERR_UNSUPPORTED
    assert dec_static(Hq=5) == tq.TQ_ERR_UNSUPPORTED
    assert dec_static(Hq=4, L=65) == tq.TQ_ERR_INVALID_ARG
    assert dec_static(Hq=4, q=None) == tq.TQ_ERR_INVALID_ARG
    assert dec_static(Hq=4, B=0) == tq.TQ_OK
    assert dec_static(Hq=4, out=P(20)) == tq.TQ_ERR_ALIGNMENT
    # dequantize: bad sizes, missing pointers, misaligned output or int32 arrays
    def deq(k=None, bt=P(16), mb=4, sl=P(16), B=1, L=8, K=P(16), V=P(16), st=None):
        return lib.tq_dequantize(ctypes.byref(c), k, bt, mb, sl, B, L, K, V, st, None)

    for bad in (dict(B=-1), dict(L=-1), dict(mb=0), dict(bt=None), dict(sl=None), dict(K=None),
                dict(V=None)):
        assert deq(**bad) == tq.TQ_ERR_INVALID_ARG, bad
    assert deq(B=0, K=None, V=None) == tq.TQ_OK and deq(L=0, K=None, V=None) == tq.TQ_OK
    for mis in (dict(K=P(20)), dict(V=P(24)), dict(bt=P(18)), dict(sl=P(6)), dict(k=P(2)), dict(st=P(1))):
        assert deq(**mis) == tq.TQ_ERR_ALIGNMENT, mis


def test_prefill_argument_validation_without_launch(lib):
    """tq_prefill_attention rejects each bad argument on the host, before any launch."""
    P = ctypes.c_void_p
    c = _cache_struct(heads=2)
    args = dict(q=P(16), k=None, bt=P(16), mb=4, sl=P(16), qs=P(16), B=1, Hq=4, T=8, mq=8, scale=0.1,
                out=P(16))

    def pre(cache=c, **kw):
        a = {**args, **kw}
        return lib.tq_prefill_attention(a["q"], ctypes.byref(cache), a["k"], a["bt"], a["mb"], a["sl"],
                                        a["qs"], a["B"], a["Hq"], a["T"], a["mq"],
                                        ctypes.c_float(a["scale"]), a["out"], None, None)

    assert pre(cache=tq._Cache(4, 2, 128, tq.TQ_CACHE_BF16, 0x1000)) == tq.TQ_ERR_UNSUPPORTED
    assert pre(cache=_cache_struct(d=96)) == tq.TQ_ERR_UNSUPPORTED
    assert pre(cache=tq._Cache(4, 2, 128, tq.TQ_CACHE_BF16 | tq.TQ_CACHE_UNROTATED, 0x1000)) == tq.TQ_ERR_INVALID_ARG
    for bad in (dict(B=-1), dict(Hq=0), dict(T=-1), dict(mq=-1), dict(mb=0), dict(q=None), dict(qs=None),
                dict(out=None), dict(sl=None), dict(bt=None), dict(scale=float("inf"))):
        assert pre(**bad) == tq.TQ_ERR_INVALID_ARG, bad
    for empty in (dict(B=0), dict(T=0), dict(mq=0)):  # nothing to do: no launch, no pointer checks
        assert pre(q=None, out=None, **empty) == tq.TQ_OK, empty
    assert pre(B=65536) == tq.TQ_ERR_UNSUPPORTED
    assert pre(Hq=5) == tq.TQ_ERR_UNSUPPORTED
    assert pre(mq=1 << 30) == tq.TQ_ERR_UNSUPPORTED  # rows of (token, head) past 2^30
    for mis in (dict(q=P(24)), dict(out=P(40)), dict(qs=P(18)), dict(sl=P(2)), dict(bt=P(6)),
                dict(k=P(2))):
        assert pre(**mis) == tq.TQ_ERR_ALIGNMENT, mis
    # the unrotated cache is accepted by the same checks (the call stops at its empty batch)
    assert pre(cache=tq._Cache(4, 2, 128, tq.TQ_CACHE_UNROTATED, 0x1000), B=0) == tq.TQ_OK


def _host_cache(num_kv_heads=2, head_dim=128, num_blocks=1):
    rec = tq.record_bytes(head_dim)
    return tq.Cache(num_blocks, num_kv_heads, head_dim,
                    data=torch.zeros((num_blocks, num_kv_heads, rec), dtype=torch.uint8))


def test_binding_refuses_host_tensors(lib):
    c = _host_cache()
    K = torch.zeros((1, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        tq.quantize_append(K, K, torch.zeros(1, dtype=torch.int32), c)


def test_binding_checks_extents_before_anything_runs(lib):
    """The library reads and writes through bare pointers, so the binding refuses every
    tensor whose extent differs from what the call would touch (before placement)."""
    c = _host_cache()  # 2 kv heads, d 128

    def bf(*shape):
        return torch.zeros(shape, dtype=torch.bfloat16)

    def i32(*shape):
        return torch.zeros(shape, dtype=torch.int32)

    f16 = torch.zeros(16, dtype=torch.float16)
    cases = [
        (lambda: tq.quantize_append(bf(4, 1, 128), bf(4, 1, 128), i32(4), c), "K has shape"),
        (lambda: tq.quantize_append(bf(4, 2, 128), bf(4, 2, 64), i32(4), c), "V has shape"),
        (lambda: tq.quantize_append(bf(4, 256), bf(4, 256), i32(4), c), "K has shape"),
        (lambda: tq.quantize_append(bf(4, 2, 128), bf(4, 2, 128), i32(3), c), "slot_mapping has shape"),
        (lambda: tq.quantize_append(bf(4, 2, 128), bf(4, 2, 128), i32(4), c, k_tables=f16),
         "k_tables holds 16 values"),
        (lambda: tq.decode_attention(bf(2, 8, 64), c, i32(2, 4), i32(2), 64, 0.1), "q has shape"),
        (lambda: tq.decode_attention(bf(2, 8, 128), c, i32(3, 4), i32(2), 64, 0.1),
         "block_tables has shape"),
        (lambda: tq.decode_attention(bf(2, 8, 128), c, i32(2, 4), i32(3), 64, 0.1), "seq_lens has shape"),
        (lambda: tq.decode_attention(bf(2, 8, 128), c, i32(2, 4), i32(2), 64, 0.1,
                                     out=torch.zeros((2, 8, 64))), "out has shape"),
        (lambda: tq.decode_attention(bf(2, 8, 128), c, i32(2, 4), i32(2), 64, 0.1, status=i32(0)),
         "status must hold"),
        (lambda: tq.decode_attention_static(bf(2, 8, 128), c, i32(2, 4), i32(1), 64, 0.1),
         "seq_lens has shape"),
        (lambda: tq.dequantize(c, i32(2, 4), i32(3), 64), "seq_lens has shape"),
        (lambda: tq.prefill_attention(bf(8, 256), c, i32(2, 4), i32(2), i32(3), 4, 0.1), "q has shape"),
        (lambda: tq.prefill_attention(bf(8, 4, 64), c, i32(2, 4), i32(2), i32(3), 4, 0.1), "q has shape"),
        (lambda: tq.prefill_attention(bf(8, 4, 128), c, i32(3, 4), i32(2), i32(3), 4, 0.1),
         "block_tables has shape"),
        (lambda: tq.prefill_attention(bf(8, 4, 128), c, i32(2, 4), i32(2), i32(2), 4, 0.1),
         "q_start has shape"),
        (lambda: tq.prefill_attention(bf(8, 4, 128), c, i32(2, 4), i32(2), i32(3), 4, 0.1,
                                      out=torch.zeros((8, 4, 64))), "out has shape"),
        (lambda: tq.prefill_attention(bf(8, 4, 128), c, i32(2, 4), i32(2), i32(3), 4, 0.1, status=i32(0)),
         "status must hold"),
    ]
    for call, msg in cases:
        with pytest.raises(ValueError, match=msg):
            call()
    # the right extents on the host are refused for their placement
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        tq.decode_attention(bf(2, 8, 128), c, i32(2, 4), i32(2), 64, 0.1)


def test_workspace_bounds_cover_the_bf16_plans(lib):
    """A bf16 cache's decode keeps per (sequence, query head, range) an fp32 partial
    output and its (max, sum): B H_q S (4 d + 8) bytes.  The workspace size the library
    asks for must cover that for every explicit split count, and for its own default
    (up to 8 ranges, within the 8 MiB of the static entry)."""
    for B, Hq, d in [(1, 8, 64), (2, 32, 128), (32, 32, 128), (64, 64, 128), (16, 16, 64)]:
        per = B * Hq * (4 * d + 8)
        for S in (2, 3, 8, 64, 1024):
            assert lib.tq_decode_workspace_bytes(B, Hq, d, S) >= per * S
        assert lib.tq_decode_workspace_bytes(B, Hq, d, 0) >= min(8 * per, 8 << 20)
        assert lib.tq_decode_workspace_bytes(B, Hq, d, 1) == 0
    assert lib.tq_cache_record_bytes(128, tq.TQ_CACHE_BF16) == 8192
    assert lib.tq_cache_record_bytes(64, tq.TQ_CACHE_BF16) == 4096
    assert lib.tq_cache_record_bytes(128, 0) == lib.tq_record_bytes(128) == 2336
    assert lib.tq_cache_record_bytes(128, tq.TQ_CACHE_UNROTATED) == 2336
    assert lib.tq_cache_record_bytes(128, tq.TQ_CACHE_BF16 | tq.TQ_CACHE_UNROTATED) == 0
    assert lib.tq_cache_record_bytes(96, 0) == 0

