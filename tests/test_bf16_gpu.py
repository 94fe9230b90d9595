"""GPU parity of the full-precision cache (TQ_CACHE_BF16, the layers a model keeps
unquantised: "TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", section 3).

The append stores each bf16 row as it is, so its records are checked byte for
byte against the inputs at their slots (through a reader of the documented
layout: [16 key rows][16 value rows] of d bf16 per (block, kv head), the 16-byte
chunk j of row r at chunk position j xor (r mod 8)).  The
decode is compared with the oracle's fp64 attention over the exact bf16 keys and
values, under the same rule as the TQ4/4 decode (max-abs 2e-3, rel-L2 1e-3).
"""
import numpy as np
import pytest
import torch

import workloads as W
from parity_util import attn_errors, check_attention
from workloads import bf16_bits

pytestmark = pytest.mark.gpu


def _cache(tq, w, fill=0):
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d, bf16=True)
    if fill:
        cache.data.fill_(fill)
    bt = torch.from_numpy(w.block_tables).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for K, V, slots in w.population():
        tq.quantize_append(K.cuda(), V.cuda(), slots.cuda(), cache, block_table=bt, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return cache, bt


def _oracle(orc, w, q_bits):
    """fp64 attention over the exact bf16 keys and values of every sequence."""
    L = int(w.seq_lens.max())
    Kh = np.zeros((w.B, max(L, 1), w.Hkv, w.d))
    Vh = np.zeros_like(Kh)
    for b in range(w.B):
        n = int(w.seq_lens[b])
        if n:
            K, V = w.kv(b)
            Kh[b, :n], Vh[b, :n] = K.double().numpy(), V.double().numpy()
    return orc.attention(q_bits, Kh, Vh, w.seq_lens, w.scale)


def _unswizzle(row, r):
    """A stored row (uint16 [..., d]) back in element order: chunk j at j ^ (r % 8)."""
    d = row.shape[-1]
    i = np.arange(d)
    return row[..., (((i >> 3) ^ (r & 7)) << 3) | (i & 7)]


@pytest.mark.parametrize("name", ["qwen3_8b_layer", "prefill_small_head"])
def test_bf16_append_stores_rows(tq, name):
    w = W.make(name, B=2, ctx=100)
    cache, _ = _cache(tq, w)
    data = cache.data.cpu().numpy()
    d = w.d
    for b in range(w.B):
        K, V = w.kv(b)
        kb, vb = bf16_bits(K), bf16_bits(V)
        for t in range(int(w.seq_lens[b])):
            pb, off = w.block_tables[b, t // 16], t % 16
            rec = data[pb].view(np.uint16).reshape(w.Hkv, 32, d)
            assert np.array_equal(_unswizzle(rec[:, off], off), kb[t])
            assert np.array_equal(_unswizzle(rec[:, 16 + off], 16 + off), vb[t])
        # the last block's rows past the length were never written
        L = int(w.seq_lens[b])
        if L % 16:
            rec = data[w.block_tables[b, L // 16]].view(np.uint16).reshape(w.Hkv, 32, d)
            assert np.all(rec[:, L % 16:16] == 0) and np.all(rec[:, 16 + L % 16:] == 0)


@pytest.mark.parametrize("name,over,S", [
    ("qwen3_8b_layer", dict(B=3, ctx=1000), 0),         # ragged last block, shuffled tables
    ("qwen3_8b_layer", dict(B=2, ctx=777), 5),
    ("prefill_small_head", dict(B=3, ctx=1500), 0),     # d 64, GQA 8
    ("tiny", dict(B=2, ctx=17), 2),                     # one full block plus one token
    ("qwen3_8b_layer", dict(B=2, ctx=300, Hq=8), 3),    # GQA 1
    ("qwen3_8b_layer", dict(B=2, ctx=200, Hq=96), 0),   # GQA 12: items of 8 and 4 heads
    ("prefill_small_head", dict(B=1, ctx=260, Hq=128), 1),  # GQA 64 at d 64
    ("long_context", dict(B=1, ctx=4100), 64),          # many splits, some empty
])
def test_bf16_decode_matches_oracle(tq, orc, name, over, S):
    w = W.make(name, **over)
    cache, bt = _cache(tq, w)
    q = w.q()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tq.decode_attention(q.cuda(), cache, bt, torch.from_numpy(w.seq_lens).cuda(), int(w.seq_lens.max()),
                              w.scale, num_splits=S, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = out.cpu().numpy()
    want = _oracle(orc, w, bf16_bits(q))
    max_abs, rel = check_attention(got, want, f"{name} S={S}")
    # exact operands, p to ~2^-16: far inside the rule
    assert max_abs < 1e-4 and rel < 1e-5, (max_abs, rel)


def test_bf16_lengths_zero_and_one_and_stale_rows(tq, orc):
    """Unwritten slots hold NaN bit patterns (the cache starts filled with 0xff):
    rows past each length must not reach the output; a length of 0 gives 0."""
    w = W.make("qwen3_8b_layer", B=3, ctx=40)
    w.seq_lens[:] = [0, 1, 37]
    cache, bt = _cache(tq, w, fill=0xFF)
    q = w.q()
    for S in (0, 1, 3):
        out = tq.decode_attention(q.cuda(), cache, bt, torch.from_numpy(w.seq_lens).cuda(), 40, w.scale,
                                  num_splits=S).cpu().numpy()
        assert np.all(out[0] == 0)
        assert np.isfinite(out).all()
        check_attention(out[1:], _oracle(orc, w, bf16_bits(q))[1:], f"S={S}")


def test_bf16_dequantize_is_exact(tq):
    w = W.make("tiny", B=2, ctx=50)
    cache, bt = _cache(tq, w)
    lens = torch.from_numpy(w.seq_lens).cuda()
    Kh, Vh = tq.dequantize(cache, bt, lens, 56)
    Kh, Vh = Kh.cpu(), Vh.cpu()
    for b in range(w.B):
        K, V = w.kv(b)
        L = int(w.seq_lens[b])
        assert torch.equal(Kh[b, :L], K.float()) and torch.equal(Vh[b, :L], V.float())
        assert torch.all(Kh[b, L:] == 0) and torch.all(Vh[b, L:] == 0)


def test_bf16_static_entry_equals_workspace_entry(tq):
    w = W.make("qwen3_8b_layer", B=2, ctx=500)
    cache, bt = _cache(tq, w)
    q, lens = w.q().cuda(), torch.from_numpy(w.seq_lens).cuda()
    for S in (0, 1, 4):
        a = tq.decode_attention(q, cache, bt, lens, 500, w.scale, num_splits=S)
        s = tq.decode_attention_static(q, cache, bt, lens, 500, w.scale, num_splits=S)
        torch.cuda.synchronize()
        assert torch.equal(a, s)


def test_bf16_cache_argument_errors(tq):
    w = W.make("tiny", B=1, ctx=32)
    cache, bt = _cache(tq, w)
    lens = torch.from_numpy(w.seq_lens).cuda()
    tables = torch.from_numpy(np.tile(tq.lloyd_max_table(w.d), (w.Hkv, 1))).cuda()
    K, V = w.kv(0)
    with pytest.raises(tq.TQError) as e:
        tq.quantize_append(K.cuda(), V.cuda(), torch.arange(32, dtype=torch.int32, device="cuda"), cache,
                           k_tables=tables)
    assert e.value.code == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TQError) as e:
        tq.decode_attention(w.q().cuda(), cache, bt, lens, 32, w.scale, k_tables=tables)
    assert e.value.code == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TQError) as e:
        tq.prefill_attention(torch.zeros((4, w.Hq, w.d), dtype=torch.bfloat16, device="cuda"), cache, bt, lens,
                             torch.tensor([0, 4], dtype=torch.int32, device="cuda"), 4, w.scale)
    assert e.value.code == tq.TQ_ERR_UNSUPPORTED
    with pytest.raises(tq.TQError):
        tq.Cache(4, 2, 128, rotate=False, bf16=True)


def test_tq_and_bf16_caches_agree(tq, orc):
    """The same data through both caches: the bf16 decode is the exact one; the TQ4/4
    decode differs from it by the quantisation alone (a sanity bound, not parity)."""
    w = W.make("prefill_small_head", B=2, ctx=700)
    cache, bt = _cache(tq, w)
    tqc = tq.Cache(w.num_blocks, w.Hkv, w.d)
    for K, V, slots in w.population():
        tq.quantize_append(K.cuda(), V.cuda(), slots.cuda(), tqc, block_table=bt)
    q, lens = w.q().cuda(), torch.from_numpy(w.seq_lens).cuda()
    a = tq.decode_attention(q, cache, bt, lens, 700, w.scale).cpu().numpy()
    b = tq.decode_attention(q, tqc, bt, lens, 700, w.scale).cpu().numpy()
    want = _oracle(orc, w, bf16_bits(w.q()))
    ea, eb = attn_errors(a, want), attn_errors(b, want)
    assert ea[1] < 1e-5 and eb[1] > 10 * ea[1] and eb[1] < 0.2
