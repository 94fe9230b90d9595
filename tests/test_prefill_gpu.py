"""GPU parity of tq_prefill_attention (chunked prefill on the tcgen05 tensor cores)
against the CPU oracle.

The cache holds every token of each sequence (the chunk is appended before the
attention, as for the decode); the chunk is the last q_len of them.  The oracle
builds its own cache from the same bf16 inputs, dequantises it, and runs its
fp64 chunked-prefill attention; outputs are compared element by element under
the attention rule (max-abs 2e-3, rel-L2 1e-3).
"""
import numpy as np
import pytest
import torch

import workloads as W
from parity_util import check_attention
from workloads import bf16_bits

pytestmark = pytest.mark.gpu


def _gpu_cache(tq, w, tables=None, rotate=True):
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d, rotate=rotate)
    bt = torch.from_numpy(w.block_tables).cuda()
    for K, V, slots in w.population():
        tq.quantize_append(K.cuda(), V.cuda(), slots.cuda(), cache, block_table=bt, k_tables=tables)
    torch.cuda.synchronize()
    return cache, bt


def _oracle_prefill(orc, w, b, q_bits_b, qlen, table_rows, rotate=True):
    """fp64 chunked-prefill attention of sequence b's last qlen tokens (oracle only)."""
    L = int(w.seq_lens[b])
    K, V = w.kv(b)
    nblk = (L + 15) // 16
    cache = np.zeros((nblk, w.Hkv, orc.record_bytes(w.d)), np.uint8)
    rc, _, _ = orc.quantize_append(bf16_bits(K), bf16_bits(V), np.arange(L, dtype=np.int32), cache,
                                   tables=table_rows, rotate=rotate)
    assert rc == 0
    bt = np.arange(nblk, dtype=np.int32)[None]
    Kh, Vh = orc.dequantize(cache, w.Hkv, w.d, bt, np.array([L], np.int32), L, tables=table_rows,
                            rotate=rotate)
    return orc.prefill_attention(q_bits_b, np.array([0, qlen], np.int32), Kh, Vh,
                                 np.array([L], np.int32), w.scale)


def _run_case(tq, orc, w, qlens, tables=None, oracle_tables=None, seed=5, rotate=True):
    cache, bt = _gpu_cache(tq, w, tables, rotate)
    qlens = np.asarray(qlens, np.int32)
    q_start = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    T = int(q_start[-1])
    rng = np.random.default_rng(seed)
    q = torch.from_numpy(rng.standard_normal((T, w.Hq, w.d)).astype(np.float32)).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tq.prefill_attention(q.cuda(), cache, bt, torch.from_numpy(w.seq_lens).cuda(),
                               torch.from_numpy(q_start).cuda(), int(qlens.max()), w.scale,
                               k_tables=tables, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out.cpu().numpy()
    q_bits = bf16_bits(q)
    for b in range(w.B):
        rows = slice(int(q_start[b]), int(q_start[b + 1]))
        want = _oracle_prefill(orc, w, b, q_bits[rows], int(qlens[b]), oracle_tables, rotate)
        check_attention(got[rows], want, f"{w.name} b={b} q_len={qlens[b]}")
    return got


@pytest.mark.parametrize("name,over,qlens", [
    ("qwen3_8b_layer", dict(B=2, ctx=700), (130, 1)),          # d 128, GQA 4: 520 rows, 5 tiles
    ("prefill_small_head", dict(B=2, ctx=600), (200, 77)),     # d 64, GQA 8
    ("tiny", dict(B=1, ctx=100), (100,)),                      # the whole sequence is the chunk
    ("qwen3_8b_layer", dict(B=1, ctx=300, Hq=24), (50,)),      # GQA 3: tokens straddle tiles
    ("qwen3_8b_layer", dict(B=1, ctx=200, Hq=8), (160,)),      # GQA 1: 128 tokens per tile
    ("prefill_small_head", dict(B=3, ctx=333, Hq=2), (17, 64, 333)),  # d 64, GQA 1, ragged
])
def test_prefill_matches_oracle(tq, orc, name, over, qlens):
    _run_case(tq, orc, W.make(name, **over), qlens)


def test_prefill_calibrated_tables(tq, orc):
    w = W.make("qwen3_8b_layer", B=1, ctx=400)
    keys = w.calibration_keys(20)
    prod, orct = [], []
    for h in range(w.Hkv):
        p, _ = tq.fit_k_table(keys[h], tq.lloyd_max_table(w.d), 100)
        o, _ = orc.kmeans_table(orc.rotated_unit_samples(bf16_bits(keys[h])), orc.default_table(w.d), 100)
        prod.append(p)
        orct.append(o)
    assert np.array_equal(np.stack(prod), np.stack(orct))
    tables = torch.from_numpy(np.stack(prod)).cuda()
    _run_case(tq, orc, w, (64,), tables=tables, oracle_tables=np.stack(orct))


def test_prefill_one_token_chunk_equals_decode(tq, orc):
    """A chunk of one token is a decode step: both entry points agree (to their
    own rounding) on the same cache."""
    w = W.make("qwen3_8b_layer", B=3, ctx=500)
    cache, bt = _gpu_cache(tq, w)
    lens = torch.from_numpy(w.seq_lens).cuda()
    q = w.q().cuda()  # [B][Hq][d]: one token per sequence
    q_start = torch.arange(w.B + 1, dtype=torch.int32).cuda()
    pre = tq.prefill_attention(q, cache, bt, lens, q_start, 1, w.scale).cpu().numpy()
    dec = tq.decode_attention(q, cache, bt, lens, int(w.seq_lens.max()), w.scale).cpu().numpy()
    check_attention(pre, dec, "one-token chunk vs decode")


def test_prefill_bad_length_sets_status_and_zeros(tq):
    w = W.make("tiny", B=2, ctx=40)
    cache, bt = _gpu_cache(tq, w)
    lens = torch.tensor([40, 5], dtype=torch.int32, device="cuda")  # 5 < q_len 8: no valid context
    q_start = torch.tensor([0, 8, 16], dtype=torch.int32, device="cuda")
    q = torch.randn((16, w.Hq, w.d), device="cuda").to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tq.prefill_attention(q, cache, bt, lens, q_start, 8, w.scale, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tq.STATUS_BAD_LEN
    assert torch.all(out[8:] == 0) and torch.isfinite(out[:8]).all() and out[:8].abs().sum() > 0


@pytest.mark.parametrize("name,over,qlens", [
    ("tiny", dict(B=1, ctx=200), (130,)),                      # d 128, outlier channels
    ("prefill_small_head", dict(B=2, ctx=300), (77, 150)),     # d 64, GQA 8
])
def test_prefill_on_unrotated_cache(tq, orc, name, over, qlens):
    """TQ_CACHE_UNROTATED: the query is not rotated either; same oracle rule."""
    _run_case(tq, orc, W.make(name, **over), qlens, rotate=False)
