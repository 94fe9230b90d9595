"""tq_append_decode: the append and the decode of one step in one launch.

The fused call must leave exactly the records that tq_quantize_append leaves
and return exactly what tq_decode_attention returns after it (the same kernels'
arithmetic, so the comparison is bit for bit), including the tokens the
append itself writes into the blocks being decoded.
"""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def _populated(tq, w, tables):
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d)
    bt = torch.from_numpy(w.block_tables).cuda()
    for K, V, s in w.population():
        tq.quantize_append(K.cuda(), V.cuda(), s.cuda(), cache, block_table=bt, k_tables=tables)
    torch.cuda.synchronize()
    return cache, bt


def _tables(tq, w, calibrated):
    if not calibrated:
        return None
    rng = np.random.default_rng(3)
    base = tq.lloyd_max_table(w.d).astype(np.float64)
    t = np.stack([np.sort(base * (1.0 + 0.05 * rng.standard_normal()) + 0.001 * h) for h in range(w.Hkv)])
    return torch.from_numpy(t.astype(np.float16)).cuda()


@pytest.mark.parametrize("name,over,S,calibrated", [
    ("qwen3_8b_layer", dict(B=4, ctx=1000), 0, False),
    ("qwen3_8b_layer", dict(B=3, ctx=777), 3, True),   # per-head tables: bins built on the device
    ("prefill_small_head", dict(B=3, ctx=900), 0, False),  # d = 64, GQA 8
    ("qwen3_8b_layer", dict(B=2, ctx=64, Hq=8), 1, False),  # one range per item
])
def test_fused_equals_separate_calls(tq, name, over, S, calibrated):
    w = W.make(name, **over)
    tables = _tables(tq, w, calibrated)
    L = int(w.seq_lens.max())
    aK, aV, aS = w.append_batch()  # the last append_tokens positions of every sequence
    aK, aV, aS = aK.cuda(), aV.cuda(), aS.cuda()
    q = w.q().cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    # separate calls on one cache, fused call on another; both start from the same population
    # with the appended positions overwritten by zero vectors, so what the decode sees there
    # can only come from the append under test
    cache_a, bt = _populated(tq, w, tables)
    cache_b, _ = _populated(tq, w, tables)
    for c in (cache_a, cache_b):
        tq.quantize_append(torch.zeros_like(aK), torch.zeros_like(aV), aS, c, block_table=bt,
                           k_tables=tables)
    tq.quantize_append(aK, aV, aS, cache_a, block_table=bt, k_tables=tables, status=st)
    want = tq.decode_attention(q, cache_a, bt, torch.from_numpy(w.seq_lens).cuda(), L, w.scale,
                               num_splits=S, k_tables=tables, status=st)
    got = tq.append_decode(aK, aV, aS, q, cache_b, bt, torch.from_numpy(w.seq_lens).cuda(), L, w.scale,
                           num_splits=S, append_block_table=bt, k_tables=tables, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(cache_a.data, cache_b.data)
    assert torch.equal(got, want)


def test_fused_sees_its_own_append(tq):
    """The appended tokens change the result: decoding a cache whose last positions
    were never written differs from the fused call, which writes them first."""
    w = W.make("qwen3_8b_layer", B=2, ctx=500)
    L = int(w.seq_lens.max())
    lens = torch.from_numpy(w.seq_lens).cuda()
    cache, bt = _populated(tq, w, None)
    aK, aV, aS = (x.cuda() for x in w.append_batch())
    # wipe the appended positions' records by appending zeros there first
    tq.quantize_append(torch.zeros_like(aK), torch.zeros_like(aV), aS, cache, block_table=bt)
    q = w.q().cuda()
    stale = tq.decode_attention(q, cache, bt, lens, L, w.scale)
    fused = tq.append_decode(aK, aV, aS, q, cache, bt, lens, L, w.scale, append_block_table=bt)
    again = tq.decode_attention(q, cache, bt, lens, L, w.scale)
    torch.cuda.synchronize()
    assert not torch.equal(stale, fused)
    assert torch.equal(fused, again)


def test_fused_degenerate_sizes(tq):
    w = W.make("tiny", B=1, ctx=40)
    cache, bt = _populated(tq, w, None)
    lens = torch.from_numpy(w.seq_lens).cuda()
    q = w.q().cuda()
    K, V = w.kv(0, 0, 2)
    slots = torch.tensor([3, 4], dtype=torch.int32, device="cuda")
    empty = torch.zeros((0, w.Hkv, w.d), dtype=torch.bfloat16, device="cuda")
    # T = 0: a plain decode
    want = tq.decode_attention(q, cache, bt, lens, 40, w.scale)
    got = tq.append_decode(empty, empty, torch.zeros(0, dtype=torch.int32, device="cuda"), q, cache, bt,
                           lens, 40, w.scale)
    assert torch.equal(got, want)
    # B = 0: a plain append (physical slots)
    c2, _ = _populated(tq, w, None)
    tq.quantize_append(K.cuda(), V.cuda(), slots, cache)
    q0 = torch.zeros((0, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    tq.append_decode(K.cuda(), V.cuda(), slots, q0, c2, bt[:0], lens[:0], 40, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(cache.data, c2.data)


def test_fused_call_replays_in_a_cuda_graph(tq):
    """Captured once and replayed, the fused call keeps its barrier: every replay
    appends before it decodes (each replay first rewrites the appended positions)."""
    w = W.make("qwen3_8b_layer", B=3, ctx=600)
    L = int(w.seq_lens.max())
    lens = torch.from_numpy(w.seq_lens).cuda()
    cache, bt = _populated(tq, w, None)
    aK, aV, aS = (x.cuda() for x in w.append_batch())
    zK, zV = torch.zeros_like(aK), torch.zeros_like(aV)
    q = w.q().cuda()
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(16, tq.workspace_bytes(w.B, w.Hq, w.d, 0)), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def step():
        tq.quantize_append(zK, zV, aS, cache, block_table=bt, stream=s)  # stale the positions
        tq.append_decode(aK, aV, aS, q, cache, bt, lens, L, w.scale, out=out, workspace=ws,
                         append_block_table=bt, status=st, stream=s)

    with torch.cuda.stream(s):
        step()
        s.synchronize()
        want = out.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            step()
        for _ in range(3):
            out.zero_()
            g.replay()
            s.synchronize()
            assert torch.equal(out, want)
    assert int(st.item()) == 0
