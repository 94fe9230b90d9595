"""The allocation-free decode entry point, tq_decode_attention_static.

It serves callers that cannot allocate device memory (an operator hosted by
another runtime gets only its tensors; the host owns the rest of the memory),
so the split partials live in a fixed array inside the library instead of a
caller workspace.  This file is collected last on purpose: if it fails, a run
that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def _state(tq, w):
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d)
    bt = torch.from_numpy(w.block_tables).cuda()
    lens = torch.from_numpy(w.seq_lens).cuda()
    for K, V, slots in w.population():
        tq.quantize_append(K.cuda(), V.cuda(), slots.cuda(), cache, block_table=bt)
    torch.cuda.synchronize()
    return cache, bt, lens


def _call_static(tq, q, cache, bt, lens, L, scale, out, S, status):
    """Through the C ABI directly (ctypes), as a non-Python caller would."""
    lib = tq.load()
    return lib.tq_decode_attention_static(
        ctypes.c_void_p(q.data_ptr()), cache.c, None, ctypes.c_void_p(bt.data_ptr()), bt.shape[1],
        ctypes.c_void_p(lens.data_ptr()), q.shape[0], q.shape[1], L, ctypes.c_float(scale),
        ctypes.c_void_p(out.data_ptr()), S, ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,over,S", [
    ("qwen3_8b_layer", dict(B=3, ctx=1000), 5),
    ("prefill_small_head", dict(B=2, ctx=1500), 0),
])
def test_static_matches_workspace_entry_point_twice(tq, name, over, S):
    w = W.make(name, **over)
    cache, bt, lens = _state(tq, w)
    L = int(w.seq_lens.max())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(11)
    for call in range(2):  # two calls in a row, different queries, same shared scratch
        q = torch.from_numpy(rng.standard_normal((w.B, w.Hq, w.d)).astype(np.float32)).to(torch.bfloat16).cuda()
        want = tq.decode_attention(q, cache, bt, lens, L, w.scale, num_splits=S).cpu().numpy()
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
        rc = _call_static(tq, q, cache, bt, lens, L, w.scale, out, S, status)
        assert rc == tq.TQ_OK, tq.load().tq_last_error()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # the same plan and the same kernels, only another home for the partials:
        # the outputs must be identical bit for bit
        assert torch.equal(out.cpu(), torch.from_numpy(want)), f"{name} call {call}"


def test_static_rejects_plans_beyond_its_scratch(tq):
    lib = tq.load()
    cap = int(lib.tq_decode_static_scratch_bytes())
    assert cap == 8 << 20
    # 64 sequences x 32 heads x 64 splits x (128 floats + 2) = 68 MB of partials
    w = W.make("qwen3_8b_layer", B=1, ctx=64)
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d)
    B, Hq, S, L = 64, 32, 64, 64 * 16 * 64
    need = int(lib.tq_decode_workspace_bytes(B, Hq, 128, S))
    assert need > cap
    bt = torch.zeros((B, L // 16), dtype=torch.int32, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((B, Hq, 128), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = _call_static(tq, q, cache, bt, lens, L, 0.1, out, S, status)
    assert rc == tq.TQ_ERR_WORKSPACE
    assert b"scratch" in lib.tq_last_error()
    torch.cuda.synchronize()
    assert torch.all(out == 0)  # nothing was enqueued
