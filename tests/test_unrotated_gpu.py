"""GPU parity of the unrotated cache (TQ_CACHE_UNROTATED) and of the table-quality
study against the CPU oracle.

The unrotated cache quantises each key's unit vector directly ("TurboQuant 在 AMD
GPU 上把長上下文延遲壓下來", section 4, the baseline of the rotation); its records
must equal the oracle's byte for byte (the same rule as the rotated cache: a code
may differ only within 1e-6 of a decision threshold), and the decode, prefill and
dequantise over it must match the oracle's fp64 results.  The study's MSEs,
computed from the library's own append and dequantise kernels, must equal the
oracle's to ~1e-6 relative.
"""
import numpy as np
import pytest
import torch

import workloads as W
from test_parity_gpu import GpuState, OracleSeq, check_pairs
from test_quality_oracle import calibrated_tables, oracle_study

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over,calibrated", [
    ("tiny", dict(B=2, ctx=140), False),                 # d 128, four x20 channels per head
    ("qwen3_8b_layer", dict(B=2, ctx=300), False),       # d 128, heavy-tailed, shuffled blocks
    ("prefill_small_head", dict(B=2, ctx=333), False),   # d 64, GQA 8
    ("qwen3_8b_layer", dict(B=1, ctx=200), True),        # per-head tables
])
def test_unrotated_records_and_decode_match_oracle(tq, orc, name, over, calibrated):
    w = W.make(name, **over)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    check_pairs(tq, orc, w, pairs, calibrated=calibrated, rotate=False)


def test_unrotated_dequantize_matches_oracle(tq, orc):
    w = W.make("tiny", B=2, ctx=100)
    g = GpuState(tq, w, rotate=False)
    Kh, Vh = tq.dequantize(g.cache, g.bt, g.seq_lens, 104)
    Kh, Vh = Kh.cpu().numpy(), Vh.cpu().numpy()
    t = orc.default_table(w.d)
    for b in range(w.B):
        for h in range(w.Hkv):
            o = OracleSeq(orc, w, b, h, t, rotate=False)
            L = o.L
            scale = np.maximum(o.norms, 1e-30)[:, None]
            assert np.max(np.abs(Kh[b, :L, h] - o.Kh[0, :, 0]) / scale) < 1e-6
            assert np.max(np.abs(Vh[b, :L, h] - o.Vh[0, :, 0]) / (1 + np.abs(o.Vh[0, :, 0]))) < 1e-6
            assert np.all(Kh[b, L:] == 0) and np.all(Vh[b, L:] == 0)


def gpu_study(tq, w, b, T, tables=None, rotate=True):
    """(K MSE, V MSE) of tokens [0, T) of sequence b, coded by the library's append
    and dequantise kernels; the error sums are taken on the GPU in fp64."""
    K, V = w.kv(b, 0, T)
    Kd, Vd = K.cuda(), V.cuda()
    nblk = (T + 15) // 16
    cache = tq.Cache(nblk, w.Hkv, w.d, rotate=rotate)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kt = None if tables is None else torch.from_numpy(np.ascontiguousarray(tables)).cuda()
    tq.quantize_append(Kd, Vd, torch.arange(T, dtype=torch.int32, device="cuda"), cache, k_tables=kt,
                       status=st)
    bt = torch.arange(nblk, dtype=torch.int32, device="cuda")[None]
    Kh, Vh = tq.dequantize(cache, bt, torch.tensor([T], dtype=torch.int32, device="cuda"), T, k_tables=kt,
                           status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    Kf, Vf = Kd.double(), Vd.double()
    n2 = (Kf * Kf).sum(-1, keepdim=True)
    live = n2[..., 0] > 0
    k_mse = (((Kf - Kh[0].double()) ** 2) / torch.where(n2 > 0, n2, torch.ones_like(n2)))[live].mean()
    v_mse = ((Vf - Vh[0].double()) ** 2).mean()
    return float(k_mse), float(v_mse)


@pytest.mark.parametrize("name,over,T", [("tiny", {}, 256), ("qwen3_8b_layer", dict(B=2, ctx=512), 512),
                                         ("prefill_small_head", dict(B=1, ctx=1024), 1024)])
def test_quality_study_matches_oracle(tq, orc, name, over, T):
    """Lloyd-Max, re-fitted and unrotated key codings: the library's MSEs equal the
    oracle's (the records are the same; only the fp32 dequantisation differs)."""
    w = W.make(name, **over)
    b = w.B - 1  # the calibration keys come from sequence 0
    tabs = calibrated_tables(orc, w)
    for tables, rotate in ((None, True), (tabs, True), (None, False)):
        gk, gv = gpu_study(tq, w, b, T, tables, rotate)
        ok, ov = oracle_study(orc, w, b, T, tables, rotate)
        assert abs(gk / ok - 1) < 1e-5, (tables is not None, rotate, gk, ok)
        assert abs(gv / ov - 1) < 1e-5, (gv, ov)
