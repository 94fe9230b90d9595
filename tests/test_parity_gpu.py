"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Inputs come from the seeded generators in `workloads`; the oracle sees the
same bf16 tensors.  Small cases are compared exhaustively (every record byte,
every output); the full-size workloads, in the launch configuration that
bench.py times, are compared on sampled (sequence, kv head) pairs that the
oracle recomputes from scratch.
"""
import numpy as np
import pytest
import torch

import workloads as W
from parity_util import (CodeReport, check_attention, fp16_midpoint_rel_distance,
                         key_boundary_distance, near_threshold_keys, unpack_record,
                         value_boundary_distance)
from workloads import bf16_bits

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- GPU side
class GpuState:
    """A workload appended into a device cache through tq_quantize_append."""

    def __init__(self, tq, w, tables=None, rotate=True):
        self.tq, self.w = tq, w
        self.cache = tq.Cache(w.num_blocks, w.Hkv, w.d, rotate=rotate)
        self.bt = torch.from_numpy(w.block_tables).cuda()
        self.seq_lens = torch.from_numpy(w.seq_lens).cuda()
        self.tables_np = tables
        self.tables = None if tables is None else torch.from_numpy(np.ascontiguousarray(tables)).cuda()
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for K, V, slots in w.population():
            tq.quantize_append(K.cuda(), V.cuda(), slots.cuda(), self.cache, block_table=self.bt,
                               k_tables=self.tables, status=self.status)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0

    def decode(self, q=None, num_splits=0, scale=None):
        w = self.w
        q = (w.q() if q is None else q).cuda()
        out = self.tq.decode_attention(q, self.cache, self.bt, self.seq_lens, int(w.seq_lens.max()),
                                       w.scale if scale is None else scale, num_splits=num_splits,
                                       k_tables=self.tables, status=self.status)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0
        return out.cpu().numpy()

    def records(self, b, h):
        nblk = (int(self.w.seq_lens[b]) + 15) // 16
        ids = torch.from_numpy(self.w.block_tables[b, :nblk].astype(np.int64)).cuda()
        return self.cache.data[ids, h].cpu().numpy()


# ---------------------------------------------------------------- oracle side
class OracleSeq:
    """The oracle's encoding, dequantisation and attention for one (sequence, kv head)."""

    def __init__(self, orc, w, b, h, table, rotate=True):
        self.w, self.b, self.h = w, b, h
        L = int(w.seq_lens[b])
        K, V = w.kv(b)
        Kb = bf16_bits(K[:, h:h + 1].contiguous())
        Vb = bf16_bits(V[:, h:h + 1].contiguous())
        nblk = (L + 15) // 16
        self.table = np.ascontiguousarray(table)
        assert self.table.dtype == np.float16
        self.cache = np.zeros((nblk, 1, orc.record_bytes(w.d)), np.uint8)
        rc, self.ky, self.vr = orc.quantize_append(Kb, Vb, np.arange(L, dtype=np.int32), self.cache,
                                                   tables=self.table[None], want_aux=True, rotate=rotate)
        assert rc == 0
        bt = np.arange(nblk, dtype=np.int32)[None]
        self.Kh, self.Vh = orc.dequantize(self.cache, 1, w.d, bt, np.array([L], np.int32), L,
                                          tables=self.table[None], rotate=rotate)
        self.norms = np.linalg.norm(K[:, h].double().numpy(), axis=-1)
        self.L = L

    def attention(self, orc, q_bits_heads, scale):
        return orc.attention(q_bits_heads[None], self.Kh, self.Vh, np.array([self.L], np.int32), scale)[0]


def compare_records(report, got_rec, o: OracleSeq, d):
    L = o.L
    gk, gn, gv, gs, gz = unpack_record(got_rec, d)
    ok_, on, ov, os_, oz = unpack_record(o.cache[:, 0], d)
    flat = lambda x: x.reshape((-1,) + x.shape[2:])[:L]
    kd = key_boundary_distance(o.ky[:, 0], o.table)
    report.add(flat(gk), flat(ok_), kd, "key codes")
    vd = value_boundary_distance(o.vr[:, 0])
    report.add(flat(gv), flat(ov), vd, "value codes")
    nd = fp16_midpoint_rel_distance(o.norms)
    report.add(flat(gn), flat(on), nd, "key norms")
    # scales and zero points have no rounding freedom: exact
    assert np.array_equal(flat(gs), flat(os_)), "value scales differ"
    assert np.array_equal(flat(gz), flat(oz)), "value zero points differ"
    # padding rows of the last block stay untouched (zero)
    assert np.all(gk.reshape(-1, d)[L:] == 0) and np.all(gv.reshape(-1, d)[L:] == 0)


def table_for(w, tq, orc, calibrated=False):
    """(product tables [Hkv][16] or None, oracle tables [Hkv][16])."""
    if not calibrated:
        t = orc.default_table(w.d)
        return None, np.tile(t, (w.Hkv, 1))
    keys = w.calibration_keys(20)
    prod, orct = [], []
    for h in range(w.Hkv):
        init = tq.lloyd_max_table(w.d)
        p, _ = tq.fit_k_table(keys[h], init, 100)
        o, _ = orc.kmeans_table(orc.rotated_unit_samples(bf16_bits(keys[h])), orc.default_table(w.d), 100)
        prod.append(p)
        orct.append(o)
    return np.stack(prod), np.stack(orct)


def check_pairs(tq, orc, w, pairs, num_splits=0, calibrated=False, decode=True, rotate=True):
    prod_t, orc_t = table_for(w, tq, orc, calibrated)
    if calibrated:
        assert np.array_equal(prod_t, orc_t), "re-fitted tables differ between library and oracle"
    g = GpuState(tq, w, prod_t, rotate=rotate)
    out = g.decode(num_splits=num_splits) if decode else None
    q_bits = bf16_bits(w.q())
    report = CodeReport()
    for b, h in pairs:
        o = OracleSeq(orc, w, b, h, orc_t[h], rotate=rotate)
        compare_records(report, g.records(b, h), o, w.d)
        if decode:
            heads = slice(h * w.G, (h + 1) * w.G)
            want = o.attention(orc, q_bits[b, heads], w.scale)
            check_attention(out[b, heads], want, f"{w.name} b={b} h={h}")
    report.check()
    return g, report


# ---------------------------------------------------------------- small, exhaustive
def test_tiny_exhaustive(tq, orc):
    w = W.make("tiny")
    for S in (1, 3, 16):
        check_pairs(tq, orc, w, [(0, h) for h in range(w.Hkv)], num_splits=S)


def test_dequantize_matches_oracle(tq, orc):
    w = W.make("qwen3_8b_layer", B=2, ctx=333)
    g = GpuState(tq, w)
    Kh, Vh = tq.dequantize(g.cache, g.bt, g.seq_lens, 340)
    Kh, Vh = Kh.cpu().numpy(), Vh.cpu().numpy()
    t = orc.default_table(w.d)
    for b in range(w.B):
        for h in (0, 5):
            o = OracleSeq(orc, w, b, h, t)
            L = o.L
            scale = np.maximum(o.norms, 1e-30)[:, None]
            assert np.max(np.abs(Kh[b, :L, h] - o.Kh[0, :, 0]) / scale) < 2e-6
            assert np.max(np.abs(Vh[b, :L, h] - o.Vh[0, :, 0]) / (1 + np.abs(o.Vh[0, :, 0]))) < 1e-6
            assert np.all(Kh[b, L:] == 0) and np.all(Vh[b, L:] == 0)


@pytest.mark.parametrize("name,over,S", [
    ("qwen3_8b_layer", dict(B=3, ctx=1000), 0),       # ragged last block, shuffled tables
    ("qwen3_8b_layer", dict(B=2, ctx=777), 5),
    ("prefill_small_head", dict(B=3, ctx=1500), 0),   # d = 64, GQA 8
    ("long_context", dict(B=1, ctx=4100), 64),        # many splits, one partly empty
    ("tiny", dict(B=2, ctx=17), 2),                   # one full block plus one token
    ("qwen3_8b_layer", dict(B=2, ctx=300, Hq=8), 3),  # GQA 1
    ("qwen3_8b_layer", dict(B=2, ctx=300, Hq=16), 0), # GQA 2
    ("qwen3_8b_layer", dict(B=2, ctx=300, Hq=64), 2), # GQA 8 at d = 128
    ("prefill_small_head", dict(B=2, ctx=200, Hq=8), 1),  # GQA 4 at d = 64
    # d = 64 items of two groups of four heads, the second one partly or wholly used
    ("prefill_small_head", dict(B=2, ctx=333, Hq=10), 0),  # GQA 5: 4 + 1
    ("prefill_small_head", dict(B=2, ctx=250, Hq=12), 3),  # GQA 6: 4 + 2, splits
    ("prefill_small_head", dict(B=2, ctx=180, Hq=24), 0),  # GQA 12: items of 8 and 4 heads
    ("prefill_small_head", dict(B=1, ctx=520, Hq=32), 2),  # GQA 16: two items of 8 heads
    ("qwen3_8b_layer", dict(B=2, ctx=200, Hq=48), 0),      # GQA 6 at d = 128: 4 + 2
    ("qwen3_8b_layer", dict(B=2, ctx=150, Hq=24), 2),      # GQA 3 at d = 128
    # the largest GQA groups the library accepts: several 8-head items per kv head at d = 64,
    # 8 and 16 four-head items per kv head at d = 128
    ("prefill_small_head", dict(B=2, ctx=300, Hq=64), 0),   # GQA 32 at d = 64
    ("prefill_small_head", dict(B=1, ctx=260, Hq=128), 3),  # GQA 64 at d = 64
    ("qwen3_8b_layer", dict(B=2, ctx=180, Hq=32, Hkv=1), 2),  # GQA 32 at d = 128
    ("qwen3_8b_layer", dict(B=2, ctx=200, Hq=64, Hkv=1), 0),  # GQA 64 at d = 128
    # the most kv heads the cache accepts
    ("qwen3_8b_layer", dict(B=2, ctx=150, Hq=32, Hkv=16), 0),  # H_kv 16
    ("qwen3_8b_layer", dict(B=1, ctx=170, Hq=32, Hkv=32), 4),  # H_kv 32, GQA 1
    ("prefill_small_head", dict(B=2, ctx=140, Hq=64, Hkv=32), 0),  # H_kv 32 at d = 64
])
def test_reduced_configs(tq, orc, name, over, S):
    w = W.make(name, **over)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    check_pairs(tq, orc, w, pairs, num_splits=S)


@pytest.mark.parametrize("B,ctx,plans", [
    (3, 700, (5, 0, 3, 64, 1, 0, 7)),
    (8, 2000, (1024, 0, 1024, 9, 0)),  # 8000 one-block ranges with 1024 splits
])
def test_workspace_reused_across_plans(tq, orc, B, ctx, plans):
    """One workspace serves calls with different split plans back to back, holding the
    last call's partials: every partial a plan reads is written by the same call, so each
    result equals the one from a fresh workspace bit for bit (and the oracle's)."""
    w = W.make("qwen3_8b_layer", B=B, ctx=ctx)
    g = GpuState(tq, w)
    L = int(w.seq_lens.max())
    nbytes = max(tq.workspace_bytes(w.B, w.Hq, w.d, S) for S in plans)
    ws = torch.full((nbytes,), 0xff, dtype=torch.uint8, device="cuda")  # NaN floats to start
    q = w.q().cuda()
    for S in plans:
        fresh = tq.decode_attention(q, g.cache, g.bt, g.seq_lens, L, w.scale, num_splits=S)
        again = tq.decode_attention(q, g.cache, g.bt, g.seq_lens, L, w.scale, num_splits=S, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(fresh, again), f"num_splits {S}"
    q_bits = bf16_bits(w.q())
    t = orc.default_table(w.d)
    out = again.cpu().numpy()
    for b, h in ((0, 0), (w.B - 1, 7)):
        o = OracleSeq(orc, w, b, h, t)
        heads = slice(h * w.G, (h + 1) * w.G)
        check_attention(out[b, heads], o.attention(orc, q_bits[b, heads], w.scale), f"b={b} h={h}")


def test_calibrated_tables_for_32_kv_heads(tq, orc):
    """Per-head re-fitted tables at the most kv heads the cache takes: the append builds
    one bin table per head in shared memory, the decode one centroid table per head."""
    w = W.make("qwen3_8b_layer", B=2, ctx=120, Hq=64, Hkv=32)
    check_pairs(tq, orc, w, [(b, h) for b in range(w.B) for h in range(0, 32, 3)], calibrated=True)


def test_agentic_reduced_calibrated(tq, orc):
    w = W.make("agentic", B=4, prefix=700, suffix_max=400)
    check_pairs(tq, orc, w, [(b, h) for b in range(w.B) for h in (0, 3, 7)], calibrated=True)


def test_dense_custom_table_exact_count_path(tq, orc):
    """A table whose midpoints crowd one bin takes the exact counting path."""
    w = W.make("qwen3_8b_layer", B=1, ctx=200)
    base = orc.default_table(w.d).astype(np.float64)
    t = base.copy()
    t[7], t[8], t[9] = -1e-4, 0.0, 1e-4  # midpoints 7 and 8 fall in one bin
    t = t.astype(np.float16)
    assert np.all(np.diff(t) > 0)
    tables = np.tile(t, (w.Hkv, 1))
    g = GpuState(tq, w, tables)
    report = CodeReport()
    for h in (0, 4):
        o = OracleSeq(orc, w, 0, h, t)
        compare_records(report, g.records(0, h), o, w.d)
    report.check()


# ---------------------------------------------------------------- edge cases
def test_seq_len_zero_and_one(tq, orc):
    w = W.make("tiny", B=3, ctx=40)
    g = GpuState(tq, w)
    lens = torch.tensor([0, 1, 40], dtype=torch.int32, device="cuda")
    out = tq.decode_attention(w.q().cuda(), g.cache, g.bt, lens, 40, w.scale, num_splits=3).cpu().numpy()
    assert np.all(out[0] == 0)
    t = orc.default_table(w.d)
    for h in range(w.Hkv):
        o = OracleSeq(orc, w, 1, h, t)
        v0 = o.Vh[0, 0, 0]
        for gq in range(h * w.G, (h + 1) * w.G):
            assert np.max(np.abs(out[1, gq] - v0)) < 1e-5


def test_skip_slots_and_modes_agree(tq, orc):
    w = W.make("qwen3_8b_layer", B=2, ctx=64)
    K, V = w.kv(0)
    T = K.shape[0]
    bt = torch.from_numpy(w.block_tables).cuda()
    logical = torch.arange(T, dtype=torch.int32)
    logical[5] = -1
    phys = torch.tensor([-1 if s < 0 else int(w.block_tables[0, s // 16]) * 16 + s % 16 for s in logical.tolist()],
                        dtype=torch.int32)
    c1 = tq.Cache(w.num_blocks, w.Hkv, w.d)
    c2 = tq.Cache(w.num_blocks, w.Hkv, w.d)
    tq.quantize_append(K.cuda(), V.cuda(), logical.cuda(), c1, block_table=bt)
    tq.quantize_append(K.cuda(), V.cuda(), phys.cuda(), c2)
    torch.cuda.synchronize()
    assert torch.equal(c1.data, c2.data)
    rec = c1.data[int(w.block_tables[0, 0])].cpu().numpy()
    kidx, kn, vq, vs, vz = unpack_record(rec, w.d)
    assert np.all(kidx[:, 5] == 0) and np.all(kn[:, 5] == 0) and np.all(vs[:, 5] == 0)
    # T == 0 is a no-op
    tq.quantize_append(K[:0].cuda(), V[:0].cuda(), logical[:0].cuda(), c1, block_table=bt)


def test_bad_block_and_slot_set_status(tq):
    w = W.make("tiny", B=1, ctx=32)
    g = GpuState(tq, w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    K, V = w.kv(0, 0, 2)
    tq.quantize_append(K.cuda(), V.cuda(), torch.tensor([10 ** 6, 3], dtype=torch.int32, device="cuda"),
                       g.cache, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tq.STATUS_BAD_SLOT
    bad_bt = g.bt.clone()
    bad_bt[0, 1] = 10 ** 6
    st.zero_()
    tq.decode_attention(w.q().cuda(), g.cache, bad_bt, g.seq_lens, 32, w.scale, num_splits=1, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tq.STATUS_BAD_BLOCK
    st.zero_()
    lens = torch.tensor([10 ** 6], dtype=torch.int32, device="cuda")
    tq.decode_attention(w.q().cuda(), g.cache, g.bt, lens, 32, w.scale, num_splits=1, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & tq.STATUS_BAD_LEN


@pytest.mark.parametrize("d", [64, 128])
def test_out_of_range_inputs_set_status(tq, orc, d):
    """Inputs whose stored fields cannot hold them set TQ_STATUS_RANGE: a key whose norm
    exceeds 65504 (the largest fp16), a value group whose range needs a scale above 65504,
    a value group whose minimum rounds down past -65504, a NaN in a value and a NaN in a
    key.  Every other token's record still equals the oracle's byte for byte."""
    H, T = 2, 48
    rng = np.random.default_rng(31 + d)
    K = rng.standard_normal((T, H, d)).astype(np.float32)
    V = rng.standard_normal((T, H, d)).astype(np.float32)
    K[3, 0, 5] = 70000.0            # norm > 65504: the fp16 norm overflows
    V[5, 1, :32] = np.linspace(-1.0, 1.0e6, 32)  # (max - z) / 15 > 65504
    V[9, 0, 32:64] = -1.0e5         # z = fp16 rounded down from -1e5: overflows
    V[20, 1, 40] = np.nan           # a NaN among the values
    K[33, 0, 7] = np.nan            # a NaN among the keys
    flagged = {3, 5, 9, 20, 33}
    Kt = torch.from_numpy(K).to(torch.bfloat16)
    Vt = torch.from_numpy(V).to(torch.bfloat16)
    cache = tq.Cache(T // 16, H, d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.quantize_append(Kt.cuda(), Vt.cuda(), torch.arange(T, dtype=torch.int32).cuda(), cache, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == tq.STATUS_RANGE
    # one overflow at a time sets the bit too
    for t in sorted(flagged):
        c1 = tq.Cache(1, H, d)
        st.zero_()
        tq.quantize_append(Kt[t:t + 1].cuda(), Vt[t:t + 1].cuda(),
                           torch.zeros(1, dtype=torch.int32).cuda(), c1, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == tq.STATUS_RANGE, f"token {t}"
    # the oracle on the tokens it can encode (a NaN has no defined code)
    keep = np.array([t not in flagged for t in range(T)])
    slots = np.where(keep, np.arange(T), -1).astype(np.int32)
    ocache = np.zeros((T // 16, H, orc.record_bytes(d)), np.uint8)
    assert orc.quantize_append(bf16_bits(Kt), bf16_bits(Vt), slots, ocache)[0] == 0
    got = cache.data.cpu().numpy()
    for blk in range(T // 16):
        for h in range(H):
            a = unpack_record(got[blk, h], d)
            b = unpack_record(ocache[blk, h], d)
            rows = [r for r in range(16) if keep[16 * blk + r]]
            for name, x, y in zip(("kidx", "knorm", "vq", "vs", "vz"), a, b):
                assert np.array_equal(x[rows], y[rows]), f"blk {blk} head {h} {name}"


@pytest.mark.parametrize("d", [64, 128])
def test_value_and_key_edge_data(tq, orc, d):
    """Zero keys, constant and integer-valued value groups (exact .5 ties), huge ranges,
    groups whose (max - z)/15 is an fp16 value, groups whose max - z is inexact in fp32,
    and groups whose quotients lie 2^-20 off a .5 point."""
    H = 2
    T = 64
    rng = np.random.default_rng(5)
    K = rng.standard_normal((T, H, d)).astype(np.float32)
    V = rng.standard_normal((T, H, d)).astype(np.float32)
    K[0] = 0.0                                    # zero key: every code ties to 7
    K[1, :, :] = 0.0
    K[1, :, 0] = K[1, :, 1] = 1.0                 # exact zeros after rotation
    V[2] = 3.25                                   # constant group
    V[3] = np.round(rng.uniform(-8, 8, (H, d)))   # integers: exact .5 ties
    V[4] = np.tile(np.arange(32, dtype=np.float32), (H, d // 32))
    V[5] *= 1000.0
    V[5, :, 7] = 1e-3                             # wide dynamic range in one group
    K[6] *= 1e-20                                 # tiny norm
    K[9] *= 1e-20
    K[9, :, :16] = 0.0                            # tiny norm, one lane's elements all zero
    # z = -1, max - z = 1.875 = 15 * 0.125 (s exact in fp16), every other value on a .5 point
    V[7] = np.tile(-1.0 + 0.0625 * np.minimum(np.arange(32), 30), (H, d // 32))
    V[8] = rng.uniform(0.0, 1.0, (H, d))
    V[8, :, ::32] = 524288.0                      # max - z needs 29 bits: inexact in fp32
    V[8, :, 1::32] = 2.0 ** -10
    # minimum 2^-24, maximum 15/16, elements (2k + 1)/32: s = 1/16 and every quotient
    # 2^-20 below a .5 point (near-ties that round down)
    k15 = np.arange(15)
    near = np.concatenate([[2.0 ** -24, 15 / 16], (2 * k15 + 1) / 32, (2 * k15[::-1] + 1) / 32])
    V[10] = np.tile(near, (H, d // 32))
    V[11] = -np.tile(near[::-1], (H, d // 32))  # mirrored: minimum -15/16
    Kt = torch.from_numpy(K).to(torch.bfloat16)
    Vt = torch.from_numpy(V).to(torch.bfloat16)
    cache = tq.Cache(4, H, d)
    tq.quantize_append(Kt.cuda(), Vt.cuda(), torch.arange(T, dtype=torch.int32).cuda(), cache)
    torch.cuda.synchronize()
    ocache = np.zeros((4, H, orc.record_bytes(d)), np.uint8)
    rc, ky, vr = orc.quantize_append(bf16_bits(Kt), bf16_bits(Vt), np.arange(T, dtype=np.int32), ocache,
                                     want_aux=True)
    assert rc == 0
    got = cache.data.cpu().numpy()
    if not np.array_equal(got, ocache):
        msgs = []
        for blk in range(4):
            for h in range(H):
                a = unpack_record(got[blk, h], d)
                b = unpack_record(ocache[blk, h], d)
                for name, x, y in zip(("kidx", "knorm", "vq", "vs", "vz"), a, b):
                    bad = np.argwhere(x != y)
                    if bad.size:
                        t0 = tuple(bad[0])
                        msgs.append(f"blk {blk} head {h} {name}: {len(bad)} differ, first at {t0}: "
                                    f"gpu {x[t0]} oracle {y[t0]}")
        raise AssertionError("records differ:\n" + "\n".join(msgs[:12]))


@pytest.mark.parametrize("d,dense", [(64, False), (128, False), (128, True)],
                         ids=["d64", "d128", "d128-dense-table"])
def test_keys_near_decision_thresholds(tq, orc, d, dense):
    """Keys whose rotated unit coordinates lie within 1e-6 of a centroid midpoint (kv
    head 0) or whose norms lie within 1e-6 (relative) of an fp16 rounding midpoint,
    exact ties included (kv head 1): every one of them takes the append's exact
    re-decision.  The records must equal the oracle's byte for byte; a differing code
    or norm is accepted only below 1e-12 of its threshold, where the two sides' binary64
    rounding orders (y - C against product with the midpoint) may split a case."""
    T, H = 64, 2
    t = orc.default_table(d)
    if dense:  # midpoints 7 and 8 in one bin: the exact counting path
        t = t.astype(np.float64)
        t[7], t[8], t[9] = -1e-4, 0.0, 1e-4
        t = t.astype(np.float16)
    Kk, dk = near_threshold_keys(d, t, T, "key", seed=301 + d)
    Kn, dn = near_threshold_keys(d, t, T, "norm", seed=401 + d)
    K = np.stack([Kk, Kn], axis=1)
    V = np.random.default_rng(7).standard_normal((T, H, d)).astype(np.float32)
    Kt = torch.from_numpy(K).to(torch.bfloat16)
    Vt = torch.from_numpy(V).to(torch.bfloat16)
    assert torch.equal(Kt.float(), torch.from_numpy(K))  # the keys are bf16 values
    tables = np.tile(t, (H, 1))
    cache = tq.Cache(T // 16, H, d)
    tq.quantize_append(Kt.cuda(), Vt.cuda(), torch.arange(T, dtype=torch.int32).cuda(), cache,
                       k_tables=torch.from_numpy(np.ascontiguousarray(tables, np.float16)).cuda())
    torch.cuda.synchronize()
    ocache = np.zeros((T // 16, H, orc.record_bytes(d)), np.uint8)
    rc, ky, vr = orc.quantize_append(bf16_bits(Kt), bf16_bits(Vt), np.arange(T, dtype=np.int32),
                                     ocache, tables=tables, want_aux=True)
    assert rc == 0
    got = cache.data.cpu().numpy()
    if np.array_equal(got, ocache):
        return
    ky = ky.reshape(T, H, d)
    n = np.linalg.norm(Kt.double().numpy(), axis=-1)
    bad = []
    for blk in range(T // 16):
        for h in range(H):
            a = unpack_record(got[blk, h], d)
            b = unpack_record(ocache[blk, h], d)
            rows = slice(16 * blk, 16 * blk + 16)
            kd = key_boundary_distance(ky[rows, h], t)
            nd = fp16_midpoint_rel_distance(n[rows, h])
            for name, x, y, dist in zip(("kidx", "knorm", "vq", "vs", "vz"), a, b,
                                        (kd, nd, None, None, None)):
                for pos in np.argwhere(x != y):
                    pos = tuple(pos)
                    if dist is None or dist[pos] >= 1e-12:
                        bad.append(f"blk {blk} head {h} {name} {pos}: gpu {x[pos]} oracle {y[pos]}"
                                   + ("" if dist is None else f" distance {dist[pos]:.3e}"))
    assert not bad, "records differ:\n" + "\n".join(bad[:12])


# ---------------------------------------------------------------- full size, sampled
FULL = [
    ("qwen3_8b_layer", 0, False, [(0, 0), (13, 5), (31, 7)]),
    ("long_context", 64, False, [(0, 2), (3, 7)]),
    ("agentic", 0, True, [(0, 0), (17, 4), (31, 7)]),
    ("prefill_small_head", 0, False, [(0, 0), (9, 1), (15, 1)]),
]


@pytest.mark.parametrize("name,S,calibrated,pairs", FULL, ids=[f[0] for f in FULL])
def test_full_size_sampled(tq, orc, name, S, calibrated, pairs):
    w = W.make(name)
    g, report = check_pairs(tq, orc, w, pairs, num_splits=S, calibrated=calibrated)
    del g
    torch.cuda.empty_cache()
