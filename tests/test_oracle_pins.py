"""Pins of the CPU oracle against what mathematics and published tables fix.

No value here comes from the CUDA path.  Each test ties one oracle function to
something independent of it: a library routine for a special case (numpy's
binary16, scipy's Hadamard matrix, scipy's normal distribution and
quadrature), a published table (Max 1960), a hand-derived worked example,
an invariant, or brute force on tiny inputs.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.special
import scipy.stats
import torch

from conftest import read_golden
from parity_util import near_threshold_keys

RNG = np.random.default_rng(12345)


def bf16_bits_of(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- scalar formats
def test_bf16_decode_matches_torch(orc):
    bits = RNG.integers(0, 1 << 16, size=4000).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite values only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([orc.bf16_to_double(b) for b in bits])
    assert np.array_equal(got, ref)


def _fp16_samples():
    xs = list(np.concatenate([
        RNG.standard_normal(3000) * 10.0 ** RNG.integers(-9, 6, 3000),
        np.ldexp(RNG.random(500), -RNG.integers(14, 26, 500)),  # subnormal range
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 70000.0, -1e9, 5.960464477539063e-08,
         2.9802322387695312e-08, 2.98023224e-08, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11],
    ]))
    return xs


def test_fp16_nearest_matches_numpy(orc):
    for x in _fp16_samples():
        got = orc.fp16_from_double(x, 0)
        with np.errstate(over="ignore"):
            ref = int(np.array([x], np.float64).astype(np.float16).view(np.uint16)[0])
        assert got == ref, (x, hex(got), hex(ref))


def test_fp16_directed_rounding_brackets(orc):
    for x in _fp16_samples():
        if abs(x) > 65504:
            continue
        dn = orc.fp16_from_double(x, -1)
        up = orc.fp16_from_double(x, +1)
        fdn = np.array([dn], np.uint16).view(np.float16)[0]
        fup = np.array([up], np.uint16).view(np.float16)[0]
        assert float(fdn) <= x <= float(fup)
        # adjacent: nothing representable strictly between the bracket and x
        with np.errstate(over="ignore"):
            assert float(np.nextafter(fdn, np.float16(np.inf))) > x or float(fdn) == x
            assert float(np.nextafter(fup, np.float16(-np.inf))) < x or float(fup) == x
        assert orc.fp16_to_double(dn) == float(fdn)
        assert orc.fp16_to_double(up) == float(fup)


def test_fp16_decode_all_finite_patterns(orc):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = bits.view(np.float16)
    fin = np.isfinite(f)
    got = np.array([orc.fp16_to_double(int(b)) for b in bits[fin][::7]])
    assert np.array_equal(got, f[fin][::7].astype(np.float64))


# ---------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128])
def test_hadamard_is_scipy_sylvester(orc, d):
    H = orc.hadamard(d)
    ref = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    assert np.array_equal(H, ref)
    assert np.allclose(H @ H, np.eye(d), atol=1e-14)  # symmetric and involutive


def test_hadamard_small_closed_forms(orc):
    s = 1 / math.sqrt(2)
    assert np.array_equal(orc.hadamard(2), np.array([[s, s], [s, -s]]))
    H = orc.hadamard(128)
    assert np.allclose(H[:, 0], np.full(128, 1 / math.sqrt(128)), atol=0)  # H e_0


# ---------------------------------------------------------------- Lloyd-Max
def test_lloyd_max_matches_max_1960(orc):
    c, iters = orc.lloyd_max_gaussian16()
    rows = read_golden("max1960_gaussian16.txt")
    levels = {int(r[1]): float(r[2]) for r in rows if r[0] == "level"}
    thr = {int(r[1]): float(r[2]) for r in rows if r[0] == "threshold"}
    for j in range(1, 9):
        # positive half: c[7+j]; negative half is the mirror
        assert abs(c[7 + j] - levels[j]) <= 5.1e-4 * max(1, levels[j]), (j, c[7 + j])
        assert abs(c[8 - j] + levels[j]) <= 5.1e-4 * max(1, levels[j])
    mids = 0.5 * (c[:-1] + c[1:])
    for j in range(1, 9):
        assert abs(mids[6 + j] - thr[j]) <= 5.1e-4 * max(1, thr[j]), (j, mids[6 + j])
    assert np.all(np.diff(c) > 0)
    assert np.allclose(c, -c[::-1], atol=1e-14)


def test_lloyd_max_is_a_fixed_point_by_quadrature(orc):
    """Each level equals the conditional mean of N(0,1) on its cell, by numerical integration."""
    c, _ = orc.lloyd_max_gaussian16()
    b = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    for j in range(16):
        mass = scipy.stats.norm.cdf(b[j + 1]) - scipy.stats.norm.cdf(b[j])
        mom, _ = scipy.integrate.quad(lambda x: x * scipy.stats.norm.pdf(x), b[j], b[j + 1],
                                      epsabs=1e-15, epsrel=1e-13)
        assert abs(mom / mass - c[j]) < 1e-9, j


def test_lloyd_max_distortion_by_quadrature(orc):
    c, _ = orc.lloyd_max_gaussian16()
    b = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    D = sum(scipy.integrate.quad(lambda x, cj=c[j]: (x - cj) ** 2 * scipy.stats.norm.pdf(x),
                                 b[j], b[j + 1], epsabs=1e-15)[0] for j in range(16))
    dist = float([r for r in read_golden("max1960_gaussian16.txt") if r[0] == "distortion"][0][2])
    assert abs(D - dist) < 1e-5
    # and the closed form for a centroid quantiser, E[X^2] - E[Q^2], agrees with the quadrature
    P = np.diff(scipy.stats.norm.cdf(b))
    assert abs((1.0 - np.sum(c ** 2 * P)) - D) < 1e-12


@pytest.mark.parametrize("d", [64, 128])
def test_default_table_scaled_by_sqrt_d(orc, d):
    c, _ = orc.lloyd_max_gaussian16()
    t = orc.default_table(d)
    assert t.dtype == np.float16
    assert np.array_equal(t, (c / math.sqrt(d)).astype(np.float16))


# ---------------------------------------------------------------- keys
def test_key_worked_example_e0(orc):
    g = {r[0]: r[1:] for r in read_golden("worked_examples.txt")}
    d = 128
    table = orc.default_table(d)
    k = np.zeros(d, np.float32)
    k[0] = 1.0
    idx, n16, y = orc.encode_k(bf16_bits_of(k), table)
    assert n16 == int(g["key_e0_norm16"][0], 16)
    assert np.all(idx == int(g["key_e0_code"][0]))
    assert np.allclose(y, 1 / math.sqrt(d), atol=1e-15)
    assert int(table.view(np.uint16)[11]) == int(g["key_e0_table11"][0], 16)
    khat = orc.decode_k(idx, n16, table)
    assert abs(khat[0] - float(g["key_e0_khat0"][0])) < 1e-6
    assert np.max(np.abs(khat[1:])) < 1e-12


def test_key_worked_example_exact_zero_ties_low(orc):
    g = {r[0]: r[1:] for r in read_golden("worked_examples.txt")}
    table = orc.default_table(128)
    k = np.zeros(128, np.float32)
    k[0] = k[1] = 1.0
    idx, n16, y = orc.encode_k(bf16_bits_of(k), table)
    assert n16 == int(g["key_e01_norm16"][0], 16)
    assert np.all(idx[0::2] == int(g["key_e01_even_code"][0]))
    assert np.all(y[1::2] == 0.0)
    assert np.all(idx[1::2] == int(g["key_e01_odd_code"][0]))


def test_key_zero_vector_ties_low(orc):
    table = orc.default_table(64)
    idx, n16, y = orc.encode_k(np.zeros(64, np.uint16), table)
    # y = 0 is exactly the midpoint of levels 7 and 8: the tie goes to the lower index
    assert np.all(idx == 7) and n16 == 0
    assert np.all(orc.decode_k(idx, n16, table) == 0.0)


@pytest.mark.parametrize("d", [64, 128])
def test_key_rotation_matches_scipy_and_keeps_norm(orc, d):
    table = orc.default_table(d)
    Hs = scipy.linalg.hadamard(d) / math.sqrt(d)
    for _ in range(20):
        kb = bf16_bits_of(RNG.standard_normal(d) * RNG.lognormal(0, 1, d))
        k = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).double().numpy()
        idx, n16, y = orc.encode_k(kb, table)
        assert np.allclose(y, Hs @ (k / np.linalg.norm(k)), atol=1e-14)
        assert abs(np.linalg.norm(y) - 1.0) < 1e-14
        assert n16 == int(np.float16(np.linalg.norm(k)).view(np.uint16))
        # brute force: the chosen level is at least as close as every other level
        dist = np.abs(y[:, None] - table[None, :].astype(np.float64))
        assert np.all(dist[np.arange(d), idx] <= dist.min(axis=1))


def _exact_code(N, nsq, d, mids):
    """Code of y = N / sqrt(nsq d) against sorted midpoints, all exact rationals:
    the count of midpoints strictly below y (a tie keeps the lower index), and
    whether y equals one of them.  y > m is decided on squares: N > m sqrt(nsq d)
    with both sides' signs known."""
    code, tie = 0, False
    for m in mids:
        tie |= (N > 0) == (m > 0) and N * N == m * m * nsq * d
        if m == 0:
            above = N > 0
        elif (N >= 0) != (m > 0):
            above = N >= 0  # opposite signs (or N = 0): y > m exactly when m < 0
        elif m > 0:
            above = N * N > m * m * nsq * d
        else:
            above = N * N < m * m * nsq * d
        code += above
    return code, tie


def _exact_fp16_of_sqrt(nsq):
    """fp16 nearest (ties to even) to sqrt(nsq), nsq an exact positive rational, and
    whether sqrt(nsq) lies exactly on the midpoint of two fp16 values."""
    lo = np.float16(math.sqrt(float(nsq)))
    while Fraction(float(lo)) ** 2 > nsq:
        lo = np.nextafter(lo, np.float16(-np.inf))
    while Fraction(float(np.nextafter(lo, np.float16(np.inf)))) ** 2 <= nsq:
        lo = np.nextafter(lo, np.float16(np.inf))
    hi = np.nextafter(lo, np.float16(np.inf))
    mid = (Fraction(float(lo)) + Fraction(float(hi))) / 2
    if nsq != mid * mid:
        return int((hi if nsq > mid * mid else lo).view(np.uint16)), False
    even = lo if int(lo.view(np.uint16)) % 2 == 0 else hi
    return int(even.view(np.uint16)), True


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("which", ["key", "norm"])
def test_key_decisions_near_thresholds_match_exact_arithmetic(orc, d, which):
    """bf16 keys chosen so that a rotated coordinate lies within 1e-6 of a centroid
    midpoint, or the norm within 1e-6 (relative) of an fp16 rounding midpoint (two-entry
    keys a e_i + b e_j searched for closeness, then N(0, 1) keys filtered).  With
    N = (S k)_i exact (S = scipy's +-1 Hadamard matrix) and nsq = |k|^2 exact, each
    coordinate y = N / sqrt(nsq d) is placed against the midpoints, and the norm
    sqrt(nsq) against the fp16 grid, in exact rational arithmetic on squares.  The
    oracle's binary64 codes and fp16 norms must agree wherever binary64 resolves the
    question (distance >= 1e-14) and wherever the exact value sits on the threshold (a
    tie: ties to even for the norm, to the lower index for a code).  Other cases
    closer than 1e-14 are the binary64 reading itself (the norm and coordinates are
    binary64 values before they are rounded or compared) and are only counted."""
    table = orc.default_table(d)
    t = np.sort(table.astype(np.float64))
    mids = [(Fraction(float(t[j])) + Fraction(float(t[j + 1]))) / 2 for j in range(15)]
    K, dist = near_threshold_keys(d, table, 40, which, seed=71 + d)
    assert len(K) == 40 and dist.max() < 1e-6
    S = scipy.linalg.hadamard(d)
    checked_near = unresolved = 0
    for k in K:
        idx, n16, y = orc.encode_k(bf16_bits_of(k), table)
        nz = np.flatnonzero(k)
        nsq = sum(Fraction(float(k[j])) ** 2 for j in nz)
        # norm
        n = math.sqrt(float(nsq))
        h = np.float16(n)
        cand = [np.nextafter(h, np.float16(-np.inf)), h, np.nextafter(h, np.float16(np.inf))]
        ndist = min(abs(n - (float(cand[i]) + float(cand[i + 1])) / 2) for i in range(2)) / n
        n_exact, n_tie = _exact_fp16_of_sqrt(nsq)
        if ndist >= 1e-14 or n_tie:
            assert n16 == n_exact, (k[nz], n16, n_tie)
            checked_near += which == "norm" and ndist < 1e-6
        else:
            unresolved += which == "norm"
        # codes: every coordinate
        for i in range(d):
            N = sum(int(S[i, j]) * Fraction(float(k[j])) for j in nz)
            kdist = float(np.min(np.abs(y[i] - np.asarray([float(m) for m in mids]))))
            code, tie = _exact_code(N, nsq, d, mids)
            if kdist >= 1e-14 or tie:
                assert idx[i] == code, (k[nz], i, y[i], idx[i], tie)
                checked_near += which == "key" and kdist < 1e-6
            else:
                unresolved += which == "key"
    # the selection reaches the thresholds: nearly every chosen key was decided within 1e-6
    assert checked_near >= 36, (checked_near, unresolved)


@pytest.mark.parametrize("d", [64, 128])
def test_key_relative_mse_matches_lloyd_max_distortion(orc, d):
    """For Gaussian keys the rotated unit coordinates are ~N(0, 1/d), so the relative
    reconstruction error is the quantiser distortion of N(0,1) (Max 1960: 0.009497)."""
    table = orc.default_table(d)
    errs = []
    for _ in range(1500):
        kb = bf16_bits_of(RNG.standard_normal(d))
        k = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).double().numpy()
        idx, n16, _ = orc.encode_k(kb, table)
        khat = orc.decode_k(idx, n16, table)
        errs.append(np.sum((k - khat) ** 2) / np.sum(k ** 2))
    mse = float(np.mean(errs))
    # the coordinates are Beta- rather than exactly Gaussian-distributed; a few % slack
    assert abs(mse - 0.009497) / 0.009497 < 0.04, mse


# ---------------------------------------------------------------- values
def test_value_worked_example_ramp(orc):
    g = {r[0]: r[1:] for r in read_golden("worked_examples.txt")}
    v = np.concatenate([np.arange(32, dtype=np.float32), np.arange(32, dtype=np.float32)])
    q, s, z, r = orc.encode_v(bf16_bits_of(v))
    assert int(z[0]) == int(g["value_ramp_zero16"][0], 16)
    assert int(s[0]) == int(g["value_ramp_scale16"][0], 16)
    assert list(q[:32]) == [int(x) for x in g["value_ramp_codes"]]


def test_value_error_bound_and_brute_force(orc):
    for trial in range(300):
        scale = 10.0 ** RNG.uniform(-3, 3)
        v = RNG.standard_t(4, 128) * scale + RNG.normal() * scale
        vb = bf16_bits_of(v)
        vd = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).double().numpy()
        q, s16, z16, r = orc.encode_v(vb)
        vh = orc.decode_v(q, s16, z16)
        for g in range(4):
            sl = slice(32 * g, 32 * g + 32)
            s = float(np.uint16(s16[g]).view(np.float16))
            z = float(np.uint16(z16[g]).view(np.float16))
            mn, mx = vd[sl].min(), vd[sl].max()
            # z is the largest fp16 <= min, s the smallest fp16 >= (max - z)/15
            assert z <= mn < float(np.nextafter(np.float16(z), np.float16(np.inf))) or z == mn
            assert s * 15 >= mx - z
            assert float(np.nextafter(np.float16(s), np.float16(-np.inf))) * 15 < mx - z
            assert np.all(np.abs(vd[sl] - vh[sl]) <= s / 2 * (1 + 1e-12))
            # brute force over the 16 grid points, ties to the even code
            cand = np.arange(16)[None, :] * s + z
            dist = np.abs(vd[sl][:, None] - cand)
            best = dist.min(axis=1, keepdims=True)
            ok = dist <= best
            for i in range(32):
                choices = np.nonzero(ok[i])[0]
                want = choices[0] if len(choices) == 1 else [c for c in choices if c % 2 == 0][0]
                assert q[32 * g + i] == want, (trial, g, i)
            assert q[32 * g + int(np.argmin(vd[sl]))] == 0
            assert q[32 * g + int(np.argmax(vd[sl]))] == 15


def test_value_constant_group_is_exact(orc):
    v = np.full(64, 3.25, np.float32)
    q, s, z, _ = orc.encode_v(bf16_bits_of(v))
    assert np.all(q == 0) and np.all(s == 0)
    assert np.all(orc.decode_v(q, s, z) == 3.25)


def test_value_near_ties_below_half_round_down(orc):
    """Worked example of near-ties: a group with minimum 2^-24, maximum 15/16 and the
    elements (2k + 1)/32 (all bf16 values).  z = fp16 down of 2^-24 = 2^-24 (0x0001),
    s = fp16 up of (15/16 - 2^-24)/15, just below 1/16, = 1/16 (0x2C00), and
    ((2k + 1)/32 - z)/s = k + 1/2 - 2^-20: 9.5e-7 below a .5 point, so every such
    element takes code k (an exact tie would send odd k up to k + 1)."""
    k = np.arange(15)
    v = np.concatenate([[2.0 ** -24, 15 / 16], (2 * k + 1) / 32, (2 * k[::-1] + 1) / 32])
    assert v.size == 32
    q, s, z, r = orc.encode_v(bf16_bits_of(v))
    assert int(z[0]) == 0x0001 and int(s[0]) == 0x2C00
    assert q[0] == 0 and q[1] == 15
    assert np.array_equal(q[2:17], k) and np.array_equal(q[17:], k[::-1])
    assert np.allclose(r[2:17], k + 0.5 - 2.0 ** -20, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- record format
def test_record_size_and_nibble_order(orc):
    g = {r[0]: r[1:] for r in read_golden("worked_examples.txt")}
    assert orc.record_bytes(128) == 2336 and orc.record_bytes(64) == 1184
    d = 128
    K = np.zeros((1, 1, d), np.float32)
    K[0, 0, 0] = 1.0
    V = np.tile(np.arange(32, dtype=np.float32), 4).reshape(1, 1, d)
    cache = np.zeros((2, 1, 2336), np.uint8)
    rc, _, _ = orc.quantize_append(bf16_bits_of(K), bf16_bits_of(V), np.array([16 + 5], np.int32),
                                   cache)
    assert rc == 0
    rec = cache[1, 0]
    assert np.all(cache[0] == 0)
    row = rec[5 * 64:6 * 64]
    assert np.all(row == int(g["key_e0_byte"][0], 16))
    assert int(rec[1024 + 10]) | (int(rec[1024 + 11]) << 8) == 0x3C00
    vc = rec[1056:1056 + 1024]
    chunk23 = [int(x, 16) for x in g["value_ramp_chunk23_d128"]]
    assert list(vc[23 * 16:24 * 16]) == chunk23
    odd_pos = [2, 3, 6, 7, 10, 11, 14, 15]
    for r in range(8):  # chunk 16 + (r + 4) % 8: 0x11*r at m-even, 0x11*(r+8) at m-odd positions
        c = 16 + (r + 4) % 8
        ch = vc[c * 16:(c + 1) * 16]
        assert list(ch[odd_pos]) == [0x11 * r, 0x11 * (r + 8)] * 4
        assert not np.any(np.delete(ch, odd_pos))
    # reading the bytes back in natural order gives the worked example's code bytes
    natural = [vc[(16 + (j % 8 + 4) % 8) * 16 + 4 * (j // 16) + 2 + (j // 8) % 2] for j in range(64)]
    want = [int(x, 16) for x in g["value_ramp_bytes"]]
    assert natural[:16] == want and natural[16:32] == want
    offs = [int(x) for x in g["value_ramp_group_offsets_d128"]]
    scale_area, zero_area = rec[2080:2208], rec[2208:2336]
    for o in offs:
        assert int(scale_area[o]) | (int(scale_area[o + 1]) << 8) == int(g["value_ramp_scale16"][0], 16)
        assert int(zero_area[o]) | (int(zero_area[o + 1]) << 8) == int(g["value_ramp_zero16"][0], 16)
    # every other byte is untouched
    mask = np.ones(2336, bool)
    mask[5 * 64:6 * 64] = False
    mask[1024 + 10:1024 + 12] = False
    for r in range(8):
        mask[1056 + (16 + r) * 16:1056 + (17 + r) * 16] = False
    for o in offs:
        mask[2080 + o:2080 + o + 2] = False
    assert np.all(rec[mask] == 0)


def _rand_kv(T, H, d, scale=1.0):
    K = bf16_bits_of(RNG.standard_normal((T, H, d)) * scale)
    V = bf16_bits_of(RNG.standard_normal((T, H, d)) * scale)
    return K, V


def test_append_slot_modes_and_skips_agree(orc):
    H, d, nb = 2, 64, 6
    K, V = _rand_kv(40, H, d)
    rec = orc.record_bytes(d)
    bt = np.array([[4, 1, 3], [0, 5, 2]], np.int32)
    # 20 tokens for each of 2 sequences, logical slots; -1 skips token 7
    logical = np.concatenate([np.arange(20), 48 + np.arange(20)]).astype(np.int32)
    logical[7] = -1
    phys = np.array([-1 if s < 0 else bt[s // 48, (s % 48) // 16] * 16 + s % 16 for s in logical],
                    np.int32)
    c1 = np.zeros((nb, H, rec), np.uint8)
    c2 = np.zeros((nb, H, rec), np.uint8)
    assert orc.quantize_append(K, V, logical, c1, block_table=bt)[0] == 0
    assert orc.quantize_append(K, V, phys, c2)[0] == 0
    assert np.array_equal(c1, c2)
    # the skipped token's slot (block 4, offset 7) stays zero
    assert np.all(c1[4, :, 7 * 32:8 * 32] == 0)


def test_dequantize_invariant_to_physical_permutation(orc):
    H, d, L = 2, 64, 70
    K, V = _rand_kv(L, H, d)
    rec = orc.record_bytes(d)
    nblk = (L + 15) // 16
    out = []
    for perm in (np.arange(nblk), RNG.permutation(nblk)):
        bt = perm.astype(np.int32)[None, :]
        cache = np.zeros((nblk, H, rec), np.uint8)
        orc.quantize_append(K, V, np.arange(L, dtype=np.int32), cache, block_table=bt)
        out.append(orc.dequantize(cache, H, d, bt, np.array([L], np.int32), L))
    assert np.array_equal(out[0][0], out[1][0]) and np.array_equal(out[0][1], out[1][1])


# ---------------------------------------------------------------- attention
def _attn_case(B=2, Hq=4, Hkv=2, d=64, L=37):
    q = bf16_bits_of(RNG.standard_normal((B, Hq, d)))
    Kh = RNG.standard_normal((B, L, Hkv, d))
    Vh = RNG.standard_normal((B, L, Hkv, d))
    return q, Kh, Vh


def test_attention_matches_scipy_softmax(orc):
    q, Kh, Vh = _attn_case()
    B, Hq, d = q.shape
    Hkv = Kh.shape[2]
    lens = np.array([37, 11], np.int32)
    out = orc.attention(q, Kh, Vh, lens, 0.125)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double().numpy()
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            a = 0.125 * Kh[b, :lens[b], kv] @ qd[b, h]
            ref = scipy.special.softmax(a) @ Vh[b, :lens[b], kv]
            assert np.allclose(out[b, h], ref, atol=1e-13)


def test_attention_special_cases(orc):
    q, Kh, Vh = _attn_case(B=1, Hq=2, Hkv=1, L=9)
    one = orc.attention(q, Kh, Vh, np.array([1], np.int32), 0.3)
    assert np.allclose(one[0], Vh[0, 0, 0][None, :], atol=1e-15)      # one token -> its value
    zero = orc.attention(q, Kh, Vh, np.array([9], np.int32), 0.0)
    assert np.allclose(zero[0], Vh[0, :, 0].mean(axis=0)[None, :], atol=1e-14)  # uniform weights
    Ks = np.repeat(Kh[:, :1], 9, axis=1)
    same = orc.attention(q, Ks, Vh, np.array([9], np.int32), 1.0)
    assert np.allclose(same[0], Vh[0, :, 0].mean(axis=0)[None, :], atol=1e-14)
    Kd = np.zeros_like(Kh)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double().numpy()
    Kd[0, 4, 0] = 1000.0 * qd[0, 0] / np.linalg.norm(qd[0, 0])
    dom = orc.attention(q[:, :1], Kd, Vh, np.array([9], np.int32), 1.0)
    assert np.allclose(dom[0, 0], Vh[0, 4, 0], atol=1e-12)             # one dominant score
    empty = orc.attention(q, Kh, Vh, np.array([0], np.int32), 1.0)
    assert np.all(empty == 0.0)


def test_attention_split_then_combine_equals_whole(orc):
    """Attention over disjoint token ranges, merged by their softmax masses
    (o = sum_s l_s o_s / sum_s l_s, l_s = sum over range s of exp(a_t - M)), equals the
    attention over the whole sequence: the identity a split-K decode relies on."""
    q, Kh, Vh = _attn_case(B=1, Hq=2, Hkv=1, L=61)
    scale = 0.7
    whole = orc.attention(q, Kh, Vh, np.array([61], np.int32), scale)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double().numpy()
    cuts = [0, 5, 6, 30, 61]  # ranges of 5, 1, 24 and 31 tokens
    for h in range(2):
        a = scale * Kh[0, :, 0] @ qd[0, h]
        M = a.max()
        o, l = 0.0, 0.0
        for c0, c1 in zip(cuts[:-1], cuts[1:]):
            part = orc.attention(q, Kh[:, c0:c1], Vh[:, c0:c1], np.array([c1 - c0], np.int32), scale)
            ls = np.exp(a[c0:c1] - M).sum()
            o, l = o + ls * part[0, h], l + ls
        assert np.allclose(o / l, whole[0, h], rtol=0, atol=1e-14)


def test_shared_prefix_tables_equal_private_copies(orc):
    """Two sequences whose first two blocks are one physical copy (block tables share
    them) dequantise, and attend, exactly as with private copies of those blocks."""
    H, d, L = 2, 64, 48
    K, V = _rand_kv(L, H, d)
    rec = orc.record_bytes(d)
    lens = np.array([L, L], np.int32)
    q = bf16_bits_of(RNG.standard_normal((2, 4, d)))

    def run(bt, seq1_positions):
        cache = np.zeros((int(bt.max()) + 1, H, rec), np.uint8)
        cap = bt.shape[1] * 16
        orc.quantize_append(K, V, np.arange(L, dtype=np.int32), cache, block_table=bt)
        p = np.asarray(seq1_positions)
        orc.quantize_append(K[p], V[p], (cap + p).astype(np.int32), cache, block_table=bt)
        Kh, Vh = orc.dequantize(cache, H, d, bt, lens, L)
        return Kh, Vh, orc.attention(q, Kh, Vh, lens, 0.125)

    shared = run(np.array([[0, 1, 2], [0, 1, 3]], np.int32), np.arange(32, L))
    private = run(np.array([[0, 1, 2], [4, 5, 3]], np.int32), np.arange(L))
    for x, y in zip(shared, private):
        assert np.array_equal(x, y)
    assert np.array_equal(shared[0][0], shared[0][1])  # both sequences hold the same tokens


@pytest.mark.parametrize("d", [64, 128])
def test_scores_in_rotated_domain_equal_original_domain(orc, d):
    """H is symmetric and orthonormal, so q . k_hat = (H q) . (n16 C[idx]): the scores can
    be taken against the stored centroids once the query is rotated (H from scipy)."""
    table = orc.default_table(d).astype(np.float64)
    Hs = scipy.linalg.hadamard(d) / math.sqrt(d)
    for _ in range(20):
        kb = bf16_bits_of(RNG.standard_normal(d) * 3.0)
        idx, n16, _ = orc.encode_k(kb, orc.default_table(d))
        khat = orc.decode_k(idx, n16, orc.default_table(d))
        qd = RNG.standard_normal(d)
        n = float(np.uint16(n16).view(np.float16))
        rot = (Hs @ qd) @ (n * table[idx])
        assert abs(qd @ khat - rot) <= 1e-12 * np.linalg.norm(qd) * np.linalg.norm(khat)


def test_attention_invariant_to_token_order(orc):
    q, Kh, Vh = _attn_case(B=1, L=30)
    p = RNG.permutation(30)
    a = orc.attention(q, Kh, Vh, np.array([30], np.int32), 0.2)
    b = orc.attention(q, Kh[:, p], Vh[:, p], np.array([30], np.int32), 0.2)
    assert np.allclose(a, b, atol=1e-14)


# ---------------------------------------------------------------- calibration
@pytest.mark.parametrize("d", [64, 128])
def test_rotated_unit_samples_are_hadamard_of_unit_keys(orc, d):
    """The calibration samples are the rotated unit keys y = H k / ||k|| (H = scipy's
    Sylvester matrix / sqrt(d)), row for row; a zero key gives zeros."""
    kb = bf16_bits_of(RNG.standard_t(4, (12, d)) * RNG.lognormal(0, 1, d))
    kb[5] = 0
    k = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).double().numpy()
    Hs = scipy.linalg.hadamard(d) / math.sqrt(d)
    n = np.linalg.norm(k, axis=1, keepdims=True)
    want = np.where(n > 0, (k / np.where(n > 0, n, 1)) @ Hs.T, 0.0)
    got = orc.rotated_unit_samples(kb)
    assert got.shape == (12, d)
    assert np.allclose(got, want, rtol=0, atol=1e-14)
    assert np.all(got[5] == 0)


def test_kmeans_table_lowers_mse_on_its_samples(orc):
    d = 128
    init = orc.default_table(d)
    kb = bf16_bits_of(RNG.standard_t(4, (20, d)) * RNG.lognormal(0, 1, d))
    y = orc.rotated_unit_samples(kb)
    assert np.allclose(np.linalg.norm(y, axis=1), 1.0, atol=1e-14)
    tab, it = orc.kmeans_table(y, init, 100)
    assert np.all(np.diff(tab) > 0)

    def mse(t):
        t = t.astype(np.float64)
        return np.mean(np.min((y.ravel()[:, None] - t[None, :]) ** 2, axis=1))

    assert mse(tab) <= mse(init) * (1 + 1e-3)  # Lloyd steps never raise the MSE (fp16 rounding aside)


def test_kmeans_on_gaussian_samples_reaches_lloyd_max_distortion(orc):
    """On many samples of N(0, 1/d), k-means from the Lloyd-Max table converges to a
    table whose distortion is no worse than Lloyd-Max's on those samples and not
    meaningfully better than the population optimum (Max 1960: 0.009497 sigma^2)."""
    d = 64
    init = orc.default_table(d)
    rng = np.random.default_rng(99)
    y = rng.standard_normal(400_000) / math.sqrt(d)
    tab, it = orc.kmeans_table(y, init, 1000)
    assert it < 1000 and np.all(np.diff(tab.astype(np.float64)) > 0)

    def mse(t):
        t = t.astype(np.float64)
        return np.mean(np.min((y[:, None] - t[None, :]) ** 2, axis=1)) * d

    assert mse(tab) <= mse(init) * (1 + 1e-4)
    assert 0.0095 * 0.98 <= mse(tab) <= 0.0095 * 1.02


@pytest.mark.parametrize("d", [64, 128])
def test_record_placement_round_trip(orc, d):
    """The oracle's placement of every field and the test-side reader (written
    separately from the documented formulas) agree on a record with every token,
    code, norm, scale and zero distinct enough to expose a swapped index."""
    from parity_util import unpack_record

    rec = orc.record_bytes(d)
    assert rec == 18 * d + 32
    r = np.random.default_rng(7)
    kidx = r.integers(0, 16, (16, d)).astype(np.uint8)
    vq = r.integers(0, 16, (16, d)).astype(np.uint8)
    kn = r.integers(0, 0x7bff, 16).astype(np.uint16)
    vs = r.integers(0, 0x7bff, (16, d // 32)).astype(np.uint16)
    vz = r.integers(0, 0xfbff, (16, d // 32)).astype(np.uint16)
    record = np.zeros(rec, np.uint8)
    for t in range(16):
        orc.pack_token(record, d, t, kidx[t], kn[t], vq[t], vs[t], vz[t])
    # every byte of the record is written by exactly one field of one token
    counts = np.zeros(rec, np.int64)
    for t in range(16):
        probe = np.zeros(rec, np.uint8)
        orc.pack_token(probe, d, t, np.full(d, 15, np.uint8), 0xffff, np.full(d, 15, np.uint8),
                       np.full(d // 32, 0xffff, np.uint16), np.full(d // 32, 0xffff, np.uint16))
        counts += probe == 0xff
    assert np.all(counts == 1)
    gk, gn, gv, gs, gz = unpack_record(record, d)
    assert np.array_equal(gk, kidx) and np.array_equal(gn, kn) and np.array_equal(gv, vq)
    assert np.array_equal(gs, vs) and np.array_equal(gz, vz)
    for t in range(16):
        k2, n2, v2, s2, z2 = orc.unpack_token(record, d, t)
        assert np.array_equal(k2, kidx[t]) and n2 == kn[t] and np.array_equal(v2, vq[t])
        assert np.array_equal(s2, vs[t]) and np.array_equal(z2, vz[t])


# ---------------------------------------------------------------- cache glue
def _glue_case(orc):
    """2 sequences x 3 kv heads at d 64, ragged lengths 37 and 50, shuffled
    physical blocks, three different per-head key tables: the default, one
    re-fitted by k-means, and the default scaled by 1.25 (still fp16-exact
    and strictly ascending)."""
    d, H = 64, 3
    r = np.random.default_rng(2024)
    lens = np.array([37, 50], np.int32)
    nblk = (lens + 15) // 16
    max_blocks = int(nblk.max()) + 1  # one spare column, never read
    perm = r.permutation(int(nblk.sum()) + 2).astype(np.int32)  # two physical blocks unused
    bt = np.full((2, max_blocks), -1, np.int32)
    bt[0, :nblk[0]] = perm[:nblk[0]]
    bt[1, :nblk[1]] = perm[nblk[0]:nblk[0] + nblk[1]]
    t0 = orc.default_table(d)
    kb = bf16_bits_of(r.standard_t(4, (20, d)))
    fitted, _ = orc.kmeans_table(orc.rotated_unit_samples(kb), t0, 100)
    scaled = (t0.astype(np.float64) * 1.25).astype(np.float16)
    tables = np.stack([t0, fitted, scaled]).astype(np.float16)
    assert not np.array_equal(tables[0], tables[1]) and not np.array_equal(tables[0], tables[2])
    T = int(lens.sum())
    K = bf16_bits_of(r.standard_normal((T, H, d)) * r.lognormal(0, 1, (1, H, d)))
    V = bf16_bits_of(r.standard_normal((T, H, d)) * 3.0)
    seq = np.repeat(np.arange(2), lens)
    pos = np.concatenate([np.arange(L) for L in lens])
    logical = (seq * max_blocks * 16 + pos).astype(np.int32)
    cache = np.zeros((len(perm), H, orc.record_bytes(d)), np.uint8)
    assert orc.quantize_append(K, V, logical, cache, tables=tables, block_table=bt)[0] == 0
    return dict(d=d, H=H, lens=lens, bt=bt, tables=tables, K=K, V=V, seq=seq, pos=pos,
                cache=cache, max_len=int(lens.max()) + 3)


def _expected_rows(orc, c):
    """Per (b, t, h): decode_k(encode_k(k, table[h])) and decode_v(encode_v(v)),
    the already pinned per-vector codecs, with no record, block or stride in between."""
    d, H = c["d"], c["H"]
    Ke = np.zeros((2, c["max_len"], H, d))
    Ve = np.zeros((2, c["max_len"], H, d))
    for i in range(len(c["seq"])):
        b, t = c["seq"][i], c["pos"][i]
        for h in range(H):
            idx, n16, _ = orc.encode_k(c["K"][i, h], c["tables"][h])
            Ke[b, t, h] = orc.decode_k(idx, n16, c["tables"][h])
            q, s, z, _ = orc.encode_v(c["V"][i, h])
            Ve[b, t, h] = orc.decode_v(q, s, z)
    return Ke, Ve


def _check_glue(c, Kh, Vh, Ke, Ve):
    """Every valid row equals the per-vector codecs' row (bit for bit); every row
    at or past a sequence's length is exactly 0."""
    for b, L in enumerate(c["lens"]):
        assert np.array_equal(Kh[b, :L], Ke[b, :L]), f"keys of sequence {b}"
        assert np.array_equal(Vh[b, :L], Ve[b, :L]), f"values of sequence {b}"
        assert np.all(Kh[b, L:] == 0) and np.all(Vh[b, L:] == 0), f"rows past length {L}"


def test_dequantize_with_per_head_tables_equals_per_vector_codecs(orc):
    """orc_dequantize and the per-head-table branch of orc_quantize_append, pinned
    against encode/decode of each vector alone (which are pinned to scipy, Max 1960,
    brute force and exact arithmetic above)."""
    c = _glue_case(orc)
    Ke, Ve = _expected_rows(orc, c)
    Kh, Vh = orc.dequantize(c["cache"], c["H"], c["d"], c["bt"], c["lens"], c["max_len"],
                            tables=c["tables"])
    _check_glue(c, Kh, Vh, Ke, Ve)
    # the records themselves, read by the test-side reader of the documented layout,
    # hold the per-vector codes of each head's own table
    from parity_util import unpack_record

    for i in range(len(c["seq"])):
        b, t = c["seq"][i], c["pos"][i]
        blk = c["bt"][b, t // 16]
        for h in range(c["H"]):
            kidx, kn, vq, vs, vz = unpack_record(c["cache"][blk, h], c["d"])
            idx, n16, _ = orc.encode_k(c["K"][i, h], c["tables"][h])
            q, s, z, _ = orc.encode_v(c["V"][i, h])
            assert np.array_equal(kidx[t % 16], idx) and kn[t % 16] == n16
            assert np.array_equal(vq[t % 16], q) and np.array_equal(vs[t % 16], s)
            assert np.array_equal(vz[t % 16], z)


def test_glue_check_catches_planted_mistakes(orc):
    """The check above fails under each plausible mistake of the glue, planted in
    the oracle's result here on the CPU: the token and head strides swapped, every
    head decoded with head 0's table, rows past the length left stale."""
    c = _glue_case(orc)
    Ke, Ve = _expected_rows(orc, c)
    d, H, ml = c["d"], c["H"], c["max_len"]
    Kh, Vh = orc.dequantize(c["cache"], H, d, c["bt"], c["lens"], ml, tables=c["tables"])
    # [b][t][h][d] written as [b][h][t][d]
    swapped = np.ascontiguousarray(Kh.transpose(0, 2, 1, 3)).reshape(Kh.shape)
    with pytest.raises(AssertionError):
        _check_glue(c, swapped, Vh, Ke, Ve)
    # head_table ignoring h
    Kw, Vw = orc.dequantize(c["cache"], H, d, c["bt"], c["lens"], ml,
                            tables=np.stack([c["tables"][0]] * H))
    with pytest.raises(AssertionError):
        _check_glue(c, Kw, Vw, Ke, Ve)
    # rows past the length not cleared (a buffer reused from a longer call)
    stale_K, stale_V = Kh.copy(), Vh.copy()
    stale_K[0, c["lens"][0]:] = 0.5
    with pytest.raises(AssertionError):
        _check_glue(c, stale_K, stale_V, Ke, Ve)


# ---------------------------------------------------------------- chunked prefill
def _prefill_case(orc, B=3, Hq=8, Hkv=2, d=64, Ls=(37, 20, 64), qlens=(5, 20, 1)):
    r = np.random.default_rng(77)
    max_len = max(Ls)
    q_start = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = bf16_bits_of(r.standard_normal((int(q_start[-1]), Hq, d)))
    Kh = r.standard_normal((B, max_len, Hkv, d))
    Vh = r.standard_normal((B, max_len, Hkv, d))
    return q, q_start, Kh, Vh, np.array(Ls, np.int32)


def test_prefill_rows_equal_decode_attention_at_their_positions(orc):
    """Each chunk token's output equals the (pinned) decode attention of that query
    over the cached tokens up to and including its own position."""
    q, q_start, Kh, Vh, L = _prefill_case(orc)
    scale = 1 / 8
    out = orc.prefill_attention(q, q_start, Kh, Vh, L, scale)
    for b in range(len(L)):
        qlen = q_start[b + 1] - q_start[b]
        for i in range(qlen):
            tok = q_start[b] + i
            n = L[b] - qlen + i + 1
            want = orc.attention(q[tok][None], Kh[b:b + 1], Vh[b:b + 1], np.array([n], np.int32), scale)[0]
            assert np.array_equal(out[tok], want), (b, i)


def test_prefill_is_causal_and_first_position_returns_first_value(orc):
    q, q_start, Kh, Vh, L = _prefill_case(orc, Ls=(20, 20, 64), qlens=(20, 3, 1))
    scale = 1 / 8
    out = orc.prefill_attention(q, q_start, Kh, Vh, L, scale)
    # sequence 0 is all chunk: its first token sees only position 0
    for h in range(8):
        assert np.allclose(out[0, h], Vh[0, 0, h // 4], atol=1e-15)
    # changing keys and values after a token's position leaves its output unchanged
    Kp, Vp = Kh.copy(), Vh.copy()
    Kp[0, 10:] += 5.0
    Vp[0, 10:] -= 3.0
    out2 = orc.prefill_attention(q, q_start, Kp, Vp, L, scale)
    assert np.array_equal(out[:10], out2[:10])  # tokens 0..9 of sequence 0
    assert not np.allclose(out[10:20], out2[10:20])


def test_prefill_matches_scipy_softmax(orc):
    q, q_start, Kh, Vh, L = _prefill_case(orc, B=1, Ls=(30,), qlens=(7,))
    scale = 0.3
    out = orc.prefill_attention(q, q_start, Kh, Vh, L, scale)
    qd = torch.tensor(q.view(np.int16)).view(torch.bfloat16).double().numpy()
    for i in range(7):
        n = 30 - 7 + i + 1
        for h in range(8):
            kv = h // 4
            a = scale * (Kh[0, :n, kv] @ qd[i, h])
            want = scipy.special.softmax(a) @ Vh[0, :n, kv]
            assert np.allclose(out[i, h], want, rtol=1e-12, atol=1e-13)
