"""Test-side helpers: read the documented TQ4/4 record layout and compare the
GPU path with the oracle under the parity rule.

Parity rule (the TQ4/4 statement of what must match):
  - packed codes bit-exact, except elements whose oracle decision input lies
    within 1e-6 of a decision threshold (a centroid midpoint for keys, a .5
    rounding point of (v - z)/s for values); such mismatches are counted and
    must be at most 1e-5 of all elements;
  - fp16 norms, scales and zero points exact, except a norm within 1e-6
    (relative) of an fp16 rounding midpoint (counted the same way);
  - attention within max-abs 2e-3 and rel-L2 1e-3 of the oracle's fp64
    attention over its own dequantised K/V.
"""
from __future__ import annotations

import numpy as np
import torch

CODE_TOL = 1e-6
COUNT_TOL = 1e-5
ATTN_MAX_ABS = 2e-3
ATTN_REL_L2 = 1e-3


def layout(d):
    row = d // 2
    kn = 16 * row
    vc = kn + 32
    vs = vc + 16 * row
    return row, kn, vc, vs, vs + d, vs + 2 * d


def value_code_positions(d):
    """[16][d/2] offsets of value byte j of token t in the value-code area:
    (8 p + (j % 8 + 2 p) % 8) (d/8) + 4 ((j // 8) // 2) + 2 (t % 2) + (j // 8) % 2, p = t // 2."""
    t = np.arange(16)[:, None]
    j = np.arange(d // 2)[None, :]
    m, r, p = j // 8, j % 8, t // 2
    return (8 * p + (r + 2 * p) % 8) * (d // 8) + 4 * (m // 2) + 2 * (t % 2) + m % 2


def group_positions(d):
    """[16][d/32] byte offsets of the scale (zero) of token t, group G in its area:
    2 (4 (c (d/32) + G) + u) with c = (t % 8) // 2, u = 2 (t // 8) + t % 2."""
    t = np.arange(16)[:, None]
    G = np.arange(d // 32)[None, :]
    c, u = (t % 8) // 2, 2 * (t // 8) + t % 2
    return 2 * (4 * (c * (d // 32) + G) + u)


def unpack_record(rec: np.ndarray, d: int):
    """rec uint8 [record] -> kidx [16][d], knorm uint16 [16], vq [16][d], vs, vz uint16 [16][d/32]."""
    row, kn, vc, vs, vz, total = layout(d)
    assert rec.shape[-1] == total
    kc = rec[..., :kn].reshape(rec.shape[:-1] + (16, row))
    kidx = np.stack([kc & 15, kc >> 4], axis=-1).reshape(rec.shape[:-1] + (16, d))
    knorm = rec[..., kn:kn + 32].copy().view(np.uint16).reshape(rec.shape[:-1] + (16,))
    vcb = rec[..., vc:vs][..., value_code_positions(d)]  # natural [16][d/2] byte order
    vq = np.stack([vcb & 15, vcb >> 4], axis=-1).reshape(rec.shape[:-1] + (16, d))
    gp = group_positions(d)

    def u16(area):
        return area[..., gp].astype(np.uint16) | (area[..., gp + 1].astype(np.uint16) << 8)

    return kidx, knorm, vq, u16(rec[..., vs:vz]), u16(rec[..., vz:total])


def key_boundary_distance(ky: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Distance of each rotated unit coordinate to the nearest fp64 midpoint of the table."""
    t = table.astype(np.float64)
    mids = 0.5 * (t[:-1] + t[1:])
    return np.min(np.abs(ky[..., None] - mids), axis=-1)


def value_boundary_distance(vr: np.ndarray) -> np.ndarray:
    return np.abs(vr - (np.floor(vr) + 0.5))


def fp16_midpoint_rel_distance(n: np.ndarray) -> np.ndarray:
    """Relative distance of a positive norm to the nearest fp16 rounding midpoint."""
    n = np.asarray(n, np.float64)
    h = n.astype(np.float16).astype(np.float64)
    up = np.nextafter(n.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(n.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    mids = np.stack([(h + up) / 2, (h + dn) / 2], axis=-1)
    return np.min(np.abs(mids - n[..., None]), axis=-1) / np.maximum(n, 1e-300)


def bf16_values(lo_exp: int, hi_exp: int) -> np.ndarray:
    """Every positive bf16 value in [2^lo_exp, 2^hi_exp), ascending."""
    e = np.arange(lo_exp, hi_exp, dtype=np.float64)
    m = np.arange(128, dtype=np.float64)
    return ((1.0 + m[None, :] / 128.0) * 2.0 ** e[:, None]).ravel()


def near_threshold_pairs(d: int, table: np.ndarray, count: int, which: str):
    """Pairs (a, b) of positive bf16 values for two-entry keys k = a e_i + b e_j.

    The Sylvester rotation of such a key has coordinates (+-a +- b) / (|k| sqrt d),
    with |k| = sqrt(a^2 + b^2).  The pairs are ranked by how close those
    coordinates come to a midpoint of `table` (which="key"), or by how close
    |k| comes, relatively, to an fp16 rounding midpoint (which="norm"), and the
    `count` closest are returned with their distances.  a spans [1, 2), b spans
    [2^-8, 2): about 147 000 candidates, so the closest sit far inside 1e-6.
    """
    A, B = np.meshgrid(bf16_values(0, 1), bf16_values(-8, 1), indexing="ij")
    A, B = A.ravel(), B.ravel()
    n = np.sqrt(A * A + B * B)
    if which == "key":
        t = np.sort(table.astype(np.float64))
        mids = 0.5 * (t[:-1] + t[1:])
        dist = np.full(A.shape, np.inf)
        dist[A == B] = -1.0  # a = b: coordinates exactly 0, a tie pinned elsewhere; not taken
        for s in (1.0, -1.0):
            y = np.abs(A + s * B) / (n * np.sqrt(d))
            dist = np.minimum(dist, np.min(np.abs(y[:, None] - np.abs(mids)[None, :]), axis=1))
    elif which == "norm":
        dist = fp16_midpoint_rel_distance(n)
    else:
        raise ValueError(which)
    order = np.argsort(np.where(dist < 0, np.inf, dist), kind="stable")[:count]
    return A[order], B[order], dist[order]


def two_entry_keys(d: int, a: np.ndarray, b: np.ndarray, rng) -> np.ndarray:
    """fp32 keys [len(a)][d], key t = a[t] e_i + b[t] e_j (signs and i != j at random).

    a and b must be bf16 values, so the keys are exact in bf16."""
    K = np.zeros((len(a), d), np.float32)
    for t in range(len(a)):
        i, j = rng.choice(d, 2, replace=False)
        K[t, i] = a[t] * rng.choice((-1.0, 1.0))
        K[t, j] = b[t] * rng.choice((-1.0, 1.0))
    return K


def near_threshold_keys(d: int, table: np.ndarray, count: int, which: str, seed: int,
                        within: float = 1e-6, pool: int = 4096, max_pools: int = 64):
    """bf16-exact fp32 keys [count][d] with a rotated unit coordinate within `within` of
    a midpoint of `table` (which="key") or a norm within `within` (relative) of an fp16
    rounding midpoint (which="norm"), drawn from pools of N(0, 1) keys; the 8 closest
    two-entry keys of `near_threshold_pairs` come first.  Returns keys, distances."""
    rng = np.random.default_rng(seed)
    a, b, dist2 = near_threshold_pairs(d, table, 8, which)
    keys, dists = [two_entry_keys(d, a, b, rng)], [dist2]
    have = len(a)
    Hs = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(d)] for i in range(d)])
    t = np.sort(table.astype(np.float64))
    mids = 0.5 * (t[:-1] + t[1:])
    for _ in range(max_pools):
        if have >= count:
            break
        K = torch.from_numpy(rng.standard_normal((pool, d)).astype(np.float32)).to(
            torch.bfloat16).float().numpy()
        Kd = K.astype(np.float64)
        n = np.sqrt(np.sum(Kd * Kd, axis=1))
        if which == "key":
            y = (Kd @ Hs.T) / (n[:, None] * np.sqrt(d))
            dist = np.min(np.abs(y[..., None] - mids), axis=-1).min(axis=1)
        else:
            dist = fp16_midpoint_rel_distance(n)
        sel = np.flatnonzero(dist < within)[: count - have]
        keys.append(K[sel])
        dists.append(dist[sel])
        have += len(sel)
    return np.concatenate(keys)[:count], np.concatenate(dists)[:count]


class CodeReport:
    def __init__(self):
        self.elements = 0
        self.mismatch = 0
        self.far_mismatch = 0
        self.notes = []

    def add(self, got, want, dist, what):
        got = np.asarray(got)
        want = np.asarray(want)
        bad = got != want
        self.elements += got.size
        n = int(bad.sum())
        self.mismatch += n
        if n:
            far = bad & (np.broadcast_to(dist, got.shape) >= CODE_TOL)
            nf = int(far.sum())
            self.far_mismatch += nf
            self.notes.append(f"{what}: {n} mismatches ({nf} not near a threshold)")

    def check(self):
        assert self.far_mismatch == 0, "; ".join(self.notes)
        assert self.mismatch <= COUNT_TOL * max(1, self.elements), \
            f"{self.mismatch} near-threshold mismatches of {self.elements}: " + "; ".join(self.notes)
        return self.mismatch


def attn_errors(got: np.ndarray, want: np.ndarray):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    max_abs = float(np.max(np.abs(got - want))) if got.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(got - want) / den) if den > 0 else float(np.linalg.norm(got - want))
    return max_abs, rel


def check_attention(got, want, what=""):
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, \
        f"{what}: max-abs {max_abs:.3e} (<= {ATTN_MAX_ABS}), rel-L2 {rel:.3e} (<= {ATTN_REL_L2})"
    return max_abs, rel
