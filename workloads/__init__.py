"""Seeded synthetic inputs for the TQ4/4 append + decode path.

This module only draws random numbers and lays out block tables; it holds none
of the method's arithmetic.  Both the CUDA path (bench, GPU tests) and the CPU
oracle (tests, CPU baseline) take their inputs from here.

Every array is reproducible from (workload name, seed, sequence index):
each sequence has its own numpy PCG64 stream, so one sequence can be
regenerated on the host without drawing the others.

Workloads (shapes of the TQ4/4 decode and prefill settings studied on the
"TurboQuant 在 AMD GPU 上把長上下文延遲壓下來" and
"UltraQuant：4-bit KV 快取加速長代理" pages; the agentic one takes the shape of
their 32-way concurrent, ~25K-token-prefix agent runs):

  tiny                 1 seq x 256 tokens, 8 q / 2 kv heads, d 128, N(0,1) with
                       4 outlier channels per head scaled x20, seed 0
  qwen3_8b_layer       32 seqs x 8192 tokens, 32 q / 8 kv heads, d 128, shuffled
                       block tables, Student-t(4) x per-channel lognormal(0,1)
                       scales, seed 1; 32-token append per sequence
  long_context         4 seqs x 131072 tokens, 32 q / 8 kv, d 128, Student-t(4)
                       x lognormal scales, seed 2
  agentic              32 seqs sharing a 25,000-token prefix (shared physical
                       blocks) + private suffixes U[0, 15000], 32 q / 8 kv,
                       d 128, Student-t(4) x lognormal scales, calibrated table
                       from 20 sampled key vectors per head, seed 3
  prefill_small_head   16 seqs, 2048-token append chunks, 16 q / 2 kv heads
                       (GQA 8), d 64, N(0,1) with 2% of tokens x10, decode at
                       32768 tokens, seed 4
  iid_normal           1 seq x 4096 tokens, 32 q / 8 kv heads, d 128, plain
                       N(0,1) (keys uniform in direction: the reference case
                       of the table-quality study), seed 5
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK = 16
CHUNK = 4096          # tokens per random stream chunk
PREFIX_KEY = 1 << 20  # stream key of a shared prefix

# stream tags: np.random.default_rng([seed, TAG, ...])
_K, _V, _KSCALE, _VSCALE, _OUTLIER, _SPIKE, _Q, _TABLE, _SUFFIX, _CALIB, _PHYS = range(11)


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    seed: int
    dist: str                      # "normal_outlier" | "student_t" | "normal_spike" | "normal"
    seq_lens: np.ndarray           # int32 [B]
    block_tables: np.ndarray       # int32 [B][max_blocks]
    num_blocks: int
    shared_prefix: int = 0         # tokens whose full blocks are shared by every sequence
    append_tokens: int = 0         # per-sequence tokens re-appended each bench step
    chunk: int = 0                 # prefill chunk length (prefill_small_head)
    calibrate: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    # ------------------------------------------------------------ draws
    def _channel_scales(self, tag: int) -> np.ndarray:
        """lognormal(0,1) scale per (kv head, channel); ones for the Gaussian workloads."""
        if self.dist != "student_t":
            return np.ones((self.Hkv, self.d), np.float32)
        rng = np.random.default_rng([self.seed, tag])
        return rng.lognormal(0.0, 1.0, size=(self.Hkv, self.d)).astype(np.float32)

    def _outlier_mask(self) -> np.ndarray:
        m = np.ones((self.Hkv, self.d), np.float32)
        if self.dist == "normal_outlier":
            rng = np.random.default_rng([self.seed, _OUTLIER])
            for h in range(self.Hkv):
                m[h, rng.choice(self.d, size=4, replace=False)] = 20.0
        return m

    def _chunk(self, tag: int, key: int, c: int) -> np.ndarray:
        """Chunk c (tokens [c*CHUNK, (c+1)*CHUNK)) of stream (tag, key): float32 [CHUNK][Hkv][d]."""
        rng = np.random.default_rng([self.seed, tag, key, c])
        shape = (CHUNK, self.Hkv, self.d)
        n = CHUNK * self.Hkv * self.d
        z = rng.standard_normal(n, dtype=np.float32)
        if self.dist == "student_t":
            # t(4) = Z / sqrt(W/4), W ~ chi-square(4) = 2 (E1 + E2), E ~ Exp(1)
            w = rng.standard_exponential(n, dtype=np.float32)
            w += rng.standard_exponential(n, dtype=np.float32)
            w *= 0.5
            np.sqrt(w, out=w)
            z /= w
        z = z.reshape(shape)
        if self.dist == "normal_spike":
            spikes = rng.random(CHUNK) < 0.02  # 2% of tokens, whole token vector x10
            z[spikes] *= 10.0
        return z

    def _draw(self, tag: int, key: int, start: int, stop: int) -> np.ndarray:
        """Tokens [start, stop) of stream (tag, key), float32 [stop-start][Hkv][d]."""
        if stop <= start:
            return np.zeros((0, self.Hkv, self.d), np.float32)
        c0, c1 = start // CHUNK, (stop - 1) // CHUNK
        if c1 - c0 >= 4:  # long ranges: draw the chunks in parallel
            with ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
                parts = list(ex.map(lambda c: self._chunk(tag, key, c), range(c0, c1 + 1)))
        else:
            parts = [self._chunk(tag, key, c) for c in range(c0, c1 + 1)]
        full = parts[0] if len(parts) == 1 else np.concatenate(parts, axis=0)
        return full[start - c0 * CHUNK: stop - c0 * CHUNK]

    def _segment(self, tag: int, b: int, start: int, stop: int) -> np.ndarray:
        """Tokens [start, stop) of sequence b before per-channel scaling (float32).

        With a shared prefix, positions below it come from one prefix stream
        (the same for every sequence) and the rest from the sequence's own stream.
        """
        P = self.shared_prefix
        if not P:
            return self._draw(tag, b, start, stop)
        parts = []
        if start < P:
            parts.append(self._draw(tag, PREFIX_KEY, start, min(stop, P)))
        if stop > P:
            parts.append(self._draw(tag, b, max(start, P) - P, stop - P))
        return parts[0] if len(parts) == 1 else np.concatenate(parts, axis=0)

    def kv(self, b: int, start: int = 0, stop: int | None = None):
        """(K, V) bf16 tensors [stop-start][Hkv][d] for tokens [start, stop) of sequence b."""
        stop = int(self.seq_lens[b]) if stop is None else stop
        ks = self._channel_scales(_KSCALE) * self._outlier_mask()
        vs = self._channel_scales(_VSCALE) * self._outlier_mask()
        K = self._segment(_K, b, start, stop) * ks[None]
        V = self._segment(_V, b, start, stop) * vs[None]
        return (torch.from_numpy(np.ascontiguousarray(K)).to(torch.bfloat16),
                torch.from_numpy(np.ascontiguousarray(V)).to(torch.bfloat16))

    def q(self) -> torch.Tensor:
        rng = np.random.default_rng([self.seed, _Q])
        x = rng.standard_normal((self.B, self.Hq, self.d), dtype=np.float32)
        return torch.from_numpy(x).to(torch.bfloat16)

    def calibration_keys(self, n_vec: int = 20) -> torch.Tensor:
        """[Hkv][n_vec][d] bf16 key vectors drawn from sequence 0 (for a re-fitted table)."""
        rng = np.random.default_rng([self.seed, _CALIB])
        L = int(self.seq_lens[0])
        pos = np.sort(rng.choice(L, size=n_vec, replace=False))
        K, _ = self.kv(0)
        return K[torch.from_numpy(pos)].permute(1, 0, 2).contiguous()

    # ------------------------------------------------------------ population
    def population(self, max_tokens: int = 1 << 17):
        """Yield (K, V, logical_slots) batches that write every token of every sequence once.

        A logical slot is seq * (max_blocks * 16) + position; tokens of the
        shared prefix's full blocks are written through sequence 0 only.
        Pieces of at most CHUNK tokens are drawn in a thread pool and grouped
        into batches of at most max_tokens tokens.
        """
        cap = self.max_blocks * BLOCK
        shared_full = (self.shared_prefix // BLOCK) * BLOCK
        pieces = []
        for b in range(self.B):
            start = 0 if (b == 0 or not shared_full) else shared_full
            L = int(self.seq_lens[b])
            s = start
            while s < L:
                e = min(L, (s // CHUNK + 1) * CHUNK)
                pieces.append((b, s, e))
                s = e
        groups, batch, size = [], [], 0
        for p in pieces:
            n = p[2] - p[1]
            if batch and size + n > max_tokens:
                groups.append(batch)
                batch, size = [], 0
            batch.append(p)
            size += n
        if batch:
            groups.append(batch)

        def make(p):
            b, s, e = p
            K, V = self.kv(b, s, e)
            slots = torch.arange(s, e, dtype=torch.int32) + b * cap
            return K, V, slots

        with ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
            for g in groups:
                parts = list(ex.map(make, g))
                yield (torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts]),
                       torch.cat([p[2] for p in parts]))

    def append_batch(self):
        """The per-step append: the last `append_tokens` positions of every sequence."""
        cap = self.max_blocks * BLOCK

        def one(b):
            L = int(self.seq_lens[b])
            s = L - self.append_tokens
            K, V = self.kv(b, s, L)
            return K, V, torch.arange(s, L, dtype=torch.int32) + b * cap

        with ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
            parts = list(ex.map(one, range(self.B)))
        return (torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts]),
                torch.cat([p[2] for p in parts]))


def _shuffled_tables(seed: int, B: int, blocks_per_seq: np.ndarray, max_blocks: int,
                     num_blocks: int) -> np.ndarray:
    rng = np.random.default_rng([seed, _TABLE])
    perm = rng.permutation(num_blocks).astype(np.int32)
    tables = np.zeros((B, max_blocks), np.int32)
    o = 0
    for b in range(B):
        n = int(blocks_per_seq[b])
        tables[b, :n] = perm[o:o + n]
        o += n
    return tables


def make(name: str, **over) -> Workload:
    """Build a named workload; keyword overrides (B, ctx, ...) shrink it for tests."""
    if name == "tiny":
        B, Hq, Hkv, d, ctx, seed, dist = 1, 8, 2, 128, 256, 0, "normal_outlier"
    elif name == "qwen3_8b_layer":
        B, Hq, Hkv, d, ctx, seed, dist = 32, 32, 8, 128, 8192, 1, "student_t"
    elif name == "long_context":
        B, Hq, Hkv, d, ctx, seed, dist = 4, 32, 8, 128, 131072, 2, "student_t"
    elif name == "agentic":
        B, Hq, Hkv, d, ctx, seed, dist = 32, 32, 8, 128, 0, 3, "student_t"
    elif name == "prefill_small_head":
        B, Hq, Hkv, d, ctx, seed, dist = 16, 16, 2, 64, 32768, 4, "normal_spike"
    elif name == "iid_normal":
        B, Hq, Hkv, d, ctx, seed, dist = 1, 32, 8, 128, 4096, 5, "normal"
    else:
        raise KeyError(name)
    B = over.pop("B", B)
    ctx = over.pop("ctx", ctx)
    seed = over.pop("seed", seed)
    Hq = over.pop("Hq", Hq)
    Hkv = over.pop("Hkv", Hkv)
    extra = {}
    if name == "agentic":
        prefix = over.pop("prefix", 25000)
        suffix_max = over.pop("suffix_max", 15000)
        rng = np.random.default_rng([seed, _SUFFIX])
        suffix = rng.integers(0, suffix_max + 1, size=B)
        seq_lens = (prefix + suffix).astype(np.int32)
        shared_blocks = prefix // BLOCK
        blocks_per_seq = (seq_lens + BLOCK - 1) // BLOCK
        max_blocks = int(blocks_per_seq.max())
        private = blocks_per_seq - shared_blocks
        num_blocks = int(shared_blocks + private.sum())
        rng = np.random.default_rng([seed, _PHYS])
        perm = rng.permutation(num_blocks).astype(np.int32)
        tables = np.zeros((B, max_blocks), np.int32)
        shared_ids = perm[:shared_blocks]
        o = shared_blocks
        for b in range(B):
            tables[b, :shared_blocks] = shared_ids
            n = int(private[b])
            tables[b, shared_blocks:shared_blocks + n] = perm[o:o + n]
            o += n
        w = Workload(name, B, Hq, Hkv, d, seed, dist, seq_lens, tables, num_blocks,
                     shared_prefix=prefix, calibrate=True, extra=extra)
    else:
        seq_lens = np.full(B, ctx, np.int32)
        blocks_per_seq = (seq_lens + BLOCK - 1) // BLOCK
        max_blocks = int(blocks_per_seq.max())
        num_blocks = int(blocks_per_seq.sum())
        tables = _shuffled_tables(seed, B, blocks_per_seq, max_blocks, num_blocks)
        w = Workload(name, B, Hq, Hkv, d, seed, dist, seq_lens, tables, num_blocks, extra=extra)
        if name == "qwen3_8b_layer":
            w.append_tokens = min(32, ctx)
        if name == "prefill_small_head":
            w.chunk = over.pop("chunk", min(2048, ctx))
    if over:
        raise TypeError(f"unknown overrides {sorted(over)}")
    return w


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
