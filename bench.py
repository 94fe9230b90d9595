"""Benchmark of the TQ4/4 hot path on B200: quantise-append + paged split-K decode.

One step = one pass of the whole path over one batch of the Qwen3-8B-shaped
layer workload (32 sequences x 8192 tokens, 32 query / 8 kv heads, d 128):
tq_quantize_append of 32 new tokens per sequence (positions 8160..8191, so
the cache state is the same every step) followed by tq_decode_attention of
one query per sequence over all 8192 tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]

Rank 0 prints one JSON line.  value = quantised KV bytes the decode reads per
step x steps / timed seconds (GB/s), over the whole step (append included),
summed over ranks (each rank runs its own batch: weak scaling).  The cache
(306 MB per rank) is larger than L2 (126 MB), so no L2 flush is needed.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

WORKLOAD = "qwen3_8b_layer"
METRIC = "decode-attn quantised-KV GB/s & % of HBM peak; quantize-append tokens/s"


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak() -> float:
    """Dense bf16 TFLOP/s of this machine's B200s (burst), else the fallback figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def decode_bytes(w) -> int:
    """Algorithmic bytes of one decode launch: the quantised records of every
    valid token (record/16 per token-head), q, block tables read, output written."""
    import bit_rotated_kv_tq_b200 as tq

    rec = tq.record_bytes(w.d)
    tokens = int(w.seq_lens.sum())
    nblk = int(((w.seq_lens + 15) // 16).sum())
    return tokens * w.Hkv * rec // 16 + w.B * w.Hq * w.d * 2 + nblk * 4 + w.B * w.Hq * w.d * 4


def decode_kv_bytes(w) -> int:
    import bit_rotated_kv_tq_b200 as tq

    return int(w.seq_lens.sum()) * w.Hkv * tq.record_bytes(w.d) // 16


def append_bytes(w, T) -> int:
    import bit_rotated_kv_tq_b200 as tq

    return T * w.Hkv * (2 * w.d * 2 + tq.record_bytes(w.d) // 16) + T * 4


class ClockSampler:
    """SM clock and clock-event reasons, polled through NVML every ~1 ms by a
    thread while the timed region runs (read-only; no setting is changed).

    mark_start()/mark_end() bracket the timed region on the host clock; the
    summary uses the samples inside it, or the nearest ones when the region is
    shorter than a polling period."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, bus_id: str):
        self.bus_id = bus_id
        self.samples = []  # (host time, sm MHz, reason bits)
        self.t0 = self.t1 = None
        self.err = None

    def __enter__(self):
        import threading

        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(self.bus_id)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it, do not fail the bench
            self.err = f"nvml unavailable: {type(e).__name__}"
            return self
        self.stop = False

        def poll():
            while not self.stop:
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((time.perf_counter(), mhz, rs))
                except Exception:
                    pass
                time.sleep(0.001)

        self.th = threading.Thread(target=poll, daemon=True)
        self.th.start()
        time.sleep(0.02)  # a few samples before the region starts
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *a):
        if self.err is None:
            time.sleep(0.005)
            self.stop = True
            self.th.join(timeout=2)

    def summary(self):
        if self.err is not None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"]}
        inside = [s for s in self.samples if self.t0 <= s[0] <= self.t1]
        if not inside:  # region shorter than a polling period: the samples around it
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - self.t0), abs(s[0] - self.t1)))[:2]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [name for name, const in self.REASONS if bits & getattr(self.nv, const, 0)]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


def smi_id(local: int) -> str:
    """The NVML / nvidia-smi id (PCI bus id when torch exposes it) of local CUDA device `local`."""
    props = torch.cuda.get_device_properties(local)
    bus = getattr(props, "pci_bus_id", None)
    if bus is not None and getattr(props, "pci_domain_id", None) is not None:
        return f"{props.pci_domain_id:08x}:{bus:02x}:{getattr(props, 'pci_device_id', 0):02x}.0"
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


def dist_setup(n_gpus):
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, 0
    import datetime

    import torch.distributed as dist

    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return dist.get_rank(), dist.get_world_size(), local


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of x over all ranks (device timings are compared this way)."""
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank processed units_per_rank per step."""
    return world * units_per_rank * steps / max_seconds


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------- oracle timing
def oracle_sample(w, n_seqs: int):
    """Prepare the oracle's cache for the first n_seqs sequences (untimed)."""
    import oracle
    from workloads import bf16_bits

    oracle.build()
    L = int(w.seq_lens[0])
    nblk = (L + 15) // 16
    cache = np.zeros((n_seqs * nblk, w.Hkv, oracle.record_bytes(w.d)), np.uint8)
    bt = np.arange(n_seqs * nblk, dtype=np.int32).reshape(n_seqs, nblk)
    kv = [w.kv(b) for b in range(n_seqs)]
    Ks = np.concatenate([bf16_bits(k) for k, _ in kv])
    Vs = np.concatenate([bf16_bits(v) for _, v in kv])
    slots = np.concatenate([np.arange(L, dtype=np.int32) + b * nblk * 16 for b in range(n_seqs)])
    rc, _, _ = oracle.quantize_append(Ks, Vs, slots, cache, block_table=bt)
    assert rc == 0
    app = [w.kv(b, L - w.append_tokens, L) for b in range(n_seqs)]
    aK = np.concatenate([bf16_bits(k) for k, _ in app])
    aV = np.concatenate([bf16_bits(v) for _, v in app])
    aS = np.concatenate([np.arange(L - w.append_tokens, L, dtype=np.int32) + b * nblk * 16
                         for b in range(n_seqs)])
    q = bf16_bits(w.q()[:n_seqs])
    return dict(cache=cache, bt=bt, lens=np.full(n_seqs, L, np.int32), L=L, aK=aK, aV=aV, aS=aS, q=q)


def oracle_step(w, s):
    """One oracle pass over the sample: append its new tokens, then decode."""
    import oracle

    oracle.quantize_append(s["aK"], s["aV"], s["aS"], s["cache"], block_table=s["bt"])
    Kh, Vh = oracle.dequantize(s["cache"], w.Hkv, w.d, s["bt"], s["lens"], s["L"])
    return oracle.attention(s["q"], Kh, Vh, s["lens"], w.scale)


def cpu_model() -> str:
    """The host CPU's model name (/proc/cpuinfo), for the CPU-baseline record."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on a bounded sample."""
    if rank != 0:
        return
    w = W.make(WORKLOAD)
    n_seqs = 1
    s = oracle_sample(w, n_seqs)
    for _ in range(args.warmup):
        oracle_step(w, s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, s)
    dt = time.perf_counter() - t0
    kv_bytes = n_seqs * s["L"] * w.Hkv * (18 * w.d + 32) // 16
    value = kv_bytes * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": cfg(w, "oracle sample"),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": f"{n_seqs} of {w.B} sequences (all 8 kv heads, 8192 tokens, "
                                   f"32-token append) per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def profiled_traffic(w):
    """DRAM bytes (read + write) per launch of the decode split kernel, from the
    committed ncu summary, or None when the kernel source has changed since it was
    taken or the workload is not the one the figure was scaled to."""
    import hashlib

    prof = os.path.join(ROOT, "profiles", "decode_split_kernel_qwen3_8b_layer.md")
    src = os.path.join(ROOT, "bit_rotated_kv_tq_b200", "csrc", "tq_decode.cu")
    if not (os.path.exists(prof) and os.path.exists(src)):
        return None
    fields = {}
    with open(prof) as f:
        for ln in f:
            if ":" in ln and not ln.startswith(("|", " ", "#")):
                k, v = ln.split(":", 1)
                fields[k.strip()] = v.strip()
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    key = f"traffic_bytes_per_launch_b{w.B}"
    if fields.get("source_sha256") != sha or key not in fields or int(w.seq_lens[0]) != 8192:
        return None
    return int(fields[key])


def combine_runs(w, S, dev) -> bool:
    """Whether tq_decode_attention launches its combine kernel: some sequence is cut
    between two ranges of the split kernel's plan (the library's rule, restated)."""
    nmax = max(1, (int(w.seq_lens.max()) + 15) // 16)
    items = w.B * w.Hkv * ((w.Hq // w.Hkv + 3) // 4)
    V = items * nmax
    if S == 0:
        halves = 2 * torch.cuda.get_device_properties(dev).multi_processor_count
        R = max(1, -(-V // halves))
    else:
        R = max(1, -(-nmax // S))
    return -(-V // R) > 1 and R % nmax != 0


def cfg(w, l2):
    return {"workload": f"{w.name}: {w.B} seqs x {int(w.seq_lens[0])} tokens, {w.Hq} q / {w.Hkv} kv heads, "
                        f"d {w.d}, block 16, shuffled block tables, {w.append_tokens}-token append per seq",
            "global_batch": w.B, "seq_len": int(w.seq_lens[0]), "l2": l2}


# ---------------------------------------------------------------- the other workloads
def other_workloads(dev, peak, reps: int = 20) -> dict:
    """Device time per call (graphs of `reps` calls, CUDA events) of the scope
    table's other measured workloads, each on its own cache.  The long-context and
    agentic decodes read more than L2 per call; the prefill chunk and its cache fit
    in L2, so each of those calls follows a 512 MB read that evicts it, and the
    read's own time is subtracted.

    long_context: decode over 4 x 131072 tokens with 64 splits per item (and the
    even cut); agentic: decode over the shared-prefix batch with calibrated
    per-head tables, as logical bytes (what the sequences attend over) and unique
    bytes (distinct records); prefill_small_head: one 2048-token chunk appended to
    every sequence, and decode at context 32768; prefill_chunk_attention: the
    chunked-prefill attention of every sequence's second 2048-token chunk (context
    4096) on the tcgen05 tensor cores, as FLOP/s against the bf16 tensor peak."""
    import bit_rotated_kv_tq_b200 as tq

    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def graph_time(fn, n):
        """ms per fn() on the device: n calls captured as one CUDA graph, the median of
        three replays timed with CUDA events on the replay stream"""
        s_ = torch.cuda.Stream(dev)
        s_.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s_):
            fn()
            s_.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s_):
                for _ in range(n):
                    fn()
            g.replay()
            s_.synchronize()
            ts = []
            for _ in range(3):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s_)
                g.replay()
                e1.record(s_)
                s_.synchronize()
                ts.append(e0.elapsed_time(e1))
        del g
        return statistics.median(ts) / n

    def timed(fn, cold):
        """ms per call on the device, without the host's launch latency; with cold,
        every call follows an L2 flush (a 512 MB read) whose own time is subtracted"""
        if not cold:
            return graph_time(fn, reps)
        return graph_time(lambda: (flush.sum(), fn()), reps) - graph_time(lambda: flush.sum(), reps)

    def build(w, tables=None, bf16=False):
        cache = tq.Cache(w.num_blocks, w.Hkv, w.d, device=dev, bf16=bf16)
        bt = torch.from_numpy(w.block_tables).to(dev)
        for K, V, slots in w.population():
            tq.quantize_append(K.to(dev), V.to(dev), slots.to(dev), cache, block_table=bt,
                               k_tables=tables, status=status)
        return cache, bt

    def decode(w, cache, bt, S, tables=None, cold=False):
        lens = torch.from_numpy(w.seq_lens).to(dev)
        q = w.q().to(dev)
        max_len = int(w.seq_lens.max())
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
        ws = torch.empty(max(16, tq.workspace_bytes(w.B, w.Hq, w.d, S)), dtype=torch.uint8, device=dev)
        return timed(lambda: tq.decode_attention(q, cache, bt, lens, max_len, w.scale, out=out,
                                                 workspace=ws, num_splits=S, k_tables=tables,
                                                 status=status), cold)

    res = {}
    w = W.make("long_context")
    cache, bt = build(w)
    kv = decode_kv_bytes(w)
    for S in (64, 0):
        ms = decode(w, cache, bt, S)
        res[f"long_context_decode_s{S}"] = {"ms": ms, "gbs": kv / ms / 1e6, "hbm_frac": kv / ms / 1e6 / peak}
    del cache

    w = W.make("agentic")
    keys = w.calibration_keys(20)
    init = tq.lloyd_max_table(w.d)
    tables = torch.from_numpy(np.stack([tq.fit_k_table(keys[h], init, 100)[0] for h in range(w.Hkv)])).to(dev)
    cache, bt = build(w, tables)
    ms = decode(w, cache, bt, 0, tables)
    rec = tq.record_bytes(w.d)
    logical = decode_kv_bytes(w)
    nblk = (w.seq_lens + 15) // 16
    used = np.unique(np.concatenate([w.block_tables[b, :nblk[b]] for b in range(w.B)]))
    unique = int(used.size) * w.Hkv * rec
    res["agentic_decode"] = {"ms": ms, "logical_gbs": logical / ms / 1e6, "unique_gbs": unique / ms / 1e6,
                             "unique_hbm_frac": unique / ms / 1e6 / peak,
                             "logical_mb": logical / 1e6, "unique_mb": unique / 1e6}
    del cache

    w = W.make("prefill_small_head")
    cache, bt = build(w)
    cap = w.max_blocks * 16
    parts = [w.kv(b, 0, 2048) for b in range(w.B)]
    K = torch.cat([p[0] for p in parts]).to(dev)
    V = torch.cat([p[1] for p in parts]).to(dev)
    slots = torch.cat([torch.arange(0, 2048, dtype=torch.int32) + b * cap for b in range(w.B)]).to(dev)
    T = K.shape[0]
    ms = timed(lambda: tq.quantize_append(K, V, slots, cache, block_table=bt, status=status), True)
    ab = append_bytes(w, T)
    # what a plain device copy moving the same bytes (half read, half written) reaches
    # at this size, L2 evicted the same way: the ceiling of a streaming kernel this short
    cbuf = torch.randint(0, 256, (ab // 2 // 16 * 16,), dtype=torch.uint8, device=dev)
    cdst = torch.zeros_like(cbuf)
    cms = timed(lambda: cdst.copy_(cbuf), True)
    del cbuf, cdst
    res["prefill_chunk_append"] = {"ms": ms, "tokens": T, "tokens_per_s": T / ms * 1e3,
                                   "gbs": ab / ms / 1e6, "hbm_frac": ab / ms / 1e6 / peak,
                                   "same_bytes_copy_ms": cms, "same_bytes_copy_hbm_frac": ab / cms / 1e6 / peak}
    kv = decode_kv_bytes(w)
    ms = decode(w, cache, bt, 0, cold=True)
    res["prefill_small_head_decode"] = {"ms": ms, "gbs": kv / ms / 1e6, "hbm_frac": kv / ms / 1e6 / peak}
    del cache

    # the full-precision (bf16) cache that boundary layers keep, on the headline shape:
    # 32 x 8192 tokens x 8 kv heads of bf16 keys and values (1.07 GB, more than L2)
    w = W.make("qwen3_8b_layer")
    cache, bt = build(w, bf16=True)
    kv = int(w.seq_lens.sum()) * w.Hkv * 4 * w.d
    ms = decode(w, cache, bt, 0)
    res["bf16_decode"] = {"ms": ms, "kv_bytes": kv, "gbs": kv / ms / 1e6, "hbm_frac": kv / ms / 1e6 / peak}
    del cache

    # chunked-prefill attention (tcgen05): the second 2048-token chunk of every
    # prefill_small_head sequence, attending causally over positions 0 .. 4095;
    # algorithmic FLOPs = 4 d per (query head, key) pair (q.k and p.v)
    w = W.make("prefill_small_head", ctx=4096)
    cache, bt = build(w)
    qlen = 2048
    lens = torch.from_numpy(w.seq_lens).to(dev)
    q_start = (torch.arange(w.B + 1, dtype=torch.int32) * qlen).to(dev)
    rng = np.random.default_rng([w.seed, 99])
    q = torch.from_numpy(rng.standard_normal((w.B * qlen, w.Hq, w.d), dtype=np.float32)).to(torch.bfloat16).to(dev)
    out = torch.empty((w.B * qlen, w.Hq, w.d), dtype=torch.float32, device=dev)
    L = int(w.seq_lens[0])
    pairs = w.B * w.Hq * sum(L - qlen + i + 1 for i in range(qlen))
    flops = 4 * w.d * pairs
    ms = graph_time(lambda: tq.prefill_attention(q, cache, bt, lens, q_start, qlen, w.scale, out=out,
                                                 status=status), 5)
    tf_peak = measured_tensor_peak()
    res["prefill_chunk_attention"] = {"ms": ms, "tokens": w.B * qlen, "context": L,
                                      "tflops": flops / ms / 1e9, "tensor_frac": flops / ms / 1e9 / tf_peak,
                                      "tensor_peak_tflops": tf_peak}
    del cache
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    res["quality"] = quality_study(dev)
    return res


def sphere_coordinate_mse(table16: np.ndarray, d: int) -> float:
    """E[(y - C[nearest(y)])^2] for a coordinate y of a uniform unit vector in R^d
    (density proportional to (1 - y^2)^((d-3)/2)): the key error of Gaussian keys."""
    import scipy.integrate

    c = table16.view(np.float16).astype(np.float64)
    edges = np.concatenate([[-1.0], (c[:-1] + c[1:]) / 2, [1.0]])
    dens = lambda y: (1.0 - y * y) ** ((d - 3) / 2.0)
    Z = scipy.integrate.quad(dens, -1, 1, limit=400)[0]
    return sum(scipy.integrate.quad(lambda y, ci=ci: (y - ci) ** 2 * dens(y), edges[i], edges[i + 1],
                                    limit=400)[0] for i, ci in enumerate(c)) / Z


def quality_study(dev) -> dict:
    """Table-quality study on the library's own kernels: per-element K MSE of the unit
    key vector, ((k - k_hat) / ||k||)^2 averaged, for the Lloyd-Max table, tables
    re-fitted (tq_fit_k_table) on 20 calibration vectors per head, and the unrotated
    cache; V MSE (v - v_hat)^2.  Evaluated on sequences other than the calibration one."""
    import bit_rotated_kv_tq_b200 as tq

    out = {}
    cases = [("qwen3_8b_layer", dict(B=2, ctx=8192)), ("tiny", dict(B=2)),
             ("prefill_small_head", dict(B=2, ctx=8192)), ("iid_normal", dict(B=2))]
    for name, over in cases:
        w = W.make(name, **over)
        T = int(w.seq_lens[1])
        K, V = w.kv(1, 0, T)
        Kd, Vd = K.to(dev), V.to(dev)
        keys = w.calibration_keys(20)
        tabs = np.stack([tq.fit_k_table(keys[h], tq.lloyd_max_table(w.d), 100)[0] for h in range(w.Hkv)])
        nblk = (T + 15) // 16
        bt = torch.arange(nblk, dtype=torch.int32, device=dev)[None]
        lens = torch.tensor([T], dtype=torch.int32, device=dev)
        slots = torch.arange(T, dtype=torch.int32, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        Kf, Vf = Kd.double(), Vd.double()
        n2 = (Kf * Kf).sum(-1, keepdim=True)
        live = n2[..., 0] > 0
        row = {"tokens": T, "kv_heads": w.Hkv, "d": w.d, "dist": w.dist}
        for label, tables, rotate in (("lloyd_max", None, True), ("calibrated", tabs, True),
                                      ("unrotated", None, False)):
            cache = tq.Cache(nblk, w.Hkv, w.d, device=dev, rotate=rotate)
            kt = None if tables is None else torch.from_numpy(np.ascontiguousarray(tables)).to(dev)
            tq.quantize_append(Kd, Vd, slots, cache, k_tables=kt, status=st)
            Kh, Vh = tq.dequantize(cache, bt, lens, T, k_tables=kt, status=st)
            ek = ((Kf - Kh[0].double()) ** 2) / torch.where(n2 > 0, n2, torch.ones_like(n2))
            row["k_mse_" + label] = float(ek[live].mean())
            if label == "lloyd_max":
                row["v_mse"] = float(((Vf - Vh[0].double()) ** 2).mean())
                row["v_rel_mse"] = float(((Vf - Vh[0].double()) ** 2).sum() / (Vf * Vf).sum())
            del cache, Kh, Vh
        torch.cuda.synchronize(dev)
        assert int(st.item()) == 0, f"device status {int(st.item())}"
        row["calibrated_vs_lloyd_max"] = row["k_mse_calibrated"] / row["k_mse_lloyd_max"] - 1
        row["unrotated_vs_lloyd_max"] = row["k_mse_unrotated"] / row["k_mse_lloyd_max"] - 1
        row["k_mse_gaussian_keys"] = sphere_coordinate_mse(tq.lloyd_max_table(w.d), w.d)
        out[name] = row
    return out


def prefill_append_case(dev):
    """One 2048-token chunk appended to each of the 16 sequences of
    prefill_small_head (d 64, 2 kv heads), 3 warm-up calls then 1: the small,
    self-contained case the append kernel is profiled on."""
    import bit_rotated_kv_tq_b200 as tq

    tq.load()
    w = W.make("prefill_small_head")
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d, device=dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    cap = w.max_blocks * 16
    parts = [w.kv(b, 0, 2048) for b in range(w.B)]
    K = torch.cat([p[0] for p in parts]).to(dev)
    V = torch.cat([p[1] for p in parts]).to(dev)
    slots = torch.cat([torch.arange(0, 2048, dtype=torch.int32) + b * cap for b in range(w.B)]).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)
    for _ in range(4):
        flush.sum()
        tq.quantize_append(K, V, slots, cache, block_table=bt, status=status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    print(json.dumps({"case": "prefill_append", "tokens": K.shape[0], "ok": True}))


def prefill_attention_case(dev):
    """Chunked-prefill attention of the second 2048-token chunk of 4 prefill_small_head
    sequences (context 4096, d 64), 3 warm-up calls then 1: the case the tcgen05
    prefill kernel is profiled on."""
    import bit_rotated_kv_tq_b200 as tq

    tq.load()
    w = W.make("prefill_small_head", B=4, ctx=4096)
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d, device=dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for K, V, slots in w.population():
        tq.quantize_append(K.to(dev), V.to(dev), slots.to(dev), cache, block_table=bt, status=status)
    qlen = 2048
    lens = torch.from_numpy(w.seq_lens).to(dev)
    q_start = (torch.arange(w.B + 1, dtype=torch.int32) * qlen).to(dev)
    q = torch.randn((w.B * qlen, w.Hq, w.d), device=dev, generator=torch.Generator(dev).manual_seed(4)).to(
        torch.bfloat16)
    for _ in range(4):
        tq.prefill_attention(q, cache, bt, lens, q_start, qlen, w.scale, status=status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    print(json.dumps({"case": "prefill_attention", "ok": True}))


def prefill_decode_case(dev):
    """Decode over the prefill_small_head cache (16 x 32768 tokens, 16 q / 2 kv
    heads, d 64), 3 warm-up calls then 1, L2 flushed before each: the case the
    d 64 decode kernel is profiled on."""
    import bit_rotated_kv_tq_b200 as tq

    tq.load()
    w = W.make("prefill_small_head")
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d, device=dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for K, V, slots in w.population():
        tq.quantize_append(K.to(dev), V.to(dev), slots.to(dev), cache, block_table=bt, status=status)
    lens = torch.from_numpy(w.seq_lens).to(dev)
    q = w.q().to(dev)
    max_len = int(w.seq_lens.max())
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, tq.workspace_bytes(w.B, w.Hq, w.d, 0)), dtype=torch.uint8, device=dev)
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)
    for _ in range(4):
        flush.sum()
        tq.decode_attention(q, cache, bt, lens, max_len, w.scale, out=out, workspace=ws, status=status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    print(json.dumps({"case": "prefill_decode", "ok": True}))


def bf16_decode_case(dev):
    """Decode over the full-precision (bf16) cache of 8 qwen3_8b_layer sequences
    (8 x 8192 tokens, 8 kv heads, d 128: 268 MB of keys and values, more than L2),
    3 warm-up calls then 1: the case the bf16 decode kernel is profiled on."""
    import bit_rotated_kv_tq_b200 as tq

    tq.load()
    w = W.make("qwen3_8b_layer", B=8)
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d, device=dev, bf16=True)
    bt = torch.from_numpy(w.block_tables).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for K, V, slots in w.population():
        tq.quantize_append(K.to(dev), V.to(dev), slots.to(dev), cache, block_table=bt, status=status)
    lens = torch.from_numpy(w.seq_lens).to(dev)
    q = w.q().to(dev)
    for _ in range(4):
        tq.decode_attention(q, cache, bt, lens, int(w.seq_lens.max()), w.scale, status=status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    print(json.dumps({"case": "bf16_decode", "ok": True}))


# ---------------------------------------------------------------- GPU arm
def run_tq(args, rank, world, local):
    import bit_rotated_kv_tq_b200 as tq

    tq.load()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = W.make(WORKLOAD, B=args.batch) if args.batch else W.make(WORKLOAD)
    cache = tq.Cache(w.num_blocks, w.Hkv, w.d, device=dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.seq_lens).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for K, V, slots in w.population():
        tq.quantize_append(K.to(dev), V.to(dev), slots.to(dev), cache, block_table=bt, status=status)
    aK, aV, aS = w.append_batch()
    aK, aV, aS = aK.to(dev), aV.to(dev), aS.to(dev)
    q = w.q().to(dev)
    max_len = int(w.seq_lens.max())
    S = tq.default_splits(w.B, w.Hkv, max_len)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, tq.workspace_bytes(w.B, w.Hq, w.d, S)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    T = aK.shape[0]

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        tq.quantize_append(aK, aV, aS, cache, block_table=bt, status=status, stream=stream)
        if ev:
            ev[1].record(stream)
        tq.decode_attention(q, cache, bt, lens, max_len, w.scale, out=out, workspace=ws, num_splits=S,
                            status=status, stream=stream)
        if ev:
            ev[2].record(stream)

    torch.cuda.synchronize(dev)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"

    # per call: CUDA events around each library call, launched one by one from Python
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    barrier(world)
    app_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    dec_call = max_over_ranks(sum(dec_ms) / len(dec_ms), world)
    app_call = max_over_ranks(sum(app_ms) / len(app_ms), world)

    # the decode alone on the device: K calls captured as one CUDA graph and replayed,
    # CUDA events around the replay on its stream, so the host's launch latency (the
    # per-call events above include it) is not counted; 306 MB per call exceeds L2
    def graph_ms(fn):
        s_ = torch.cuda.Stream(dev)
        s_.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s_):
            fn(s_)
            s_.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s_):
                for _ in range(args.steps):
                    fn(s_)
            g.replay()
            s_.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier(world)
            e0.record(s_)
            g.replay()
            e1.record(s_)
            s_.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        del g
        return ms

    dec_avg = graph_ms(lambda s_: tq.decode_attention(q, cache, bt, lens, max_len, w.scale, out=out,
                                                      workspace=ws, num_splits=S, status=status,
                                                      stream=s_))
    # the append alone on the device, each call right after a 512 MB read that evicts
    # L2 (its inputs, 4.4 MB, would otherwise stay there over back-to-back calls):
    # graph-replayed (read + append) less graph-replayed reads
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)
    app_flush = graph_ms(lambda s_: (flush.sum(), tq.quantize_append(aK, aV, aS, cache, block_table=bt,
                                                                     status=status, stream=s_)))
    app_avg = app_flush - graph_ms(lambda s_: flush.sum())
    del flush

    # whole steps: the step (append, then decode) captured once as a CUDA graph, the way
    # a serving engine launches a decode step, and replayed; CUDA events around K replays
    gs = torch.cuda.Stream(dev)
    gs.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(gs):
        tq.quantize_append(aK, aV, aS, cache, block_table=bt, status=status, stream=gs)
        tq.decode_attention(q, cache, bt, lens, max_len, w.scale, out=out, workspace=ws, num_splits=S,
                            status=status, stream=gs)
        gs.synchronize()
        step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(step_graph, stream=gs):
            tq.quantize_append(aK, aV, aS, cache, block_table=bt, status=status, stream=gs)
            tq.decode_attention(q, cache, bt, lens, max_len, w.scale, out=out, workspace=ws,
                                num_splits=S, status=status, stream=gs)
        for _ in range(max(args.warmup, 3)):
            step_graph.replay()
        gs.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        with ClockSampler(smi_id(local)) as clk:
            clk.mark_start()
            start.record(gs)
            for _ in range(args.steps):
                step_graph.replay()
            end.record(gs)
            gs.synchronize()
            clk.mark_end()
    barrier(world)
    total_ms = max_over_ranks(start.elapsed_time(end), world)

    # end to end through the same public calls with host buffers, driven the way a
    # serving engine drives them: one CUDA graph per step.  Every step copies one set
    # of inputs in from pinned host memory and reads one result back.  The graph of
    # step k runs step k on the compute stream while it copies step k + 1's inputs
    # into the other device buffer set on a copy stream, then reads step k's result
    # back on a third stream; the timed region ends when the last read-back has landed.
    nbuf = 2
    h_q = w.q().pin_memory()
    h_K, h_V, h_S = aK.cpu().pin_memory(), aV.cpu().pin_memory(), aS.cpu().pin_memory()
    h_outs = [torch.empty((w.B, w.Hq, w.d), dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    d_in = [(torch.empty_like(q), torch.empty_like(aK), torch.empty_like(aV), torch.empty_like(aS))
            for _ in range(nbuf)]
    d_out = [torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev) for _ in range(nbuf)]
    cs = torch.cuda.Stream(dev)  # the stream the graphs are captured and replayed on
    copy_s, read_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def copy_in(i):
        d_q, d_K, d_V, d_S = d_in[i]
        d_q.copy_(h_q, non_blocking=True)
        d_K.copy_(h_K, non_blocking=True)
        d_V.copy_(h_V, non_blocking=True)
        d_S.copy_(h_S, non_blocking=True)

    def read_out(i):
        with torch.cuda.stream(read_s):
            h_outs[i].copy_(d_out[i], non_blocking=True)

    def step_body(i):  # captured: step on set i, next step's inputs into set 1 - i,
        # and the previous step's result (set 1 - i) read back, both beside the step
        copy_s.wait_stream(cs)
        with torch.cuda.stream(copy_s):
            copy_in(1 - i)
        read_s.wait_stream(cs)
        read_out(1 - i)
        d_q, d_K, d_V, d_S = d_in[i]
        tq.quantize_append(d_K, d_V, d_S, cache, block_table=bt, status=status, stream=cs)
        tq.decode_attention(d_q, cache, bt, lens, max_len, w.scale, out=d_out[i], workspace=ws,
                            num_splits=S, status=status, stream=cs)
        cs.wait_stream(copy_s)  # the graph ends when both side branches are done, so the
        cs.wait_stream(read_s)  # next step may reuse what they read and write

    cs.wait_stream(torch.cuda.current_stream(dev))
    graphs = []
    with torch.cuda.stream(cs):
        for i in range(nbuf):
            copy_in(i)  # every buffer set holds real inputs before any step reads one
        for i in range(nbuf):
            step_body(i)  # once outside capture (first-use setup of the library)
        cs.synchronize()
        for i in range(nbuf):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cs):
                step_body(i)
            graphs.append(g)
        copy_in(0)
        for k in range(4):
            graphs[k % nbuf].replay()
        cs.synchronize()
        barrier(world)
        t0 = time.perf_counter()
        # steps 0 .. K-1; graph k reads back step k - 1's result, and the last result
        # is read back after the loop, inside the timed region
        for k in range(args.steps):
            graphs[k % nbuf].replay()
        read_s.wait_stream(cs)
        read_out((args.steps - 1) % nbuf)
        read_s.synchronize()
        cs.synchronize()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world)
    torch.cuda.synchronize(dev)
    # the read-back results are the device-timed path's (same inputs, same cache state)
    assert torch.equal(h_outs[(args.steps - 1) % nbuf], out.cpu()), "end-to-end result differs"
    assert torch.equal(h_outs[(args.steps - 2) % nbuf], out.cpu()), "end-to-end result differs"
    h2d = h_q.numel() * 2 + h_K.numel() * 2 + h_V.numel() * 2 + h_S.numel() * 4
    d2h = h_outs[0].numel() * 4
    # the host link alone: one step's input copies with nothing else running, the floor
    # under the end-to-end step time
    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(copy_s):
        copy_in(0)
        l0.record(copy_s)
        for _ in range(5):
            copy_in(0)
        l1.record(copy_s)
    copy_s.synchronize()
    h2d_link_gbs = h2d * 5 / (l0.elapsed_time(l1) / 1e3) / 1e9

    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"

    kv = decode_kv_bytes(w)
    value = weak_scaling_value(kv, args.steps, world, total_ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    dec_bytes = decode_bytes(w)
    achieved = dec_bytes / (dec_avg / 1e3) / 1e9
    clocks = clk.summary()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        s = oracle_sample(w, 1)
        oracle_step(w, s)
        # passes until about 10 s of CPU work (at least 3, at most 60)
        n_rep = 0
        t0 = time.perf_counter()
        while n_rep < 3 or (n_rep < 60 and time.perf_counter() - t0 < 10.0):
            oracle_step(w, s)
            n_rep += 1
        dt = (time.perf_counter() - t0) / n_rep
        cpu = {"value": s["L"] * w.Hkv * tq.record_bytes(w.d) // 16 / dt / 1e9, "unit": "GB/s", "cores": 1,
               "kind": "oracle", "cpu_model": cpu_model(),
               "sample": f"1 of {w.B} sequences (8 kv heads x {s['L']} tokens + {w.append_tokens}-token append), "
                         f"{n_rep} passes, {dt:.2f} s each"}

    others = None
    if rank == 0 and world == 1 and not args.no_workloads:
        others = other_workloads(dev, peak)
        # the same decode over the full-precision cache, against this one
        others["bf16_decode"]["tq_speedup"] = others["bf16_decode"]["ms"] / dec_avg

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": cfg(w, f"inputs larger than L2: {kv / 1e6:.0f} MB cache read per rank vs 126 MB L2, no flush"),
            "decode_gbs": kv / (dec_avg / 1e3) / 1e9,
            "decode_hbm_frac": kv / (dec_avg / 1e3) / 1e9 / peak,
            "decode_ms": dec_avg, "append_ms": app_avg, "decode_call_ms": dec_call, "append_call_ms": app_call,
            "append_tokens_per_s": T / (app_avg / 1e3),
            "append_hbm_frac": append_bytes(w, T) / (app_avg / 1e3) / 1e9 / peak,
            "num_splits": S,
            "partition": "even cut of (item, block) space over the grid" if S == 0 else f"{S} splits per item",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(w),
                         "kernel": "tq_decode_attention (split kernel + combine)",
                         "peak_source": f"{peak_kind} hbm_gbs"},
            "e2e": {"value": weak_scaling_value(kv, args.steps, world, e2e_s) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_s * 1e3 / args.steps, "h2d_link_gbs": h2d_link_gbs},
            "gpu_launches": args.steps * (2 + (1 if combine_runs(w, S, dev) else 0)),
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        if others is not None:
            line["workloads"] = others
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["prefill_append", "prefill_decode", "prefill_attention", "bf16_decode"],
                    default=None,
                    help="run one small profiling case instead of the bench")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the long-context, agentic and prefill-chunk measurements")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per rank (default: the workload's 32); smaller values make the "
                         "profiling case, not a bench line")
    args = ap.parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        world = int(os.environ.get("WORLD_SIZE", args.gpus))
        run_reference(args, rank, world)
        return
    if args.case == "prefill_append":
        prefill_append_case(torch.device("cuda", 0))
        return
    if args.case == "prefill_decode":
        prefill_decode_case(torch.device("cuda", 0))
        return
    if args.case == "prefill_attention":
        prefill_attention_case(torch.device("cuda", 0))
        return
    if args.case == "bf16_decode":
        bf16_decode_case(torch.device("cuda", 0))
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_tq(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
