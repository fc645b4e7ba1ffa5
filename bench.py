"""Benchmark of the hierarchically pruned attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--layers L]

One step is one pass of the whole hot path (a fresh mask and the sparse
attention over it, i.e. one attention layer) over one batch of the workload:
hip_mask_sparse_attn for decode (one launch for bf16 groups of <= 4 query
rows; --two-calls times hip_mask + hip_sparse_attn instead), hip_mask +
hip_sparse_attn for prefill. The default workload is
Llama-3.1-8B-shaped decode at T = 128k (32 query / 8 KV heads, d = 128,
k = 2048, b_k = 2, sink 128 + window 1024, bf16). Inputs are synthetic
(seeded AR(1) keys/values, Gaussian queries, needle keys) and resident in
HBM; steps rotate over L layer buffers whose total exceeds the 126 MB L2, so
every step reads cold data. The K timed steps are replays of a CUDA graph of
L steps, bracketed by a barrier and device synchronisation, timed with CUDA
events on the launch stream (max over ranks); the last full replay is a copy
of the graph with event nodes around each kernel, whose intervals give the
kernel durations of the roofline. Rank 0 prints one JSON line.

With N > 1 (torchrun) every rank runs its own replica of the workload on its
own GPU (weak scaling; the path has no exchange step, so there is no
collective on the data path).

--impl reference times the CPU oracle (the plain C reference) on the host
cores on the same workload and metric, on a bounded sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hierarchically_pruned_sparse_b200 import workloads as W  # noqa: E402

METRIC = "decode mask+sparse-attn µs/layer @T=128k, % of HBM roofline; prefill TFLOP/s"
DEFAULT_WORKLOAD = W.DECODE_128K.name
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--layers", type=int, default=0, help="rotating layer buffers (0 = auto)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--head-masks", action="store_true",
                    help="one mask per query head (head-reduce off) instead of per KV-head group")
    ap.add_argument("--two-calls", action="store_true",
                    help="decode: time hip_mask + hip_sparse_attn instead of hip_mask_sparse_attn")
    ap.add_argument("--no-prefill", action="store_true",
                    help="default run: leave out the nested prefill measurement")
    ap.add_argument("--no-dense", action="store_true",
                    help="decode: leave out the dense-attention comparison")
    ap.add_argument("--stages", default="",
                    help="InfiniteHiP pruning stages before the mask, chunk_size:stage_k:stride_q "
                         "per stage, comma-separated (topk is then second_stage_k)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- work accounting


HEAD_MASKS = False  # --head-masks: one mask per query head instead of per KV-head group
STAGES = ()  # --stages: InfiniteHiP pruning stages (chunk_size, stage_k, stride_q) before the mask


def stage_launches() -> int:
    """Kernel launches the stages add to a mask call: a scoring and a
    selection launch per stage that ranks, or one selection launch when
    none ranks."""
    if not STAGES:
        return 0
    ranked = sum(1 for _, k, _ in STAGES if k > 0)
    return 2 * ranked if ranked else 1


def counting_view(w: W.Workload) -> W.Workload:
    """The workload as the mask sees it: with one mask per query head, every
    query head is its own group (for unit counts and the work counters)."""
    return w.replace(n_kvheads=w.n_qheads) if HEAD_MASKS else w


def oracle_layer_shape(w: W.Workload):
    import oracle
    return oracle.shape(head_dim=w.head_dim, per_head=int(HEAD_MASKS), stages=STAGES,
                        **layer_shape(w))


def layer_shape(w: W.Workload):
    T = w.seq_len
    return dict(batch=w.batch, n_qheads=w.n_qheads, n_kvheads=w.n_kvheads, seq_len=T,
                q_len=w.q_len, q_pos0=T - 1 if w.kind == "decode" else 0, block_q=w.block_q,
                block_k=w.block_k, topk=w.topk, sink=w.sink, window=w.window,
                kv_capacity=w.capacity)


def elem_bytes(w: W.Workload):
    """Bytes of a q / out element and of a k / v element."""
    if w.dtype == "e5m2":
        return 2, 1
    return (2, 2) if w.dtype == "bf16" else (4, 4)


def oracle_inputs(w: W.Workload, x: dict) -> dict:
    """The inputs as the oracle takes them: e5m2 codes decoded by the oracle."""
    if w.dtype != "e5m2":
        return x
    import oracle
    return dict(x, k=oracle.decode_e5m2(x["k"]), v=oracle.decode_e5m2(x["v"]))


def mask_algorithmic_bytes(w: W.Workload, scored: int) -> int:
    """Bytes the mask must read: every round reads the representative key block
    (b_k keys x d) of each candidate chunk, plus q; it writes the idx rows.
    ``scored`` is the number of candidates the kernels scored in one call
    (each candidate of each round exactly once)."""
    esz, kv_esz = elem_bytes(w)
    units = w.batch * w.n_kvheads * (-(-w.q_len // w.block_q))
    stride = 1 + w.topk // w.block_k + -(-w.sink // w.block_k) + (
        (-(-(w.window + w.block_q - 1) // w.block_k) + 1) if w.window else 0)
    q_bytes = w.batch * w.n_qheads * w.q_len * w.head_dim * esz
    return scored * w.block_k * w.head_dim * kv_esz + q_bytes + units * stride * 4


def mask_algorithmic_flops(w: W.Workload, scored: int) -> int:
    """Multiply-adds of the mask scores: every candidate's b_k keys against the
    G * b_q query rows of its mask (d = 128), two flops each."""
    return 2 * scored * w.block_k * w.group * w.block_q * w.head_dim


def attn_algorithmic_flops(w: W.Workload, idx: np.ndarray) -> int:
    """QK^T and PV flops (4 d per attended (row, key) pair), counted from the
    idx rows: a row at position p attends the listed keys j <= p."""
    bk, bq, T, G = w.block_k, w.block_q, w.seq_len, w.group
    rows = idx.reshape(-1, idx.shape[-1])
    nqb = rows.shape[0] // (w.batch * w.n_kvheads)
    pairs = 0
    for u, r in enumerate(rows):
        qb = u % nqb
        blocks = r[1:1 + r[0]].astype(np.int64)
        keys = (blocks[:, None] * bk + np.arange(bk)[None, :]).reshape(-1)
        keys = np.sort(keys[keys < T])
        pos = np.arange(qb * bq, min(qb * bq + bq, w.q_len))
        pairs += G * int(np.searchsorted(keys, pos, side="right").sum())
    return 4 * w.head_dim * pairs


def attn_algorithmic_bytes(w: W.Workload, idx: np.ndarray, seq_len: int, mask_len: int) -> int:
    """Bytes the sparse attention must read: K and V rows of every attended
    key (counted from the actual idx rows), q and idx; it writes the output."""
    esz, kv_esz = elem_bytes(w)
    bk = w.block_k
    rows = idx.reshape(-1, idx.shape[-1])
    keys = 0
    for r in rows:
        blocks = r[1:1 + r[0]].astype(np.int64)
        keys += int(np.minimum(bk, mask_len - blocks * bk).clip(min=0).sum())
    keys += rows.shape[0] * max(0, seq_len - mask_len)
    qo = 2 * w.batch * w.n_qheads * w.q_len * w.head_dim * esz
    return keys * 2 * w.head_dim * kv_esz + qo + int(sum(int(r[0]) + 1 for r in rows)) * 4


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:  # the NVML index need not match the CUDA index
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # NVML missing: record nothing, say so
            self.err = str(exc)
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((sm, rs, pw))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "no NVML samples" if not self.ok else "timed region shorter than one sample"}
        sms = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= int(s[1])
        reasons = [name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": float(np.median(sms)), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(sms),
                "power_w_max": float(max(s[2] for s in self.samples))}


# ---------------------------------------------------------------- distributed


def dist_setup(n_gpus: int, backend: str | None = None):
    """Join the job's process group (one process per GPU; a no-op at N=1).

    ``backend`` defaults to NCCL; gloo serves the CPU tests of these helpers.
    The group's timeout is short so that ranks waiting on a lost peer end with
    an error instead of hanging.
    """
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = backend or "nccl"
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_layer(max_total_ms: float, steps: int, world: int) -> float:
    """Whole-job decode throughput: every rank serves one layer per step, so
    the job serves steps * world layers in the slowest rank's time."""
    return max_total_ms * 1e3 / (steps * world)


# ---------------------------------------------------------------- reference arm


def reference_arm(args, w: W.Workload, world: int, rank: int):
    """The CPU oracle, as it stands, on the host cores: each step runs the mask
    and attention of a sample of the layer's (sequence, KV head, query block)
    units, sized so that the whole run stays within a few minutes, and the
    time is scaled to one layer. Same metric and unit as the GPU arm."""
    if rank != 0:
        return
    import oracle
    cores = oracle.set_threads(0)
    x = oracle_inputs(w, W.make_inputs(w))  # e5m2 codes decoded once, before timing
    sh = oracle_layer_shape(w)
    w = counting_view(w)
    nqb = -(-w.q_len // w.block_q)
    units = w.batch * w.n_kvheads * nqb
    prefill = w.kind == "prefill"
    rng = np.random.default_rng(0)
    # calibrate on a spread sample (a whole prefill layer would take hours)
    cal = np.unique(np.linspace(0, units - 1, min(units, max(cores, 8))).astype(np.int64))
    t0 = time.perf_counter()
    _oracle_units(w, x, sh, cal)
    t_layer = (time.perf_counter() - t0) * units / cal.size
    budget = 150.0
    u = units
    while u > 1 and (args.steps + args.warmup) * t_layer * u / units > budget:
        u //= 2
    picks = [rng.choice(units, u, replace=False) for _ in range(args.steps + max(0, args.warmup - 1))]
    for pick in picks[args.steps:]:
        _oracle_units(w, x, sh, pick)
    flops = 0
    t0 = time.perf_counter()
    for pick in picks[:args.steps]:
        _oracle_units(w, x, sh, pick)
    elapsed = time.perf_counter() - t0
    us_layer = elapsed / args.steps * (units / u) * 1e6
    sample = (f"{u} of {units} (sequence, KV head, query block) units per step: their mask rows "
              f"and the attention of their query rows; scaled to one layer")
    value, unit, hib = us_layer, "us/layer", False
    if prefill:
        # the flops of the sampled units (same count as the GPU arm), per second
        for pick in picks[:1]:
            idx, _, _, scored = oracle.mask(x["q"][0], x["k"], sh, units=pick, with_scored=True)
            full = np.full((units, idx.shape[1]), -1, np.int32)
            full[pick] = idx
            flops = mask_algorithmic_flops(w, int(scored.sum()))
            for uu in np.sort(pick):
                qb = uu % nqb
                r = full[uu]
                blocks = r[1:1 + r[0]].astype(np.int64)
                keys = np.sort(((blocks[:, None] * w.block_k + np.arange(w.block_k)[None, :])
                                .reshape(-1)))
                pos = np.arange(qb * w.block_q, min(qb * w.block_q + w.block_q, w.q_len))
                flops += 4 * w.head_dim * w.group * int(np.searchsorted(keys, pos, side="right").sum())
        value, unit, hib = flops / (elapsed / args.steps) / 1e12, "TFLOP/s", True
    line = {"metric": METRIC, "value": value, "unit": unit, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": hib,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_of(w, 0),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _oracle_units(w: W.Workload, x: dict, sh, units: np.ndarray):
    """Oracle mask + attention of the given (sequence, KV head, query block) units."""
    import oracle
    nqb = -(-w.q_len // w.block_q)
    idx, _, _ = oracle.mask(x["q"][0], x["k"], sh, units=units)
    full = np.full((w.batch * w.n_kvheads * nqb, idx.shape[1]), -1, np.int32)
    full[units] = idx
    rows = []
    for u in units:
        qb, g, b = u % nqb, (u // nqb) % w.n_kvheads, u // (nqb * w.n_kvheads)
        for h in range(g * w.group, (g + 1) * w.group):
            base = (b * w.n_qheads + h) * w.q_len
            rows.extend(range(base + qb * w.block_q, base + min(qb * w.block_q + w.block_q, w.q_len)))
    oracle.attention(x["q"][0], x["k"], x["v"], full, sh, rows=np.asarray(rows, np.int64))


def cpu_baseline(w: W.Workload, x: dict, min_seconds: float = 10.0):
    """The oracle timed on the host cores: whole layers (decode) until
    min_seconds pass, or a spread sample of query blocks scaled to a layer
    (prefill, where a whole layer takes hours)."""
    import oracle
    cores = oracle.set_threads(0)
    x = oracle_inputs(w, x)  # e5m2 codes decoded once, before timing
    sh = oracle_layer_shape(w)
    w = counting_view(w)
    if w.kind == "prefill":
        nqb = -(-w.q_len // w.block_q)
        units_total = w.batch * w.n_kvheads * nqb
        pick = np.unique(np.linspace(0, units_total - 1, max(cores, 8)).astype(np.int64))
        t0 = time.perf_counter()
        _oracle_units(w, x, sh, pick)
        el = time.perf_counter() - t0
        per_layer = el * units_total / pick.size
        return {"value": per_layer * 1e6, "unit": "us/layer", "cores": cores, "kind": "oracle",
                "sample": f"{pick.size} of {units_total} query blocks spread over the layer "
                          f"(mask + attention), extrapolated linearly to the layer"}
    n = 0
    t0 = time.perf_counter()
    while True:
        idx, _, _ = oracle.mask(x["q"][0], x["k"], sh)
        oracle.attention(x["q"][0], x["k"], x["v"], idx, sh)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return {"value": el / n * 1e6, "unit": "us/layer", "cores": cores, "kind": "oracle",
            "sample": f"{n} whole layer(s) of the workload (mask + attention of all heads)"}


def traffic_from_profile(kernel: str, workload: str):
    """DRAM bytes per launch of ``kernel`` from the committed ncu summary, if
    it was taken on the current sources of the kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        ent = json.load(f).get("entries", {}).get(f"{kernel}:{workload}")
    if not ent:
        return None
    h = hashlib.sha256()
    for src in ent["sources"]:
        p = os.path.join(ROOT, src)
        if not os.path.exists(p):
            return None
        with open(p, "rb") as f:
            h.update(f.read())
    if h.hexdigest() != ent["sha256"]:
        return None
    return ent["dram_bytes_per_launch"]


# ---------------------------------------------------------------- our arm


def touched_bytes(w: W.Workload) -> int:
    """Bytes one step of the workload reads (to size the rotating layer
    buffers so that a layer's data has left L2 before it is used again):
    prefill reads all of q, k and v; a decode refresh reads each round's
    representative blocks and then the attended blocks."""
    esz, kv_esz = elem_bytes(w)
    wc = counting_view(w)
    if w.kind == "prefill":
        return (2 * w.batch * w.n_kvheads * w.capacity * kv_esz
                + w.batch * w.n_qheads * w.q_len * esz) * w.head_dim
    n = -(-w.seq_len // w.block_k)
    n0 = min(w.topk // w.block_k, n)
    rounds = max(0, math.ceil(math.log2(max(1, -(-n // n0)))))
    units = wc.batch * wc.n_kvheads
    attended = n0 + -(-w.sink // w.block_k) + (-(-w.window // w.block_k) + 1 if w.window else 0)
    return units * (rounds * 2 * n0 + 2 * attended) * w.block_k * w.head_dim * kv_esz


def layer_count(w: W.Workload, layer_bytes: int, requested: int) -> int:
    """Rotating layer buffers: enough that the bytes the steps between two uses
    of a layer touch exceed 4x the L2, within 64 layers and 64 GB."""
    if requested:
        return requested
    n = max(2, math.ceil(4 * L2_BYTES / max(1, touched_bytes(w))))
    return max(2, min(n, 64, (64 << 30) // max(1, layer_bytes)))


def config_of(w: W.Workload, layers: int):
    cfg = {"workload": w.name, "kind": w.kind, "batch": w.batch, "seq_len": w.seq_len,
           "n_qheads": w.n_qheads, "n_kvheads": w.n_kvheads, "head_dim": w.head_dim,
           "topk": w.topk, "block_q": w.block_q, "block_k": w.block_k, "sink": w.sink,
           "window": w.window, "parallelism": "replicas",
           "masks": "per query head" if HEAD_MASKS else "per KV-head group",
           "kv_cache": {"e5m2": "fp8 e5m2 (bf16 q and out)"}.get(w.dtype, w.dtype)}
    if w.kind == "decode" and w.refresh > 1:
        cfg["mask_refresh"] = w.refresh
    if STAGES:
        cfg["stages"] = [{"chunk_size": c, "stage_k": k or None, "stride_q": r} for c, k, r in STAGES]
    if layers:
        cfg["l2"] = (f"{layers} rotating layer buffers; the steps between two uses of a layer "
                     f"touch {layers * touched_bytes(w) / L2_BYTES:.1f}x the L2 (no flush)")
    return cfg


def time_regions(replay, world: int, stream, dev, min_seconds: float = 1.0, max_regions: int = 5000):
    """Device time of the timed region (K steps), repeated until at least
    ``min_seconds`` of device time has passed: each repeat is bracketed by a
    barrier and a device synchronisation on both sides and timed with CUDA
    events on ``stream``; returns the per-repeat times (ms, max over ranks)."""
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def once():
        barrier(world)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            start.record(stream)
            replay()
            end.record(stream)
        end.synchronize()
        torch.cuda.synchronize(dev)
        barrier(world)
        return max_over_ranks(start.elapsed_time(end), world)

    first = once()  # every rank sees the same maximum, so all agree on the count
    n = int(min(max_regions, max(1, math.ceil(min_seconds * 1e3 / max(first, 1e-3)))))
    return [first] + [once() for _ in range(n - 1)]


class Layers:
    """Device buffers of `layers` copies of a workload's layer: each layer's K
    and V caches in one [2, ...] tensor (so that one copy appends a key row
    and a value row), its own query per decode step, idx and output."""

    def __init__(self, w: W.Workload, x: dict, layers: int, dev):
        import torch
        self.dt = torch.float32 if w.dtype == "f32" else torch.bfloat16  # q and out
        self.kt = torch.uint8 if w.dtype == "e5m2" else self.dt          # k and v
        k0 = torch.from_numpy(x["k"]).to(dev).to(self.kt).contiguous()
        v0 = torch.from_numpy(x["v"]).to(dev).to(self.kt).contiguous()
        self.kvs = [torch.stack([k0, v0]) for _ in range(layers)]
        del k0, v0
        self.ks = [kv[0] for kv in self.kvs]
        self.vs = [kv[1] for kv in self.kvs]
        steps = x["q"].shape[0]
        qd = [torch.from_numpy(np.ascontiguousarray(x["q"][s])).to(dev).to(self.dt).contiguous()
              for s in range(steps)]
        self.qs = [[q.clone() for q in qd] for _ in range(layers)]  # [layer][decode step]
        self.outs = [torch.empty_like(qd[0]) for _ in range(layers)]
        self.n = layers


def build_graph(stream, calls):
    """A CUDA graph of the given calls, captured on ``stream``."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    return g


def ours(args, w: W.Workload, world: int, rank: int, local: int, nested: bool = False):
    """Our arm on workload ``w``; returns the JSON line (printed by main)."""
    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if w.kind == "prefill":
        return ours_prefill(args, w, world, rank, dev, nested)
    return ours_decode(args, w, world, rank, dev)


def _scored_and_idx(hb, sess, lay, stream):
    """Scored candidates of one mask call (status block counter) and its idx."""
    hb.workspace_init(sess.p)
    with torch_stream(stream):
        hb.hip_mask(lay.qs[0][0], lay.ks[0], sess.p, lay.idxs[0])
    stream.synchronize()
    base = sess.p.workspace - sess.workspace.data_ptr()
    scored = int(sess.workspace[base + 8: base + 16].cpu().numpy().view(np.uint64)[0])
    sess.check()
    return scored, lay.idxs[0].cpu().numpy()


def torch_stream(stream):
    import torch
    return torch.cuda.stream(stream)


def ours_decode(args, w: W.Workload, world: int, rank: int, dev):
    """Decode: a bench step is r_m decode steps of one layer (one mask refresh
    through hip_mask_sparse_attn, then r_m - 1 steps of hip_sparse_attn that
    reuse the mask while the cache grows by one key per step); with r_m = 1
    every step refreshes. The calls run phase-major over the rotating layers
    (decode step s of every layer, then step s + 1), as in a model."""
    import torch

    from hierarchically_pruned_sparse_b200 import binding as hb
    x = W.make_inputs(w)
    esz, kv_esz = elem_bytes(w)
    wc = counting_view(w)
    rm = w.refresh
    layer_bytes = 2 * x["k"].size * kv_esz + x["q"][0].size * esz
    layers = layer_count(w, layer_bytes, args.layers)
    lay = Layers(w, x, layers, dev)
    stream = torch.cuda.Stream(device=dev)
    shp = layer_shape(w)
    code = {"bf16": hb.HIPS_BF16, "f32": hb.HIPS_F32, "e5m2": hb.HIPS_BF16_E5M2}[w.dtype]
    T = w.seq_len
    # the workspace is sized at the longest cache of the reuse steps
    shp.update(seq_len=T + rm - 1, q_pos0=T + rm - 2)
    sess = hb.Session(dtype=code, flags=hb.FLAG_HEAD_MASKS if HEAD_MASKS else 0, stream=stream,
                      stages=STAGES,
                      mask_len=T, **shp)
    sess.set(seq_len=T, q_pos0=T - 1)
    lay.idxs = [sess.new_idx() for _ in range(layers)]
    two = bool(args.two_calls)
    one_launch = not two and w.dtype != "f32" and wc.group * min(w.block_q, w.q_len) <= 4

    def call(l, s, q=None):
        """Decode step s (0 = refresh) of layer l on query q (its own by default)."""
        q = lay.qs[l][s] if q is None else q
        sess.set(seq_len=T + s, mask_len=T, q_pos0=T + s - 1)
        if s == 0 and not two:
            hb.hip_mask_sparse_attn(q, lay.ks[l], lay.vs[l], sess.p, lay.idxs[l], lay.outs[l])
        else:
            if s == 0:
                hb.hip_mask(q, lay.ks[l], sess.p, lay.idxs[l])
            hb.hip_sparse_attn(q, lay.ks[l], lay.vs[l], lay.idxs[l], sess.p, lay.outs[l])

    def cycle(nl):
        """Calls of bench steps on layers [0, nl): phase-major."""
        return [(l, s) for s in range(rm) for l in range(nl)]

    with torch_stream(stream):
        for i in range(max(args.warmup, 3)):  # untimed bench steps
            for s in range(rm):
                call(i % layers, s)
    stream.synchronize()
    sess.check()
    sess.set(seq_len=T, mask_len=T, q_pos0=T - 1)
    scored, idx_host = _scored_and_idx(hb, sess, lay, stream)
    mask_bytes = mask_algorithmic_bytes(wc, scored)
    attn_bytes = [attn_algorithmic_bytes(wc, idx_host, T + s, T) for s in range(rm)]
    step_bytes = mask_bytes + sum(attn_bytes)  # one bench step: r_m decode steps of a layer

    steps = max(1, args.steps)
    reps, rem = divmod(steps, layers)
    g_full = build_graph(stream, [lambda l=l, s=s: call(l, s) for l, s in cycle(layers)])
    g_rem = build_graph(stream, [lambda l=l, s=s: call(l, s) for l, s in cycle(rem)]) if rem else None

    def replay():
        for _ in range(reps):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()

    with torch_stream(stream):
        for _ in range(2):
            replay()
    stream.synchronize()
    with ClockSampler(int(dev.index or 0)) as clk:
        regions = time_regions(replay, world, stream, dev)
    sess.check()
    region_ms = float(np.median(regions))
    step_us = region_ms * 1e3 / steps                      # one bench step (r_m decode steps)
    us_layer = whole_job_us_per_layer(region_ms, steps * rm, world)  # per layer decode step

    # split of a bench step by kernel: CUDA event nodes around each call of
    # the first layer, in graph replays outside the timed region (the nodes
    # add a little time of their own; the shares are what is reported)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3 * rm)]

    def evcall(s):
        def f():
            ev[3 * s].record(stream)
            sess.set(seq_len=T + s, mask_len=T, q_pos0=T + s - 1)
            q = lay.qs[0][s]
            if s == 0 and not two:
                hb.hip_mask_sparse_attn(q, lay.ks[0], lay.vs[0], sess.p, lay.idxs[0], lay.outs[0])
                ev[1].record(stream)
            else:
                if s == 0:
                    hb.hip_mask(q, lay.ks[0], sess.p, lay.idxs[0])
                ev[3 * s + 1].record(stream)
                hb.hip_sparse_attn(q, lay.ks[0], lay.vs[0], lay.idxs[0], sess.p, lay.outs[0])
            ev[3 * s + 2].record(stream)
        return f

    calls_ev = []
    for l, s in cycle(layers):
        calls_ev.append(evcall(s) if l == 0 else (lambda l=l, s=s: call(l, s)))
    g_ev = build_graph(stream, calls_ev)
    mask_ev, attn_ev = [], [[] for _ in range(rm)]
    with torch_stream(stream):
        for _ in range(max(3, min(30, 3000 // max(1, layers * rm)))):
            g_ev.replay()
            stream.synchronize()
            mask_ev.append(ev[0].elapsed_time(ev[1]))
            for s in range(rm):
                attn_ev[s].append(ev[3 * s + 1].elapsed_time(ev[3 * s + 2]))
    sess.check()
    m_ev = float(np.median(mask_ev)) * 1e3
    a_ev = [float(np.median(a)) * 1e3 for a in attn_ev]
    # scale the event-node intervals to the measured step so that the
    # per-kernel times add up to it (they cannot exceed the step)
    ev_total = m_ev + sum(a_ev)
    scale = step_us / ev_total if ev_total > 0 else 1.0
    refresh_us = (m_ev + a_ev[0]) * scale
    mask_us = m_ev * scale
    attn0_us = a_ev[0] * scale
    reuse_us = [a * scale for a in a_ev[1:]]

    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    if one_launch:
        # the refresh is one kernel (after the stages' launches, if any):
        # mask and attention bytes over its time
        dom_bytes, dom_us = mask_bytes + attn_bytes[0], refresh_us
        dom_kernel = "mask_mma_kernel (mask + attention)"
        traffic = traffic_from_profile("mask_mma_kernel+attn", w.name)
        if STAGES:
            dom_kernel = "stage_score/stage_select + " + dom_kernel
            traffic = None
    else:
        dom_bytes, dom_us = mask_bytes, mask_us
        dom_kernel = "mask_mma_kernel" if w.dtype != "f32" else "mask_fma_kernel"
        traffic = traffic_from_profile(dom_kernel, w.name) if not STAGES else None
    dom_gbs = dom_bytes / (dom_us * 1e-6) / 1e9
    roofline = {"bound": "hbm", "kernel": dom_kernel, "achieved": dom_gbs, "peak": hbm,
                "peak_kind": f"{pk_kind} HBM copy", "unit": "GB/s", "frac": dom_gbs / hbm,
                "traffic": traffic, "algorithmic_bytes": dom_bytes,
                "time_us": dom_us,
                "how": ("the refresh step's share of the median timed step (event-node "
                        "split), algorithmic bytes over it" if rm > 1 or not one_launch else
                        "the step is the stage launches and this one launch: algorithmic bytes "
                        "over the median step time" if STAGES else
                        "the step is this one launch: algorithmic bytes over the median step time")}
    step_gbs = step_bytes / (step_us * 1e-6) / 1e9
    launches_refresh = (1 if one_launch else 2) + stage_launches()
    launches_per_step = launches_refresh + (rm - 1)

    kern = {"how": "median timed step split by CUDA event-node intervals of one layer "
                   "(replays outside the timed region), scaled to the step",
            "step_call": "hip_mask + hip_sparse_attn" if two else "hip_mask_sparse_attn",
            "one_launch": one_launch and not STAGES, "scored_candidates": scored,
            "mask_bytes": mask_bytes, "attn_bytes": attn_bytes[0]}
    if one_launch:
        kern["refresh_us"] = refresh_us
    else:
        kern.update(mask_us=mask_us, attn_us=attn0_us)
    if rm > 1:
        kern["refresh_us"] = refresh_us
        kern["reuse_us_mean"] = float(np.mean(reuse_us))
        kern["reuse_bytes_mean"] = float(np.mean(attn_bytes[1:]))
        kern["reuse_gbs"] = kern["reuse_bytes_mean"] / (kern["reuse_us_mean"] * 1e-6) / 1e9
    kern["event_node_us"] = {"mask_or_fused": m_ev, "attn": a_ev}

    # the library's dense decode kernel on the same layers (comparison only)
    dense = None
    if not args.no_dense:
        sess.set(seq_len=T, mask_len=T, q_pos0=T - 1)
        gd = build_graph(stream, [lambda l=l: hb.hip_dense_attn(lay.qs[l][0], lay.ks[l], lay.vs[l],
                                                                 sess.p, lay.outs[l])
                                  for l in range(layers)])
        with torch_stream(stream):
            gd.replay()
        stream.synchronize()
        dts = time_regions(lambda: gd.replay(), world, stream, dev, min_seconds=0.3)
        sess.check()
        d_us = float(np.median(dts)) * 1e3 / layers
        d_bytes = (wc.batch * w.n_kvheads * T * 2 * w.head_dim * kv_esz
                   + 2 * w.batch * w.n_qheads * w.head_dim * esz)
        dense = {"kernel": "attn_fma_kernel (dense)", "us_per_layer": d_us,
                 "bytes": d_bytes, "gbs": d_bytes / (d_us * 1e-6) / 1e9,
                 "frac": d_bytes / (d_us * 1e-6) / 1e9 / hbm,
                 "speedup_of_sparse": d_us / us_layer}
        del gd

    e2e = None if args.no_e2e else decode_e2e(args, w, x, lay, sess, call, cycle, steps, layers,
                                               world, stream, dev, esz)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x)

    line = {
        "metric": METRIC, "value": us_layer, "unit": "us/layer", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": region_ms / steps,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if lay.dt == torch.bfloat16 else "f32",
        "data": "synthetic (seeded AR(1) keys/values, Gaussian queries, needle keys)",
        "config": config_of(w, layers),
        "roofline": roofline,
        "step_roofline": {"bound": "hbm", "achieved": step_gbs, "peak": hbm, "unit": "GB/s",
                          "frac": step_gbs / hbm, "algorithmic_bytes": step_bytes},
        "kernels": kern,
        "timing": {"regions": len(regions), "region_ms_median": region_ms,
                   "region_ms_min": float(np.min(regions)), "region_ms_max": float(np.max(regions)),
                   "decode_steps_per_bench_step": rm},
        "gpu_launches": launches_per_step * steps,
        "clocks": clk.summary(),
    }
    if dense:
        line["dense"] = dense
    if e2e:
        line["e2e"] = e2e
    if cpu:
        line["cpu_baseline"] = cpu
    return line


def decode_e2e(args, w, x, lay, sess, call, cycle, steps, layers, world, stream, dev, esz):
    """End to end through the C ABI: per decode call one H2D (pinned host) of
    the call's query and new key and value rows, packed, on a copy stream;
    one copy appends the rows to the caches; the call itself on the query in
    the staging buffer; and a D2H of the output. The uploads of later calls
    overlap the kernels of earlier ones (they do not depend on them)."""
    import torch
    dt, kt = lay.dt, lay.kt
    T = w.seq_len
    rm = w.refresh
    copy_stream = torch.cuda.Stream(device=dev)
    n_calls = layers * rm
    q_host = [torch.from_numpy(np.ascontiguousarray(x["q"][s])).to(dt).contiguous().view(torch.uint8)
              for s in range(rm)]
    rows = [torch.from_numpy(np.ascontiguousarray(
        np.stack([x["k"][:, :, T - 1 + s], x["v"][:, :, T - 1 + s]]))).to(kt).contiguous()
        for s in range(rm)]
    packed = [torch.cat([q_host[s].reshape(-1), rows[s].view(torch.uint8).reshape(-1)]) for s in range(rm)]
    hstage = [[packed[s].clone().pin_memory() for s in range(rm)] for _ in range(layers)]
    dstage = [[torch.empty(packed[s].numel(), dtype=torch.uint8, device=dev) for s in range(rm)]
              for _ in range(layers)]
    nq = q_host[0].numel()
    qv = [[d[:nq].view(dt).view(lay.qs[0][0].shape) for d in dl] for dl in dstage]
    kvrow = [[d[nq:].view(kt).view(rows[0].shape) for d in dl] for dl in dstage]
    hout = [[torch.empty(lay.outs[0].shape, dtype=dt).pin_memory() for _ in range(rm)]
            for _ in range(layers)]
    up = [torch.cuda.Event() for _ in range(n_calls)]

    def e2e_calls(nl):
        order = cycle(nl)

        def run():
            cur = torch.cuda.current_stream()
            copy_stream.wait_stream(cur)
            # uploads, in call order, on the copy stream
            with torch.cuda.stream(copy_stream):
                for i, (l, s) in enumerate(order):
                    dstage[l][s].copy_(hstage[l][s], non_blocking=True)
                    up[i].record(copy_stream)
            for i, (l, s) in enumerate(order):
                cur.wait_event(up[i])
                lay.kvs[l][:, :, :, T - 1 + s].copy_(kvrow[l][s])
                call(l, s, qv[l][s])
                hout[l][s].copy_(lay.outs[l], non_blocking=True)
            cur.wait_stream(copy_stream)
        return run

    reps, rem = divmod(steps, layers)
    g2 = build_graph(stream, [e2e_calls(layers)])
    g2_rem = build_graph(stream, [e2e_calls(rem)]) if rem else None

    def replay():
        for _ in range(reps):
            g2.replay()
        if g2_rem is not None:
            g2_rem.replay()

    with torch_stream(stream):
        replay()
    stream.synchronize()
    regions = time_regions(replay, world, stream, dev, min_seconds=0.5)
    sess.check()
    e2e_ms = float(np.median(regions))
    h2d = int(np.mean([p.numel() for p in packed]))
    return {"value": whole_job_us_per_layer(e2e_ms, steps * rm, world), "unit": "us/layer",
            "h2d_bytes_per_step": h2d * rm, "d2h_bytes_per_step": int(lay.outs[0].numel() * esz) * rm,
            "regions": len(regions),
            "how": "CUDA graph per group of steps: per decode call one H2D (pinned) of q and "
                   "the new k/v rows on a copy stream (overlapping earlier calls' kernels), "
                   "their append to the caches, the C-ABI call, D2H of out"}


def ours_prefill(args, w: W.Workload, world: int, rank: int, dev, nested: bool):
    """Prefill: a step is hip_mask (key-norm pre-pass and mask) and
    hip_sparse_attn over the whole sequence, rotating over layer buffers."""
    import torch

    from hierarchically_pruned_sparse_b200 import binding as hb
    x = W.make_inputs(w)
    esz, kv_esz = elem_bytes(w)
    wc = counting_view(w)
    layer_bytes = 2 * x["k"].size * kv_esz + x["q"][0].size * esz
    layers = layer_count(w, layer_bytes, 0 if nested else args.layers)
    lay = Layers(w, x, layers, dev)
    stream = torch.cuda.Stream(device=dev)
    code = {"bf16": hb.HIPS_BF16, "f32": hb.HIPS_F32, "e5m2": hb.HIPS_BF16_E5M2}[w.dtype]
    sess = hb.Session(dtype=code, flags=hb.FLAG_HEAD_MASKS if HEAD_MASKS else 0, stream=stream,
                      stages=STAGES,
                      **layer_shape(w))
    lay.idxs = [sess.new_idx() for _ in range(layers)]

    def call(l):
        hb.hip_mask(lay.qs[l][0], lay.ks[l], sess.p, lay.idxs[l])
        hb.hip_sparse_attn(lay.qs[l][0], lay.ks[l], lay.vs[l], lay.idxs[l], sess.p, lay.outs[l])

    with torch_stream(stream):
        for i in range(max(args.warmup, 3)):
            call(i % layers)
    stream.synchronize()
    sess.check()
    scored, idx_host = _scored_and_idx(hb, sess, lay, stream)
    mask_flops = mask_algorithmic_flops(wc, scored)
    attn_flops = attn_algorithmic_flops(wc, idx_host)
    steps = max(1, args.steps)
    reps, rem = divmod(steps, layers)
    g_full = build_graph(stream, [lambda l=l: call(l) for l in range(layers)])
    g_rem = build_graph(stream, [lambda l=l: call(l) for l in range(rem)]) if rem else None

    def replay():
        for _ in range(reps):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()

    with torch_stream(stream):
        replay()
    stream.synchronize()
    with ClockSampler(int(dev.index or 0)) as clk:
        regions = time_regions(replay, world, stream, dev)
    sess.check()
    region_ms = float(np.median(regions))
    step_ms = region_ms / steps
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]

    def evcall():
        ev[0].record(stream)
        hb.hip_mask(lay.qs[0][0], lay.ks[0], sess.p, lay.idxs[0])
        ev[1].record(stream)
        hb.hip_sparse_attn(lay.qs[0][0], lay.ks[0], lay.vs[0], lay.idxs[0], sess.p, lay.outs[0])
        ev[2].record(stream)

    g_ev = build_graph(stream, [evcall] + [lambda l=l: call(l) for l in range(1, layers)])
    m_ev, a_ev = [], []
    with torch_stream(stream):
        for _ in range(5):
            g_ev.replay()
            stream.synchronize()
            m_ev.append(ev[0].elapsed_time(ev[1]))
            a_ev.append(ev[1].elapsed_time(ev[2]))
    sess.check()
    m_ev, a_ev = float(np.median(m_ev)), float(np.median(a_ev))
    scale = step_ms / (m_ev + a_ev)
    mask_ms, attn_ms = m_ev * scale, a_ev * scale
    pk, pk_kind = peaks()
    burst = float(pk["bf16_tflops"])
    sustained = float(pk.get("bf16_tflops_sustained", burst))
    mask_tf = mask_flops / (mask_ms * 1e-3) / 1e12
    attn_tf = attn_flops / (attn_ms * 1e-3) / 1e12
    step_tf = (mask_flops + attn_flops) * world / (region_ms * 1e-3 / steps) / 1e12

    def tensor_roof(kernel, tf, flops, ms):
        return {"bound": "tensor", "kernel": kernel, "achieved": tf, "peak": burst,
                "peak_kind": f"{pk_kind} bf16 burst (cuBLAS)", "unit": "TFLOP/s", "frac": tf / burst,
                "frac_of_sustained": tf / sustained, "sustained_peak": sustained,
                "traffic": traffic_from_profile(kernel, w.name), "algorithmic_flops": flops,
                "time_ms": ms}

    mask_kernel = "mask_mma_kernel"
    roofline = (tensor_roof(mask_kernel, mask_tf, mask_flops, mask_ms) if mask_ms >= attn_ms
                else tensor_roof("attn_mma_kernel", attn_tf, attn_flops, attn_ms))
    e2e = None
    if not args.no_e2e:
        hq = torch.from_numpy(np.ascontiguousarray(x["q"][0])).to(lay.dt).pin_memory()
        hk = torch.from_numpy(x["k"]).to(lay.kt).pin_memory()
        hv = torch.from_numpy(x["v"]).to(lay.kt).pin_memory()
        hout = torch.empty(lay.outs[0].shape, dtype=lay.dt).pin_memory()
        n_e2e = max(1, min(steps, 10))

        def e2e_replay():
            for i in range(n_e2e):
                l = i % layers
                lay.qs[l][0].copy_(hq, non_blocking=True)
                lay.ks[l].copy_(hk, non_blocking=True)
                lay.vs[l].copy_(hv, non_blocking=True)
                call(l)
                hout.copy_(lay.outs[l], non_blocking=True)

        regions_e = time_regions(e2e_replay, world, stream, dev, min_seconds=0.0, max_regions=3)
        sess.check()
        e2e_ms = float(np.median(regions_e))
        e2e = {"value": (mask_flops + attn_flops) * n_e2e * world / (e2e_ms * 1e-3) / 1e12,
               "unit": "TFLOP/s",
               "h2d_bytes_per_step": int((hq.numel() * esz + (hk.numel() + hv.numel()) * kv_esz)),
               "d2h_bytes_per_step": int(lay.outs[0].numel() * esz), "steps": n_e2e,
               "how": "per step: H2D of q, k, v (pinned), hip_mask, hip_sparse_attn, D2H of out"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x)
        if cpu:
            cpu = dict(cpu, value_tflops=(mask_flops + attn_flops) / (cpu["value"] * 1e-6) / 1e12)
    line = {
        "metric": METRIC, "value": step_tf, "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if lay.dt == torch.bfloat16 else "f32",
        "data": "synthetic (seeded AR(1) queries, keys and values)",
        "config": config_of(w, layers),
        "roofline": roofline,
        "attn_roofline": tensor_roof("attn_mma_kernel", attn_tf, attn_flops, attn_ms),
        "mask_roofline": tensor_roof(mask_kernel, mask_tf, mask_flops, mask_ms),
        "kernels": {"how": "median timed step split by CUDA event-node intervals (replays "
                           "outside the timed region), scaled to the step",
                    "mask_ms": mask_ms, "attn_ms": attn_ms, "mask_flops": mask_flops,
                    "attn_flops": attn_flops, "scored_candidates": scored,
                    "us_per_layer": step_ms * 1e3},
        "timing": {"regions": len(regions), "region_ms_median": region_ms,
                   "region_ms_min": float(np.min(regions)), "region_ms_max": float(np.max(regions))},
        "gpu_launches": (3 + stage_launches()) * steps,  # key-norm pre-pass, mask, attention
        "clocks": clk.summary(),
    }
    if e2e:
        line["e2e"] = e2e
    if cpu:
        line["cpu_baseline"] = cpu
    return line


def main():
    global HEAD_MASKS, STAGES
    args = parse()
    HEAD_MASKS = args.head_masks
    if args.stages:
        STAGES = tuple(tuple(int(v) for v in st.split(":")) for st in args.stages.split(","))
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores alone; no process group
        reference_arm(args, w, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        line = ours(args, w, world, rank, local)
        if (args.workload == DEFAULT_WORKLOAD and not args.no_prefill and not HEAD_MASKS
                and not args.two_calls and not STAGES):
            # the other half of the metric: prefill TFLOP/s, in the same line
            pw = W.PREFILL_32K
            pre = ours(args, pw, world, rank, local, nested=True)
            line["prefill"] = {k: pre[k] for k in ("value", "unit", "ms_per_step", "config",
                                                   "roofline", "attn_roofline", "mask_roofline",
                                                   "kernels", "timing", "gpu_launches", "clocks",
                                                   "e2e", "cpu_baseline") if k in pre}
            line["gpu_launches_prefill"] = pre["gpu_launches"]
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
