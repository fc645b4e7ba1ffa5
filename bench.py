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
    ap.add_argument("--steps", type=int, default=2000)
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


def counting_view(w: W.Workload) -> W.Workload:
    """The workload as the mask sees it: with one mask per query head, every
    query head is its own group (for unit counts and the work counters)."""
    return w.replace(n_kvheads=w.n_qheads) if HEAD_MASKS else w


def oracle_layer_shape(w: W.Workload):
    import oracle
    return oracle.shape(head_dim=w.head_dim, per_head=int(HEAD_MASKS), **layer_shape(w))


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


def config_of(w: W.Workload, layers: int):
    return {"workload": w.name, "kind": w.kind, "batch": w.batch, "seq_len": w.seq_len,
            "n_qheads": w.n_qheads, "n_kvheads": w.n_kvheads, "head_dim": w.head_dim,
            "topk": w.topk, "block_q": w.block_q, "block_k": w.block_k, "sink": w.sink,
            "window": w.window, "parallelism": "replicas",
            "masks": "per query head" if HEAD_MASKS else "per KV-head group",
            "kv_cache": {"e5m2": "fp8 e5m2 (bf16 q and out)"}.get(w.dtype, w.dtype),
            "l2": f"{layers} rotating layer buffers > L2 (no flush)" if layers else None}


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


def ours(args, w: W.Workload, world: int, rank: int, local: int):
    import torch

    from hierarchically_pruned_sparse_b200 import binding as hb
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    x = W.make_inputs(w)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16  # q and out
    kt = torch.uint8 if w.dtype == "e5m2" else dt                # k and v
    esz, kv_esz = elem_bytes(w)
    prefill = w.kind == "prefill"
    layer_bytes = 2 * x["k"].size * kv_esz + x["q"][0].size * esz
    layers = args.layers or max(2, math.ceil(4 * L2_BYTES / layer_bytes))
    layers = min(layers, 64)
    k0 = torch.from_numpy(x["k"]).to(dev).to(kt).contiguous()
    v0 = torch.from_numpy(x["v"]).to(dev).to(kt).contiguous()
    q0 = torch.from_numpy(np.ascontiguousarray(x["q"][0])).to(dev).to(dt).contiguous()
    # each layer's K and V caches sit in one [2, ...] tensor, so that one copy
    # appends a new key row and value row to both
    kvs = [torch.stack([k0, v0]) for _ in range(layers)]
    del k0, v0
    ks = [kv[0] for kv in kvs]
    vs = [kv[1] for kv in kvs]
    qs = [q0.clone() for _ in range(layers)]
    stream = torch.cuda.Stream(device=dev)
    shp = layer_shape(w)
    code = {"bf16": hb.HIPS_BF16, "f32": hb.HIPS_F32, "e5m2": hb.HIPS_BF16_E5M2}[w.dtype]
    sess = hb.Session(dtype=code,
                      flags=hb.FLAG_HEAD_MASKS if HEAD_MASKS else 0,
                      stream=stream, **shp)
    idxs = [sess.new_idx() for _ in range(layers)]
    outs = [torch.empty_like(q0) for _ in range(layers)]

    # decode steps go through hip_mask_sparse_attn (a fresh mask and the
    # attention over it); the library runs it as one launch for bf16 groups of
    # at most 4 query rows, as the two kernels otherwise
    fused = not prefill and not args.two_calls
    wc = counting_view(w)
    one_launch = fused and w.dtype != "f32" and wc.group * min(w.block_q, w.q_len) <= 4

    def two_calls(l, q=None):
        q = qs[l] if q is None else q
        hb.hip_mask(q, ks[l], sess.p, idxs[l])
        hb.hip_sparse_attn(q, ks[l], vs[l], idxs[l], sess.p, outs[l])

    def step(l, q=None):
        if fused:
            hb.hip_mask_sparse_attn(qs[l] if q is None else q, ks[l], vs[l], sess.p, idxs[l],
                                    outs[l])
        else:
            two_calls(l, q)

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            step(i % layers)
    stream.synchronize()
    sess.check()
    # one more mask call on a cleared status block counts the scored candidates
    hb.workspace_init(sess.p)
    with torch.cuda.stream(stream):
        hb.hip_mask(qs[0], ks[0], sess.p, idxs[0])
    stream.synchronize()
    base = sess.p.workspace - sess.workspace.data_ptr()
    scored = int(sess.workspace[base + 8: base + 16].cpu().numpy().view(np.uint64)[0])
    sess.check()
    idx_host = idxs[0].cpu().numpy()
    mask_bytes = mask_algorithmic_bytes(wc, scored)
    attn_bytes = attn_algorithmic_bytes(wc, idx_host, w.seq_len, w.seq_len)
    mask_flops = mask_algorithmic_flops(wc, scored)
    attn_flops = attn_algorithmic_flops(wc, idx_host) if prefill else 0

    # CUDA graphs of `layers` steps (and of the remainder of K); a copy of
    # the full graph with event nodes around each kernel gives the kernel
    # durations inside the timed region
    def graph_with_events(ev, fused_step):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for l in range(layers):
                ev[3 * l].record(stream)
                if fused_step:
                    hb.hip_mask_sparse_attn(qs[l], ks[l], vs[l], sess.p, idxs[l], outs[l])
                    ev[3 * l + 1].record(stream)
                else:
                    hb.hip_mask(qs[l], ks[l], sess.p, idxs[l])
                    ev[3 * l + 1].record(stream)
                    hb.hip_sparse_attn(qs[l], ks[l], vs[l], idxs[l], sess.p, outs[l])
                ev[3 * l + 2].record(stream)
        return gr

    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3 * layers)]
    g_ev = graph_with_events(ev, fused)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for l in range(layers):
            step(l)
    steps = max(1, args.steps)
    reps, rem = divmod(steps, layers)
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=stream):
            for l in range(rem):
                step(l)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g.replay()
            g_ev.replay()
            if g_rem is not None:
                g_rem.replay()
    stream.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        # graphs replay on the current stream: make it the stream the events use
        start.record(stream)
        # the last full replay carries the event nodes that time each kernel
        for i in range(reps):
            (g_ev if i == reps - 1 else g).replay()
        if g_rem is not None:
            g_rem.replay()
        end.record(stream)
        end.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    sess.check()
    total_ms = start.elapsed_time(end)
    mask_ms = np.mean([ev[3 * l].elapsed_time(ev[3 * l + 1]) for l in range(layers)])
    attn_ms = np.mean([ev[3 * l + 1].elapsed_time(ev[3 * l + 2]) for l in range(layers)])
    total_ms = max_over_ranks(total_ms, world)
    us_layer = whole_job_us_per_layer(total_ms, steps, world)
    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    tensor_peak = float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
    mask_gbs = mask_bytes / (mask_ms * 1e-3) / 1e9
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9
    step_gbs = (mask_bytes + attn_bytes) / (total_ms * 1e-3 / (steps)) / 1e9
    mask_tf = mask_flops / (mask_ms * 1e-3) / 1e12
    attn_tf = attn_flops / (attn_ms * 1e-3) / 1e12
    step_tf = (mask_flops + attn_flops) / (total_ms * 1e-3 / steps) / 1e12
    # hip_mask + hip_sparse_attn (their split merge is fused), or one launch
    launches_per_step = 1 if one_launch else 2
    if w.dtype == "bf16" and wc.group * min(w.block_q, w.q_len) > 32:
        launches_per_step += 1  # the key-block norm pre-pass of a many-row mask
    two_call = None
    if fused:
        # the same step as the two separate calls, for comparison (not timed above)
        ev2 = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3 * layers)]
        g3 = graph_with_events(ev2, False)
        with torch.cuda.stream(stream):
            for _ in range(max(3, min(50, reps))):
                g3.replay()
        stream.synchronize()
        sess.check()
        m2 = np.mean([ev2[3 * l].elapsed_time(ev2[3 * l + 1]) for l in range(layers)])
        a2 = np.mean([ev2[3 * l + 1].elapsed_time(ev2[3 * l + 2]) for l in range(layers)])
        two_call = {"mask_us": m2 * 1e3, "attn_us": a2 * 1e3, "step_us": (m2 + a2) * 1e3,
                    "how": "hip_mask + hip_sparse_attn, CUDA event nodes, last of up to 50 replays"}
        del g3

    # e2e: per step, one H2D from pinned host memory of the step's query and
    # its new key and value rows (packed), one copy that appends the rows to the
    # caches, the C-ABI call(s) on the query in the staging buffer, and D2H of
    # the output; captured as a graph
    e2e = None
    if not args.no_e2e and not prefill:
        # q (as bf16/f32 bytes) then the new key and value rows (native bytes)
        q_host = torch.from_numpy(np.ascontiguousarray(x["q"][0])).to(dt).contiguous().view(torch.uint8)
        rows = torch.from_numpy(np.ascontiguousarray(
            np.stack([x["k"][:, :, w.seq_len - 1], x["v"][:, :, w.seq_len - 1]])))
        rows = rows.to(kt).contiguous()
        rb = rows.view(torch.uint8).reshape(-1)
        packed = torch.cat([q_host.reshape(-1), rb])
        hstage = [packed.clone().pin_memory() for _ in range(layers)]
        dstage = [torch.empty(packed.numel(), dtype=torch.uint8, device=dev) for _ in range(layers)]
        qv = [d[:q_host.numel()].view(dt).view(q0.shape) for d in dstage]
        kvrow = [d[q_host.numel():].view(kt).view(rows.shape) for d in dstage]
        hout = [torch.empty(q0.shape, dtype=dt).pin_memory() for _ in range(layers)]

        def e2e_step(l):
            dstage[l].copy_(hstage[l], non_blocking=True)
            kvs[l][:, :, :, w.seq_len - 1].copy_(kvrow[l])
            step(l, qv[l])
            hout[l].copy_(outs[l], non_blocking=True)

        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            for l in range(layers):
                e2e_step(l)
        g2_rem = None
        if rem:
            g2_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2_rem, stream=stream):
                for l in range(rem):
                    e2e_step(l)
        with torch.cuda.stream(stream):
            g2.replay()
        stream.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            s2.record(stream)
            for _ in range(reps):
                g2.replay()
            if g2_rem is not None:
                g2_rem.replay()
            e2.record(stream)
        e2.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(s2.elapsed_time(e2), world)
        h2d = packed.numel()
        e2e = {"value": whole_job_us_per_layer(e2e_ms, steps, world), "unit": "us/layer",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(q0.numel() * esz),
               "how": "CUDA graph per step: one H2D (pinned) of q and the new k/v rows, "
                      "their append to the caches, "
                      + ("hip_mask_sparse_attn" if fused else "hip_mask + hip_sparse_attn")
                      + ", D2H of out"}
        sess.check()

    if not args.no_e2e and prefill:
        hq = torch.from_numpy(np.ascontiguousarray(x["q"][0])).to(dt).pin_memory()
        hk = torch.from_numpy(x["k"]).to(dt).pin_memory()
        hv = torch.from_numpy(x["v"]).to(dt).pin_memory()
        hout = torch.empty(q0.shape, dtype=dt).pin_memory()
        n_e2e = max(1, min(steps, 20))
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            s2.record(stream)
            for i in range(n_e2e):
                l = i % layers
                qs[l].copy_(hq, non_blocking=True)
                ks[l].copy_(hk, non_blocking=True)
                vs[l].copy_(hv, non_blocking=True)
                step(l)
                hout.copy_(outs[l], non_blocking=True)
            e2.record(stream)
        e2.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(s2.elapsed_time(e2), world)
        fl = (mask_flops + attn_flops) * n_e2e * world
        e2e = {"value": fl / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int((hq.numel() + hk.numel() + hv.numel()) * esz),
               "d2h_bytes_per_step": int(q0.numel() * esz), "steps": n_e2e,
               "how": "per step: H2D of q, k, v (pinned), hip_mask, hip_sparse_attn, D2H of out"}
        sess.check()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x)

    mask_kernel = "mask_mma_kernel" if w.dtype != "f32" else "mask_fma_kernel"
    attn_kernel = "attn_mma_kernel" if prefill else "attn_fma_kernel"
    if prefill:
        dom_attn = attn_ms >= mask_ms
        dom_tf = attn_tf if dom_attn else mask_tf
        roofline = {"bound": "tensor", "kernel": attn_kernel if dom_attn else mask_kernel,
                    "achieved": dom_tf, "peak": tensor_peak, "peak_kind": f"{pk_kind} bf16 sustained",
                    "unit": "TFLOP/s", "frac": dom_tf / tensor_peak,
                    "traffic": traffic_from_profile(attn_kernel if dom_attn else mask_kernel, w.name),
                    "algorithmic_flops": attn_flops if dom_attn else mask_flops}
        value, unit, hib = step_tf, "TFLOP/s", True
    else:
        if one_launch:
            # one kernel does the whole step: its bytes are the mask's and the attention's
            fused_gbs = (mask_bytes + attn_bytes) / (mask_ms * 1e-3) / 1e9
            roofline = {"bound": "hbm", "kernel": mask_kernel + " (mask + attention)",
                        "achieved": fused_gbs, "peak": hbm, "peak_kind": pk_kind, "unit": "GB/s",
                        "frac": fused_gbs / hbm,
                        "traffic": traffic_from_profile(mask_kernel + "+attn", w.name),
                        "algorithmic_bytes": mask_bytes + attn_bytes}
        else:
            roofline = {"bound": "hbm", "kernel": mask_kernel, "achieved": mask_gbs,
                        "peak": hbm, "peak_kind": pk_kind, "unit": "GB/s", "frac": mask_gbs / hbm,
                        "traffic": traffic_from_profile(mask_kernel, w.name),
                        "algorithmic_bytes": mask_bytes}
        value, unit, hib = us_layer, "us/layer", False
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": total_ms / steps,
        "higher_is_better": hib, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if dt == torch.bfloat16 else "f32",
        "data": "synthetic (seeded AR(1) keys/values, Gaussian queries, needle keys)",
        "config": config_of(w, layers),
        "roofline": roofline,
        "step_roofline": {"bound": "hbm", "achieved": step_gbs, "peak": hbm, "unit": "GB/s",
                          "frac": step_gbs / hbm, "algorithmic_bytes": mask_bytes + attn_bytes},
        "kernels": {"how": "CUDA event nodes around each call, last full graph replay of the timed region",
                    "step_call": "hip_mask_sparse_attn" if fused else "hip_mask + hip_sparse_attn",
                    "one_launch": one_launch,
                    "mask_kernel": mask_kernel, "attn_kernel": None if one_launch else attn_kernel,
                    "mask_us": mask_ms * 1e3, "mask_bytes": mask_bytes, "mask_gbs": mask_gbs,
                    "mask_tflops": mask_tf, "mask_flops": mask_flops, "scored_candidates": scored,
                    "attn_us": attn_ms * 1e3, "attn_bytes": attn_bytes, "attn_gbs": attn_gbs,
                    "attn_tflops": attn_tf, "attn_flops": attn_flops},
        "gpu_launches": launches_per_step * steps,
        "clocks": clk.summary(),
    }
    if two_call:
        line["kernels"]["two_calls"] = two_call
    if prefill:
        line["step_tflops"] = step_tf
        line["us_per_layer"] = us_layer
    if e2e:
        line["e2e"] = e2e
    if cpu:
        line["cpu_baseline"] = cpu
    del g, g_ev, g_rem
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    global HEAD_MASKS
    args = parse()
    HEAD_MASKS = args.head_masks
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores alone; no process group
        reference_arm(args, w, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
