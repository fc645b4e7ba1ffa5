"""Seeded synthetic workloads for hierarchically pruned attention.

This module only describes workload shapes and draws random inputs. It holds
none of the method's arithmetic (no scoring, no pruning, no attention), so the
CPU oracle tests and the CUDA parity tests can both take their inputs from it.

Input recipe (the pages run on PG19 / LongBench text with trained Llama3.1-8B
weights, neither of which is available here; these synthetic inputs stand in
for them):

* ``numpy.random.default_rng(seed)`` (PCG64), ``standard_normal`` in float32.
* K and V are AR(1) sequences along the time axis, drawn head-major:
  x_0 ~ N(0, I), x_t = 0.9 x_{t-1} + 0.436 e_t. The stationary variance is
  0.436^2 / (1 - 0.81) ~= 1.0005, and neighbouring keys are correlated,
  which gives the "attention locality" that HiP relies on (HiP paper,
  Approach; rebuttal to reviewer RsGC, Q2).
* Decode queries are i.i.d. N(0, I). Prefill queries are AR(1) like K and V.
* Needles: the j-th needle of KV head g is aligned with query head
  g*G + (j mod G) and replaces the key at its position with
  3 q/|q| + 0.1 N(0, I). Positions are uniform without replacement over
  [0, T) ("uniform"), or at distances floor(exp(U(0, ln(T-1)))) before the
  query, resampled on collision ("loguniform").
* Draw order: all of K, then V, then Q, then needle positions and noise;
  the draws of one head are taken in [dim][t] order.
* bf16 workloads round every tensor to bf16 (round to nearest even) after
  drawing; the float32 arrays returned hold exactly the bf16 values.
* e5m2 workloads (an fp8 KV cache) round q to bf16 and return k and v as
  uint8 fp8 e5m2 codes of the bf16 values, each rounded once to the nearest
  e5m2 value (ties to even). Needles are coded the same way.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch
from scipy.signal import lfilter

AR_RHO = np.float32(0.9)
AR_SIGMA = np.float32(0.436)
NEEDLE_GAIN = np.float32(3.0)
NEEDLE_NOISE = np.float32(0.1)


@dataclass(frozen=True)
class Workload:
    """Shape and recipe of one synthetic attention workload.

    ``seq_len`` is the key count T when the mask is computed. Decode queries
    sit at position T-1; with ``refresh`` > 1 the cache grows by one key per
    step and the mask of step 0 is reused for ``refresh`` steps.
    """

    name: str
    kind: str  # "decode" | "prefill"
    batch: int
    n_qheads: int
    n_kvheads: int
    head_dim: int
    seq_len: int
    block_q: int
    block_k: int
    topk: int
    sink: int
    window: int
    dtype: str  # "f32" | "bf16" | "e5m2" (bf16 q, fp8 e5m2 k and v)
    needles: int = 0  # per KV head
    needle_mode: str = "none"  # "uniform" | "loguniform" | "none"
    refresh: int = 1  # decode steps served by one mask (r_m)
    seed: int = 0  # batch entry b uses seed + b

    @property
    def group(self) -> int:
        return self.n_qheads // self.n_kvheads

    @property
    def q_len(self) -> int:
        return 1 if self.kind == "decode" else self.seq_len

    @property
    def capacity(self) -> int:
        """Keys held per sequence (the mask-time keys plus decode growth)."""
        return self.seq_len + (self.refresh - 1 if self.kind == "decode" else 0)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: small fp32 decode, Llama-3.1-8B-shaped decode at 128k,
# causal prefill at 32k, batched decode with mask reuse, and decode at 1M.
DECODE_8K_F32 = Workload("decode_T8k_h1_f32", "decode", 1, 1, 1, 128, 8192,
                         1, 16, 512, 0, 0, "f32", needles=4, needle_mode="uniform")
DECODE_128K = Workload("decode_T128k_h32x8_bf16", "decode", 1, 32, 8, 128, 131072,
                       1, 2, 2048, 128, 1024, "bf16", needles=16, needle_mode="uniform")
PREFILL_32K = Workload("prefill_T32k_h32x8_bf16", "prefill", 1, 32, 8, 128, 32768,
                       64, 2, 2048, 128, 1024, "bf16")
DECODE_B16_REUSE = Workload("decode_B16_T128k_h32x8_bf16_rm8", "decode", 16, 32, 8, 128,
                            131072, 1, 2, 2048, 128, 1024, "bf16", needles=16,
                            needle_mode="uniform", refresh=8)
DECODE_1M = Workload("decode_T1M_h32x8_bf16", "decode", 1, 32, 8, 128, 1048576,
                     1, 4, 4096, 256, 2048, "bf16", needles=64, needle_mode="loguniform")

# the 128k decode step over an fp8 e5m2 KV cache (bf16 queries)
DECODE_128K_E5M2 = dataclasses.replace(DECODE_128K, name="decode_T128k_h32x8_e5m2", dtype="e5m2")

WORKLOADS = {w.name: w for w in (DECODE_8K_F32, DECODE_128K, PREFILL_32K,
                                 DECODE_B16_REUSE, DECODE_1M, DECODE_128K_E5M2)}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even); returns float32 values."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of bf16-exact float32 values, as uint16."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def e5m2_codes(x: np.ndarray) -> np.ndarray:
    """fp8 e5m2 codes (uint8) of float32 values, rounded once to the nearest
    e5m2 value (ties to even): 2 mantissa bits kept on the float32 encoding,
    multiples of 2^-16 below 2^-14 (the subnormals). The rounded value is
    exact in binary16, whose encoding's upper byte is the code. Values must
    stay below the e5m2 range limit."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u + np.uint32(0xFFFFF) + ((u >> np.uint32(21)) & np.uint32(1))) & np.uint32(0xFFE00000)
    y = r.view(np.float32).copy()
    small = np.abs(x) < np.float32(2.0 ** -14)
    y[small] = (np.rint(x[small].astype(np.float64) * 2.0 ** 16) / 2.0 ** 16).astype(np.float32)
    return (y.astype(np.float16).view(np.uint16) >> np.uint16(8)).astype(np.uint8)


def _ar1(rng: np.random.Generator, heads: int, length: int, dim: int) -> np.ndarray:
    """[heads, length, dim] AR(1) sequences along ``length`` (float32).

    The draws of one head are taken in [dim][t] order. x_0 = e_0 and
    x_t = 0.9 x_{t-1} + 0.436 e_t, run as a first-order IIR filter over t
    (direct form II transposed, with state 0.9 x_0 entering at t = 1).
    """
    e = rng.standard_normal((heads, dim, length), dtype=np.float32)
    if length > 1:
        zi = (AR_RHO * e[:, :, :1]).astype(np.float32)
        e[:, :, 1:], _ = lfilter(np.array([AR_SIGMA], np.float32),
                                 np.array([1.0, -AR_RHO], np.float32),
                                 e[:, :, 1:], axis=-1, zi=zi)
    return torch.from_numpy(e).transpose(1, 2).contiguous().numpy()


def _needle_positions(rng: np.random.Generator, w: Workload, count: int, qpos: int) -> np.ndarray:
    if w.needle_mode == "uniform":
        return rng.choice(w.seq_len, size=count, replace=False)
    if w.needle_mode == "loguniform":
        used: set[int] = set()
        out = []
        hi = np.log(qpos) if qpos > 1 else 0.0
        while len(out) < count:
            dist = int(np.floor(np.exp(rng.uniform(0.0, hi))))
            pos = qpos - max(dist, 1)
            if pos < 0 or pos in used:
                continue
            used.add(pos)
            out.append(pos)
        return np.asarray(out, dtype=np.int64)
    raise ValueError(w.needle_mode)


def make_sequence(w: Workload, b: int = 0) -> dict:
    """Inputs of batch entry ``b`` (seed ``w.seed + b``).

    Returns float32 arrays ``k``/``v`` [Hkv, capacity, d] (uint8 e5m2 codes
    for e5m2 workloads) and ``q``
    [steps, Hq, Lq, d] (steps = ``refresh`` for decode, 1 for prefill), plus
    ``needle_pos`` [Hkv, needles].
    """
    rng = np.random.default_rng(w.seed + b)
    d, hkv, hq, cap = w.head_dim, w.n_kvheads, w.n_qheads, w.capacity
    k = _ar1(rng, hkv, cap, d)
    v = _ar1(rng, hkv, cap, d)
    if w.kind == "decode":
        q = rng.standard_normal((w.refresh, hq, 1, d), dtype=np.float32)
    else:
        q = _ar1(rng, hq, w.seq_len, d)[None]
    if w.dtype in ("bf16", "e5m2"):
        k, v, q = bf16_round(k), bf16_round(v), bf16_round(q)
    needle_pos = np.zeros((hkv, w.needles), dtype=np.int64)
    if w.needles:
        if w.kind != "decode":
            raise ValueError("needles are defined for decode workloads only")
        g = w.group
        qpos = w.seq_len - 1
        for h in range(hkv):
            pos = _needle_positions(rng, w, w.needles, qpos)
            noise = rng.standard_normal((w.needles, d), dtype=np.float32)
            for j in range(w.needles):
                qv = q[0, h * g + (j % g), 0]
                key = NEEDLE_GAIN * qv / np.float32(np.linalg.norm(qv)) + NEEDLE_NOISE * noise[j]
                k[h, pos[j]] = bf16_round(key) if w.dtype in ("bf16", "e5m2") else key
            needle_pos[h] = pos
    if w.dtype == "e5m2":
        k, v = e5m2_codes(k), e5m2_codes(v)
    return {"q": q, "k": k, "v": v, "needle_pos": needle_pos}


def make_inputs(w: Workload) -> dict:
    """Whole-batch inputs: q [steps, B, Hq, Lq, d], k/v [B, Hkv, capacity, d]."""
    seqs = [make_sequence(w, b) for b in range(w.batch)]
    q = np.stack([s["q"] for s in seqs], axis=1)
    k = np.stack([s["k"] for s in seqs])
    v = np.stack([s["v"] for s in seqs])
    return {"q": q, "k": k, "v": v,
            "needle_pos": np.stack([s["needle_pos"] for s in seqs])}
