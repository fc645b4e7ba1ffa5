"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np

import oracle
from hierarchically_pruned_sparse_b200 import binding as hb
from hierarchically_pruned_sparse_b200 import workloads as W

# Attention tolerance for bf16 inputs (stated with the method's targets):
# max |gpu - oracle| <= 2e-2 and mean <= 5e-3. For fp32 inputs the only error
# sources are fp32 accumulation and exp2f over <= 10^6 keys: 2e-4 / 2e-5.
# fp8 e5m2 K/V widen exactly and the outputs are bf16: the bf16 tolerance.
TOL = {"bf16": (2e-2, 5e-3), "f32": (2e-4, 2e-5), "e5m2": (2e-2, 5e-3)}
NEAR_TIE = 1e-3          # rows whose oracle cut gap is below this may differ
NEAR_TIE_MAX_FRAC = 0.005


def torch_inputs(x: dict, w: W.Workload, step: int = 0):
    """Device q, k, v of a workload (e5m2: bf16 q, uint8 code k and v)."""
    import torch
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    kt = torch.uint8 if w.dtype == "e5m2" else dt
    q = torch.from_numpy(np.ascontiguousarray(x["q"][step])).to("cuda").to(dt).contiguous()
    k = torch.from_numpy(x["k"]).to("cuda").to(kt).contiguous()
    v = torch.from_numpy(x["v"]).to("cuda").to(kt).contiguous()
    return q, k, v


def oracle_kv(x: dict, w: W.Workload):
    """float32 k, v for the oracle: the oracle decodes e5m2 codes itself."""
    if w.dtype == "e5m2":
        return oracle.decode_e5m2(x["k"]), oracle.decode_e5m2(x["v"])
    return x["k"], x["v"]


def shapes(w: W.Workload, step: int = 0):
    """(oracle shape, binding kwargs) of step ``step`` of a workload."""
    T = w.seq_len + (step if w.kind == "decode" else 0)
    q_len = w.q_len
    q_pos0 = T - 1 if w.kind == "decode" else 0
    common = dict(batch=w.batch, n_qheads=w.n_qheads, n_kvheads=w.n_kvheads, seq_len=T,
                  q_len=q_len, q_pos0=q_pos0, block_q=w.block_q, block_k=w.block_k,
                  topk=w.topk, sink=w.sink, window=w.window, mask_len=w.seq_len,
                  kv_capacity=w.capacity)
    osh = oracle.shape(head_dim=w.head_dim, **common)
    code = {"bf16": hb.HIPS_BF16, "f32": hb.HIPS_F32, "e5m2": hb.HIPS_BF16_E5M2}[w.dtype]
    bkw = dict(dtype=code, **common)
    return osh, bkw


def compare_masks(idx_gpu: np.ndarray, idx_ref: np.ndarray, gap: np.ndarray) -> dict:
    """Bit-exact rows except near-ties; returns counts and asserts the rule."""
    g = idx_gpu.reshape(idx_ref.shape)
    diff = np.any(g != idx_ref, axis=1)
    n_diff = int(diff.sum())
    bad = diff & ~(gap < NEAR_TIE)
    stats = {"rows": int(idx_ref.shape[0]), "mismatched": n_diff,
             "near_tie_rows": int((gap < NEAR_TIE).sum()), "bad": int(bad.sum())}
    assert stats["bad"] == 0, f"mask rows differ away from near-ties: {np.nonzero(bad)[0][:10]} {stats}"
    assert n_diff <= NEAR_TIE_MAX_FRAC * idx_ref.shape[0], stats
    return stats


def compare_outputs(out_gpu: np.ndarray, out_ref: np.ndarray, dtype: str) -> dict:
    err = np.abs(out_gpu.astype(np.float64) - out_ref.astype(np.float64))
    mx, mean = float(err.max()), float(err.mean())
    tmax, tmean = TOL[dtype]
    assert np.all(np.isfinite(out_gpu)), "non-finite outputs"
    assert mx <= tmax and mean <= tmean, f"max {mx:.3g} mean {mean:.3g} (tol {tmax}, {tmean})"
    return {"max_abs": mx, "mean_abs": mean}
