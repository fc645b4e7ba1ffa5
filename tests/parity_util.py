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


def unit_range(sh, unit: int):
    """(N, n0): key blocks in the causal range of a mask row, and its chunk count."""
    nqb = -(-sh.q_len // sh.block_q)
    qb = unit % nqb
    i1 = min(qb * sh.block_q + sh.block_q, sh.q_len)
    tc = min(sh.q_pos0 + i1, sh.seq_len)
    n = -(-tc // sh.block_k)
    return n, min(sh.topk // sh.block_k, n)


def union_row(sh, unit: int, kept) -> np.ndarray:
    """Ascending block ids of kept plus the sink blocks [0, ceil(sink/b_k)) and
    the window blocks over keys [max(0, q_first - window + 1), q_last]."""
    nqb = -(-sh.q_len // sh.block_q)
    qb = unit % nqb
    bk = sh.block_k
    n, _ = unit_range(sh, unit)
    q_first = sh.q_pos0 + qb * sh.block_q
    q_last = sh.q_pos0 + min(qb * sh.block_q + sh.block_q, sh.q_len) - 1
    s = set(int(c) for c in kept) | set(range(min(-(-sh.sink // bk), n)))
    if sh.window > 0:
        s |= set(range(max(0, q_first - sh.window + 1) // bk, min(q_last // bk + 1, n)))
    return np.array(sorted(s), dtype=np.int64)


def replay_selection(q, k, sh, unit: int, kept, tol_raw: float = 0.0):
    """Check that ``kept`` (a mask row's chosen blocks before the sink/window
    union) is a result of the rounds ("Author Rebuttal to the Reviewer RsGC",
    Q2, steps 1-4) in which every cut is right up to ``tol_raw`` (raw q.k
    units). Returns None when valid, else the first violation as text.

    The rounds are replayed with the oracle's block scores (step 3). In each
    round the candidates that hold a kept block must be among the n0 chosen;
    the remaining places go to the best other candidates by (score desc, start
    asc), and every chosen candidate must score at least the best unchosen one
    minus ``tol_raw``. With tol_raw = 0 this accepts exactly the selection by
    (score desc, start asc) and nothing else. With tol_raw > 0 it accepts
    near-tie swaps, and could reject a valid row only where a near-tie chunk
    that was chosen in one round loses both halves in a later one."""
    kept = np.asarray(kept, dtype=np.int64)
    n, n0 = unit_range(sh, unit)
    if kept.size != n0:
        return f"{kept.size} kept blocks, expected n0 = {n0}"
    if kept.size and (np.any(np.diff(kept) <= 0) or kept[0] < 0 or kept[-1] >= n):
        return "kept blocks not strictly ascending within [0, N)"
    i = np.arange(n0, dtype=np.int64)
    s, e = i * n // n0, (i + 1) * n // n0
    rnd = 0
    while n0 and np.max(e - s) > 1:
        ln = e - s
        split = ln > 1
        m = s + ln // 2
        cs = np.concatenate([s, m[split]])
        ce = np.concatenate([np.where(split, m, e), e[split]])
        o = np.argsort(cs, kind="stable")
        cs, ce = cs[o], ce[o]
        sc = oracle.block_scores(q, k, sh, unit, cs + (ce - cs) // 2).astype(np.float64)
        want = min(n0, cs.size)
        required = np.searchsorted(kept, ce) > np.searchsorted(kept, cs)
        if int(required.sum()) > want:
            return f"round {rnd}: {int(required.sum())} candidates hold kept blocks, more than {want}"
        order = np.lexsort((cs, -sc))  # score desc, then start asc
        chosen = required.copy()
        fill = want - int(required.sum())
        for c in order:
            if fill == 0:
                break
            if not chosen[c]:
                chosen[c] = True
                fill -= 1
        if cs.size > n0:
            exact = np.zeros(cs.size, bool)
            exact[order[:n0]] = True
            if not np.array_equal(exact, chosen):
                worst = float(np.max(sc[~chosen]) - np.min(sc[chosen]))
                if tol_raw == 0.0 or not worst < tol_raw:
                    return (f"round {rnd}: an unchosen candidate outscores a chosen one by "
                            f"{worst:.3g} (allowed below {tol_raw:.3g})")
        s, e = cs[chosen], ce[chosen]
        rnd += 1
    if not np.array_equal(np.sort(s), kept):
        return "the replayed chunks are not the kept blocks"
    return None


def compare_masks(idx_gpu: np.ndarray, idx_ref: np.ndarray, gap: np.ndarray, exact: bool = True,
                  validate=None) -> dict:
    """Mask rows against the oracle.

    The method's rule: rows match bit-exactly except where the oracle's cut
    gap is below 1e-3 (q.k/sqrt(d) units), and such rows stay under 0.5 % of
    all rows. Every mismatched row must also be a valid selection:
    ``validate(r, gpu_row)`` (see ``gpu_validator``) returns None for a valid
    row.
    With ``exact`` (the kernels select by the canonical scores, so they claim
    bit-exact rows) no row may differ at all."""
    g = idx_gpu.reshape(idx_ref.shape)
    diff = np.any(g != idx_ref, axis=1)
    n_diff = int(diff.sum())
    bad = diff & ~(gap < NEAR_TIE)
    stats = {"rows": int(idx_ref.shape[0]), "mismatched": n_diff,
             "near_tie_rows": int((gap < NEAR_TIE).sum()), "bad": int(bad.sum())}
    invalid = []
    if validate is not None:
        for r in np.nonzero(diff)[0][:16]:
            msg = validate(int(r), g[r])
            if msg is not None:
                invalid.append((int(r), msg))
    stats["invalid"] = invalid
    assert stats["bad"] == 0, f"mask rows differ away from near-ties: {np.nonzero(bad)[0][:10]} {stats}"
    assert not invalid, f"mismatched rows that are no valid selection: {invalid[:4]} {stats}"
    assert n_diff <= NEAR_TIE_MAX_FRAC * idx_ref.shape[0], stats
    if exact:
        assert n_diff == 0, f"the kernels select by canonical scores, yet rows differ: {stats}"
    return stats


def gpu_validator(x_q, x_k, osh, session, q, k, units=None):
    """``validate(r, gpu_row)`` for compare_masks: the GPU's kept blocks of
    row r (one more mask call with no sink and no window, which leaves the
    rounds unchanged) must rebuild the GPU row with the sink and window blocks,
    and must be a valid selection up to near-ties (replay_selection with the
    1e-3 near-tie bound in raw q.k units). Row r of the compared rows is
    unit ``units[r]`` when a sample of units is compared."""
    cache = {}

    def kept_rows():
        if "rows" not in cache:
            import torch
            sink, window = session.p.sink, session.p.window
            session.set(sink=0, window=0)
            try:
                idx = session.mask(q, k)
                torch.cuda.synchronize()
                session.check()
            finally:
                session.set(sink=sink, window=window)
            cache["rows"] = idx.cpu().numpy().reshape(-1, idx.shape[-1])
        return cache["rows"]

    tol = NEAR_TIE * float(np.sqrt(osh.head_dim))

    def validate(r, gpu_row):
        r = int(units[r]) if units is not None else r
        kept = kept_rows()[r]
        kept = kept[1:1 + kept[0]].astype(np.int64)
        nnz = int(gpu_row[0])
        if nnz < 0 or nnz >= gpu_row.size or np.any(gpu_row[1 + nnz:] != -1):
            return "nnz out of range or padding not -1"
        if not np.array_equal(union_row(osh, r, kept), gpu_row[1:1 + nnz]):
            return "the row is not the kept blocks plus the sink and window blocks"
        return replay_selection(x_q, x_k, osh, r, kept, tol)

    return validate


def compare_outputs(out_gpu: np.ndarray, out_ref: np.ndarray, dtype: str) -> dict:
    err = np.abs(out_gpu.astype(np.float64) - out_ref.astype(np.float64))
    mx, mean = float(err.max()), float(err.mean())
    tmax, tmean = TOL[dtype]
    assert np.all(np.isfinite(out_gpu)), "non-finite outputs"
    assert mx <= tmax and mean <= tmean, f"max {mx:.3g} mean {mean:.3g} (tol {tmax}, {tmean})"
    return {"max_abs": mx, "mean_abs": mean}
