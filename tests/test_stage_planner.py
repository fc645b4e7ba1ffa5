"""The host planner of the pruning stages (hips_stage; "[Feature] Support
Efficient Sparse HiP Attention (InfiniteHiP)" stages) against a restatement
of its bounds, on the CPU.

For a schedule the planner must accept exactly the shapes whose lists fit
(every ranking stage at most 36864 chunks per mask row, at most
topk / block_k chunks before the iteration, bounds taken over the worst
mask row), size the workspace as the plain mask's plus one score array and
two chunk lists per mask row, and its bounds must hold for every mask row
of the shape: the chunk counts each stage really sees (restated here from
the stage rule, which keeps min(keep, count) chunks and cuts each into
pieces) never exceed them, so the kernels' device-side bound check cannot
fire.
"""
import numpy as np
import pytest

from hierarchically_pruned_sparse_b200 import binding as hb

MAX_CHUNKS = 36864


def _up(n):
    return (n + 255) // 256 * 256


def _bounds(stages, bk, topk, n_max):
    """(accepted, cap) of the planner's rule."""
    ranked = [s for s in stages if s[1] > 0]
    c_last = stages[-1][0] // bk
    n0max = topk // bk
    cap, kept, kept_c = n0max, 0, 1
    for t, (c_keys, k, _) in enumerate(ranked):
        c = c_keys // bk
        cands = -(-n_max // c) if t == 0 else kept * (kept_c // c)
        if cands > MAX_CHUNKS:
            return False, 0
        cap = max(cap, cands)
        kept, kept_c = min(k // c_keys, cands), c
    pieces = kept * (kept_c // c_last) if ranked else -(-n_max // c_last)
    if pieces > n0max or cap > (1 << 22):
        return False, 0
    return True, max(cap, pieces)


def _row_counts(stages, bk, n_blocks):
    """Chunk counts one mask row of n_blocks key blocks sees: per ranking
    stage, and the chunks the iteration starts from (any kept subset has the
    same counts, so the first chunks stand in for the best ones)."""
    chunks = [(0, n_blocks)]
    seen = []
    for c_keys, k, _ in stages:
        c = c_keys // bk
        chunks = [(p, min(p + c, e)) for s, e in chunks for p in range(s, e, c)]
        if k > 0:
            seen.append(len(chunks))
            chunks = chunks[:k // c_keys] if len(chunks) > k // c_keys else chunks
    return seen, len(chunks)


def _schedule(rng, bk):
    sizes = [bk * int(rng.choice([1, 2, 4, 8]))]
    for _ in range(int(rng.integers(0, 3))):
        sizes.insert(0, sizes[0] * int(rng.choice([1, 2, 4, 8])))
    out = []
    for c in sizes:
        keep = 0 if rng.random() < 0.3 else c * int(rng.choice([1, 4, 16, 64, 256, 1024]))
        out.append((c, keep, 1))
    return tuple(out)


def _cases():
    rng = np.random.default_rng(5)
    cases = []
    for _ in range(120):
        bk = int(rng.choice([1, 2, 4, 16]))
        kind = "decode" if rng.random() < 0.6 else "prefill"
        T = int(rng.choice([1000, 4096, 65536, 131072, 1 << 20]))
        if kind == "prefill":
            T = min(T, 8192)
        topk = bk * int(rng.choice([8, 64, 512, 1024, 2048]))
        cases.append((kind, T, bk, topk, _schedule(rng, bk)))
    return cases


@pytest.mark.parametrize("case", _cases())
def test_planner_accepts_exactly_the_bounded_schedules(case):
    kind, T, bk, topk, stages = case
    q_len = 1 if kind == "decode" else T
    bq = 1 if kind == "decode" else 64
    kw = dict(batch=1, n_qheads=8, n_kvheads=2, seq_len=T, q_len=q_len, q_pos0=T - q_len,
              dtype=hb.HIPS_BF16, block_q=bq, block_k=bk, topk=topk, sink=0, window=0)
    plain = hb.workspace_size(hb.params(**kw), hb.OP_MASK)
    staged = hb.workspace_size(hb.params(**kw, stages=stages), hb.OP_MASK)
    n_max = -(-T // bk)
    ok, cap = _bounds(stages, bk, topk, n_max)
    if plain == 0 or not ok:
        assert staged == 0, (case, staged)
        return
    units = 2 * -(-q_len // bq)
    want = _up(plain) + _up(units * cap * 4) + 2 * _up(units * (4 + 2 * cap) * 4)
    assert staged == want, (case, staged, want)
    # the bounds hold for every mask row: the last query block sees all keys,
    # earlier ones fewer
    rows = [n_max] if kind == "decode" else sorted({-(-min(T, (qb + 1) * bq) // bk)
                                                    for qb in range(0, -(-T // bq), 7)} | {n_max})
    for n in rows:
        seen, start = _row_counts(stages, bk, n)
        assert all(m <= cap for m in seen), (case, n, seen, cap)
        assert start <= topk // bk, (case, n, start)
