"""CPU checks of the mask-row validator the GPU parity tests use.

``parity_util.replay_selection`` replays the halving rounds ("Author Rebuttal
to the Reviewer RsGC", Q2, steps 1-4) along the selection path a row implies
and checks each cut with the oracle's block scores. It must accept the
oracle's own rows exactly and reject rows with a wrong block, a missing
block, an extra block or a reversed tie; ``union_row`` must rebuild the
oracle's idx row from the kept blocks plus the sink and window blocks.
"""
import numpy as np
import pytest

import oracle
from hierarchically_pruned_sparse_b200 import workloads as W
from tests import parity_util as pu

CASES = [
    # decode, GQA 4:1, ragged T, sink + window
    W.Workload("v1", "decode", 1, 4, 1, 64, 1001, 1, 2, 64, 8, 20, "f32", 2, "uniform"),
    # two KV heads, 4-key blocks, N / n0 not a power of two
    W.Workload("v2", "decode", 2, 4, 2, 64, 700, 1, 4, 96, 0, 0, "f32"),
    # prefill query blocks of 8 rows, causal ranges of every length
    W.Workload("v3", "prefill", 1, 2, 1, 64, 300, 8, 2, 32, 4, 12, "f32"),
]


def _kept(x, w, sh):
    """The oracle's kept blocks (a run without sink and window) and its idx."""
    bare = oracle.shape(head_dim=w.head_dim, **{**_kw(w), "sink": 0, "window": 0})
    kept, _, _ = oracle.mask(x["q"][0], x["k"], bare)
    idx, gap, _ = oracle.mask(x["q"][0], x["k"], sh)
    return kept, idx, gap


def _kw(w):
    T = w.seq_len
    return dict(batch=w.batch, n_qheads=w.n_qheads, n_kvheads=w.n_kvheads, seq_len=T,
                q_len=w.q_len, q_pos0=T - 1 if w.kind == "decode" else 0, block_q=w.block_q,
                block_k=w.block_k, topk=w.topk, sink=w.sink, window=w.window)


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_validator_accepts_the_oracle_rows_and_rebuilds_the_union(w):
    x = W.make_inputs(w)
    sh = oracle.shape(head_dim=w.head_dim, **_kw(w))
    kept, idx, _ = _kept(x, w, sh)
    for u in range(idx.shape[0]):
        row = kept[u, 1:1 + kept[u, 0]]
        assert pu.replay_selection(x["q"][0], x["k"], sh, u, row) is None, u
        assert np.array_equal(pu.union_row(sh, u, row), idx[u, 1:1 + idx[u, 0]]), u


@pytest.mark.parametrize("w", CASES[:2], ids=[w.name for w in CASES[:2]])
def test_validator_rejects_planted_rows(w):
    x = W.make_inputs(w)
    sh = oracle.shape(head_dim=w.head_dim, **_kw(w))
    kept, _, _ = _kept(x, w, sh)
    rng = np.random.default_rng(1)
    for u in range(kept.shape[0]):
        row = kept[u, 1:1 + kept[u, 0]].astype(np.int64)
        n, n0 = pu.unit_range(sh, u)
        if n0 == n:
            continue  # every block is kept: no other row is possible
        outside = np.setdiff1d(np.arange(n), row)
        # one kept block swapped for a block the oracle dropped
        for _ in range(3):
            bad = row.copy()
            bad[rng.integers(row.size)] = rng.choice(outside)
            bad = np.unique(bad)
            msg = pu.replay_selection(x["q"][0], x["k"], sh, u, bad)
            assert msg is not None, (u, bad)
        assert pu.replay_selection(x["q"][0], x["k"], sh, u, row[1:]) is not None
        extra = np.unique(np.concatenate([row, outside[:1]]))
        assert pu.replay_selection(x["q"][0], x["k"], sh, u, extra) is not None


def test_validator_applies_the_tie_rule_and_the_tolerance():
    # all keys equal: every cut is a tie, and the rule keeps the lowest blocks
    T, bk, topk, d = 64, 1, 8, 64
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 1, d)).astype(np.float32)
    k = np.ascontiguousarray(np.broadcast_to(rng.standard_normal(d).astype(np.float32),
                                             (1, 1, T, d)))
    sh = oracle.shape(batch=1, n_qheads=1, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                      q_pos0=T - 1, block_q=1, block_k=bk, topk=topk)
    idx, _, _ = oracle.mask(q, k, sh)
    row = idx[0, 1:1 + idx[0, 0]]
    assert list(row) == list(range(topk))
    assert pu.replay_selection(q, k, sh, 0, row) is None
    # block 8 in place of block 7: the same score, the higher start -- a
    # reversed tie, invalid exactly and valid once near-ties are allowed
    alt = np.array(list(range(topk - 1)) + [topk], np.int64)
    assert pu.replay_selection(q, k, sh, 0, alt) is not None
    assert pu.replay_selection(q, k, sh, 0, alt, tol_raw=1e-3) is None


def test_compare_masks_rules():
    ref = np.array([[2, 0, 1, -1], [2, 1, 2, -1]], np.int32)
    same = ref.copy()
    st = pu.compare_masks(same, ref, np.array([1.0, 1.0]))
    assert st["mismatched"] == 0
    other = ref.copy()
    other[1, 2] = 3
    with pytest.raises(AssertionError):  # away from a near-tie
        pu.compare_masks(other, ref, np.array([1.0, 1.0]), exact=False)
    with pytest.raises(AssertionError):  # exactness claimed
        pu.compare_masks(other, ref, np.array([1.0, 1e-5]))
    with pytest.raises(AssertionError):  # near-tie, but no valid selection
        pu.compare_masks(other, ref, np.array([1.0, 1e-5]), exact=False,
                         validate=lambda r, row: "planted")


def test_every_planted_oracle_slip_still_has_its_target():
    # tests/oracle_mutants.py plants each slip by replacing one exact piece of
    # the oracle's text; a target that no longer occurs exactly once would
    # silently drop that slip from the check
    from tests import oracle_mutants
    assert oracle_mutants.stale_targets() == []
