"""Pins of the CPU oracle to facts outside itself (no GPU needed).

* hand-traced worked examples of the iteration (tests/golden/);
* brute force: an independent recursive restatement of the pruning rule on
  integer inputs, where every score is exact, ties included;
* the dense special case (budget >= T keeps every block, so the output is
  textbook softmax attention);
* closed forms (monotone keys keep the last blocks; equal keys keep the
  first blocks through the tie rule) and the count invariant;
* the canonical fp32 dot: exact on one-hot inputs, within the fp32
  rounding bound of the exact dot, and the hand-derived order example;
* multi-stage pruning (InfiniteHiP stages): brute force on random schedules,
  a single keep-all stage of the initial chunks equals the plain iteration,
  and the monotone / equal-key closed forms through a three-stage schedule.
"""
import math
import os
import zlib

import numpy as np
import pytest

import oracle
from hierarchically_pruned_sparse_b200 import workloads as W
from tests import brute_force as bf


def _shape(**kw):
    return oracle.shape(**kw)


def _read_fixture(path):
    out = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            out.setdefault(key, []).append(vals)
    return out


# ---------------------------------------------------------------- golden


@pytest.mark.parametrize("name", ["hand_trace_T16_k4.txt", "hand_trace_ties_T16_k4.txt"])
def test_hand_traced_iteration(golden_dir, name):
    fx = _read_fixture(os.path.join(golden_dir, name))
    T = int(fx["T"][0][0])
    topk = int(fx["topk"][0][0])
    bk = int(fx["block_k"][0][0])
    scores = np.array([float(x) for x in fx["scores"][0]], dtype=np.float32)
    d = 64
    q = np.zeros((1, 1, 1, d), np.float32)
    q[..., 0] = 1.0
    rng = np.random.default_rng(3)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)  # junk outside element 0
    k[0, 0, :, 0] = scores
    sh = _shape(batch=1, n_qheads=1, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=topk)
    idx, gap, rounds = oracle.mask(q, k, sh)
    want = [int(x) for x in fx["expect_idx"][0]]
    assert idx[0, 0] == len(want)
    assert list(idx[0, 1:1 + len(want)]) == want
    assert np.all(idx[0, 1 + len(want):] == -1)
    assert gap[0] == pytest.approx(float(fx["expect_gap_raw"][0][0]) / math.sqrt(d), abs=0)
    assert rounds[0] == int(fx["expect_rounds"][0][0])


def test_canonical_dot_worked_order(golden_dir):
    fx = _read_fixture(os.path.join(golden_dir, "canonical_dot_order.txt"))
    d = int(fx["d"][0][0])
    q = np.zeros(d, np.float32)
    k = np.zeros(d, np.float32)
    for i, val in fx["q"]:
        q[int(i)] = np.float32(val)
    for i, val in fx["k"]:
        k[int(i)] = np.float32(val)
    want = np.float32(fx["expect"][0][0])
    assert want == np.float32(1.0) + np.float32(2.0 ** -23)
    assert oracle.canonical_dot(q, k) == want


def test_canonical_dot_one_hot_exact():
    # every element enters the sum exactly once (a dropped term or a wrong
    # index fails here)
    rng = np.random.default_rng(1)
    k = rng.standard_normal(128).astype(np.float32)
    for i in range(128):
        q = np.zeros(128, np.float32)
        q[i] = 1.0
        assert oracle.canonical_dot(q, k) == k[i]
        q[i] = -2.0
        assert oracle.canonical_dot(q, k) == np.float32(-2.0) * k[i]


def test_canonical_dot_rounding_bound():
    # |fl(q.k) - q.k| <= gamma_n * sum|q_i k_i| with n = 16 chained fmas + 3
    # tree levels (Higham, Accuracy and Stability of Numerical Algorithms, 3.1)
    rng = np.random.default_rng(2)
    u = 2.0 ** -24
    n = 16 + 3
    gamma = n * u / (1 - n * u)
    worst = 0.0
    for _ in range(2000):
        q = rng.standard_normal(128).astype(np.float32) * np.float32(rng.uniform(0.1, 10))
        k = rng.standard_normal(128).astype(np.float32)
        exact = float(np.dot(q.astype(np.float64), k.astype(np.float64)))
        bound = gamma * float(np.abs(q.astype(np.float64) * k).sum())
        err = abs(float(oracle.canonical_dot(q, k)) - exact)
        assert err <= bound
        worst = max(worst, err / bound)
    assert worst > 0  # the fp32 path really rounds (it is not an fp64 dot)


# ---------------------------------------------------------------- brute force


def _int_inputs(rng, B, Hq, Hkv, Lq, T, d=64, lo=-3, hi=3):
    q = rng.integers(lo, hi + 1, size=(B, Hq, Lq, d)).astype(np.float32)
    k = rng.integers(lo, hi + 1, size=(B, Hkv, T, d)).astype(np.float32)
    return q, k


def _brute_cases():
    rng = np.random.default_rng(7)
    cases = []
    for T in (1, 2, 3, 7, 16, 33, 64, 100, 257, 512):
        for bk in (1, 2, 4, 16):
            for _ in range(2):
                nb = -(-T // bk)
                topk = bk * int(rng.integers(1, max(2, nb + 2)))
                kind = "decode" if rng.random() < 0.5 else "prefill"
                Lq = 1 if kind == "decode" else T
                bq = 1 if kind == "decode" else int(rng.choice([1, 3, 8, 64]))
                G = int(rng.choice([1, 2]))
                sink = int(rng.choice([0, 0, bk, 5]))
                window = int(rng.choice([0, 0, 3, 2 * bk + 1]))
                cases.append((T, bk, topk, kind, Lq, bq, G, sink, window))
    return cases


@pytest.mark.parametrize("case", _brute_cases())
def test_mask_matches_brute_force_on_exact_scores(case):
    T, bk, topk, kind, Lq, bq, G, sink, window = case
    rng = np.random.default_rng(zlib.crc32(repr(case).encode()))
    B, Hkv = 2, 2
    q, k = _int_inputs(rng, B, Hkv * G, Hkv, Lq, T)
    q_pos0 = T - Lq
    sh = _shape(batch=B, n_qheads=Hkv * G, n_kvheads=Hkv, head_dim=64, seq_len=T, q_len=Lq,
                q_pos0=q_pos0, block_q=bq, block_k=bk, topk=topk, sink=sink, window=window)
    idx, gap, rounds = oracle.mask(q, k, sh)
    nqb = -(-Lq // bq)
    units = [(b, g, qb) for b in range(B) for g in range(Hkv) for qb in range(nqb)]
    if len(units) > 24:  # prefill with bq=1 on long T: sample rows
        pick = rng.choice(len(units), 24, replace=False)
    else:
        pick = range(len(units))
    for u in pick:
        b, g, qb = units[u]
        want, want_gap, want_rounds = bf.mask_row(
            q, k, b=b, g=g, qb=qb, group=G, block_q=bq, block_k=bk, topk=topk, q_len=Lq,
            q_pos0=q_pos0, seq_len=T, sink=sink, window=window)
        row = idx[u]
        assert row[0] == len(want), (case, u)
        assert list(row[1:1 + row[0]]) == want, (case, u)
        assert rounds[u] == want_rounds
        if math.isinf(want_gap):
            assert math.isinf(gap[u])
        else:
            assert gap[u] == pytest.approx(want_gap / math.sqrt(64), rel=1e-12, abs=0)


def test_float_mask_matches_brute_force_away_from_ties():
    # real-valued AR(1)-like data: decisions agree wherever the cut gap is
    # well above the fp32 rounding of a dot (1e-4 in q.k/sqrt(d) units)
    rng = np.random.default_rng(11)
    hits = 0
    for trial in range(30):
        T, bk, topk = 256, 2, 32
        q = rng.standard_normal((1, 2, 1, 128)).astype(np.float32)
        k = rng.standard_normal((1, 1, T, 128)).astype(np.float32)
        sh = _shape(batch=1, n_qheads=2, n_kvheads=1, head_dim=128, seq_len=T, q_len=1,
                    q_pos0=T - 1, block_q=1, block_k=bk, topk=topk)
        idx, gap, _ = oracle.mask(q, k, sh)
        qd, kd = q.astype(np.float64), k.astype(np.float64)

        def score(c):
            return max(float(qd[0, h, 0] @ kd[0, 0, j]) for h in range(2)
                       for j in range(c * bk, c * bk + bk))

        want, _, _ = bf.prune(score, T // bk, topk // bk)
        if gap[0] > 1e-4:
            hits += 1
            assert list(idx[0, 1:1 + idx[0, 0]]) == want
    assert hits >= 20


# ---------------------------------------------------------------- dense case


@pytest.mark.parametrize("kind", ["decode", "prefill"])
def test_budget_at_least_T_is_dense_attention(kind):
    rng = np.random.default_rng(5)
    B, Hq, Hkv, d, T, bk = 2, 4, 2, 128, 200, 4
    Lq = 1 if kind == "decode" else T
    bq = 1 if kind == "decode" else 16
    q = rng.standard_normal((B, Hq, Lq, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    sh = _shape(batch=B, n_qheads=Hq, n_kvheads=Hkv, head_dim=d, seq_len=T, q_len=Lq,
                q_pos0=T - Lq, block_q=bq, block_k=bk, topk=bk * (T // bk + 1))
    idx, gap, rounds = oracle.mask(q, k, sh)
    assert np.all(rounds == 0) and np.all(np.isinf(gap))
    out = oracle.attention(q, k, v, idx, sh).reshape(B, Hq, Lq, d)
    dense = oracle.attention(q, k, v, None, sh).reshape(B, Hq, Lq, d)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            pos = np.arange(Lq) + (T - Lq)
            allowed = np.arange(T)[None, :] <= pos[:, None]
            ref = bf.textbook_attention(q[b, h], k[b, h // G], v[b, h // G], allowed)
            np.testing.assert_allclose(out[b, h], ref, atol=2e-6, rtol=0)
            np.testing.assert_allclose(dense[b, h], ref, atol=2e-6, rtol=0)


def test_sparse_attention_is_masked_softmax_with_reuse_tail():
    # keys of the selected blocks below mask_len, plus every key appended
    # since the refresh (mask reuse over r_m decode steps)
    rng = np.random.default_rng(9)
    B, Hq, Hkv, d, bk = 1, 4, 2, 128, 2
    T0, steps = 300, 5
    cap = T0 + steps
    q = rng.standard_normal((B, Hq, 1, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, cap, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, cap, d)).astype(np.float32)
    sh0 = _shape(batch=B, n_qheads=Hq, n_kvheads=Hkv, head_dim=d, seq_len=T0, q_len=1,
                 q_pos0=T0 - 1, block_q=1, block_k=bk, topk=16, sink=4, window=8,
                 kv_capacity=cap)
    idx, _, _ = oracle.mask(q, k, sh0)
    for s in range(steps):
        T = T0 + s
        sh = _shape(batch=B, n_qheads=Hq, n_kvheads=Hkv, head_dim=d, seq_len=T, q_len=1,
                    q_pos0=T - 1, block_q=1, block_k=bk, topk=16, sink=4, window=8,
                    mask_len=T0, kv_capacity=cap)
        out = oracle.attention(q, k, v, idx, sh).reshape(B, Hq, d)
        for h in range(Hq):
            g = h // 2
            row = idx[g]
            keys = {j for c in row[1:1 + row[0]] for j in range(c * bk, c * bk + bk) if j < T0}
            keys |= set(range(T0, T))
            allowed = np.zeros((1, cap), bool)
            allowed[0, sorted(keys)] = True
            ref = bf.textbook_attention(q[0, h], k[0, g], v[0, g], allowed)
            np.testing.assert_allclose(out[0, h], ref[0], atol=2e-6, rtol=0)


# ---------------------------------------------------------------- closed forms


@pytest.mark.parametrize("bk,topk,T,G", [(1, 8, 256, 1), (2, 64, 1024, 4), (16, 512, 8192, 1),
                                         (4, 128, 4096, 2)])
def test_monotone_keys_keep_last_blocks(bk, topk, T, G):
    d = 128
    q = np.ones((1, G, 1, d), np.float32)
    k = np.broadcast_to(((np.arange(T) + 1) / T).astype(np.float32)[:, None], (T, d))
    k = np.ascontiguousarray(k)[None, None]
    sh = _shape(batch=1, n_qheads=G, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=topk)
    idx, _, rounds = oracle.mask(q, k, sh)
    n0, N = topk // bk, T // bk
    assert list(idx[0, 1:1 + idx[0, 0]]) == list(range(N - n0, N))
    assert rounds[0] == int(math.log2(N // n0))


def test_monotone_keys_prefill_each_block_keeps_its_last_blocks():
    d, T, bq, bk, topk = 128, 1024, 64, 2, 128
    q = np.ones((1, 1, T, d), np.float32)
    k = np.ascontiguousarray(np.broadcast_to(((np.arange(T) + 1) / T).astype(np.float32)[:, None],
                                             (T, d)))[None, None]
    sh = _shape(batch=1, n_qheads=1, n_kvheads=1, head_dim=d, seq_len=T, q_len=T, q_pos0=0,
                block_q=bq, block_k=bk, topk=topk)
    idx, _, _ = oracle.mask(q, k, sh)
    for qb in range(T // bq):
        N = (qb * bq + bq) // bk
        n0 = min(topk // bk, N)
        assert list(idx[qb, 1:1 + idx[qb, 0]]) == list(range(N - n0, N))


@pytest.mark.parametrize("bk,topk,T", [(1, 8, 64), (2, 64, 1024), (16, 512, 8192)])
def test_equal_keys_keep_first_blocks(bk, topk, T):
    d = 128
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 1, 1, d)).astype(np.float32)
    k = np.ascontiguousarray(np.broadcast_to(rng.standard_normal(d).astype(np.float32), (T, d)))
    sh = _shape(batch=1, n_qheads=1, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=topk)
    idx, gap, _ = oracle.mask(q, k[None, None], sh)
    assert list(idx[0, 1:1 + idx[0, 0]]) == list(range(topk // bk))
    assert gap[0] == 0.0


@pytest.mark.parametrize("T,bk,topk", [(8192, 16, 512), (4096, 2, 2048), (1000, 4, 64),
                                       (64, 2, 128), (131072, 2, 2048)])
def test_count_invariant_decode(T, bk, topk):
    rng = np.random.default_rng(T)
    d = 128
    q = rng.standard_normal((1, 4, 1, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    sh = _shape(batch=1, n_qheads=4, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=topk)
    idx, _, _ = oracle.mask(q, k, sh)
    N = -(-T // bk)
    n0 = min(topk // bk, N)
    blocks = idx[0, 1:1 + idx[0, 0]]
    assert idx[0, 0] == n0
    assert np.all(np.diff(blocks) > 0) and blocks[0] >= 0 and blocks[-1] < N
    if T % bk == 0:
        assert n0 * bk == min(topk, T)


def test_count_invariant_prefill_with_ragged_tail():
    rng = np.random.default_rng(4)
    d, T, bq, bk, topk = 128, 1000, 64, 2, 256
    q = rng.standard_normal((1, 2, T, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    sh = _shape(batch=1, n_qheads=2, n_kvheads=1, head_dim=d, seq_len=T, q_len=T, q_pos0=0,
                block_q=bq, block_k=bk, topk=topk)
    idx, _, _ = oracle.mask(q, k, sh)
    for qb in range(-(-T // bq)):
        t_c = min(qb * bq + bq, T)
        N = -(-t_c // bk)
        assert idx[qb, 0] == min(topk // bk, N)
        blocks = idx[qb, 1:1 + idx[qb, 0]]
        assert np.all(np.diff(blocks) > 0) and blocks[-1] < N


def test_sink_and_window_blocks_always_present():
    rng = np.random.default_rng(8)
    d, T, bk = 128, 4096, 2
    q = rng.standard_normal((1, 4, 1, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    sh = _shape(batch=1, n_qheads=4, n_kvheads=1, head_dim=d, seq_len=T, q_len=1, q_pos0=T - 1,
                block_q=1, block_k=bk, topk=256, sink=128, window=1024)
    idx, _, _ = oracle.mask(q, k, sh)
    plain = _shape(batch=1, n_qheads=4, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                   q_pos0=T - 1, block_q=1, block_k=bk, topk=256)
    idx0, _, _ = oracle.mask(q, k, plain)
    got = set(idx[0, 1:1 + idx[0, 0]])
    want = set(idx0[0, 1:1 + idx0[0, 0]]) | set(range(64)) | set(range((T - 1024) // 2, T // 2))
    assert got == want
    assert idx[0, 0] <= oracle.idx_cap(sh)


@pytest.mark.parametrize("T,bk,topk", [(8192, 16, 512), (131072, 2, 2048), (4096, 4, 256)])
def test_scored_candidates_closed_form(T, bk, topk):
    # equal-length chunks: every round scores exactly 2 n0 candidates
    rng = np.random.default_rng(1)
    d = 128
    q = rng.standard_normal((1, 2, 1, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    sh = _shape(batch=1, n_qheads=2, n_kvheads=1, head_dim=d, seq_len=T, q_len=1, q_pos0=T - 1,
                block_q=1, block_k=bk, topk=topk)
    _, _, rounds, scored = oracle.mask(q, k, sh, with_scored=True)
    n0 = topk // bk
    assert rounds[0] == int(math.log2((T // bk) // n0))
    assert scored[0] == 2 * n0 * rounds[0]


# ---------------------------------------------------------------- per-head masks


@pytest.mark.parametrize("kind,G,bk,topk,T", [("decode", 2, 2, 16, 200), ("decode", 4, 1, 8, 77),
                                              ("prefill", 2, 4, 32, 150), ("prefill", 4, 2, 8, 64)])
def test_per_head_masks_match_brute_force_per_head(kind, G, bk, topk, T):
    # one mask per query head: each head's chunks are scored over its own rows
    # only, against its KV head's keys (brute force on that head alone)
    rng = np.random.default_rng(zlib.crc32(repr((kind, G, bk, topk, T)).encode()))
    B, Hkv = 2, 2
    Hq = Hkv * G
    Lq = 1 if kind == "decode" else T
    bq = 1 if kind == "decode" else 8
    q, k = _int_inputs(rng, B, Hq, Hkv, Lq, T)
    q_pos0 = T - Lq
    sh = _shape(batch=B, n_qheads=Hq, n_kvheads=Hkv, head_dim=64, seq_len=T, q_len=Lq,
                q_pos0=q_pos0, block_q=bq, block_k=bk, topk=topk, sink=bk, window=3,
                per_head=1)
    idx, gap, rounds = oracle.mask(q, k, sh)
    nqb = -(-Lq // bq)
    assert idx.shape[0] == B * Hq * nqb
    for u in rng.choice(idx.shape[0], min(24, idx.shape[0]), replace=False):
        b, h, qb = u // (Hq * nqb), (u // nqb) % Hq, u % nqb
        want, want_gap, want_rounds = bf.mask_row(
            q[:, h:h + 1], k[:, h // G:h // G + 1], b=b, g=0, qb=qb, group=1, block_q=bq,
            block_k=bk, topk=topk, q_len=Lq, q_pos0=q_pos0, seq_len=T, sink=bk, window=3)
        row = idx[u]
        assert list(row[1:1 + row[0]]) == want, (u, b, h, qb)
        assert rounds[u] == want_rounds


def test_per_head_masks_equal_group_masks_with_one_query_head_per_kv_head():
    rng = np.random.default_rng(21)
    q = rng.standard_normal((1, 3, 1, 128)).astype(np.float32)
    k = rng.standard_normal((1, 3, 500, 128)).astype(np.float32)
    common = dict(batch=1, n_qheads=3, n_kvheads=3, head_dim=128, seq_len=500, q_len=1,
                  q_pos0=499, block_q=1, block_k=2, topk=32, sink=4, window=8)
    a, ga, ra = oracle.mask(q, k, _shape(per_head=0, **common))
    b, gb, rb = oracle.mask(q, k, _shape(per_head=1, **common))
    assert np.array_equal(a, b) and np.array_equal(ra, rb)


def test_per_head_attention_reads_each_heads_own_row():
    rng = np.random.default_rng(23)
    B, Hq, Hkv, d, bk, T = 1, 4, 2, 128, 2, 300
    q = rng.standard_normal((B, Hq, 1, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    sh = _shape(batch=B, n_qheads=Hq, n_kvheads=Hkv, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=16, sink=4, window=8, per_head=1)
    idx, _, _ = oracle.mask(q, k, sh)
    assert idx.shape[0] == Hq
    out = oracle.attention(q, k, v, idx, sh).reshape(B, Hq, d)
    for h in range(Hq):
        g = h // 2
        row = idx[h]
        keys = {j for c in row[1:1 + row[0]] for j in range(c * bk, c * bk + bk) if j < T}
        allowed = np.zeros((1, T), bool)
        allowed[0, sorted(keys)] = True
        ref = bf.textbook_attention(q[0, h], k[0, g], v[0, g], allowed)
        np.testing.assert_allclose(out[0, h], ref[0], atol=2e-6, rtol=0)
    # the two query heads of a group do pick different blocks here
    assert not np.array_equal(idx[0], idx[1]) or not np.array_equal(idx[2], idx[3])


# ---- fp8 e5m2 codes (the KV cache type of the SGLang integration's serving
# commands, "[Feature] Support Efficient Sparse HiP Attention (InfiniteHiP)";
# values per the OCP 8-bit floating-point format, E5M2)


def test_e5m2_codes_are_the_upper_byte_of_binary16():
    # numpy's IEEE binary16 conversion is an independent statement of the
    # format: an e5m2 code c is the binary16 encoding c << 8
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.decode_e5m2(codes)
    ref = (codes.astype(np.uint16) << np.uint16(8)).view(np.float16).astype(np.float32)
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x80, -0.0),
    (0x3C, 1.0), (0xBC, -1.0), (0x40, 2.0), (0x3D, 1.25), (0x3F, 1.75),
    (0x04, 2.0 ** -14),              # smallest normal
    (0x01, 2.0 ** -16),              # smallest subnormal: 1/4 * 2^-14
    (0x03, 3.0 * 2.0 ** -16),
    (0x7B, 57344.0),                 # largest finite: 1.75 * 2^15
    (0x7C, np.inf), (0xFC, -np.inf),
])
def test_e5m2_closed_form_values(code, value):
    got = oracle.decode_e5m2(np.array([code], dtype=np.uint8))[0]
    assert got == value and np.signbit(got) == np.signbit(value)


def test_e5m2_nan_codes():
    got = oracle.decode_e5m2(np.array([0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF], dtype=np.uint8))
    assert np.all(np.isnan(got))


def test_e5m2_generator_codes_round_to_nearest():
    # the generator's codes decode to a value nearest the drawn one among
    # the finite e5m2 values (checked by brute force over the code table)
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(4000) * np.float32(3.0)).astype(np.float32)
    codes = W.e5m2_codes(x)
    table = oracle.decode_e5m2(np.arange(256, dtype=np.uint8)).astype(np.float64)
    finite = np.isfinite(table)
    got = oracle.decode_e5m2(codes).astype(np.float64)
    best = np.min(np.abs(table[finite][None, :] - x[:, None].astype(np.float64)), axis=1)
    assert np.all(np.abs(got - x) <= best * (1 + 1e-12))


# ---------------------------------------------------------------- stages
# The stage schedule of "[Feature] Support Efficient Sparse HiP Attention
# (InfiniteHiP)" (serving command, --hip-attention-config): per stage a chunk
# size, a stage_k (null: keep all) and a query-row stride; second_stage_k is
# the iteration's budget (topk here).


def _schedule(rng, bk, T, bq):
    """1-3 stages; chunk sizes multiples of b_k, each dividing the previous;
    stage_k 0 (keep all) or a multiple of the chunk size; random strides."""
    sizes = [bk * int(rng.choice([1, 2, 3, 4]))]
    for _ in range(int(rng.integers(0, 3))):
        sizes.insert(0, sizes[0] * int(rng.choice([1, 2, 4])))
    out = []
    for c in sizes:
        keep = 0 if rng.random() < 0.3 else c * int(rng.integers(1, max(2, T // c + 2)))
        out.append((c, keep, int(rng.choice([1, 2, 3, bq]))))
    return tuple(out)


def _stage_cases():
    rng = np.random.default_rng(23)
    cases = []
    for T in (5, 16, 33, 100, 257, 600):
        for bk in (1, 2, 4):
            for _ in range(2):
                kind = "decode" if rng.random() < 0.5 else "prefill"
                Lq = 1 if kind == "decode" else min(T, 48)
                bq = 1 if kind == "decode" else int(rng.choice([4, 8, 16]))
                G = int(rng.choice([1, 2]))
                nb = -(-T // bk)
                topk = bk * int(rng.integers(1, max(2, nb // 2 + 2)))
                sink = int(rng.choice([0, 0, bk, 5]))
                window = int(rng.choice([0, 0, 3, 2 * bk + 1]))
                cases.append((T, bk, topk, kind, Lq, bq, G, sink, window, _schedule(rng, bk, T, bq)))
    return cases


@pytest.mark.parametrize("case", _stage_cases())
def test_staged_mask_matches_brute_force_on_exact_scores(case):
    T, bk, topk, kind, Lq, bq, G, sink, window, stages = case
    rng = np.random.default_rng(zlib.crc32(repr(case).encode()))
    B, Hkv = 1, 2
    q, k = _int_inputs(rng, B, Hkv * G, Hkv, Lq, T)
    q_pos0 = T - Lq
    sh = _shape(batch=B, n_qheads=Hkv * G, n_kvheads=Hkv, head_dim=64, seq_len=T, q_len=Lq,
                q_pos0=q_pos0, block_q=bq, block_k=bk, topk=topk, sink=sink, window=window,
                stages=stages)
    idx, gap, rounds = oracle.mask(q, k, sh)
    nqb = -(-Lq // bq)
    units = [(b, g, qb) for b in range(B) for g in range(Hkv) for qb in range(nqb)]
    for u, (b, g, qb) in enumerate(units):
        want, want_gap, want_rounds = bf.mask_row(
            q, k, b=b, g=g, qb=qb, group=G, block_q=bq, block_k=bk, topk=topk, q_len=Lq,
            q_pos0=q_pos0, seq_len=T, sink=sink, window=window, stages=stages)
        row = idx[u]
        assert list(row[1:1 + row[0]]) == want, (case, u)
        assert rounds[u] == want_rounds, (case, u)
        if math.isinf(want_gap):
            assert math.isinf(gap[u])
        else:
            assert gap[u] == pytest.approx(want_gap / math.sqrt(64), rel=1e-12, abs=0)


@pytest.mark.parametrize("T,bk,topk", [(4096, 2, 256), (8192, 4, 512), (2048, 1, 64)])
def test_one_keep_all_stage_of_the_initial_chunks_is_the_plain_iteration(T, bk, topk):
    # n0 divides N: the plain iteration's n0 initial chunks are the aligned
    # chunks of b_k N / n0 keys, so a stage of that size that keeps every
    # chunk (stage_k null, or at least T) leaves the iteration unchanged
    rng = np.random.default_rng(T + bk)
    d, G = 128, 4
    q = rng.standard_normal((1, G, 1, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    N, n0 = T // bk, topk // bk
    assert N % n0 == 0
    base = dict(batch=1, n_qheads=G, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=topk, sink=bk, window=3 * bk)
    want = oracle.mask(q, k, _shape(**base), with_scored=True)
    for keep in (0, T):
        got = oracle.mask(q, k, _shape(**base, stages=((bk * N // n0, keep, 1),)), with_scored=True)
        for a, b in zip(got, want):
            np.testing.assert_array_equal(a, b)


# a schedule shaped like the serving command's (chunks of 128, 32 and 8
# keys; the first keeps all, the others a quarter of the range each time)
PR_LIKE = ((128, 0, 4), (32, 2048, 4), (8, 512, 1))


@pytest.mark.parametrize("T", [8192, 8000])
def test_staged_monotone_keys_keep_last_blocks(T):
    # every stage and round keeps its right-most chunks: the last n0 blocks
    d, bk, topk = 128, 2, 256
    q = np.ones((1, 2, 1, d), np.float32)
    k = np.ascontiguousarray(np.broadcast_to(((np.arange(T) + 1) / T).astype(np.float32)[:, None],
                                             (T, d)))[None, None]
    sh = _shape(batch=1, n_qheads=2, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=topk, stages=PR_LIKE)
    idx, _, rounds, scored = oracle.mask(q, k, sh, with_scored=True)
    N, n0 = -(-T // bk), topk // bk
    assert list(idx[0, 1:1 + idx[0, 0]]) == list(range(N - n0, N))
    # ranked: stages 2 and 3, then the rounds from 64 chunks of 4 blocks:
    # halves (128 = n0, kept unranked), then 256 single blocks
    assert rounds[0] == 3
    assert scored[0] == -(-T // 32) + 512 // 8 * 4 + 256


def test_staged_equal_keys_keep_first_blocks():
    # every score ties: the lower start wins each time, down to [0, n0)
    d, T, bk, topk = 128, 8192, 2, 256
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, 1, d)).astype(np.float32)
    k = np.ascontiguousarray(np.broadcast_to(rng.standard_normal(d).astype(np.float32), (T, d)))
    sh = _shape(batch=1, n_qheads=1, n_kvheads=1, head_dim=d, seq_len=T, q_len=1,
                q_pos0=T - 1, block_q=1, block_k=bk, topk=topk, stages=PR_LIKE)
    idx, gap, _ = oracle.mask(q, k[None, None], sh)
    assert list(idx[0, 1:1 + idx[0, 0]]) == list(range(topk // bk))
    assert gap[0] == 0.0


def test_stage_rows_are_counted_back_from_the_last_row():
    # one query block of 4 rows at stride 4: only the last row scores the
    # stage, so a key block that only the first row favours is pruned
    d, T, bk = 64, 64, 4
    q = np.zeros((1, 1, 4, d), np.float32)
    k = np.zeros((1, 1, T, d), np.float32)
    q[0, 0, 0, 0] = 1.0    # row 0 (position 60) wants dimension 0
    q[0, 0, 3, 1] = 1.0    # row 3 (position 63) wants dimension 1
    k[0, 0, 8, 0] = 5.0    # block 2 (chunk [0, 4) of 4 blocks) matches row 0
    k[0, 0, 40, 1] = 1.0   # block 10 (chunk [8, 12)) matches row 3
    base = dict(batch=1, n_qheads=1, n_kvheads=1, head_dim=d, seq_len=T, q_len=4, q_pos0=T - 4,
                block_q=4, block_k=bk, topk=bk * 4)
    rep = lambda c: c * 4 + 2  # noqa: E731 -- the centre block of chunk c
    k[0, 0, rep(0) * bk, 0] = 5.0
    k[0, 0, rep(2) * bk, 1] = 1.0
    for stride, want_chunk in ((4, 2), (1, 0)):
        sh = _shape(**base, stages=((16, 16, stride),))
        idx, _, _ = oracle.mask(q, k, sh)
        kept = list(idx[0, 1:1 + idx[0, 0]])
        assert kept == list(range(want_chunk * 4, want_chunk * 4 + 4)), (stride, kept)
