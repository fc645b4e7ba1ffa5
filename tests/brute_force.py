"""Independent restatement of the hierarchical pruning rule, for pinning the oracle.

Written separately from the oracle (recursive, on Python intervals, with
scores given by a callback) from the iteration in "A Training-free
Sub-quadratic Cost Transformer Model Serving Framework With Hierarchically
Pruned Attention", Author Rebuttal to the Reviewer RsGC, Q2, steps 1-4.
Tests feed it integer-valued inputs so every score is an exact integer and
no evaluation order can change a decision.
"""
from __future__ import annotations

import math

import numpy as np


def _halves(iv):
    s, e = iv
    if e - s <= 1:
        return [iv]
    m = s + (e - s) // 2
    return [(s, m), (m, e)]


def _rep(iv):
    return iv[0] + (iv[1] - iv[0]) // 2


def prune(score, n_blocks: int, budget: int):
    """Returns (kept blocks sorted, smallest raw cut gap, rounds)."""
    n0 = min(budget, n_blocks)
    start = [(i * n_blocks // n0, (i + 1) * n_blocks // n0) for i in range(n0)]

    def refine(chunks, gap, rounds):
        if max(e - s for s, e in chunks) <= 1:
            return chunks, gap, rounds
        cands = [h for iv in chunks for h in _halves(iv)]
        ranked = sorted(cands, key=lambda iv: (-score(_rep(iv)), iv[0]))
        if len(ranked) > n0:
            gap = min(gap, score(_rep(ranked[n0 - 1])) - score(_rep(ranked[n0])))
        return refine(ranked[:n0], gap, rounds + 1)

    chunks, gap, rounds = refine(start, math.inf, 0)
    return sorted(s for s, _ in chunks), gap, rounds


def mask_row(q, k, *, b, g, qb, group, block_q, block_k, topk, q_len, q_pos0,
             seq_len, sink, window):
    """One mask row (sorted block ids, raw gap, rounds) from integer q, k."""
    i0, i1 = qb * block_q, min(qb * block_q + block_q, q_len)
    q_first, q_last = q_pos0 + i0, q_pos0 + i1 - 1
    t_c = min(q_last + 1, seq_len)
    n_blocks = -(-t_c // block_k)
    rows = [(h, q_pos0 + i) for h in range(g * group, (g + 1) * group) for i in range(i0, i1)]
    qi = q.astype(np.int64)
    ki = k.astype(np.int64)

    cache = {}

    def score(c):
        if c not in cache:
            vals = [int(qi[b, h, p - q_pos0] @ ki[b, g, j])
                    for (h, p) in rows
                    for j in range(c * block_k, min(c * block_k + block_k, t_c)) if j <= p]
            cache[c] = max(vals)
        return cache[c]

    kept, gap, rounds = prune(score, n_blocks, topk // block_k)
    blocks = set(kept)
    blocks |= set(range(min(-(-sink // block_k), n_blocks)))
    if window > 0:
        lo = max(0, q_first - window + 1)
        blocks |= {c for c in range(lo // block_k, q_last // block_k + 1) if c < n_blocks}
    return sorted(blocks), gap, rounds


def textbook_attention(q, k, v, allowed):
    """softmax(q k^T / sqrt(d) restricted to ``allowed``) v, in fp64 matrix form.

    q: [R, d]; k, v: [T, d]; allowed: bool [R, T] (every row has a key).
    """
    d = q.shape[-1]
    s = (q.astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(d)
    s = np.where(allowed, s, -np.inf)
    w = np.exp(s - s.max(axis=1, keepdims=True))
    return (w @ v.astype(np.float64)) / w.sum(axis=1, keepdims=True)
