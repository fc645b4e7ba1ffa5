"""Independent restatement of the hierarchical pruning rule, for pinning the oracle.

Written separately from the oracle (recursive, on Python intervals, with
scores given by a callback) from the iteration in "A Training-free
Sub-quadratic Cost Transformer Model Serving Framework With Hierarchically
Pruned Attention", Author Rebuttal to the Reviewer RsGC, Q2, steps 1-4, and
from the multi-stage schedule of "[Feature] Support Efficient Sparse HiP
Attention (InfiniteHiP)" (the serving command's stages: chunk size, stage_k,
query-row stride), read as: every stage cuts the surviving intervals into
pieces of its chunk size (stage 1 cuts the whole range) and keeps the
stage_k / chunk_size best pieces (all when stage_k is 0), and the iteration
then starts from the survivors. Tests feed it integer-valued inputs so every
score is an exact integer and no evaluation order can change a decision.
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


def _pieces(iv, size):
    s, e = iv
    return [(p, min(p + size, e)) for p in range(s, e, size)]


def _staged(stage_score, n_blocks, stages, block_k):
    """Intervals surviving the stages (chunk_size, stage_k, stride), with the
    smallest raw cut gap and the number of stages that ranked."""
    chunks, gap, rounds = [(0, n_blocks)], math.inf, 0
    for chunk_size, stage_k, stride in stages:
        cands = [p for iv in chunks for p in _pieces(iv, chunk_size // block_k)]
        keep = stage_k // chunk_size
        if stage_k == 0 or len(cands) <= keep:
            chunks = cands
            continue

        def sc(iv, stride=stride):
            return stage_score(_rep(iv), stride)

        ranked = sorted(cands, key=lambda iv: (-sc(iv), iv[0]))
        gap = min(gap, sc(ranked[keep - 1]) - sc(ranked[keep]))
        chunks, rounds = ranked[:keep], rounds + 1
    return chunks, gap, rounds


def prune(score, n_blocks: int, budget: int, stages=(), block_k: int = 1, stage_score=None):
    """Returns (kept blocks sorted, smallest raw cut gap, rounds). With
    stages, stage_score(block, stride) scores a stage's representative."""
    n0 = min(budget, n_blocks)
    if stages:
        start, gap0, rounds0 = _staged(stage_score, n_blocks, stages, block_k)
    else:
        start = [(i * n_blocks // n0, (i + 1) * n_blocks // n0) for i in range(n0)]
        gap0, rounds0 = math.inf, 0

    def refine(chunks, gap, rounds):
        # done when single blocks, at most n0 of them, are left
        if max(e - s for s, e in chunks) <= 1 and len(chunks) <= n0:
            return chunks, gap, rounds
        cands = [h for iv in chunks for h in _halves(iv)]
        if len(cands) <= n0:
            return refine(cands, gap, rounds)
        ranked = sorted(cands, key=lambda iv: (-score(_rep(iv)), iv[0]))
        gap = min(gap, score(_rep(ranked[n0 - 1])) - score(_rep(ranked[n0])))
        return refine(ranked[:n0], gap, rounds + 1)

    chunks, gap, rounds = refine(start, gap0, rounds0)
    return sorted(s for s, _ in chunks), gap, rounds


def mask_row(q, k, *, b, g, qb, group, block_q, block_k, topk, q_len, q_pos0,
             seq_len, sink, window, stages=()):
    """One mask row (sorted block ids, raw gap, rounds) from integer q, k."""
    i0, i1 = qb * block_q, min(qb * block_q + block_q, q_len)
    q_first, q_last = q_pos0 + i0, q_pos0 + i1 - 1
    t_c = min(q_last + 1, seq_len)
    n_blocks = -(-t_c // block_k)
    heads = range(g * group, (g + 1) * group)
    # exact integer dots of the unit's rows with its keys, -inf where causal
    # order hides the key (j > p)
    dots = np.stack([q[b, h, i0:i1].astype(np.int64) @ k[b, g, :t_c].astype(np.int64).T
                     for h in heads]).astype(np.float64)
    pos = q_pos0 + np.arange(i0, i1)
    dots[:, pos[:, None] < np.arange(t_c)[None, :]] = -math.inf

    def stage_score(c, stride):
        # rows: the block's last query row and every stride-th one before it
        rows = np.arange(i1 - 1 - i0, -1, -stride)
        return dots[:, rows, c * block_k:min(c * block_k + block_k, t_c)].max()

    kept, gap, rounds = prune(lambda c: stage_score(c, 1), n_blocks, topk // block_k,
                              stages=stages, block_k=block_k, stage_score=stage_score)
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
