"""GPU parity of the InfiniteHiP pruning stages against the oracle.

The stages of the serving command's --hip-attention-config in "[Feature]
Support Efficient Sparse HiP Attention (InfiniteHiP)" (chunk size, stage_k,
query-row stride; second_stage_k as the iteration's budget) run before the
hierarchical iteration. The stage kernels rank by the canonical fp32 scores,
as the mask kernels do, so the masks must match the oracle's bit for bit;
the work counter (candidates scored, stages included) must equal the
oracle's; attention is checked on the GPU's idx against the oracle's.
"""
import functools

import numpy as np
import pytest

import oracle
from hierarchically_pruned_sparse_b200 import workloads as W
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    from hierarchically_pruned_sparse_b200 import build
    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    build.build()
    oracle.set_threads(0)


@functools.lru_cache(maxsize=4)
def _inputs(w: W.Workload):
    return W.make_inputs(w)


def _scored(sess) -> int:
    base = sess.p.workspace - sess.workspace.data_ptr()
    return int(sess.workspace[base + 8: base + 16].cpu().numpy().view(np.uint64)[0])


def _check(w: W.Workload, stages, fused: bool, flags: int = 0):
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    x = _inputs(w)
    kf, vf = pu.oracle_kv(x, w)
    osh, bkw = pu.shapes(w)
    per_head = bool(flags & hb.FLAG_HEAD_MASKS)
    fields = {f: getattr(osh, f) for f, _ in oracle.Shape._fields_
              if f not in ("n_stages", "stages", "pad0", "per_head")}
    osh = oracle.shape(**fields, per_head=int(per_head), stages=stages)
    q, k, v = pu.torch_inputs(x, w)
    s = hb.Session(flags=flags, stages=stages, **bkw)
    hb.workspace_init(s.p)
    if fused:
        idx_g, out = s.mask_sparse_attn(q, k, v)
        torch.cuda.synchronize()
    else:
        idx_g = s.mask(q, k)
        torch.cuda.synchronize()
        scored = _scored(s)
        out = s.sparse_attn(q, k, v, idx_g)
        torch.cuda.synchronize()
    s.check()
    idx_ref, gap, _, scored_ref = oracle.mask(x["q"][0], kf, osh, with_scored=True)
    ig = idx_g.cpu().numpy().reshape(idx_ref.shape)
    st = pu.compare_masks(ig, idx_ref, gap)
    if not fused:
        assert scored == int(scored_ref.sum())
    out_ref = oracle.attention(x["q"][0], kf, vf, ig, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(out_ref.shape), out_ref, w.dtype)
    return st


# (workload, stages, fused): each covers a kernel the iteration continues on
SMALL = [
    # bf16 decode, one launch (tensor-core mask + attention): two ranking
    # stages; the survivors need one halving that keeps all, then one round
    (W.Workload("s1", "decode", 1, 4, 1, 128, 5001, 1, 2, 256, 16, 100, "bf16", 4, "uniform"),
     ((64, 0, 1), (16, 1024, 1), (8, 512, 1)), True),
    # the same, survivors that halve down to single blocks (no round left)
    (W.Workload("s1b", "decode", 1, 4, 1, 128, 5001, 1, 2, 256, 16, 100, "bf16", 4, "uniform"),
     ((64, 0, 1), (16, 1024, 1), (4, 256, 1)), False),
    # fp32 decode of one head (CUDA-core mask), 16-key blocks
    (W.Workload("s2", "decode", 1, 1, 1, 128, 8192, 1, 16, 512, 0, 0, "f32", 4, "uniform"),
     ((1024, 0, 1), (256, 4096, 1), (64, 2048, 1)), False),
    # e5m2 keys, 8 rows per mask, batch of 2, two calls
    (W.Workload("s3", "decode", 2, 16, 2, 128, 3001, 1, 4, 128, 0, 32, "e5m2", 2, "uniform"),
     ((32, 0, 2), (16, 256, 1)), False),
    # bf16 prefill in 64-row query blocks (tensor-core mask with many rows),
    # strided stage rows, early blocks with fewer chunks than a stage keeps
    (W.Workload("s4", "prefill", 1, 8, 2, 128, 1000, 64, 2, 128, 16, 32, "bf16"),
     ((64, 0, 4), (16, 512, 4), (4, 128, 1)), False),
    # fp32 prefill in 4-row blocks (CUDA-core mask), stride 3, ragged T
    (W.Workload("s5", "prefill", 1, 2, 1, 128, 600, 4, 4, 64, 4, 8, "f32"),
     ((32, 0, 1), (16, 128, 3)), False),
    # no ranking stage: the iteration starts from the 64-key tiling
    (W.Workload("s6", "decode", 1, 4, 1, 128, 5001, 1, 2, 256, 0, 0, "bf16", 4, "uniform"),
     ((64, 0, 1),), True),
    # a cache shorter than one chunk
    (W.Workload("s7", "decode", 1, 4, 2, 128, 7, 1, 2, 4, 0, 0, "bf16"),
     ((16, 16, 1), (4, 4, 1)), False),
]


@pytest.mark.parametrize("w,stages,fused", SMALL, ids=[w.name for w, _, _ in SMALL])
def test_small_staged_shapes(w, stages, fused):
    _check(w, stages, fused)


def test_staged_per_head_masks():
    from hierarchically_pruned_sparse_b200 import binding as hb
    w = W.Workload("s8", "decode", 1, 8, 2, 128, 4000, 1, 2, 128, 8, 64, "bf16", 4, "uniform")
    _check(w, ((32, 0, 1), (8, 256, 1)), False, flags=hb.FLAG_HEAD_MASKS)


# A schedule shaped like the serving command's (chunks of 128, 32 and 8
# keys; the first keeps every chunk, stride 4 for the first two stages) at
# the 128k decode shape, with the decode budget of 2048 keys as
# second_stage_k: stage 2 keeps a quarter of the keys, stage 3 a quarter of
# those, and the iteration then runs two rounds.
PR_LIKE_128K = ((128, 0, 4), (32, 32768, 4), (8, 8192, 1))


def test_decode_128k_pr_schedule_one_launch():
    st = _check(W.DECODE_128K, PR_LIKE_128K, True)
    assert st["rows"] == 8


def test_decode_128k_pr_schedule_two_calls():
    _check(W.DECODE_128K, PR_LIKE_128K, False)


@pytest.mark.parametrize("stages", [((4, 1024, 1),), ((2, 2048, 1),)],
                         ids=["ties_in_one_bucket", "ties_past_the_bucket_band"])
def test_equal_keys_keep_the_lowest_starts(stages):
    # every key row is the same, so every score ties: each stage and round
    # keeps the chunks with the lowest starts. 2048 tied chunks are ranked
    # in the selection's cut bucket; 4096 exceed its band and take the
    # digit-by-digit selection instead.
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    T, d = 8192, 128
    rng = np.random.default_rng(9)
    qf = rng.standard_normal((1, 1, 1, d)).astype(np.float32)
    row = rng.standard_normal(d).astype(np.float32)
    kf = np.ascontiguousarray(np.broadcast_to(row, (1, 1, T, d)))
    vf = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)  # noqa: E731
    q, k, v = to(qf), to(kf), to(vf)
    qb, kb, vb = (x.float().cpu().numpy() for x in (q, k, v))
    common = dict(batch=1, n_qheads=1, n_kvheads=1, seq_len=T, q_len=1, q_pos0=T - 1,
                  block_q=1, block_k=1, topk=1024)
    s = hb.Session(dtype=hb.HIPS_BF16, stages=stages, **common)
    idx, out = s.mask_sparse_attn(q, k, v)
    torch.cuda.synchronize()
    s.check()
    osh = oracle.shape(head_dim=d, stages=stages, **common)
    idx_ref, gap, _ = oracle.mask(qb, kb, osh)
    got = idx.cpu().numpy().reshape(idx_ref.shape)
    assert list(idx_ref[0, 1:1 + idx_ref[0, 0]]) == list(range(1024))
    np.testing.assert_array_equal(got, idx_ref)
    ref = oracle.attention(qb, kb, vb, got, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(ref.shape), ref, "bf16")
