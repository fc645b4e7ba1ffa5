"""GPU parity of the decode path (and small query blocks) against the oracle.

The kernels select by the canonical fp32 scores, so masks must match the
oracle bit-exactly (stricter than the method's rule, which lets rows whose
oracle cut gap is below 1e-3 q.k/sqrt(d) differ when they stay under 0.5 % of
rows and are valid selections). Attention is checked twice: fed the oracle's
idx (isolates the attention kernel) and end to end from the CUDA mask,
against the oracle's attention over the GPU's own idx.
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


def _session(bkw):
    from hierarchically_pruned_sparse_b200 import binding as hb
    return hb.Session(**bkw)


def _run_step(w, step=0, idx_ref=None):
    """GPU mask (at the refresh) and attention of step ``step`` against the
    oracle. Masks must match exactly (with the validity replay of any
    mismatched row); attention is checked on the oracle's idx (isolates the
    attention kernel) and end to end, the GPU's idx against the oracle's
    attention over that same idx."""
    import torch
    x = _inputs(w)
    osh, bkw = pu.shapes(w, step)
    q, k, v = pu.torch_inputs(x, w, step)
    s = _session(bkw)
    # the mask of a refresh is computed at mask_len keys
    s.set(seq_len=w.seq_len, q_pos0=osh.q_pos0 - step)
    q0 = pu.torch_inputs(x, w, 0)[0]
    idx_g = s.mask(q0, k)
    osh0, _ = pu.shapes(w, 0)
    osh0.kv_capacity = w.capacity
    if idx_ref is None:
        idx_ref, gap, _ = oracle.mask(x["q"][0], x["k"], osh0)
    else:
        idx_ref, gap = idx_ref
    torch.cuda.synchronize()
    ig = idx_g.cpu().numpy().reshape(idx_ref.shape)
    st = pu.compare_masks(ig, idx_ref, gap,
                          validate=pu.gpu_validator(x["q"][0], x["k"], osh0, s, q0, k))
    s.set(seq_len=osh.seq_len, q_pos0=osh.q_pos0)
    out_e2e = s.sparse_attn(q, k, v, idx_g)
    idx_ref_dev = torch.from_numpy(idx_ref).to("cuda").reshape(idx_g.shape).contiguous()
    out_on_ref = s.sparse_attn(q, k, v, idx_ref_dev)
    torch.cuda.synchronize()
    s.check()
    out_ref = oracle.attention(x["q"][step], x["k"], x["v"], idx_ref, osh)
    pu.compare_outputs(out_on_ref.float().cpu().numpy().reshape(out_ref.shape), out_ref, w.dtype)
    ref_g = out_ref if np.array_equal(ig, idx_ref) else oracle.attention(
        x["q"][step], x["k"], x["v"], ig, osh)
    pu.compare_outputs(out_e2e.float().cpu().numpy().reshape(out_ref.shape), ref_g, w.dtype)
    return st


def _check(w, step=0):
    return _run_step(w, step)


SMALL = [
    # several tiles, ragged T (not a multiple of b_k), sink + window, GQA
    W.Workload("r1", "decode", 1, 4, 1, 128, 5001, 1, 2, 256, 16, 100, "bf16", 4, "uniform"),
    W.Workload("r2", "decode", 2, 8, 2, 128, 3001, 1, 4, 128, 0, 0, "bf16", 2, "uniform"),
    W.Workload("r3", "decode", 1, 2, 2, 128, 777, 1, 1, 64, 3, 5, "f32", 2, "uniform"),
    # N/n0 not a power of two: chunks of 11 and 12 blocks, single-block chunks pass through
    W.Workload("r4", "decode", 1, 4, 1, 128, 3000, 1, 2, 256, 0, 0, "bf16", 2, "uniform"),
    # budget >= T: every block kept (dense)
    W.Workload("r5", "decode", 1, 4, 2, 128, 500, 1, 2, 512, 0, 0, "bf16"),
    # 8 query heads per KV head
    W.Workload("r6", "decode", 1, 8, 1, 128, 4096, 1, 2, 512, 32, 64, "bf16", 4, "uniform"),
    # one key per block, long
    W.Workload("r7", "decode", 1, 1, 1, 128, 20000, 1, 1, 1024, 0, 0, "f32", 4, "uniform"),
    # 16-key blocks in bf16, 2 query heads per group
    W.Workload("r8", "decode", 1, 4, 2, 128, 9000, 1, 16, 1024, 64, 256, "bf16", 4, "uniform"),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_decode(w):
    _check(w)


FUSED = SMALL + [W.DECODE_128K]


@pytest.mark.parametrize("w", FUSED, ids=[w.name for w in FUSED])
def test_mask_then_attention_in_one_call(w):
    """hip_mask_sparse_attn: the same idx as hip_mask, and attention within
    tolerance of the oracle (one launch for bf16 groups of <= 4 rows, the two
    calls otherwise)."""
    import torch
    x = _inputs(w)
    osh, bkw = pu.shapes(w)
    q, k, v = pu.torch_inputs(x, w)
    s = _session(bkw)
    idx_f, out_f = s.mask_sparse_attn(q, k, v)
    idx_m = s.mask(q, k)
    torch.cuda.synchronize()
    s.check()
    idx_f = idx_f.cpu().numpy()
    assert np.array_equal(idx_f, idx_m.cpu().numpy())
    idx_ref, gap, _ = oracle.mask(x["q"][0], x["k"], osh)
    idx_f = idx_f.reshape(idx_ref.shape)
    pu.compare_masks(idx_f, idx_ref, gap, validate=pu.gpu_validator(x["q"][0], x["k"], osh, s, q, k))
    ref = oracle.attention(x["q"][0], x["k"], x["v"], idx_f, osh)  # on the GPU's own idx
    pu.compare_outputs(out_f.float().cpu().numpy().reshape(ref.shape), ref, w.dtype)


def test_decode_8k_f32():
    _check(W.DECODE_8K_F32)


def test_decode_128k_llama_shape():
    _check(W.DECODE_128K)


def test_dense_attention_128k():
    import torch
    w = W.DECODE_128K
    x = _inputs(w)
    osh, bkw = pu.shapes(w)
    q, k, v = pu.torch_inputs(x, w)
    s = _session(bkw)
    out = s.dense_attn(q, k, v)
    torch.cuda.synchronize()
    s.check()
    ref = oracle.attention(x["q"][0], x["k"], x["v"], None, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(ref.shape), ref, w.dtype)


def test_small_prefill_blocks_on_cuda_cores():
    # query blocks of 4 rows x 2 heads: the CUDA-core mask and attention kernels
    import torch
    w = W.Workload("p1", "prefill", 1, 4, 2, 128, 700, 4, 2, 128, 8, 16, "bf16")
    x = _inputs(w)
    osh, bkw = pu.shapes(w)
    q, k, v = pu.torch_inputs(x, w)
    s = _session(bkw)
    idx = s.mask(q, k)
    out = s.sparse_attn(q, k, v, idx)
    torch.cuda.synchronize()
    s.check()
    idx_ref, gap, _ = oracle.mask(x["q"][0], x["k"], osh)
    ig = idx.cpu().numpy().reshape(idx_ref.shape)
    pu.compare_masks(ig, idx_ref, gap, validate=pu.gpu_validator(x["q"][0], x["k"], osh, s, q, k))
    ref = oracle.attention(x["q"][0], x["k"], x["v"], ig, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(ref.shape), ref, w.dtype)


def test_mask_reuse_small():
    w = W.Workload("m1", "decode", 2, 4, 1, 128, 3000, 1, 2, 256, 16, 64, "bf16", 2,
                   "uniform", refresh=5)
    for step in range(w.refresh):
        _check(w, step)


def test_batched_decode_mask_reuse_128k():
    w = W.DECODE_B16_REUSE
    x = _inputs(w)
    osh0, _ = pu.shapes(w, 0)
    idx_ref, gap, _ = oracle.mask(x["q"][0], x["k"], osh0)
    for step in (0, 3, 7):
        _run_step(w, step, (idx_ref, gap))


def test_decode_1m():
    _check(W.DECODE_1M)
