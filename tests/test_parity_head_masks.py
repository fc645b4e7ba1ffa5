"""GPU parity of one mask per query head (the head-reduce switch off) against
the oracle's per-head mode: masks bit-exact,
attention within tolerance, through hip_mask, hip_sparse_attn and the
one-call hip_mask_sparse_attn."""
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


@functools.lru_cache(maxsize=2)
def _inputs(w: W.Workload):
    return W.make_inputs(w)


def _check(w: W.Workload, fused: bool):
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    x = _inputs(w)
    osh, bkw = pu.shapes(w)
    osh.per_head = 1
    q, k, v = pu.torch_inputs(x, w)
    s = hb.Session(flags=hb.FLAG_HEAD_MASKS, **bkw)
    if fused:
        idx, out_f = s.mask_sparse_attn(q, k, v)
        assert torch.equal(idx, s.mask(q, k))
    else:
        idx, out_f = s.mask(q, k), None
    assert idx.shape[1] == w.n_qheads
    idx_ref, gap, _ = oracle.mask(x["q"][0], x["k"], osh)
    out = s.sparse_attn(q, k, v, torch.from_numpy(idx_ref).cuda().reshape(idx.shape).contiguous())
    if out_f is None:
        out_f = s.sparse_attn(q, k, v, idx)  # end to end through the two calls
    torch.cuda.synchronize()
    s.check()
    ig = idx.cpu().numpy().reshape(idx_ref.shape)
    pu.compare_masks(ig, idx_ref, gap, validate=pu.gpu_validator(x["q"][0], x["k"], osh, s, q, k))
    ref = oracle.attention(x["q"][0], x["k"], x["v"], idx_ref, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(ref.shape), ref, w.dtype)
    ref_g = ref if np.array_equal(ig, idx_ref) else oracle.attention(x["q"][0], x["k"], x["v"], ig, osh)
    pu.compare_outputs(out_f.float().cpu().numpy().reshape(ref.shape), ref_g, w.dtype)
    return idx_ref


DECODE = [
    W.Workload("h1", "decode", 1, 4, 1, 128, 5001, 1, 2, 256, 16, 100, "bf16", 4, "uniform"),
    W.Workload("h2", "decode", 2, 8, 2, 128, 3001, 1, 4, 128, 0, 0, "bf16", 2, "uniform"),
    W.Workload("h3", "decode", 1, 4, 2, 128, 777, 1, 1, 64, 3, 5, "f32", 2, "uniform"),
]


@pytest.mark.parametrize("w", DECODE, ids=[w.name for w in DECODE])
def test_head_masks_small_decode(w):
    idx = _check(w, fused=True)
    # heads of one group see the same keys but generally pick different blocks
    assert idx.shape[0] == w.batch * w.n_qheads


def test_head_masks_decode_128k():
    _check(W.DECODE_128K, fused=True)


PREFILL = [
    # 64 rows per mask (one head x b_q 64) on the tensor-core kernels, ragged tail
    W.Workload("hp64", "prefill", 1, 4, 1, 128, 1500, 64, 2, 128, 8, 32, "bf16"),
    # 16-row masks (b_q 16), two KV heads
    W.Workload("hp16", "prefill", 1, 4, 2, 128, 900, 16, 4, 128, 0, 16, "bf16"),
]


@pytest.mark.parametrize("w", PREFILL, ids=[w.name for w in PREFILL])
def test_head_masks_prefill(w):
    _check(w, fused=False)
