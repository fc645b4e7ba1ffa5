"""GPU parity of the fp8 e5m2 KV cache (bf16 queries and outputs) against
the oracle, which decodes the same codes itself.

The serving commands of "[Feature] Support Efficient Sparse HiP Attention
(InfiniteHiP)" (SGLang pull request) run HiP attention over a KV cache
stored as fp8 e5m2. Every e5m2 code widens exactly to bf16, so the masks
must match the oracle's bit-exactly (the kernels select by canonical scores) and the
outputs stay within the bf16 tolerance. The e5m2 path must also give the
same masks as the bf16 path run on the widened keys, and the one-launch
decode the same outputs bit for bit (both attend in 64-key tiles in the same
order). Shapes with no e5m2 kernel (prefill query blocks, attention of more
than 8 rows per block) run on widened rows and are checked the same way.
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


@functools.lru_cache(maxsize=2)
def _inputs(w: W.Workload):
    return W.make_inputs(w)


def _check(w: W.Workload, fused: bool, step: int = 0):
    """GPU mask (exact, with the validity replay of any mismatched row) and
    attention of decode step ``step`` against the oracle: outputs on the
    oracle's idx, and end to end on the GPU's idx against the oracle's
    attention over that same idx."""
    import numpy as np
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    x = _inputs(w)
    kf, vf = pu.oracle_kv(x, w)
    osh, bkw = pu.shapes(w, step)
    q, k, v = pu.torch_inputs(x, w, step)
    q0 = pu.torch_inputs(x, w, 0)[0]
    s = hb.Session(**bkw)
    if step == 0 and fused:
        idx_g, out_e2e = s.mask_sparse_attn(q, k, v)
    else:
        s.set(seq_len=w.seq_len, q_pos0=osh.q_pos0 - step)
        idx_g = s.mask(q0, k)
        s.set(seq_len=osh.seq_len, q_pos0=osh.q_pos0)
        out_e2e = s.sparse_attn(q, k, v, idx_g)
    osh0, _ = pu.shapes(w, 0)
    osh0.kv_capacity = w.capacity
    idx_ref, gap, _ = oracle.mask(x["q"][0], kf, osh0)
    idx_ref_dev = torch.from_numpy(idx_ref).to("cuda").reshape(idx_g.shape).contiguous()
    out_on_ref = s.sparse_attn(q, k, v, idx_ref_dev)
    torch.cuda.synchronize()
    s.check()
    ig = idx_g.cpu().numpy().reshape(idx_ref.shape)
    s.set(seq_len=w.seq_len, q_pos0=osh.q_pos0 - step)
    st = pu.compare_masks(ig, idx_ref, gap,
                          validate=pu.gpu_validator(x["q"][0], kf, osh0, s, q0, k))
    s.set(seq_len=osh.seq_len, q_pos0=osh.q_pos0)
    out_ref = oracle.attention(x["q"][step], kf, vf, idx_ref, osh)
    pu.compare_outputs(out_on_ref.float().cpu().numpy().reshape(out_ref.shape), out_ref, w.dtype)
    ref_g = out_ref if np.array_equal(ig, idx_ref) else oracle.attention(x["q"][step], kf, vf, ig, osh)
    pu.compare_outputs(out_e2e.float().cpu().numpy().reshape(out_ref.shape), ref_g, w.dtype)
    return st


SMALL = [
    # one launch (4 rows per mask): ragged T, sink + window, needles
    (W.Workload("e1", "decode", 1, 4, 1, 128, 5001, 1, 2, 256, 16, 100, "e5m2", 4, "uniform"), True),
    # two calls: 8 rows per mask (split-K attention with 8 rows), batch of 2, b_k = 4
    (W.Workload("e2", "decode", 2, 16, 2, 128, 3001, 1, 4, 128, 0, 32, "e5m2", 2, "uniform"), True),
    # a cache of a few keys (fewer than one budget)
    (W.Workload("e4", "decode", 1, 4, 2, 128, 7, 1, 2, 4, 0, 0, "e5m2"), True),
    # 2048 chunks per mask: more than the tensor-core mask kernel holds, so
    # the CUDA-core decode kernel plans it (one launch, 4 rows, ragged T)
    (W.Workload("e5", "decode", 1, 4, 1, 128, 20011, 1, 2, 4096, 16, 256, "e5m2", 4, "uniform"), True),
    # the same kernel for the mask alone: 8 rows, b_k = 4, batch of 2
    (W.Workload("e6", "decode", 2, 16, 2, 128, 9001, 1, 4, 8192, 0, 64, "e5m2", 2, "uniform"), False),
]


@pytest.mark.parametrize("w,fused", SMALL, ids=[w.name for w, _ in SMALL])
def test_small_decode_shapes(w, fused):
    _check(w, fused)


def test_sixteen_row_mask_and_its_attention():
    # 16 rows per mask is the largest e5m2 mask (one MMA column block); the
    # attention of more than 8 rows per query block has no e5m2 kernel and
    # runs on widened rows
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    w = W.Workload("e16", "decode", 1, 16, 1, 128, 2500, 1, 2, 64, 2, 8, "e5m2")
    x = _inputs(w)
    kf, vf = pu.oracle_kv(x, w)
    osh, bkw = pu.shapes(w)
    q, k, v = pu.torch_inputs(x, w)
    s = hb.Session(**bkw)
    idx = s.mask(q, k)
    out = s.sparse_attn(q, k, v, idx)
    torch.cuda.synchronize()
    s.check()
    idx_ref, gap, _ = oracle.mask(x["q"][0], kf, osh)
    ig = idx.cpu().numpy().reshape(idx_ref.shape)
    pu.compare_masks(ig, idx_ref, gap, validate=pu.gpu_validator(x["q"][0], kf, osh, s, q, k))
    ref = oracle.attention(x["q"][0], kf, vf, ig, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(ref.shape), ref, "e5m2")


def test_reused_mask_with_appended_keys():
    w = W.Workload("e_reuse", "decode", 2, 8, 2, 128, 4000, 1, 2, 256, 8, 64, "e5m2", 2,
                   "uniform", refresh=4)
    _check(w, fused=False, step=3)


def test_decode_128k_one_launch():
    st = _check(W.DECODE_128K_E5M2, fused=True)
    assert st["rows"] == 8


def test_decode_128k_two_calls():
    _check(W.DECODE_128K_E5M2, fused=False)


def test_e5m2_matches_bf16_on_the_widened_values():
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    w = W.DECODE_128K_E5M2
    x = _inputs(w)
    _, bkw = pu.shapes(w)
    q, k8, v8 = pu.torch_inputs(x, w)
    kf, vf = pu.oracle_kv(x, w)
    kb = torch.from_numpy(kf).to("cuda").to(torch.bfloat16).contiguous()
    vb = torch.from_numpy(vf).to("cuda").to(torch.bfloat16).contiguous()
    assert torch.equal(kb.float().cpu(), torch.from_numpy(kf))  # widening is exact
    s8 = hb.Session(**bkw)
    sb = hb.Session(**dict(bkw, dtype=hb.HIPS_BF16))
    idx8, out8 = s8.mask_sparse_attn(q, k8, v8)
    idxb, outb = sb.mask_sparse_attn(q, kb, vb)
    idx8_2 = s8.mask(q, k8)
    torch.cuda.synchronize()
    s8.check()
    sb.check()
    assert torch.equal(idx8, idxb)
    assert torch.equal(idx8_2, idxb)
    assert torch.equal(out8, outb)


def test_dense_attention_over_e5m2():
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    w = W.Workload("e_dense", "decode", 1, 8, 2, 128, 3000, 1, 2, 64, 0, 0, "e5m2")
    x = _inputs(w)
    kf, vf = pu.oracle_kv(x, w)
    osh, bkw = pu.shapes(w)
    q, k, v = pu.torch_inputs(x, w)
    s = hb.Session(**bkw)
    out = torch.empty_like(q)
    hb.hip_dense_attn(q, k, v, s.p, out)
    torch.cuda.synchronize()
    s.check()
    ref = oracle.attention(x["q"][0], kf, vf, None, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(ref.shape), ref, "e5m2")


# Shapes with no e5m2 kernel run on the bf16 kernels after the library widens
# K and V exactly into the workspace (the e5m2 path is defined as the bf16 one
# on the widened values): prefill query blocks, and attention of more than 8
# rows per query block.
PREFILL = W.Workload("e_pre", "prefill", 1, 8, 2, 128, 1000, 64, 2, 128, 16, 32, "e5m2")


@pytest.mark.parametrize("fused", [True, False], ids=["one_call", "two_calls"])
def test_prefill_blocks_by_widening(fused):
    st = _check(PREFILL, fused)
    assert st["rows"] == 2 * 16


def test_dense_prefill_over_e5m2_by_widening():
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    x = _inputs(PREFILL)
    kf, vf = pu.oracle_kv(x, PREFILL)
    osh, bkw = pu.shapes(PREFILL)
    q, k, v = pu.torch_inputs(x, PREFILL)
    s = hb.Session(**bkw)
    out = torch.empty_like(q)
    hb.hip_dense_attn(q, k, v, s.p, out)
    torch.cuda.synchronize()
    s.check()
    rows = np.arange(0, q.numel() // 128, 7)  # every 7th (head, position) row
    ref = oracle.attention(x["q"][0], kf, vf, None, osh, rows=rows)
    got = out.float().cpu().numpy().reshape(-1, 128)[rows]
    pu.compare_outputs(got, ref, "e5m2")
