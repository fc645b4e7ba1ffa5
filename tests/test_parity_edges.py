"""GPU parity on the edges of the method's shapes, against the oracle:
a prefill chunk whose query rows start after the first key (q_pos0 > 0),
caches of one to a few keys, sink and window longer than the cache, a
budget larger than the cache in prefill, and decode groups through the
one-call entry point. Masks must match the oracle bit-exactly; attention is
compared on the oracle's idx and end to end on the GPU's idx."""
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


def _run(x_q, x_k, x_v, dtype, *, batch, hq, hkv, T, q_len, q_pos0, bq, bk, topk, sink, window,
         fused=False):
    """Mask and attention of one call shape on the GPU and in the oracle."""
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    common = dict(batch=batch, n_qheads=hq, n_kvheads=hkv, seq_len=T, q_len=q_len, q_pos0=q_pos0,
                  block_q=bq, block_k=bk, topk=topk, sink=sink, window=window)
    osh = oracle.shape(head_dim=128, **common)
    s = hb.Session(dtype=hb.HIPS_BF16 if dtype == "bf16" else hb.HIPS_F32, **common)
    q = torch.from_numpy(np.ascontiguousarray(x_q)).cuda().to(dt).contiguous()
    k = torch.from_numpy(np.ascontiguousarray(x_k)).cuda().to(dt).contiguous()
    v = torch.from_numpy(np.ascontiguousarray(x_v)).cuda().to(dt).contiguous()
    if fused:
        idx, out_f = s.mask_sparse_attn(q, k, v)
    else:
        idx, out_f = s.mask(q, k), None
    idx_ref, gap, _ = oracle.mask(x_q, x_k, osh)
    idx_ref_dev = torch.from_numpy(idx_ref).cuda().reshape(idx.shape).contiguous()
    out = s.sparse_attn(q, k, v, idx_ref_dev)
    if out_f is None:
        out_f = s.sparse_attn(q, k, v, idx)  # end to end through the two calls
    torch.cuda.synchronize()
    s.check()
    ig = idx.cpu().numpy().reshape(idx_ref.shape)
    pu.compare_masks(ig, idx_ref, gap, validate=pu.gpu_validator(x_q, x_k, osh, s, q, k))
    ref = oracle.attention(x_q, x_k, x_v, idx_ref, osh)
    pu.compare_outputs(out.float().cpu().numpy().reshape(ref.shape), ref, dtype)
    ref_g = ref if np.array_equal(ig, idx_ref) else oracle.attention(x_q, x_k, x_v, ig, osh)
    pu.compare_outputs(out_f.float().cpu().numpy().reshape(ref.shape), ref_g, dtype)
    return idx_ref


def _draw(w: W.Workload):
    x = W.make_inputs(w)
    return x["q"][0], x["k"], x["v"]


def test_prefill_chunk_after_cached_keys():
    # 1000 query rows at positions 2000..2999 over a 3000-key cache (chunked prefill)
    w = W.Workload("chunk", "prefill", 1, 4, 1, 128, 3000, 64, 2, 256, 16, 64, "bf16")
    q, k, v = _draw(w)
    _run(q[:, :, 2000:], k, v, "bf16", batch=1, hq=4, hkv=1, T=3000, q_len=1000, q_pos0=2000,
         bq=64, bk=2, topk=256, sink=16, window=64)


@pytest.mark.parametrize("T", [1, 2, 3, 7])
def test_decode_caches_of_a_few_keys(T):
    # fewer keys than one budget, one block, or a ragged last block
    w = W.Workload(f"tiny{T}", "decode", 1, 4, 1, 128, T, 1, 2, 4, 0, 0, "bf16")
    q, k, v = _draw(w)
    idx = _run(q, k, v, "bf16", batch=1, hq=4, hkv=1, T=T, q_len=1, q_pos0=T - 1, bq=1, bk=2,
               topk=4, sink=0, window=0, fused=True)
    assert idx[0, 0] == min(4 // 2, (T + 1) // 2)  # k / b_k blocks, or every block


def test_sink_and_window_longer_than_the_cache():
    w = W.Workload("longsw", "decode", 1, 4, 2, 128, 100, 1, 4, 32, 0, 0, "bf16")
    q, k, v = _draw(w)
    idx = _run(q, k, v, "bf16", batch=1, hq=4, hkv=2, T=100, q_len=1, q_pos0=99, bq=1, bk=4,
               topk=32, sink=200, window=500, fused=True)
    assert np.all(idx[:, 0] == 25)  # the union is every block


def test_prefill_budget_above_the_cache_is_dense():
    w = W.Workload("pdense", "prefill", 1, 4, 1, 128, 300, 64, 2, 512, 0, 0, "bf16")
    q, k, v = _draw(w)
    idx = _run(q, k, v, "bf16", batch=1, hq=4, hkv=1, T=300, q_len=300, q_pos0=0, bq=64, bk=2,
               topk=512, sink=0, window=0)
    # query block qb sees keys < min(64 (qb + 1), 300): all of their blocks
    for qb in range(5):
        assert idx[qb, 0] == (min(64 * (qb + 1), 300) + 1) // 2


def test_prefill_tiny_cache_one_ragged_query_block():
    w = W.Workload("ptiny", "prefill", 1, 4, 1, 128, 5, 64, 2, 2, 0, 0, "bf16")
    q, k, v = _draw(w)
    _run(q, k, v, "bf16", batch=1, hq=4, hkv=1, T=5, q_len=5, q_pos0=0, bq=64, bk=2, topk=2,
         sink=0, window=0)


def test_fused_decode_batch_of_sequences_fp32_falls_back():
    # fp32 has no one-launch form: the call runs the two kernels and must agree
    w = W.Workload("f32b", "decode", 2, 4, 2, 128, 700, 1, 2, 64, 4, 16, "f32", 2, "uniform")
    q, k, v = _draw(w)
    _run(q, k, v, "f32", batch=2, hq=4, hkv=2, T=700, q_len=1, q_pos0=699, bq=1, bk=2, topk=64,
         sink=4, window=16, fused=True)
