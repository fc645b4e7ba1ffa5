"""GPU parity of the prefill mask (query blocks of b_q rows scored on tensor
cores with the exact re-score band) against the oracle."""
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


def _gpu_mask(w, x):
    """(oracle shape, GPU idx rows, validator factory) of a prefill workload."""
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    osh, bkw = pu.shapes(w)
    q, k, _ = pu.torch_inputs(x, w)
    s = hb.Session(**bkw)
    idx = s.mask(q, k)
    torch.cuda.synchronize()
    s.check()

    def validator(units=None):
        return pu.gpu_validator(x["q"][0], x["k"], osh, s, q, k, units)

    return osh, idx.cpu().numpy().reshape(-1, idx.shape[-1]), validator


SMALL = [
    # 4 heads x 64 positions = 256 rows per mask, ragged last query block
    W.Workload("p256", "prefill", 1, 4, 1, 128, 3000, 64, 2, 256, 16, 64, "bf16"),
    # 2 heads x 64 = 128 rows, 4-key blocks, two KV heads, batch 2
    W.Workload("p128", "prefill", 2, 4, 2, 128, 2100, 64, 4, 256, 0, 0, "bf16"),
    # 1 head x 64 = 64 rows, one-key blocks
    W.Workload("p64", "prefill", 1, 1, 1, 128, 1500, 64, 1, 128, 4, 32, "bf16"),
    # 16-key blocks, 8 rows per mask (b_q = 2, 4 heads)
    W.Workload("p8", "prefill", 1, 4, 1, 128, 1200, 2, 16, 256, 0, 16, "bf16"),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_prefill_mask(w):
    x = _inputs(w)
    osh, got, validator = _gpu_mask(w, x)
    ref, gap, _ = oracle.mask(x["q"][0], x["k"], osh)
    pu.compare_masks(got, ref, gap, validate=validator())


def prefill_32k_sample(nqb: int, n_kvheads: int) -> np.ndarray:
    """Mask rows of the 32k prefill that are checked one by one: every KV head
    at 64 query blocks -- 0 (one round or none), 31, 32 and 33 (around the
    first full budget of 2048 keys), the last one, and 59 more drawn
    uniformly -- 512 of the 4096 rows."""
    rng = np.random.default_rng(0)
    fixed = {0, 31, 32, 33, nqb - 1}
    rest = rng.choice(sorted(set(range(nqb)) - fixed), 64 - len(fixed), replace=False)
    qbs = np.array(sorted(fixed | set(int(r) for r in rest)), dtype=np.int64)
    return np.array([g * nqb + qb for g in range(n_kvheads) for qb in qbs], dtype=np.int64)


def test_prefill_32k_mask_sampled():
    w = W.PREFILL_32K
    x = _inputs(w)
    osh, got, validator = _gpu_mask(w, x)
    units = prefill_32k_sample(oracle.num_qblocks(osh), w.n_kvheads)
    assert units.size >= 512
    ref, gap, _ = oracle.mask(x["q"][0], x["k"], osh, units=units)
    pu.compare_masks(got[units], ref, gap, validate=validator(units))


def test_equal_keys_every_candidate_in_the_band():
    # every score ties: the whole candidate set is re-scored canonically and
    # the tie rule keeps the lowest blocks
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    T, bk, topk = 4096, 2, 256
    rng = np.random.default_rng(0)
    q = W.bf16_round(rng.standard_normal((1, 4, 1, 128)).astype(np.float32))
    k = np.ascontiguousarray(np.broadcast_to(W.bf16_round(rng.standard_normal(128).astype(np.float32)),
                                             (1, 1, T, 128)))
    s = hb.Session(batch=1, n_qheads=4, n_kvheads=1, seq_len=T, q_len=1, q_pos0=T - 1,
                   dtype=hb.HIPS_BF16, block_q=1, block_k=bk, topk=topk)
    idx = s.mask(torch.from_numpy(q).cuda().to(torch.bfloat16).contiguous(),
                 torch.from_numpy(k).cuda().to(torch.bfloat16).contiguous())
    torch.cuda.synchronize()
    s.check()
    got = idx.cpu().numpy().reshape(-1)
    assert got[0] == topk // bk
    assert list(got[1:1 + got[0]]) == list(range(topk // bk))


def _gpu_attention(w, x, idx_ref=None, dense=False):
    """(gpu idx, gpu out on gpu idx, gpu out on the oracle idx) for a prefill workload."""
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    osh, bkw = pu.shapes(w)
    q, k, v = pu.torch_inputs(x, w)
    s = hb.Session(**bkw)
    if dense:
        out = s.dense_attn(q, k, v)
        torch.cuda.synchronize()
        s.check()
        return None, out.float().cpu().numpy().reshape(-1, 128), None
    idx = s.mask(q, k)
    out = s.sparse_attn(q, k, v, idx)
    out_ref_idx = None
    if idx_ref is not None:
        ri = torch.from_numpy(idx_ref).to("cuda").reshape(idx.shape).contiguous()
        out_ref_idx = s.sparse_attn(q, k, v, ri).float().cpu().numpy().reshape(-1, 128)
    torch.cuda.synchronize()
    s.check()
    return (idx.cpu().numpy().reshape(-1, idx.shape[-1]), out.float().cpu().numpy().reshape(-1, 128),
            out_ref_idx)


@pytest.mark.parametrize("w", SMALL[:3], ids=[w.name for w in SMALL[:3]])
def test_small_prefill_attention_on_tensor_cores(w):
    x = _inputs(w)
    osh, _ = pu.shapes(w)
    ref_idx, gap, _ = oracle.mask(x["q"][0], x["k"], osh)
    got_idx, out_e2e, out_on_ref = _gpu_attention(w, x, ref_idx)
    ref = oracle.attention(x["q"][0], x["k"], x["v"], ref_idx, osh)
    pu.compare_outputs(out_on_ref, ref, w.dtype)
    pu.compare_masks(got_idx, ref_idx, gap)
    ref_g = ref if np.array_equal(got_idx, ref_idx) else oracle.attention(
        x["q"][0], x["k"], x["v"], got_idx, osh)
    pu.compare_outputs(out_e2e, ref_g, w.dtype)


def test_small_prefill_dense_attention():
    w = W.Workload("pd", "prefill", 1, 4, 2, 128, 1500, 64, 2, 256, 0, 0, "bf16")
    x = _inputs(w)
    osh, _ = pu.shapes(w)
    _, out, _ = _gpu_attention(w, x, dense=True)
    ref = oracle.attention(x["q"][0], x["k"], x["v"], None, osh)
    pu.compare_outputs(out, ref, w.dtype)


def test_prefill_32k_attention_sampled():
    w = W.PREFILL_32K
    x = _inputs(w)
    osh, _ = pu.shapes(w)
    got_idx, out, _ = _gpu_attention(w, x)
    nqb = oracle.num_qblocks(osh)
    G, bq, T = w.group, w.block_q, w.seq_len
    picks = [(0, 0), (3, 31), (5, 32), (7, 33), (2, 200), (6, nqb - 1), (1, 400)]
    units = np.array([g * nqb + qb for g, qb in picks], dtype=np.int64)
    ref_idx, gap, _ = oracle.mask(x["q"][0], x["k"], osh, units=units)
    pu.compare_masks(got_idx[units], ref_idx, gap)
    # the oracle's attention over the GPU's own idx rows of those units
    full_idx = np.full((got_idx.shape[0], got_idx.shape[1]), -1, np.int32)
    full_idx[units] = got_idx[units]
    rows = np.array([(g * G + h) * T + qb * bq + i for g, qb in picks for h in range(G)
                     for i in range(0, bq, 7)], dtype=np.int64)
    ref = oracle.attention(x["q"][0], x["k"], x["v"], full_idx, osh, rows=rows)
    pu.compare_outputs(out[rows], ref, w.dtype)
