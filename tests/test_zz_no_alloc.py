"""The no-allocation sparse attention entry point (hip_sparse_attn_noalloc).

Some callers cannot allocate device memory at call time (a memory pool that
is frozen after start-up, or a decode loop that must never meet a cudaMalloc
and the synchronisation it can bring). For them the library keeps its split-K
scratch in a fixed device array. This checks, through the C ABI, that the
entry point gives the same output as hip_sparse_attn on two calls in a row
(the array keeps the previous call's contents), and that a request larger
than the array is refused before anything runs. It lives in its own file so
that a run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest

from hierarchically_pruned_sparse_b200 import binding as hb
from hierarchically_pruned_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2e-2, 5e-3  # the bf16 attention tolerance of the parity tests


def _setup(w):
    import torch
    from hierarchically_pruned_sparse_b200 import build
    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    build.build()
    x = W.make_inputs(w)
    T = w.seq_len
    s = hb.Session(batch=w.batch, n_qheads=w.n_qheads, n_kvheads=w.n_kvheads, seq_len=T,
                   q_len=1, q_pos0=T - 1, dtype=hb.HIPS_BF16, block_q=1, block_k=w.block_k,
                   topk=w.topk, sink=w.sink, window=w.window)
    q = torch.from_numpy(x["q"][0]).cuda().to(torch.bfloat16).contiguous()
    k = torch.from_numpy(x["k"]).cuda().to(torch.bfloat16).contiguous()
    v = torch.from_numpy(x["v"]).cuda().to(torch.bfloat16).contiguous()
    return s, q, k, v


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    w = W.Workload("noalloc", "decode", 2, 32, 8, 128, 16384, 1, 2, 1024, 128, 512, "bf16",
                   needles=4, needle_mode="uniform")
    s, q, k, v = _setup(w)
    assert hb.workspace_size(s.p, hb.OP_SPARSE) <= hb.NOALLOC_SCRATCH_BYTES
    idx = s.mask(q, k)
    ref = s.sparse_attn(q, k, v, idx)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        hb.hip_sparse_attn_noalloc(q, k, v, idx, s.p, out)
        torch.cuda.synchronize()
        hb.noalloc_check_status()  # no bounded wait of the call gave up
        err = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= TOL_MAX and err.mean().item() <= TOL_MEAN
    s.check()


def test_noalloc_refuses_requests_beyond_its_array():
    # 64 query heads over 8 KV heads at 128k: the split-K partials of 64 rows
    # (about 0.6 MB) need more than the 512 KiB array holds
    big = hb.params(batch=1, n_qheads=64, n_kvheads=8, seq_len=131072, q_len=1,
                    q_pos0=131071, dtype=hb.HIPS_BF16, block_q=1, block_k=2, topk=2048,
                    sink=128, window=1024)
    need = hb.workspace_size(big, hb.OP_SPARSE)
    assert need > hb.NOALLOC_SCRATCH_BYTES, need
    f = 1 << 20  # never dereferenced: refused before any launch
    assert hb.sparse_attn_noalloc_ptr(f, f, f, f, big, f) == hb.HIPS_ERR_TOO_LARGE
    assert "scratch" in hb.error_string(hb.HIPS_ERR_TOO_LARGE)
