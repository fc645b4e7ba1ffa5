"""Calls from several host threads at once, each on its own stream and
workspace, give the same masks and outputs as the same calls made one after
another. The shapes differ per thread, so the threads also plan new kernel
shapes concurrently (the launch-attribute and residency caches)."""
import threading

import numpy as np
import pytest

from hierarchically_pruned_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    from hierarchically_pruned_sparse_b200 import build
    assert torch.cuda.is_available(), "gpu tests need a CUDA device"
    build.build()


# (name, kind, Hq, Hkv, T, b_q, b_k, k, sink, window, dtype): a fused decode
# group, a two-call decode in fp32, and two small prefill shapes
CASES = [
    ("thr_dec", "decode", 8, 2, 3000, 1, 2, 128, 4, 32, "bf16"),
    ("thr_f32", "decode", 4, 2, 1500, 1, 2, 64, 0, 16, "f32"),
    ("thr_pre", "prefill", 4, 1, 700, 64, 2, 128, 8, 64, "bf16"),
    ("thr_pre16", "prefill", 4, 2, 900, 16, 4, 64, 0, 32, "bf16"),
]


def _setup(case):
    import torch
    from hierarchically_pruned_sparse_b200 import binding as hb
    name, kind, hq, hkv, T, bq, bk, topk, sink, window, dtype = case
    w = W.Workload(name, kind, 1, hq, hkv, 128, T, bq, bk, topk, sink, window, dtype)
    x = W.make_inputs(w)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q_np = x["q"][0]
    q_len = 1 if kind == "decode" else T
    q_pos0 = T - 1 if kind == "decode" else 0
    stream = torch.cuda.Stream()
    s = hb.Session(batch=1, n_qheads=hq, n_kvheads=hkv, seq_len=T, q_len=q_len, q_pos0=q_pos0,
                   block_q=bq, block_k=bk, topk=topk, sink=sink, window=window,
                   dtype=hb.HIPS_BF16 if dtype == "bf16" else hb.HIPS_F32, stream=stream)
    q = torch.from_numpy(np.ascontiguousarray(q_np)).cuda().to(dt).contiguous()
    k = torch.from_numpy(x["k"]).cuda().to(dt).contiguous()
    v = torch.from_numpy(x["v"]).cuda().to(dt).contiguous()
    return dict(s=s, q=q, k=k, v=v, kind=kind, stream=stream)


def _run(c, reps):
    import torch
    outs = []
    with torch.cuda.stream(c["stream"]):
        for _ in range(reps):
            if c["kind"] == "decode":
                idx, out = c["s"].mask_sparse_attn(c["q"], c["k"], c["v"])
            else:
                idx = c["s"].mask(c["q"], c["k"])
                out = c["s"].sparse_attn(c["q"], c["k"], c["v"], idx)
            outs.append((idx, out))
    c["stream"].synchronize()
    c["s"].check()
    return [(i.cpu().numpy(), o.float().cpu().numpy()) for i, o in outs]


def test_concurrent_host_threads_match_sequential_calls():
    import torch
    cases = [_setup(c) for c in CASES]
    torch.cuda.synchronize()
    results = [None] * len(cases)
    errors = []
    start = threading.Barrier(len(cases))

    def worker(i):
        try:
            start.wait(timeout=60)
            results[i] = _run(cases[i], reps=4)
        except Exception as e:  # reported below, with the thread's case
            errors.append((CASES[i][0], repr(e)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a host thread did not finish"
    assert not errors, errors
    for i, c in enumerate(cases):
        ref_idx, ref_out = _run(c, reps=1)[0]
        for idx, out in results[i]:
            np.testing.assert_array_equal(idx, ref_idx, err_msg=CASES[i][0])
            np.testing.assert_array_equal(out, ref_out, err_msg=CASES[i][0])
