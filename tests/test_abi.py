"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/hip_sparse.h, and rejects bad arguments on the host
before anything is launched (no compute call is made here)."""
import os
import re

import pytest

from hierarchically_pruned_sparse_b200 import binding as hb
from hierarchically_pruned_sparse_b200 import build as hbuild
from hierarchically_pruned_sparse_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def lib():
    hbuild.build()
    return hb.load()


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"HIPS_API\s+[\w\s\*]+?\b(hip_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert len(declared) >= 9
    assert set(hb.EXPORTS) <= set(declared)
    for name in declared:
        assert hasattr(lib, name), name


def test_error_strings(lib):
    for code in (0, -1, -2, -3, -4, -5):
        assert hb.error_string(code)
    assert hb.error_string(-99) == "unknown status"


def _decode_params(**kw):
    base = dict(batch=1, n_qheads=32, n_kvheads=8, seq_len=131072, q_len=1, q_pos0=131071,
                dtype=hb.HIPS_BF16, block_q=1, block_k=2, topk=2048, sink=128, window=1024)
    base.update(kw)
    return hb.params(**base)


def test_row_stride_and_workspace_sizes():
    p = _decode_params()
    # 1 (nnz) + topk/bk + ceil(sink/bk) + ceil((window + bq - 1)/bk) + 1
    assert hb.idx_row_stride(p) == 1 + 1024 + 64 + 512 + 1
    assert hb.workspace_size(p, hb.OP_MASK) >= 256
    assert hb.workspace_size(p, hb.OP_SPARSE) > 256  # split-K partials
    assert hb.workspace_size(p, hb.OP_DENSE) > 256
    p2 = _decode_params(window=0, sink=0)
    assert hb.idx_row_stride(p2) == 1 + 1024


@pytest.mark.parametrize("bad,code", [
    (dict(n_qheads=30), hb.HIPS_ERR_INVALID_ARG),        # head ratio
    (dict(topk=2047), hb.HIPS_ERR_INVALID_ARG),          # topk % block_k
    (dict(block_k=3, topk=3 * 512), hb.HIPS_ERR_INVALID_ARG),  # block_k not a power of two
    (dict(head_dim=64), hb.HIPS_ERR_UNSUPPORTED),
    (dict(dtype=7), hb.HIPS_ERR_UNSUPPORTED),
    (dict(q_pos0=131072), hb.HIPS_ERR_INVALID_ARG),      # query past the cache
    (dict(mask_len=131073), hb.HIPS_ERR_INVALID_ARG),
    (dict(kv_capacity=1000), hb.HIPS_ERR_INVALID_ARG),
    (dict(topk=2 * 4096), hb.HIPS_ERR_UNSUPPORTED),      # more than 2048 chunks
    (dict(batch=0), hb.HIPS_ERR_INVALID_ARG),
    (dict(sink=-1), hb.HIPS_ERR_INVALID_ARG),
])
def test_bad_arguments_rejected_on_host(bad, code):
    p = _decode_params(**bad)
    fake = 1 << 20  # never dereferenced: validation fails first
    assert hb.mask_ptr(fake, fake, p, fake) == code
    assert hb.sparse_attn_ptr(fake, fake, fake, fake, p, fake) == code
    assert hb.mask_sparse_attn_ptr(fake, fake, fake, p, fake, fake) == code
    assert hb.workspace_size(p, hb.OP_MASK) == 0
    assert hb.workspace_size(p, hb.OP_MASK_SPARSE) == 0


def test_null_and_misaligned_pointers_rejected():
    p = _decode_params(workspace=1 << 20, workspace_bytes=1 << 30)
    f = 1 << 20
    assert hb.mask_ptr(0, f, p, f) == hb.HIPS_ERR_INVALID_ARG
    assert hb.mask_ptr(f, 0, p, f) == hb.HIPS_ERR_INVALID_ARG
    assert hb.mask_ptr(f, f, p, 0) == hb.HIPS_ERR_INVALID_ARG
    assert hb.mask_ptr(f + 8, f, p, f) == hb.HIPS_ERR_INVALID_ARG  # q not 16-byte aligned
    assert hb.sparse_attn_ptr(f, f, f, 0, p, f) == hb.HIPS_ERR_INVALID_ARG
    assert hb.dense_attn_ptr(f, f, 0, p, f) == hb.HIPS_ERR_INVALID_ARG


def test_workspace_checked_before_launch():
    f = 1 << 20
    p = _decode_params()  # no workspace
    assert hb.mask_ptr(f, f, p, f) == hb.HIPS_ERR_WORKSPACE
    need = hb.workspace_size(p, hb.OP_SPARSE)
    p = _decode_params(workspace=f, workspace_bytes=need - 1)
    assert hb.sparse_attn_ptr(f, f, f, f, p, f) == hb.HIPS_ERR_WORKSPACE
    p = _decode_params(workspace=f + 16, workspace_bytes=need)  # not 256-byte aligned
    assert hb.sparse_attn_ptr(f, f, f, f, p, f) == hb.HIPS_ERR_WORKSPACE


def test_unknown_flag_bits_rejected_and_head_masks_accepted():
    f = 1 << 20
    bad = _decode_params(flags=2)
    assert hb.mask_ptr(f, f, bad, f) == hb.HIPS_ERR_INVALID_ARG
    assert hb.workspace_size(bad, hb.OP_MASK) == 0
    p = _decode_params(flags=hb.FLAG_HEAD_MASKS)
    assert hb.workspace_size(p, hb.OP_MASK) >= 256
    assert hb.idx_row_stride(p) == hb.idx_row_stride(_decode_params())
    assert hb.mask_ptr(f, f, p, f) == hb.HIPS_ERR_WORKSPACE  # valid up to the missing workspace


def test_fused_call_checks_on_host():
    f = 1 << 20
    need = hb.workspace_size(_decode_params(), hb.OP_MASK_SPARSE)
    assert need == max(hb.workspace_size(_decode_params(), hb.OP_MASK),
                       hb.workspace_size(_decode_params(), hb.OP_SPARSE))
    # a reused mask (keys appended since it was computed) is not a fresh mask
    p = _decode_params(seq_len=131080, kv_capacity=131080, q_pos0=131079, mask_len=131072,
                       workspace=f, workspace_bytes=need)
    assert hb.mask_sparse_attn_ptr(f, f, f, p, f, f) == hb.HIPS_ERR_INVALID_ARG
    p = _decode_params(workspace=f, workspace_bytes=need)
    assert hb.mask_sparse_attn_ptr(f, f, 0, p, f, f) == hb.HIPS_ERR_INVALID_ARG   # v missing
    assert hb.mask_sparse_attn_ptr(f, f, f, p, f, f + 8) == hb.HIPS_ERR_INVALID_ARG  # out misaligned
    assert hb.mask_sparse_attn_ptr(f, f, f, _decode_params(), f, f) == hb.HIPS_ERR_WORKSPACE


def test_prefill_shapes_plan():
    p = hb.params(batch=1, n_qheads=32, n_kvheads=8, seq_len=32768, q_len=32768, q_pos0=0,
                  dtype=hb.HIPS_BF16, block_q=64, block_k=2, topk=2048, sink=128, window=1024)
    assert hb.idx_row_stride(p) == 1 + 1024 + 64 + 544 + 1


def _up(n):
    return (n + 255) // 256 * 256


def test_e5m2_kv_plans_decode_natively_and_other_shapes_by_widening():
    f = 1 << 20
    p = _decode_params(dtype=hb.HIPS_BF16_E5M2)
    for op in (hb.OP_MASK, hb.OP_SPARSE, hb.OP_DENSE, hb.OP_MASK_SPARSE):
        assert hb.workspace_size(p, op) >= 256, op
    assert hb.mask_ptr(f, f, p, f) == hb.HIPS_ERR_WORKSPACE  # valid up to the missing workspace
    # the decode shapes have e5m2 kernels: no room for widened rows
    assert hb.workspace_size(p, hb.OP_MASK) < 8 * 131072 * 128 * 2

    def widened(**kw):
        # shapes without an e5m2 kernel: the bf16 plan (compact rows), then
        # K (mask) or K and V (attention) widened to bf16 in the workspace
        e = hb.params(**kw, dtype=hb.HIPS_BF16_E5M2)
        b = hb.params(**kw, dtype=hb.HIPS_BF16)
        rows = _up(kw["batch"] * kw["n_kvheads"] * kw["seq_len"] * 128 * 2)
        for op, n in ((hb.OP_MASK, 1), (hb.OP_SPARSE, 2), (hb.OP_DENSE, 2), (hb.OP_MASK_SPARSE, 2)):
            w = hb.workspace_size(b, op)
            want = _up(w) + n * rows if w else 0  # no bf16 plan: none either
            assert hb.workspace_size(e, op) == want, (op, hb.workspace_size(e, op), want)

    # more than 16 rows per mask (one MMA column block) has no e5m2 mask kernel
    widened(batch=1, n_qheads=64, n_kvheads=2, seq_len=131072, q_len=1, q_pos0=131071,
            block_q=1, block_k=2, topk=2048, sink=128, window=1024)
    # prefill query blocks: neither the mask nor the attention has an e5m2 kernel
    widened(batch=1, n_qheads=32, n_kvheads=8, seq_len=32768, q_len=32768, q_pos0=0,
            block_q=64, block_k=2, topk=2048, sink=128, window=1024)
    # 2048 chunks per mask do not fit beside the tensor-core kernel's tiles:
    # e5m2 decode masks (one query position, at most 8 rows) then run on the
    # CUDA-core decode kernel, bf16 ones on the CUDA-core mask kernel
    big = _decode_params(dtype=hb.HIPS_BF16_E5M2, topk=4096)
    assert 256 <= hb.workspace_size(big, hb.OP_MASK) < 8 * 131072 * 128 * 2
    assert hb.workspace_size(_decode_params(topk=4096), hb.OP_MASK) >= 256


@pytest.mark.parametrize("name", sorted(W.WORKLOADS))
def test_every_workload_plans_every_op(name):
    # each benchmarked workload (and its mask reuse steps) has a kernel plan
    # for the mask, the sparse and dense attention and the one-call step
    w = W.WORKLOADS[name]
    code = {"bf16": hb.HIPS_BF16, "f32": hb.HIPS_F32, "e5m2": hb.HIPS_BF16_E5M2}[w.dtype]
    T = w.seq_len
    q_len = 1 if w.kind == "decode" else T
    p = hb.params(batch=w.batch, n_qheads=w.n_qheads, n_kvheads=w.n_kvheads, seq_len=T,
                  q_len=q_len, q_pos0=T - q_len, dtype=code, block_q=w.block_q,
                  block_k=w.block_k, topk=w.topk, sink=w.sink, window=w.window,
                  kv_capacity=w.capacity)
    for op in (hb.OP_MASK, hb.OP_SPARSE, hb.OP_DENSE, hb.OP_MASK_SPARSE):
        assert hb.workspace_size(p, op) >= 256, (name, op)
    if w.refresh > 1:  # a later step attends the keys appended since the refresh
        later = hb.params(batch=w.batch, n_qheads=w.n_qheads, n_kvheads=w.n_kvheads,
                          seq_len=T + w.refresh - 1, q_len=1, q_pos0=T + w.refresh - 2,
                          dtype=code, block_q=w.block_q, block_k=w.block_k, topk=w.topk,
                          sink=w.sink, window=w.window, mask_len=T, kv_capacity=w.capacity)
        assert hb.workspace_size(later, hb.OP_SPARSE) >= 256


@pytest.mark.parametrize("flags", [0, 1])
def test_head_masks_plan_decode_and_prefill(flags):
    for q_len, bq in ((1, 1), (4096, 64)):
        p = hb.params(batch=1, n_qheads=32, n_kvheads=8, seq_len=4096, q_len=q_len,
                      q_pos0=4096 - q_len, dtype=hb.HIPS_BF16, block_q=bq, block_k=2,
                      topk=512, sink=16, window=64, flags=flags)
        assert hb.workspace_size(p, hb.OP_MASK) >= 256
        assert hb.workspace_size(p, hb.OP_SPARSE) >= 256


# ---------------------------------------------------------------- pruning stages
# (struct hips_stage: the stages of the serving command's --hip-attention-config
# in "[Feature] Support Efficient Sparse HiP Attention (InfiniteHiP)")
PR_LIKE = ((128, 0, 4), (32, 32768, 4), (8, 8192, 1))


def test_stage_schedules_are_sized_by_their_bounds():
    plain = hb.workspace_size(_decode_params(), hb.OP_MASK)
    staged = hb.workspace_size(_decode_params(stages=PR_LIKE), hb.OP_MASK)
    # 8 mask rows: scores for 4096 chunks (65536 blocks in chunks of 16) and
    # two lists of 4 + 2 x 4096 int32, each area rounded up to 256 bytes
    cap, rows = 4096, 8

    def up(n):
        return (n + 255) // 256 * 256

    assert staged == up(plain) + up(rows * cap * 4) + 2 * up(rows * (4 + 2 * cap) * 4)
    # attention-only calls ignore the stages
    assert hb.workspace_size(_decode_params(stages=PR_LIKE), hb.OP_SPARSE) == \
        hb.workspace_size(_decode_params(), hb.OP_SPARSE)


@pytest.mark.parametrize("stages", [
    ((3, 0, 1),),                    # not a whole number of 2-key blocks
    ((32, 48, 1),),                  # stage_k not a whole number of chunks
    ((32, 0, 1), (128, 0, 1)),       # a chunk size that does not divide the previous one
    ((32, 0, 0),),                   # stride 0
    ((32, -32, 1),),                 # negative stage_k
    tuple((2, 0, 1) for _ in range(9)),  # more than HIPS_MAX_STAGES
])
def test_bad_stage_schedules_are_rejected(stages):
    p = _decode_params(stages=stages)
    assert hb.workspace_size(p, hb.OP_MASK) == 0
    assert hb.workspace_size(p, hb.OP_MASK_SPARSE) == 0
    assert hb.workspace_size(p, hb.OP_SPARSE) > 0  # the attention does not read them


def test_a_stage_count_without_a_stage_array_is_rejected():
    p = _decode_params()
    p.n_stages = 2  # and no array
    assert hb.workspace_size(p, hb.OP_MASK) == 0
    assert hb.mask_ptr(1 << 20, 1 << 20, p, 1 << 20) == hb.HIPS_ERR_INVALID_ARG


def test_stage_schedules_that_leave_more_than_n0_chunks_are_unsupported():
    # the iteration starts from at most topk / block_k = 1024 chunks: 8-key
    # chunks that all survive (16384 of them at 128k keys) are too many, so
    # are 2048 survivors of a stage that keeps 16384 keys in 8-key chunks
    assert hb.workspace_size(_decode_params(stages=((8, 0, 1),)), hb.OP_MASK) == 0
    assert hb.workspace_size(_decode_params(stages=((8, 16384, 1),)), hb.OP_MASK) == 0
    assert hb.workspace_size(_decode_params(stages=((8, 8192, 1),)), hb.OP_MASK) > 0


def test_binding_structs_match_the_header_layout(tmp_path):
    # sizes and field offsets of hips_params and hips_stage as a C compiler
    # lays them out from include/hip_sparse.h, against the ctypes mirrors
    import ctypes
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    fields = [f for f, _ in hb.Params._fields_]
    sfields = [f for f, _ in hb.Stage._fields_]
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "hip_sparse.h"', 'int main(void) {',
             '  printf("%zu %zu\\n", sizeof(hips_params), sizeof(hips_stage));']
    lines += [f'  printf("%zu\\n", offsetof(hips_params, {f}));' for f in fields]
    lines += [f'  printf("%zu\\n", offsetof(hips_stage, {f}));' for f in sfields]
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", f"-I{os.path.join(root, 'include')}", str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    vals = [int(v) for v in out]
    assert vals[0] == ctypes.sizeof(hb.Params) and vals[1] == ctypes.sizeof(hb.Stage)
    assert vals[2:2 + len(fields)] == [getattr(hb.Params, f).offset for f in fields]
    assert vals[2 + len(fields):] == [getattr(hb.Stage, f).offset for f in sfields]
