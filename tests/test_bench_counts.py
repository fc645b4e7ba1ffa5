"""The benchmark's algorithmic byte counts (the roofline numerators), on CPU.

The counts are closed forms of the workload shape and of the scored-candidate
and idx contents: each scored candidate reads its representative block of b_k
key rows, each attended key one K and one V row, plus q, the output and the
idx rows. An fp8 e5m2 KV cache halves the key and value bytes and leaves the
q and output bytes at bf16.
"""
import dataclasses
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from hierarchically_pruned_sparse_b200 import workloads as W  # noqa: E402


def _idx_rows(w: W.Workload, nnz: int) -> np.ndarray:
    """idx rows that each list blocks 0..nnz-1 (within the cache)."""
    units = w.batch * w.n_kvheads * (-(-w.q_len // w.block_q))
    rows = np.full((units, 1 + nnz + 3), -1, np.int32)
    rows[:, 0] = nnz
    rows[:, 1:1 + nnz] = np.arange(nnz)
    return rows


def test_element_sizes():
    assert bench.elem_bytes(W.DECODE_128K) == (2, 2)
    assert bench.elem_bytes(W.DECODE_128K_E5M2) == (2, 1)
    assert bench.elem_bytes(W.DECODE_8K_F32) == (4, 4)


def test_mask_bytes_closed_form():
    w = W.DECODE_128K
    scored = 12345
    units = w.batch * w.n_kvheads
    stride = 1 + w.topk // w.block_k + w.sink // w.block_k + (w.window + 1 - 1) // w.block_k + 1
    q_bytes = w.batch * w.n_qheads * w.head_dim * 2
    assert bench.mask_algorithmic_bytes(w, scored) == (
        scored * w.block_k * w.head_dim * 2 + q_bytes + units * stride * 4)


def test_e5m2_halves_key_and_value_bytes_only():
    wb, w8 = W.DECODE_128K, W.DECODE_128K_E5M2
    scored = 98304
    kv = scored * wb.block_k * wb.head_dim
    assert bench.mask_algorithmic_bytes(wb, scored) - bench.mask_algorithmic_bytes(w8, scored) == kv
    idx = _idx_rows(wb, 1600)
    keys = idx.shape[0] * 1600 * wb.block_k
    diff = (bench.attn_algorithmic_bytes(wb, idx, wb.seq_len, wb.seq_len)
            - bench.attn_algorithmic_bytes(w8, idx, w8.seq_len, w8.seq_len))
    assert diff == keys * 2 * wb.head_dim  # K and V rows, one byte less per element


def test_attention_bytes_count_the_reuse_tail_and_clip_at_the_mask():
    w = dataclasses.replace(W.DECODE_128K, n_qheads=4, n_kvheads=1)
    idx = _idx_rows(w, 10)
    base = bench.attn_algorithmic_bytes(w, idx, w.seq_len, w.seq_len)
    # 7 keys appended since the refresh: each unit reads them too
    grown = bench.attn_algorithmic_bytes(w, idx, w.seq_len + 7, w.seq_len)
    assert grown - base == idx.shape[0] * 7 * 2 * w.head_dim * 2
    # a listed block past mask_len contributes no keys
    idx2 = idx.copy()
    idx2[:, 10] = (w.seq_len + 100) // w.block_k
    assert (bench.attn_algorithmic_bytes(w, idx2, w.seq_len, w.seq_len)
            == base - idx.shape[0] * w.block_k * 2 * w.head_dim * 2)


def test_oracle_inputs_decode_e5m2_and_pass_others_through():
    x = {"q": np.zeros((1, 1, 1, 1, 128), np.float32),
         "k": np.array([[0x3C, 0xC0]], np.uint8), "v": np.array([[0x40, 0x01]], np.uint8)}
    out = bench.oracle_inputs(W.DECODE_128K_E5M2, x)
    np.testing.assert_array_equal(out["k"], np.array([[1.0, -2.0]], np.float32))
    np.testing.assert_array_equal(out["v"], np.array([[2.0, 2.0 ** -16]], np.float32))
    assert bench.oracle_inputs(W.DECODE_128K, x) is x


def test_layer_buffers_outgrow_the_l2_by_the_bytes_a_step_touches():
    # decode at 128k touches ~63 MB per step (six rounds of 2048 two-key
    # candidates per KV head, then ~1600 attended blocks of K and V): at
    # least 4x the 126 MB L2 between two uses of a layer takes 9 layers
    w = W.DECODE_128K
    t = bench.touched_bytes(w)
    assert t == 8 * (6 * 2048 + 2 * (1024 + 64 + 513)) * 2 * 128 * 2
    n = bench.layer_count(w, 537 << 20, 0)
    assert n * t >= 4 * bench.L2_BYTES and (n - 1) * t < 4 * bench.L2_BYTES
    # prefill reads all of q, k and v; a requested count is kept
    assert bench.touched_bytes(W.PREFILL_32K) == (2 * 8 + 32) * 32768 * 128 * 2
    assert bench.layer_count(W.PREFILL_32K, 400 << 20, 5) == 5


def test_stage_launch_counts():
    # a scoring and a selection launch per stage that ranks; one selection
    # launch (cut and halve only) when none ranks; nothing without stages
    saved = bench.STAGES
    try:
        bench.STAGES = ()
        assert bench.stage_launches() == 0
        bench.STAGES = ((128, 0, 4), (32, 32768, 4), (8, 8192, 1))
        assert bench.stage_launches() == 4
        bench.STAGES = ((64, 0, 1),)
        assert bench.stage_launches() == 1
        cfg = bench.config_of(W.DECODE_128K, 0)
        assert cfg["stages"] == [{"chunk_size": 64, "stage_k": None, "stride_q": 1}]
    finally:
        bench.STAGES = saved
