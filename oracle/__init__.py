"""CPU oracle for hierarchically pruned attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library (the CUDA path)
never imports, links or calls it; the two share no code.

The arithmetic lives in ``hip_oracle.c`` (plain C, compiled here with gcc);
this module only builds it and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hip_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-mfma",
          "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile hip_oracle.c into liboracle.so (skipped when up to date)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


class Stage(ctypes.Structure):
    """Mirror of ``oracle_stage`` in hip_oracle.c: one pruning stage."""

    _fields_ = [("chunk_size", ctypes.c_int32), ("stage_k", ctypes.c_int32),
                ("stride_q", ctypes.c_int32), ("pad", ctypes.c_int32)]


class Shape(ctypes.Structure):
    """Mirror of ``oracle_shape`` in hip_oracle.c."""

    _fields_ = [
        ("batch", ctypes.c_int32), ("n_qheads", ctypes.c_int32),
        ("n_kvheads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("seq_len", ctypes.c_int64), ("mask_len", ctypes.c_int64),
        ("kv_capacity", ctypes.c_int64), ("q_len", ctypes.c_int32),
        ("pad0", ctypes.c_int32), ("q_pos0", ctypes.c_int64),
        ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
        ("topk", ctypes.c_int32), ("sink", ctypes.c_int32),
        ("window", ctypes.c_int32), ("per_head", ctypes.c_int32),
        ("n_stages", ctypes.c_int32), ("stages", ctypes.POINTER(Stage)),
    ]


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    try:
        build()
        lib = ctypes.CDLL(_LIB)
    except OSError:
        build(force=True)
        lib = ctypes.CDLL(_LIB)
    P = ctypes.POINTER
    f32p, i32p, i64p, f64p = (P(ctypes.c_float), P(ctypes.c_int32),
                              P(ctypes.c_int64), P(ctypes.c_double))
    lib.oracle_canonical_dot.restype = ctypes.c_float
    lib.oracle_canonical_dot.argtypes = [f32p, f32p, ctypes.c_int]
    lib.oracle_idx_cap.restype = ctypes.c_int64
    lib.oracle_idx_cap.argtypes = [P(Shape)]
    lib.oracle_num_qblocks.restype = ctypes.c_int64
    lib.oracle_num_qblocks.argtypes = [P(Shape)]
    lib.oracle_set_threads.restype = ctypes.c_int
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_mask.restype = ctypes.c_int
    lib.oracle_mask.argtypes = [f32p, f32p, P(Shape), i64p, ctypes.c_int64, i32p, f64p, i32p, i64p]
    lib.oracle_block_scores.restype = ctypes.c_int
    lib.oracle_block_scores.argtypes = [f32p, f32p, P(Shape), ctypes.c_int64, i64p, ctypes.c_int64,
                                        f32p]
    lib.oracle_decode_e5m2.restype = None
    lib.oracle_decode_e5m2.argtypes = [P(ctypes.c_uint8), ctypes.c_int64, f32p]
    lib.oracle_attention.restype = ctypes.c_int
    lib.oracle_attention.argtypes = [f32p, f32p, f32p, i32p, P(Shape), i64p, ctypes.c_int64, f32p]
    _lib = lib
    return lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def shape(*, batch, n_qheads, n_kvheads, head_dim, seq_len, q_len, q_pos0, block_q,
          block_k, topk, sink=0, window=0, mask_len=None, kv_capacity=None, per_head=0,
          stages=()) -> Shape:
    """per_head=1: one mask per query head (idx rows [B, Hq, n_qblocks]) instead of
    one per KV-head group. stages: (chunk_size, stage_k, stride_q) per pruning
    stage before the iteration (stage_k 0 keeps every chunk); topk is then
    the iteration's budget (second_stage_k)."""
    st = (Stage * max(1, len(stages)))(*[Stage(int(c), int(k), int(r), 0) for c, k, r in stages])
    sh = Shape(batch=batch, n_qheads=n_qheads, n_kvheads=n_kvheads, head_dim=head_dim,
               seq_len=seq_len, mask_len=seq_len if mask_len is None else mask_len,
               kv_capacity=seq_len if kv_capacity is None else kv_capacity,
               q_len=q_len, pad0=0, q_pos0=q_pos0, block_q=block_q, block_k=block_k,
               topk=topk, sink=sink, window=window, per_head=int(per_head),
               n_stages=len(stages), stages=ctypes.cast(st, ctypes.POINTER(Stage)))
    sh._stage_array = st  # keeps the stage list alive with the shape
    return sh


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (n <= 0 keeps it); returns the count in use."""
    return int(_load().oracle_set_threads(int(n)))


def decode_e5m2(codes) -> np.ndarray:
    """float32 values of fp8 e5m2 codes (uint8 array of any shape)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float32)
    _load().oracle_decode_e5m2(_ptr(c, ctypes.c_uint8), c.size, _ptr(out, ctypes.c_float))
    return out


def canonical_dot(q, k) -> np.float32:
    q, k = _f32(q), _f32(k)
    assert q.shape == k.shape and q.ndim == 1 and q.size % 64 == 0
    return np.float32(_load().oracle_canonical_dot(_ptr(q, ctypes.c_float),
                                                   _ptr(k, ctypes.c_float), q.size))


def idx_cap(sh: Shape) -> int:
    return int(_load().oracle_idx_cap(ctypes.byref(sh)))


def num_qblocks(sh: Shape) -> int:
    return int(_load().oracle_num_qblocks(ctypes.byref(sh)))


def mask(q, k, sh: Shape, units=None, with_scored=False):
    """Hierarchical top-k masks.

    q: [B, Hq, Lq, d]; k: [B, Hkv, kv_capacity, d] (float32 values).
    Returns (idx [n_units, 1 + cap] int32, gap [n_units] float64,
    rounds [n_units] int32) -- plus scored [n_units] int64, the candidates
    scored over all rounds, when with_scored -- units in (b, g, qb) row-major
    order (g a KV head, or a query head with sh.per_head) unless an explicit
    list of flattened unit ids is given.
    """
    lib = _load()
    q, k = _f32(q), _f32(k)
    total = sh.batch * (sh.n_qheads if sh.per_head else sh.n_kvheads) * num_qblocks(sh)
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int64)
    n = total if u is None else u.size
    idx = np.empty((n, 1 + idx_cap(sh)), dtype=np.int32)
    gap = np.empty(n, dtype=np.float64)
    rounds = np.empty(n, dtype=np.int32)
    scored = np.empty(n, dtype=np.int64)
    st = lib.oracle_mask(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float), ctypes.byref(sh),
                         None if u is None else _ptr(u, ctypes.c_int64), n,
                         _ptr(idx, ctypes.c_int32), _ptr(gap, ctypes.c_double),
                         _ptr(rounds, ctypes.c_int32), _ptr(scored, ctypes.c_int64))
    if st != 0:
        raise RuntimeError(f"oracle_mask failed ({st})")
    if with_scored:
        return idx, gap, rounds, scored
    return idx, gap, rounds


def block_scores(q, k, sh: Shape, unit: int, blocks) -> np.ndarray:
    """float32 scores (step 3 of the rounds: max over the unit's query rows and
    the block's visible keys of the canonical dot) of the given key blocks of
    one mask row; -inf outside the unit's block range."""
    lib = _load()
    q, k = _f32(q), _f32(k)
    b = np.ascontiguousarray(blocks, dtype=np.int64)
    out = np.empty(b.size, dtype=np.float32)
    st = lib.oracle_block_scores(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                 ctypes.byref(sh), int(unit), _ptr(b, ctypes.c_int64), b.size,
                                 _ptr(out, ctypes.c_float))
    if st != 0:
        raise RuntimeError(f"oracle_block_scores failed ({st})")
    return out


def attention(q, k, v, idx, sh: Shape, rows=None) -> np.ndarray:
    """Sparse (idx given, [B*Hkv*nQB, 1 + cap]) or dense causal (idx None)
    attention; returns [n_rows, d] float32 for the flattened (b, h, i) rows."""
    lib = _load()
    q, k, v = _f32(q), _f32(k), _f32(v)
    total = sh.batch * sh.n_qheads * sh.q_len
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = total if r is None else r.size
    out = np.empty((n, sh.head_dim), dtype=np.float32)
    ix = None if idx is None else np.ascontiguousarray(idx, dtype=np.int32)
    st = lib.oracle_attention(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                              _ptr(v, ctypes.c_float),
                              None if ix is None else _ptr(ix, ctypes.c_int32),
                              ctypes.byref(sh), None if r is None else _ptr(r, ctypes.c_int64),
                              n, _ptr(out, ctypes.c_float))
    if st != 0:
        raise RuntimeError(f"oracle_attention failed ({st})")
    return out
