"""ctypes binding of libhip_sparse.so (argument marshalling only).

Every step of the hot path runs in the library's CUDA kernels; this module
only turns torch tensors (device memory) and a torch stream into the plain
pointers and sizes of the C ABI declared in include/hip_sparse.h. It fails
loudly when the library is missing; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

HIPS_OK = 0
HIPS_ERR_INVALID_ARG = -1
HIPS_ERR_UNSUPPORTED = -2
HIPS_ERR_WORKSPACE = -3
HIPS_ERR_CUDA = -4
HIPS_ERR_TIMEOUT = -5
HIPS_ERR_TOO_LARGE = -6
HIPS_ERR_INTERNAL = -7
MAX_STAGES = 8
NOALLOC_SCRATCH_BYTES = 512 << 10

HIPS_F32 = 0
HIPS_BF16 = 1
HIPS_BF16_E5M2 = 2  # bf16 q and out, fp8 e5m2 k and v (uint8 codes)

OP_MASK = 0
OP_SPARSE = 1
OP_DENSE = 2
OP_MASK_SPARSE = 3
FLAG_HEAD_MASKS = 1  # one mask per query head (idx [B, Hq, n_qblocks, row_stride])

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhip_sparse.so")
EXPORTS = ("hip_idx_row_stride", "hip_workspace_size", "hip_workspace_init", "hip_check_status",
           "hip_mask", "hip_sparse_attn", "hip_mask_sparse_attn", "hip_dense_attn",
           "hip_sparse_attn_noalloc", "hip_noalloc_check_status", "hip_last_cuda_error",
           "hip_error_string")


class HipsError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({detail})")


class Stage(ctypes.Structure):
    """Mirror of ``hips_stage`` (include/hip_sparse.h): one pruning stage."""

    _fields_ = [("chunk_size", ctypes.c_int32), ("stage_k", ctypes.c_int32),
                ("stride_q", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class Params(ctypes.Structure):
    """Mirror of ``hips_params`` (include/hip_sparse.h)."""

    _fields_ = [
        ("batch", ctypes.c_int32), ("n_qheads", ctypes.c_int32),
        ("n_kvheads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("seq_len", ctypes.c_int64), ("mask_len", ctypes.c_int64),
        ("kv_capacity", ctypes.c_int64), ("q_len", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("q_pos0", ctypes.c_int64),
        ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
        ("topk", ctypes.c_int32), ("sink", ctypes.c_int32),
        ("window", ctypes.c_int32), ("flags", ctypes.c_int32),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("stream", ctypes.c_void_p),
        ("n_stages", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("stages", ctypes.POINTER(Stage)),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m hierarchically_pruned_sparse_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp = ctypes.c_void_p
    lib.hip_idx_row_stride.restype = ctypes.c_int64
    lib.hip_idx_row_stride.argtypes = [P]
    lib.hip_workspace_size.restype = ctypes.c_size_t
    lib.hip_workspace_size.argtypes = [P, ctypes.c_int]
    lib.hip_workspace_init.restype = ctypes.c_int
    lib.hip_workspace_init.argtypes = [P]
    lib.hip_check_status.restype = ctypes.c_int
    lib.hip_check_status.argtypes = [P]
    lib.hip_mask.restype = ctypes.c_int
    lib.hip_mask.argtypes = [vp, vp, P, vp]
    lib.hip_sparse_attn.restype = ctypes.c_int
    lib.hip_sparse_attn.argtypes = [vp, vp, vp, vp, P, vp]
    lib.hip_mask_sparse_attn.restype = ctypes.c_int
    lib.hip_mask_sparse_attn.argtypes = [vp, vp, vp, P, vp, vp]
    lib.hip_dense_attn.restype = ctypes.c_int
    lib.hip_dense_attn.argtypes = [vp, vp, vp, P, vp]
    lib.hip_sparse_attn_noalloc.restype = ctypes.c_int
    lib.hip_sparse_attn_noalloc.argtypes = [vp, vp, vp, vp, P, vp]
    lib.hip_noalloc_check_status.restype = ctypes.c_int
    lib.hip_noalloc_check_status.argtypes = [vp]
    lib.hip_last_cuda_error.restype = ctypes.c_int
    lib.hip_last_cuda_error.argtypes = []
    lib.hip_error_string.restype = ctypes.c_char_p
    lib.hip_error_string.argtypes = [ctypes.c_int]
    _lib = lib
    return lib


def error_string(code: int) -> str:
    return load().hip_error_string(int(code)).decode()


def _check(fn: str, code: int) -> None:
    if code != HIPS_OK:
        detail = error_string(code)
        if code == HIPS_ERR_CUDA:
            detail += f", cudaError {load().hip_last_cuda_error()}"
        raise HipsError(fn, code, detail)


def params(*, batch, n_qheads, n_kvheads, seq_len, q_len, q_pos0, dtype, block_q=1, block_k=1,
           topk=1, sink=0, window=0, mask_len=None, kv_capacity=None, head_dim=128,
           workspace=0, workspace_bytes=0, stream=0, flags=0, stages=()) -> Params:
    """stages: (chunk_size, stage_k, stride_q) per pruning stage (stage_k 0
    keeps every chunk); topk is then the iteration's budget."""
    p = Params(batch=batch, n_qheads=n_qheads, n_kvheads=n_kvheads, head_dim=head_dim,
               seq_len=seq_len, mask_len=seq_len if mask_len is None else mask_len,
               kv_capacity=seq_len if kv_capacity is None else kv_capacity, q_len=q_len,
               dtype=dtype, q_pos0=q_pos0, block_q=block_q, block_k=block_k, topk=topk,
               sink=sink, window=window, flags=flags, workspace=workspace or None,
               workspace_bytes=workspace_bytes, stream=stream or None)
    set_stages(p, stages)
    return p


def set_stages(p: Params, stages) -> None:
    """Point p at a stage list (kept alive with p)."""
    arr = (Stage * max(1, len(stages)))(*[Stage(int(c), int(k), int(r), 0) for c, k, r in stages])
    p._stage_array = arr
    p.n_stages = len(stages)
    p.stages = ctypes.cast(arr, ctypes.POINTER(Stage)) if stages else None


def idx_row_stride(p: Params) -> int:
    return int(load().hip_idx_row_stride(ctypes.byref(p)))


def workspace_size(p: Params, op: int) -> int:
    return int(load().hip_workspace_size(ctypes.byref(p), int(op)))


def workspace_init(p: Params) -> None:
    _check("hip_workspace_init", load().hip_workspace_init(ctypes.byref(p)))


def check_status(p: Params) -> None:
    _check("hip_check_status", load().hip_check_status(ctypes.byref(p)))


def mask_ptr(q: int, k: int, p: Params, idx_out: int) -> int:
    return int(load().hip_mask(q or None, k or None, ctypes.byref(p), idx_out or None))


def sparse_attn_ptr(q: int, k: int, v: int, idx: int, p: Params, out: int) -> int:
    return int(load().hip_sparse_attn(q or None, k or None, v or None, idx or None,
                                      ctypes.byref(p), out or None))


def mask_sparse_attn_ptr(q: int, k: int, v: int, p: Params, idx_out: int, out: int) -> int:
    return int(load().hip_mask_sparse_attn(q or None, k or None, v or None, ctypes.byref(p),
                                           idx_out or None, out or None))


def sparse_attn_noalloc_ptr(q: int, k: int, v: int, idx: int, p: Params, out: int) -> int:
    """hip_sparse_attn on the library's fixed scratch array (no workspace)."""
    return int(load().hip_sparse_attn_noalloc(q or None, k or None, v or None, idx or None,
                                              ctypes.byref(p), out or None))


def dense_attn_ptr(q: int, k: int, v: int, p: Params, out: int) -> int:
    return int(load().hip_dense_attn(q or None, k or None, v or None, ctypes.byref(p),
                                     out or None))


# ---------------------------------------------------------------- torch tensors


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return HIPS_BF16
    if t.dtype == torch.float32:
        return HIPS_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t) -> int:
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return t.data_ptr()


def hip_mask(q, k, p: Params, idx_out) -> None:
    """idx_out[...] = hierarchical top-k mask of (q, k) (see include/hip_sparse.h)."""
    _check("hip_mask", mask_ptr(_dev(q), _dev(k), p, _dev(idx_out)))


def hip_sparse_attn(q, k, v, idx, p: Params, out) -> None:
    _check("hip_sparse_attn", sparse_attn_ptr(_dev(q), _dev(k), _dev(v), _dev(idx), p, _dev(out)))


def hip_mask_sparse_attn(q, k, v, p: Params, idx_out, out) -> None:
    """hip_mask then hip_sparse_attn on its idx (one launch for decode shapes)."""
    _check("hip_mask_sparse_attn",
           mask_sparse_attn_ptr(_dev(q), _dev(k), _dev(v), p, _dev(idx_out), _dev(out)))


def hip_sparse_attn_noalloc(q, k, v, idx, p: Params, out) -> None:
    """Sparse attention for callers that cannot allocate device memory: the
    split-K scratch is a fixed array inside the library (see the header)."""
    _check("hip_sparse_attn_noalloc",
           sparse_attn_noalloc_ptr(_dev(q), _dev(k), _dev(v), _dev(idx), p, _dev(out)))


def noalloc_check_status(stream=None) -> None:
    """Raise if the last hip_sparse_attn_noalloc call on this device gave up a
    bounded wait (synchronises the stream; torch's current one by default)."""
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    _check("hip_noalloc_check_status", load().hip_noalloc_check_status(stream.cuda_stream or None))


def hip_dense_attn(q, k, v, p: Params, out) -> None:
    _check("hip_dense_attn", dense_attn_ptr(_dev(q), _dev(k), _dev(v), p, _dev(out)))


class Session:
    """Shapes, a device workspace and a stream for repeated calls.

    ``q`` is [B, Hq, q_len, d]; ``k``/``v`` are [B, Hkv, kv_capacity, d] torch
    tensors (bf16 or fp32) on the current device. The workspace is sized for
    every op and its status block is cleared once.
    """

    def __init__(self, *, batch, n_qheads, n_kvheads, seq_len, q_len, q_pos0, dtype, block_q=1,
                 block_k=1, topk=1, sink=0, window=0, mask_len=None, kv_capacity=None,
                 stream=None, flags=0, stages=()):
        import torch
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.p = params(batch=batch, n_qheads=n_qheads, n_kvheads=n_kvheads, seq_len=seq_len,
                        q_len=q_len, q_pos0=q_pos0, dtype=dtype, block_q=block_q,
                        block_k=block_k, topk=topk, sink=sink, window=window,
                        mask_len=mask_len, kv_capacity=kv_capacity,
                        stream=self.stream.cuda_stream, flags=flags, stages=stages)
        need = max(workspace_size(self.p, op) for op in (OP_MASK, OP_SPARSE, OP_DENSE, OP_MASK_SPARSE))
        if need == 0:
            raise HipsError("hip_workspace_size", HIPS_ERR_INVALID_ARG, "invalid parameters")
        self.workspace = torch.empty(need + 256, dtype=torch.uint8, device="cuda")
        base = self.workspace.data_ptr()
        self.p.workspace = (base + 255) // 256 * 256
        self.p.workspace_bytes = need
        workspace_init(self.p)
        self.nqb = -(-q_len // block_q)
        self.row_stride = idx_row_stride(self.p)

    def set(self, **kw) -> None:
        """Change scalar fields (seq_len, mask_len, q_pos0 ...) in place."""
        for key, val in kw.items():
            setattr(self.p, key, val)
        need = max(workspace_size(self.p, op) for op in (OP_MASK, OP_SPARSE, OP_DENSE, OP_MASK_SPARSE))
        if need > self.p.workspace_bytes:
            raise HipsError("hip_workspace_size", HIPS_ERR_WORKSPACE, "workspace too small")
        self.row_stride = idx_row_stride(self.p)

    def new_idx(self):
        import torch
        heads = self.p.n_qheads if self.p.flags & FLAG_HEAD_MASKS else self.p.n_kvheads
        return torch.empty((self.p.batch, heads, self.nqb, self.row_stride),
                           dtype=torch.int32, device="cuda")

    def mask(self, q, k, idx_out=None):
        idx = self.new_idx() if idx_out is None else idx_out
        hip_mask(q, k, self.p, idx)
        return idx

    def sparse_attn(self, q, k, v, idx, out=None):
        import torch
        o = torch.empty_like(q) if out is None else out
        hip_sparse_attn(q, k, v, idx, self.p, o)
        return o

    def mask_sparse_attn(self, q, k, v, idx_out=None, out=None):
        """Fresh mask and attention over it; returns (idx, out)."""
        import torch
        idx = self.new_idx() if idx_out is None else idx_out
        o = torch.empty_like(q) if out is None else out
        hip_mask_sparse_attn(q, k, v, self.p, idx, o)
        return idx, o

    def dense_attn(self, q, k, v, out=None):
        import torch
        o = torch.empty_like(q) if out is None else out
        hip_dense_attn(q, k, v, self.p, o)
        return o

    def check(self) -> None:
        check_status(self.p)
