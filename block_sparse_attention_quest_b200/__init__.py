"""Python binding of libresa.so (ReSA decode hot path on B200, sm_100a).

Argument marshalling only: every function below checks tensor shapes, passes
device pointers, sizes and the current CUDA stream to the C ABI declared in
include/resa.h, and raises on a non-zero status. All arithmetic happens in the
library's CUDA kernels. PyTorch provides device memory and streams.

The library must be built (``python block_sparse_attention_quest_b200/build.py``
or ``__graft_entry__.build()``); importing this module fails loudly when
libresa.so is missing. There is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libresa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libresa.so not found at {LIB_PATH}; build it with "
        "`python block_sparse_attention_quest_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

RESA_OK = 0
RESA_ERR_INVALID_ARG = -1
RESA_ERR_UNSUPPORTED = -2
RESA_ERR_CAPACITY = -3
RESA_ERR_WORKSPACE = -4
RESA_ERR_CUDA = -5
RESA_ERR_TIMEOUT = -6
RESA_ERR_BAD_INDEX = -7
RESA_F32 = 0
RESA_BF16 = 1
BLOCK = 16

EXPORTED = ("resa_num_selected", "resa_workspace_bytes", "resa_build_desc",
            "resa_decode_sparse", "resa_select_blocks", "resa_attend_blocks",
            "resa_decode_dense", "resa_rectify",
            "resa_workspace_status", "resa_status_string", "resa_decode_sparse_noalloc",
            "resa_build_desc_varlen", "resa_decode_sparse_varlen", "resa_decode_dense_varlen",
            "resa_rectify_varlen", "resa_prefill", "resa_wait_check", "resa_noalloc_status")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("max_len", ctypes.c_int64)]


_P = ctypes.c_void_p
_lib.resa_num_selected.restype = ctypes.c_int32
_lib.resa_num_selected.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_int32]
_lib.resa_workspace_bytes.restype = ctypes.c_size_t
_lib.resa_workspace_bytes.argtypes = [ctypes.POINTER(Dims), ctypes.c_int64, ctypes.c_int32]
_lib.resa_build_desc.restype = ctypes.c_int
_lib.resa_build_desc.argtypes = [ctypes.POINTER(Dims), _P, ctypes.c_int64, _P, _P]
_lib.resa_decode_sparse.restype = ctypes.c_int
_lib.resa_decode_sparse.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, ctypes.c_int64,
                                    ctypes.c_double, ctypes.c_int32, ctypes.c_float, _P, _P, _P,
                                    _P, ctypes.c_size_t, _P]
_lib.resa_select_blocks.restype = ctypes.c_int
_lib.resa_select_blocks.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, ctypes.c_int64,
                                    ctypes.c_double, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]
_lib.resa_attend_blocks.restype = ctypes.c_int
_lib.resa_attend_blocks.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, ctypes.c_int64, _P,
                                    ctypes.c_int32, ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]
_lib.resa_decode_dense.restype = ctypes.c_int
_lib.resa_decode_dense.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, ctypes.c_int64,
                                   ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]
_lib.resa_rectify.restype = ctypes.c_int
_lib.resa_rectify.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, ctypes.c_int64,
                              ctypes.c_int32, ctypes.c_float, _P, _P, ctypes.c_size_t, _P]
_lib.resa_decode_sparse_noalloc.restype = ctypes.c_int
_lib.resa_decode_sparse_noalloc.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P,
                                            ctypes.c_int64, ctypes.c_double, ctypes.c_int32,
                                            ctypes.c_float, _P, _P, _P, _P]
_lib.resa_build_desc_varlen.restype = ctypes.c_int
_lib.resa_build_desc_varlen.argtypes = [ctypes.POINTER(Dims), _P, _P, ctypes.c_int64, _P, _P]
_lib.resa_decode_sparse_varlen.restype = ctypes.c_int
_lib.resa_decode_sparse_varlen.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P,
                                           ctypes.c_int64, ctypes.c_double, ctypes.c_int32,
                                           ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.resa_decode_dense_varlen.restype = ctypes.c_int
_lib.resa_decode_dense_varlen.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_int64, ctypes.c_float, _P, _P, _P,
                                          ctypes.c_size_t, _P]
_lib.resa_rectify_varlen.restype = ctypes.c_int
_lib.resa_rectify_varlen.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P,
                                     ctypes.c_int64, ctypes.c_int32, ctypes.c_float, _P, _P,
                                     ctypes.c_size_t, _P]
_lib.resa_prefill.restype = ctypes.c_int
_lib.resa_prefill.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, ctypes.c_int64, ctypes.c_float,
                              _P, _P, ctypes.c_size_t, _P]
_lib.resa_wait_check.restype = ctypes.c_int
_lib.resa_wait_check.argtypes = [_P, ctypes.c_int32, ctypes.c_uint32, _P, _P]
_lib.resa_workspace_status.restype = ctypes.c_int
_lib.resa_workspace_status.argtypes = [_P, _P]
_lib.resa_noalloc_status.restype = ctypes.c_int
_lib.resa_noalloc_status.argtypes = [_P]
_lib.resa_status_string.restype = ctypes.c_char_p
_lib.resa_status_string.argtypes = [ctypes.c_int]


class ResaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def status_string(status: int) -> str:
    return _lib.resa_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != RESA_OK:
        raise ResaError(status, what)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return RESA_F32
    if dt == torch.bfloat16:
        return RESA_BF16
    raise ValueError(f"unsupported dtype {dt}")


def dims_for(k_cache: torch.Tensor, n_q_heads: int) -> Dims:
    """Dims of a cache [B, H_kv, max_len, d] serving n_q_heads query heads."""
    B, H, L, d = k_cache.shape
    return Dims(B, int(n_q_heads), H, d, BLOCK, _dtype_code(k_cache.dtype), L)


def num_selected(length: int, r: float, n_min: int) -> int:
    n = _lib.resa_num_selected(int(length), BLOCK, float(r), int(n_min))
    if n < 0:
        raise ResaError(n, "resa_num_selected")
    return n


def workspace_bytes(dims: Dims, length: int, f: int = 0) -> int:
    n = _lib.resa_workspace_bytes(ctypes.byref(dims), int(length), int(f))
    if n == 0:
        raise ResaError(RESA_ERR_INVALID_ARG, "resa_workspace_bytes")
    return n


def alloc_workspace(dims: Dims, length: int, f: int = 0, device=None) -> torch.Tensor:
    """Zero-filled workspace (uint8) of the size the library asks for."""
    n = workspace_bytes(dims, length, f)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def build_desc(k_cache: torch.Tensor, length: int, desc: torch.Tensor, n_q_heads: int,
               stream=None) -> None:
    dims = dims_for(k_cache, n_q_heads)
    _check(_lib.resa_build_desc(ctypes.byref(dims), _ptr(k_cache), int(length), _ptr(desc),
                                _stream(stream)), "resa_build_desc")


def decode_sparse(q, k_new, v_new, k_cache, v_cache, desc, length: int, r: float, n_min: int,
                  softmax_scale: float, out, workspace, lse=None, sel=None, stream=None) -> None:
    dims = dims_for(k_cache, q.shape[1])
    _check(_lib.resa_decode_sparse(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), int(length), float(r), int(n_min), float(softmax_scale), _ptr(out), _ptr(lse),
        _ptr(sel), _ptr(workspace), workspace.numel(), _stream(stream)), "resa_decode_sparse")


def select_blocks(q, k_new, v_new, k_cache, v_cache, desc, length: int, r: float, n_min: int,
                  sel, workspace, stream=None) -> None:
    dims = dims_for(k_cache, q.shape[1])
    _check(_lib.resa_select_blocks(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), int(length), float(r), int(n_min), _ptr(sel), _ptr(workspace),
        workspace.numel(), _stream(stream)), "resa_select_blocks")


def attend_blocks(q, k_cache, v_cache, length: int, sel, softmax_scale: float, out, workspace,
                  lse=None, stream=None) -> None:
    dims = dims_for(k_cache, q.shape[1])
    _check(_lib.resa_attend_blocks(
        ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), int(length), _ptr(sel),
        int(sel.shape[-1]), float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream(stream)), "resa_attend_blocks")


def decode_dense(q, k_new, v_new, k_cache, v_cache, desc, length: int, softmax_scale: float, out,
                 workspace, lse=None, stream=None) -> None:
    dims = dims_for(k_cache, q.shape[1])
    _check(_lib.resa_decode_dense(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), int(length), float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream(stream)), "resa_decode_dense")


def rectify(q_f, k_f, v_f, k_cache, v_cache, desc, length: int, f: int, softmax_scale: float,
            out_f, workspace, stream=None) -> None:
    dims = dims_for(k_cache, q_f.shape[2])
    _check(_lib.resa_rectify(
        ctypes.byref(dims), _ptr(q_f), _ptr(k_f), _ptr(v_f), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), int(length), int(f), float(softmax_scale), _ptr(out_f), _ptr(workspace),
        workspace.numel(), _stream(stream)), "resa_rectify")


def decode_sparse_noalloc(q, k_new, v_new, k_cache, v_cache, desc, length: int, r: float,
                          n_min: int, softmax_scale: float, out, lse=None, sel=None,
                          stream=None) -> None:
    """resa_decode_sparse with the library's own fixed scratch (no workspace)."""
    dims = dims_for(k_cache, q.shape[1])
    _check(_lib.resa_decode_sparse_noalloc(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), int(length), float(r), int(n_min), float(softmax_scale), _ptr(out), _ptr(lse),
        _ptr(sel), _stream(stream)), "resa_decode_sparse_noalloc")


def noalloc_status(stream=None) -> int:
    """Synchronise and read (and clear) the device error flag of the fixed
    scratch that decode_sparse_noalloc uses on the current device."""
    return _lib.resa_noalloc_status(_stream(stream))


def workspace_status(workspace, stream=None) -> int:
    """Synchronise and read (and clear) the device error flag of a workspace."""
    return _lib.resa_workspace_status(_ptr(workspace), _stream(stream))


# ---- variable-length batches: `lens` is an int32 CUDA tensor [batch] of row
# lengths, `len_bound` an upper bound on its entries (sizes grids, workspace and
# the stride of `sel`)


def _lens(lens):
    if lens is None or lens.dtype != torch.int32 or not lens.is_cuda or lens.dim() != 1:
        raise ValueError("lens must be a 1-D int32 CUDA tensor")
    return _ptr(lens)


def build_desc_varlen(k_cache, lens, len_bound: int, desc, n_q_heads: int, stream=None) -> None:
    dims = dims_for(k_cache, n_q_heads)
    _check(_lib.resa_build_desc_varlen(ctypes.byref(dims), _ptr(k_cache), _lens(lens),
                                       int(len_bound), _ptr(desc), _stream(stream)),
           "resa_build_desc_varlen")


def decode_sparse_varlen(q, k_new, v_new, k_cache, v_cache, desc, lens, len_bound: int, r: float,
                         n_min: int, softmax_scale: float, out, workspace, lse=None, sel=None,
                         stream=None) -> None:
    dims = dims_for(k_cache, q.shape[1])
    _check(_lib.resa_decode_sparse_varlen(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), _lens(lens), int(len_bound), float(r), int(n_min), float(softmax_scale),
        _ptr(out), _ptr(lse), _ptr(sel), _ptr(workspace), workspace.numel(), _stream(stream)),
        "resa_decode_sparse_varlen")


def decode_dense_varlen(q, k_new, v_new, k_cache, v_cache, desc, lens, len_bound: int,
                        softmax_scale: float, out, workspace, lse=None, stream=None) -> None:
    dims = dims_for(k_cache, q.shape[1])
    _check(_lib.resa_decode_dense_varlen(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), _lens(lens), int(len_bound), float(softmax_scale), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel(), _stream(stream)), "resa_decode_dense_varlen")


def rectify_varlen(q_f, k_f, v_f, k_cache, v_cache, desc, lens, len_bound: int, f: int,
                   softmax_scale: float, out_f, workspace, windows=None, stream=None) -> None:
    """windows: optional int32 CUDA tensor [batch] of per-row windows in [0, f]
    (0 = row not rectified); None = every row uses f."""
    dims = dims_for(k_cache, q_f.shape[2])
    _check(_lib.resa_rectify_varlen(
        ctypes.byref(dims), _ptr(q_f), _ptr(k_f), _ptr(v_f), _ptr(k_cache), _ptr(v_cache),
        _ptr(desc), _lens(lens), None if windows is None else _lens(windows), int(len_bound), int(f), float(softmax_scale), _ptr(out_f),
        _ptr(workspace), workspace.numel(), _stream(stream)), "resa_rectify_varlen")


def prefill(q, k_cache, v_cache, desc, length: int, softmax_scale: float, out, workspace,
            stream=None) -> None:
    """Causal attention of every prompt position (q, out: [B, len, Hq, d]) and
    the descriptors of the prompt's keys, in one pass."""
    dims = dims_for(k_cache, q.shape[2])
    _check(_lib.resa_prefill(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(desc),
                             int(length), float(softmax_scale), _ptr(out), _ptr(workspace),
                             workspace.numel(), _stream(stream)), "resa_prefill")


def wait_check(flag, target: int, limit_us: int, workspace, stream=None) -> None:
    """Enqueue the device's bounded wait on `flag` (int32 CUDA tensor) reaching
    `target`; a wait that runs out shows as RESA_ERR_TIMEOUT in
    workspace_status()."""
    _check(_lib.resa_wait_check(_ptr(flag), int(target), int(limit_us), _ptr(workspace),
                                _stream(stream)), "resa_wait_check")
