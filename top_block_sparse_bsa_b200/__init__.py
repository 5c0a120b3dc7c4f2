"""Python binding of libbsa, the B200 (sm_100a) library for query-aware
top-k block-sparse causal attention.

Argument marshalling only: every function here forwards torch tensors'
device pointers and the current CUDA stream to the C entry point of the same
name declared in ``include/bsa.h``; all computation runs in the library's
CUDA kernels.  There is no CPU fallback: importing the package fails if
``libbsa.so`` has not been built (``python top_block_sparse_bsa_b200/_build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "BsaError", "BsaShape", "lib", "LIB_PATH",
    "BSA_F32", "BSA_BF16",
    "BSA_SCORE_PREFILL", "BSA_SCORE_DECODE", "BSA_SCORE_GIST", "BSA_SCORE_DECODE_HEADS",
    "BSA_TOPK_CAUSAL_BLOCK", "BSA_TOPK_LAST_BLOCK", "BSA_TOPK_PLAIN",
    "BSA_OP_DECODE", "BSA_OP_GIST_DECODE", "BSA_OP_DECODE_HEADS",
    "make_shape", "bsa_score_blocks", "bsa_topk_select", "bsa_sparse_attn_prefill",
    "bsa_gated_attn_fwd", "bsa_sparse_attn_decode", "bsa_gist_expand_decode",
    "bsa_workspace_bytes", "bsa_status_string", "bsa_device_status", "bsa_version",
    "bsa_sparse_attn_decode_noalloc", "bsa_decode_split_override", "bsa_selftest_wait_expiry",
    "bsa_prefill_kernel_override", "bsa_decode_select", "bsa_topk_select_pattern",
    "bsa_topk_select_joint_heads", "bsa_sparse_attn_decode_heads", "bsa_sparse_attn_decode_paged",
    "bsa_paged_append", "bsa_hssa_decode", "bsa_workspace_bytes_hssa", "bsa_gated_attn_bwd",
    "bsa_workspace_bytes_bwd", "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbsa.so")

BSA_OK, BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED, BSA_ERR_CUDA, BSA_ERR_TIMEOUT, BSA_ERR_DEVICE = range(6)
BSA_F32, BSA_BF16 = 0, 1
BSA_SCORE_PREFILL, BSA_SCORE_DECODE, BSA_SCORE_GIST, BSA_SCORE_DECODE_HEADS = 0, 1, 2, 3
BSA_TOPK_CAUSAL_BLOCK, BSA_TOPK_LAST_BLOCK, BSA_TOPK_PLAIN = 0, 1, 2
BSA_OP_DECODE, BSA_OP_GIST_DECODE, BSA_OP_DECODE_HEADS = 0, 1, 2

# Every symbol the C header declares.
EXPORTED_SYMBOLS = (
    "bsa_score_blocks", "bsa_topk_select", "bsa_sparse_attn_prefill", "bsa_gated_attn_fwd",
    "bsa_sparse_attn_decode", "bsa_gist_expand_decode", "bsa_workspace_bytes",
    "bsa_status_string", "bsa_device_status", "bsa_version", "bsa_sparse_attn_decode_noalloc",
    "bsa_decode_split_override", "bsa_selftest_wait_expiry", "bsa_prefill_kernel_override",
    "bsa_decode_select", "bsa_topk_select_pattern", "bsa_topk_select_joint_heads", "bsa_sparse_attn_decode_heads",
    "bsa_sparse_attn_decode_paged", "bsa_paged_append", "bsa_hssa_decode", "bsa_workspace_bytes_hssa",
    "bsa_gated_attn_bwd", "bsa_workspace_bytes_bwd",
)


class BsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {_status_name(code)}")


class BsaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("Nq", ctypes.c_int),
                ("Nk", ctypes.c_int), ("d", ctypes.c_int), ("block", ctypes.c_int), ("dtype", ctypes.c_int)]

    def __repr__(self):
        return (f"BsaShape(B={self.B}, Hq={self.Hq}, Hkv={self.Hkv}, Nq={self.Nq}, Nk={self.Nk}, "
                f"d={self.d}, block={self.block}, dtype={self.dtype})")


_p = ctypes.c_void_p
_i = ctypes.c_int
_SIGS = {
    "bsa_score_blocks": (_i, [ctypes.POINTER(BsaShape), _i, _p, _p, _p, _p, _p, _p, _p]),
    "bsa_topk_select": (_i, [_p, _i, _i, _i, _i, _p, _i, _p, _p]),
    "bsa_decode_select": (_i, [ctypes.POINTER(BsaShape), _p, _p, _i, _p, _p, _p, _i, _p, _p]),
    "bsa_topk_select_pattern": (_i, [_p, _i, _i, _i, _i, _i, _p, _i, _p, _p]),
    "bsa_sparse_attn_decode_paged": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _i, _p, _i, _p, _i, ctypes.c_float,
                                          _p, ctypes.c_size_t, _p, _p, _p]),
    "bsa_paged_append": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _i, _i, _p, _p, _p, _p]),
    "bsa_hssa_decode": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _p, _p, _p, _i, _i, _p, _p, ctypes.c_float,
                             _p, ctypes.c_size_t, _p, _p, _p]),
    "bsa_workspace_bytes_hssa": (ctypes.c_size_t, [ctypes.POINTER(BsaShape), _i, _i]),
    "bsa_gated_attn_bwd": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _p, _p, _i, _p, ctypes.c_float, _p, _p,
                                _p, _p, _p, ctypes.c_size_t, _p]),
    "bsa_workspace_bytes_bwd": (ctypes.c_size_t, [ctypes.POINTER(BsaShape), _i]),
    "bsa_topk_select_joint_heads": (_i, [_p, _i, _i, _i, _i, _p, _i, _p, _p]),
    "bsa_sparse_attn_decode_heads": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _i, ctypes.c_float, _p,
                                          ctypes.c_size_t, _p, _p, _p]),
    "bsa_sparse_attn_prefill": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _i, ctypes.c_float, _p, _p, _p]),
    "bsa_gated_attn_fwd": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _i, _p, ctypes.c_float, _p, _p, _p]),
    "bsa_sparse_attn_decode": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _i, ctypes.c_float, _p,
                                    ctypes.c_size_t, _p, _p, _p]),
    "bsa_gist_expand_decode": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _p, _i, _p, _p, ctypes.c_float,
                                    _p, ctypes.c_size_t, _p, _p, _p]),
    "bsa_sparse_attn_decode_noalloc": (_i, [ctypes.POINTER(BsaShape), _p, _p, _p, _p, _i, ctypes.c_float, _p,
                                            _p, _p]),
    "bsa_workspace_bytes": (ctypes.c_size_t, [_i, ctypes.POINTER(BsaShape), _i]),
    "bsa_status_string": (ctypes.c_char_p, [_i]),
    "bsa_device_status": (_i, [ctypes.POINTER(ctypes.c_uint), _i]),
    "bsa_version": (_i, []),
    "bsa_decode_split_override": (_i, [_i]),
    "bsa_prefill_kernel_override": (_i, [_i]),
    "bsa_selftest_wait_expiry": (_i, [ctypes.c_longlong, _p]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbsa.so is not built at {LIB_PATH}; build it with "
                          "`python top_block_sparse_bsa_b200/_build.py`")
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def _status_name(code: int) -> str:
    return lib.bsa_status_string(code).decode()


def _check(fn: str, code: int) -> None:
    if code != BSA_OK:
        raise BsaError(fn, code)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libbsa takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libbsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BSA_BF16
    if t.dtype == torch.float32:
        return BSA_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def make_shape(B, Hq, Hkv, Nq, Nk, d, block, dtype) -> BsaShape:
    if isinstance(dtype, torch.dtype):
        dtype = BSA_BF16 if dtype == torch.bfloat16 else BSA_F32
    return BsaShape(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d), int(block), int(dtype))


def bsa_version() -> int:
    return int(lib.bsa_version())


def bsa_status_string(code: int) -> str:
    return _status_name(code)


def bsa_device_status(reset: bool = False):
    """(status code, flag bits) of the current device; synchronises it."""
    flags = ctypes.c_uint(0)
    code = lib.bsa_device_status(ctypes.byref(flags), 1 if reset else 0)
    return int(code), int(flags.value)


def bsa_decode_split_override(num_splits: int) -> int:
    """Fix the decode split-K range count (> 0) or restore the default (<= 0); returns the previous setting."""
    return int(lib.bsa_decode_split_override(int(num_splits)))


def bsa_prefill_kernel_override(kernel: int) -> int:
    """Force a bf16 prefill kernel (1 paired tiles, 2 one tile per SM, 3 SM pair) or 0 for the
    shape's default; returns the previous setting."""
    return int(lib.bsa_prefill_kernel_override(int(kernel)))


def bsa_selftest_wait_expiry(budget_cycles: int, stream=None) -> None:
    """Enqueue the bounded-wait expiry self-test kernel (sets BSA_DEV_TIMEOUT in the status word)."""
    _check("bsa_selftest_wait_expiry", lib.bsa_selftest_wait_expiry(int(budget_cycles), _stream(stream)))


def bsa_workspace_bytes(op: int, shape: BsaShape, budget: int) -> int:
    return int(lib.bsa_workspace_bytes(op, ctypes.byref(shape), int(budget)))


def bsa_score_blocks(shape: BsaShape, mode: int, q, k=None, pooled_k_in=None, pooled_q_out=None,
                     pooled_k_out=None, scores=None, stream=None) -> None:
    _check("bsa_score_blocks", lib.bsa_score_blocks(
        ctypes.byref(shape), int(mode), _ptr(q), _ptr(k), _ptr(pooled_k_in), _ptr(pooled_q_out),
        _ptr(pooled_k_out), _ptr(scores), _stream(stream)))


def bsa_topk_select(scores, rows: int, ncols: int, mode: int, kb: int, idx_out, idx_stride: int,
                    count_out=None, stream=None) -> None:
    _check("bsa_topk_select", lib.bsa_topk_select(
        _ptr(scores), int(rows), int(ncols), int(mode), int(kb), _ptr(idx_out), int(idx_stride),
        _ptr(count_out), _stream(stream)))


def bsa_topk_select_pattern(scores, rows: int, ncols: int, sink: int, local: int, kb: int, idx_out,
                            idx_stride: int, count_out=None, stream=None) -> None:
    _check("bsa_topk_select_pattern", lib.bsa_topk_select_pattern(
        _ptr(scores), int(rows), int(ncols), int(sink), int(local), int(kb), _ptr(idx_out), int(idx_stride),
        _ptr(count_out), _stream(stream)))


def bsa_topk_select_joint_heads(scores, rows: int, heads: int, ncols: int, kb_total: int, idx_out,
                                idx_stride: int, count_out=None, stream=None) -> None:
    _check("bsa_topk_select_joint_heads", lib.bsa_topk_select_joint_heads(
        _ptr(scores), int(rows), int(heads), int(ncols), int(kb_total), _ptr(idx_out), int(idx_stride),
        _ptr(count_out), _stream(stream)))


def bsa_sparse_attn_decode_heads(shape: BsaShape, q, k_cache, v_cache, idx, idx_stride: int, softmax_scale: float,
                                 workspace, o, lse=None, stream=None) -> None:
    _check("bsa_sparse_attn_decode_heads", lib.bsa_sparse_attn_decode_heads(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx), int(idx_stride),
        ctypes.c_float(softmax_scale), _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        _ptr(o), _ptr(lse), _stream(stream)))


def bsa_sparse_attn_decode_paged(shape: BsaShape, q, k_pool, v_pool, block_table, idx, idx_stride: int,
                                 softmax_scale: float, workspace, o, lse=None, stream=None) -> None:
    """Decode over a paged cache: pools [P,Hkv,64,d], block_table [B, table_stride]."""
    _check("bsa_sparse_attn_decode_paged", lib.bsa_sparse_attn_decode_paged(
        ctypes.byref(shape), _ptr(q), _ptr(k_pool), _ptr(v_pool), int(k_pool.shape[0]), _ptr(block_table),
        int(block_table.shape[-1]), _ptr(idx), int(idx_stride), ctypes.c_float(softmax_scale), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _ptr(o), _ptr(lse), _stream(stream)))


def bsa_paged_append(shape: BsaShape, k_new, v_new, seq_lens, block_table, k_pool, v_pool, pooled_k=None,
                     stream=None) -> None:
    """Write k_new/v_new [B,Hkv,T,d] at positions seq_lens[b]+t of the paged cache; pool completed blocks."""
    _check("bsa_paged_append", lib.bsa_paged_append(
        ctypes.byref(shape), _ptr(k_new), _ptr(v_new), _ptr(seq_lens), _ptr(block_table), int(block_table.shape[-1]),
        int(k_pool.shape[0]), _ptr(k_pool), _ptr(v_pool), _ptr(pooled_k), _stream(stream)))


def bsa_hssa_decode(shape: BsaShape, q, k_cache, v_cache, gist_k, gist_v, meta_k, meta_v, km: int, topk: int,
                    meta_out=None, idx_out=None, softmax_scale: float = 0.0, workspace=None, o=None, lse=None,
                    stream=None) -> None:
    _check("bsa_hssa_decode", lib.bsa_hssa_decode(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(gist_k), _ptr(gist_v), _ptr(meta_k),
        _ptr(meta_v), int(km), int(topk), _ptr(meta_out), _ptr(idx_out), ctypes.c_float(softmax_scale),
        _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size() if workspace is not None else 0),
        _ptr(o), _ptr(lse), _stream(stream)))


def bsa_workspace_bytes_hssa(shape: BsaShape, km: int, topk: int) -> int:
    return int(lib.bsa_workspace_bytes_hssa(ctypes.byref(shape), int(km), int(topk)))


def bsa_gated_attn_bwd(shape: BsaShape, q, k, v, lse, d_o, idx, idx_stride: int, sel_scores, softmax_scale: float,
                       dq, dk, dv, dsel=None, workspace=None, stream=None) -> None:
    """Backward of the sparse (sel_scores None) or gated prefill attention: fp32 dq, dk, dv (and dsel)."""
    _check("bsa_gated_attn_bwd", lib.bsa_gated_attn_bwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(lse), _ptr(d_o), _ptr(idx), int(idx_stride),
        _ptr(sel_scores), ctypes.c_float(softmax_scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dsel), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size() if workspace is not None else 0),
        _stream(stream)))


def bsa_workspace_bytes_bwd(shape: BsaShape, idx_stride: int) -> int:
    return int(lib.bsa_workspace_bytes_bwd(ctypes.byref(shape), int(idx_stride)))


def bsa_decode_select(shape: BsaShape, q, pooled_k, kb: int, scores, idx_out, idx_stride: int,
                      pooled_q_out=None, count_out=None, stream=None) -> None:
    _check("bsa_decode_select", lib.bsa_decode_select(
        ctypes.byref(shape), _ptr(q), _ptr(pooled_k), int(kb), _ptr(pooled_q_out), _ptr(scores), _ptr(idx_out),
        int(idx_stride), _ptr(count_out), _stream(stream)))


def bsa_sparse_attn_prefill(shape: BsaShape, q, k, v, idx, idx_stride: int, softmax_scale: float, o,
                            lse=None, stream=None) -> None:
    _check("bsa_sparse_attn_prefill", lib.bsa_sparse_attn_prefill(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), int(idx_stride),
        ctypes.c_float(softmax_scale), _ptr(o), _ptr(lse), _stream(stream)))


def bsa_gated_attn_fwd(shape: BsaShape, q, k, v, idx, idx_stride: int, sel_scores, softmax_scale: float, o,
                       lse=None, stream=None) -> None:
    _check("bsa_gated_attn_fwd", lib.bsa_gated_attn_fwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), int(idx_stride), _ptr(sel_scores),
        ctypes.c_float(softmax_scale), _ptr(o), _ptr(lse), _stream(stream)))


def bsa_sparse_attn_decode(shape: BsaShape, q, k_cache, v_cache, idx, idx_stride: int, softmax_scale: float,
                           workspace, o, lse=None, stream=None) -> None:
    _check("bsa_sparse_attn_decode", lib.bsa_sparse_attn_decode(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx), int(idx_stride),
        ctypes.c_float(softmax_scale), _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        _ptr(o), _ptr(lse), _stream(stream)))


def bsa_gist_expand_decode(shape: BsaShape, q, k_cache, v_cache, gist_k, gist_v, topk: int, idx_in=None,
                           idx_out=None, softmax_scale: float = 0.0, workspace=None, o=None, lse=None,
                           stream=None) -> None:
    _check("bsa_gist_expand_decode", lib.bsa_gist_expand_decode(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(gist_k), _ptr(gist_v), int(topk),
        _ptr(idx_in), _ptr(idx_out), ctypes.c_float(softmax_scale), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size() if workspace is not None else 0),
        _ptr(o), _ptr(lse), _stream(stream)))


def bsa_sparse_attn_decode_noalloc(shape: BsaShape, q, k_cache, v_cache, idx, idx_stride: int,
                                   softmax_scale: float, o, lse=None, stream=None) -> None:
    """Decode without a caller-provided workspace (scratch lives in the library)."""
    _check("bsa_sparse_attn_decode_noalloc", lib.bsa_sparse_attn_decode_noalloc(
        ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx), int(idx_stride),
        ctypes.c_float(softmax_scale), _ptr(o), _ptr(lse), _stream(stream)))
