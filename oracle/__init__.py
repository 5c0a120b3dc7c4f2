"""CPU oracle for query-aware top-k block-sparse causal attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``top_block_sparse_bsa_b200``) never imports it and shares no code with it.

The arithmetic lives in ``bsa_oracle.c`` (plain C, fp64 attention, fixed-order
fp32 selector); this module compiles it with gcc, loads it with ctypes and
converts arrays.  Every function documents the passage it follows in the C
source.

Inputs may be torch tensors or numpy arrays; bf16 tensors are upcast to fp32
exactly before the call.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")

# -ffp-contract=off: no fused multiply-add, so every fp32 product and sum of
# the selector is rounded separately, in source order.
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-std=c11", "-Wall"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle's C source into a shared library (gcc)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def _declare(L):
    sig = {
        "oracle_pool_keys": [_p, _i64, _i64, _i64, _i64, _i64, _p],
        "oracle_pool_queries_grouped": [_p, _i64, _i64, _i64, _i64, _i64, _i64, _p],
        "oracle_group_mean_query": [_p, _i64, _i64, _i64, _i64, _p],
        "oracle_scores_prefill": [_p, _p, _i64, _i64, _i64, _i64, _p],
        "oracle_scores_decode": [_p, _p, _i64, _i64, _i64, _i64, _p],
        "oracle_scores_gist": [_p, _p, _i64, _i64, _i64, _i64, _i64, _p],
        "oracle_topk": [_p, _i64, _i64, ctypes.c_int, _i64, _p, _i64, _p],
        "oracle_prefill_mask": [_i64, _i64, _p, _i64, _p],
        "oracle_attend_prefill_rows": [_p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p, _i64,
                                       _p, ctypes.c_double, _p, _i64, _p, _p],
        "oracle_attend_decode_rows": [_p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p, _i64,
                                      ctypes.c_double, _p, _i64, _p, _p],
        "oracle_attend_gist_rows": [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p,
                                    _i64, ctypes.c_double, _p, _i64, _p, _p],
        "oracle_topk_pattern": [_p, _i64, _i64, _i64, _i64, _i64, _p, _i64, _p],
        "oracle_topk_joint_heads": [_p, _i64, _i64, _i64, _i64, _p, _i64, _p],
        "oracle_attend_decode_heads_rows": [_p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p, _i64,
                                            ctypes.c_double, _p, _i64, _p, _p],
        "oracle_paged_gather": [_p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p],
        "oracle_hssa_select": [_p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _p, _i64, _p, _i64],
        "oracle_attend_hssa_rows": [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _p, _i64,
                                    _p, _i64, ctypes.c_double, _p, _i64, _p, _p],
        "oracle_attend_prefill_bwd": [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64, _p, _i64, _p,
                                      ctypes.c_double, _p, _p, _p, _p],
        "oracle_max_threads": [],
        "oracle_set_threads": [ctypes.c_int],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int if name == "oracle_max_threads" else None


# ----------------------------------------------------------------------------
# array helpers
# ----------------------------------------------------------------------------

def _f32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float32).contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.int32).contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())


# ----------------------------------------------------------------------------
# 1-2. pooling and selector scores (fixed-order fp32)
# ----------------------------------------------------------------------------

def pool_keys(k, bs: int) -> np.ndarray:
    """k [B,H,N,d] -> kbar [B,H,N/bs,d]; block means, tokens ascending."""
    k = _f32(k)
    B, H, N, d = k.shape
    out = np.empty((B, H, N // bs, d), np.float32)
    lib().oracle_pool_keys(_ptr(k), B, H, N, d, bs, _ptr(out))
    return out


def pool_queries_grouped(q, Hkv: int, bs: int) -> np.ndarray:
    """q [B,Hq,N,d] -> qbar [B,Hkv,N/bs,d]; mean over the group's heads and the block's tokens."""
    q = _f32(q)
    B, Hq, N, d = q.shape
    out = np.empty((B, Hkv, N // bs, d), np.float32)
    lib().oracle_pool_queries_grouped(_ptr(q), B, Hq, Hkv, N, d, bs, _ptr(out))
    return out


def group_mean_query(q, Hkv: int) -> np.ndarray:
    """q [B,Hq,d] -> qbar [B,Hkv,d]; mean over the group's heads."""
    q = _f32(q)
    B, Hq, d = q.shape
    out = np.empty((B, Hkv, d), np.float32)
    lib().oracle_group_mean_query(_ptr(q), B, Hq, Hkv, d, _ptr(out))
    return out


def scores_prefill(qbar, kbar) -> np.ndarray:
    qbar, kbar = _f32(qbar), _f32(kbar)
    B, Hkv, nb, d = qbar.shape
    out = np.empty((B, Hkv, nb, nb), np.float32)
    lib().oracle_scores_prefill(_ptr(qbar), _ptr(kbar), B, Hkv, nb, d, _ptr(out))
    return out


def scores_decode(qbar, kbar) -> np.ndarray:
    qbar, kbar = _f32(qbar), _f32(kbar)
    B, Hkv, nb, d = kbar.shape
    out = np.empty((B, Hkv, nb), np.float32)
    lib().oracle_scores_decode(_ptr(qbar), _ptr(kbar), B, Hkv, nb, d, _ptr(out))
    return out


def scores_gist(q, gk) -> np.ndarray:
    q, gk = _f32(q), _f32(gk)
    B, Hq, d = q.shape
    _, Hkv, nc, _ = gk.shape
    out = np.empty((B, Hq, nc), np.float32)
    lib().oracle_scores_gist(_ptr(q), _ptr(gk), B, Hq, Hkv, nc, d, _ptr(out))
    return out


# ----------------------------------------------------------------------------
# 3. selection
# ----------------------------------------------------------------------------

TOPK_CAUSAL_BLOCK = 0
TOPK_LAST_BLOCK = 1
TOPK_PLAIN = 2


def topk(scores, mode: int, kb: int, idx_stride: Optional[int] = None
         ) -> Tuple[np.ndarray, np.ndarray]:
    """scores [..., ncols] -> (idx [..., idx_stride] ascending, -1 padded; count [...])."""
    s = _f32(scores)
    ncols = s.shape[-1]
    lead = s.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    forced = 0 if mode == TOPK_PLAIN else 1
    if idx_stride is None:
        idx_stride = kb + forced
    idx = np.empty(lead + (idx_stride,), np.int32)
    cnt = np.empty(lead, np.int32)
    lib().oracle_topk(_ptr(s), rows, ncols, mode, kb, _ptr(idx), idx_stride, _ptr(cnt))
    return idx, cnt


# ----------------------------------------------------------------------------
# 4. mask, 5-6. attention
# ----------------------------------------------------------------------------

def prefill_mask(N: int, bs: int, idx) -> np.ndarray:
    """idx [nb, idx_stride] of one (batch, group) -> bool mask [N, N] (True = M is 0)."""
    idx = _i32(idx)
    m = np.empty((N, N), np.uint8)
    lib().oracle_prefill_mask(N, bs, _ptr(idx), idx.shape[-1], _ptr(m))
    return m.astype(bool)


def _rows_arg(rows, total: int) -> np.ndarray:
    if rows is None:
        return np.arange(total, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def attend_prefill(q, k, v, bs: int, idx, gate_scores=None, scale: Optional[float] = None,
                   rows=None) -> Tuple[np.ndarray, np.ndarray]:
    """Sparse causal prefill attention (fp64) for the listed query rows.

    q [B,Hq,N,d], k/v [B,Hkv,N,d], idx [B,Hkv,nb,stride]; gate_scores
    [B,Hkv,nb,nb] turns on the SAS log-gate.  rows: flat ids (b*Hq+h)*N+t
    (default: all).  Returns out [nrows,d] fp64, lse [nrows] fp64.
    """
    q, k, v, idx = _f32(q), _f32(k), _f32(v), _i32(idx)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    r = _rows_arg(rows, B * Hq * N)
    out = np.empty((len(r), d), np.float64)
    lse = np.empty((len(r),), np.float64)
    gs = _f32(gate_scores) if gate_scores is not None else None
    lib().oracle_attend_prefill_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, N, d, bs,
                                     _ptr(idx), idx.shape[-1],
                                     _ptr(gs) if gs is not None else None, float(scale),
                                     _ptr(r), len(r), _ptr(out), _ptr(lse))
    return out, lse


def attend_decode(q, k, v, bs: int, idx, scale: Optional[float] = None, rows=None
                  ) -> Tuple[np.ndarray, np.ndarray]:
    """Sparse decode attention (fp64).  q [B,Hq,d], k/v [B,Hkv,Nk,d], idx [B,Hkv,stride]."""
    q, k, v, idx = _f32(q), _f32(k), _f32(v), _i32(idx)
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    r = _rows_arg(rows, B * Hq)
    out = np.empty((len(r), d), np.float64)
    lse = np.empty((len(r),), np.float64)
    lib().oracle_attend_decode_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nk, d, bs,
                                    _ptr(idx), idx.shape[-1], float(scale),
                                    _ptr(r), len(r), _ptr(out), _ptr(lse))
    return out, lse


def attend_gist(q, k, v, gk, gv, chunk: int, idx, scale: Optional[float] = None, rows=None
                ) -> Tuple[np.ndarray, np.ndarray]:
    """Gist selective-expansion decode attention (fp64).  idx [B,Hq,stride]."""
    q, k, v, gk, gv, idx = _f32(q), _f32(k), _f32(v), _f32(gk), _f32(gv), _i32(idx)
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    r = _rows_arg(rows, B * Hq)
    out = np.empty((len(r), d), np.float64)
    lse = np.empty((len(r),), np.float64)
    lib().oracle_attend_gist_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(gk), _ptr(gv),
                                  B, Hq, Hkv, Nk, d, chunk, _ptr(idx), idx.shape[-1],
                                  float(scale), _ptr(r), len(r), _ptr(out), _ptr(lse))
    return out, lse


# ----------------------------------------------------------------------------
# whole steps (pool -> score -> select -> attend), in the pages' order
# ----------------------------------------------------------------------------

def prefill_select(q, k, Hkv: int, bs: int, kb: int):
    """Steps 1-3 of prefill: returns (qbar, kbar, scores, idx, count)."""
    qbar = pool_queries_grouped(q, Hkv, bs)
    kbar = pool_keys(k, bs)
    s = scores_prefill(qbar, kbar)
    idx, cnt = topk(s, TOPK_CAUSAL_BLOCK, kb)
    return qbar, kbar, s, idx, cnt


def decode_select(q, kbar, Hkv: int, kb: int):
    """Steps 2-3 of decode from the pooled-key summary: (qbar, scores, idx, count)."""
    qbar = group_mean_query(q, Hkv)
    s = scores_decode(qbar, kbar)
    idx, cnt = topk(s, TOPK_LAST_BLOCK, kb)
    return qbar, s, idx, cnt


def gist_select(q, gk, kb: int):
    """Gist scoring and per-head expansion choice: (scores, idx, count)."""
    s = scores_gist(q, gk)
    idx, cnt = topk(s, TOPK_PLAIN, kb)
    return s, idx, cnt


# ----------------------------------------------------------------------------
# 7-9. fixed pattern + dynamic blocks, shared head budget, paged cache
# ----------------------------------------------------------------------------

def topk_pattern(scores, sink: int, local: int, kb: int, idx_stride: Optional[int] = None
                 ) -> Tuple[np.ndarray, np.ndarray]:
    """scores [..., nb, nb] (row = query block i) -> kept blocks: the first
    `sink` blocks, the `local` most recent (current included) and the kb best
    of the others (MInference block-sparse, Sparse Frontier review §2.2.3)."""
    s = _f32(scores)
    ncols = s.shape[-1]
    lead = s.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    if idx_stride is None:
        idx_stride = sink + local + kb
    idx = np.empty(lead + (idx_stride,), np.int32)
    cnt = np.empty(lead, np.int32)
    lib().oracle_topk_pattern(_ptr(s), rows, ncols, sink, local, kb, _ptr(idx), idx_stride, _ptr(cnt))
    return idx, cnt


def topk_joint_heads(scores, kb_total: int, idx_stride: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """scores [B, Hkv, G, nb] per-head decode scores -> per-head kept blocks
    [B, Hkv, G, idx_stride] under one budget of kb_total (head, block) pairs per
    group, the last block kept by every head (Ada-KV, review §2.3.2)."""
    s = _f32(scores)
    B, Hkv, G, nb = s.shape
    if idx_stride is None:
        idx_stride = min(kb_total, nb - 1) + 1
    idx = np.empty((B, Hkv, G, idx_stride), np.int32)
    cnt = np.empty((B, Hkv, G), np.int32)
    lib().oracle_topk_joint_heads(_ptr(s), B * Hkv, G, nb, kb_total, _ptr(idx), idx_stride, _ptr(cnt))
    return idx, cnt


def attend_decode_heads(q, k, v, bs: int, idx, scale: Optional[float] = None, rows=None
                        ) -> Tuple[np.ndarray, np.ndarray]:
    """Decode attention (fp64) with each query head's own kept blocks.
    q [B,Hq,d], k/v [B,Hkv,Nk,d], idx [B,Hq,stride]."""
    q, k, v, idx = _f32(q), _f32(k), _f32(v), _i32(idx)
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    r = _rows_arg(rows, B * Hq)
    out = np.empty((len(r), d), np.float64)
    lse = np.empty((len(r),), np.float64)
    lib().oracle_attend_decode_heads_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nk, d, bs,
                                          _ptr(idx), idx.shape[-1], float(scale),
                                          _ptr(r), len(r), _ptr(out), _ptr(lse))
    return out, lse


def paged_gather(pool, table, nb: int) -> np.ndarray:
    """pool [P, Hkv, bs, d], table [B, max_blocks] -> the logical cache
    [B, Hkv, nb*bs, d] of the first nb blocks (PagedAttention, tutorial §7)."""
    pool, table = _f32(pool), _i32(table)
    P, Hkv, bs, d = pool.shape
    B, max_blocks = table.shape
    out = np.empty((B, Hkv, nb * bs, d), np.float32)
    lib().oracle_paged_gather(_ptr(pool), _ptr(table), B, Hkv, nb, bs, d, max_blocks, _ptr(out))
    return out


# ----------------------------------------------------------------------------
# 10. two-level gist routing (H-SSA)
# ----------------------------------------------------------------------------

def hssa_select(q, gk, mk, M: int, km: int, k: int):
    """Meta-gist then gist selection per query head (SSA page, H-SSA).
    q [B,Hq,d], gk [B,Hkv,nc,d], mk [B,Hkv,nc/M,d] -> (meta_idx [B,Hq,km],
    chunk_idx [B,Hq,k]), ascending, -1 padded."""
    q, gk, mk = _f32(q), _f32(gk), _f32(mk)
    B, Hq, d = q.shape
    Hkv, nc = gk.shape[1], gk.shape[2]
    meta = np.empty((B, Hq, max(km, 1)), np.int32)
    chunks = np.empty((B, Hq, max(k, 1)), np.int32)
    lib().oracle_hssa_select(_ptr(q), _ptr(gk), _ptr(mk), B, Hq, Hkv, nc, M, d, km, k,
                             _ptr(meta), meta.shape[-1], _ptr(chunks), chunks.shape[-1])
    return meta, chunks


def attend_hssa(q, k, v, gk, gv, mk, mv, chunk: int, M: int, meta_idx, chunk_idx,
                scale: Optional[float] = None, rows=None) -> Tuple[np.ndarray, np.ndarray]:
    """H-SSA decode attention (fp64): expanded chunks' tokens, gists of the
    other chunks of kept groups, meta-gists of groups not kept."""
    q, k, v, gk, gv, mk, mv = (_f32(x) for x in (q, k, v, gk, gv, mk, mv))
    meta_idx, chunk_idx = _i32(meta_idx), _i32(chunk_idx)
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    r = _rows_arg(rows, B * Hq)
    out = np.empty((len(r), d), np.float64)
    lse = np.empty((len(r),), np.float64)
    lib().oracle_attend_hssa_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(gk), _ptr(gv), _ptr(mk), _ptr(mv),
                                  B, Hq, Hkv, Nk, d, chunk, M, _ptr(meta_idx), meta_idx.shape[-1],
                                  _ptr(chunk_idx), chunk_idx.shape[-1], float(scale), _ptr(r), len(r),
                                  _ptr(out), _ptr(lse))
    return out, lse


# ----------------------------------------------------------------------------
# 11. backward of the (gated) sparse prefill attention
# ----------------------------------------------------------------------------

def attend_prefill_bwd(q, k, v, dO, bs: int, idx, gate_scores=None, scale: Optional[float] = None):
    """Gradients (fp64) of sum(dO * O) for O = attend_prefill(q, k, v, bs, idx,
    gate_scores): (dq [B,Hq,N,d], dk, dv [B,Hkv,N,d], ds [B,Hkv,nb,nb] or None)."""
    q, k, v, dO, idx = _f32(q), _f32(k), _f32(v), _f32(dO), _i32(idx)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    nb = N // bs
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.empty((B, Hq, N, d), np.float64)
    dk = np.empty((B, Hkv, N, d), np.float64)
    dv = np.empty((B, Hkv, N, d), np.float64)
    gs = _f32(gate_scores) if gate_scores is not None else None
    ds = np.empty((B, Hkv, nb, nb), np.float64) if gs is not None else None
    lib().oracle_attend_prefill_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), B, Hq, Hkv, N, d, bs, _ptr(idx),
                                    idx.shape[-1], _ptr(gs) if gs is not None else None, float(scale),
                                    _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds) if ds is not None else None)
    return dq, dk, dv, ds
