"""Whole steps of the hot path, composed from the C entry points.

A step is the pages' sequence -- score the blocks, keep the top-k (with the
current / last block), attend over the kept blocks -- issued as consecutive
library calls on one stream.  Buffers are allocated once (torch is only the
device-memory provider here) and reused, so a step launches kernels and
nothing else.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import torch

from . import (bsa_gated_attn_bwd, bsa_workspace_bytes_bwd, BSA_OP_DECODE, BSA_OP_DECODE_HEADS, BSA_OP_GIST_DECODE, BSA_SCORE_DECODE,
               BSA_SCORE_DECODE_HEADS, BSA_SCORE_PREFILL, BSA_TOPK_CAUSAL_BLOCK, bsa_decode_select,
               bsa_gated_attn_fwd, bsa_gist_expand_decode, bsa_score_blocks, bsa_sparse_attn_decode,
               bsa_hssa_decode, bsa_paged_append, bsa_sparse_attn_decode_heads, bsa_workspace_bytes_hssa, bsa_sparse_attn_decode_paged, bsa_sparse_attn_prefill,
               bsa_topk_select, bsa_topk_select_joint_heads, bsa_topk_select_pattern, bsa_workspace_bytes,
               make_shape)


def _dev(t: torch.Tensor):
    return t.device


@dataclass
class PrefillStep:
    """pool+score -> top-k -> sparse (or gated) attention for q [B,Hq,N,d], k/v [B,Hkv,N,d].

    pattern=(sink, local) keeps, besides the kb best blocks, the first `sink`
    blocks and the `local` most recent ones (MInference block-sparse); the
    default keeps the current block only."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    block: int
    kb: int
    gated: bool = False
    softmax_scale: Optional[float] = None
    pattern: Optional[Tuple[int, int]] = None
    bufs: Dict[str, torch.Tensor] = field(default_factory=dict)

    def __post_init__(self):
        B, Hq, N, d = self.q.shape
        Hkv = self.k.shape[1]
        nb = N // self.block
        self.shape = make_shape(B, Hq, Hkv, N, N, d, self.block, self.q.dtype)
        self.nb = nb
        self.idx_stride = self.kb + 1 if self.pattern is None else self.kb + self.pattern[0] + self.pattern[1]
        if self.softmax_scale is None:
            self.softmax_scale = 1.0 / math.sqrt(d)
        dev = _dev(self.q)
        f32 = torch.float32
        b = self.bufs
        b.setdefault("qbar", torch.empty((B, Hkv, nb, d), dtype=f32, device=dev))
        b.setdefault("kbar", torch.empty((B, Hkv, nb, d), dtype=f32, device=dev))
        b.setdefault("scores", torch.empty((B, Hkv, nb, nb), dtype=f32, device=dev))
        b.setdefault("idx", torch.empty((B, Hkv, nb, self.idx_stride), dtype=torch.int32, device=dev))
        b.setdefault("count", torch.empty((B, Hkv, nb), dtype=torch.int32, device=dev))
        b.setdefault("o", torch.empty_like(self.q))
        b.setdefault("lse", torch.empty((B, Hq, N), dtype=f32, device=dev))

    def select(self, stream=None):
        b = self.bufs
        bsa_score_blocks(self.shape, BSA_SCORE_PREFILL, self.q, self.k, None, b["qbar"], b["kbar"],
                         b["scores"], stream=stream)
        rows = self.shape.B * self.shape.Hkv * self.nb
        if self.pattern is None:
            bsa_topk_select(b["scores"], rows, self.nb, BSA_TOPK_CAUSAL_BLOCK, self.kb, b["idx"], self.idx_stride,
                            b["count"], stream=stream)
        else:
            sink, local = self.pattern
            bsa_topk_select_pattern(b["scores"], rows, self.nb, sink, local, self.kb, b["idx"], self.idx_stride,
                                    b["count"], stream=stream)

    def attend(self, idx: Optional[torch.Tensor] = None, stream=None, with_lse: bool = True):
        b = self.bufs
        idx = b["idx"] if idx is None else idx
        lse = b["lse"] if with_lse else None
        if self.gated:
            bsa_gated_attn_fwd(self.shape, self.q, self.k, self.v, idx, idx.shape[-1], b["scores"],
                               self.softmax_scale, b["o"], lse, stream=stream)
        else:
            bsa_sparse_attn_prefill(self.shape, self.q, self.k, self.v, idx, idx.shape[-1], self.softmax_scale,
                                    b["o"], lse, stream=stream)

    def run(self, stream=None, with_lse: bool = True):
        self.select(stream)
        self.attend(stream=stream, with_lse=with_lse)
        return self.bufs

    def backward(self, d_o: torch.Tensor, idx: Optional[torch.Tensor] = None, stream=None):
        """Gradients of sum(d_o * O) for the last attend() (run with its LSE):
        fp32 dq, dk, dv and, gated, dsel (the selector scores' gradient)."""
        b = self.bufs
        idx = b["idx"] if idx is None else idx
        dev = _dev(self.q)
        f32 = torch.float32
        b.setdefault("dq", torch.empty(self.q.shape, dtype=f32, device=dev))
        b.setdefault("dk", torch.empty(self.k.shape, dtype=f32, device=dev))
        b.setdefault("dv", torch.empty(self.v.shape, dtype=f32, device=dev))
        if self.gated:
            b.setdefault("dsel", torch.empty(b["scores"].shape, dtype=f32, device=dev))
        ws = bsa_workspace_bytes_bwd(self.shape, idx.shape[-1])
        if "bwd_workspace" not in b or b["bwd_workspace"].numel() < ws:
            b["bwd_workspace"] = torch.empty((max(ws, 256),), dtype=torch.uint8, device=dev)
        bsa_gated_attn_bwd(self.shape, self.q, self.k, self.v, b["lse"], d_o, idx, idx.shape[-1],
                           b["scores"] if self.gated else None, self.softmax_scale, b["dq"], b["dk"], b["dv"],
                           b["dsel"] if self.gated else None, b["bwd_workspace"], stream=stream)
        return b


@dataclass
class DecodeStep:
    """score (against the resident pooled-key summary) -> top-k -> split-K sparse decode.

    q [B,Hq,d]; k_cache/v_cache [B,Hkv,Nk,d]; kbar [B,Hkv,nb,d] fp32 is the
    block-mean summary kept next to the cache (built once by ``pool_cache``).
    """
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block: int
    kb: int
    softmax_scale: Optional[float] = None
    bufs: Dict[str, torch.Tensor] = field(default_factory=dict)

    def __post_init__(self):
        B, Hq, d = self.q.shape
        Hkv, Nk = self.k_cache.shape[1], self.k_cache.shape[2]
        nb = Nk // self.block
        self.nb = nb
        self.shape = make_shape(B, Hq, Hkv, 1, Nk, d, self.block, self.q.dtype)
        self.idx_stride = self.kb + 1
        if self.softmax_scale is None:
            self.softmax_scale = 1.0 / math.sqrt(d)
        dev = _dev(self.q)
        f32 = torch.float32
        b = self.bufs
        b.setdefault("kbar", torch.empty((B, Hkv, nb, d), dtype=f32, device=dev))
        b.setdefault("qbar", torch.empty((B, Hkv, d), dtype=f32, device=dev))
        b.setdefault("scores", torch.empty((B, Hkv, nb), dtype=f32, device=dev))
        b.setdefault("idx", torch.empty((B, Hkv, self.idx_stride), dtype=torch.int32, device=dev))
        b.setdefault("count", torch.empty((B, Hkv), dtype=torch.int32, device=dev))
        ws = bsa_workspace_bytes(BSA_OP_DECODE, self.shape, self.idx_stride)
        b.setdefault("workspace", torch.empty((max(ws, 256),), dtype=torch.uint8, device=dev))
        b.setdefault("o", torch.empty_like(self.q))
        b.setdefault("lse", torch.empty((B, Hq), dtype=f32, device=dev))

    def pool_cache(self, stream=None):
        """Build the pooled-key summary from the cache (off the per-step path)."""
        b = self.bufs
        bsa_score_blocks(self.shape, BSA_SCORE_DECODE, self.q, self.k_cache, None, b["qbar"], b["kbar"],
                         b["scores"], stream=stream)

    def select(self, stream=None):
        b = self.bufs
        bsa_decode_select(self.shape, self.q, b["kbar"], self.kb, b["scores"], b["idx"], self.idx_stride,
                          pooled_q_out=b["qbar"], count_out=b["count"], stream=stream)

    def attend(self, idx: Optional[torch.Tensor] = None, stream=None, with_lse: bool = True):
        b = self.bufs
        idx = b["idx"] if idx is None else idx
        bsa_sparse_attn_decode(self.shape, self.q, self.k_cache, self.v_cache, idx, idx.shape[-1],
                               self.softmax_scale, b["workspace"], b["o"], b["lse"] if with_lse else None,
                               stream=stream)

    def run(self, stream=None, with_lse: bool = True):
        self.select(stream)
        self.attend(stream=stream, with_lse=with_lse)
        return self.bufs


@dataclass
class GistStep:
    """SSA decode: gist scores -> per-head top-k chunks -> mixed attention (one C call)."""
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    gist_k: torch.Tensor
    gist_v: torch.Tensor
    chunk: int
    topk: int
    softmax_scale: Optional[float] = None
    bufs: Dict[str, torch.Tensor] = field(default_factory=dict)

    def __post_init__(self):
        B, Hq, d = self.q.shape
        Hkv, Nk = self.k_cache.shape[1], self.k_cache.shape[2]
        self.shape = make_shape(B, Hq, Hkv, 1, Nk, d, self.chunk, self.q.dtype)
        if self.softmax_scale is None:
            self.softmax_scale = 1.0 / math.sqrt(d)
        dev = _dev(self.q)
        b = self.bufs
        ws = bsa_workspace_bytes(BSA_OP_GIST_DECODE, self.shape, self.topk)
        b.setdefault("workspace", torch.empty((max(ws, 256),), dtype=torch.uint8, device=dev))
        b.setdefault("idx", torch.empty((B, Hq, max(self.topk, 1)), dtype=torch.int32, device=dev))
        b.setdefault("o", torch.empty_like(self.q))
        b.setdefault("lse", torch.empty((B, Hq), dtype=torch.float32, device=dev))

    def run(self, idx_in: Optional[torch.Tensor] = None, stream=None, with_lse: bool = True):
        b = self.bufs
        bsa_gist_expand_decode(self.shape, self.q, self.k_cache, self.v_cache, self.gist_k, self.gist_v,
                               self.topk, idx_in, b["idx"] if self.topk > 0 else None, self.softmax_scale,
                               b["workspace"], b["o"], b["lse"] if with_lse else None, stream=stream)
        return b


@dataclass
class HeadBudgetDecodeStep:
    """Decode with one budget shared by the query heads of each KV group
    (Ada-KV): per-head scores against the pooled-key summary -> the best
    kb_total (head, block) pairs of the group, the last block kept by every
    head -> attention with each head's own kept blocks."""
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block: int
    kb_total: int
    softmax_scale: Optional[float] = None
    bufs: Dict[str, torch.Tensor] = field(default_factory=dict)

    def __post_init__(self):
        B, Hq, d = self.q.shape
        Hkv, Nk = self.k_cache.shape[1], self.k_cache.shape[2]
        nb = Nk // self.block
        self.nb = nb
        self.G = Hq // Hkv
        self.shape = make_shape(B, Hq, Hkv, 1, Nk, d, self.block, self.q.dtype)
        self.idx_stride = min(self.kb_total, nb - 1) + 1
        if self.softmax_scale is None:
            self.softmax_scale = 1.0 / math.sqrt(d)
        dev = _dev(self.q)
        f32 = torch.float32
        b = self.bufs
        b.setdefault("kbar", torch.empty((B, Hkv, nb, d), dtype=f32, device=dev))
        b.setdefault("qbar", torch.empty((B, Hkv, d), dtype=f32, device=dev))
        b.setdefault("scores", torch.empty((B, Hq, nb), dtype=f32, device=dev))
        b.setdefault("idx", torch.empty((B, Hq, self.idx_stride), dtype=torch.int32, device=dev))
        b.setdefault("count", torch.empty((B, Hq), dtype=torch.int32, device=dev))
        ws = bsa_workspace_bytes(BSA_OP_DECODE_HEADS, self.shape, self.idx_stride)
        b.setdefault("workspace", torch.empty((max(ws, 256),), dtype=torch.uint8, device=dev))
        b.setdefault("o", torch.empty_like(self.q))
        b.setdefault("lse", torch.empty((B, Hq), dtype=f32, device=dev))

    def pool_cache(self, stream=None):
        b = self.bufs
        group_scores = torch.empty((self.shape.B, self.shape.Hkv, self.nb), dtype=torch.float32, device=self.q.device)
        bsa_score_blocks(self.shape, BSA_SCORE_DECODE, self.q, self.k_cache, None, b["qbar"], b["kbar"],
                         group_scores, stream=stream)

    def select(self, stream=None):
        b = self.bufs
        bsa_score_blocks(self.shape, BSA_SCORE_DECODE_HEADS, self.q, None, b["kbar"], None, None, b["scores"],
                         stream=stream)
        bsa_topk_select_joint_heads(b["scores"], self.shape.B * self.shape.Hkv, self.G, self.nb, self.kb_total,
                                    b["idx"], self.idx_stride, b["count"], stream=stream)

    def attend(self, idx: Optional[torch.Tensor] = None, stream=None, with_lse: bool = True):
        b = self.bufs
        idx = b["idx"] if idx is None else idx
        bsa_sparse_attn_decode_heads(self.shape, self.q, self.k_cache, self.v_cache, idx, idx.shape[-1],
                                     self.softmax_scale, b["workspace"], b["o"], b["lse"] if with_lse else None,
                                     stream=stream)

    def run(self, stream=None, with_lse: bool = True):
        self.select(stream)
        self.attend(stream=stream, with_lse=with_lse)
        return self.bufs


@dataclass
class PagedDecodeStep:
    """Decode over a paged KV cache (PagedAttention): pools [P,Hkv,64,d] of
    physical blocks and a block table [B, nb] mapping each sequence's logical
    blocks to them.  The pooled-key summary [B,Hkv,nb,d] is kept by
    ``append`` (each block is pooled when it completes); ``select`` scores
    the query against it and keeps the top-kb logical blocks with the last;
    ``attend`` gathers the kept blocks through the table."""
    q: torch.Tensor
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    block_table: torch.Tensor
    block: int
    kb: int
    softmax_scale: Optional[float] = None
    bufs: Dict[str, torch.Tensor] = field(default_factory=dict)

    def __post_init__(self):
        B, Hq, d = self.q.shape
        Hkv = self.k_pool.shape[1]
        nb = self.block_table.shape[1]
        self.nb = nb
        self.shape = make_shape(B, Hq, Hkv, 1, nb * self.block, d, self.block, self.q.dtype)
        self.idx_stride = self.kb + 1
        if self.softmax_scale is None:
            self.softmax_scale = 1.0 / math.sqrt(d)
        dev = _dev(self.q)
        f32 = torch.float32
        b = self.bufs
        b.setdefault("kbar", torch.zeros((B, Hkv, nb, d), dtype=f32, device=dev))
        b.setdefault("qbar", torch.empty((B, Hkv, d), dtype=f32, device=dev))
        b.setdefault("scores", torch.empty((B, Hkv, nb), dtype=f32, device=dev))
        b.setdefault("idx", torch.empty((B, Hkv, self.idx_stride), dtype=torch.int32, device=dev))
        b.setdefault("count", torch.empty((B, Hkv), dtype=torch.int32, device=dev))
        ws = bsa_workspace_bytes(BSA_OP_DECODE, self.shape, self.idx_stride)
        b.setdefault("workspace", torch.empty((max(ws, 256),), dtype=torch.uint8, device=dev))
        b.setdefault("o", torch.empty_like(self.q))
        b.setdefault("lse", torch.empty((B, Hq), dtype=f32, device=dev))

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, seq_lens: torch.Tensor, stream=None):
        """Write k_new/v_new [B,Hkv,T,d] after seq_lens[b] tokens; completed blocks are pooled."""
        B, Hkv, T, d = k_new.shape
        shape = make_shape(B, Hkv, Hkv, T, self.nb * self.block, d, self.block, k_new.dtype)
        bsa_paged_append(shape, k_new, v_new, seq_lens, self.block_table, self.k_pool, self.v_pool,
                         self.bufs["kbar"], stream=stream)

    def select(self, stream=None):
        b = self.bufs
        bsa_decode_select(self.shape, self.q, b["kbar"], self.kb, b["scores"], b["idx"], self.idx_stride,
                          pooled_q_out=b["qbar"], count_out=b["count"], stream=stream)

    def attend(self, idx: Optional[torch.Tensor] = None, stream=None, with_lse: bool = True):
        b = self.bufs
        idx = b["idx"] if idx is None else idx
        bsa_sparse_attn_decode_paged(self.shape, self.q, self.k_pool, self.v_pool, self.block_table, idx,
                                     idx.shape[-1], self.softmax_scale, b["workspace"], b["o"],
                                     b["lse"] if with_lse else None, stream=stream)

    def run(self, stream=None, with_lse: bool = True):
        self.select(stream)
        self.attend(stream=stream, with_lse=with_lse)
        return self.bufs


@dataclass
class HssaStep:
    """Two-level gist routing decode (H-SSA): meta-gist scores -> km groups
    per head -> gist scores inside them -> topk chunks per head -> attention
    over expanded tokens, gists of kept groups, meta-gists of the rest (one C
    call).  Groups are 64 chunks; meta_k/meta_v [B,Hkv,nc/64,d]."""
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    gist_k: torch.Tensor
    gist_v: torch.Tensor
    meta_k: torch.Tensor
    meta_v: torch.Tensor
    chunk: int
    km: int
    topk: int
    softmax_scale: Optional[float] = None
    bufs: Dict[str, torch.Tensor] = field(default_factory=dict)

    def __post_init__(self):
        B, Hq, d = self.q.shape
        Hkv, Nk = self.k_cache.shape[1], self.k_cache.shape[2]
        self.shape = make_shape(B, Hq, Hkv, 1, Nk, d, self.chunk, self.q.dtype)
        if self.softmax_scale is None:
            self.softmax_scale = 1.0 / math.sqrt(d)
        dev = _dev(self.q)
        b = self.bufs
        ws = bsa_workspace_bytes_hssa(self.shape, self.km, self.topk)
        b.setdefault("workspace", torch.empty((max(ws, 256),), dtype=torch.uint8, device=dev))
        b.setdefault("meta_idx", torch.empty((B, Hq, self.km), dtype=torch.int32, device=dev))
        b.setdefault("idx", torch.empty((B, Hq, max(self.topk, 1)), dtype=torch.int32, device=dev))
        b.setdefault("o", torch.empty_like(self.q))
        b.setdefault("lse", torch.empty((B, Hq), dtype=torch.float32, device=dev))

    def run(self, stream=None, with_lse: bool = True):
        b = self.bufs
        bsa_hssa_decode(self.shape, self.q, self.k_cache, self.v_cache, self.gist_k, self.gist_v, self.meta_k,
                        self.meta_v, self.km, self.topk, b["meta_idx"], b["idx"] if self.topk > 0 else None,
                        self.softmax_scale, b["workspace"], b["o"], b["lse"] if with_lse else None, stream=stream)
        return b
