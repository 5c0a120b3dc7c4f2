"""Algorithmic work of the hot path, for throughput and roofline figures.

Counts are taken from the kept-block index lists (host copies), not from
what a kernel happens to execute:

* pairs: causal-valid (query, key) pairs inside kept blocks; a query block's
  own block contributes bs*(bs+1)/2 pairs, every earlier kept block bs*bs
  ("稀疏注意力" tutorial §1 counts n x n pairs for dense attention);
* FLOPs: 4*d per pair (QK^T and PV, a multiply and an add each);
* bytes: the kept K and V tiles, each counted once per unit that reads it
  (per (batch, KV group, query block) in prefill, per (batch, KV group) in
  decode; in gist decode the union of the group's expanded chunks plus every
  gist key/value);
* sparsity = 1 - computed / full ("稀疏注意力的Trade-offs" review §1.2).
"""
from __future__ import annotations

import numpy as np


def dense_pairs(n: int, causal: bool = False) -> int:
    """Query-key pairs of dense attention over n tokens (n*n, or n(n+1)/2 causal)."""
    return n * (n + 1) // 2 if causal else n * n


def sparsity(computed: float, full: float) -> float:
    return 1.0 - computed / full


def _kept(idx: np.ndarray) -> np.ndarray:
    """Boolean mask of the valid (non-negative, before the first -1) entries."""
    idx = np.asarray(idx)
    valid = idx >= 0
    return np.logical_and.accumulate(valid, axis=-1)


def prefill_pairs(idx: np.ndarray, bs: int, G: int) -> int:
    """idx [B,Hkv,nb,stride] -> causal pairs over all G heads of every group."""
    idx = np.asarray(idx)
    kept = _kept(idx)
    nb = idx.shape[2]
    i = np.arange(nb).reshape(1, 1, nb, 1)
    diag = (idx == i) & kept
    full = (idx < i) & kept
    per_head = full.sum() * bs * bs + diag.sum() * (bs * (bs + 1) // 2)
    return int(per_head) * G


def prefill_kv_bytes(idx: np.ndarray, bs: int, d: int, elem: int) -> int:
    """Kept K+V bytes, each kept tile counted once per (b, group, query block)."""
    return int(_kept(idx).sum()) * bs * d * elem * 2


def decode_kv_bytes(idx: np.ndarray, bs: int, d: int, elem: int) -> int:
    """idx [B,Hkv,stride] -> kept K+V bytes, once per (b, group)."""
    return int(_kept(idx).sum()) * bs * d * elem * 2


def decode_pairs(idx: np.ndarray, bs: int, G: int) -> int:
    return int(_kept(idx).sum()) * bs * G


def gist_union_chunks(idx: np.ndarray, G: int) -> int:
    """idx [B,Hq,k] -> sum over (b, group) of the number of distinct expanded chunks."""
    idx = np.asarray(idx)
    B, Hq, _ = idx.shape
    total = 0
    for b in range(B):
        for g in range(Hq // G):
            sel = idx[b, g * G:(g + 1) * G].ravel()
            total += len(np.unique(sel[sel >= 0]))
    return total


def gist_kv_bytes(idx: np.ndarray, G: int, chunk: int, nc: int, d: int, elem: int) -> int:
    """Bytes the gist attention must read: the union of expanded chunks' K/V
    plus every gist key/value, per (b, group)."""
    idx = np.asarray(idx)
    groups = idx.shape[0] * (idx.shape[1] // G)
    return (gist_union_chunks(idx, G) * chunk + groups * nc) * d * elem * 2


def gist_pairs(idx: np.ndarray, chunk: int, nc: int) -> int:
    """Keys attended per head: expanded tokens plus unexpanded gists, summed over heads."""
    idx = np.asarray(idx)
    k = (idx >= 0).sum(axis=-1)
    return int((k * chunk + (nc - k)).sum())


def heads_kv_bytes(idx: np.ndarray, G: int, bs: int, d: int, elem: int) -> int:
    """idx [B,Hq,stride] per-head kept blocks -> bytes of the union of each
    (b, group)'s blocks (each gathered once for the group's heads), K and V."""
    idx = np.asarray(idx)
    B, Hq, _ = idx.shape
    total = 0
    for b in range(B):
        for g in range(Hq // G):
            sel = idx[b, g * G:(g + 1) * G].ravel()
            total += len(np.unique(sel[sel >= 0]))
    return total * bs * d * elem * 2


def hssa_kv_bytes(chunks: np.ndarray, groups: np.ndarray, G: int, chunk: int, d: int, elem: int) -> int:
    """Two-level gist decode: per (b, group) the union of the heads' expanded
    chunks (chunk tokens each), the gists of the union of their kept groups
    (64 per group) and the 64-row meta-gist tile, K and V."""
    chunks, groups = np.asarray(chunks), np.asarray(groups)
    B, Hq, _ = chunks.shape
    rows = 0
    for b in range(B):
        for g in range(Hq // G):
            c = chunks[b, g * G:(g + 1) * G].ravel()
            m = groups[b, g * G:(g + 1) * G].ravel()
            rows += len(np.unique(c[c >= 0])) * chunk + len(np.unique(m[m >= 0])) * 64 + 64
    return rows * d * elem * 2
