"""Pins for the CPU oracle: every check compares the oracle with something
other than itself -- the pages' worked examples (tests/golden/), closed forms,
invariants, a library routine the special case reduces to, or brute force.

Runs on CPU only (no GPU marker).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden_sets(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, vals = line.split(":")
            rows[int(key)] = [int(x) for x in vals.split()]
    return rows


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa64(q, k, v, mask=None, causal=False):
    """Library attention in fp64 on CPU (the dense formula's own routine)."""
    q = torch.as_tensor(q, dtype=torch.float64)
    k = torch.as_tensor(k, dtype=torch.float64)
    v = torch.as_tensor(v, dtype=torch.float64)
    if mask is not None:
        mask = torch.as_tensor(mask)
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, is_causal=causal).numpy()


# ----------------------------------------------------------------------------
# pooling: closed forms and the fixed summation order
# ----------------------------------------------------------------------------

def test_pool_keys_constant_input_is_exact():
    k = np.full((2, 3, 128, 16), 0.375, np.float32)
    kbar = oracle.pool_keys(k, 64)
    assert kbar.shape == (2, 3, 2, 16)
    assert np.all(kbar == np.float32(0.375))


def test_pool_keys_integer_input_exact_mean():
    r = _rng(1)
    k = r.integers(-8, 9, size=(2, 2, 256, 8)).astype(np.float32)
    kbar = oracle.pool_keys(k, 64)
    exact = k.reshape(2, 2, 4, 64, 8).astype(np.int64).sum(axis=3) / 64.0
    assert np.array_equal(kbar.astype(np.float64), exact)


def test_pool_keys_sequential_fp32_order():
    # np.add.accumulate is a strictly left-to-right fp32 running sum: the
    # oracle's fixed order must reproduce its last element bit for bit.
    r = _rng(2)
    k = r.standard_normal((1, 2, 192, 8)).astype(np.float32)
    kbar = oracle.pool_keys(k, 64)
    blocks = k.reshape(1, 2, 3, 64, 8)
    seq = np.add.accumulate(blocks, axis=3, dtype=np.float32)[:, :, :, -1, :]
    assert np.array_equal(kbar, seq / np.float32(64))


def test_pool_queries_grouped_heads_then_tokens():
    r = _rng(3)
    B, Hq, Hkv, N, d, bs = 1, 6, 2, 128, 8, 32
    q = r.standard_normal((B, Hq, N, d)).astype(np.float32)
    qbar = oracle.pool_queries_grouped(q, Hkv, bs)
    G = Hq // Hkv
    # group g, block i: the G*bs rows in (head asc, token asc) order
    seqs = q.reshape(B, Hkv, G, N // bs, bs, d).transpose(0, 1, 3, 2, 4, 5)
    seqs = seqs.reshape(B, Hkv, N // bs, G * bs, d)
    ref = np.add.accumulate(seqs, axis=3, dtype=np.float32)[:, :, :, -1, :] / np.float32(G * bs)
    assert np.array_equal(qbar, ref)


def test_group_mean_query():
    r = _rng(4)
    q = r.integers(-4, 5, size=(3, 8, 16)).astype(np.float32)
    qbar = oracle.group_mean_query(q, 2)
    exact = q.reshape(3, 2, 4, 16).astype(np.int64).sum(axis=2) / 4.0
    assert np.array_equal(qbar.astype(np.float64), exact)


# ----------------------------------------------------------------------------
# selector scores
# ----------------------------------------------------------------------------

def test_scores_prefill_integer_exact_and_causal():
    r = _rng(5)
    B, Hkv, nb, d = 1, 2, 6, 16
    qbar = r.integers(-3, 4, size=(B, Hkv, nb, d)).astype(np.float32)
    kbar = r.integers(-3, 4, size=(B, Hkv, nb, d)).astype(np.float32)
    s = oracle.scores_prefill(qbar, kbar)
    scale = np.float32(1.0 / math.sqrt(d))
    dots = np.einsum("bgic,bgjc->bgij", qbar.astype(np.int64), kbar.astype(np.int64))
    for i in range(nb):
        for j in range(nb):
            if j <= i:
                assert np.array_equal(s[:, :, i, j], (dots[:, :, i, j].astype(np.float32) * scale))
            else:
                assert np.all(np.isneginf(s[:, :, i, j]))


def test_scores_sequential_fp32_products():
    r = _rng(6)
    B, Hkv, nb, d = 1, 1, 5, 32
    qbar = r.standard_normal((B, Hkv, nb, d)).astype(np.float32)
    kbar = r.standard_normal((B, Hkv, nb, d)).astype(np.float32)
    s = oracle.scores_prefill(qbar, kbar)
    scale = np.float32(1.0 / math.sqrt(d))
    for i in range(nb):
        for j in range(i + 1):
            prods = (qbar[0, 0, i] * kbar[0, 0, j]).astype(np.float32)
            acc = np.add.accumulate(prods, dtype=np.float32)[-1]
            assert s[0, 0, i, j] == np.float32(acc * scale)


def test_group_score_is_mean_of_head_scores():
    # Linearity: pooled-over-heads query . pooled key = mean of the per-head
    # pooled scores, up to fp32 rounding.
    r = _rng(7)
    B, Hq, Hkv, N, d, bs = 1, 4, 1, 256, 64, 64
    q = r.standard_normal((B, Hq, N, d)).astype(np.float32)
    k = r.standard_normal((B, Hkv, N, d)).astype(np.float32)
    s_group = oracle.scores_prefill(oracle.pool_queries_grouped(q, Hkv, bs), oracle.pool_keys(k, bs))
    per_head = []
    for h in range(Hq):
        qh = q[:, h:h + 1]
        per_head.append(oracle.scores_prefill(oracle.pool_queries_grouped(qh, 1, bs),
                                              oracle.pool_keys(k, bs)))
    mean = np.mean(np.stack(per_head), axis=0)
    tri = np.tril(np.ones((N // bs, N // bs), bool))
    assert np.allclose(s_group[0, 0][tri], mean[0, 0][tri], atol=1e-5)


def test_scores_decode_and_gist_shapes_and_values():
    r = _rng(8)
    B, Hq, Hkv, nb, d = 2, 4, 2, 7, 16
    q = r.integers(-2, 3, size=(B, Hq, d)).astype(np.float32)
    kbar = r.integers(-2, 3, size=(B, Hkv, nb, d)).astype(np.float32)
    scale = np.float32(1.0 / math.sqrt(d))
    qbar = oracle.group_mean_query(q, Hkv)
    s = oracle.scores_decode(qbar, kbar)
    ref = np.einsum("bgc,bgjc->bgj", qbar.astype(np.float64), kbar.astype(np.float64))
    assert np.array_equal(s, ref.astype(np.float32) * scale)
    sg = oracle.scores_gist(q, kbar)
    G = Hq // Hkv
    refg = np.einsum("bhc,bhjc->bhj", q.astype(np.int64), np.repeat(kbar, G, axis=1).astype(np.int64))
    assert np.array_equal(sg, refg.astype(np.float32) * scale)


# ----------------------------------------------------------------------------
# top-k selection: brute force over every subset
# ----------------------------------------------------------------------------

def _brute_topk(scores, cand, kb):
    """Max-sum subset of size min(kb,|cand|); ties -> lexicographically smallest."""
    take = min(kb, len(cand))
    best, best_sum = None, None
    for comb in itertools.combinations(sorted(cand), take):
        ssum = sum(scores[j] for j in comb)
        if best is None or ssum > best_sum or (ssum == best_sum and comb < best):
            best, best_sum = comb, ssum
    return list(best)


@pytest.mark.parametrize("mode", [oracle.TOPK_CAUSAL_BLOCK, oracle.TOPK_LAST_BLOCK, oracle.TOPK_PLAIN])
def test_topk_matches_bruteforce(mode):
    r = _rng(10 + mode)
    for trial in range(40):
        nb = int(r.integers(1, 10))
        kb = int(r.integers(0, nb + 2))
        s = r.integers(-3, 4, size=(nb, nb)).astype(np.float32)   # many ties
        idx, cnt = oracle.topk(s, mode, kb)
        for row in range(nb):
            if mode == oracle.TOPK_CAUSAL_BLOCK:
                cand, forced = list(range(row)), [row]
            elif mode == oracle.TOPK_LAST_BLOCK:
                cand, forced = list(range(nb - 1)), [nb - 1]
            else:
                cand, forced = list(range(nb)), []
            want = sorted(_brute_topk(s[row].tolist(), cand, kb) + forced)
            got = [int(x) for x in idx[row] if x >= 0]
            assert got == want, (trial, row, s[row], kb)
            assert cnt[row] == len(want)
            assert np.all(idx[row][len(want):] == -1)


def test_topk_ties_go_to_lowest_index():
    s = np.array([[1.0, 2.0, 2.0, 2.0, 0.5, 2.0]], np.float32)
    idx, _ = oracle.topk(s, oracle.TOPK_PLAIN, 2)
    assert idx.tolist() == [[1, 2]]


def test_topk_nan_ranks_last():
    s = np.array([[np.nan, -np.inf, 0.0, np.nan, -1.0]], np.float32)
    idx, _ = oracle.topk(s, oracle.TOPK_PLAIN, 3)
    assert idx.tolist() == [[1, 2, 4]]
    idx, _ = oracle.topk(s, oracle.TOPK_PLAIN, 4)
    assert idx.tolist() == [[0, 1, 2, 4]]


# ----------------------------------------------------------------------------
# the mask: the pages' two worked examples
# ----------------------------------------------------------------------------

def test_sliding_window_w3_pattern_from_tutorial():
    """bs = 1 (one token per block), budget 2 history blocks, recency scores
    s_{i,j} = j: selection + forced current block must give the page's w=3
    causal window, and the mask must equal its printed 6x6 pattern."""
    golden = _read_golden_sets("sliding_window_w3.txt")
    N = 6
    s = np.full((N, N), -np.inf, np.float32)
    for i in range(N):
        for j in range(i + 1):
            s[i, j] = float(j)
    idx, _ = oracle.topk(s, oracle.TOPK_CAUSAL_BLOCK, 2)
    mask = oracle.prefill_mask(N, 1, idx)
    for t in range(N):
        seen = [u + 1 for u in range(N) if mask[t, u]]
        assert seen == golden[t + 1], (t, seen)


def test_block_sparse_4block_pattern_from_tutorial():
    golden = _read_golden_sets("block_sparse_4blocks.txt")
    idx = np.full((4, 3), -1, np.int32)
    for qb, ks in golden.items():
        idx[qb - 1, :len(ks)] = [x - 1 for x in ks]
    mask = oracle.prefill_mask(4, 1, idx)
    for t in range(4):
        assert [u + 1 for u in range(4) if mask[t, u]] == golden[t + 1]
    # At bs > 1 the same block pattern holds, with causality inside the
    # diagonal block only.
    bs = 3
    mask3 = oracle.prefill_mask(4 * bs, bs, idx)
    for t in range(4 * bs):
        for u in range(4 * bs):
            want = ((u // bs) + 1 in golden[t // bs + 1]) and u <= t
            assert mask3[t, u] == want


# ----------------------------------------------------------------------------
# attention: special cases that reduce to the dense library routine
# ----------------------------------------------------------------------------

def _small_prefill(seed, B=1, Hq=4, Hkv=2, N=192, d=16):
    r = _rng(seed)
    q = r.standard_normal((B, Hq, N, d)).astype(np.float32)
    k = r.standard_normal((B, Hkv, N, d)).astype(np.float32)
    v = r.standard_normal((B, Hkv, N, d)).astype(np.float32)
    return q, k, v


def test_prefill_full_budget_equals_dense_causal():
    q, k, v = _small_prefill(20)
    bs = 32
    Hkv = k.shape[1]
    G = q.shape[1] // Hkv
    _, _, _, idx, cnt = oracle.prefill_select(q, k, Hkv, bs, kb=64)
    nb = q.shape[2] // bs
    assert np.all(cnt == np.arange(nb)[None, None, :] + 1)
    out, lse = oracle.attend_prefill(q, k, v, bs, idx)
    ref = _sdpa64(q, np.repeat(k, G, 1), np.repeat(v, G, 1), causal=True)
    assert np.allclose(out.reshape(ref.shape), ref, atol=1e-10, rtol=0)
    # lse against the library logsumexp of the causal logits
    qt = torch.as_tensor(q, dtype=torch.float64)
    kt = torch.as_tensor(np.repeat(k, G, 1), dtype=torch.float64)
    logits = qt @ kt.transpose(-1, -2) / math.sqrt(q.shape[-1])
    causal = torch.ones(logits.shape[-2:], dtype=torch.bool).tril()
    ref_lse = torch.logsumexp(logits.masked_fill(~causal, -math.inf), dim=-1).numpy()
    assert np.allclose(lse.reshape(ref_lse.shape), ref_lse, atol=1e-10)


def test_prefill_sparse_equals_masked_library_attention():
    q, k, v = _small_prefill(21, B=2)
    bs, kb = 32, 2
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    _, _, _, idx, _ = oracle.prefill_select(q, k, Hkv, bs, kb)
    out, _ = oracle.attend_prefill(q, k, v, bs, idx)
    mask = np.zeros((B, Hq, N, N), bool)
    for b in range(B):
        for h in range(Hq):
            for t in range(N):
                blocks = set(int(x) for x in idx[b, h // G, t // bs] if x >= 0)
                for u in range(t + 1):
                    mask[b, h, t, u] = (u // bs) in blocks
    ref = _sdpa64(q, np.repeat(k, G, 1), np.repeat(v, G, 1), mask=mask)
    assert np.allclose(out.reshape(ref.shape), ref, atol=1e-10, rtol=0)


def test_prefill_selection_keeps_current_and_budget():
    q, k, v = _small_prefill(22, N=512)
    bs, kb = 32, 3
    _, _, _, idx, cnt = oracle.prefill_select(q, k, k.shape[1], bs, kb)
    nb = 512 // bs
    for i in range(nb):
        row = idx[0, 0, i]
        kept = [int(x) for x in row if x >= 0]
        assert kept[-1] == i                       # current block kept, list ascending
        assert kept == sorted(kept)
        assert len(kept) == min(kb, i) + 1


# ----------------------------------------------------------------------------
# the gate (SAS): invariants and the library routine with an additive bias
# ----------------------------------------------------------------------------

def test_gate_with_uniform_scores_equals_ungated():
    q, k, v = _small_prefill(30)
    bs, kb = 32, 2
    _, _, s, idx, _ = oracle.prefill_select(q, k, k.shape[1], bs, kb)
    ungated, lse_u = oracle.attend_prefill(q, k, v, bs, idx)
    uniform = np.full_like(s, 0.7)
    gated, _ = oracle.attend_prefill(q, k, v, bs, idx, gate_scores=uniform)
    assert np.allclose(gated, ungated, atol=1e-12, rtol=0)


def test_gate_is_shift_invariant():
    q, k, v = _small_prefill(31)
    bs, kb = 32, 2
    _, _, s, idx, _ = oracle.prefill_select(q, k, k.shape[1], bs, kb)
    # dyadic scores (multiples of 2^-10, |s| < 8) so that s + 3 is exact in fp32
    s = (np.round(s * 1024) / 1024).astype(np.float32)
    a, _ = oracle.attend_prefill(q, k, v, bs, idx, gate_scores=s)
    b, _ = oracle.attend_prefill(q, k, v, bs, idx, gate_scores=s + np.float32(3.0))
    assert np.allclose(a, b, atol=1e-12, rtol=0)


def test_gate_equals_library_attention_with_log_softmax_bias():
    q, k, v = _small_prefill(32)
    bs, kb = 32, 2
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    _, _, s, idx, _ = oracle.prefill_select(q, k, Hkv, bs, kb)
    s = s * np.float32(5.0)   # make the gate far from uniform
    out, _ = oracle.attend_prefill(q, k, v, bs, idx, gate_scores=s)
    bias = np.full((B, Hq, N, N), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(N // bs):
                kept = [int(x) for x in idx[b, g, i] if x >= 0]
                logg = torch.log_softmax(torch.tensor([float(s[b, g, i, j]) for j in kept],
                                                      dtype=torch.float64), 0).numpy()
                for t in range(i * bs, (i + 1) * bs):
                    for jj, j in enumerate(kept):
                        for u in range(j * bs, (j + 1) * bs):
                            if u <= t:
                                bias[b, h, t, u] = logg[jj]
    ref = _sdpa64(q, np.repeat(k, G, 1), np.repeat(v, G, 1), mask=bias)
    assert np.allclose(out.reshape(ref.shape), ref, atol=1e-10, rtol=0)


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------

def _small_decode(seed, B=2, Hq=8, Hkv=2, Nk=512, d=16):
    r = _rng(seed)
    q = r.standard_normal((B, Hq, d)).astype(np.float32)
    k = r.standard_normal((B, Hkv, Nk, d)).astype(np.float32)
    v = r.standard_normal((B, Hkv, Nk, d)).astype(np.float32)
    return q, k, v


def test_decode_full_budget_equals_dense():
    q, k, v = _small_decode(40)
    bs = 32
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kbar = oracle.pool_keys(k, bs)
    _, _, idx, cnt = oracle.decode_select(q, kbar, Hkv, kb=Nk // bs)
    assert np.all(cnt == Nk // bs)
    out, _ = oracle.attend_decode(q, k, v, bs, idx)
    ref = _sdpa64(q[:, :, None, :], np.repeat(k, G, 1), np.repeat(v, G, 1))
    assert np.allclose(out.reshape(B, Hq, d), ref[:, :, 0], atol=1e-10, rtol=0)


def test_decode_sparse_keeps_last_block_and_matches_library():
    q, k, v = _small_decode(41)
    bs, kb = 32, 3
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kbar = oracle.pool_keys(k, bs)
    _, _, idx, cnt = oracle.decode_select(q, kbar, Hkv, kb)
    assert np.all(idx[:, :, kb] == Nk // bs - 1)
    out, _ = oracle.attend_decode(q, k, v, bs, idx)
    mask = np.zeros((B, Hq, 1, Nk), bool)
    for b in range(B):
        for h in range(Hq):
            for j in idx[b, h // G]:
                mask[b, h, 0, j * bs:(j + 1) * bs] = True
    ref = _sdpa64(q[:, :, None, :], np.repeat(k, G, 1), np.repeat(v, G, 1), mask=mask)
    assert np.allclose(out.reshape(B, Hq, d), ref[:, :, 0], atol=1e-10, rtol=0)


# ----------------------------------------------------------------------------
# gist selective expansion (SSA)
# ----------------------------------------------------------------------------

def _small_gist(seed, B=2, Hq=4, Hkv=2, Nk=256, d=16, chunk=32):
    r = _rng(seed)
    q, k, v = _small_decode(seed, B, Hq, Hkv, Nk, d)
    nc = Nk // chunk
    gk = r.standard_normal((B, Hkv, nc, d)).astype(np.float32)
    gv = r.standard_normal((B, Hkv, nc, d)).astype(np.float32)
    return q, k, v, gk, gv


def test_gist_all_chunks_expanded_equals_dense():
    q, k, v, gk, gv = _small_gist(50)
    chunk = 32
    B, Hq, d = q.shape
    G = Hq // k.shape[1]
    _, idx, _ = oracle.gist_select(q, gk, kb=k.shape[2] // chunk)
    out, _ = oracle.attend_gist(q, k, v, gk, gv, chunk, idx)
    ref = _sdpa64(q[:, :, None, :], np.repeat(k, G, 1), np.repeat(v, G, 1))
    assert np.allclose(out.reshape(B, Hq, d), ref[:, :, 0], atol=1e-10, rtol=0)


def test_gist_nothing_expanded_equals_attention_over_gists():
    q, k, v, gk, gv = _small_gist(51)
    chunk = 32
    B, Hq, d = q.shape
    G = Hq // k.shape[1]
    _, idx, cnt = oracle.gist_select(q, gk, kb=0)
    assert np.all(cnt == 0)
    out, _ = oracle.attend_gist(q, k, v, gk, gv, chunk, np.full((B, Hq, 1), -1, np.int32))
    ref = _sdpa64(q[:, :, None, :], np.repeat(gk, G, 1), np.repeat(gv, G, 1))
    assert np.allclose(out.reshape(B, Hq, d), ref[:, :, 0], atol=1e-10, rtol=0)


def test_gist_mixture_matches_library_on_explicit_key_set():
    q, k, v, gk, gv = _small_gist(52)
    chunk, kb = 32, 3
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    nc = Nk // chunk
    s, idx, _ = oracle.gist_select(q, gk, kb)
    # per-head choices are independent: heads of one group may differ
    out, _ = oracle.attend_gist(q, k, v, gk, gv, chunk, idx)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            chosen = set(int(x) for x in idx[b, h] if x >= 0)
            assert len(chosen) == kb
            top = np.argsort(-s[b, h], kind="stable")[:kb]
            assert chosen == set(int(x) for x in top)
            keys, vals = [], []
            for c in range(nc):
                if c in chosen:
                    keys.append(k[b, g, c * chunk:(c + 1) * chunk]); vals.append(v[b, g, c * chunk:(c + 1) * chunk])
                else:
                    keys.append(gk[b, g, c:c + 1]); vals.append(gv[b, g, c:c + 1])
            K = np.concatenate(keys)[None, None]
            V = np.concatenate(vals)[None, None]
            ref = _sdpa64(q[b, h][None, None, None, :], K, V)
            assert np.allclose(out[b * Hq + h], ref[0, 0, 0], atol=1e-10, rtol=0)


# ----------------------------------------------------------------------------
# fixed pattern + dynamic blocks (MInference block-sparse): brute force, the
# tutorial's sliding window, and the plain causal top-k it reduces to
# ----------------------------------------------------------------------------

def test_topk_pattern_matches_bruteforce():
    r = _rng(70)
    for trial in range(60):
        nb = int(r.integers(1, 10))
        sink = int(r.integers(0, 3))
        local = int(r.integers(1, 4))
        kb = int(r.integers(0, nb + 1))
        s = r.integers(-3, 4, size=(nb, nb)).astype(np.float32)   # many ties
        idx, cnt = oracle.topk_pattern(s, sink, local, kb)
        for i in range(nb):
            forced = [j for j in range(i + 1) if j < sink or j > i - local]
            cand = [j for j in range(i) if j not in forced]
            want = sorted(_brute_topk(s[i].tolist(), cand, kb) + forced)
            got = [int(x) for x in idx[i] if x >= 0]
            assert got == want, (trial, i, sink, local, kb)
            assert cnt[i] == len(want) and np.all(idx[i][len(want):] == -1)


def test_topk_pattern_without_sink_and_window_is_the_causal_topk():
    r = _rng(71)
    s = r.standard_normal((2, 3, 40, 40)).astype(np.float32)
    for kb in (0, 3, 17, 40):
        got, gcnt = oracle.topk_pattern(s, 0, 1, kb, idx_stride=kb + 1)
        want, wcnt = oracle.topk(s, oracle.TOPK_CAUSAL_BLOCK, kb)
        assert np.array_equal(got, want) and np.array_equal(gcnt, wcnt)


def test_topk_pattern_window_only_is_the_tutorial_w3_window():
    """No sink, a local window of 3 blocks of one token, no dynamic blocks:
    the tutorial's 6-token, w = 3 causal sliding window (§3)."""
    golden = _read_golden_sets("sliding_window_w3.txt")
    N = 6
    s = _rng(72).standard_normal((N, N)).astype(np.float32)   # scores play no part
    idx, _ = oracle.topk_pattern(s, 0, 3, 0)
    mask = oracle.prefill_mask(N, 1, idx)
    for t in range(N):
        assert [u + 1 for u in range(N) if mask[t, u]] == golden[t + 1]


def test_topk_pattern_streaming_sink_plus_window_closed_form():
    """One sink block, a window of w blocks, no dynamic blocks: the
    StreamingLLM-style set {0} u {i-w+1, ..., i} (review §2.2.3)."""
    nb, w = 20, 4
    s = _rng(73).standard_normal((nb, nb)).astype(np.float32)
    idx, cnt = oracle.topk_pattern(s, 1, w, 0)
    for i in range(nb):
        want = sorted(set([0]) | set(range(max(0, i - w + 1), i + 1)))
        assert [int(x) for x in idx[i] if x >= 0] == want and cnt[i] == len(want)


# ----------------------------------------------------------------------------
# one budget shared by a group's heads (Ada-KV)
# ----------------------------------------------------------------------------

def test_topk_joint_heads_matches_bruteforce():
    r = _rng(74)
    for trial in range(40):
        G = int(r.integers(1, 4))
        nb = int(r.integers(1, 6))
        kb_total = int(r.integers(0, G * nb + 1))
        s = r.integers(-2, 3, size=(1, 1, G, nb)).astype(np.float32)
        idx, cnt = oracle.topk_joint_heads(s, kb_total, idx_stride=G * nb + 1)
        flat = [float(s[0, 0, h, j]) for h in range(G) for j in range(nb - 1)]
        chosen = _brute_topk(flat, list(range(len(flat))), kb_total)
        for h in range(G):
            want = sorted([c % (nb - 1) for c in chosen if c // (nb - 1) == h] + [nb - 1]) if nb > 1 else [0]
            got = [int(x) for x in idx[0, 0, h] if x >= 0]
            assert got == want, (trial, G, nb, kb_total, h)
            assert cnt[0, 0, h] == len(want)
        assert sum(int(c) for c in cnt[0, 0]) == min(kb_total, G * (nb - 1)) + G


def test_topk_joint_heads_single_head_is_the_decode_topk():
    r = _rng(75)
    s = r.standard_normal((3, 2, 1, 300)).astype(np.float32)
    for kb in (0, 5, 96, 400):
        got, gcnt = oracle.topk_joint_heads(s, kb, idx_stride=min(kb, 299) + 1)
        want, wcnt = oracle.topk(s[:, :, 0], oracle.TOPK_LAST_BLOCK, kb, idx_stride=min(kb, 299) + 1)
        assert np.array_equal(got[:, :, 0], want) and np.array_equal(gcnt[:, :, 0], wcnt)


def test_decode_heads_with_shared_lists_is_the_group_decode():
    q, k, v = _small_decode(76)
    bs, kb = 32, 4
    Hkv = k.shape[1]
    G = q.shape[1] // Hkv
    kbar = oracle.pool_keys(k, bs)
    _, _, idx, _ = oracle.decode_select(q, kbar, Hkv, kb)
    per_head = np.repeat(idx, G, axis=1)   # every head of a group keeps the group's blocks
    a, la = oracle.attend_decode(q, k, v, bs, idx)
    b, lb = oracle.attend_decode_heads(q, k, v, bs, per_head)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_decode_heads_matches_library_with_per_head_masks():
    q, k, v = _small_decode(77)
    bs = 32
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    nb = Nk // bs
    r = _rng(78)
    idx = np.full((B, Hq, 6), -1, np.int32)
    mask = np.zeros((B, Hq, 1, Nk), bool)
    for b in range(B):
        for h in range(Hq):
            sel = sorted(r.choice(nb, size=int(r.integers(1, 6)), replace=False).tolist())
            idx[b, h, :len(sel)] = sel
            for j in sel:
                mask[b, h, 0, j * bs:(j + 1) * bs] = True
    out, _ = oracle.attend_decode_heads(q, k, v, bs, idx)
    ref = _sdpa64(q[:, :, None, :], np.repeat(k, G, 1), np.repeat(v, G, 1), mask=mask)
    assert np.allclose(out.reshape(B, Hq, d), ref[:, :, 0], atol=1e-10, rtol=0)


# ----------------------------------------------------------------------------
# paged KV cache
# ----------------------------------------------------------------------------

def test_paged_gather_identity_table_is_the_contiguous_cache():
    B, Hkv, nb, bs, d = 2, 3, 5, 4, 8
    k = _rng(79).standard_normal((B, Hkv, nb * bs, d)).astype(np.float32)
    # pool laid out [P][Hkv][bs][d] with P = B*nb and the identity mapping
    pool = k.reshape(B, Hkv, nb, bs, d).transpose(0, 2, 1, 3, 4).reshape(B * nb, Hkv, bs, d)
    table = np.arange(B * nb, dtype=np.int32).reshape(B, nb)
    assert np.array_equal(oracle.paged_gather(pool, table, nb), k)


def test_paged_gather_permuted_pages():
    r = _rng(80)
    B, Hkv, nb, bs, d, P = 2, 2, 4, 3, 5, 11
    pool = r.standard_normal((P, Hkv, bs, d)).astype(np.float32)
    table = np.stack([r.permutation(P)[:nb] for _ in range(B)]).astype(np.int32)
    out = oracle.paged_gather(pool, table, nb)
    for b in range(B):
        for j in range(nb):
            for g in range(Hkv):
                assert np.array_equal(out[b, g, j * bs:(j + 1) * bs], pool[table[b, j], g])


# ----------------------------------------------------------------------------
# two-level gist routing (H-SSA)
# ----------------------------------------------------------------------------

def _small_hssa(seed, B=2, Hq=4, Hkv=2, Nk=512, d=16, chunk=16, M=4):
    r = _rng(seed)
    nc = Nk // chunk
    q = r.standard_normal((B, Hq, d)).astype(np.float32)
    k = r.standard_normal((B, Hkv, Nk, d)).astype(np.float32)
    v = r.standard_normal((B, Hkv, Nk, d)).astype(np.float32)
    gk = r.standard_normal((B, Hkv, nc, d)).astype(np.float32)
    gv = r.standard_normal((B, Hkv, nc, d)).astype(np.float32)
    mk = r.standard_normal((B, Hkv, nc // M, d)).astype(np.float32)
    mv = r.standard_normal((B, Hkv, nc // M, d)).astype(np.float32)
    return q, k, v, gk, gv, mk, mv


def test_hssa_with_every_group_kept_is_ssa():
    """Keeping every group, the fine step scores every gist: H-SSA's choice
    and attention are SSA's (SSA page, 推理时的关键模块)."""
    q, k, v, gk, gv, mk, mv = _small_hssa(90)
    chunk, M, kk = 16, 4, 5
    nm = gk.shape[2] // M
    meta, chunks = oracle.hssa_select(q, gk, mk, M, nm, kk)
    assert np.array_equal(meta, np.broadcast_to(np.arange(nm, dtype=np.int32), meta.shape))
    _, idx, _ = oracle.gist_select(q, gk, kk)
    assert np.array_equal(chunks, idx)
    a, la = oracle.attend_hssa(q, k, v, gk, gv, mk, mv, chunk, M, meta, chunks)
    b, lb = oracle.attend_gist(q, k, v, gk, gv, chunk, idx)
    assert np.allclose(a, b, atol=1e-12, rtol=0) and np.allclose(la, lb, atol=1e-12, rtol=0)


def test_hssa_with_nothing_kept_attends_the_meta_gists():
    q, k, v, gk, gv, mk, mv = _small_hssa(91)
    B, Hq, d = q.shape
    G = Hq // k.shape[1]
    meta, chunks = oracle.hssa_select(q, gk, mk, 4, 0, 0)
    assert np.all(meta == -1) and np.all(chunks == -1)
    out, _ = oracle.attend_hssa(q, k, v, gk, gv, mk, mv, 16, 4, meta, chunks)
    ref = _sdpa64(q[:, :, None, :], np.repeat(mk, G, 1), np.repeat(mv, G, 1))
    assert np.allclose(out.reshape(B, Hq, d), ref[:, :, 0], atol=1e-10, rtol=0)


def test_hssa_one_chunk_groups_expanding_every_kept_group():
    """Groups of one chunk, every kept group expanded: the keys are the kept
    chunks' tokens and the meta-gists of the rest, i.e. SSA with the
    meta-gists as the gists and the meta selection as the expanded set."""
    q, k, v, gk, gv, mk, mv = _small_hssa(92, M=1)
    chunk, km = 16, 6
    meta, chunks = oracle.hssa_select(q, gk, mk, 1, km, km)
    assert np.array_equal(meta, chunks)
    a, _ = oracle.attend_hssa(q, k, v, gk, gv, mk, mv, chunk, 1, meta, chunks)
    b, _ = oracle.attend_gist(q, k, v, mk, mv, chunk, meta)
    assert np.allclose(a, b, atol=1e-12, rtol=0)


def test_hssa_selection_matches_bruteforce():
    """Integer-valued queries and keys make every score exact, with many
    ties: the two-level choice equals brute force over subsets."""
    r = _rng(93)
    for trial in range(20):
        B, Hq, Hkv, d, M = 1, 2, 1, 4, 3
        nc = 3 * M
        km = int(r.integers(0, 4))
        kk = int(r.integers(0, km * M + 2))
        q = r.integers(-2, 3, (B, Hq, d)).astype(np.float32)
        gk = r.integers(-2, 3, (B, Hkv, nc, d)).astype(np.float32)
        mk = r.integers(-2, 3, (B, Hkv, nc // M, d)).astype(np.float32)
        meta, chunks = oracle.hssa_select(q, gk, mk, M, km, kk)
        for h in range(Hq):
            ms = [float(np.dot(q[0, h], mk[0, 0, m])) for m in range(nc // M)]
            want_m = sorted(_brute_topk(ms, list(range(nc // M)), km))
            assert [int(x) for x in meta[0, h] if x >= 0] == want_m
            cand = [c for m in want_m for c in range(m * M, (m + 1) * M)]
            cs = {c: float(np.dot(q[0, h], gk[0, 0, c])) for c in cand}
            want_c = sorted(_brute_topk([cs.get(c, 0.0) for c in range(nc)], cand, kk))
            assert [int(x) for x in chunks[0, h] if x >= 0] == want_c, (trial, h)


def test_hssa_attention_matches_library_on_explicit_key_set():
    q, k, v, gk, gv, mk, mv = _small_hssa(94)
    chunk, M, km, kk = 16, 4, 3, 4
    B, Hq, d = q.shape
    G = Hq // k.shape[1]
    nc, nm = gk.shape[2], mk.shape[2]
    meta, chunks = oracle.hssa_select(q, gk, mk, M, km, kk)
    out, _ = oracle.attend_hssa(q, k, v, gk, gv, mk, mv, chunk, M, meta, chunks)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            keys, vals = [], []
            kept = set(int(x) for x in meta[b, h] if x >= 0)
            exp = set(int(x) for x in chunks[b, h] if x >= 0)
            for m in range(nm):
                if m not in kept:
                    keys.append(mk[b, g, m]); vals.append(mv[b, g, m]); continue
                for c in range(m * M, (m + 1) * M):
                    if c in exp:
                        keys.extend(k[b, g, c * chunk:(c + 1) * chunk]); vals.extend(v[b, g, c * chunk:(c + 1) * chunk])
                    else:
                        keys.append(gk[b, g, c]); vals.append(gv[b, g, c])
            ref = _sdpa64(q[b, h][None, None], np.array(keys)[None], np.array(vals)[None])
            assert np.allclose(out[b * Hq + h], ref[0, 0], atol=1e-10, rtol=0)


# ----------------------------------------------------------------------------
# backward of the (gated) sparse prefill attention
# ----------------------------------------------------------------------------

def _bwd_case(seed, B=1, Hq=4, Hkv=2, N=96, d=8, bs=16, kb=2):
    r = _rng(seed)
    q = r.standard_normal((B, Hq, N, d)).astype(np.float32)
    k = r.standard_normal((B, Hkv, N, d)).astype(np.float32)
    v = r.standard_normal((B, Hkv, N, d)).astype(np.float32)
    dO = r.standard_normal((B, Hq, N, d)).astype(np.float32)
    _, _, s, idx, _ = oracle.prefill_select(q, k, Hkv, bs, kb)
    return q, k, v, dO, s, idx


def _autograd_reference(q, k, v, dO, s, idx, bs, gated):
    """torch autograd (fp64) of sum(dO * SDPA(q, k, v, bias)) where bias is the
    sparse causal mask (-inf off the kept blocks) plus, gated, log_softmax of
    the kept blocks' scores broadcast over each block's keys."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G, nb = Hq // Hkv, N // bs
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    ts = torch.tensor(s, dtype=torch.float64, requires_grad=True)
    kept = torch.zeros((B, Hkv, nb, nb), dtype=torch.bool)
    for b in range(B):
        for g in range(Hkv):
            for i in range(nb):
                for j in idx[b, g, i]:
                    if j >= 0:
                        kept[b, g, i, j] = True
    bias_blk = torch.where(kept, torch.zeros((), dtype=torch.float64), torch.tensor(float("-inf"), dtype=torch.float64))
    if gated:
        logits = ts.masked_fill(~kept, float("-inf"))
        bias_blk = bias_blk + torch.log_softmax(logits, dim=-1).masked_fill(~kept, 0.0)
    bias = bias_blk.repeat_interleave(bs, dim=2).repeat_interleave(bs, dim=3)          # [B,Hkv,N,N]
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    bias = bias.masked_fill(~causal, float("-inf")).repeat_interleave(G, dim=1)       # [B,Hq,N,N]
    o = F.scaled_dot_product_attention(tq, tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1), attn_mask=bias)
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy(), (ts.grad.numpy() if gated else None)


@pytest.mark.parametrize("gated", [False, True])
def test_backward_matches_library_autograd(gated):
    q, k, v, dO, s, idx = _bwd_case(100 + gated)
    dq, dk, dv, ds = oracle.attend_prefill_bwd(q, k, v, dO, 16, idx, gate_scores=s if gated else None)
    rq, rk, rv, rs = _autograd_reference(q, k, v, dO, s, idx, 16, gated)
    for got, want in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.allclose(got, want, atol=1e-10, rtol=1e-9)
    if gated:
        assert np.allclose(ds, rs, atol=1e-10, rtol=1e-9)


def test_backward_central_differences():
    """d/dx of sum(dO * O) by central differences of the oracle's own forward,
    at sampled coordinates of q, k, v and the selector scores."""
    q, k, v, dO, s, idx = _bwd_case(102, N=48, d=4, bs=8, kb=2)
    dq, dk, dv, ds = oracle.attend_prefill_bwd(q, k, v, dO, 8, idx, gate_scores=s)

    def loss(q_, k_, v_, s_):
        o, _ = oracle.attend_prefill(q_, k_, v_, 8, idx, gate_scores=s_)
        return float((o.reshape(dO.shape) * dO.astype(np.float64)).sum())

    r = _rng(103)
    eps = 1e-2
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("s", s, ds)):
        for _ in range(6):
            pos = tuple(int(r.integers(0, n)) for n in arr.shape)
            if name == "s" and not np.isfinite(arr[pos]):
                continue
            hi, lo = arr.copy(), arr.copy()
            hi[pos] += eps
            lo[pos] -= eps
            args = {"q": q, "k": k, "v": v, "s": s}
            args_hi = dict(args, **{name: hi})
            args_lo = dict(args, **{name: lo})
            fd = (loss(args_hi["q"], args_hi["k"], args_hi["v"], args_hi["s"]) -
                  loss(args_lo["q"], args_lo["k"], args_lo["v"], args_lo["s"])) / (float(hi[pos]) - float(lo[pos]))
            assert abs(fd - grad[pos]) <= 1e-4 * max(1.0, abs(grad[pos])), (name, pos, fd, grad[pos])


def test_backward_score_gradient_sums_to_zero_per_unit():
    """log g_j = s_j - log sum exp(s_kept): adding a constant to a unit's
    scores changes nothing, so the unit's score gradients sum to zero."""
    q, k, v, dO, s, idx = _bwd_case(104)
    _, _, _, ds = oracle.attend_prefill_bwd(q, k, v, dO, 16, idx, gate_scores=s)
    assert np.abs(ds.sum(axis=-1)).max() < 1e-12
    assert np.abs(ds).max() > 1e-3


def test_backward_uniform_gate_equals_ungated():
    q, k, v, dO, s, idx = _bwd_case(105)
    flat = np.zeros_like(s)
    a = oracle.attend_prefill_bwd(q, k, v, dO, 16, idx, gate_scores=flat)
    b = oracle.attend_prefill_bwd(q, k, v, dO, 16, idx)
    for x, y in zip(a[:3], b[:3]):
        assert np.allclose(x, y, atol=1e-12, rtol=0)


def test_backward_full_budget_is_dense_causal():
    q, k, v, dO, _, _ = _bwd_case(106)
    N, bs = q.shape[2], 16
    nb = N // bs
    _, _, s, idx, _ = oracle.prefill_select(q, k, k.shape[1], bs, nb)
    dq, dk, dv, _ = oracle.attend_prefill_bwd(q, k, v, dO, bs, idx)
    G = q.shape[1] // k.shape[1]
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    o = F.scaled_dot_product_attention(tq, tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1), is_causal=True)
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    assert np.allclose(dq, tq.grad.numpy(), atol=1e-10, rtol=1e-9)
    assert np.allclose(dk, tk.grad.numpy(), atol=1e-10, rtol=1e-9)
    assert np.allclose(dv, tv.grad.numpy(), atol=1e-10, rtol=1e-9)
