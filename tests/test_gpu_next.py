"""GPU parity of the widened path against the CPU oracle: the fixed pattern +
dynamic blocks selection (MInference block-sparse), one budget shared by a
group's heads with per-head decode attention (Ada-KV), decode over a paged
KV cache with the pooled summary kept up by appends (PagedAttention),
two-level gist routing (H-SSA), and the backward of the sparse / gated
prefill attention (SAS: gradients reach the selector scores through the
inner log-gate).

Selections are compared bit for bit (both sides use the same fixed-order fp32
scores); attention runs on the oracle's index sets and must be within
max-abs 2e-2 / mean-abs 2e-3 of the oracle's fp64 result (bf16 inputs).
"""
import numpy as np
import pytest
import torch

import bsa_workloads as W
import oracle

pytestmark = pytest.mark.gpu

TOL_BF16 = dict(max_abs=2e-2, mean_abs=2e-3)
TOL_LSE = dict(max_abs=2e-3, mean_abs=2e-4)


def _bsa():
    import top_block_sparse_bsa_b200 as bsa
    return bsa


def _pipe():
    from top_block_sparse_bsa_b200 import pipeline
    return pipeline


def _assert_close(got, want, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    assert err.max() <= tol["max_abs"], f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= tol["mean_abs"], f"{what}: mean-abs {err.mean():.3e}"


def _status_clean():
    code, flags = _bsa().bsa_device_status(reset=True)
    assert code == 0 and flags == 0, f"device status {code} flags {flags:#x}"


# ----------------------------------------------------------------------------
# fixed pattern + dynamic blocks
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("ncols", [1, 7, 33, 300, 2048, 5000])
def test_topk_pattern_ties_nan_and_budgets(ncols):
    bsa = _bsa()
    r = np.random.default_rng(500 + ncols)
    rows = 2 * ncols if ncols < 100 else 40
    for sink, local, kb in ((0, 1, 3), (1, 2, 5), (2, 4, 0), (3, 1, 64), (1, 3, ncols + 5)):
        s = r.integers(-4, 5, size=(rows, ncols)).astype(np.float32)
        s[0, ::3] = np.nan
        s[1 % rows, :] = 0.0
        s[2 % rows, ::2] = -np.inf
        stride = sink + local + kb + 1
        want, cnt = oracle.topk_pattern(s, sink, local, kb, idx_stride=stride)
        idx = torch.full((rows, stride), -7, dtype=torch.int32, device="cuda")
        count = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
        bsa.bsa_topk_select_pattern(torch.from_numpy(s).cuda(), rows, ncols, sink, local, kb, idx, stride, count)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), want), (ncols, sink, local, kb)
        assert np.array_equal(count.cpu().numpy(), cnt)
    _status_clean()


@pytest.mark.parametrize("gated", [False, True])
def test_prefill_with_pattern_selection(gated):
    """Selection with one sink block and a two-block window on the GQA prefill
    shape (scaled), then the tcgen05 attention on the oracle's lists."""
    pipe = _pipe()
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=8, Hkv=2, N=4096, kb=4)
    inp = W.make_inputs(w, "cuda")
    step = pipe.PrefillStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb, gated=gated, pattern=(1, 2))
    step.select()
    torch.cuda.synchronize()
    qc, kc, vc = (inp[x].float().cpu() for x in ("q", "k", "v"))
    _, _, s, _, _ = oracle.prefill_select(qc, kc, w.Hkv, w.bs, w.kb)
    assert np.array_equal(step.bufs["scores"].cpu().numpy(), s)
    idx, cnt = oracle.topk_pattern(s, 1, 2, w.kb)
    assert np.array_equal(step.bufs["idx"].cpu().numpy(), idx)
    assert np.array_equal(step.bufs["count"].cpu().numpy(), cnt)
    step.attend(idx=torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    _status_clean()
    want, want_lse = oracle.attend_prefill(qc, kc, vc, w.bs, idx, gate_scores=s if gated else None)
    _assert_close(step.bufs["o"].float().reshape(-1, w.d).cpu().numpy(), want, TOL_BF16, "pattern prefill")
    _assert_close(step.bufs["lse"].reshape(-1).cpu().numpy(), want_lse, TOL_LSE, "pattern lse")


# ----------------------------------------------------------------------------
# one budget across a group's heads
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("G,nb", [(1, 300), (4, 64), (4, 2048), (16, 100), (3, 2)])
def test_topk_joint_heads_ties_nan_and_budgets(G, nb):
    bsa = _bsa()
    r = np.random.default_rng(600 + G * nb)
    rows = 6
    for kb_total in (0, 1, 7, 96 * G, G * nb + 3):
        s = r.integers(-4, 5, size=(rows, G, nb)).astype(np.float32)
        s[0, 0, ::3] = np.nan
        s[1, :, :] = 0.0
        s[2, -1, ::2] = -np.inf
        stride = min(kb_total, nb - 1) + 1
        want, cnt = oracle.topk_joint_heads(s.reshape(1, rows, G, nb), kb_total, idx_stride=stride)
        idx = torch.full((rows, G, stride), -7, dtype=torch.int32, device="cuda")
        count = torch.full((rows, G), -7, dtype=torch.int32, device="cuda")
        bsa.bsa_topk_select_joint_heads(torch.from_numpy(s).cuda(), rows, G, nb, kb_total, idx, stride, count)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), want[0]), (G, nb, kb_total)
        assert np.array_equal(count.cpu().numpy(), cnt[0])
    _status_clean()


def _head_budget_case(w, kb_total, groups=None):
    pipe = _pipe()
    inp = W.make_inputs(w, "cuda")
    q, kc, vc = inp["q"], inp["k"], inp["v"]
    step = pipe.HeadBudgetDecodeStep(q, kc, vc, w.bs, kb_total)
    step.pool_cache()
    step.select()
    torch.cuda.synchronize()
    G = w.G
    if groups is None:
        groups = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    got_s = step.bufs["scores"].cpu().numpy()
    got_idx = step.bufs["idx"].cpu().numpy()
    for (b, g) in groups:
        qs = q[b:b + 1, g * G:(g + 1) * G].float().cpu()
        kbar = oracle.pool_keys(kc[b:b + 1, g:g + 1].float().cpu(), w.bs)
        assert np.array_equal(step.bufs["kbar"][b:b + 1, g:g + 1].cpu().numpy(), kbar)
        s = oracle.scores_gist(qs, kbar)           # q_h . kbar_j / sqrt(d), per head
        assert np.array_equal(got_s[b, g * G:(g + 1) * G], s[0]), (b, g)
        idx, _ = oracle.topk_joint_heads(s.reshape(1, 1, G, -1), kb_total, idx_stride=step.idx_stride)
        assert np.array_equal(got_idx[b, g * G:(g + 1) * G], idx[0, 0]), (b, g)
    step.attend()
    torch.cuda.synchronize()
    _status_clean()
    for (b, g) in groups:
        qs = q[b:b + 1, g * G:(g + 1) * G].float().cpu()
        want, want_lse = oracle.attend_decode_heads(qs, kc[b:b + 1, g:g + 1].float().cpu(),
                                                    vc[b:b + 1, g:g + 1].float().cpu(), w.bs,
                                                    got_idx[b:b + 1, g * G:(g + 1) * G])
        _assert_close(step.bufs["o"][b, g * G:(g + 1) * G].float().cpu().numpy(), want, TOL_BF16, f"({b},{g})")
        _assert_close(step.bufs["lse"][b, g * G:(g + 1) * G].cpu().numpy(), want_lse, TOL_LSE, "lse")


@pytest.mark.parametrize("hq,hkv,kb_total", [(8, 2, 48), (4, 1, 1), (16, 2, 300), (2, 2, 10), (32, 2, 64)])
def test_head_budget_decode_small(hq, hkv, kb_total):
    w = W.get("decode_bf16").scaled(B=2, Hq=hq, Hkv=hkv, N=8192, kb=kb_total)
    _head_budget_case(w, kb_total)


def test_head_budget_decode_full_size_sampled():
    """The decode workload (16 sequences, 131072 tokens) with a budget of
    96 blocks per head on average (384 per group of four heads)."""
    w = W.get("decode_bf16")
    _head_budget_case(w, 96 * w.G, groups=[(0, 0), (7, 3), (15, 7)])


# ----------------------------------------------------------------------------
# paged KV cache
# ----------------------------------------------------------------------------

def _pages(w, table):
    """Pools [P, Hkv, 64, d] holding the contiguous cache's blocks at the
    table's physical ids (test set-up: plain indexing, no method arithmetic)."""
    inp = W.make_inputs(w, "cuda")
    B, Hkv, N, d = inp["k"].shape
    nb = N // w.bs
    P = int(table.max().item()) + 1
    pools = []
    for name in ("k", "v"):
        blocks = inp[name].view(B, Hkv, nb, w.bs, d).permute(0, 2, 1, 3, 4).reshape(B * nb, Hkv, w.bs, d)
        pool = torch.zeros((P, Hkv, w.bs, d), dtype=inp[name].dtype, device="cuda")
        pool[table.reshape(-1).long()] = blocks
        pools.append(pool)
    return inp, pools[0], pools[1]


def test_paged_decode_identity_table_equals_contiguous_decode():
    pipe = _pipe()
    w = W.get("decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=12)
    nb = w.N // w.bs
    table = torch.arange(w.B * nb, dtype=torch.int32, device="cuda").view(w.B, nb)
    inp, kp, vp = _pages(w, table)
    ref = pipe.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
    ref.pool_cache()
    ref.run()
    paged = pipe.PagedDecodeStep(inp["q"], kp, vp, table, w.bs, w.kb)
    paged.bufs["kbar"].copy_(ref.bufs["kbar"])
    paged.run()
    torch.cuda.synchronize()
    assert torch.equal(paged.bufs["idx"], ref.bufs["idx"])
    assert torch.equal(paged.bufs["o"], ref.bufs["o"])
    assert torch.equal(paged.bufs["lse"], ref.bufs["lse"])
    _status_clean()


@pytest.mark.parametrize("chunks", [[8192], [100, 37, 1000, 64, 6991]])
def test_paged_append_then_decode_matches_oracle(chunks):
    """Build the cache by appends into permuted pages (whole, or in ragged
    pieces that complete blocks mid-append), then decode: the pages hold the
    logical cache, the summary equals pooling the logical cache, and the
    selection and output match the oracle's."""
    pipe = _pipe()
    w = W.get("decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=20)
    nb = w.N // w.bs
    r = np.random.default_rng(81)
    P = w.B * nb + 7
    table = torch.from_numpy(r.permutation(P)[:w.B * nb].reshape(w.B, nb).astype(np.int32)).cuda()
    inp = W.make_inputs(w, "cuda")
    kp = torch.zeros((P, w.Hkv, w.bs, w.d), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    step = pipe.PagedDecodeStep(inp["q"], kp, vp, table, w.bs, w.kb)
    pos = 0
    for T in chunks:
        lens = torch.full((w.B,), pos, dtype=torch.int32, device="cuda")
        step.append(inp["k"][:, :, pos:pos + T].contiguous(), inp["v"][:, :, pos:pos + T].contiguous(), lens)
        pos += T
    assert pos == w.N
    step.run()
    torch.cuda.synchronize()
    _status_clean()
    kc, vc, qc = inp["k"].float().cpu(), inp["v"].float().cpu(), inp["q"].float().cpu()
    logical_k = oracle.paged_gather(kp.float().cpu(), table.cpu(), nb)
    assert np.array_equal(logical_k, kc.numpy())
    assert np.array_equal(oracle.paged_gather(vp.float().cpu(), table.cpu(), nb), vc.numpy())
    kbar = oracle.pool_keys(logical_k, w.bs)
    assert np.array_equal(step.bufs["kbar"].cpu().numpy(), kbar)
    _, s, idx, _ = oracle.decode_select(qc, kbar, w.Hkv, w.kb)
    assert np.array_equal(step.bufs["scores"].cpu().numpy(), s)
    assert np.array_equal(step.bufs["idx"].cpu().numpy(), idx)
    want, want_lse = oracle.attend_decode(qc, logical_k, vc, w.bs, idx)
    _assert_close(step.bufs["o"].float().reshape(-1, w.d).cpu().numpy(), want, TOL_BF16, "paged decode")
    _assert_close(step.bufs["lse"].reshape(-1).cpu().numpy(), want_lse, TOL_LSE, "paged lse")


def test_paged_decode_full_size_permuted_pages_sampled():
    """The decode workload (16 x 131072 tokens) in randomly permuted pages:
    selection on every row and outputs of sampled groups against the oracle."""
    pipe = _pipe()
    w = W.get("decode_bf16")
    nb = w.N // w.bs
    r = np.random.default_rng(82)
    table = torch.from_numpy(r.permutation(w.B * nb).reshape(w.B, nb).astype(np.int32)).cuda()
    inp, kp, vp = _pages(w, table)
    ref = pipe.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
    ref.pool_cache()
    step = pipe.PagedDecodeStep(inp["q"], kp, vp, table, w.bs, w.kb)
    step.bufs["kbar"].copy_(ref.bufs["kbar"])
    step.run()
    torch.cuda.synchronize()
    _status_clean()
    idx = step.bufs["idx"].cpu().numpy()
    for (b, g) in [(0, 0), (6, 2), (15, 7)]:
        kbar = oracle.pool_keys(inp["k"][b:b + 1, g:g + 1].float().cpu(), w.bs)
        qs = inp["q"][b:b + 1, g * w.G:(g + 1) * w.G].float().cpu()
        _, _, want_idx, _ = oracle.decode_select(qs, kbar, 1, w.kb)
        assert np.array_equal(idx[b, g], want_idx[0, 0])
        want, _ = oracle.attend_decode(qs, inp["k"][b:b + 1, g:g + 1].float().cpu(),
                                       inp["v"][b:b + 1, g:g + 1].float().cpu(), w.bs, want_idx)
        _assert_close(step.bufs["o"][b, g * w.G:(g + 1) * w.G].float().cpu().numpy(), want, TOL_BF16, f"({b},{g})")


# ----------------------------------------------------------------------------
# two-level gist routing (H-SSA)
# ----------------------------------------------------------------------------

def _hssa_case(w, km, topk, rows_per_batch=None):
    pipe = _pipe()
    inp = W.make_inputs(w, "cuda")
    step = pipe.HssaStep(inp["q"], inp["k"], inp["v"], inp["gk"], inp["gv"], inp["mk"], inp["mv"], w.bs, km, topk)
    step.run()
    torch.cuda.synchronize()
    _status_clean()
    got_meta = step.bufs["meta_idx"].cpu().numpy()
    got_idx = step.bufs["idx"].cpu().numpy()
    for b in range(w.B):
        sl = slice(b, b + 1)
        q = inp["q"][sl].float().cpu()
        gk, gv = inp["gk"][sl].float().cpu(), inp["gv"][sl].float().cpu()
        mk, mv = inp["mk"][sl].float().cpu(), inp["mv"][sl].float().cpu()
        meta, chunks = oracle.hssa_select(q, gk, mk, 64, km, topk)
        assert np.array_equal(got_meta[sl], meta), b
        if topk > 0:
            assert np.array_equal(got_idx[sl], chunks), b
        rows = None if rows_per_batch is None else np.arange(rows_per_batch)
        want, want_lse = oracle.attend_hssa(q, inp["k"][sl].float().cpu(), inp["v"][sl].float().cpu(), gk, gv, mk, mv,
                                            w.bs, 64, meta, chunks, rows=rows)
        got = step.bufs["o"][b].float().cpu().numpy()
        got_lse = step.bufs["lse"][b].cpu().numpy()
        if rows is not None:
            got, got_lse = got[rows], got_lse[rows]
        _assert_close(got, want, TOL_BF16, f"hssa b={b}")
        _assert_close(got_lse, want_lse, TOL_LSE, "hssa lse")


@pytest.mark.parametrize("hq,hkv,km,topk", [(8, 2, 2, 8), (4, 1, 1, 0), (4, 1, 4, 256), (16, 2, 3, 5), (2, 2, 1, 64)])
def test_hssa_small(hq, hkv, km, topk):
    """16384 tokens = 256 chunks = 4 groups of 64 chunks: one group kept (all
    its chunks expanded at topk 64), no chunk expanded (gists and meta-gists
    only), every group kept with every chunk expanded (dense over tokens)."""
    w = W.get("hssa_decode_bf16").scaled(B=2, Hq=hq, Hkv=hkv, N=16384, kb=topk)
    _hssa_case(w, km, topk)


@pytest.mark.parametrize("km,ngroups,topk", [(6, 8, 40), (12, 16, 100), (20, 24, 33)])
def test_hssa_many_kept_groups(km, ngroups, topk):
    """More kept groups per head (6, 12, 20 of 8, 16, 24 groups of 64 chunks):
    the fine top-k then runs over 384, 768 or 1280 positions (two, four or
    eight keys per thread in the select that shares the scoring launch)."""
    w = W.get("hssa_decode_bf16").scaled(B=1, Hq=4, Hkv=1, N=ngroups * 64 * 64, kb=topk)
    _hssa_case(w, km, topk)


def test_hssa_full_size():
    """The gist workload's shape with meta-gists: 8 sequences x 131072 tokens,
    2048 chunks in 32 groups, 4 groups kept and 32 chunks expanded per head;
    every head's choice compared, outputs of every head of the first two
    sequences."""
    w = W.get("hssa_decode_bf16")
    _hssa_case(w.scaled(B=2, name=w.name), W.HSSA_GROUPS_KEPT, w.kb)


# ----------------------------------------------------------------------------
# backward of the sparse / gated prefill attention
# ----------------------------------------------------------------------------

def _bwd_case(w, gated, empty_frac=0.0):
    pipe = _pipe()
    inp = W.make_inputs(w, "cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    step = pipe.PrefillStep(q, k, v, w.bs, w.kb, gated=gated)
    step.select()
    torch.cuda.synchronize()
    qc, kc, vc = q.float().cpu(), k.float().cpu(), v.float().cpu()
    _, _, s, idx, _ = oracle.prefill_select(qc, kc, w.Hkv, w.bs, w.kb)
    if empty_frac > 0:
        empty = np.random.default_rng(12).random(idx.shape[:3]) < empty_frac
        idx = idx.copy()
        idx[empty] = -1
    idx_dev = torch.from_numpy(idx).cuda()
    step.attend(idx=idx_dev)
    g = torch.Generator(device="cuda").manual_seed(77)
    d_o = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    step.backward(d_o, idx=idx_dev)
    torch.cuda.synchronize()
    _status_clean()
    dq, dk, dv, ds = oracle.attend_prefill_bwd(qc, kc, vc, d_o.float().cpu(), w.bs, idx,
                                               gate_scores=s if gated else None)
    b = step.bufs
    _assert_close(b["dq"].cpu().numpy(), dq, TOL_BF16, "dq")
    _assert_close(b["dk"].cpu().numpy(), dk, TOL_BF16, "dk")
    _assert_close(b["dv"].cpu().numpy(), dv, TOL_BF16, "dv")
    if gated:
        _assert_close(b["dsel"].cpu().numpy(), ds, TOL_BF16, "dsel")
        kept = ds != 0
        assert np.all(b["dsel"].cpu().numpy()[~kept] == 0.0)


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("hq,hkv,bs,kb", [(4, 2, 64, 3), (5, 1, 64, 4), (7, 1, 128, 3)])
def test_backward_small(gated, hq, hkv, bs, kb):
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=hq, Hkv=hkv, N=2048, bs=bs, kb=kb)
    _bwd_case(w, gated)


def test_backward_full_budget_and_empty_lists():
    base = W.get("prefill_gqa_bf16")
    _bwd_case(base.scaled(B=1, Hq=4, Hkv=1, N=2048, kb=31), gated=True)
    _bwd_case(base.scaled(B=2, Hq=4, Hkv=2, N=2048, kb=4), gated=True, empty_frac=0.4)


def test_backward_gated_workload_shape_sampled():
    """The gated workload's head layout (28 query / 4 KV heads, 128-token
    blocks, budget 8 + current) at 4096 tokens, checked element by element."""
    w = W.get("gated_prefill_bf16").scaled(B=1, N=4096)
    _bwd_case(w, gated=True)
