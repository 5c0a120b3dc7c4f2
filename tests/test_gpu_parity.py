"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Selection: the selector is computed in the same fixed fp32 order on both
sides, so pooled means, scores and kept indices are compared bit for bit.
Attention: both sides are fed the oracle's index set, and the outputs must
be within max-abs 2e-2 / mean-abs 2e-3 (bf16 inputs) or max-abs 1e-4 (fp32
inputs) of the oracle's fp64 result.

Small cases span several tiles and odd (ragged) kept lists and are checked on
every output row; the full workload sizes are checked on sampled rows.
"""
import numpy as np
import pytest
import torch

import bsa_workloads as W
import oracle

pytestmark = pytest.mark.gpu

TOL_BF16 = dict(max_abs=2e-2, mean_abs=2e-3)
TOL_F32 = dict(max_abs=1e-4, mean_abs=1e-4)


def _bsa():
    import top_block_sparse_bsa_b200 as bsa
    return bsa


def _pipe():
    from top_block_sparse_bsa_b200 import pipeline
    return pipeline


def _tol(dtype):
    return TOL_F32 if dtype == "f32" else TOL_BF16


def _assert_close(got, want, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    assert err.max() <= tol["max_abs"], f"{what}: max-abs {err.max():.3e} > {tol['max_abs']}"
    assert err.mean() <= tol["mean_abs"], f"{what}: mean-abs {err.mean():.3e} > {tol['mean_abs']}"


def _status_clean():
    bsa = _bsa()
    code, flags = bsa.bsa_device_status(reset=True)
    assert code == 0 and flags == 0, f"device status {code} flags {flags:#x}"


# ----------------------------------------------------------------------------
# prefill (ungated and gated)
# ----------------------------------------------------------------------------

def _prefill_case(w: W.Workload, gated: bool, rows_sample=None):
    pipe = _pipe()
    inp = W.make_inputs(w, "cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    step = pipe.PrefillStep(q, k, v, w.bs, w.kb, gated=gated)
    step.select()
    torch.cuda.synchronize()
    qc, kc, vc = q.float().cpu(), k.float().cpu(), v.float().cpu()
    qbar, kbar, s, idx, cnt = oracle.prefill_select(qc, kc, w.Hkv, w.bs, w.kb)
    b = step.bufs
    # selector: bit-exact
    assert np.array_equal(b["kbar"].cpu().numpy(), kbar), "pooled keys differ"
    assert np.array_equal(b["qbar"].cpu().numpy(), qbar), "pooled queries differ"
    assert np.array_equal(b["scores"].cpu().numpy(), s), "scores differ"
    assert np.array_equal(b["idx"].cpu().numpy(), idx), "kept indices differ"
    assert np.array_equal(b["count"].cpu().numpy(), cnt)
    # attention on the oracle's index set
    idx_dev = torch.from_numpy(idx).cuda()
    step.attend(idx=idx_dev)
    torch.cuda.synchronize()
    _status_clean()
    total = w.B * w.Hq * w.N
    rows = np.arange(total) if rows_sample is None else np.asarray(rows_sample, dtype=np.int64)
    want, want_lse = oracle.attend_prefill(qc, kc, vc, w.bs, idx, gate_scores=s if gated else None, rows=rows)
    got = b["o"].float().reshape(total, w.d)[torch.from_numpy(rows).cuda()].cpu().numpy()
    got_lse = b["lse"].reshape(total)[torch.from_numpy(rows).cuda()].cpu().numpy()
    _assert_close(got, want, _tol(w.dtype), f"{w.name} out")
    _assert_close(got_lse, want_lse, dict(max_abs=2e-3, mean_abs=2e-4) if w.dtype == "bf16" else TOL_F32,
                  f"{w.name} lse")


@pytest.mark.parametrize("gated", [False, True])
def test_tiny_prefill_f32_full_config(gated):
    _prefill_case(W.get("tiny_prefill_f32"), gated)


@pytest.mark.parametrize("bs,hq", [(64, 1), (64, 3), (64, 5), (128, 1), (128, 3)])
def test_prefill_bf16_ragged_tiles(bs, hq):
    # G*bs stacked rows that do not fill 128-row tiles (64, 192, 320 rows at
    # bs 64) and units with an odd tile count (single-tile items)
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=hq, Hkv=1, N=2048, bs=bs, kb=3)
    _prefill_case(w, gated=False)
    _prefill_case(w, gated=True)


@pytest.mark.parametrize("kb", [4, 5])
def test_prefill_gqa_bf16_small(kb):
    # 32 blocks, kept lists of odd and even length, two 128-row tiles per CTA
    w = W.get("prefill_gqa_bf16").scaled(Hq=8, Hkv=2, N=2048, kb=kb)
    _prefill_case(w, gated=False)


def test_gated_bf16_small_group_of_seven():
    # G = 7 heads x 128 rows: seven tiles per unit, an odd count (one-tile-per-item kernel)
    w = W.get("gated_prefill_bf16").scaled(B=1, Hq=7, Hkv=1, N=2048, kb=3)
    _prefill_case(w, gated=True)


def test_gated_bf16_small_gqa():
    w = W.get("gated_prefill_bf16").scaled(B=2, Hq=8, Hkv=2, N=1024, kb=2)
    _prefill_case(w, gated=True)


def test_prefill_bf16_block128_ungated():
    w = W.get("gated_prefill_bf16").scaled(B=1, Hq=4, Hkv=2, N=2048, kb=4, kind="prefill")
    _prefill_case(w, gated=False)


@pytest.mark.parametrize("kernel", [1, 2, 3])
@pytest.mark.parametrize("hq,bs,gated", [(4, 64, False), (5, 64, True), (7, 128, True), (3, 64, False)])
def test_prefill_every_kernel_matches_the_oracle(kernel, hq, bs, gated):
    """Each bf16 prefill kernel, forced through the testing hook (1 paired
    tiles, 2 one tile per SM, 3 SM pair with MMAs of M = 256), on even and
    odd tile counts per unit, ungated and gated, with odd and even kept lists."""
    bsa = _bsa()
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=hq, Hkv=1, N=4096, bs=bs, kb=5)
    prev = bsa.bsa_prefill_kernel_override(kernel)
    try:
        _prefill_case(w, gated=gated)
    finally:
        bsa.bsa_prefill_kernel_override(prev)


def test_sm_pair_prefill_full_budget_and_empty_lists():
    """The SM-pair kernel on the longest lists (dense causal at full budget)
    and with emptied lists between items."""
    bsa = _bsa()
    prev = bsa.bsa_prefill_kernel_override(3)
    try:
        _prefill_case(W.get("prefill_gqa_bf16").scaled(B=1, Hq=4, Hkv=1, N=8192, kb=127), gated=True)
        _prefill_case(W.get("gated_prefill_bf16").scaled(B=2, Hq=14, Hkv=2, N=4096, kb=8), gated=True)
    finally:
        bsa.bsa_prefill_kernel_override(prev)


def _sample_rows(w: W.Workload, n: int, seed: int):
    r = np.random.default_rng(seed)
    b = r.integers(0, w.B, n)
    h = r.integers(0, w.Hq, n)
    t = r.integers(0, w.N, n)
    t[:4] = [0, w.bs - 1, w.N - 1, w.N - w.bs]   # first / last rows of the first and last blocks
    return (b * w.Hq + h) * w.N + t


def test_prefill_gqa_bf16_full_size_sampled():
    w = W.get("prefill_gqa_bf16")
    _prefill_case(w, gated=False, rows_sample=_sample_rows(w, 96, 1))


def test_gated_bf16_full_size_sampled():
    w = W.get("gated_prefill_bf16")
    _prefill_case(w, gated=True, rows_sample=_sample_rows(w, 96, 3))


@pytest.mark.parametrize("fp32_d", [128])
@pytest.mark.parametrize("gated", [False, True])
def test_tiny_prefill_f32_head_dim_128(fp32_d, gated):
    # the fp32 path at the other head dimension it is built for
    w = W.get("tiny_prefill_f32").scaled(d=fp32_d)
    _prefill_case(w, gated)


# Budgets at or above the number of history blocks: every block j <= i is
# kept, so the sparse result must be dense causal attention (the tutorial's
# softmax(QK^T/sqrt(d))V with the causal mask, §1).  These runs also reach the
# longest kept lists the prefill kernels take.
@pytest.mark.parametrize("hq,gated", [(4, False), (4, True), (5, False), (5, True)])
def test_prefill_bf16_full_budget_dense_causal(hq, gated):
    # G 4: 256 stacked rows, two tiles (paired kernel); G 5: 320 rows, three
    # tiles (one-tile-per-item kernel).  128 blocks, budget 127 + current.
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=hq, Hkv=1, N=8192, kb=127)
    _prefill_case(w, gated=gated)


def test_gated_bf16_block128_full_budget_group_of_seven():
    # 128-token blocks, G 7 (seven tiles per unit), 64 blocks, budget 63 + current
    w = W.get("gated_prefill_bf16").scaled(B=1, Hq=7, Hkv=1, N=8192, kb=63)
    _prefill_case(w, gated=True)


def test_prefill_bf16_longest_lists():
    """256 blocks with budget 255 + current: kept lists of up to 256 entries,
    the longest the prefill entry points accept (idx_stride <= 256)."""
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=4, Hkv=1, N=16384, kb=255)
    _prefill_case(w, gated=False)


def test_prefill_full_budget_equals_dense_causal_closed_form():
    """The closed form itself, on the GPU output: at full budget the sparse
    prefill equals dense causal attention computed as one fp64 softmax over
    every earlier token (no index list involved)."""
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=4, Hkv=1, N=2048, kb=31)
    pipe = _pipe()
    inp = W.make_inputs(w, "cuda")
    step = pipe.PrefillStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
    step.run()
    torch.cuda.synchronize()
    _status_clean()
    q = inp["q"].double().cpu()[0]
    k = inp["k"].double().cpu()[0, 0]
    v = inp["v"].double().cpu()[0, 0]
    logits = torch.einsum("htd,ud->htu", q, k) / np.sqrt(w.d)
    causal = torch.ones(w.N, w.N, dtype=torch.bool).tril()
    logits = logits.masked_fill(~causal, float("-inf"))
    want = torch.softmax(logits, dim=-1) @ v
    _assert_close(step.bufs["o"][0].float().cpu().numpy(), want.numpy(), TOL_BF16, "dense causal")


def test_prefill_empty_and_bad_lists():
    """A query block with an empty list gives zero rows and LSE -inf; an entry
    in the future (> i) is skipped and flagged, never read."""
    bsa = _bsa()
    pipe = _pipe()
    w = W.get("prefill_gqa_bf16").scaled(Hq=4, Hkv=1, N=512, kb=2)
    inp = W.make_inputs(w, "cuda")
    step = pipe.PrefillStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
    step.select()
    idx = step.bufs["idx"].clone()
    a = int(idx[0, 0, 5, 0].item())
    idx[0, 0, 3, :] = -1                                                   # empty list
    idx[0, 0, 5, :] = torch.tensor([a, 7, -1], dtype=torch.int32)          # 7 > 5: future block
    good = idx.clone()
    good[0, 0, 5, :] = torch.tensor([a, -1, -1], dtype=torch.int32)
    bsa.bsa_device_status(reset=True)
    step.attend(idx=idx)
    code, flags = bsa.bsa_device_status(reset=True)
    assert flags & 2, "bad index not flagged"
    o_bad = step.bufs["o"].clone()
    lse_bad = step.bufs["lse"].clone()
    # block 3 rows are zero with LSE -inf
    assert torch.all(o_bad[0, :, 3 * w.bs:4 * w.bs] == 0)
    assert torch.all(torch.isneginf(lse_bad[0, :, 3 * w.bs:4 * w.bs]))
    # block 5 equals the run without the bad entry
    step.attend(idx=good)
    torch.cuda.synchronize()
    assert torch.equal(o_bad[0, :, 5 * w.bs:6 * w.bs], step.bufs["o"][0, :, 5 * w.bs:6 * w.bs])
    _status_clean()


@pytest.mark.parametrize("hq,gated", [(10, False), (10, True), (8, False)])
def test_prefill_empty_lists_between_items(hq, gated):
    """Empty kept lists on a seeded half of the query blocks, with enough
    units that every persistent CTA walks several items, so items without
    keys sit between items with keys (G 5: three 128-row tiles per unit, the
    one-tile-per-item kernel; G 4: two tiles, the paired kernel).  Both sides
    get the oracle's index set with the same lists emptied; every output row
    is compared, the emptied blocks' rows are exactly zero with LSE -inf."""
    pipe = _pipe()
    w = W.get("prefill_gqa_bf16").scaled(B=1, Hq=hq, Hkv=2, N=8192, kb=3)
    inp = W.make_inputs(w, "cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    step = pipe.PrefillStep(q, k, v, w.bs, w.kb, gated=gated)
    step.select()
    qc, kc, vc = q.float().cpu(), k.float().cpu(), v.float().cpu()
    _, _, s, idx, _ = oracle.prefill_select(qc, kc, w.Hkv, w.bs, w.kb)
    nb = w.N // w.bs
    empty = np.random.default_rng(11).random((w.Hkv, nb)) < 0.5
    idx = idx.copy()
    idx[0][empty] = -1
    step.attend(idx=torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    _status_clean()
    want, want_lse = oracle.attend_prefill(qc, kc, vc, w.bs, idx, gate_scores=s if gated else None)
    got = step.bufs["o"].float().reshape(-1, w.d).cpu().numpy()
    got_lse = step.bufs["lse"].reshape(-1).cpu().numpy().astype(np.float64)
    _assert_close(got, want, TOL_BF16, "out")
    fin = np.isfinite(want_lse)
    assert (~fin).sum() > 0 and np.array_equal(np.isneginf(got_lse), ~fin), "LSE -inf rows differ"
    _assert_close(got_lse[fin], want_lse[fin], dict(max_abs=2e-3, mean_abs=2e-4), "lse")
    assert np.all(got[~fin] == 0.0), "rows of emptied blocks are not zero"


# ----------------------------------------------------------------------------
# top-k selection on crafted scores (ties, NaN, budgets)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [0, 1, 2])
def test_topk_ties_nan_and_budgets(mode):
    bsa = _bsa()
    r = np.random.default_rng(100 + mode)
    for ncols in (1, 7, 33, 300, 2048):
        for kb in (0, 1, 5, 64, ncols + 3):
            rows = 9
            s = r.integers(-4, 5, size=(rows, ncols)).astype(np.float32)
            s[0, ::3] = np.nan
            s[1, :] = 0.0
            s[2, ::2] = -np.inf
            s[3, 1::2] = -0.0
            forced = 0 if mode == 2 else 1
            stride = kb + forced + 2
            want, cnt = oracle.topk(s, mode, kb, idx_stride=stride)
            sd = torch.from_numpy(s).cuda()
            idx = torch.empty((rows, stride), dtype=torch.int32, device="cuda")
            count = torch.empty((rows,), dtype=torch.int32, device="cuda")
            bsa.bsa_topk_select(sd, rows, ncols, mode, kb, idx, stride, count)
            torch.cuda.synchronize()
            assert np.array_equal(idx.cpu().numpy(), want), (ncols, kb)
            assert np.array_equal(count.cpu().numpy(), cnt)


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------

def _decode_case(w: W.Workload, groups=None):
    """groups: list of (b, g) to check (default: all)."""
    pipe = _pipe()
    inp = W.make_inputs(w, "cuda")
    q, kc, vc = inp["q"], inp["k"], inp["v"]
    step = pipe.DecodeStep(q, kc, vc, w.bs, w.kb)
    step.pool_cache()
    step.select()
    torch.cuda.synchronize()
    b_ = step.bufs
    G = w.G
    if groups is None:
        groups = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    idx_all = b_["idx"].cpu().numpy()
    oracle_idx = idx_all.copy()
    for (b, g) in groups:
        ks = kc[b:b + 1, g:g + 1].float().cpu()
        qs = q[b:b + 1, g * G:(g + 1) * G].float().cpu()
        kbar = oracle.pool_keys(ks, w.bs)
        assert np.array_equal(b_["kbar"][b:b + 1, g:g + 1].cpu().numpy(), kbar), (b, g)
        _, s, idx, cnt = oracle.decode_select(qs, kbar, 1, w.kb)
        assert np.array_equal(b_["scores"][b, g].cpu().numpy(), s[0, 0]), (b, g)
        assert np.array_equal(idx_all[b, g], idx[0, 0]), (b, g)
        oracle_idx[b, g] = idx[0, 0]
    step.attend(idx=torch.from_numpy(oracle_idx).cuda())
    torch.cuda.synchronize()
    _status_clean()
    for (b, g) in groups:
        ks = kc[b:b + 1, g:g + 1].float().cpu()
        vs = vc[b:b + 1, g:g + 1].float().cpu()
        qs = q[b:b + 1, g * G:(g + 1) * G].float().cpu()
        want, want_lse = oracle.attend_decode(qs, ks, vs, w.bs, oracle_idx[b:b + 1, g:g + 1])
        got = b_["o"][b, g * G:(g + 1) * G].float().cpu().numpy()
        _assert_close(got, want, TOL_BF16, f"{w.name} decode ({b},{g})")
        _assert_close(b_["lse"][b, g * G:(g + 1) * G].cpu().numpy(), want_lse,
                      dict(max_abs=2e-3, mean_abs=2e-4), "decode lse")


@pytest.mark.parametrize("nb,kb,d,dtype", [(128, 12, 128, "bf16"), (200, 17, 128, "bf16"), (2048, 96, 128, "bf16"),
                                          (1, 3, 128, "bf16"), (129, 0, 128, "bf16"), (300, 400, 128, "bf16"),
                                          (256, 20, 128, "f32"), (96, 7, 64, "bf16"), (2500, 30, 128, "bf16")])
def test_decode_select_one_call_equals_score_then_topk(nb, kb, d, dtype):
    """bsa_decode_select (one kernel for d 128 and up to 2048 blocks, the two
    kernels otherwise) gives the bits of bsa_score_blocks(DECODE) followed by
    bsa_topk_select(LAST_BLOCK), and the oracle's scores and kept blocks:
    ragged last chunks (200, 129, 300 blocks), one block, budget 0 and a
    budget above the candidates, fp32 queries, d 64 and 2500 blocks (the two
    kernel path)."""
    bsa = _bsa()
    B, Hq, Hkv, bs = 2, 8, 2, 64
    g = torch.Generator(device="cuda").manual_seed(nb * 7 + kb)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.randn((B, Hq, d), generator=g, device="cuda").to(tdt)
    kbar = torch.randn((B, Hkv, nb, d), generator=g, device="cuda")
    shape = bsa.make_shape(B, Hq, Hkv, 1, nb * bs, d, bs, tdt)
    stride = kb + 3
    outs = []
    for fused in (True, False):
        sc = torch.full((B, Hkv, nb), float("nan"), device="cuda")
        qb = torch.full((B, Hkv, d), float("nan"), device="cuda")
        idx = torch.full((B, Hkv, stride), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
        if fused:
            bsa.bsa_decode_select(shape, q, kbar, kb, sc, idx, stride, pooled_q_out=qb, count_out=cnt)
        else:
            bsa.bsa_score_blocks(shape, bsa.BSA_SCORE_DECODE, q, None, kbar, qb, None, sc)
            bsa.bsa_topk_select(sc, B * Hkv, nb, bsa.BSA_TOPK_LAST_BLOCK, kb, idx, stride, cnt)
        torch.cuda.synchronize()
        outs.append((sc.cpu().numpy(), qb.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()))
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b)
    qbar, s, want_idx, want_cnt = oracle.decode_select(q.float().cpu(), kbar.cpu(), Hkv, kb)
    assert np.array_equal(outs[0][0], s)
    assert np.array_equal(outs[0][1], qbar)
    assert np.array_equal(outs[0][2][..., :want_idx.shape[-1]], want_idx)
    assert np.all(outs[0][2][..., want_idx.shape[-1]:] == -1)
    assert np.array_equal(outs[0][3], want_cnt)
    _status_clean()


def test_decode_bf16_small():
    w = W.get("decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=12)
    _decode_case(w)


def test_decode_bf16_small_even_list_and_full_budget():
    w = W.get("decode_bf16").scaled(B=1, Hq=4, Hkv=1, N=4096, kb=63)   # every block kept
    _decode_case(w)


def test_decode_bf16_full_size_every_row():
    """The full decode workload (16 sequences x 131072 cached tokens): pooled
    keys, scores and kept indices of all 128 (sequence, group) rows compared
    bit for bit, and the outputs of all 512 query heads against the oracle,
    one sequence at a time on the host."""
    pipe = _pipe()
    w = W.get("decode_bf16")
    inp = W.make_inputs(w, "cuda")
    q, kc, vc = inp["q"], inp["k"], inp["v"]
    step = pipe.DecodeStep(q, kc, vc, w.bs, w.kb)
    step.pool_cache()
    step.select()
    torch.cuda.synchronize()
    b_ = step.bufs
    idx_gpu = b_["idx"].cpu().numpy()
    oracle_idx = np.empty_like(idx_gpu)
    for b in range(w.B):
        kbar = oracle.pool_keys(kc[b:b + 1].float().cpu(), w.bs)
        assert np.array_equal(b_["kbar"][b:b + 1].cpu().numpy(), kbar), b
        _, s, idx, _ = oracle.decode_select(q[b:b + 1].float().cpu(), kbar, w.Hkv, w.kb)
        assert np.array_equal(b_["scores"][b:b + 1].cpu().numpy(), s), b
        assert np.array_equal(idx_gpu[b:b + 1], idx), b
        oracle_idx[b] = idx[0]
    step.attend(idx=torch.from_numpy(oracle_idx).cuda())
    torch.cuda.synchronize()
    _status_clean()
    got = b_["o"].float().cpu().numpy()
    got_lse = b_["lse"].cpu().numpy()
    for b in range(w.B):
        want, want_lse = oracle.attend_decode(q[b:b + 1].float().cpu(), kc[b:b + 1].float().cpu(),
                                              vc[b:b + 1].float().cpu(), w.bs, oracle_idx[b:b + 1])
        _assert_close(got[b], want, TOL_BF16, f"decode sequence {b}")
        _assert_close(got_lse[b], want_lse, dict(max_abs=2e-3, mean_abs=2e-4), f"decode lse {b}")


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (16, 2), (32, 2)])
def test_decode_group_widths(hq, hkv):
    # G = 1, 2, 8, 16 query heads per KV group (the softmax is specialised on
    # the padded group width 4 / 8 / 16)
    w = W.get("decode_bf16").scaled(B=1, Hq=hq, Hkv=hkv, N=4096, kb=10)
    _decode_case(w)


def test_decode_split_count_invariance():
    bsa = _bsa()
    pipe = _pipe()
    w = W.get("decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=40)
    inp = W.make_inputs(w, "cuda")
    outs = []
    for splits in (1, 3, 7, 0):
        prev = bsa.bsa_decode_split_override(splits)
        try:
            step = pipe.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
            step.pool_cache()
            step.run()
            torch.cuda.synchronize()
            outs.append(step.bufs["o"].float().cpu())
        finally:
            bsa.bsa_decode_split_override(prev)
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 1e-2
    _status_clean()


def test_bounded_wait_expiry_reports_timeout_and_leaves_the_device_usable():
    """The bounded-wait expiry path: a self-test kernel waits, through the
    same helper every kernel uses, on a barrier nothing arrives on, with a
    budget of 1e5 cycles.  It returns, the status word reports a timeout, a
    reset clears it, and a following real call runs clean."""
    bsa = _bsa()
    pipe = _pipe()
    bsa.bsa_device_status(reset=True)
    bsa.bsa_selftest_wait_expiry(100_000)
    code, flags = bsa.bsa_device_status(reset=True)
    assert code == bsa.BSA_ERR_TIMEOUT and flags & 1, (code, flags)
    code, flags = bsa.bsa_device_status(reset=False)
    assert code == 0 and flags == 0
    w = W.get("decode_bf16").scaled(B=1, Hq=8, Hkv=2, N=4096, kb=6)
    inp = W.make_inputs(w, "cuda")
    step = pipe.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
    step.pool_cache()
    step.run()
    torch.cuda.synchronize()
    assert torch.isfinite(step.bufs["o"].float()).all()
    _status_clean()


def test_decode_and_gist_graph_replay_match_eager():
    """The decode and gist steps captured into CUDA graphs (as the benchmark
    replays them) give the same bytes as the eager C-ABI calls."""
    pipe = _pipe()
    w = W.get("decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=24)
    inp = W.make_inputs(w, "cuda")
    step = pipe.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
    step.pool_cache()
    step.run()
    torch.cuda.synchronize()
    eager = {k: step.bufs[k].clone() for k in ("scores", "idx", "o", "lse")}
    for k in ("scores", "o", "lse"):
        step.bufs[k].zero_()
    step.bufs["idx"].fill_(-7)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        step.run()
    g.replay()
    torch.cuda.synchronize()
    for k, v in eager.items():
        assert torch.equal(step.bufs[k], v), k
    wg = W.get("gist_decode_bf16").scaled(B=1, Hq=8, Hkv=2, N=8192, kb=6)
    ig = W.make_inputs(wg, "cuda")
    gs = pipe.GistStep(ig["q"], ig["k"], ig["v"], ig["gk"], ig["gv"], wg.bs, wg.kb)
    gs.run()
    torch.cuda.synchronize()
    o_eager = gs.bufs["o"].clone()
    gs.bufs["o"].zero_()
    gg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gg, capture_error_mode="thread_local"):
        gs.run()
    gg.replay()
    torch.cuda.synchronize()
    assert torch.equal(gs.bufs["o"], o_eager)
    del g, gg
    _status_clean()


# ----------------------------------------------------------------------------
# gist selective expansion (SSA)
# ----------------------------------------------------------------------------

def _gist_case(w: W.Workload, groups=None, topk=None):
    pipe = _pipe()
    inp = W.make_inputs(w, "cuda")
    topk = w.kb if topk is None else topk
    G = w.G
    nc = w.N // w.bs
    step = pipe.GistStep(inp["q"], inp["k"], inp["v"], inp["gk"], inp["gv"], w.bs, topk)
    step.run()
    torch.cuda.synchronize()
    _status_clean()
    if groups is None:
        groups = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    for (b, g) in groups:
        qs = inp["q"][b:b + 1, g * G:(g + 1) * G].float().cpu()
        gks = inp["gk"][b:b + 1, g:g + 1].float().cpu()
        gvs = inp["gv"][b:b + 1, g:g + 1].float().cpu()
        ks = inp["k"][b:b + 1, g:g + 1].float().cpu()
        vs = inp["v"][b:b + 1, g:g + 1].float().cpu()
        s, idx, _ = oracle.gist_select(qs, gks, topk)
        if topk > 0:
            assert np.array_equal(step.bufs["idx"][b, g * G:(g + 1) * G, :topk].cpu().numpy(), idx[0]), (b, g)
        else:
            idx = np.full((1, G, 1), -1, np.int32)
        want, want_lse = oracle.attend_gist(qs, ks, vs, gks, gvs, w.bs, idx)
        got = step.bufs["o"][b, g * G:(g + 1) * G].float().cpu().numpy()
        _assert_close(got, want, TOL_BF16, f"gist ({b},{g}) topk={topk}")
        _assert_close(step.bufs["lse"][b, g * G:(g + 1) * G].cpu().numpy(), want_lse,
                      dict(max_abs=2e-3, mean_abs=2e-4), "gist lse")


def test_gist_bf16_small():
    w = W.get("gist_decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=8)
    _gist_case(w)


@pytest.mark.parametrize("topk", [0, 1, 128])
def test_gist_bf16_edge_budgets(topk):
    w = W.get("gist_decode_bf16").scaled(B=1, Hq=4, Hkv=1, N=8192, kb=topk)
    _gist_case(w, topk=topk)


@pytest.mark.parametrize("hq,hkv,nc", [(8, 2, 2048), (6, 2, 128), (7, 1, 96), (2, 2, 64), (32, 2, 256)])
def test_gist_scores_bit_exact(hq, hkv, nc):
    """The gist scores themselves (SSA page, 推理时的关键模块 1: the query
    against every chunk's gist key), fixed-order fp32, bit for bit against the
    oracle for several group widths (odd ones leave one head of a pair empty)
    and gist counts (a partial last tile of 64)."""
    bsa = _bsa()
    g = torch.Generator(device="cuda").manual_seed(31)
    B, d = 2, 128
    q = torch.randn((B, hq, d), generator=g, device="cuda").to(torch.bfloat16)
    gk = torch.randn((B, hkv, nc, d), generator=g, device="cuda").to(torch.bfloat16)
    scores = torch.empty((B, hq, nc), dtype=torch.float32, device="cuda")
    shape = bsa.make_shape(B, hq, hkv, 1, nc * 64, d, 64, torch.bfloat16)
    bsa.bsa_score_blocks(shape, bsa.BSA_SCORE_GIST, q, gk, None, None, None, scores)
    torch.cuda.synchronize()
    _status_clean()
    want = oracle.scores_gist(q.float().cpu(), gk.float().cpu())
    assert np.array_equal(scores.cpu().numpy(), want)


@pytest.mark.parametrize("hq,hkv", [(2, 2), (6, 2), (7, 1), (16, 2), (32, 2)])
def test_gist_group_widths(hq, hkv):
    w = W.get("gist_decode_bf16").scaled(B=1, Hq=hq, Hkv=hkv, N=8192, kb=5)
    _gist_case(w)


def test_gist_union_kernel_above_2048_chunks():
    """Above 2048 chunks per row the union of the heads' expanded chunks is
    built by its own kernel instead of inside the attention kernel: 4096
    chunks, two groups of widths 3."""
    w = W.get("gist_decode_bf16").scaled(B=1, Hq=6, Hkv=2, N=4096 * 64, kb=9)
    _gist_case(w)


def test_gist_injected_lists_with_padding_and_repeats():
    """Injected per-head lists with -1 padding, a chunk kept by every head and
    a head that expands nothing: the union and the per-head masks built in the
    attention kernel."""
    pipe = _pipe()
    w = W.get("gist_decode_bf16").scaled(B=1, Hq=4, Hkv=1, N=8192, kb=4)
    inp = W.make_inputs(w, "cuda")
    idx = torch.tensor([[[3, 40, 127, -1], [3, 4, -1, -1], [-1, -1, -1, -1], [0, 3, 64, 126]]],
                       dtype=torch.int32, device="cuda")
    step = pipe.GistStep(inp["q"], inp["k"], inp["v"], inp["gk"], inp["gv"], w.bs, 4)
    step.run(idx_in=idx)
    torch.cuda.synchronize()
    want, _ = oracle.attend_gist(inp["q"].float().cpu(), inp["k"].float().cpu(), inp["v"].float().cpu(),
                                 inp["gk"].float().cpu(), inp["gv"].float().cpu(), w.bs, idx.cpu().numpy())
    _assert_close(step.bufs["o"][0].float().cpu().numpy(), want, TOL_BF16, "gist padded lists")
    _status_clean()


def test_gist_bf16_full_size_every_group():
    """The full gist workload (8 sequences x 131072 tokens, 2048 gists): the
    chosen chunks of all 256 query heads compared exactly, and the outputs of
    all 256 heads against the oracle, one sequence at a time on the host."""
    pipe = _pipe()
    w = W.get("gist_decode_bf16")
    inp = W.make_inputs(w, "cuda")
    step = pipe.GistStep(inp["q"], inp["k"], inp["v"], inp["gk"], inp["gv"], w.bs, w.kb)
    step.run()
    torch.cuda.synchronize()
    _status_clean()
    got_idx = step.bufs["idx"].cpu().numpy()
    got = step.bufs["o"].float().cpu().numpy()
    got_lse = step.bufs["lse"].cpu().numpy()
    for b in range(w.B):
        qs = inp["q"][b:b + 1].float().cpu()
        gks = inp["gk"][b:b + 1].float().cpu()
        _, idx, _ = oracle.gist_select(qs, gks, w.kb)
        assert np.array_equal(got_idx[b:b + 1], idx), b
        want, want_lse = oracle.attend_gist(qs, inp["k"][b:b + 1].float().cpu(), inp["v"][b:b + 1].float().cpu(),
                                            gks, inp["gv"][b:b + 1].float().cpu(), w.bs, idx)
        _assert_close(got[b], want, TOL_BF16, f"gist sequence {b}")
        _assert_close(got_lse[b], want_lse, dict(max_abs=2e-3, mean_abs=2e-4), f"gist lse {b}")


def test_gist_injected_index_set():
    """idx_in bypasses scoring/selection: the given chunks are expanded."""
    pipe = _pipe()
    w = W.get("gist_decode_bf16").scaled(B=1, Hq=4, Hkv=1, N=8192, kb=3)
    inp = W.make_inputs(w, "cuda")
    idx = torch.tensor([[[0, 5, 127], [1, 2, 3], [7, 64, 100], [0, 1, 2]]], dtype=torch.int32, device="cuda")
    step = pipe.GistStep(inp["q"], inp["k"], inp["v"], inp["gk"], inp["gv"], w.bs, 3)
    step.run(idx_in=idx)
    torch.cuda.synchronize()
    want, _ = oracle.attend_gist(inp["q"].float().cpu(), inp["k"].float().cpu(), inp["v"].float().cpu(),
                                 inp["gk"].float().cpu(), inp["gv"].float().cpu(), w.bs, idx.cpu().numpy())
    _assert_close(step.bufs["o"][0].float().cpu().numpy(), want, TOL_BF16, "gist injected")
    _status_clean()


# ----------------------------------------------------------------------------
# host-side argument checks (nothing is launched when they fail)
# ----------------------------------------------------------------------------

def test_invalid_arguments_rejected():
    bsa = _bsa()
    q = torch.zeros((1, 4, 256, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 256, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    idx = torch.zeros((1, 1, 4, 3), dtype=torch.int32, device="cuda")
    bad_g = bsa.make_shape(1, 4, 3, 256, 256, 128, 64, torch.bfloat16)   # Hq % Hkv != 0
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_sparse_attn_prefill(bad_g, q, k, k, idx, 3, 0.1, o)
    assert e.value.code == 1
    bad_block = bsa.make_shape(1, 4, 1, 256, 256, 128, 32, torch.bfloat16)  # block 32 not built
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_sparse_attn_prefill(bad_block, q, k, k, idx, 3, 0.1, o)
    assert e.value.code == 2
    good = bsa.make_shape(1, 4, 1, 256, 256, 128, 64, torch.bfloat16)
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_sparse_attn_prefill(good, q, k, k, idx, 3, -1.0, o)   # bad scale
    assert e.value.code == 1
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_topk_select(torch.zeros((2, 8), device="cuda"), 2, 8, 0, 4, idx, 3)   # stride < kb+1
    assert e.value.code == 1
    _status_clean()
