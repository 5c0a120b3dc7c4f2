"""Host-side logic: work accounting against the pages' figures and the
oracle's mask, and the seeded workload generator."""
import os

import numpy as np
import pytest
import torch

import bsa_workloads as W
import oracle
from top_block_sparse_bsa_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_numbers():
    vals = {}
    for line in open(os.path.join(GOLDEN, "pair_counts.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def test_dense_pair_counts_from_tutorial():
    g = _golden_numbers()
    assert acc.dense_pairs(4) == g["dense_pairs_4"]
    assert abs(acc.dense_pairs(128000) - g["dense_pairs_128000_approx"]) / g["dense_pairs_128000_approx"] < 0.01


def test_sparsity_definition_from_review():
    g = _golden_numbers()
    assert acc.sparsity(g["sparsity_095_kept_fraction"], 1.0) == pytest.approx(0.95)
    # decode workload: 96 history blocks + the last block out of 2048
    w = W.get("decode_bf16")
    assert acc.sparsity(w.kb + 1, w.nb) == pytest.approx(0.95264, abs=1e-5)


def test_prefill_pairs_equal_the_oracle_mask_count():
    r = np.random.default_rng(0)
    for kb in (0, 2, 100):
        q = r.standard_normal((1, 4, 256, 16)).astype(np.float32)
        k = r.standard_normal((1, 2, 256, 16)).astype(np.float32)
        bs = 32
        _, _, _, idx, _ = oracle.prefill_select(q, k, 2, bs, kb)
        want = sum(int(oracle.prefill_mask(256, bs, idx[0, g]).sum()) for g in range(2)) * 2   # G = 2
        assert acc.prefill_pairs(idx, bs, G=2) == want
    # full budget = dense causal pairs per head
    _, _, _, idx, _ = oracle.prefill_select(q, k, 2, 32, 100)
    assert acc.prefill_pairs(idx, 32, 2) == acc.dense_pairs(256, causal=True) * 4


def test_decode_bytes_closed_form():
    w = W.get("decode_bf16")
    idx = np.tile(np.arange(w.kb + 1, dtype=np.int32), (w.B, w.Hkv, 1))
    assert acc.decode_kv_bytes(idx, w.bs, w.d, 2) == w.B * w.Hkv * (w.kb + 1) * w.bs * w.d * 2 * 2
    assert acc.decode_kv_bytes(idx, w.bs, w.d, 2) == 406_847_488


def test_gist_accounting():
    w = W.get("gist_decode_bf16")
    nc = w.N // w.bs
    idx = np.zeros((1, 4, w.kb), np.int32)
    idx[0, 0] = np.arange(w.kb)
    idx[0, 1] = np.arange(w.kb)
    idx[0, 2] = np.arange(w.kb) + w.kb
    idx[0, 3] = np.arange(w.kb) + 2 * w.kb
    assert acc.gist_union_chunks(idx, G=4) == 3 * w.kb
    assert acc.gist_pairs(idx[:, :1], w.bs, nc) == w.kb * w.bs + nc - w.kb == 4064


def test_pair_counts_of_a_tiny_block_pattern():
    # the tutorial's 4-block example at bs = 2: Q3 sees {K2,K3}, Q4 sees {K1,K3,K4}
    idx = np.array([[[[0, -1, -1], [0, 1, -1], [1, 2, -1], [0, 2, 3]]]], np.int32)
    assert acc.prefill_pairs(idx, 2, 1) == int(oracle.prefill_mask(8, 2, idx[0, 0]).sum())


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_workload_shapes_and_determinism(name):
    w = W.get(name)
    small = w.scaled(B=1, N=w.bs * 4, Hq=w.G, Hkv=1)
    a = W.make_inputs(small, "cpu")
    b = W.make_inputs(small, "cpu")
    for key in a:
        assert torch.equal(a[key], b[key]), key
        assert a[key].dtype == w.torch_dtype
    if w.kind in ("prefill", "gated"):
        assert a["q"].shape == (1, w.G, w.bs * 4, w.d)
        assert a["k"].shape == (1, 1, w.bs * 4, w.d)
    else:
        assert a["q"].shape == (1, w.G, w.d)
    if w.kind == "gist":
        assert a["gk"].shape == (1, 1, 4, w.d)
