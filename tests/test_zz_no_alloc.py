"""The allocation-free decode entry point (bsa_sparse_attn_decode_noalloc).

It exists for callers that cannot allocate device memory -- a server that
reserves all its memory at start-up, a plugin whose host framework owns every
buffer -- and so cannot hand the decode a scratch workspace.  It must give the
same result as bsa_sparse_attn_decode with a caller workspace, call after
call, while the library's built-in scratch array keeps the previous call's
contents.  This file is collected last on purpose.
"""
import math

import numpy as np
import pytest
import torch

import bsa_workloads as W

pytestmark = pytest.mark.gpu

TOL = dict(max_abs=2e-2, mean_abs=2e-3)


def _close(a, b):
    err = (a.float() - b.float()).abs()
    assert torch.isfinite(a.float()).all()
    assert err.max().item() <= TOL["max_abs"] and err.mean().item() <= TOL["mean_abs"]


def test_noalloc_decode_matches_workspace_decode_twice():
    import top_block_sparse_bsa_b200 as bsa
    from top_block_sparse_bsa_b200 import pipeline
    torch.cuda.set_device(0)
    for seed, kb in ((2, 12), (7, 30)):
        w = W.get("decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=kb, seed=seed)
        inp = W.make_inputs(w, "cuda")
        step = pipeline.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
        step.pool_cache()
        step.run()
        torch.cuda.synchronize()
        want_o = step.bufs["o"].clone()
        want_lse = step.bufs["lse"].clone()
        idx = step.bufs["idx"]
        scale = 1.0 / math.sqrt(w.d)
        for _ in range(2):   # two calls in a row share the built-in scratch
            o = torch.full_like(want_o, float("nan"))
            lse = torch.full_like(want_lse, float("nan"))
            bsa.bsa_sparse_attn_decode_noalloc(step.shape, inp["q"], inp["k"], inp["v"], idx, idx.shape[-1],
                                               scale, o, lse)
            torch.cuda.synchronize()
            _close(o, want_o)
            assert torch.allclose(lse, want_lse, atol=2e-3, rtol=0)
    code, flags = bsa.bsa_device_status(reset=True)
    assert code == 0 and flags == 0


def test_noalloc_decode_after_a_call_with_another_split_layout():
    """Stale partial records: a call with many split ranges (the scratch laid
    out with more slots per row) runs first, then calls with the default
    plan read the same array.  Each result must still equal the workspace
    decode run with the same plan."""
    import top_block_sparse_bsa_b200 as bsa
    from top_block_sparse_bsa_b200 import pipeline
    torch.cuda.set_device(0)
    w = W.get("decode_bf16").scaled(B=2, Hq=8, Hkv=2, N=8192, kb=40, seed=5)
    inp = W.make_inputs(w, "cuda")
    scale = 1.0 / math.sqrt(w.d)
    for splits in (61, 0, 7):
        prev = bsa.bsa_decode_split_override(splits)
        try:
            step = pipeline.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
            step.pool_cache()
            step.run()
            torch.cuda.synchronize()
            idx = step.bufs["idx"]
            o = torch.full_like(step.bufs["o"], float("nan"))
            lse = torch.full_like(step.bufs["lse"], float("nan"))
            bsa.bsa_sparse_attn_decode_noalloc(step.shape, inp["q"], inp["k"], inp["v"], idx, idx.shape[-1],
                                               scale, o, lse)
            torch.cuda.synchronize()
            assert torch.equal(o, step.bufs["o"]), splits
            assert torch.equal(lse, step.bufs["lse"]), splits
        finally:
            bsa.bsa_decode_split_override(prev)
    code, flags = bsa.bsa_device_status(reset=True)
    assert code == 0 and flags == 0


def test_noalloc_decode_rejects_shapes_beyond_its_scratch():
    import top_block_sparse_bsa_b200 as bsa
    torch.cuda.set_device(0)
    # 64 sequences x 64 query heads need far more than the built-in 4 MiB of partials
    shape = bsa.make_shape(64, 64, 8, 1, 1 << 20, 128, 64, torch.bfloat16)
    assert bsa.bsa_workspace_bytes(bsa.BSA_OP_DECODE, shape, 4097) > (4 << 20)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_sparse_attn_decode_noalloc(shape, dummy, dummy, dummy, idx, 4097, 0.1, dummy)
    assert e.value.code == bsa.BSA_ERR_UNSUPPORTED
