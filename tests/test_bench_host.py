"""Host-side logic of bench.py that needs no GPU: which prefill kernel (and
so which committed ncu summary) a workload's shape selects."""
from __future__ import annotations

import importlib.util
import os

import bsa_workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_prefill_kernel_follows_the_tile_count():
    b = _bench()
    # G*bs rows per unit: 4*64 = 256 (two tiles) -> paired; 7*128 = 896 (seven) -> split
    assert b.prefill_kernel_of(W.get("prefill_gqa_bf16"))[0] == "attn_prefill.cu"
    assert b.prefill_kernel_of(W.get("gated_prefill_bf16"))[0] == "attn_prefill_split.cu"
    assert b.prefill_kernel_of(W.get("tiny_prefill_f32"))[0] == "attn_f32.cu"
    base = W.get("prefill_gqa_bf16")
    for hq, bs, want in ((1, 64, "split"), (3, 64, "paired"), (5, 64, "split"), (1, 128, "split"),
                         (3, 128, "split"), (2, 128, "paired")):
        f = b.prefill_kernel_of(base.scaled(Hq=hq, Hkv=1, bs=bs))[0]
        assert f == ("attn_prefill_split.cu" if want == "split" else "attn_prefill.cu"), (hq, bs, f)


def test_committed_prefill_summaries_carry_traffic_and_source_hash():
    """Each committed prefill ncu summary carries the traffic figure and the
    hash of the sources its counters were taken on (bench.py reports the
    traffic only while that hash matches the current sources)."""
    b = _bench()
    for name in ("prefill_gqa_bf16", "gated_prefill_bf16"):
        kfile, _ = b.prefill_kernel_of(W.get(name))
        traffic, sha = b.profile_traffic(kfile, f"{kfile[:-3]}_{name}.md")
        assert traffic is not None and traffic > 0, name
        assert sha is not None and len(sha) == 64, name


def test_reference_arm_prints_the_same_config_as_ours():
    """Both arms describe the workload with the same config object, so the
    two lines can be matched config for config."""
    b = _bench()
    for name in ("prefill_gqa_bf16", "gated_prefill_bf16", "tiny_prefill_f32"):
        w = W.get(name)
        c = b.prefill_config(w, 1)
        assert c["workload"] == name and c["seq_len"] == w.N and c["Hq"] == w.Hq
        assert c == b.prefill_config(W.get(name), 1)
