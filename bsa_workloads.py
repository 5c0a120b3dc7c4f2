"""Seeded synthetic workloads for top-k block-sparse causal attention.

This module only draws random inputs and names workload shapes.  It holds
none of the method's arithmetic (no pooling, scoring, selection or
attention): both the CUDA path and the CPU oracle receive the bytes drawn
here, so the two sides are compared on identical inputs.

Shapes mirror the workloads described on the source pages:
  * GQA shapes with 28/4 and 32/8 query/KV heads and head dim 128 follow the
    model table of "稀疏注意力的Trade-offs" (§3.1, Qwen 2.5 / Llama 3.1 rows).
  * Context lengths up to 128K and sparsity up to 0.95 follow the same page,
    §3.4 (evaluation settings) and §1.2 (sparsity definition).
  * The 64-token chunk followed by one gist key/value follows
    "通过Gist Token的简化稀疏注意力" (SSA), "输入与训练阶段".

Every draw comes from one ``torch.Generator`` seeded per workload, in a fixed
order (Q, then K, then V, then the extra tensors), drawn as fp32 N(0,1) and
cast to the workload dtype.  The same seed on a CPU generator and on a CUDA
generator gives different streams; a test always hands the SAME tensors to
both sides, so that does not matter.
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill", "gated", "decode", "gist", "hssa"
    B: int
    Hq: int
    Hkv: int
    N: int               # tokens (prefill) or cached tokens (decode / gist)
    d: int
    bs: int              # KV block size, or gist chunk size
    kb: int              # history budget (prefill/decode) or top-k chunks (gist)
    dtype: str           # "f32" or "bf16"
    seed: int
    key_offset_std: float = 0.0   # per-block key offset, std (prefill GQA)
    plant_frac: float = 0.0       # fraction of blocks with a planted key shift (decode)
    plant_alpha: float = 0.0      # size of the planted shift along the group query direction

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nb(self) -> int:
        return self.N // self.bs

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        """Same structure (kind, dtype, block size, distributions), other sizes."""
        fields = dataclasses.asdict(self)
        fields.update(kw)
        if "name" not in kw:
            fields["name"] = self.name + "_scaled"
        return Workload(**fields)


# The five workloads.  Config 1 is the small case the oracle finishes in
# seconds; config 2 is the prefill workload the headline metric is quoted on.
WORKLOADS: Dict[str, Workload] = {
    "tiny_prefill_f32": Workload(
        name="tiny_prefill_f32", kind="prefill", B=1, Hq=1, Hkv=1, N=1024, d=64,
        bs=64, kb=4, dtype="f32", seed=0),
    "prefill_gqa_bf16": Workload(
        name="prefill_gqa_bf16", kind="prefill", B=1, Hq=32, Hkv=8, N=32768, d=128,
        bs=64, kb=16, dtype="bf16", seed=1, key_offset_std=0.5),
    "decode_bf16": Workload(
        name="decode_bf16", kind="decode", B=16, Hq=32, Hkv=8, N=131072, d=128,
        bs=64, kb=96, dtype="bf16", seed=2, plant_frac=0.01, plant_alpha=2.0),
    "gated_prefill_bf16": Workload(
        name="gated_prefill_bf16", kind="gated", B=2, Hq=28, Hkv=4, N=16384, d=128,
        bs=128, kb=8, dtype="bf16", seed=3),
    "gist_decode_bf16": Workload(
        name="gist_decode_bf16", kind="gist", B=8, Hq=32, Hkv=8, N=131072, d=128,
        bs=64, kb=32, dtype="bf16", seed=4),
}

# Workloads of the widened path (not among the five above): the gist workload
# with one meta-gist per 64 chunks, 4 groups kept per head, 32 chunks expanded.
EXTRA_WORKLOADS: Dict[str, Workload] = {
    "hssa_decode_bf16": Workload(
        name="hssa_decode_bf16", kind="hssa", B=8, Hq=32, Hkv=8, N=131072, d=128,
        bs=64, kb=32, dtype="bf16", seed=5),
}
HSSA_GROUPS_KEPT = 4


def _randn(shape, gen: torch.Generator, device, dtype) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def _randn_big(shape, gen: torch.Generator, device, dtype) -> torch.Tensor:
    """N(0,1) drawn slice by slice along dim 0, so the fp32 staging buffer
    stays one slice in size.  Deterministic for a given generator state."""
    out = torch.empty(shape, device=device, dtype=dtype)
    for b in range(shape[0]):
        out[b] = torch.randn(shape[1:], generator=gen, device=device,
                             dtype=torch.float32).to(dtype)
    return out


def make_inputs(w: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """Draw the inputs of workload ``w`` on ``device``.

    prefill / gated: q [B,Hq,N,d], k [B,Hkv,N,d], v [B,Hkv,N,d]
    decode:          q [B,Hq,d],   k [B,Hkv,N,d], v [B,Hkv,N,d]
    gist:            q [B,Hq,d],   k, v [B,Hkv,N,d], gk, gv [B,Hkv,N/bs,d]
    hssa:            as gist, plus mk, mv [B,Hkv,N/bs/64,d]
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    out: Dict[str, torch.Tensor] = {}
    if w.kind in ("prefill", "gated"):
        out["q"] = _randn_big((w.B, w.Hq, w.N, w.d), gen, device, torch.float32)
        out["k"] = _randn_big((w.B, w.Hkv, w.N, w.d), gen, device, torch.float32)
        out["v"] = _randn_big((w.B, w.Hkv, w.N, w.d), gen, device, dt)
        if w.key_offset_std > 0.0:
            # One offset vector per (batch, KV head, block), added to every key
            # of the block before the cast, so block scores are separable.
            off = torch.randn((w.B, w.Hkv, w.nb, 1, w.d), generator=gen, device=device,
                              dtype=torch.float32) * w.key_offset_std
            k = out["k"].view(w.B, w.Hkv, w.nb, w.bs, w.d)
            k += off
        out["q"] = out["q"].to(dt)
        out["k"] = out["k"].to(dt)
    elif w.kind == "decode":
        out["q"] = _randn((w.B, w.Hq, w.d), gen, device, torch.float32)
        out["k"] = _randn_big((w.B, w.Hkv, w.N, w.d), gen, device, dt)
        out["v"] = _randn_big((w.B, w.Hkv, w.N, w.d), gen, device, dt)
        if w.plant_frac > 0.0:
            # Plant a shift toward the group's query direction in a few history
            # blocks (never the always-kept last block), so that the selected
            # set is not decided by noise alone.
            n_plant = int(round(w.plant_frac * w.nb))
            qg = out["q"].view(w.B, w.Hkv, w.G, w.d).sum(dim=2)
            u = qg / qg.norm(dim=-1, keepdim=True)
            k = out["k"].view(w.B, w.Hkv, w.nb, w.bs, w.d)
            for b in range(w.B):
                for g in range(w.Hkv):
                    blocks = torch.randperm(w.nb - 1, generator=gen, device=device)[:n_plant]
                    shift = (w.plant_alpha * u[b, g]).to(torch.float32)
                    kb = k[b, g, blocks].to(torch.float32) + shift
                    k[b, g, blocks] = kb.to(dt)
        out["q"] = out["q"].to(dt)
    elif w.kind in ("gist", "hssa"):
        nc = w.N // w.bs
        out["q"] = _randn((w.B, w.Hq, w.d), gen, device, dt)
        out["k"] = _randn_big((w.B, w.Hkv, w.N, w.d), gen, device, dt)
        out["v"] = _randn_big((w.B, w.Hkv, w.N, w.d), gen, device, dt)
        out["gk"] = _randn((w.B, w.Hkv, nc, w.d), gen, device, dt)
        out["gv"] = _randn((w.B, w.Hkv, nc, w.d), gen, device, dt)
        if w.kind == "hssa":
            # one meta-gist key/value per group of 64 chunks ("gist-of-gist")
            out["mk"] = _randn((w.B, w.Hkv, nc // 64, w.d), gen, device, dt)
            out["mv"] = _randn((w.B, w.Hkv, nc // 64, w.d), gen, device, dt)
    else:
        raise ValueError(f"unknown workload kind {w.kind!r}")
    return out


def get(name: str) -> Workload:
    return WORKLOADS[name] if name in WORKLOADS else EXTRA_WORKLOADS[name]
