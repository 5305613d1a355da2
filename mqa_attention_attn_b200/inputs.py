"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws seeded bf16 tensors
of the shapes below, so that the CUDA path and the fp64 oracle can be fed the
very same values. Both sides import it; it imports neither.

Recipe (for every workload):
  * one ``torch.Generator`` seeded with the workload's seed, on the device
    the tensors are made on;
  * for decode workloads the per-sequence cache lengths are drawn first, from
    a CPU generator with the same seed, uniformly in [lo, hi] (inclusive);
  * then q, k, v in that order, each ``torch.randn`` in fp32 (N(0, 1)),
    rounded to bf16 (round-to-nearest-even); large tensors are drawn in
    slices along the leading dimension, in order, from the same generator;
  * cache rows beyond a sequence's length are drawn like the rest, so a
    kernel that reads past ``seqlens`` produces a wrong answer.

The workloads stand in for the shapes the pages discuss: a Llama-3-8B-like
GQA layer (32 query / 8 KV heads, head dim 128), a Llama-3-70B-like layer
(64 / 8), and the DeepSeek-V3 MLA latent cache (512 latent + 64 rotary).
No dataset or trained weight is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" | "decode" | "mla_decode"
    B: int
    n_q: int
    n_kv: int
    d_qk: int
    d_v: int
    seed: int
    Sq: int = 1
    Skv: int = 0               # prefill: key count; decode: S_max (cache capacity)
    causal: bool = False
    scale: float = 0.0
    seqlen_range: tuple = ()   # decode: (lo, hi) inclusive, drawn per sequence
    description: str = ""

    @property
    def G(self) -> int:
        return self.n_q // self.n_kv


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_prefill", "prefill", B=1, n_q=4, n_kv=2, d_qk=32, d_v=32, seed=1,
                 Sq=64, Skv=64, causal=True, scale=1 / math.sqrt(32),
                 description="tiny causal GQA forward, B=1 S=64 n_q=4 n_kv=2 d=32"),
        Workload("llama3_8b_prefill", "prefill", B=1, n_q=32, n_kv=8, d_qk=128, d_v=128, seed=2,
                 Sq=4096, Skv=4096, causal=True, scale=1 / math.sqrt(128),
                 description="Llama-3-8B-shaped causal GQA prefill, B=1 S=4096 n_q=32 n_kv=8 d=128"),
        Workload("gqa_decode", "decode", B=32, n_q=32, n_kv=8, d_qk=128, d_v=128, seed=3,
                 Sq=1, Skv=32768, seqlen_range=(1024, 32768), scale=1 / math.sqrt(128),
                 description="GQA decode, B=32, cache length ~U[1024, 32768], n_q=32 n_kv=8 d=128"),
        Workload("llama3_70b_long_prefill", "prefill", B=1, n_q=64, n_kv=8, d_qk=128, d_v=128,
                 seed=4, Sq=32768, Skv=32768, causal=True, scale=1 / math.sqrt(128),
                 description="70B-shaped causal GQA prefill, B=1 S=32768 n_q=64 n_kv=8 d=128"),
        Workload("mla_decode", "mla_decode", B=64, n_q=128, n_kv=1, d_qk=576, d_v=512, seed=5,
                 Sq=1, Skv=4096, seqlen_range=(4096, 4096), scale=1 / math.sqrt(192),
                 description="MLA absorbed-latent decode (MQA form), B=64 S=4096 n_q=128, "
                             "key = 576-wide latent row, value = its first 512 columns"),
    ]
}


def _randn_bf16(shape, gen, device, chunk_elems=1 << 27) -> torch.Tensor:
    """N(0,1) fp32 rounded to bf16, drawn in order along dim 0 in slices."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if out.numel() == 0:
        return out
    flat = out.view(shape[0], -1)
    per_row = flat.shape[1]
    rows_per_chunk = max(1, chunk_elems // max(per_row, 1))
    for r0 in range(0, shape[0], rows_per_chunk):
        r1 = min(shape[0], r0 + rows_per_chunk)
        flat[r0:r1] = torch.randn((r1 - r0, per_row), generator=gen, device=device,
                                  dtype=torch.float32).to(torch.bfloat16)
    return out


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return g


def prefill_inputs(B, Sq, Skv, n_q, n_kv, d_qk, d_v, seed, device="cpu"):
    """q [B,n_q,Sq,d_qk], k [B,n_kv,Skv,d_qk], v [B,n_kv,Skv,d_v], all bf16."""
    g = _gen(seed, device)
    q = _randn_bf16((B, n_q, Sq, d_qk), g, device)
    k = _randn_bf16((B, n_kv, Skv, d_qk), g, device)
    v = _randn_bf16((B, n_kv, Skv, d_v), g, device)
    return q, k, v


def draw_seqlens(B, lo, hi, seed) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    return torch.randint(int(lo), int(hi) + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def decode_inputs(B, n_q, n_kv, d_qk, d_v, S_max, seqlen_range, seed, device="cpu"):
    """seqlens int32 [B]; q [B,n_q,d_qk]; kcache [B,n_kv,S_max,d_qk];
    vcache [B,n_kv,S_max,d_v]."""
    seqlens = draw_seqlens(B, seqlen_range[0], seqlen_range[1], seed)
    g = _gen(seed, device)
    q = _randn_bf16((B, n_q, d_qk), g, device)
    k = _randn_bf16((B, n_kv, S_max, d_qk), g, device)
    v = _randn_bf16((B, n_kv, S_max, d_v), g, device)
    return seqlens, q, k, v


def mla_inputs(B, n_q, d_latent, S_max, seqlen_range, seed, device="cpu"):
    """seqlens int32 [B]; q [B,n_q,d_latent]; latent cache [B,S_max,d_latent].
    The key of token j is cache[b, j, :d_latent]; its value is a prefix of the
    same row."""
    seqlens = draw_seqlens(B, seqlen_range[0], seqlen_range[1], seed)
    g = _gen(seed, device)
    q = _randn_bf16((B, n_q, d_latent), g, device)
    cache = _randn_bf16((B, S_max, d_latent), g, device)
    return seqlens, q, cache


def make(w: Workload, device="cpu"):
    """Inputs of a named workload (see the recipe above)."""
    if w.kind == "prefill":
        return prefill_inputs(w.B, w.Sq, w.Skv, w.n_q, w.n_kv, w.d_qk, w.d_v, w.seed, device)
    if w.kind == "decode":
        return decode_inputs(w.B, w.n_q, w.n_kv, w.d_qk, w.d_v, w.Skv, w.seqlen_range, w.seed, device)
    if w.kind == "mla_decode":
        return mla_inputs(w.B, w.n_q, w.d_qk, w.Skv, w.seqlen_range, w.seed, device)
    raise ValueError(w.kind)


def sample_rows(n_rows, B, n_q, Sq, seed, must=()):
    """A seeded sample of (b, h, i) row triples for sampled checks at full
    size, stratified: every (b, h) contributes its first and last row, both
    rows at every 128-row tile boundary (i = 128t - 1 and 128t, each with a
    seeded (b, h)) are included, and the rest are uniform. The forced rows
    alone can exceed n_rows at long S; the result then holds all of them.
    Returns an int32 tensor [n, 3], sorted."""
    g = torch.Generator().manual_seed(int(seed) + 7919)
    picks = set()
    for b in range(B):
        for h in range(n_q):
            picks.add((b, h, 0))
            picks.add((b, h, Sq - 1))
    for i in list(range(127, Sq, 128)) + list(range(128, Sq, 128)):
        picks.add((int(torch.randint(B, (1,), generator=g)), int(torch.randint(n_q, (1,), generator=g)), i))
    for t in must:
        picks.add(tuple(int(x) for x in t))
    while len(picks) < n_rows:
        picks.add((int(torch.randint(B, (1,), generator=g)),
                   int(torch.randint(n_q, (1,), generator=g)),
                   int(torch.randint(Sq, (1,), generator=g))))
    rows = sorted(picks)
    return torch.tensor(rows, dtype=torch.int32)
