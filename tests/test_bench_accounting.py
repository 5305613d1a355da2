"""The algorithmic work the benchmark divides by: FLOPs and bytes per launch,
checked against closed forms and brute force (CPU only)."""
import math

import numpy as np
import torch

import bench
from mqa_attention_attn_b200 import inputs


def _brute_pairs(Sq, Skv, causal):
    i = np.arange(Sq)[:, None]
    j = np.arange(Skv)[None, :]
    return int(((j <= i + (Skv - Sq)) if causal else np.ones((Sq, Skv), bool)).sum())


def test_prefill_flops_closed_forms():
    w = inputs.WORKLOADS["llama3_8b_prefill"]
    # 4 d FLOPs per visible pair and head, S (S + 1) / 2 pairs under the causal mask
    assert bench.prefill_flops(w) == 4 * 128 * 32 * 4096 * 4097 / 2
    assert abs(bench.prefill_flops(w) / 1e9 - 137.47) < 0.01
    w70 = inputs.WORKLOADS["llama3_70b_long_prefill"]
    assert abs(bench.prefill_flops(w70) / 1e12 - 17.59) < 0.01
    tiny = inputs.WORKLOADS["tiny_prefill"]
    assert bench.prefill_flops(tiny) == 4 * 4 * 32 * (64 * 65 // 2)


def test_prefill_flops_bottom_right_and_full_masks_by_brute_force():
    for Sq, Skv, causal in [(5, 9, True), (9, 9, True), (7, 3, False), (1, 12, True)]:
        w = inputs.Workload("x", "prefill", B=2, n_q=6, n_kv=3, d_qk=16, d_v=16, seed=0, Sq=Sq, Skv=Skv,
                            causal=causal, scale=0.25)
        assert bench.prefill_flops(w) == 2 * 6 * _brute_pairs(Sq, Skv, causal) * 2 * 32


def test_decode_bytes_and_flops():
    w = inputs.WORKLOADS["gqa_decode"]
    seqlens = inputs.draw_seqlens(w.B, w.seqlen_range[0], w.seqlen_range[1], w.seed)
    L = int(seqlens.sum())
    # K and V rows below each length (bf16), plus q, o (bf16) and lse (fp32)
    expect = L * 8 * 256 * 2 + 32 * 32 * (128 * 2 + 128 * 2 + 4)
    assert bench.decode_bytes(w, seqlens) == expect
    assert bench.decode_bytes(w, seqlens, cache_elem_bytes=1) == L * 8 * 256 + 32 * 32 * 516
    assert bench.decode_flops(w, seqlens) == L * 32 * 2 * 256
    # about 2.2 GB for this seed, arithmetic intensity about n_q / n_kv
    assert 2.0e9 < expect < 2.4e9
    assert abs(bench.decode_flops(w, seqlens) / (L * 8 * 256 * 2) - 4.0) < 1e-12


def test_mla_bytes_read_each_latent_row_once():
    w = inputs.WORKLOADS["mla_decode"]
    seqlens = torch.full((w.B,), w.Skv, dtype=torch.int32)
    cache = 64 * 4096 * 576 * 2
    assert abs(cache / 1e6 - 302.0) < 0.1
    assert bench.mla_bytes(w, seqlens) == cache + 64 * 128 * (576 * 2 + 512 * 2 + 4)
    flops = bench.decode_flops(w, seqlens)
    assert abs(flops / 1e9 - 73.0) < 0.1
    assert math.isclose(flops, 2 * 64 * 128 * 4096 * (576 + 512))


def test_fp8_prefill_bytes():
    """The FP8 prefill's algorithmic bytes: one byte per q, k, v element, a
    fp32 scale per 128-row tile of each (sequence, head), bf16 o, fp32 lse;
    for the Llama-3-8B layout 16 + 4 + 4 MiB of e4m3 inputs, 32 MiB of o."""
    w = inputs.WORKLOADS["llama3_8b_prefill"]
    tiles = (w.B * w.n_q + 2 * w.B * w.n_kv) * 32
    expect = (16 + 4 + 4 + 32) * 2 ** 20 + 4 * tiles + 4 * w.B * w.n_q * w.Sq
    assert bench.prefill_fp8_bytes(w) == expect
