"""MLA absorbed-latent decode (attn_decode with d_qk=576, d_v=512, n_kv=1 and
the value rows being the first 512 columns of the key rows) against the fp64
oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def _run(seqlens, q, cache, scale, what):
    binding = need_gpu()
    c4 = cache[:, None]                                  # [B, 1, S_max, 576] view
    sl = seqlens.cuda()
    o, lse = binding.attn_decode(q, c4, c4, sl, scale, d_v=512)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, l_ref = oracle.sdpa(q[:, :, None, :], c4, c4, False, scale, seqlens=seqlens.numpy(), d_v=512)
    check_parity(o, lse, o_ref[:, :, 0], l_ref[:, :, 0], what)
    return o, lse


def test_mla_workload_full():
    """B=64 sequences of 4096 latent rows, 128 heads: every output row."""
    w = inputs.WORKLOADS["mla_decode"]
    seqlens, q, cache = inputs.make(w, device="cuda")
    _run(seqlens, q, cache, w.scale, "mla_decode")


@pytest.mark.parametrize("seqlens", [[1, 63, 64, 65], [1000, 4096, 2049], [0, 5]])
def test_mla_ragged(seqlens):
    B, S_max = len(seqlens), max(max(seqlens), 1)
    sl = torch.tensor(seqlens, dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(B * 7 + S_max)
    q = torch.randn(B, 128, 576, generator=g, device="cuda").to(torch.bfloat16)
    cache = torch.randn(B, S_max, 576, generator=g, device="cuda").to(torch.bfloat16)
    o, lse = _run(sl, q, cache, 1 / math.sqrt(192), f"mla {seqlens}")
    for b, L in enumerate(seqlens):
        if L == 0:
            assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))


def test_mla_ignores_nonfinite_rows_past_the_length():
    """Latent rows at or beyond a sequence's length hold NaN and +Inf, inside
    the same 64-row tile as valid rows: the result must equal the oracle's on
    the valid rows."""
    seqlens = [1, 100, 4000]
    B, S_max = len(seqlens), 4096
    sl = torch.tensor(seqlens, dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(17)
    q = torch.randn(B, 128, 576, generator=g, device="cuda").to(torch.bfloat16)
    cache = torch.randn(B, S_max, 576, generator=g, device="cuda").to(torch.bfloat16)
    for b, L in enumerate(seqlens):
        cache[b, L:, :288] = float("nan")
        cache[b, L:, 288:] = float("inf")
    o, lse = _run(sl, q, cache, 1 / math.sqrt(192), "mla non-finite rows past the length")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_mla_two_head_blocks_and_padded_rows():
    """256 heads (two 128-head tiles) and a cache whose rows are padded to 640."""
    binding = need_gpu()
    B, S_max = 2, 700
    g = torch.Generator(device="cuda").manual_seed(91)
    q = torch.randn(B, 256, 576, generator=g, device="cuda").to(torch.bfloat16)
    buf = torch.randn(B, S_max, 640, generator=g, device="cuda").to(torch.bfloat16)
    cache = buf[:, :, :576]                              # row stride 640 elements
    sl = torch.tensor([700, 333], dtype=torch.int32)
    c4 = cache[:, None]
    o, lse = binding.attn_decode(q, c4, c4, sl.cuda(), 0.07, d_v=512)
    o_ref, l_ref = oracle.sdpa(q[:, :, None, :], c4, c4, False, 0.07, seqlens=sl.numpy(), d_v=512)
    check_parity(o, lse, o_ref[:, :, 0], l_ref[:, :, 0], "mla 256 heads padded rows")


def test_mla_deterministic():
    binding = need_gpu()
    w = inputs.WORKLOADS["mla_decode"]
    seqlens, q, cache = inputs.mla_inputs(8, 128, 576, 2048, (1, 2048), 55, device="cuda")
    c4 = cache[:, None]
    sl = seqlens.cuda()
    o1, l1 = binding.attn_decode(q, c4, c4, sl, w.scale, d_v=512)
    for _ in range(3):
        o2, l2 = binding.attn_decode(q, c4, c4, sl, w.scale, d_v=512)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_mla_rejects_unaliased_value():
    binding = need_gpu()
    q = torch.zeros(1, 128, 576, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(1, 1, 64, 576, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(1, 1, 64, 576, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.AttnError) as e:
        binding.attn_decode(q, c, v, torch.ones(1, dtype=torch.int32, device="cuda"), 0.1, d_v=512)
    assert e.value.code == -2


@pytest.mark.parametrize("B", [1, 4])
def test_mla_small_batch_split_over_the_sms(B):
    """A batch too small to fill the GPU by whole sequences (S=4096, 128
    heads): the keys are cut into chunks, each a 2-CTA cluster of its own
    writing a partial output to the workspace, merged by their log-sum-exp
    weights; every output row against the oracle."""
    binding = need_gpu()
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    S = 4096
    ws = binding.decode_workspace_bytes(B, 128, 1, 576, 512, S)
    # clusters of two SMs; at least two 64-key tiles per chunk
    s = min((n_sm // 2) // B, S // 128)
    ch = -(-(-(-S // s)) // 64) * 64
    splits = -(-S // ch)
    assert splits > 1
    rows = B * 128 * splits
    assert ws == ((rows * 512 * 4 + 255) // 256) * 256 + rows * 8, (ws, splits)
    seqlens, q, cache = inputs.mla_inputs(B, 128, 576, S, (S, S), 40 + B, device="cuda")
    _run(seqlens, q, cache, 1 / math.sqrt(192), f"mla split B={B}")


def test_mla_full_batch_needs_no_workspace():
    """The MLA workload's batch (64 sequences) fills the clusters by itself:
    one chunk per sequence, no workspace."""
    binding = need_gpu()
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    B = max(64, n_sm // 2)
    assert binding.decode_workspace_bytes(B, 128, 1, 576, 512, 4096) == 0
