"""attn_fwd_varlen (prefill over a packed batch of sequences of different
lengths) on the GPU against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu

pytestmark = pytest.mark.gpu


def _packed(lens_q, lens_k, n_q, n_kv, d, seed):
    need_gpu()
    g = torch.Generator(device="cuda").manual_seed(seed)
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    q = torch.randn(tq, n_q, d, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(max(tk, 1), n_kv, d, generator=g, device="cuda").to(torch.bfloat16)[:tk].contiguous()
    v = torch.randn(max(tk, 1), n_kv, d, generator=g, device="cuda").to(torch.bfloat16)[:tk].contiguous()
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lens_k)]), dtype=torch.int32)
    return q, k, v, cq, ck


def _run(lens_q, lens_k, n_q, n_kv, d, causal, seed, scale=None):
    binding = need_gpu()
    scale = scale or 1.0 / math.sqrt(d)
    q, k, v, cq, ck = _packed(lens_q, lens_k, n_q, n_kv, d, seed)
    o, lse = binding.attn_fwd_varlen(q, k, v, cq.cuda(), ck.cuda(), max(lens_q), causal, scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa_varlen(q, k, v, cq, ck, causal, scale)
    check_parity(o, lse, o_ref, lse_ref, f"varlen {lens_q}/{lens_k} {n_q}/{n_kv} d{d} c{causal}")
    return o, lse


@pytest.mark.parametrize("lens,n_q,n_kv,d,causal", [
    ([1, 300, 64, 129, 1000], 32, 8, 128, True),     # G=4: one-row, ragged and tile-aligned sequences
    ([700, 5, 256], 16, 2, 128, True),               # G=8
    ([513, 77], 4, 4, 64, True),                     # MHA (G=1): two 128-row tiles per CTA
    ([200, 31, 2048], 8, 1, 128, False),             # MQA, non-causal
    ([97, 160], 2, 1, 32, True),                     # d=32
])
def test_varlen_self_attention(lens, n_q, n_kv, d, causal):
    _run(lens, lens, n_q, n_kv, d, causal, seed=len(lens) * 100 + n_q)


def test_varlen_queries_shorter_than_keys():
    """Chunked prefill: each sequence appends its last Sq_b queries to a longer
    context (bottom-right causal alignment per sequence)."""
    _run([64, 1, 300], [1000, 77, 300], 32, 8, 128, True, seed=5)


def test_varlen_empty_rows_and_sequences():
    """A sequence with no queries, one with no keys, and one with more causal
    queries than keys: rows that see no key give O = 0, LSE = -inf."""
    o, lse = _run([5, 0, 40, 3], [5, 3, 0, 1], 8, 2, 128, True, seed=6)
    # sequence 2 (rows 5..44) has no keys at all
    assert torch.all(o[5:45] == 0) and torch.all(torch.isneginf(lse[:, 5:45]))


def test_varlen_equals_batched_prefill():
    """Equal-length sequences packed are the BHSD batch: same numbers as attn_fwd."""
    binding = need_gpu()
    B, S, n_q, n_kv, d = 3, 700, 32, 8, 128
    g = torch.Generator(device="cuda").manual_seed(9)
    q = torch.randn(B, n_q, S, d, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, n_kv, S, d, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, n_kv, S, d, generator=g, device="cuda").to(torch.bfloat16)
    o1, l1 = binding.attn_fwd(q, k, v, True, 0.1)
    pack = lambda x: x.transpose(1, 2).reshape(B * S, x.shape[1], d).contiguous()
    cu = torch.arange(B + 1, dtype=torch.int32, device="cuda") * S
    o2, l2 = binding.attn_fwd_varlen(pack(q), pack(k), pack(v), cu, cu, S, True, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(pack(o1), o2)
    assert torch.equal(l1.transpose(0, 1).reshape(n_q, B * S), l2)


def test_varlen_writes_only_its_rows():
    """Rows of the output outside every sequence (here: none exist, so the
    check is on a guard band around the packed output) stay untouched, and
    the tile that straddles a sequence end does not spill into the next
    sequence."""
    binding = need_gpu()
    lens = [70, 300, 1]
    q, k, v, cq, ck = _packed(lens, lens, 16, 4, 128, 12)
    total = sum(lens)
    guard = 4096
    buf = torch.full((total * 16 * 128 + 2 * guard,), 3.0, dtype=torch.bfloat16, device="cuda")
    o = buf[guard:guard + total * 16 * 128].view(total, 16, 128)
    binding.attn_fwd_varlen(q, k, v, cq.cuda(), ck.cuda(), max(lens), True, 0.1, o=o)
    torch.cuda.synchronize()
    assert torch.all(buf[:guard] == 3.0) and torch.all(buf[guard + o.numel():] == 3.0)
    o_ref, _ = oracle.sdpa_varlen(q, k, v, cq, ck, True, 0.1)
    assert float(np.abs(o.float().cpu().numpy() - o_ref).max()) <= 2e-2


def test_varlen_malformed_offsets_are_skipped_and_reported():
    binding = need_gpu()
    lens = [100, 50]
    q, k, v, cq, ck = _packed(lens, lens, 8, 2, 128, 13)
    bad_q = torch.tensor([0, 100, 90], dtype=torch.int32, device="cuda")    # decreasing: sequence 1 malformed
    o = torch.full((150, 8, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    binding.attn_fwd_varlen(q, k, v, bad_q, ck.cuda(), 100, True, 0.1, o=o)
    assert binding.device_status() == -7
    assert torch.all(o[100:] == 7.0)                 # skipped sequence left as it was
    o_ref, _ = oracle.sdpa_varlen(q[:100], k[:100], v[:100], [0, 100], [0, 100], True, 0.1)
    assert float(np.abs(o[:100].float().cpu().numpy() - o_ref).max()) <= 2e-2
