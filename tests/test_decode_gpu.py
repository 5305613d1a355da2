"""attn_decode (single-token decode against a KV cache) on the GPU against the
fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def _decode_and_check(seqlens, q, kc, vc, scale, what, d_v=None):
    binding = need_gpu()
    sl = seqlens.to("cuda")
    o, lse = binding.attn_decode(q, kc, vc, sl, scale, d_v=d_v)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    B, n_q, d_qk = q.shape
    o_ref, lse_ref = oracle.sdpa(q[:, :, None, :], kc, vc, False, scale, seqlens=seqlens.numpy(),
                                 d_v=d_v)
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], what)
    return o, lse


@pytest.mark.parametrize("B,n_q,n_kv,S_max,seqlens", [
    (3, 8, 2, 1100, [1, 700, 1100]),        # G=4, ragged, 1..3 chunks
    (2, 32, 8, 2048, [2048, 1537]),         # Llama-3-8B heads
    (2, 4, 4, 600, [513, 64]),              # MHA (G=1)
    (1, 16, 8, 300, [300]),                 # G=2
    (2, 64, 8, 900, [899, 1]),              # G=8
    (1, 32, 2, 1030, [1030]),               # G=16 (two head blocks)
    (2, 32, 1, 700, [700, 65]),             # MQA, G=32 (two head blocks)
    (2, 8, 2, 100, [100, 37]),              # cache shorter than one 128-key tile
    (1, 2, 2, 513, [513]),                  # MHA with fewer heads than the MMA's 8 columns
])
def test_decode_shapes(B, n_q, n_kv, S_max, seqlens):
    seq = torch.tensor(seqlens, dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(B * 1000 + n_q + S_max)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    _decode_and_check(seq, q, kc, vc, 1 / math.sqrt(128), f"decode {B} {n_q}/{n_kv} {S_max}")


def test_decode_strided_cache():
    """A cache stored [B, S_max, n_kv, d] (token-major) passed through strides."""
    B, n_q, n_kv, S_max = 2, 16, 4, 1500
    seq = torch.tensor([1500, 999], dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(5)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kb = torch.randn(B, S_max, n_kv, 128, generator=g, device="cuda").to(torch.bfloat16)
    vb = torch.randn(B, S_max, n_kv, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc, vc = kb.permute(0, 2, 1, 3), vb.permute(0, 2, 1, 3)      # views, not copies
    _decode_and_check(seq, q, kc, vc, 0.1, "strided cache")


def test_gqa_decode_workload_full():
    """The GQA decode workload at full size (B=32, cache lengths ~U[1024, 32768],
    32/8 heads): every (b, h) output row against the oracle."""
    binding = need_gpu()
    w = inputs.WORKLOADS["gqa_decode"]
    seqlens, q, kc, vc = inputs.make(w, device="cuda")
    o, lse = binding.attn_decode(q, kc, vc, seqlens.cuda(), w.scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref = np.zeros((w.B, w.n_q, w.d_v))
    l_ref = np.zeros((w.B, w.n_q))
    for b in range(w.B):
        L = int(seqlens[b])
        ob, lb = oracle.sdpa(q[b:b + 1, :, None, :], kc[b:b + 1, :, :L], vc[b:b + 1, :, :L], False, w.scale)
        o_ref[b], l_ref[b] = ob[0, :, 0], lb[0, :, 0]
    check_parity(o, lse, o_ref, l_ref, "gqa_decode")


def test_decode_equals_last_prefill_row():
    """Decode of token L-1 against a cache of L tokens == row L-1 of causal prefill."""
    binding = need_gpu()
    n_q, n_kv, L = 32, 8, 1234
    q, k, v = inputs.prefill_inputs(1, L, L, n_q, n_kv, 128, 128, 21, device="cuda")
    o_p, l_p = binding.attn_fwd(q, k, v, True, 0.08)
    o_d, l_d = binding.attn_decode(q[:, :, L - 1].contiguous(), k, v,
                                   torch.tensor([L], dtype=torch.int32, device="cuda"), 0.08)
    assert (o_p[:, :, L - 1].float() - o_d.float()).abs().max() <= 2e-2
    assert (l_p[:, :, L - 1] - l_d).abs().max() <= 1e-3


@pytest.mark.parametrize("L", [2047, 2048, 2049, 4097, 6500])
def test_decode_independent_of_split_count(L):
    """The split-KV decode (one sequence of 8 KV heads: the keys are cut into
    as many chunks as it takes to reach every SM, chunk lengths of whole
    128-key tiles, merged by their log-sum-exp weights) equals the unsplit
    computation: row L-1 of the causal prefill over the same L tokens."""
    binding = need_gpu()
    n_q, n_kv = 32, 8
    q, k, v = inputs.prefill_inputs(1, L, L, n_q, n_kv, 128, 128, 31 + L, device="cuda")
    o_p, l_p = binding.attn_fwd(q, k, v, True, 0.08)
    o_d, l_d = binding.attn_decode(q[:, :, L - 1].contiguous(), k, v,
                                   torch.tensor([L], dtype=torch.int32, device="cuda"), 0.08)
    assert binding.device_status() == 0
    assert (o_p[:, :, L - 1].float() - o_d.float()).abs().max() <= 2e-2
    assert (l_p[:, :, L - 1] - l_d).abs().max() <= 1e-3


def test_decode_zero_length_and_range_status():
    binding = need_gpu()
    B, n_q, n_kv, S_max = 3, 8, 2, 256
    g = torch.Generator(device="cuda").manual_seed(6)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    seq = torch.tensor([0, 100, 1000], dtype=torch.int32, device="cuda")   # 1000 > S_max: clamped
    o, lse = binding.attn_decode(q, kc, vc, seq, 0.1)
    assert binding.device_status() == -7                                     # ATTN_ERR_DEVICE_RANGE
    assert binding.device_status() == 0                                      # cleared by the read
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    o_ref, l_ref = oracle.sdpa(q[:, :, None, :], kc, vc, False, 0.1,
                               seqlens=np.array([0, 100, 256], np.int32))
    check_parity(o, lse, o_ref[:, :, 0], l_ref[:, :, 0], "zero/clamped lengths")


def test_decode_ignores_nonfinite_cache_rows_past_the_length():
    """Cache rows at or beyond a sequence's length take no part, whatever they
    hold: they are filled with NaN and +Inf here, inside the same 128-key
    tile as valid rows, and the result must equal the oracle's on the valid
    rows."""
    B, n_q, n_kv, S_max = 3, 32, 8, 1100
    seq = torch.tensor([1, 700, 1029], dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(8)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    for b, L in enumerate(seq.tolist()):
        kc[b, :, L:] = float("nan")
        vc[b, :, L:] = float("inf")
    o, lse = _decode_and_check(seq, q, kc, vc, 0.1, "non-finite rows past the length")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_decode_workspace_checks():
    binding = need_gpu()
    B, n_q, n_kv, S_max = 2, 8, 2, 1024
    q = torch.zeros(B, n_q, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(B, n_kv, S_max, 128, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([5, 6], dtype=torch.int32, device="cuda")
    need = binding.decode_workspace_bytes(B, n_q, n_kv, 128, 128, S_max)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.AttnError) as e:
        binding.attn_decode(q, kc, kc, seq, 0.1, workspace=ws)
    assert e.value.code == -4


def test_decode_deterministic():
    binding = need_gpu()
    w = inputs.WORKLOADS["gqa_decode"]
    seqlens, q, kc, vc = inputs.decode_inputs(4, 32, 8, 128, 128, 8192, (1, 8192), 31, device="cuda")
    sl = seqlens.cuda()
    o1, l1 = binding.attn_decode(q, kc, vc, sl, w.scale)
    for _ in range(5):
        o2, l2 = binding.attn_decode(q, kc, vc, sl, w.scale)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_timeout_path_reports_status():
    """A bounded wait that nothing completes ends with ATTN_ERR_DEVICE_TIMEOUT
    and leaves the context usable."""
    binding = need_gpu()
    binding.selftest_timeout(20000)
    assert binding.device_status() == -6
    assert binding.device_status() == 0
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


def _planned_splits(B, n_kv, G, S_max):
    """The split count the launch plans for a bf16 cache (two CTAs per SM at
    up to 8 heads per unit): every unit of a full-length batch gets a slot of
    the persistent grid when the batch alone does not fill it."""
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    GT = min(G, 16)
    largest = 2048 if GT <= 8 else 1024
    s = (2 * n_sm) // (B * n_kv * (G // GT))
    ch = largest if s <= 1 else min(largest, -(-(-(-S_max // s)) // 128) * 128)
    return -(-S_max // ch)


@pytest.mark.parametrize("B,L,seqlens", [
    (1, 32768, [32768]),                   # one long sequence: chunks over every SM
    (4, 8192, [8192, 8192, 5000, 1]),     # a small batch, ragged
])
def test_small_batch_decode_spreads_over_the_sms(B, L, seqlens):
    """Llama-3-8B heads (32 / 8), a batch too small to fill the GPU by whole
    sequences: the keys are cut into enough chunks that every SM gets work
    (the workspace has that many splits), and the result matches the oracle."""
    binding = need_gpu()
    n_q, n_kv = 32, 8
    splits = _planned_splits(B, n_kv, n_q // n_kv, L)
    assert splits > L // 2048, splits          # more chunks than the largest chunk gives
    rows = B * n_q * splits
    assert binding.decode_workspace_bytes(B, n_q, n_kv, 128, 128, L) == ((rows * 512 + 255) // 256) * 256 + rows * 8
    seq = torch.tensor(seqlens, dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(B * 7 + L)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, L, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, L, 128, generator=g, device="cuda").to(torch.bfloat16)
    _decode_and_check(seq, q, kc, vc, 1 / math.sqrt(128), f"small-batch decode B={B} L={L}")


def test_large_batch_decode_keeps_the_largest_chunk():
    """A batch that fills every slot of the persistent grid by itself keeps
    the largest chunk (2048 keys at 4 query heads per KV head); lengths on
    both sides of chunk boundaries, against the oracle."""
    binding = need_gpu()
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    n_q, n_kv, S_max = 32, 8, 6500
    B = -(-2 * n_sm // n_kv)                       # B * n_kv >= the resident CTAs
    assert _planned_splits(B, n_kv, n_q // n_kv, S_max) == 4
    base = [2047, 2048, 2049, 4096, 4097, 6500, 1, 128, 129]
    seq = torch.tensor([base[b % len(base)] for b in range(B)], dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(77)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    _decode_and_check(seq, q, kc, vc, 1 / math.sqrt(128), f"large-batch decode B={B}")


def test_decode_split_ignores_workspace_contents_and_replays():
    """The split-KV decode writes each key chunk's partial output to the
    workspace and a second kernel merges them. Whatever the workspace holds on
    entry (all ones, then random bytes), the result is the oracle's and
    repeats bit for bit; a CUDA graph replays both launches with new queries,
    each replay against the oracle. A zero-length sequence in the batch gets
    O = 0, LSE = -inf."""
    binding = need_gpu()
    B, n_q, n_kv, L = 3, 32, 8, 8192
    scale = 1 / math.sqrt(128)
    seq = torch.tensor([8192, 0, 3000], dtype=torch.int32)
    sl = seq.to("cuda")
    g = torch.Generator(device="cuda").manual_seed(4242)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, L, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, L, 128, generator=g, device="cuda").to(torch.bfloat16)
    assert _planned_splits(B, n_kv, n_q // n_kv, L) > 1
    nbytes = binding.decode_workspace_bytes(B, n_q, n_kv, 128, 128, L)
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")

    def check(o, lse, what):
        assert torch.all(o[1] == 0) and torch.all(torch.isneginf(lse[1])), what
        keep = [0, 2]
        o_ref, lse_ref = oracle.sdpa(q[keep][:, :, None, :], kc[keep], vc[keep], False, scale,
                                     seqlens=seq.numpy()[keep])
        check_parity(o[keep], lse[keep], o_ref[:, :, 0], lse_ref[:, :, 0], what)

    o1, lse1 = binding.attn_decode(q, kc, vc, sl, scale, workspace=ws)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    check(o1, lse1, "workspace of all ones")
    ws.random_(0, 256, generator=g)
    o2, lse2 = binding.attn_decode(q, kc, vc, sl, scale, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)

    o3, lse3 = torch.empty_like(o1), torch.empty_like(lse1)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        binding.attn_decode(q, kc, vc, sl, scale, o=o3, lse=lse3, workspace=ws)
    for rep in range(3):
        q.copy_(torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16))
        graph.replay()
        torch.cuda.synchronize()
        assert binding.device_status() == 0
        check(o3, lse3, f"graph replay {rep}")
    del graph
