"""attn_fwd_paged (prefill or chunked prefill of a packed batch whose keys and
values live in a paged cache) on the GPU against the fp64 oracle: the cache
the page table describes (oracle.paged_to_cache) attended as a packed batch
(oracle.sdpa_varlen)."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def _paged_case(seqs, n_q, n_kv, d, page_size, seed, spare_pages=3):
    """Random packed queries and a page pool holding each sequence's cached
    tokens in pages placed in a seeded random order; unused pages and rows
    past each length hold NaN. seqs: [(Sq_b, Skv_b)]."""
    g = torch.Generator().manual_seed(seed)
    B = len(seqs)
    pages_per_seq = max(1, max(-(-skv // page_size) for _, skv in seqs))
    used = [-(-skv // page_size) for _, skv in seqs]
    num_pages = sum(used) + spare_pages
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((B, pages_per_seq), -1, dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(used):
        table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    k_pages = torch.full((num_pages, page_size, n_kv, d), float("nan"))
    v_pages = torch.full((num_pages, page_size, n_kv, d), float("nan"))
    k_rows, v_rows = [], []
    for b, (_, skv) in enumerate(seqs):
        kb = torch.randn(skv, n_kv, d, generator=g)
        vb = torch.randn(skv, n_kv, d, generator=g)
        for j in range(skv):
            pg = int(table[b, j // page_size])
            k_pages[pg, j % page_size] = kb[j]
            v_pages[pg, j % page_size] = vb[j]
        k_rows.append(kb)
        v_rows.append(vb)
    total_q = sum(sq for sq, _ in seqs)
    q = torch.randn(total_q, n_q, d, generator=g)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum([sq for sq, _ in seqs])]), dtype=torch.int32)
    seqlens_k = torch.tensor([skv for _, skv in seqs], dtype=torch.int32)
    bf = lambda t: t.to(torch.bfloat16).cuda()
    return bf(q), bf(k_pages), bf(v_pages), table.cuda(), cu_q.cuda(), seqlens_k.cuda(), cu_q, seqlens_k


def _reference(q, k_pages, v_pages, table, cu_q, seqlens_k, causal, scale):
    kc = oracle.paged_to_cache(k_pages, table, seqlens_k)            # [B, n_kv, P*page, d]
    vc = oracle.paged_to_cache(v_pages, table, seqlens_k)
    lens = seqlens_k.numpy()
    kp = np.concatenate([kc[b, :, :lens[b]].transpose(1, 0, 2) for b in range(len(lens))])
    vp = np.concatenate([vc[b, :, :lens[b]].transpose(1, 0, 2) for b in range(len(lens))])
    cu_k = np.concatenate([[0], np.cumsum(lens)])
    return oracle.sdpa_varlen(q, kp, vp, cu_q.numpy(), cu_k, causal, scale)


@pytest.mark.parametrize("seqs,n_q,n_kv,d,page_size,causal", [
    ([(300, 300), (5, 700), (128, 130)], 8, 2, 128, 64, True),        # G=4: prefill, chunked, chunked
    ([(200, 517)], 16, 2, 128, 16, True),                              # G=8, 16-token pages
    ([(130, 390), (64, 64)], 4, 4, 64, 256, True),                    # MHA, pages larger than a tile
    ([(77, 77), (1, 1000), (0, 50)], 4, 2, 32, 32, False),            # non-causal, a decode-like row, no query
    ([(100, 40), (60, 0)], 8, 1, 128, 128, True),                     # MQA; queries before the first key; no key
])
def test_paged_prefill_matches_oracle(seqs, n_q, n_kv, d, page_size, causal):
    binding = need_gpu()
    q, kp, vp, table, cu_q, sk, cu_q_h, sk_h = _paged_case(seqs, n_q, n_kv, d, page_size, len(seqs) * 100 + d)
    max_q = max(max(sq for sq, _ in seqs), 1)
    scale = 1 / math.sqrt(d)
    o, lse = binding.attn_fwd_paged(q, kp, vp, table, cu_q, sk, max_q, causal, scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = _reference(q, kp, vp, table.cpu(), cu_q_h, sk_h, causal, scale)
    check_parity(o, lse, o_ref, lse_ref, f"paged prefill {seqs} page {page_size}")


def test_paged_prefill_bit_identical_to_varlen_on_contiguous_pages():
    """Pages laid out in order (identity table, the pool being the packed keys
    themselves): the same arithmetic as attn_fwd_varlen, bit for bit."""
    binding = need_gpu()
    n_q, n_kv, d, page = 16, 4, 128, 128
    lens = [(384, 384), (256, 640)]
    g = torch.Generator(device="cuda").manual_seed(9)
    total_q = sum(a for a, _ in lens)
    q = torch.randn(total_q, n_q, d, generator=g, device="cuda").to(torch.bfloat16)
    kp = torch.randn(sum(b for _, b in lens), n_kv, d, generator=g, device="cuda").to(torch.bfloat16)
    vp = torch.randn_like(kp)
    cu_q = torch.tensor([0, 384, 640], dtype=torch.int32, device="cuda")
    cu_k = torch.tensor([0, 384, 1024], dtype=torch.int32, device="cuda")
    o1, l1 = binding.attn_fwd_varlen(q, kp, vp, cu_q, cu_k, 384, True, 0.09)
    table = torch.tensor([[0, 1, 2, 2, 2], [3, 4, 5, 6, 7]], dtype=torch.int32, device="cuda")
    pool_k = kp.view(8, page, n_kv, d)
    pool_v = vp.view(8, page, n_kv, d)
    sk = torch.tensor([384, 640], dtype=torch.int32, device="cuda")
    o2, l2 = binding.attn_fwd_paged(q, pool_k, pool_v, table, cu_q, sk, 384, True, 0.09)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_paged_prefill_out_of_pool_page_reads_zeros():
    """A page id outside the pool reads as zeros (keys and values) and raises
    the range status; the result equals the oracle on that zeroed cache."""
    binding = need_gpu()
    seqs = [(100, 200)]
    q, kp, vp, table, cu_q, sk, cu_q_h, sk_h = _paged_case(seqs, 8, 2, 64, 64, 5)
    table[0, 1] = 10_000                                                 # keys 64..127
    o, lse = binding.attn_fwd_paged(q, kp, vp, table, cu_q, sk, 100, True, 0.125)
    assert binding.device_status() == -7                                # ATTN_ERR_DEVICE_RANGE
    o_ref, lse_ref = _reference(q, kp, vp, table.cpu(), cu_q_h, sk_h, True, 0.125)
    check_parity(o, lse, o_ref, lse_ref, "paged prefill with an out-of-pool page")


def test_paged_prefill_llama3_8b_sampled():
    """The Llama-3-8B prefill (S=4096, 32 / 8 heads) with its keys and values
    in 64-token pages shuffled in a pool: sampled rows against the oracle."""
    binding = need_gpu()
    w = inputs.WORKLOADS["llama3_8b_prefill"]
    q4, k4, v4 = inputs.make(w, device="cuda")
    page = 64
    P = w.Skv // page
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(3)).to(torch.int32)
    table = perm[None].cuda()
    kd = k4[0].permute(1, 0, 2).reshape(P, page, w.n_kv, w.d_qk)      # [page][token][head][d] in logical order
    vd = v4[0].permute(1, 0, 2).reshape(P, page, w.n_kv, w.d_v)
    pool_k, pool_v = torch.empty_like(kd), torch.empty_like(vd)
    pool_k[perm.long().cuda()] = kd
    pool_v[perm.long().cuda()] = vd
    qp = q4[0].permute(1, 0, 2).contiguous()                            # [S][n_q][d]
    cu_q = torch.tensor([0, w.Sq], dtype=torch.int32, device="cuda")
    sk = torch.tensor([w.Skv], dtype=torch.int32, device="cuda")
    o, lse = binding.attn_fwd_paged(qp, pool_k, pool_v, table, cu_q, sk, w.Sq, True, w.scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    rows = inputs.sample_rows(1500, w.B, w.n_q, w.Sq, 21)
    rb, rh, ri = rows[:, 0].long(), rows[:, 1].long(), rows[:, 2].long()
    o_ref, lse_ref = oracle.sdpa_rows(q4[rb.cuda(), rh.cuda(), ri.cuda()], rows.numpy(), k4, v4, w.B, w.n_q, w.Sq,
                                      True, w.scale)
    check_parity(o[ri.cuda(), rh.cuda()], lse[rh.cuda(), ri.cuda()], o_ref, lse_ref, "paged llama3_8b_prefill")


def test_paged_prefill_rejects_bad_arguments():
    binding = need_gpu()
    q, kp, vp, table, cu_q, sk, _, _ = _paged_case([(10, 10)], 4, 2, 64, 16, 1)
    kp48 = torch.zeros(4, 48, 2, 64, dtype=torch.bfloat16, device="cuda")      # 48-token pages
    with pytest.raises(binding.AttnError) as e:
        binding.attn_fwd_paged(q, kp48, kp48, table, cu_q, sk, 10, True, 0.1)
    assert e.value.code == -2
    q6 = torch.zeros(10, 6, 64, dtype=torch.bfloat16, device="cuda")            # 6 % 4 heads
    kp4 = torch.zeros(4, 16, 4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.AttnError) as e:
        binding.attn_fwd_paged(q6, kp4, kp4, table, cu_q, sk, 10, True, 0.1)
    assert e.value.code == -1
