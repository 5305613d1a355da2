"""attn_decode_paged (decode against a paged KV cache) on the GPU against the
fp64 oracle, with the logical cache gathered through the page table."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu

pytestmark = pytest.mark.gpu


def _pool(num_pages, page_size, n_kv, gen, fill=None):
    pool = torch.randn(num_pages, page_size, n_kv, 128, generator=gen, device="cuda").to(torch.bfloat16)
    if fill is not None:
        pool.fill_(fill)
    return pool


def _case(B, n_q, n_kv, page_size, pages_per_seq, lens, seed):
    """Random page assignment: each sequence's pages drawn without
    replacement from a pool with spare pages; table entries past a
    sequence's pages hold garbage ids."""
    need_gpu()
    g = torch.Generator(device="cuda").manual_seed(seed)
    rng = np.random.default_rng(seed)
    need = sum((L + page_size - 1) // page_size for L in lens)
    num_pages = need + 7
    pool_k = _pool(num_pages, page_size, n_kv, g)
    pool_v = _pool(num_pages, page_size, n_kv, g)
    ids = rng.permutation(num_pages)
    table = np.full((B, pages_per_seq), -12345, dtype=np.int32)      # garbage past the pages in use
    at = 0
    for b, L in enumerate(lens):
        n = (L + page_size - 1) // page_size
        table[b, :n] = ids[at:at + n]
        at += n
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    return q, pool_k, pool_v, torch.tensor(table, device="cuda"), torch.tensor(lens, dtype=torch.int32)


def _check(q, pk, pv, table, lens, scale, what):
    binding = need_gpu()
    o, lse = binding.attn_decode_paged(q, pk, pv, table, lens.cuda(), scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    kc = oracle.paged_to_cache(pk, table, lens)
    vc = oracle.paged_to_cache(pv, table, lens)
    o_ref, lse_ref = oracle.sdpa(q[:, :, None, :], kc, vc, False, scale, seqlens=lens.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], what)
    return o, lse


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_paged_decode_page_sizes(page_size):
    lens = [1, 700, 2049, 130]
    pps = (max(lens) + page_size - 1) // page_size
    q, pk, pv, table, sl = _case(4, 32, 8, page_size, pps, lens, 40 + page_size)
    _check(q, pk, pv, table, sl, 1 / math.sqrt(128), f"paged ps={page_size}")


@pytest.mark.parametrize("n_q,n_kv", [(8, 8), (16, 1), (64, 4)])
def test_paged_decode_group_sizes(n_q, n_kv):
    lens = [333, 1024, 65]
    q, pk, pv, table, sl = _case(3, n_q, n_kv, 64, 16, lens, 7 + n_q)
    _check(q, pk, pv, table, sl, 0.1, f"paged {n_q}/{n_kv}")


def test_paged_identity_table_equals_contiguous_decode():
    """A pool laid out sequence by sequence with the identity table is the
    contiguous cache: the same tiles in the same order, so the result is
    bit-identical to attn_decode."""
    binding = need_gpu()
    B, n_q, n_kv, S, ps = 3, 32, 8, 4096, 128
    g = torch.Generator(device="cuda").manual_seed(3)
    kc = torch.randn(B, n_kv, S, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S, 128, generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    sl = torch.tensor([4096, 1000, 3333], dtype=torch.int32, device="cuda")
    P = S // ps
    pool_k = kc.view(B, n_kv, P, ps, 128).permute(0, 2, 3, 1, 4).reshape(B * P, ps, n_kv, 128).contiguous()
    pool_v = vc.view(B, n_kv, P, ps, 128).permute(0, 2, 3, 1, 4).reshape(B * P, ps, n_kv, 128).contiguous()
    table = torch.arange(B * P, dtype=torch.int32, device="cuda").view(B, P)
    o1, l1 = binding.attn_decode(q, kc, vc, sl, 0.09)
    o2, l2 = binding.attn_decode_paged(q, pool_k, pool_v, table, sl, 0.09)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_paged_nonfinite_rows_past_the_length_and_unused_pages():
    """Rows of a sequence's last page past its length, and every page the
    table does not reference, hold NaN / Inf: no effect on the result."""
    lens = [5, 300, 1000]
    q, pk, pv, table, sl = _case(3, 16, 4, 64, 16, lens, 99)
    used = set()
    t = table.cpu().numpy()
    for b, L in enumerate(lens):
        n = (L + 63) // 64
        used.update(int(x) for x in t[b, :n])
        last = int(t[b, n - 1])
        r = L - (n - 1) * 64                        # valid rows of the last page
        pk[last, r:] = float("nan")
        pv[last, r:] = float("inf")
    for p in range(pk.shape[0]):
        if p not in used:
            pk[p] = float("nan")
            pv[p] = float("nan")
    o, lse = _check(q, pk, pv, table, sl, 0.1, "paged non-finite padding")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_paged_out_of_pool_page_reads_zeros_and_is_reported():
    binding = need_gpu()
    lens = [256, 256]
    q, pk, pv, table, sl = _case(2, 8, 2, 64, 4, lens, 5)
    table[1, 2] = pk.shape[0] + 100                  # outside the pool, below the length
    o, lse = binding.attn_decode_paged(q, pk, pv, table, sl.cuda(), 0.1)
    assert binding.device_status() == -7             # ATTN_ERR_DEVICE_RANGE
    kc = oracle.paged_to_cache(pk, table, sl)        # that page reads as zeros
    vc = oracle.paged_to_cache(pv, table, sl)
    o_ref, lse_ref = oracle.sdpa(q[:, :, None, :], kc, vc, False, 0.1, seqlens=sl.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], "page id outside the pool")


def test_paged_zero_length_and_rejects_bad_arguments():
    binding = need_gpu()
    lens = [0, 100]
    q, pk, pv, table, sl = _case(2, 8, 2, 32, 4, lens, 11)
    o, lse = _check(q, pk, pv, table, sl, 0.1, "paged zero length")
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    g = torch.Generator(device="cuda").manual_seed(1)
    bad = torch.randn(10, 48, 2, 128, generator=g, device="cuda").to(torch.bfloat16)   # page size 48
    with pytest.raises(binding.AttnError) as e:
        binding.attn_decode_paged(q, bad, bad, table, sl.cuda(), 0.1)
    assert e.value.code == -2
    with pytest.raises(binding.AttnError) as e:
        binding.attn_decode_paged(q, pk, pv, table, sl.cuda(), 0.1, workspace=torch.empty(256, dtype=torch.uint8,
                                                                                          device="cuda"))
    assert e.value.code == -4
