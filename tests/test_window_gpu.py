"""Sliding-window attention with sink keys (attn_fwd_window, attn_decode_window)
on the GPU against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Sq,Skv,n_q,n_kv,d,W,ns", [
    (1, 1000, 1000, 32, 8, 128, 256, 0),     # G=4, window of two key tiles
    (1, 1000, 1000, 32, 8, 128, 300, 4),     # window with 4 sink keys
    (2, 700, 700, 16, 2, 128, 1, 0),         # window of one: each row returns its own value
    (1, 513, 513, 4, 4, 64, 129, 130),       # MHA (G=1), sinks spanning two tiles
    (1, 300, 1300, 8, 1, 128, 200, 16),      # bottom-right: queries at the end of a longer context
    (1, 640, 640, 8, 2, 32, 5000, 0),        # window wider than the sequence = causal
])
def test_window_prefill(B, Sq, Skv, n_q, n_kv, d, W, ns):
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(B, Sq, Skv, n_q, n_kv, d, d, 300 + W + ns, device="cuda")
    scale = 1 / math.sqrt(d)
    o, lse = binding.attn_fwd_window(q, k, v, W, ns, scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa_window(q, k, v, True, W, ns, scale)
    check_parity(o, lse, o_ref, lse_ref, f"window W={W} sinks={ns}")
    if W == 1 and ns == 0:
        G = n_q // n_kv
        for h in range(n_q):
            assert torch.equal(o[:, h], v[:, h // G, Skv - Sq:])


def test_window_wider_than_context_equals_causal_bitwise():
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(1, 1024, 1024, 32, 8, 128, 128, 17, device="cuda")
    o1, l1 = binding.attn_fwd(q, k, v, True, 0.08)
    o2, l2 = binding.attn_fwd_window(q, k, v, 1024, 0, 0.08)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("W,ns", [(512, 0), (1000, 4), (3000, 1030), (1, 0), (40000, 0)])
def test_window_decode(W, ns):
    binding = need_gpu()
    B, n_q, n_kv, S_max = 4, 32, 8, 6000
    seq = torch.tensor([1, 700, 2500, 6000], dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(W + ns)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    o, lse = binding.attn_decode_window(q, kc, vc, seq.cuda(), W, ns, 0.1)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa_window(q[:, :, None, :], kc, vc, False, W, ns, 0.1, seqlens=seq.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], f"decode window W={W} sinks={ns}")


def test_window_decode_skips_unread_chunks():
    """Keys outside the window and the sinks may hold NaN: the chunks that
    hold only such keys are not read, and the masked keys of partly visible
    chunks get weight 0 (finite values there, as the cache below the length
    must hold)."""
    binding = need_gpu()
    B, n_q, n_kv, S_max, W, ns = 2, 16, 4, 8192, 700, 2
    seq = torch.tensor([8192, 5000], dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(4)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    for b, L in enumerate(seq.tolist()):
        # whole 2048-key spans between the sinks' chunk and the window's first
        # chunk: never read, whatever chunk length (a whole number of 128-key
        # tiles up to 2048) the launch plans
        lo = (L - W) // 2048 * 2048
        kc[b, :, 2048:lo] = float("nan")
        vc[b, :, 2048:lo] = float("nan")
    o, lse = binding.attn_decode_window(q, kc, vc, seq.cuda(), W, ns, 0.1)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    o_ref, lse_ref = oracle.sdpa_window(q[:, :, None, :], kc, vc, False, W, ns, 0.1, seqlens=seq.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], "decode window with NaN outside")


def test_window_rejects_bad_arguments():
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(1, 64, 64, 4, 2, 64, 64, 1, device="cuda")
    for W, ns in [(0, 0), (5, -1)]:
        with pytest.raises(binding.AttnError) as e:
            binding.attn_fwd_window(q, k, v, W, ns, 0.1)
        assert e.value.code == -1
    q2, k2, v2 = inputs.prefill_inputs(1, 65, 64, 4, 2, 64, 64, 1, device="cuda")
    with pytest.raises(binding.AttnError) as e:                         # Sq > Skv
        binding.attn_fwd_window(q2, k2, v2, 8, 0, 0.1)
    assert e.value.code == -2
