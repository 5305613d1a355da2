"""Randomised shapes through the CUDA path against the fp64 oracle.

The parametrised tests elsewhere pin chosen shapes (tile edges, ragged tails,
head-group sizes); these draw shapes at random (a fixed, derandomised
hypothesis search, so a run is repeatable) over the supported space: head
group sizes, head dims, lengths on and off the 128-row/128-key tiles, causal
and not, batches with empty sequences, windows with sink keys, the MLA
latent decode and the paged decode.
"""
import math

import pytest
import torch
from hypothesis import given, settings, HealthCheck
from hypothesis import strategies as st

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu

_SETTINGS = settings(max_examples=24, deadline=None, derandomize=True, database=None,
                     suppress_health_check=list(HealthCheck))


@st.composite
def prefill_shapes(draw):
    n_kv = draw(st.sampled_from([1, 2, 4]))
    G = draw(st.sampled_from([1, 2, 4, 8, 16]))
    d = draw(st.sampled_from([32, 64, 128]))
    B = draw(st.integers(1, 2))
    causal = draw(st.booleans())
    Sq = draw(st.integers(1, 384))
    Skv = Sq + draw(st.integers(0, 320)) if causal else draw(st.integers(1, 600))
    return B, Sq, Skv, n_kv * G, n_kv, d, causal


@_SETTINGS
@given(prefill_shapes(), st.integers(0, 2**31 - 1))
def test_prefill_random_shapes(shape, seed):
    binding = need_gpu()
    B, Sq, Skv, n_q, n_kv, d, causal = shape
    scale = 1.0 / math.sqrt(d)
    q, k, v = inputs.prefill_inputs(B, Sq, Skv, n_q, n_kv, d, d, seed, device="cuda")
    o, lse = binding.attn_fwd(q, k, v, causal, scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa(q, k, v, causal, scale)
    check_parity(o, lse, o_ref, lse_ref, f"prefill {shape}")


@st.composite
def decode_shapes(draw):
    n_kv = draw(st.sampled_from([1, 2, 8]))
    G = draw(st.sampled_from([1, 2, 4, 8, 16, 32]))
    B = draw(st.integers(1, 5))
    S_max = draw(st.integers(1, 3000))
    # lengths anywhere in [0, S_max], an empty sequence included sometimes
    lens = draw(st.lists(st.integers(0, S_max), min_size=B, max_size=B))
    return B, n_kv * G, n_kv, S_max, lens


@_SETTINGS
@given(decode_shapes(), st.integers(0, 2**31 - 1))
def test_decode_random_shapes(shape, seed):
    binding = need_gpu()
    B, n_q, n_kv, S_max, lens = shape
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    seq = torch.tensor(lens, dtype=torch.int32)
    scale = 1.0 / math.sqrt(128)
    o, lse = binding.attn_decode(q, kc, vc, seq.cuda(), scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa(q[:, :, None, :], kc, vc, False, scale, seqlens=seq.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], f"decode {shape}")


@st.composite
def window_shapes(draw):
    n_kv = draw(st.sampled_from([1, 2, 4]))
    G = draw(st.sampled_from([1, 2, 4, 8]))
    Sq = draw(st.integers(1, 320))
    Skv = Sq + draw(st.integers(0, 400))
    W = draw(st.integers(1, Skv + 64))
    n_sink = draw(st.integers(0, 200))
    return 1, Sq, Skv, n_kv * G, n_kv, W, n_sink


@_SETTINGS
@given(window_shapes(), st.integers(0, 2**31 - 1))
def test_window_prefill_random_shapes(shape, seed):
    binding = need_gpu()
    B, Sq, Skv, n_q, n_kv, W, n_sink = shape
    scale = 1.0 / math.sqrt(128)
    q, k, v = inputs.prefill_inputs(B, Sq, Skv, n_q, n_kv, 128, 128, seed, device="cuda")
    o, lse = binding.attn_fwd_window(q, k, v, W, n_sink, scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa_window(q, k, v, True, W, n_sink, scale)
    check_parity(o, lse, o_ref, lse_ref, f"window prefill {shape}")


@_SETTINGS
@given(decode_shapes(), st.integers(1, 3000), st.integers(0, 300), st.integers(0, 2**31 - 1))
def test_window_decode_random_shapes(shape, W, n_sink, seed):
    binding = need_gpu()
    B, n_q, n_kv, S_max, lens = shape
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    seq = torch.tensor(lens, dtype=torch.int32)
    o, lse = binding.attn_decode_window(q, kc, vc, seq.cuda(), W, n_sink, 0.1)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa_window(q[:, :, None, :], kc, vc, False, W, n_sink, 0.1, seqlens=seq.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], f"window decode {shape} W={W} sinks={n_sink}")


@st.composite
def mla_shapes(draw):
    B = draw(st.integers(1, 3))
    n_q = draw(st.sampled_from([128, 256]))
    S_max = draw(st.integers(1, 2500))
    lens = draw(st.lists(st.integers(0, S_max), min_size=B, max_size=B))
    return B, n_q, S_max, lens


@settings(max_examples=12, deadline=None, derandomize=True, database=None, suppress_health_check=list(HealthCheck))
@given(mla_shapes(), st.integers(0, 2**31 - 1))
def test_mla_decode_random_shapes(shape, seed):
    """The absorbed MLA decode (576-wide latent rows, values = their first
    512 columns) over random batches, lengths and one or two head blocks:
    batches too small to fill the SMs are split over key chunks."""
    binding = need_gpu()
    B, n_q, S_max, lens = shape
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, n_q, 576, generator=g, device="cuda").to(torch.bfloat16)
    cache = torch.randn(B, S_max, 576, generator=g, device="cuda").to(torch.bfloat16)
    seq = torch.tensor(lens, dtype=torch.int32)
    c4 = cache[:, None]
    scale = 1.0 / math.sqrt(192)
    o, lse = binding.attn_decode(q, c4, c4, seq.cuda(), scale, d_v=512)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa(q[:, :, None, :], c4, c4, False, scale, seqlens=seq.numpy(), d_v=512)
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], f"mla decode {shape}")


@st.composite
def paged_shapes(draw):
    page = draw(st.sampled_from([16, 32, 64, 128, 256]))
    n_kv = draw(st.sampled_from([1, 2, 8]))
    G = draw(st.sampled_from([1, 2, 4, 8]))
    B = draw(st.integers(1, 4))
    lens = draw(st.lists(st.integers(0, 2000), min_size=B, max_size=B))
    return B, n_kv * G, n_kv, page, lens


@settings(max_examples=16, deadline=None, derandomize=True, database=None, suppress_health_check=list(HealthCheck))
@given(paged_shapes(), st.integers(0, 2**31 - 1))
def test_paged_decode_random_shapes(shape, seed):
    """The paged decode with random page sizes, group sizes and lengths, each
    sequence's pages drawn at random from a pool with spare pages."""
    from test_paged_decode_gpu import _case, _check
    B, n_q, n_kv, page, lens = shape
    pages_per_seq = max(1, -(-max(lens) // page)) + 1
    q, pk, pv, table, sl = _case(B, n_q, n_kv, page, pages_per_seq, lens, seed % 100000)
    _check(q, pk, pv, table, sl, 1.0 / math.sqrt(128), f"paged decode {shape}")
