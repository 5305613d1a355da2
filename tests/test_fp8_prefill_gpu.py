"""attn_fwd_fp8 (e4m3 Q, K, V with one scale per 128-row tile) on the GPU
against the fp64 oracle's FP8 mode (per-tile dequantisation, then the plain
definition). The kernel sees the same e4m3 bytes and scales; its operands
are the exact bf16 images of the bytes, so the tolerances are the bf16
path's."""
import math

import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def quantize_tiles(x, tile_mag=None):
    """One scale per 128-row tile of each (sequence, head) of a [B, H, S, d]
    tensor: the tile's largest |value| maps to 448 (e4m3's largest finite).
    tile_mag, if given, multiplies each tile's values first (to spread the
    tiles' magnitudes). Returns (e4m3 bytes as float8_e4m3fn, scales fp32)."""
    B, H, S, d = x.shape
    nt = (S + 127) // 128
    xp = torch.nn.functional.pad(x.float(), (0, 0, 0, nt * 128 - S)).view(B, H, nt, 128, d)
    if tile_mag is not None:
        xp = xp * tile_mag.view(1, 1, nt, 1, 1)
    amax = xp.abs().amax(dim=(3, 4)).clamp_min(1e-6)
    scale = (amax / 448.0).to(torch.float32).contiguous()
    q8 = (xp / scale[..., None, None]).view(B, H, nt * 128, d)[:, :, :S]
    return q8.to(torch.float8_e4m3fn).contiguous(), scale


def _case(B, Sq, Skv, n_q, n_kv, causal, seed, spread=False):
    q, k, v = inputs.prefill_inputs(B, Sq, Skv, n_q, n_kv, 128, 128, seed, device="cuda")
    mag = (lambda n: torch.tensor([(0.5, 1.0, 2.0)[i % 3] for i in range(n)], device="cuda")) if spread else (
        lambda n: None)
    q8, qs = quantize_tiles(q, mag((Sq + 127) // 128))
    k8, ks = quantize_tiles(k, mag((Skv + 127) // 128))
    v8, vs = quantize_tiles(v, mag((Skv + 127) // 128))
    return q8, k8, v8, qs, ks, vs


def _check(q8, k8, v8, qs, ks, vs, causal, scale, what):
    binding = need_gpu()
    o, lse = binding.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal, scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    u8 = lambda t: t.view(torch.uint8)
    o_ref, lse_ref = oracle.sdpa_fp8(u8(q8), u8(k8), u8(v8), qs, ks, vs, causal, scale)
    check_parity(o, lse, o_ref, lse_ref, what)
    return o, lse


@pytest.mark.parametrize("B,Sq,Skv,n_q,n_kv,causal", [
    (1, 300, 300, 8, 2, True),        # G=4, ragged tail
    (2, 257, 513, 4, 4, False),       # MHA, non-causal, Sq != Skv
    (1, 1000, 1000, 32, 8, True),     # Llama-3-8B head layout
    (1, 100, 333, 16, 2, True),       # G=8, bottom-right causal
    (1, 1, 700, 8, 2, True),          # one query row
    (3, 77, 77, 2, 1, True),          # G=2
    (1, 200, 200, 1, 1, True),        # G=1, two position tiles
])
def test_fp8_prefill_shapes(B, Sq, Skv, n_q, n_kv, causal):
    q8, k8, v8, qs, ks, vs = _case(B, Sq, Skv, n_q, n_kv, causal, 500 + Sq + n_q)
    _check(q8, k8, v8, qs, ks, vs, causal, 1 / math.sqrt(128), f"fp8 prefill {B} {Sq}/{Skv} {n_q}/{n_kv} c{causal}")


def test_fp8_prefill_tile_scales_differ():
    """Tiles whose magnitudes differ by a factor of 4 (so their scales do):
    every tile's scale must reach exactly its own rows (queries: the score
    row; keys: the score column; values: the weights of the tile's rows).
    The spread stays small enough that the outputs keep unit scale, where
    the absolute O bound applies."""
    q8, k8, v8, qs, ks, vs = _case(1, 700, 900, 8, 2, True, 77, spread=True)
    assert float(ks.max() / ks.min()) > 3 and float(qs.max() / qs.min()) > 3 and float(vs.max() / vs.min()) > 3
    _check(q8, k8, v8, qs, ks, vs, True, 0.02, "fp8 prefill, tiles of spread magnitudes")


def test_fp8_prefill_llama3_8b_sampled():
    """The Llama-3-8B layout in full (B=1, S=4096, 32/8 heads), the inputs of
    the bf16 workload quantised per tile: 2000 sampled rows against the
    single-row oracle on the dequantised operands."""
    binding = need_gpu()
    w = inputs.WORKLOADS["llama3_8b_prefill"]
    q, k, v = inputs.make(w, device="cuda")
    q8, qs = quantize_tiles(q)
    k8, ks = quantize_tiles(k)
    v8, vs = quantize_tiles(v)
    o, lse = binding.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, w.causal, w.scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    qd = oracle.dequant_e4m3_tiles(q8.view(torch.uint8), qs)
    kd = oracle.dequant_e4m3_tiles(k8.view(torch.uint8), ks)
    vd = oracle.dequant_e4m3_tiles(v8.view(torch.uint8), vs)
    rows = inputs.sample_rows(2000, w.B, w.n_q, w.Sq, 21)
    rb, rh, ri = rows[:, 0].long(), rows[:, 1].long(), rows[:, 2].long()
    q_rows = qd[rb.numpy(), rh.numpy(), ri.numpy()]
    o_ref, lse_ref = oracle.sdpa_rows(q_rows, rows.numpy(), kd, vd, w.B, w.n_q, w.Sq, w.causal, w.scale)
    o_rows = o[rb.cuda(), rh.cuda(), ri.cuda()]
    lse_rows = lse[rb.cuda(), rh.cuda(), ri.cuda()]
    check_parity(o_rows, lse_rows, o_ref, lse_ref, "fp8 llama3_8b_prefill")


def test_fp8_prefill_rejects_bad_arguments():
    binding = need_gpu()
    q8, k8, v8, qs, ks, vs = _case(1, 130, 130, 4, 2, True, 3)
    with pytest.raises(ValueError):
        binding.attn_fwd_fp8(q8, k8, v8, qs[:, :, :1].contiguous(), ks, vs, True, 0.1)   # wrong scale shape
    q64 = torch.zeros(1, 4, 130, 64, dtype=torch.uint8, device="cuda")
    k64 = torch.zeros(1, 2, 130, 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.AttnError) as e:
        binding.attn_fwd_fp8(q64, k64, k64, qs, ks, vs, True, 0.1)                       # head dim 64
    assert e.value.code == -2
