"""attn_decode_fp8 (GQA decode against an e4m3 KV cache with per-KV-head
scales) and attn_decode_fp8_tiles (one scale per 128-key tile of each
sequence and KV head) on the GPU against the fp64 oracle run on the
dequantized cache."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def _quantize(x, n_kv):
    """Per-KV-head scale so that the head's largest |value| maps to 448."""
    amax = x.float().abs().amax(dim=(0, 2, 3)).clamp_min(1e-6)
    scale = (amax / 448.0).to(torch.float32)
    q8 = (x.float() / scale[None, :, None, None]).to(torch.float8_e4m3fn)
    return q8, scale.contiguous()


def _case(B, n_q, n_kv, S_max, lens, seed, spread=1.0):
    need_gpu()
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda") * spread
    v = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda") * spread
    k8, ks = _quantize(k, n_kv)
    v8, vs = _quantize(v, n_kv)
    return q, k8, v8, ks, vs, torch.tensor(lens, dtype=torch.int32)


def _check(q, k8, v8, ks, vs, sl, scale, what):
    binding = need_gpu()
    o, lse = binding.attn_decode_fp8(q, k8, v8, ks, vs, sl.cuda(), scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    kd = oracle.dequant_e4m3(k8.view(torch.uint8), ks)
    vd = oracle.dequant_e4m3(v8.view(torch.uint8), vs)
    o_ref, lse_ref = oracle.sdpa(q[:, :, None, :], kd, vd, False, scale, seqlens=sl.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], what)
    return o, lse


@pytest.mark.parametrize("B,n_q,n_kv,S_max,lens", [
    (3, 32, 8, 3000, [1, 700, 3000]),        # G=4, ragged, tail tiles
    (2, 8, 8, 1100, [1100, 513]),            # MHA
    (2, 16, 2, 2048, [2048, 129]),           # G=8
    (1, 32, 1, 1500, [1500]),                # MQA (G=32: two head blocks of 16)
])
def test_fp8_decode_shapes(B, n_q, n_kv, S_max, lens):
    q, k8, v8, ks, vs, sl = _case(B, n_q, n_kv, S_max, lens, B * 10 + n_q)
    _check(q, k8, v8, ks, vs, sl, 1 / 128 ** 0.5, f"fp8 {B} {n_q}/{n_kv}")


def test_fp8_decode_scales_and_small_values():
    """Values over the whole e4m3 range (the per-head amax maps to 448, so the
    small ones are subnormal) and different scales per head: sharper and
    flatter softmaxes, larger and smaller values (kept to outputs of a few
    units, where the bf16 output rounding stays inside the tolerance)."""
    q, k8, v8, ks, vs, sl = _case(2, 16, 4, 2000, [2000, 777], 5)
    ks = ks * torch.tensor([1.0, 3.0, 0.01, 2.0], device="cuda")
    vs = vs * torch.tensor([0.1, 1.0, 1.5, 0.5], device="cuda")
    _check(q, k8, v8, ks.contiguous(), vs.contiguous(), sl, 0.05, "fp8 scales")


def test_fp8_decode_nan_past_the_length():
    """e4m3 NaN bytes past each sequence's length take no part."""
    q, k8, v8, ks, vs, sl = _case(2, 32, 8, 1000, [37, 1000 - 5], 6)
    kb, vb = k8.view(torch.uint8), v8.view(torch.uint8)
    for b, L in enumerate(sl.tolist()):
        kb[b, :, L:] = 0x7F
        vb[b, :, L:] = 0xFF
    o, lse = _check(q, k8, v8, ks, vs, sl, 0.1, "fp8 NaN padding")
    assert torch.isfinite(o.float()).all()


def test_fp8_decode_gqa_workload_against_oracle_and_bf16_path():
    """The GQA decode workload quantized to e4m3: every row equals attn_decode
    on the dequantized cache (rounded back to bf16, exact for e4m3 values
    times a power-of-two scale) within the parity tolerances, and the rows of
    four of its sequences (every head, the shortest and longest lengths
    among them) equal the fp64 oracle on the dequantized cache."""
    binding = need_gpu()
    w = inputs.WORKLOADS["gqa_decode"]
    seqlens, q, kc, vc = inputs.make(w, device="cuda")
    # power-of-two scales keep e4m3 * scale exact in bf16
    ks = torch.full((w.n_kv,), 2.0 ** -6, device="cuda")
    vs = torch.full((w.n_kv,), 2.0 ** -6, device="cuda")
    k8 = (kc.float() / 2.0 ** -6).to(torch.float8_e4m3fn)
    v8 = (vc.float() / 2.0 ** -6).to(torch.float8_e4m3fn)
    sl = seqlens.cuda()
    o8, l8 = binding.attn_decode_fp8(q, k8, v8, ks, vs, sl, w.scale)
    kd = (k8.float() * 2.0 ** -6).to(torch.bfloat16)
    vd = (v8.float() * 2.0 ** -6).to(torch.bfloat16)
    ob, lb = binding.attn_decode(q, kd, vd, sl, w.scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    assert float((o8.float() - ob.float()).abs().max()) <= 2e-2
    assert float((l8 - lb).abs().max()) <= 1e-3
    order = torch.argsort(seqlens)
    pick = sorted({int(order[0]), int(order[-1]), 1, 2})
    for b in pick:
        L = int(seqlens[b])
        kq = oracle.dequant_e4m3(k8[b:b + 1, :, :L].view(torch.uint8), ks)
        vq = oracle.dequant_e4m3(v8[b:b + 1, :, :L].view(torch.uint8), vs)
        o_ref, l_ref = oracle.sdpa(q[b:b + 1, :, None, :], kq, vq, False, w.scale)
        check_parity(o8[b:b + 1], l8[b:b + 1], o_ref[:, :, 0], l_ref[:, :, 0], f"fp8 gqa_decode sequence {b} (L={L})")


def test_fp8_decode_rejects_bad_arguments():
    binding = need_gpu()
    q, k8, v8, ks, vs, sl = _case(1, 8, 2, 256, [100], 7)
    with pytest.raises(binding.AttnError) as e:
        binding.attn_decode_fp8(q, k8, v8, ks, vs, sl.cuda(), 0.1, workspace=torch.empty(256, dtype=torch.uint8,
                                                                                         device="cuda"))
    assert e.value.code == -4
    q6 = torch.zeros(1, 6, 128, dtype=torch.bfloat16, device="cuda")   # 6 query heads over 2: G = 3
    with pytest.raises(binding.AttnError) as e:
        binding.attn_decode_fp8(q6, k8, v8, ks, vs, sl.cuda(), 0.1)
    assert e.value.code == -2


def _quantize_tiles(x):
    """One scale per 128-key tile of each (sequence, KV head): the tile's
    largest |value| maps to 448. Returns (e4m3 cache, scales [B, n_kv, tiles])."""
    B, n_kv, S, d = x.shape
    nt = (S + 127) // 128
    xp = torch.nn.functional.pad(x.float(), (0, 0, 0, nt * 128 - S))
    amax = xp.view(B, n_kv, nt, 128, d).abs().amax(dim=(3, 4)).clamp_min(1e-6)
    scale = (amax / 448.0).to(torch.float32).contiguous()
    q8 = (xp.view(B, n_kv, nt, 128, d) / scale[..., None, None]).view(B, n_kv, nt * 128, d)[:, :, :S]
    return q8.to(torch.float8_e4m3fn).contiguous(), scale


def _check_tiles(q, k8, v8, ks, vs, sl, scale, what):
    binding = need_gpu()
    o, lse = binding.attn_decode_fp8_tiles(q, k8, v8, ks, vs, sl.cuda(), scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    kd = oracle.dequant_e4m3_tiles(k8.view(torch.uint8), ks)
    vd = oracle.dequant_e4m3_tiles(v8.view(torch.uint8), vs)
    o_ref, lse_ref = oracle.sdpa(q[:, :, None, :], kd, vd, False, scale, seqlens=sl.numpy())
    check_parity(o, lse, o_ref[:, :, 0], lse_ref[:, :, 0], what)
    return o, lse


@pytest.mark.parametrize("B,n_q,n_kv,S_max,lens", [
    (3, 32, 8, 3000, [1, 700, 3000]),        # G=4, ragged, tail tiles
    (2, 8, 8, 1100, [1100, 513]),            # MHA
    (2, 16, 2, 2300, [2300, 129]),           # G=8, more than one chunk
])
def test_fp8_tile_scales_shapes(B, n_q, n_kv, S_max, lens):
    need_gpu()
    g = torch.Generator(device="cuda").manual_seed(B * 7 + n_q)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda")
    v = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda")
    k8, ks = _quantize_tiles(k)
    v8, vs = _quantize_tiles(v)
    _check_tiles(q, k8, v8, ks, vs, torch.tensor(lens, dtype=torch.int32), 1 / 128 ** 0.5,
                 f"fp8 tile scales {B} {n_q}/{n_kv}")


def test_fp8_tile_scales_varying_magnitudes():
    """Tiles whose keys and values differ in magnitude by up to 100x (so that
    per-head scales would leave the small tiles to a few e4m3 levels): each
    tile's own scale keeps them exact to e4m3 precision."""
    need_gpu()
    g = torch.Generator(device="cuda").manual_seed(17)
    B, n_q, n_kv, S = 2, 16, 4, 1500
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    mag = torch.exp2(torch.randint(-5, 2, (B, n_kv, (S + 127) // 128, 1, 1), generator=g,
                                   device="cuda").float())
    grow = lambda x: (x.view(B, n_kv, -1, 128, 128) * mag[:, :, :x.shape[2] // 128]).view(x.shape)
    k = torch.randn(B, n_kv, 1536, 128, generator=g, device="cuda")
    v = torch.randn(B, n_kv, 1536, 128, generator=g, device="cuda")
    k, v = grow(k)[:, :, :S], grow(v)[:, :, :S]
    k8, ks = _quantize_tiles(k)
    v8, vs = _quantize_tiles(v)
    _check_tiles(q, k8, v8, ks, vs, torch.tensor([S, 901], dtype=torch.int32), 0.05, "fp8 tile magnitudes")


def test_fp8_tile_scales_equal_to_per_head():
    """Tile scales all equal to the per-head scale: the same attention as
    attn_decode_fp8 on the same bytes."""
    binding = need_gpu()
    q, k8, v8, ks, vs, sl = _case(2, 32, 8, 2100, [2100, 640], 23)
    nt = (2100 + 127) // 128
    kt = ks[None, :, None].expand(2, 8, nt).contiguous()
    vt = vs[None, :, None].expand(2, 8, nt).contiguous()
    o1, l1 = binding.attn_decode_fp8(q, k8, v8, ks, vs, sl.cuda(), 0.09)
    o2, l2 = binding.attn_decode_fp8_tiles(q, k8, v8, kt, vt, sl.cuda(), 0.09)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2
    assert float((l1 - l2).abs().max()) <= 1e-3


def test_fp8_tile_scales_rejects_bad_arguments():
    binding = need_gpu()
    q, k8, v8, ks, vs, sl = _case(1, 8, 2, 300, [300], 29)
    good = torch.ones(1, 2, 3, device="cuda")
    with pytest.raises(ValueError):
        binding.attn_decode_fp8_tiles(q, k8, v8, torch.ones(1, 2, 2, device="cuda"), good, sl.cuda(), 0.1)
    with pytest.raises(ValueError):
        binding.attn_decode_fp8_tiles(q, k8, v8, good, good.double(), sl.cuda(), 0.1)
