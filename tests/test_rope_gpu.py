"""Rotary position embedding on the GPU (attn_rope_tables, attn_rope_apply,
attn_fwd_rope, attn_decode_rope) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def _bf16_ulp(x):
    """One unit in the last place of bf16 at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def _rotated_bf16(x, c, s, pos):
    """The oracle's rotated operand rounded to bf16, and per element the size
    of a possible disagreement with the kernel's: the kernel rotates in fp32
    (error below 4 * 2^-24 * (|x_2j| + |x_2j+1|)), so where the fp64 value lies
    that close to a bf16 rounding midpoint the two may round one ulp apart."""
    r64 = oracle.rope(x, c, s, pos)
    r = oracle.round_bf16(r64)
    xa = np.abs(x.double().cpu().numpy())
    eps = 4 * 2.0 ** -24 * np.repeat(xa[..., 0::2] + xa[..., 1::2], 2, axis=-1)
    ulp = np.maximum(_bf16_ulp(r), _bf16_ulp(r64))
    flip = np.where(np.abs(np.abs(r64 - r) - _bf16_ulp(r) / 2) <= eps, ulp, 0.0)
    return r, flip


def _check_rope_prefill(o, lse, q, k, v, causal, scale, c, s, what):
    """O against the oracle on bf16-rounded rotated operands with the usual
    tolerances; LSE within 1e-3 plus, per row, the largest score change that
    the possible one-ulp rounding disagreements of its q and of the visible
    keys can make (LSE moves by at most the largest score change)."""
    B, n_q, Sq, d = q.shape
    _, n_kv, Skv, _ = k.shape
    qr, fq = _rotated_bf16(q, c, s, np.arange(Skv - Sq, Skv))
    kr, fk = _rotated_bf16(k, c, s, np.arange(Skv))
    o_ref, lse_ref = oracle.sdpa(qr, kr, v, causal, scale)
    check_parity(o, None, o_ref, None, what)
    G = n_q // n_kv
    g = np.repeat(np.arange(n_kv), G)
    kra, qra = np.abs(kr[:, g]), np.abs(qr)
    ds = scale * (np.einsum("bhid,bhjd->bhij", fq, kra + fk[:, g]) + np.einsum("bhid,bhjd->bhij", qra, fk[:, g]))
    if causal:
        vis = np.arange(Skv)[None, :] <= (np.arange(Sq) + Skv - Sq)[:, None]
        ds = np.where(vis, ds, 0.0)
    widen = ds.max(axis=3)
    tol = 1e-3 + widen
    lg = lse.double().cpu().numpy()
    assert np.all(np.abs(lg - lse_ref) <= tol), f"{what}: LSE excess {float((np.abs(lg - lse_ref) - tol).max()):.3e}"
    # the widening is a worst-case rounding allowance (every possible flip
    # against the largest entries), not the error seen: report both, and the
    # rows whose deviation actually needed it
    w_max = float(widen.max()) if widen.size else 0.0
    dl = np.abs(lg - lse_ref)
    print(f"{what}: largest per-row LSE widening {w_max:.3e}, rows widened {int((widen > 0).sum())} of {widen.size}, "
          f"largest |dLSE| {float(dl.max()):.3e}, rows beyond 1e-3 {int((dl > 1e-3).sum())}")
    return int((fq > 0).sum() + (fk > 0).sum()), w_max


@pytest.mark.parametrize("n_pos,d,base", [(32768, 128, 500000.0), (4096, 64, 10000.0), (77, 32, 10000.0)])
def test_tables_match_oracle(n_pos, d, base):
    binding = need_gpu()
    c, s = binding.rope_tables(n_pos, d, base)
    torch.cuda.synchronize()
    cr, sr = oracle.rope_tables(n_pos, d, base)
    # one fp32 rounding of values in [-1, 1]
    assert np.max(np.abs(c.cpu().numpy() - cr)) <= 6e-8
    assert np.max(np.abs(s.cpu().numpy() - sr)) <= 6e-8


@pytest.mark.parametrize("B,H,S,d,pos0", [(2, 3, 257, 128, 0), (1, 8, 100, 64, 900), (3, 1, 5, 32, 7)])
def test_apply_matches_oracle(B, H, S, d, pos0):
    binding = need_gpu()
    c, s = binding.rope_tables(pos0 + S + 3, d, 10000.0)
    g = torch.Generator(device="cuda").manual_seed(S + d)
    x = (torch.randn(B, H, S, d, generator=g, device="cuda") * 3).to(torch.bfloat16)
    y = binding.rope_apply(x, c, s, pos0=pos0)
    torch.cuda.synchronize()
    ref = oracle.rope(x, c, s, np.arange(pos0, pos0 + S))
    diff = np.abs(y.double().cpu().numpy() - ref)
    # bf16 rounding of the result, plus the fp32 error of the two products
    # (which matters where they cancel): |x_2j| + |x_2j+1| per plane
    xa = np.abs(x.double().cpu().numpy())
    plane = np.repeat(xa[..., 0::2] + xa[..., 1::2], 2, axis=-1)
    tol = _bf16_ulp(ref) / 2 + 4 * 2.0 ** -24 * plane
    assert np.all(diff <= tol), float((diff / tol).max())
    # in place gives the same words
    x2 = x.clone()
    binding.rope_apply(x2, c, s, pos0=pos0, out=x2)
    torch.cuda.synchronize()
    assert torch.equal(x2, y)
    # position 0 is the identity
    if pos0 == 0:
        assert torch.equal(y[:, :, 0], x[:, :, 0])


@pytest.mark.parametrize("B,Sq,Skv,n_q,n_kv,d,causal", [
    (2, 300, 300, 8, 2, 128, True),      # G=4, ragged last tile
    (1, 200, 517, 16, 2, 128, False),    # G=8, queries at the end of a longer context
    (1, 130, 390, 4, 4, 64, True),       # MHA, bottom-right causal
    (2, 64, 64, 4, 2, 32, True),         # the tiny layout
    (1, 1, 700, 32, 8, 128, True),       # one query row
])
def test_fwd_rope_matches_oracle(B, Sq, Skv, n_q, n_kv, d, causal):
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(B, Sq, Skv, n_q, n_kv, d, d, 500 + Sq + d, device="cuda")
    c, s = binding.rope_tables(Skv + 5, d, 500000.0)
    scale = 1 / math.sqrt(d)
    o, lse, k_rot = binding.attn_fwd_rope(q, k, v, causal, scale, c, s)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    _check_rope_prefill(o, lse, q, k, v, causal, scale, c, s, f"rope prefill {B},{Sq},{Skv},{n_q},{n_kv},{d}")
    # the rotated keys it wrote are the rotation of k
    assert torch.equal(k_rot, binding.rope_apply(k, c, s))


def test_fwd_rope_equals_attention_on_rotated_inputs_bitwise():
    """Rotating Q in shared memory gives the very bf16 words of the separate
    rotation, so the fused path equals attn_fwd on rope_apply'd q and k bit
    for bit."""
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(1, 1024, 1024, 32, 8, 128, 128, 41, device="cuda")
    c, s = binding.rope_tables(1024, 128, 500000.0)
    o1, l1, _ = binding.attn_fwd_rope(q, k, v, True, 0.08, c, s)
    o2, l2 = binding.attn_fwd(binding.rope_apply(q, c, s), binding.rope_apply(k, c, s), v, True, 0.08)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_rope_in_place_keys():
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(1, 256, 256, 8, 2, 128, 128, 43, device="cuda")
    c, s = binding.rope_tables(256, 128, 10000.0)
    o1, l1, kr = binding.attn_fwd_rope(q, k, v, True, 0.09, c, s)
    k2 = k.clone()
    o2, l2, kr2 = binding.attn_fwd_rope(q, k2, v, True, 0.09, c, s, k_rot=k2)
    torch.cuda.synchronize()
    assert kr2.data_ptr() == k2.data_ptr()
    assert torch.equal(k2, kr) and torch.equal(o1, o2) and torch.equal(l1, l2)


def test_llama3_8b_prefill_rope_sampled():
    """Full-size Llama-3-8B layout with RoPE (base 500000, 4096 positions):
    2000 sampled rows against the single-row oracle on rotated q and k."""
    binding = need_gpu()
    w = inputs.WORKLOADS["llama3_8b_prefill"]
    q, k, v = inputs.make(w, device="cuda")
    c, s = binding.rope_tables(w.Skv, w.d_qk, 500000.0)
    o, lse, _ = binding.attn_fwd_rope(q, k, v, w.causal, w.scale, c, s)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    rows = inputs.sample_rows(2000, w.B, w.n_q, w.Sq, 12)
    rb, rh, ri = rows[:, 0].long(), rows[:, 1].long(), rows[:, 2].long()
    # rotated operands are bf16 activations (see oracle.sdpa_rope)
    q_rows, fq = _rotated_bf16(q[rb.cuda(), rh.cuda(), ri.cuda()], c, s, (ri + (w.Skv - w.Sq)).numpy())
    k_rot, fk = _rotated_bf16(k, c, s, np.arange(w.Skv))
    o_ref, lse_ref = oracle.sdpa_rows(q_rows, rows.numpy(), k_rot, v, w.B, w.n_q, w.Sq, w.causal, w.scale)
    check_parity(o[rb.cuda(), rh.cuda(), ri.cuda()], None, o_ref, None, "llama3_8b_prefill rope")
    # LSE: 1e-3 plus the largest score change possible one-ulp disagreements
    # of the row's q (against the largest key entries) and of the keys make
    kabs = np.abs(k_rot).max(axis=2)[0]                                        # [n_kv, d]
    fkmax = fk.max(axis=2)[0]
    g = (rows[:, 1].numpy() // (w.n_q // w.n_kv))
    tol = 1e-3 + w.scale * (np.einsum("nd,nd->n", fq, kabs[g] + fkmax[g]) +
                            np.einsum("nd,nd->n", np.abs(q_rows), fkmax[g]))
    lg = lse[rb.cuda(), rh.cuda(), ri.cuda()].double().cpu().numpy()
    dl = np.abs(lg - lse_ref)
    print(f"llama3_8b_prefill rope: largest per-row LSE widening {float((tol - 1e-3).max()):.3e}, "
          f"largest |dLSE| {float(dl.max()):.3e}, rows beyond 1e-3 {int((dl > 1e-3).sum())} of {len(dl)}")
    assert np.all(dl <= tol)


@pytest.mark.parametrize("n_q,n_kv", [(32, 8), (64, 4), (8, 8)])
def test_decode_rope_matches_oracle(n_q, n_kv):
    binding = need_gpu()
    B, S_max = 4, 3000
    seq = torch.tensor([1, 129, 2048, 3000], dtype=torch.int32)
    g = torch.Generator(device="cuda").manual_seed(n_q)
    q = torch.randn(B, n_q, 128, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)   # rotated keys
    vc = torch.randn(B, n_kv, S_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    c, s = binding.rope_tables(S_max, 128, 500000.0)
    o, lse = binding.attn_decode_rope(q, kc, vc, seq.cuda(), 0.088, c, s)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    q_rot, fq = _rotated_bf16(q, c, s, (seq.numpy() - 1)[:, None])
    o_ref, lse_ref = oracle.sdpa(q_rot[:, :, None, :], kc, vc, False, 0.088, seqlens=seq.numpy())
    check_parity(o, None, o_ref[:, :, 0], None, f"rope decode G={n_q // n_kv}")
    # LSE: 1e-3 plus the score change a one-ulp rounding disagreement of q can make
    kmax = np.abs(kc.double().cpu().numpy()).max(axis=2)                     # [B, n_kv, d]
    tol = 1e-3 + 0.088 * np.einsum("bhd,bhd->bh", fq, kmax[:, np.arange(n_q) // (n_q // n_kv)])
    assert np.all(np.abs(lse.double().cpu().numpy() - lse_ref[:, :, 0]) <= tol)
    # bitwise: the same as attn_decode on the separately rotated query
    q_sep = torch.empty_like(q)
    for b in range(B):
        q_sep[b] = binding.rope_apply(q[b:b + 1, :, None, :].contiguous(), c, s, pos0=int(seq[b]) - 1)[0, :, 0]
    o2, l2 = binding.attn_decode(q_sep, kc, vc, seq.cuda(), 0.088)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_decode_rope_length_past_tables_is_reported():
    binding = need_gpu()
    B, n_q, n_kv, S_max = 2, 8, 2, 600
    seq = torch.tensor([600, 10], dtype=torch.int32, device="cuda")
    q = torch.randn(B, n_q, 128, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, n_kv, S_max, 128, device="cuda").to(torch.bfloat16)
    c, s = binding.rope_tables(300, 128, 10000.0)     # positions 0 .. 299 only
    o, _ = binding.attn_decode_rope(q, kc, kc, seq, 0.1, c, s)
    status = binding.device_status()
    assert status == -7, status          # ATTN_ERR_DEVICE_RANGE
    assert torch.isfinite(o.float()).all()


def test_rope_argument_checks():
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(1, 64, 64, 4, 2, 128, 128, 1, device="cuda")
    c, s = binding.rope_tables(63, 128, 10000.0)            # fewer positions than keys
    with pytest.raises(RuntimeError):
        binding.attn_fwd_rope(q, k, v, True, 0.1, c, s)
    with pytest.raises(RuntimeError):
        binding.rope_apply(k, c, s, pos0=1)                 # positions 1 .. 64 > 62
    with pytest.raises(RuntimeError):                      # MLA shape: no rotation there
        binding.attn_decode_rope(torch.zeros(1, 128, 576, dtype=torch.bfloat16, device="cuda"),
                                 torch.zeros(1, 1, 64, 576, dtype=torch.bfloat16, device="cuda"),
                                 torch.zeros(1, 1, 64, 576, dtype=torch.bfloat16, device="cuda"),
                                 torch.ones(1, dtype=torch.int32, device="cuda"), 0.1, c, s)
