"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import torch
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(oracle.load())


def test_paged_to_cache_round_trip():
    """A cache cut into pages under a random page permutation and gathered
    back through the table is the cache again; an identity table on a pool
    laid out sequence by sequence is a plain reshape; ids outside the pool
    and rows past the length read as zero."""
    rng = np.random.default_rng(5)
    B, n_kv, P, ps, d = 3, 2, 5, 4, 3
    cache = rng.standard_normal((B, n_kv, P * ps, d))
    perm = rng.permutation(B * P)                  # logical page (b, p) -> pool page perm[b*P+p]
    pool = np.zeros((B * P, ps, n_kv, d))
    for b in range(B):
        for p in range(P):
            pool[perm[b * P + p]] = cache[b, :, p * ps:(p + 1) * ps, :].transpose(1, 0, 2)
    table = perm.reshape(B, P)
    full = [P * ps] * B
    assert np.array_equal(oracle.paged_to_cache(pool, table, full), cache)
    # identity table: pool page b*P+p holds tokens p*ps .. of sequence b
    ident = np.arange(B * P).reshape(B, P)
    pool2 = cache.reshape(B, n_kv, P, ps, d).transpose(0, 2, 3, 1, 4).reshape(B * P, ps, n_kv, d)
    assert np.array_equal(oracle.paged_to_cache(pool2, ident, full), cache)
    # a length of 6 keeps rows 0..5; an id past the pool reads zeros
    t2 = table.copy()
    t2[1, 0] = B * P + 3
    got = oracle.paged_to_cache(pool, t2, [6, P * ps, 0])
    assert np.array_equal(got[0, :, :6], cache[0, :, :6]) and not got[0, :, 6:].any()
    assert not got[1, :, :ps].any() and np.array_equal(got[1, :, ps:], cache[1, :, ps:])
    assert not got[2].any()


def test_sdpa_varlen_equals_batched_sdpa_on_equal_lengths():
    """A packed batch of equal-length sequences is the BHSD batch reshaped;
    a packed batch of one sequence is that sequence; with lengths 0 and
    Sq > Skv (causal) the empty rows give O = 0 and LSE = -inf."""
    rng = np.random.default_rng(8)
    B, S, n_q, n_kv, d = 3, 7, 4, 2, 5
    q = rng.standard_normal((B, n_q, S, d))
    k = rng.standard_normal((B, n_kv, S, d))
    v = rng.standard_normal((B, n_kv, S, d))
    o_ref, l_ref = oracle.sdpa(q, k, v, True, 0.4)
    pack = lambda x: x.transpose(0, 2, 1, 3).reshape(B * S, x.shape[1], d)
    cu = np.arange(B + 1) * S
    o, l = oracle.sdpa_varlen(pack(q), pack(k), pack(v), cu, cu, True, 0.4)
    assert np.array_equal(o, pack(o_ref))
    assert np.array_equal(l, l_ref.transpose(1, 0, 2).reshape(n_q, B * S))
    # lengths (2, 0, 3) queries against (1, 2, 3) keys, causal
    cq, ck = np.array([0, 2, 2, 5]), np.array([0, 1, 3, 6])
    qv, kv_, vv = rng.standard_normal((5, n_q, d)), rng.standard_normal((6, n_kv, d)), rng.standard_normal((6, n_kv, d))
    o, l = oracle.sdpa_varlen(qv, kv_, vv, cq, ck, True, 0.5)
    # sequence 0: Sq 2 > Skv 1 -> query 0 sees no key, query 1 sees key 0
    assert not o[0].any() and np.all(np.isneginf(l[:, 0]))
    G = n_q // n_kv
    for h in range(n_q):
        assert np.allclose(o[1, h], vv[0, h // G])
    ob, lb = oracle.sdpa(qv[2:5].transpose(1, 0, 2)[None], kv_[3:6].transpose(1, 0, 2)[None],
                         vv[3:6].transpose(1, 0, 2)[None], True, 0.5)
    assert np.array_equal(o[2:5], ob[0].transpose(1, 0, 2)) and np.array_equal(l[:, 2:5], lb[0])


def test_sdpa_window_pins():
    """Sliding window + sinks against what fixes it: a window covering every
    key is the causal forward; a window of 1 without sinks returns each
    row's own value row (LSE = scale q.k of that key); and an independent
    library (torch SDPA in fp64 with the explicit boolean mask of "Attention
    deep dive" section 6, (j <= i) and (i - j < W), or j < n_sink)."""
    import torch
    rng = np.random.default_rng(21)
    B, n_q, n_kv, S, d = 2, 4, 2, 37, 8
    q = rng.standard_normal((B, n_q, S, d))
    k = rng.standard_normal((B, n_kv, S, d))
    v = rng.standard_normal((B, n_kv, S, d))
    o_c, l_c = oracle.sdpa(q, k, v, True, 0.3)
    o_w, l_w = oracle.sdpa_window(q, k, v, True, S, 0, 0.3)
    assert np.array_equal(o_w, o_c) and np.array_equal(l_w, l_c)
    o1, l1 = oracle.sdpa_window(q, k, v, True, 1, 0, 0.3)
    G = n_q // n_kv
    for h in range(n_q):
        assert np.array_equal(o1[:, h], v[:, h // G])
        assert np.allclose(l1[:, h], 0.3 * (q[:, h] * k[:, h // G]).sum(-1), atol=1e-12)
    for W, ns in [(5, 0), (5, 3), (11, 4), (1, 2)]:
        o_w, l_w = oracle.sdpa_window(q, k, v, True, W, ns, 0.3)
        i = np.arange(S)[:, None]
        j = np.arange(S)[None, :]
        mask = (j <= i) & ((i - j < W) | (j < ns))
        kr = torch.tensor(k).repeat_interleave(G, dim=1)
        vr = torch.tensor(v).repeat_interleave(G, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q), kr, vr, attn_mask=torch.tensor(mask), scale=0.3).numpy()
        assert np.allclose(o_w, ref, atol=1e-12, rtol=0), (W, ns)
    # decode form: the window ends at the last visible key seqlens[b] - 1
    o_d, l_d = oracle.sdpa_window(q[:, :, :1], k, v, False, 4, 1, 0.3, seqlens=[20, 2])
    keep = [0, 16, 17, 18, 19]
    o_r, l_r = oracle.sdpa(q[:1, :, :1], k[:1, :, keep], v[:1, :, keep], False, 0.3)
    assert np.allclose(o_d[:1], o_r, atol=1e-12) and np.allclose(l_d[:1], l_r, atol=1e-12)


def test_dequant_e4m3_matches_an_independent_decoder():
    """All 256 byte patterns against torch's float8_e4m3fn conversion (an
    independent implementation), plus the format's landmarks: 448 is the
    largest finite value, 2^-9 the smallest subnormal, 0x7F / 0xFF are NaN."""
    import torch
    raw = np.arange(256, dtype=np.uint8)
    got = oracle.dequant_e4m3(raw)
    ref = torch.from_numpy(raw.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0x38] == 1.0 and got[0xB8] == -1.0
    # per-head scale along axis 1
    x = np.full((2, 3, 4), 0x38, np.uint8)
    assert np.array_equal(oracle.dequant_e4m3(x, [1.0, 0.5, 2.0])[0, :, 0], [1.0, 0.5, 2.0])


def test_dequant_e4m3_tiles():
    """Per-tile scales: a hand case (1.0 bytes over two tiles of two tokens
    scaled by 2 and 3; a NaN byte stays NaN), and constant scales per
    (sequence, KV head) reduce to the per-head form."""
    x = np.full((1, 1, 4, 2), 0x38, np.uint8)
    x[0, 0, 3, 1] = 0x7F
    got = oracle.dequant_e4m3_tiles(x, [[[2.0, 3.0]]], tile=2)
    assert np.array_equal(got[0, 0, :3], [[2.0, 2.0], [2.0, 2.0], [3.0, 3.0]])
    assert got[0, 0, 3, 0] == 3.0 and np.isnan(got[0, 0, 3, 1])
    rng = np.random.default_rng(4)
    raw = rng.integers(0, 126, size=(2, 3, 300, 8)).astype(np.uint8)   # no NaN patterns
    per_head = np.array([0.5, 2.0, 0.125])
    tiles = np.broadcast_to(per_head[None, :, None], (2, 3, 3))
    assert np.array_equal(oracle.dequant_e4m3_tiles(raw, tiles), oracle.dequant_e4m3(raw, per_head))


def test_round_bf16_matches_torch():
    """The oracle's bf16 rounding against torch's fp32 -> bf16 conversion
    (round to nearest even) on fp32 values, ties and near-ties included."""
    g = torch.Generator().manual_seed(5)
    x = torch.randn(200000, generator=g, dtype=torch.float32) * torch.exp2(torch.randint(-20, 20, (200000,)).float())
    ties = torch.tensor([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3 * 2 ** -9 + 2 ** -30, 255.5, 256.5],
                        dtype=torch.float32)
    x = torch.cat([x, ties])
    ref = x.to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(x.double().numpy()), ref)


def test_sdpa_fp8_scaling_and_tiles():
    """The FP8 oracle mode against closed forms. Uniform power-of-two scales
    2^a, 2^b, 2^c on q, k, v: the scores scale by 2^(a+b) (the softmax scale
    times 2^(a+b) on the unscaled values) and the output by 2^c, exactly in
    fp64. Per-tile scales: query rows of tile 1 and key rows of tiles 1 and
    2 carry their own factors, which must land on rows 128.. and 256..
    (compared with sdpa on values multiplied row by row)."""
    rng = np.random.default_rng(9)
    B, n_q, n_kv, Sq, Skv, d = 1, 4, 2, 200, 300, 16
    q8 = rng.integers(0, 126, size=(B, n_q, Sq, d)).astype(np.uint8) | (rng.integers(0, 2, (B, n_q, Sq, d)) << 7).astype(np.uint8)
    k8 = rng.integers(0, 120, size=(B, n_kv, Skv, d)).astype(np.uint8)
    v8 = rng.integers(0, 126, size=(B, n_kv, Skv, d)).astype(np.uint8)
    q, k, v = oracle.dequant_e4m3(q8), oracle.dequant_e4m3(k8), oracle.dequant_e4m3(v8)
    tq, tk = (Sq + 127) // 128, (Skv + 127) // 128
    for causal in (False, True):
        o, lse = oracle.sdpa_fp8(q8, k8, v8, np.full((B, n_q, tq), 0.25), np.full((B, n_kv, tk), 2.0),
                                 np.full((B, n_kv, tk), 8.0), causal, 0.1)
        o_ref, lse_ref = oracle.sdpa(q, k, v, causal, 0.1 * 0.25 * 2.0)
        assert np.allclose(o, 8.0 * o_ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)
    qs = np.ones((B, n_q, tq)); qs[:, :, 1] = 3.0
    ks = np.ones((B, n_kv, tk)); ks[:, :, 1] = 0.5; ks[:, :, 2] = 2.0
    vs = np.ones((B, n_kv, tk)); vs[:, :, 2] = 4.0
    qm = np.where(np.arange(Sq) >= 128, 3.0, 1.0)[None, None, :, None]
    km = np.select([np.arange(Skv) >= 256, np.arange(Skv) >= 128], [2.0, 0.5], 1.0)[None, None, :, None]
    vm = np.where(np.arange(Skv) >= 256, 4.0, 1.0)[None, None, :, None]
    o, lse = oracle.sdpa_fp8(q8, k8, v8, qs, ks, vs, True, 0.1)
    o_ref, lse_ref = oracle.sdpa(q * qm, k * km, v * vm, True, 0.1)
    assert np.allclose(o, o_ref, rtol=1e-12, atol=1e-12) and np.allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)
