"""Pins of the fp64 oracle to facts outside itself.

Each ``check_*`` function takes an oracle library handle (the real build, or
a build of a deliberately mutated copy) and raises AssertionError when the
oracle disagrees with:
  * the worked example printed on "Attention, Worked Out by Hand (Part 2)"
    (tests/golden/worked_example_on_row.txt),
  * closed forms of softmax attention (value shift, key shift, constant keys,
    first causal row),
  * structural identities stated on the pages (GQA == repeated MHA,
    MHA == independent heads, MQA as one shared head),
  * an independent library implementation (torch's scaled_dot_product_attention
    on CPU in fp64),
  * the FlashAttention-2 recurrence reaching the same result as the two-pass
    softmax, to 1e-12.

test_oracle_pins.py runs them against the real oracle; test_oracle_mutations.py
shows that plausible mistakes planted in a copy of the oracle fail at least one.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name="worked_example_on_row.txt"):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rhs = line.split("=", 1)
            vals[key.strip()] = np.array([float(x) for x in rhs.split()])
    return vals


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def _bf16_rand(shape, seed):
    return _rand(shape, seed).to(torch.bfloat16).to(torch.float64)


# --------------------------------------------------------------------------
# worked example
# --------------------------------------------------------------------------
def worked_example_instance(gold):
    """q, K, V (as [1,1,S,4] fp64) reproducing the page's on-row scores."""
    s = gold["scaled_scores"]
    q = np.zeros((1, 1, 4, 4))
    q[0, 0, 3] = [2.0, 0, 0, 0]          # the "on" query (row 3)
    q[0, 0, 0:3] = _rand((3, 4), 11).numpy()  # other rows: arbitrary
    k = np.zeros((1, 1, 4, 4))
    k[0, 0, :, 0] = s                    # 2 * s_j * (1/2) = s_j
    v = np.zeros((1, 1, 4, 4))
    v[0, 0, 0] = gold["tile0_acc"]        # V[the]; V[cat] = 0
    v[0, 0, 2] = gold["tile1_acc"] - gold["rescale"] * gold["tile0_acc"]  # V[sat]; V[on] = 0
    return q, k, v


def check_worked_example(lib):
    gold = load_golden()
    q, k, v = worked_example_instance(gold)
    o, lse = oracle.sdpa(q, k, v, causal=True, scale=0.5, lib=lib)
    assert np.allclose(o[0, 0, 3], gold["out"], atol=2e-3), (o[0, 0, 3], gold["out"])
    # LSE = running max + ln(l) at the end of the trace
    want_lse = gold["tile1_max"][0] + math.log(gold["final_l"][0])
    assert abs(lse[0, 0, 3] - want_lse) < 2e-3, (lse[0, 0, 3], want_lse)
    _, _, w, nv = oracle.row_weights(q[0, 0, 3], 0, 0, 3, k, v, 1, 1, 4, causal=True,
                                     scale=0.5, lib=lib)
    assert nv == 4
    assert np.allclose(w, gold["weights"], atol=2e-3), (w, gold["weights"])
    # the first token attends only to itself
    _, _, w0, nv0 = oracle.row_weights(q[0, 0, 0], 0, 0, 0, k, v, 1, 1, 4, causal=True,
                                       scale=0.5, lib=lib)
    assert nv0 == 1
    assert np.array_equal(w0, gold["first_row_weights"]), w0
    assert np.array_equal(o[0, 0, 0], v[0, 0, 0])


def check_worked_example_first_tile(lib):
    """Only the first tile's keys visible: O = acc0 / l0, LSE = m0 + ln l0."""
    gold = load_golden()
    q, k, v = worked_example_instance(gold)
    o, lse = oracle.sdpa(q[:, :, 3:4], k[:, :, :2], v[:, :, :2], causal=False, scale=0.5, lib=lib)
    assert np.allclose(o[0, 0, 0], gold["tile0_acc"] / gold["tile0_l"][0], atol=2e-3)
    assert abs(lse[0, 0, 0] - (gold["scaled_scores"][0] + math.log(gold["tile0_l"][0]))) < 2e-3


def check_worked_example_online(lib):
    """Tile size 2 reproduces the printed result and equals the two-pass
    softmax to 1e-12 (the page's "same numbers, to 1e-12")."""
    gold = load_golden()
    q, k, v = worked_example_instance(gold)
    o2, l2 = oracle.sdpa(q, k, v, causal=True, scale=0.5, lib=lib)
    oo, lo = oracle.online(q, k, v, causal=True, scale=0.5, block_r=4, block_c=2, lib=lib)
    assert np.allclose(oo[0, 0, 3], gold["out"], atol=2e-3)
    assert np.max(np.abs(oo - o2)) <= 1e-12
    assert np.max(np.abs(lo - l2)) <= 1e-12


# --------------------------------------------------------------------------
# closed forms and special cases
# --------------------------------------------------------------------------
def check_first_causal_row(lib):
    """Causal row 0 sees only key 0: O = v_0 exactly, LSE = scale * q_0.k_0."""
    B, n_q, n_kv, S, d = 2, 4, 2, 9, 8
    q, k, v = _bf16_rand((B, n_q, S, d), 1), _bf16_rand((B, n_kv, S, d), 2), _bf16_rand((B, n_kv, S, d), 3)
    scale = 0.3
    o, lse = oracle.sdpa(q, k, v, causal=True, scale=scale, lib=lib)
    for b in range(B):
        for h in range(n_q):
            g = h // (n_q // n_kv)
            assert np.array_equal(o[b, h, 0], v[b, g, 0].numpy())
            want = scale * float(torch.dot(q[b, h, 0], k[b, g, 0]))
            assert abs(lse[b, h, 0] - want) <= 1e-12 * max(1.0, abs(want))


def check_rows_sum_to_one(lib):
    B, n_q, n_kv, S, d = 1, 4, 2, 13, 8
    q, k, v = _rand((B, n_q, S, d), 4), _rand((B, n_kv, S, d), 5), _rand((B, n_kv, S, d), 6)
    for causal in (True, False):
        for i in (0, 5, 12):
            _, _, w, nv = oracle.row_weights(q[0, 1, i], 0, 1, i, k, v, B, n_q, S, causal=causal,
                                             scale=0.4, lib=lib)
            assert nv == (i + 1 if causal else S)
            assert abs(w.sum() - 1.0) <= 1e-14
            assert np.all(w[nv:] == 0.0) and np.all(w[:nv] > 0.0)


def check_value_shift(lib):
    """V + 1 w^T  ->  O + w   (softmax rows sum to one)."""
    B, n_q, n_kv, S, d = 1, 4, 1, 17, 8
    q, k, v = _rand((B, n_q, S, d), 7), _rand((B, n_kv, S, d), 8), _rand((B, n_kv, S, d), 9)
    w = _rand((d,), 10)
    for causal in (True, False):
        o1, l1 = oracle.sdpa(q, k, v, causal, 0.35, lib=lib)
        o2, l2 = oracle.sdpa(q, k, v + w, causal, 0.35, lib=lib)
        assert np.max(np.abs(o2 - (o1 + w.numpy()))) <= 1e-12
        assert np.max(np.abs(l2 - l1)) <= 1e-12


def check_key_shift(lib):
    """K + 1 u^T  ->  O unchanged, LSE_i += scale * q_i.u   (shift invariance)."""
    B, n_q, n_kv, S, d = 1, 2, 1, 11, 8
    q, k, v = _rand((B, n_q, S, d), 12), _rand((B, n_kv, S, d), 13), _rand((B, n_kv, S, d), 14)
    u = _rand((d,), 15)
    scale = 0.5
    for causal in (True, False):
        o1, l1 = oracle.sdpa(q, k, v, causal, scale, lib=lib)
        o2, l2 = oracle.sdpa(q, k + u, v, causal, scale, lib=lib)
        assert np.max(np.abs(o2 - o1)) <= 1e-12
        shift = scale * (q @ u).numpy()
        assert np.max(np.abs(l2 - (l1 + shift))) <= 1e-12


def check_constant_keys(lib):
    """All keys equal k: O_i = mean of the visible v_j, LSE_i = scale q_i.k + ln|V(i)|."""
    B, n_q, n_kv, Sq, Skv, d = 1, 4, 2, 6, 10, 8
    q = _rand((B, n_q, Sq, d), 16)
    k = _rand((1, 1, 1, d), 17).expand(B, n_kv, Skv, d).contiguous()
    v = _rand((B, n_kv, Skv, d), 18)
    scale = 0.7
    o, lse = oracle.sdpa(q, k, v, causal=True, scale=scale, lib=lib)
    for h in range(n_q):
        g = h // 2
        for i in range(Sq):
            n = i + (Skv - Sq) + 1          # bottom-right aligned causal
            assert np.max(np.abs(o[0, h, i] - v[0, g, :n].mean(0).numpy())) <= 1e-12
            want = scale * float(q[0, h, i] @ k[0, g, 0]) + math.log(n)
            assert abs(lse[0, h, i] - want) <= 1e-12


def check_huge_logits_finite(lib):
    """Scores of magnitude ~1e4: the max-subtracted softmax stays finite."""
    B, n_q, n_kv, S, d = 1, 2, 1, 8, 4
    q = _rand((B, n_q, S, d), 19) * 100
    k = _rand((B, n_kv, S, d), 20) * 100
    v = _rand((B, n_kv, S, d), 21)
    o, lse = oracle.sdpa(q, k, v, causal=False, scale=1.0, lib=lib)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    # one key dominates: O equals that key's value
    s = torch.einsum("hid,jd->hij", q[0], k[0, 0])
    top = s.argmax(-1)
    gap = (s.sort(-1).values[..., -1] - s.sort(-1).values[..., -2])
    for h in range(n_q):
        for i in range(S):
            if gap[h, i] > 50:
                assert np.allclose(o[0, h, i], v[0, 0, top[h, i]].numpy(), atol=1e-12)
                assert abs(lse[0, h, i] - float(s[h, i].max())) <= 1e-9 * abs(float(s[h, i].max()))


# --------------------------------------------------------------------------
# structural identities
# --------------------------------------------------------------------------
def check_gqa_equals_repeated_mha(lib):
    """Grouped heads == MHA over K/V repeated G times (query head h -> group h // G)."""
    for n_q, n_kv in ((8, 2), (6, 3), (4, 1), (4, 4)):
        B, S, d = 2, 12, 8
        q, k, v = _rand((B, n_q, S, d), 22), _rand((B, n_kv, S, d), 23), _rand((B, n_kv, S, d), 24)
        G = n_q // n_kv
        kr = k.repeat_interleave(G, dim=1)
        vr = v.repeat_interleave(G, dim=1)
        for causal in (True, False):
            o1, l1 = oracle.sdpa(q, k, v, causal, 0.3, lib=lib)
            o2, l2 = oracle.sdpa(q, kr, vr, causal, 0.3, lib=lib)
            assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def check_mha_independent_heads(lib):
    """n_kv == n_q: each head is an independent one-head problem."""
    B, n, S, d = 1, 3, 10, 8
    q, k, v = _rand((B, n, S, d), 25), _rand((B, n, S, d), 26), _rand((B, n, S, d), 27)
    o, lse = oracle.sdpa(q, k, v, True, 0.3, lib=lib)
    for h in range(n):
        oh, lh = oracle.sdpa(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], True, 0.3, lib=lib)
        assert np.array_equal(o[:, h:h + 1], oh) and np.array_equal(lse[:, h:h + 1], lh)


def check_permutations(lib):
    """Non-causal: permuting key/value rows jointly changes nothing; permuting
    query heads inside a group permutes the output heads."""
    B, n_q, n_kv, S, d = 1, 4, 2, 9, 8
    q, k, v = _rand((B, n_q, S, d), 28), _rand((B, n_kv, S, d), 29), _rand((B, n_kv, S, d), 30)
    perm = torch.randperm(S, generator=torch.Generator().manual_seed(31))
    o1, l1 = oracle.sdpa(q, k, v, False, 0.3, lib=lib)
    o2, l2 = oracle.sdpa(q, k[:, :, perm], v[:, :, perm], False, 0.3, lib=lib)
    assert np.max(np.abs(o1 - o2)) <= 1e-12 and np.max(np.abs(l1 - l2)) <= 1e-12
    hp = torch.tensor([1, 0, 3, 2])       # swaps inside groups {0,1} and {2,3}
    o3, l3 = oracle.sdpa(q[:, hp], k, v, False, 0.3, lib=lib)
    assert np.array_equal(o3, o1[:, hp.numpy()]) and np.array_equal(l3, l1[:, hp.numpy()])
    # swapping the two groups together with their query-head blocks
    gp = torch.tensor([2, 3, 0, 1])
    o4, _ = oracle.sdpa(q[:, gp], k[:, [1, 0]], v[:, [1, 0]], False, 0.3, lib=lib)
    assert np.array_equal(o4, o1[:, gp.numpy()])


def check_torch_sdpa_fp64(lib):
    """An independent implementation: torch's SDPA on CPU in fp64."""
    cases = [(1, 4, 2, 64, 64, 32, True), (2, 8, 2, 33, 33, 16, True),
             (1, 6, 3, 20, 45, 16, False), (1, 4, 4, 1, 77, 8, False)]
    for B, n_q, n_kv, Sq, Skv, d, causal in cases:
        q, k, v = _rand((B, n_q, Sq, d), 40), _rand((B, n_kv, Skv, d), 41), _rand((B, n_kv, Skv, d), 42)
        scale = 1 / math.sqrt(d)
        o, _ = oracle.sdpa(q, k, v, causal, scale, lib=lib)
        ref = F.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=scale, enable_gqa=True)
        assert np.max(np.abs(o - ref.numpy())) <= 1e-10


def check_bottom_right_causal(lib):
    """Sq < Skv causal: query i sits at position Skv - Sq + i. Checked against
    torch SDPA with the explicit boolean mask of that reading."""
    B, n_q, n_kv, Sq, Skv, d = 1, 4, 2, 7, 19, 8
    q, k, v = _rand((B, n_q, Sq, d), 43), _rand((B, n_kv, Skv, d), 44), _rand((B, n_kv, Skv, d), 45)
    mask = torch.arange(Skv)[None, :] <= (torch.arange(Sq)[:, None] + (Skv - Sq))
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=0.3, enable_gqa=True)
    o, _ = oracle.sdpa(q, k, v, True, 0.3, lib=lib)
    assert np.max(np.abs(o - ref.numpy())) <= 1e-10


def check_decode(lib):
    """Decode with per-sequence lengths == SDPA on the truncated cache, and ==
    the last row of a causal prefill over those tokens."""
    B, n_q, n_kv, S_max, d = 3, 8, 2, 40, 16
    q = _rand((B, n_q, 1, d), 46)
    k, v = _rand((B, n_kv, S_max, d), 47), _rand((B, n_kv, S_max, d), 48)
    seqlens = np.array([1, 17, 40], dtype=np.int32)
    o, lse = oracle.sdpa(q, k, v, False, 0.25, seqlens=seqlens, lib=lib)
    for b in range(B):
        L = int(seqlens[b])
        ref = F.scaled_dot_product_attention(q[b:b + 1], k[b:b + 1, :, :L], v[b:b + 1, :, :L],
                                             scale=0.25, enable_gqa=True)
        assert np.max(np.abs(o[b:b + 1] - ref.numpy())) <= 1e-10
        qp = _rand((1, n_q, L, d), 49)
        qp[:, :, L - 1] = q[b, :, 0]
        op, lp = oracle.sdpa(qp, k[b:b + 1, :, :L], v[b:b + 1, :, :L], True, 0.25, lib=lib)
        assert np.max(np.abs(op[0, :, L - 1] - o[b, :, 0])) <= 1e-12
        assert np.max(np.abs(lp[0, :, L - 1] - lse[b, :, 0])) <= 1e-12


def check_empty_visible_set(lib):
    """seqlen 0: o = 0, lse = -inf (the empty-sum limit)."""
    q = _rand((1, 2, 1, 4), 50)
    k, v = _rand((1, 1, 5, 4), 51), _rand((1, 1, 5, 4), 52)
    o, lse = oracle.sdpa(q, k, v, False, 1.0, seqlens=np.array([0], np.int32), lib=lib)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def check_mla_alias(lib):
    """Latent cache: key = full 576-wide row, value = its first 512 columns of
    the same storage; equal to passing an explicit copy of those columns."""
    B, n_q, S, dl, dv = 2, 4, 9, 24, 16      # small stand-ins for 576 / 512
    q = _rand((B, n_q, 1, dl), 53)
    cache = _rand((B, 1, S, dl), 54)
    seqlens = np.array([9, 5], np.int32)
    o1, l1 = oracle.sdpa(q, cache, cache, False, 0.2, seqlens=seqlens, d_v=dv, lib=lib)
    o2, l2 = oracle.sdpa(q, cache, cache[..., :dv].contiguous(), False, 0.2, seqlens=seqlens, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    ref = F.scaled_dot_product_attention(q[1:], cache[1:, :, :5], cache[1:, :, :5, :dv], scale=0.2,
                                         enable_gqa=True)
    assert np.max(np.abs(o1[1:] - ref.numpy())) <= 1e-10


def check_online_equals_two_pass(lib):
    """The FlashAttention-2 recurrence equals the two-pass softmax (fp64, 1e-12)."""
    B, n_q, n_kv, d = 1, 4, 2, 8
    for Sq, Skv, causal in ((23, 23, True), (10, 31, True), (12, 29, False)):
        q, k, v = _rand((B, n_q, Sq, d), 55), _rand((B, n_kv, Skv, d), 56), _rand((B, n_kv, Skv, d), 57)
        o2, l2 = oracle.sdpa(q, k, v, causal, 0.3, lib=lib)
        for br, bc in ((1, 1), (3, 5), (7, 4), (16, 16), (64, 64), (5, 13)):
            oo, lo = oracle.online(q, k, v, causal, 0.3, br, bc, lib=lib)
            assert np.max(np.abs(oo - o2)) <= 1e-12, (Sq, Skv, causal, br, bc)
            assert np.max(np.abs(lo - l2)) <= 1e-12


def check_rows_mode(lib):
    """Sampled-row mode returns exactly the full forward's rows."""
    B, n_q, n_kv, S, d = 2, 4, 2, 15, 8
    q, k, v = _rand((B, n_q, S, d), 58), _rand((B, n_kv, S, d), 59), _rand((B, n_kv, S, d), 60)
    o, lse = oracle.sdpa(q, k, v, True, 0.3, lib=lib)
    rows = np.array([[0, 0, 0], [1, 3, 14], [0, 2, 7], [1, 1, 3]], np.int32)
    qr = torch.stack([q[b, h, i] for b, h, i in rows])
    orr, lr = oracle.sdpa_rows(qr, rows, k, v, B, n_q, S, True, 0.3, lib=lib)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(orr[r], o[b, h, i]) and lr[r] == lse[b, h, i]


def check_sliding_window(lib):
    """Sliding window and sinks against torch SDPA with the explicit boolean
    mask of "Attention deep dive" section 6, (j <= p) and (p - j < W), widened
    by the first n_sink keys; bottom-right alignment (Sq < Skv) and the
    decode form (window ending at seqlens[b] - 1) included."""
    B, n_q, n_kv, Sq, Skv, d = 2, 4, 2, 13, 29, 8
    q, k, v = _rand((B, n_q, Sq, d), 60), _rand((B, n_kv, Skv, d), 61), _rand((B, n_kv, Skv, d), 62)
    pos = torch.arange(Sq)[:, None] + (Skv - Sq)
    j = torch.arange(Skv)[None, :]
    for W, ns in [(1, 0), (4, 0), (4, 2), (9, 5), (40, 0)]:
        mask = (j <= pos) & ((pos - j < W) | (j < ns))
        ref = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=0.3, enable_gqa=True)
        o, _ = oracle.sdpa_window(q, k, v, True, W, ns, 0.3, lib=lib)
        assert np.max(np.abs(o - ref.numpy())) <= 1e-10, (W, ns)
    seqlens = np.array([29, 6], dtype=np.int32)
    o, _ = oracle.sdpa_window(q[:, :, :1], k, v, False, 3, 2, 0.3, seqlens=seqlens, lib=lib)
    for b, L in enumerate(seqlens):
        keep = sorted(set(range(min(2, L))) | set(range(max(0, L - 3), L)))
        ref = F.scaled_dot_product_attention(q[b:b + 1, :, :1], k[b:b + 1, :, keep], v[b:b + 1, :, keep],
                                             scale=0.3, enable_gqa=True)
        assert np.max(np.abs(o[b:b + 1] - ref.numpy())) <= 1e-10



# --------------------------------------------------------------------------
# rotary position embedding
# --------------------------------------------------------------------------
def check_rope_tables(lib):
    """Closed forms of the tables of "Attention Engineering: From MHA to GQA,
    MLA & FlashAttention", section 1 (theta_j = base^(-2j/d)): plane 0 turns
    by exactly m radians, plane d/4 of d = 128 at base 10^4 by m / 100, plane
    d/2 - 1 by m * base^(-(d-2)/d); position 0 is the identity."""
    n_pos, d, base = 300, 128, 10000.0
    c, s = oracle.rope_tables(n_pos, d, base, lib=lib)
    m = np.arange(n_pos, dtype=np.float64)
    assert np.max(np.abs(c[:, 0] - np.cos(m))) <= 1e-14 and np.max(np.abs(s[:, 0] - np.sin(m))) <= 1e-14
    assert np.max(np.abs(c[:, 32] - np.cos(m / 100.0))) <= 1e-14
    assert np.max(np.abs(s[:, 32] - np.sin(m / 100.0))) <= 1e-14
    last = m * 10000.0 ** (-126.0 / 128.0)
    assert np.max(np.abs(s[:, 63] - np.sin(last))) <= 1e-14
    assert np.all(c[0] == 1.0) and np.all(s[0] == 0.0)
    c8, s8 = oracle.rope_tables(5, 8, 500000.0, lib=lib)        # Llama-3 base, tiny d
    assert abs(s8[3, 1] - math.sin(3 * 500000.0 ** -0.25)) <= 1e-15


def check_rope_complex_form(lib):
    """The rotation equals multiplying z_j = x_{2j} + i x_{2j+1} by
    exp(i m theta_j) (section 1, complex-plane derivation), here with numpy's
    complex exponential and tables built outside the oracle."""
    d, S = 16, 11
    x = _rand((3, S, d), 70).numpy()
    theta = 10000.0 ** (-np.arange(d // 2) * 2.0 / d)
    pos = np.array([0, 1, 2, 5, 7, 8, 20, 33, 34, 40, 63], dtype=np.int32)
    ang = np.arange(64)[:, None] * theta[None, :]
    got = oracle.rope(x, np.cos(ang), np.sin(ang), pos, lib=lib)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * pos[:, None] * theta[None, :])
    ref = np.empty_like(x)
    ref[..., 0::2], ref[..., 1::2] = z.real, z.imag
    assert np.max(np.abs(got - ref)) <= 1e-13


def check_rope_relative_position(lib):
    """<RoPE(q, m), RoPE(k, n)> depends on m - n only (section 1, the
    relative-distance invariance identity), and the rotation keeps each
    plane's length."""
    d = 32
    c, s = oracle.rope_tables(400, d, 10000.0, lib=lib)
    q, k = _rand((1, d), 71).numpy(), _rand((1, d), 72).numpy()
    dots = []
    for m, n in [(5, 2), (105, 102), (303, 300), (3, 0)]:
        rq = oracle.rope(q, c, s, [m], lib=lib)
        rk = oracle.rope(k, c, s, [n], lib=lib)
        dots.append(float((rq @ rk.T)[0, 0]))
    assert max(dots) - min(dots) <= 1e-12 * max(1.0, abs(dots[0]))
    assert abs(dots[0] - float((q @ k.T)[0, 0])) > 1e-3     # the rotation does act
    rq = oracle.rope(q, c, s, [123], lib=lib)
    assert np.max(np.abs(np.hypot(rq[:, 0::2], rq[:, 1::2]) - np.hypot(q[:, 0::2], q[:, 1::2]))) <= 1e-13


def check_rope_attention(lib):
    """sdpa_rope: a lone query (decode) sits at the last key's position, so it
    equals the last row of the causal prefill; and the rotated scores of the
    first causal row are those of q_0 and k_0 unrotated (position 0)."""
    B, n_q, n_kv, S, d = 1, 4, 2, 9, 16
    q, k, v = _rand((B, n_q, S, d), 73), _rand((B, n_kv, S, d), 74), _rand((B, n_kv, S, d), 75)
    c, s = oracle.rope_tables(S, d, 10000.0, lib=lib)
    o, lse = oracle.sdpa_rope(q, k, v, True, 0.25, c, s, operand_bf16=False, lib=lib)
    o1, lse1 = oracle.sdpa_rope(q[:, :, -1:], k, v, False, 0.25, c, s, operand_bf16=False, lib=lib)
    assert np.max(np.abs(o1[:, :, 0] - o[:, :, -1])) <= 1e-12
    assert np.max(np.abs(lse1[:, :, 0] - lse[:, :, -1])) <= 1e-12
    kv0 = k[0, :, 0].numpy()
    ref = 0.25 * np.einsum("hd,hd->h", q[0, :, 0].numpy(), np.repeat(kv0, n_q // n_kv, axis=0))
    assert np.max(np.abs(lse[0, :, 0] - ref)) <= 1e-12
    # shifting every position by t leaves attention unchanged
    c2, s2 = oracle.rope_tables(S + 7, d, 10000.0, lib=lib)
    qs = oracle.rope(q, c2, s2, np.arange(7, 7 + S), lib=lib)
    ks = oracle.rope(k, c2, s2, np.arange(7, 7 + S), lib=lib)
    o2, _ = oracle.sdpa(qs, ks, v, True, 0.25, lib=lib)
    assert np.max(np.abs(o2 - o)) <= 1e-12


ALL_CHECKS = [
    check_worked_example, check_worked_example_first_tile, check_worked_example_online,
    check_first_causal_row, check_rows_sum_to_one, check_value_shift, check_key_shift,
    check_constant_keys, check_huge_logits_finite, check_gqa_equals_repeated_mha,
    check_mha_independent_heads, check_permutations, check_torch_sdpa_fp64,
    check_bottom_right_causal, check_decode, check_empty_visible_set, check_mla_alias,
    check_online_equals_two_pass, check_rows_mode,
    check_sliding_window,
    check_rope_tables, check_rope_complex_form, check_rope_relative_position, check_rope_attention,
]
