"""attn_fwd (prefill) on the GPU against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle_pins
from gpu_util import check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def _run_full(B, Sq, Skv, n_q, n_kv, d, causal, seed, scale=None):
    binding = need_gpu()
    scale = scale or 1.0 / math.sqrt(d)
    q, k, v = inputs.prefill_inputs(B, Sq, Skv, n_q, n_kv, d, d, seed, device="cuda")
    o, lse = binding.attn_fwd(q, k, v, causal, scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    o_ref, lse_ref = oracle.sdpa(q, k, v, causal, scale)
    return check_parity(o, lse, o_ref, lse_ref, f"B{B} Sq{Sq} Skv{Skv} {n_q}/{n_kv} d{d} c{causal}")


def test_tiny_workload_full():
    w = inputs.WORKLOADS["tiny_prefill"]
    _run_full(w.B, w.Sq, w.Skv, w.n_q, w.n_kv, w.d_qk, w.causal, w.seed, w.scale)


@pytest.mark.parametrize("B,Sq,Skv,n_q,n_kv,d,causal", [
    (2, 300, 300, 8, 2, 128, True),      # several tiles, ragged tail, G=4
    (1, 1000, 1000, 32, 8, 128, True),   # Llama-3-8B head layout, ragged
    (1, 130, 389, 4, 4, 64, False),      # MHA (G=1), non-causal, Sq != Skv
    (1, 100, 333, 16, 2, 128, True),     # G=8, bottom-right causal, Sq < Skv
    (2, 257, 257, 8, 1, 128, True),      # MQA
    (1, 513, 513, 4, 2, 64, True),       # G=2, d=64
    (3, 77, 77, 2, 1, 32, True),         # d=32, G=2
    (1, 1, 1, 4, 1, 128, True),          # one row, one key
    (1, 1, 700, 8, 2, 128, True),        # one query row against a long context
    (1, 200, 200, 1, 1, 128, True),      # MHA, two position tiles of which one is ragged
    (1, 96, 96, 256, 1, 64, True),       # G=256: one position per tile
])
def test_shapes_full(B, Sq, Skv, n_q, n_kv, d, causal):
    _run_full(B, Sq, Skv, n_q, n_kv, d, causal, seed=100 + Sq + n_q)


def test_worked_example_on_gpu():
    """The worked example of "Attention, Worked Out by Hand (Part 2)" run
    through the kernel (head dim padded with zeros to 32)."""
    binding = need_gpu()
    gold = oracle_pins.load_golden()
    q4, k4, v4 = oracle_pins.worked_example_instance(gold)
    pad = lambda a: np.concatenate([a, np.zeros(a.shape[:-1] + (28,))], axis=-1)
    q = torch.tensor(pad(q4), dtype=torch.bfloat16, device="cuda").contiguous()
    k = torch.tensor(pad(k4), dtype=torch.bfloat16, device="cuda").contiguous()
    v = torch.tensor(pad(v4), dtype=torch.bfloat16, device="cuda").contiguous()
    o, lse = binding.attn_fwd(q, k, v, True, 0.5)
    o_ref, lse_ref = oracle.sdpa(q, k, v, True, 0.5)
    check_parity(o, lse, o_ref, lse_ref, "worked example")
    out = o[0, 0, 3, :4].float().cpu().numpy()
    assert np.allclose(out, gold["out"], atol=1e-2), out       # bf16 inputs: looser than 2e-3
    assert torch.equal(o[0, 0, 0], v[0, 0, 0])                  # the first token attends to itself


def test_first_causal_row_exact():
    """Row 0 under the causal mask returns v_0 bit for bit; LSE = scale q0.k0."""
    binding = need_gpu()
    B, S, n_q, n_kv, d = 2, 384, 8, 2, 128
    q, k, v = inputs.prefill_inputs(B, S, S, n_q, n_kv, d, d, 7, device="cuda")
    o, lse = binding.attn_fwd(q, k, v, True, 1 / math.sqrt(d))
    G = n_q // n_kv
    for h in range(n_q):
        assert torch.equal(o[:, h, 0], v[:, h // G, 0])
        want = (q[:, h, 0].double() * k[:, h // G, 0].double()).sum(-1) / math.sqrt(d)
        assert torch.allclose(lse[:, h, 0].double(), want, atol=1e-3)


def test_deterministic():
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(1, 777, 777, 16, 4, 128, 128, 8, device="cuda")
    o1, l1 = binding.attn_fwd(q, k, v, True, 0.09)
    for _ in range(5):
        o2, l2 = binding.attn_fwd(q, k, v, True, 0.09)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_output_guard_bands_untouched():
    """Outputs written only inside their tensors (canary bands around O and LSE)."""
    binding = need_gpu()
    B, S, n_q, n_kv, d = 1, 333, 8, 2, 128
    q, k, v = inputs.prefill_inputs(B, S, S, n_q, n_kv, d, d, 9, device="cuda")
    n_o, n_l, guard = B * n_q * S * d, B * n_q * S, 4096
    obuf = torch.full((n_o + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((n_l + 2 * guard,), -3.0, dtype=torch.float32, device="cuda")
    o = obuf[guard:guard + n_o].view(B, n_q, S, d)
    lse = lbuf[guard:guard + n_l].view(B, n_q, S)
    binding.attn_fwd(q, k, v, True, 0.1, o=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(obuf[:guard] == 7.0) and torch.all(obuf[guard + n_o:] == 7.0)
    assert torch.all(lbuf[:guard] == -3.0) and torch.all(lbuf[guard + n_l:] == -3.0)
    o_ref, lse_ref = oracle.sdpa(q, k, v, True, 0.1)
    check_parity(o, lse, o_ref, lse_ref, "guarded")


def _sampled(w, n_rows, seed):
    binding = need_gpu()
    q, k, v = inputs.make(w, device="cuda")
    o, lse = binding.attn_fwd(q, k, v, w.causal, w.scale)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    rows = inputs.sample_rows(n_rows, w.B, w.n_q, w.Sq, seed)
    rb, rh, ri = rows[:, 0].long(), rows[:, 1].long(), rows[:, 2].long()
    q_rows = q[rb.cuda(), rh.cuda(), ri.cuda()]
    o_ref, lse_ref = oracle.sdpa_rows(q_rows, rows.numpy(), k, v, w.B, w.n_q, w.Sq, w.causal, w.scale)
    o_rows = o[rb.cuda(), rh.cuda(), ri.cuda()]
    lse_rows = lse[rb.cuda(), rh.cuda(), ri.cuda()]
    check_parity(o_rows, lse_rows, o_ref, lse_ref, w.name)
    return q, k, v, o, lse


def test_llama3_8b_prefill_sampled():
    """Full-size Llama-3-8B layout: 3000 sampled rows (every head's first and
    last row, tile boundaries, uniform rest) against the single-row oracle."""
    w = inputs.WORKLOADS["llama3_8b_prefill"]
    q, k, v, o, lse = _sampled(w, 3000, 11)
    # a property at full size: no output is larger than the largest value
    # (a convex combination of value rows)
    assert float(o.abs().max()) <= float(v.abs().max()) + 1e-2


def test_llama3_70b_long_prefill_sampled():
    """Full-size 70B layout at S=32768: 4096 stratified (b, h, i) triples
    (every head's first and last row, both sides of all 256 tile boundaries,
    uniform rest) against the single-row oracle."""
    w = inputs.WORKLOADS["llama3_70b_long_prefill"]
    rows = inputs.sample_rows(4096, w.B, w.n_q, w.Sq, 12)
    assert len(rows) == 4096
    i = set(rows[:, 2].tolist())
    assert all(t in i for t in range(127, w.Sq, 128)) and all(t in i for t in range(128, w.Sq, 128))
    assert set(rows[:, 1].tolist()) == set(range(w.n_q))
    _sampled(w, 4096, 12)


def test_constant_keys_closed_form_full_size():
    """All keys equal: O_i = running mean of v, LSE_i = scale q_i.k + ln(i+1),
    checked on every row at S=4096 (Llama-3-8B layout)."""
    binding = need_gpu()
    B, S, n_q, n_kv, d = 1, 4096, 32, 8, 128
    q, k, v = inputs.prefill_inputs(B, S, S, n_q, n_kv, d, d, 13, device="cuda")
    k = k[:, :, :1].expand(B, n_kv, S, d).contiguous()
    scale = 1 / math.sqrt(d)
    o, lse = binding.attn_fwd(q, k, v, True, scale)
    G = n_q // n_kv
    vr = v.double().repeat_interleave(G, dim=1)
    mean = vr.cumsum(2) / torch.arange(1, S + 1, device="cuda", dtype=torch.float64)[None, None, :, None]
    kk = k[:, :, 0].double().repeat_interleave(G, dim=1)
    want_lse = scale * (q.double() * kk[:, :, None, :]).sum(-1) + torch.log(
        torch.arange(1, S + 1, device="cuda", dtype=torch.float64))
    check_parity(o, lse, mean.cpu().numpy(), want_lse.cpu().numpy(), "constant keys")


def test_rejects_bad_arguments():
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(1, 64, 64, 6, 4, 64, 64, 1, device="cuda")
    with pytest.raises(binding.AttnError) as e:      # 6 % 4 != 0
        binding.attn_fwd(q, k, v, True, 0.1)
    assert e.value.code == -1
    q, k, v = inputs.prefill_inputs(1, 64, 64, 4, 2, 96, 96, 1, device="cuda")
    with pytest.raises(binding.AttnError) as e:      # head dim 96 not compiled
        binding.attn_fwd(q, k, v, True, 0.1)
    assert e.value.code == -2
    q, k, v = inputs.prefill_inputs(1, 65, 64, 4, 2, 64, 64, 1, device="cuda")
    with pytest.raises(binding.AttnError) as e:      # causal with Sq > Skv
        binding.attn_fwd(q, k, v, True, 0.1)
    assert e.value.code == -2
    q, k, v = inputs.prefill_inputs(1, 64, 64, 4, 2, 64, 64, 1, device="cuda")
    with pytest.raises(binding.AttnError) as e:
        binding.attn_fwd(q, k, v, True, float("nan"))
    assert e.value.code == -1
    buf = torch.empty(q.numel() + 1, dtype=torch.bfloat16, device="cuda")
    qm = buf[1:].view_as(q)                           # 2-byte offset: not 16-byte aligned
    qm.copy_(q)
    with pytest.raises(binding.AttnError) as e:
        binding.attn_fwd(qm, k, v, True, 0.1)
    assert e.value.code == -3


def test_empty_batch_is_noop():
    binding = need_gpu()
    q, k, v = inputs.prefill_inputs(0, 64, 64, 4, 2, 64, 64, 1, device="cuda")
    o, lse = binding.attn_fwd(q, k, v, True, 0.1)
    assert o.numel() == 0 and lse.numel() == 0


def test_exponential_accuracy():
    """The FMA-pipe 2^x (range reduction + fitted cubic) against float64 2^x:
    relative error below 1e-4 on the softmax's input range; clamped at -125
    (2^-125 stands in for 0); the special-function unit's ex2 as a control."""
    binding = need_gpu()
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_003), torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0])])
    yp, ys = binding.selftest_ex2(x.cuda())
    ref = torch.exp2(x.double())
    rel_p = ((yp.double().cpu() - ref) / ref).abs().max().item()
    rel_s = ((ys.double().cpu() - ref) / ref).abs().max().item()
    assert rel_p < 1e-4, rel_p
    assert rel_s < 1e-5, rel_s
    yp2, _ = binding.selftest_ex2(torch.tensor([-1e4, -200.0, float("-inf")], device="cuda"))
    y2 = yp2.double().cpu()
    assert torch.all((y2 - 2.0 ** -125).abs() <= 1e-4 * 2.0 ** -125), y2
