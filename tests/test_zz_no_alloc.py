"""attn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a plugin inside a framework that owns every device
allocation, a serving loop that must not enter an allocator, host code with
no allocator of its own). It keeps its scratch in a static device array held
by the library, so the caller passes only inputs and outputs.

Checked through the C ABI against attn_decode (which takes a caller-owned
workspace) on two calls in a row, within the parity tolerances used by every
GPU test here, and on a smaller problem also against the fp64 oracle. This
file is collected last on purpose."""
import ctypes

import pytest
import torch

import oracle
from gpu_util import LSE_ABS, O_MAX_ABS, check_parity, need_gpu
from mqa_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu

SCRATCH_MAX = 36 * 1024 * 1024     # ATTN_NOALLOC_SCRATCH_BYTES in include/attn.h


def _noalloc_fn(binding):
    fn = binding.lib().attn_decode_noalloc
    vp, i, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    fn.argtypes = [vp] * 6 + [i] * 6 + [i64] * 6 + [ctypes.c_float, vp]
    fn.restype = i
    return fn


def _call_noalloc(fn, q, kc, vc, seqlens, o, lse, scale):
    B, n_q, d = q.shape
    _, n_kv, S_max, _ = kc.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(p(q), p(kc), p(vc), p(seqlens), p(o), p(lse), B, n_q, n_kv, d, d, S_max,
              kc.stride(0), kc.stride(1), kc.stride(2), vc.stride(0), vc.stride(1), vc.stride(2),
              float(scale), stream)


def test_noalloc_matches_attn_decode_twice():
    binding = need_gpu()
    fn = _noalloc_fn(binding)
    w = inputs.WORKLOADS["gqa_decode"]
    # the full GQA decode workload fits the static scratch
    need = binding.decode_workspace_bytes(w.B, w.n_q, w.n_kv, w.d_qk, w.d_v, w.Skv)
    assert need <= SCRATCH_MAX
    seqlens, q, kc, vc = inputs.make(w, device="cuda")
    sl = seqlens.cuda()
    o_ref, lse_ref = binding.attn_decode(q, kc, vc, sl, w.scale)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        rc = _call_noalloc(fn, q, kc, vc, sl, o, lse, w.scale)
        assert rc == 0, binding.status_string(rc)
        torch.cuda.synchronize()
        assert binding.device_status() == 0
        assert float((o.float() - o_ref.float()).abs().max()) <= O_MAX_ABS, f"call {call}"
        assert float((lse - lse_ref).abs().max()) <= LSE_ABS, f"call {call}"


def test_noalloc_second_problem_after_first():
    """A smaller problem after a larger one: the leftover scratch contents of
    the previous call must not leak into the result. Checked against
    attn_decode and against the fp64 oracle, on two calls in a row."""
    binding = need_gpu()
    fn = _noalloc_fn(binding)
    seqlens, q, kc, vc = inputs.decode_inputs(3, 16, 4, 128, 128, 3000, (1, 3000), 77, device="cuda")
    sl = seqlens.cuda()
    o_ref, lse_ref = binding.attn_decode(q, kc, vc, sl, 0.1)
    o64, l64 = oracle.sdpa(q[:, :, None, :], kc, vc, False, 0.1, seqlens=seqlens.numpy())
    for call in range(2):
        o, lse = torch.empty_like(o_ref), torch.empty_like(lse_ref)
        rc = _call_noalloc(fn, q, kc, vc, sl, o, lse, 0.1)
        assert rc == 0, binding.status_string(rc)
        torch.cuda.synchronize()
        assert binding.device_status() == 0, f"call {call}"
        assert float((o.float() - o_ref.float()).abs().max()) <= O_MAX_ABS
        assert float((lse - lse_ref).abs().max()) <= LSE_ABS
        check_parity(o, lse, o64[:, :, 0], l64[:, :, 0], f"no-alloc decode, call {call}")


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    binding = need_gpu()
    fn = _noalloc_fn(binding)
    B, n_q, n_kv, S_max = 64, 32, 8, 131072         # needs ~68 MB of scratch
    assert binding.decode_workspace_bytes(B, n_q, n_kv, 128, 128, S_max) > SCRATCH_MAX
    q = torch.zeros(B, n_q, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(1, n_kv, S_max, 128, dtype=torch.bfloat16, device="cuda").expand(B, n_kv, S_max, 128)
    sl = torch.ones(B, dtype=torch.int32, device="cuda")
    o = torch.empty(B, n_q, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, n_q, dtype=torch.float32, device="cuda")
    assert _call_noalloc(fn, q, kc, kc, sl, o, lse, 0.1) == -4    # ATTN_ERR_WORKSPACE
