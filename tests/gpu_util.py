"""Shared helpers of the GPU parity tests: library loading and the tolerance
checks. The tolerances are the ones stated for this method's bf16 outputs
with fp32 accumulation: output max |diff| <= 2e-2 and relative L2 <= 5e-3
against the fp64 oracle, LSE within 1e-3 absolute."""
from __future__ import annotations

import numpy as np
import pytest
import torch

O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
LSE_ABS = 1e-3


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from mqa_attention_attn_b200 import build
    build.build_library()
    from mqa_attention_attn_b200 import binding
    binding.lib()
    return binding


def check_parity(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Element-by-element comparison against the oracle (fp64)."""
    og = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert og.shape == o_ref.shape, (og.shape, o_ref.shape)
    assert np.all(np.isfinite(og)), f"{what}: non-finite outputs"
    diff = np.abs(og - o_ref)
    max_abs = float(diff.max()) if diff.size else 0.0
    denom = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(og - o_ref) / denom) if denom > 0 else float(np.linalg.norm(og))
    assert max_abs <= O_MAX_ABS, f"{what}: O max|diff| {max_abs:.3e} > {O_MAX_ABS}"
    assert rel <= O_REL_L2, f"{what}: O rel-L2 {rel:.3e} > {O_REL_L2}"
    if lse_gpu is not None and lse_ref is not None:
        lg = lse_gpu.detach().double().cpu().numpy()
        lse_ref = np.asarray(lse_ref, dtype=np.float64)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin), f"{what}: LSE finiteness differs"
        if fin.any():
            ld = float(np.abs(lg[fin] - lse_ref[fin]).max())
            assert ld <= LSE_ABS, f"{what}: LSE max|diff| {ld:.3e} > {LSE_ABS}"
        assert np.array_equal(lg[~fin], lse_ref[~fin]), f"{what}: non-finite LSE values differ"
    return max_abs, rel
