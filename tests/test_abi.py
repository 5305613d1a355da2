"""The C-ABI library loads and exports every symbol include/attn.h declares;
argument validation answers without a GPU (no compute call is made here)."""
import ctypes

import pytest

from mqa_attention_attn_b200 import binding, build


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return binding.lib()


def test_header_declares_the_boundary():
    names = binding.header_functions()
    for required in ("attn_fwd", "attn_decode", "attn_decode_workspace_bytes", "attn_status_string",
                     "attn_device_status"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in binding.header_functions():
        assert hasattr(lib, name), f"{name} declared in include/attn.h but not exported"


def test_status_strings(lib):
    for code in range(0, -8, -1):
        assert binding.status_string(code) not in ("", "unknown status")
    assert binding.status_string(-99) == "unknown status"


def test_validation_rejects_before_any_launch(lib):
    vp = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    # n_q % n_kv != 0
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 8, 6, 4, 64, 64, 1, 0.1, None) == -1
    # causal must be 0 or 1
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 8, 4, 2, 64, 64, 2, 0.1, None) == -1
    # non-finite / non-positive scale
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 8, 4, 2, 64, 64, 1, float("inf"), None) == -1
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 8, 4, 2, 64, 64, 1, -1.0, None) == -1
    # Skv = 0
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 0, 4, 2, 64, 64, 0, 0.1, None) == -1
    # null pointers
    assert lib.attn_fwd(None, vp, vp, vp, None, 1, 8, 8, 4, 2, 64, 64, 1, 0.1, None) == -1
    # head dim outside the compiled set, d_qk != d_v
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 8, 4, 2, 96, 96, 1, 0.1, None) == -2
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 8, 4, 2, 128, 64, 1, 0.1, None) == -2
    # group size not a power of two
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 8, 8, 6, 2, 64, 64, 1, 0.1, None) == -2
    # causal with Sq > Skv
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 9, 8, 4, 2, 64, 64, 1, 0.1, None) == -2
    # misaligned pointer
    assert lib.attn_fwd(ctypes.c_void_p(18), vp, vp, vp, None, 1, 8, 8, 4, 2, 64, 64, 1, 0.1, None) == -3
    # empty batch / no query rows: nothing to do
    assert lib.attn_fwd(vp, vp, vp, vp, None, 0, 8, 8, 4, 2, 64, 64, 1, 0.1, None) == 0
    assert lib.attn_fwd(vp, vp, vp, vp, None, 1, 0, 8, 4, 2, 64, 64, 1, 0.1, None) == 0


def test_decode_validation(lib):
    vp = ctypes.c_void_p(256)
    out = ctypes.c_size_t(0)
    assert lib.attn_decode_workspace_bytes(32, 32, 8, 128, 128, 32768, ctypes.byref(out)) == 0
    # partial outputs (fp32, 128 wide) + (m, l) per (b, h, chunk); G = 4 heads
    # per unit: chunks of 2048 keys
    assert out.value == 32 * 32 * 16 * 128 * 4 + 32 * 32 * 16 * 8
    # G = 16: chunks of 1024 keys
    assert lib.attn_decode_workspace_bytes(2, 32, 2, 128, 128, 4096, ctypes.byref(out)) == 0
    assert out.value == 2 * 32 * 4 * 128 * 4 + 2 * 32 * 4 * 8
    assert lib.attn_decode_workspace_bytes(32, 32, 8, 96, 96, 4096, ctypes.byref(out)) == -2
    args = dict(B=2, n_q=8, n_kv=2, d_qk=128, d_v=128, S_max=1024)
    need = ctypes.c_size_t(0)
    lib.attn_decode_workspace_bytes(2, 8, 2, 128, 128, 1024, ctypes.byref(need))

    def call(ws_bytes=need.value, ws=vp, n_q=8, n_kv=2, d_qk=128, d_v=128, k_s=(8 * 1024 * 128, 1024 * 128, 128)):
        return lib.attn_decode(vp, vp, vp, vp, vp, vp, 2, n_q, n_kv, d_qk, d_v, 1024, *k_s, *k_s, 0.1, ws,
                               ws_bytes, None)
    assert call(ws_bytes=need.value - 1) == -4          # workspace too small
    assert call(ws=None) == -4                          # no workspace
    assert call(ws=ctypes.c_void_p(272)) == -3          # workspace not 256-byte aligned
    assert call(n_q=7) == -1                            # n_q % n_kv != 0
    assert call(d_qk=64, d_v=64) == -2                  # not a compiled decode shape
    assert call(k_s=(8 * 1024 * 128, 1024 * 128, 130)) == -3   # row stride not a multiple of 8


def test_rope_validation(lib):
    vp, al = ctypes.c_void_p(16), ctypes.c_void_p(4096)
    # tables: d must be even, base finite and positive; no positions is a no-op
    assert lib.attn_rope_tables(vp, vp, 8, 7, 10000.0, None) == -1
    assert lib.attn_rope_tables(vp, vp, 8, 8, 0.0, None) == -1
    assert lib.attn_rope_tables(vp, vp, 8, 8, float("inf"), None) == -1
    assert lib.attn_rope_tables(None, vp, 8, 8, 10000.0, None) == -1
    assert lib.attn_rope_tables(None, None, 0, 8, 10000.0, None) == 0
    # rotation pass: d a multiple of 8, every position inside the tables, 16-byte alignment
    assert lib.attn_rope_apply(vp, vp, 1, 2, 16, 12, 0, al, al, 64, None) == -1
    assert lib.attn_rope_apply(vp, vp, 1, 2, 16, 64, 49, al, al, 64, None) == -1
    assert lib.attn_rope_apply(vp, vp, 1, 2, 16, 64, -1, al, al, 64, None) == -1
    assert lib.attn_rope_apply(ctypes.c_void_p(24), vp, 1, 2, 16, 64, 0, al, al, 64, None) == -3
    assert lib.attn_rope_apply(vp, vp, 0, 2, 16, 64, 0, al, al, 64, None) == 0
    # prefill: tables covering every key, a key buffer, the prefill shape rules
    args = lambda n_pos=64, k_rot=vp, d=64, Sq=8, Skv=64, tab=al: (
        vp, vp, vp, vp, None, 1, Sq, Skv, 4, 2, d, d, 1, 0.125, tab, tab, n_pos, k_rot, None)
    assert lib.attn_fwd_rope(*args(n_pos=63)) == -1
    assert lib.attn_fwd_rope(*args(k_rot=None)) == -1
    assert lib.attn_fwd_rope(*args(tab=None)) == -1
    assert lib.attn_fwd_rope(*args(d=96)) == -2
    assert lib.attn_fwd_rope(*args(Sq=65, n_pos=65)) == -2
    assert lib.attn_fwd_rope(*args(tab=ctypes.c_void_p(4100))) == -3
    # decode: tables required, head dim 128 only (no MLA form)
    k_s = (2 * 1024 * 128, 1024 * 128, 128)
    assert lib.attn_decode_rope(vp, vp, vp, vp, vp, vp, 2, 8, 2, 128, 128, 1024, *k_s, *k_s, None, None, 64,
                                0.1, al, 1 << 20, None) == -1
    assert lib.attn_decode_rope(vp, vp, vp, vp, vp, vp, 1, 128, 1, 576, 512, 1024, *k_s, *k_s, al, al, 64,
                                0.1, al, 1 << 20, None) == -2


def test_window_fp8_paged_validation(lib):
    vp = ctypes.c_void_p(256)
    # sliding window: window >= 1, n_sink >= 0, queries no longer than keys
    assert lib.attn_fwd_window(vp, vp, vp, vp, None, 1, 8, 8, 4, 2, 64, 64, 0, 0, 0.1, None) == -1
    assert lib.attn_fwd_window(vp, vp, vp, vp, None, 1, 8, 8, 4, 2, 64, 64, 4, -1, 0.1, None) == -1
    assert lib.attn_fwd_window(vp, vp, vp, vp, None, 1, 9, 8, 4, 2, 64, 64, 4, 0, 0.1, None) == -2
    # e4m3 cache: scales required, strides in multiples of 16 bytes, workspace size
    need = ctypes.c_size_t(0)
    assert lib.attn_decode_fp8_workspace_bytes(2, 8, 2, 1024, ctypes.byref(need)) == 0
    s8 = (2 * 1024 * 128, 1024 * 128, 128)
    fp8 = lambda ks=vp, strides=s8, ws=need.value: lib.attn_decode_fp8(
        vp, vp, vp, ks, vp, vp, vp, None, 2, 8, 2, 1024, *strides, *strides, 0.1, vp, ws, None)
    assert fp8(ks=None) == -1
    assert fp8(strides=(2 * 1024 * 136, 1024 * 136, 136)) == -3
    assert fp8(ws=need.value - 1) == -4
    # paged cache: page sizes of whole TMA boxes, a positive pool, workspace size
    ps = (64 * 2 * 128, 2 * 128, 128)
    paged = lambda page=64, pool=100, ws=1 << 24: lib.attn_decode_paged(
        vp, vp, vp, vp, vp, vp, None, 2, 8, 2, 128, 128, page, 16, pool, *ps, *ps, 0.1, vp, ws, None)
    assert paged(page=0) == -1
    assert paged(pool=0) == -1
    assert paged(page=48) == -2
    assert paged(ws=16) == -4


def test_fp8_prefill_validation(lib):
    """attn_fwd_fp8 answers argument errors before any launch, and sizes its
    workspace as the keys and values widened to bf16 (256-byte aligned)."""
    vp = ctypes.c_void_p(256)
    out = ctypes.c_size_t(0)
    assert lib.attn_fwd_fp8_workspace_bytes(1, 4096, 4096, 32, 8, 128, ctypes.byref(out)) == 0
    assert out.value == 2 * (1 * 8 * 4096 * 128 * 2)
    assert lib.attn_fwd_fp8_workspace_bytes(2, 100, 130, 8, 2, 128, ctypes.byref(out)) == 0
    assert out.value == 2 * ((2 * 2 * 130 * 128 * 2 + 255) // 256 * 256)
    assert lib.attn_fwd_fp8_workspace_bytes(1, 64, 64, 4, 2, 64, ctypes.byref(out)) == -2     # d != 128
    lib.attn_fwd_fp8_workspace_bytes(1, 256, 256, 8, 2, 128, ctypes.byref(out))
    need = out.value

    def call(q=vp, qs=vp, n_q=8, n_kv=2, d=128, Sq=256, Skv=256, causal=1, scale=0.1, ws=vp, ws_bytes=need):
        return lib.attn_fwd_fp8(q, vp, vp, qs, vp, vp, vp, None, 1, Sq, Skv, n_q, n_kv, d, causal, scale, ws,
                                ws_bytes, None)
    assert call(n_q=7) == -1                      # n_q % n_kv
    assert call(causal=2) == -1
    assert call(scale=float("nan")) == -1
    assert call(q=None) == -1                     # null operand
    assert call(qs=None) == -1                    # null scales
    assert call(d=64) == -2                       # head dim 128 only
    assert call(n_q=12, n_kv=2) == -2             # group size not a power of two
    assert call(Sq=300, Skv=256) == -2            # causal with Sq > Skv
    assert call(q=ctypes.c_void_p(264)) == -3     # misaligned operand
    assert call(ws=None) == -4                    # workspace missing
    assert call(ws_bytes=need - 1) == -4          # workspace too small
    assert call(ws=ctypes.c_void_p(272)) == -3    # workspace not 256-byte aligned
    assert lib.attn_fwd_fp8(vp, vp, vp, vp, vp, vp, vp, None, 0, 256, 256, 8, 2, 128, 1, 0.1, None, 0, None) == 0
