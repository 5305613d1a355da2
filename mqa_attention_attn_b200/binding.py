"""Python binding of libattn_b200.so (argument marshalling only).

Every function here forwards torch tensors' device pointers and sizes to the
C ABI declared in include/attn.h; all arithmetic runs in the library's CUDA
kernels. There is no fallback: if the library is missing or a call fails, a
RuntimeError is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn_b200.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "attn.h")

ATTN_OK = 0
STATUS = {
    0: "ATTN_OK", -1: "ATTN_ERR_INVALID_ARG", -2: "ATTN_ERR_UNSUPPORTED", -3: "ATTN_ERR_MISALIGNED",
    -4: "ATTN_ERR_WORKSPACE", -5: "ATTN_ERR_CUDA", -6: "ATTN_ERR_DEVICE_TIMEOUT", -7: "ATTN_ERR_DEVICE_RANGE",
}

_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({status_string(code)})")


def header_functions() -> list[str]:
    """Names of the functions include/attn.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(attn_\w+)\s*\(", text, flags=re.M)


def lib() -> ctypes.CDLL:
    """The loaded library. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} not built: run `python -m mqa_attention_attn_b200.build` "
                               "(no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        L.attn_fwd.argtypes = [_vp] * 5 + [_i] * 8 + [ctypes.c_float, _vp]
        L.attn_fwd.restype = _i
        L.attn_fwd_fp8_workspace_bytes.argtypes = [_i] * 6 + [ctypes.POINTER(ctypes.c_size_t)]
        L.attn_fwd_fp8_workspace_bytes.restype = _i
        L.attn_fwd_fp8.argtypes = [_vp] * 8 + [_i] * 7 + [ctypes.c_float, _vp, ctypes.c_size_t, _vp]
        L.attn_fwd_fp8.restype = _i
        L.attn_fwd_varlen.argtypes = [_vp] * 7 + [_i] * 9 + [ctypes.c_float, _vp]
        L.attn_fwd_window.argtypes = [_vp] * 5 + [_i] * 9 + [ctypes.c_float, _vp]
        L.attn_fwd_window.restype = _i
        L.attn_fwd_varlen.restype = _i
        L.attn_decode_workspace_bytes.argtypes = [_i] * 6 + [ctypes.POINTER(ctypes.c_size_t)]
        L.attn_decode_workspace_bytes.restype = _i
        L.attn_decode.argtypes = ([_vp] * 6 + [_i] * 6 + [_i64] * 6 +
                                  [ctypes.c_float, _vp, ctypes.c_size_t, _vp])
        L.attn_decode.restype = _i
        L.attn_decode_window.argtypes = ([_vp] * 6 + [_i] * 6 + [_i64] * 6 + [_i, _i] +
                                         [ctypes.c_float, _vp, ctypes.c_size_t, _vp])
        L.attn_decode_window.restype = _i
        L.attn_decode_fp8_workspace_bytes.argtypes = [_i] * 4 + [ctypes.POINTER(ctypes.c_size_t)]
        L.attn_decode_fp8_workspace_bytes.restype = _i
        L.attn_decode_fp8.argtypes = ([_vp] * 8 + [_i] * 4 + [_i64] * 6 +
                                      [ctypes.c_float, _vp, ctypes.c_size_t, _vp])
        L.attn_decode_fp8.restype = _i
        L.attn_decode_fp8_tiles.argtypes = ([_vp] * 8 + [_i] * 4 + [_i64] * 6 +
                                            [ctypes.c_float, _vp, ctypes.c_size_t, _vp])
        L.attn_decode_fp8_tiles.restype = _i
        L.attn_decode_paged.argtypes = ([_vp] * 7 + [_i] * 8 + [_i64] * 6 +
                                        [ctypes.c_float, _vp, ctypes.c_size_t, _vp])
        L.attn_fwd_paged.argtypes = [_vp] * 8 + [_i] * 10 + [_i64] * 6 + [_i, ctypes.c_float, _vp]
        L.attn_fwd_paged.restype = _i
        L.attn_decode_paged.restype = _i
        L.attn_rope_tables.argtypes = [_vp, _vp, _i, _i, ctypes.c_double, _vp]
        L.attn_rope_tables.restype = _i
        L.attn_rope_apply.argtypes = [_vp, _vp] + [_i] * 5 + [_vp, _vp, _i, _vp]
        L.attn_rope_apply.restype = _i
        L.attn_fwd_rope.argtypes = [_vp] * 5 + [_i] * 8 + [ctypes.c_float, _vp, _vp, _i, _vp, _vp]
        L.attn_fwd_rope.restype = _i
        L.attn_decode_rope.argtypes = ([_vp] * 6 + [_i] * 6 + [_i64] * 6 + [_vp, _vp, _i] +
                                       [ctypes.c_float, _vp, ctypes.c_size_t, _vp])
        L.attn_decode_rope.restype = _i
        L.attn_status_string.argtypes = [_i]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_device_status.argtypes = [_vp]
        L.attn_device_status.restype = _i
        L.attn_selftest_timeout.argtypes = [_i, _vp]
        L.attn_selftest_timeout.restype = _i
        L.attn_selftest_ex2.argtypes = [_vp, _vp, _vp, _i, _vp]
        L.attn_selftest_ex2.restype = _i
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().attn_status_string(int(code)).decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(code: int, what: str):
    if code != ATTN_OK:
        raise AttnError(code, what)


def attn_fwd(q, k, v, causal: bool, scale: float, o=None, lse=None, stream=None, want_lse=True):
    """Prefill forward. q [B,n_q,Sq,d], k/v [B,n_kv,Skv,d] bf16 CUDA tensors
    (contiguous). Returns (o [B,n_q,Sq,d] bf16, lse [B,n_q,Sq] fp32 or None)."""
    B, n_q, Sq, d_qk = q.shape
    _, n_kv, Skv, _ = k.shape
    d_v = v.shape[3]
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    if o is None:
        o = torch.empty((B, n_q, Sq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Sq), dtype=torch.float32, device=q.device)
    rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Sq, Skv, n_q, n_kv, d_qk, d_v,
                        int(bool(causal)), float(scale), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_fwd")
    return o, lse


def fwd_fp8_workspace_bytes(B, Sq, Skv, n_q, n_kv, d) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().attn_fwd_fp8_workspace_bytes(B, Sq, Skv, n_q, n_kv, d, ctypes.byref(out)),
           "attn_fwd_fp8_workspace_bytes")
    return out.value


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, causal: bool, scale: float, o=None, lse=None,
                 workspace=None, stream=None, want_lse=True):
    """Prefill forward on e4m3 operands with one scale per 128-row tile.
    q8 [B,n_q,Sq,d], k8/v8 [B,n_kv,Skv,d]: contiguous one-byte CUDA tensors
    (float8_e4m3fn or uint8 bytes); q_scale [B,n_q,ceil(Sq/128)],
    k_scale/v_scale [B,n_kv,ceil(Skv/128)]: contiguous fp32 CUDA tensors.
    Returns (o [B,n_q,Sq,d] bf16, lse [B,n_q,Sq] fp32 or None)."""
    B, n_q, Sq, d = q8.shape
    _, n_kv, Skv, _ = k8.shape
    for t in (q8, k8, v8):
        if t.element_size() != 1 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q8, k8, v8 must be contiguous one-byte CUDA tensors")
    shapes = ((q_scale, (B, n_q, (Sq + 127) // 128)), (k_scale, (B, n_kv, (Skv + 127) // 128)),
              (v_scale, (B, n_kv, (Skv + 127) // 128)))
    for t, shp in shapes:
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shp:
            raise ValueError(f"scales must be contiguous fp32 CUDA tensors of shape {shp}")
    if o is None:
        o = torch.empty((B, n_q, Sq, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Sq), dtype=torch.float32, device=q8.device)
    if workspace is None:
        workspace = torch.empty(max(fwd_fp8_workspace_bytes(B, Sq, Skv, n_q, n_kv, d), 1), dtype=torch.uint8,
                                device=q8.device)
    rc = lib().attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), _ptr(o),
                            _ptr(lse), B, Sq, Skv, n_q, n_kv, d, int(bool(causal)), float(scale), _ptr(workspace),
                            workspace.numel(), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_fwd_fp8")
    return o, lse


def attn_fwd_window(q, k, v, window: int, n_sink: int, scale: float, o=None, lse=None, stream=None, want_lse=True):
    """Causal prefill with a sliding window of `window` keys and `n_sink`
    always-visible initial keys. Layouts as attn_fwd."""
    B, n_q, Sq, d_qk = q.shape
    _, n_kv, Skv, _ = k.shape
    d_v = v.shape[3]
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    if o is None:
        o = torch.empty((B, n_q, Sq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Sq), dtype=torch.float32, device=q.device)
    rc = lib().attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Sq, Skv, n_q, n_kv, d_qk, d_v,
                               int(window), int(n_sink), float(scale), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_fwd_window")
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool, scale: float, o=None,
                    lse=None, stream=None, want_lse=True):
    """Prefill over a packed batch. q [total_q,n_q,d], k/v [total_k,n_kv,d]
    bf16 contiguous CUDA tensors; cu_seqlens_q/k int32 [B+1] on the device.
    Returns (o [total_q,n_q,d] bf16, lse [n_q,total_q] fp32 or None)."""
    total_q, n_q, d_qk = q.shape
    total_k, n_kv, _ = k.shape
    d_v = v.shape[2]
    B = cu_seqlens_q.numel() - 1
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    for t in (cu_seqlens_q, cu_seqlens_k):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.numel() != B + 1:
            raise ValueError("cu_seqlens must be contiguous int32 CUDA tensors of B + 1 offsets")
    if o is None:
        o = torch.empty((total_q, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((n_q, total_q), dtype=torch.float32, device=q.device)
    rc = lib().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                               _ptr(cu_seqlens_k), B, int(max_seqlen_q), total_q, total_k, n_q, n_kv, d_qk, d_v,
                               int(bool(causal)), float(scale), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_fwd_varlen")
    return o, lse


def decode_workspace_bytes(B, n_q, n_kv, d_qk, d_v, S_max) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().attn_decode_workspace_bytes(B, n_q, n_kv, d_qk, d_v, S_max, ctypes.byref(out)),
           "attn_decode_workspace_bytes")
    return int(out.value)


def _elem_strides(t):
    """Element strides of the three outer dimensions of a 4-D cache or page
    pool whose innermost dimension is unit-stride."""
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("cache must be 4-D with a unit inner stride")
    return t.stride(0), t.stride(1), t.stride(2)


def attn_decode(q, kcache, vcache, seqlens, scale: float, d_v=None, o=None, lse=None, workspace=None,
                stream=None, want_lse=True):
    """Decode one query token per sequence. q [B,n_q,d_qk]; kcache/vcache
    [B,n_kv,S_max,row] (any strides with a unit inner stride; they may be the
    same tensor); seqlens int32 [B] on the device. Returns (o, lse)."""
    B, n_q, d_qk = q.shape
    _, n_kv, S_max, _ = kcache.shape
    d_v = d_v or vcache.shape[3]
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()):
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    if seqlens.dtype != torch.int32 or not seqlens.is_cuda:
        raise ValueError("seqlens must be an int32 CUDA tensor")
    ks, vs = _elem_strides(kcache), _elem_strides(vcache)
    if o is None:
        o = torch.empty((B, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_workspace_bytes(B, n_q, n_kv, d_qk, d_v, S_max)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    rc = lib().attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(o), _ptr(lse),
                           B, n_q, n_kv, d_qk, d_v, S_max, *ks, *vs, float(scale),
                           _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_decode")
    return o, lse


def attn_decode_window(q, kcache, vcache, seqlens, window: int, n_sink: int, scale: float, o=None, lse=None,
                       workspace=None, stream=None, want_lse=True):
    """attn_decode keeping only the last `window` keys of each sequence and
    its first `n_sink` keys. Arguments as attn_decode (head dim 128)."""
    B, n_q, d_qk = q.shape
    _, n_kv, S_max, _ = kcache.shape
    d_v = vcache.shape[3]
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()):
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    if seqlens.dtype != torch.int32 or not seqlens.is_cuda:
        raise ValueError("seqlens must be an int32 CUDA tensor")
    ks, vs = _elem_strides(kcache), _elem_strides(vcache)
    if o is None:
        o = torch.empty((B, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_workspace_bytes(B, n_q, n_kv, d_qk, d_v, S_max)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    rc = lib().attn_decode_window(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(o), _ptr(lse),
                                  B, n_q, n_kv, d_qk, d_v, S_max, *ks, *vs, int(window), int(n_sink), float(scale),
                                  _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_decode_window")
    return o, lse


def decode_fp8_workspace_bytes(B, n_q, n_kv, S_max) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().attn_decode_fp8_workspace_bytes(B, n_q, n_kv, S_max, ctypes.byref(out)),
           "attn_decode_fp8_workspace_bytes")
    return int(out.value)


def attn_decode_fp8(q, kcache, vcache, k_scale, v_scale, seqlens, scale: float, o=None, lse=None, workspace=None,
                    stream=None, want_lse=True):
    """Decode against an e4m3 cache: kcache/vcache [B,n_kv,S_max,128] of
    torch.float8_e4m3fn (or uint8 bytes), any strides with a unit inner
    stride; k_scale/v_scale fp32 [n_kv] on the device."""
    B, n_q, d = q.shape
    _, n_kv, S_max, _ = kcache.shape
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()):
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    for t in (kcache, vcache):
        if t.element_size() != 1 or not t.is_cuda:
            raise ValueError("the FP8 cache must be a one-byte-per-element CUDA tensor")
    for t in (k_scale, v_scale):
        if t.dtype != torch.float32 or not t.is_cuda or t.numel() != n_kv:
            raise ValueError("k_scale / v_scale must be fp32 CUDA tensors of n_kv entries")
    ks, vs = _elem_strides(kcache), _elem_strides(vcache)
    if o is None:
        o = torch.empty((B, n_q, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(decode_fp8_workspace_bytes(B, n_q, n_kv, S_max), 1), dtype=torch.uint8,
                                device=q.device)
    rc = lib().attn_decode_fp8(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(k_scale), _ptr(v_scale), _ptr(seqlens),
                               _ptr(o), _ptr(lse), B, n_q, n_kv, S_max, *ks, *vs, float(scale), _ptr(workspace),
                               workspace.numel(), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_decode_fp8")
    return o, lse


def attn_decode_fp8_tiles(q, kcache, vcache, k_scales, v_scales, seqlens, scale: float, o=None, lse=None,
                          workspace=None, stream=None, want_lse=True):
    """attn_decode_fp8 with one scale per 128-key tile: k_scales/v_scales
    contiguous fp32 [B, n_kv, ceil(S_max / 128)] on the device."""
    B, n_q, d = q.shape
    _, n_kv, S_max, _ = kcache.shape
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()):
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    for t in (kcache, vcache):
        if t.element_size() != 1 or not t.is_cuda:
            raise ValueError("the FP8 cache must be a one-byte-per-element CUDA tensor")
    n_tiles = (S_max + 127) // 128
    for t in (k_scales, v_scales):
        if (t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous()
                or tuple(t.shape) != (B, n_kv, n_tiles)):
            raise ValueError("k_scales / v_scales must be contiguous fp32 CUDA tensors [B, n_kv, ceil(S_max/128)]")
    ks, vs = _elem_strides(kcache), _elem_strides(vcache)
    if o is None:
        o = torch.empty((B, n_q, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(decode_fp8_workspace_bytes(B, n_q, n_kv, S_max), 1), dtype=torch.uint8,
                                device=q.device)
    rc = lib().attn_decode_fp8_tiles(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(k_scales), _ptr(v_scales),
                                     _ptr(seqlens), _ptr(o), _ptr(lse), B, n_q, n_kv, S_max, *ks, *vs, float(scale),
                                     _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_decode_fp8_tiles")
    return o, lse


def attn_decode_paged(q, k_pages, v_pages, block_table, seqlens, scale: float, o=None, lse=None, workspace=None,
                      stream=None, want_lse=True):
    """Decode against a paged cache. q [B,n_q,128]; k_pages/v_pages indexed
    [page, token in page, kv head, dim] (any strides with a unit inner
    stride); block_table int32 [B, pages_per_seq] and seqlens int32 [B] on the
    device. Returns (o, lse)."""
    B, n_q, d = q.shape
    num_pages, page_size, n_kv, _ = k_pages.shape
    pages_per_seq = block_table.shape[1]
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()):
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    for t in (block_table, seqlens):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("block_table and seqlens must be contiguous int32 CUDA tensors")
    ks, vs = _elem_strides(k_pages), _elem_strides(v_pages)
    if o is None:
        o = torch.empty((B, n_q, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_workspace_bytes(B, n_q, n_kv, d, d, page_size * pages_per_seq)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    rc = lib().attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seqlens), _ptr(o),
                                 _ptr(lse), B, n_q, n_kv, d, d, page_size, pages_per_seq, num_pages, *ks, *vs,
                                 float(scale), _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_decode_paged")
    return o, lse


def attn_fwd_paged(q, k_pages, v_pages, block_table, cu_seqlens_q, seqlens_k, max_seqlen_q: int, causal: bool,
                   scale: float, o=None, lse=None, stream=None, want_lse=True):
    """Prefill of a packed batch against a paged cache. q [total_q,n_q,d] bf16
    contiguous; k_pages/v_pages indexed [page, token in page, kv head, dim]
    (any strides with a unit inner stride); block_table int32 [B,
    pages_per_seq], cu_seqlens_q int32 [B+1] and seqlens_k int32 [B] on the
    device. Returns (o [total_q,n_q,d] bf16, lse [n_q,total_q] fp32 or None)."""
    total_q, n_q, d = q.shape
    num_pages, page_size, n_kv, d_k = k_pages.shape
    B, pages_per_seq = block_table.shape
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()):
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    for t in (block_table, cu_seqlens_q, seqlens_k):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("block_table, cu_seqlens_q and seqlens_k must be contiguous int32 CUDA tensors")
    if cu_seqlens_q.numel() != B + 1 or seqlens_k.numel() != B:
        raise ValueError("cu_seqlens_q needs B + 1 offsets and seqlens_k B lengths")
    ks, vs = _elem_strides(k_pages), _elem_strides(v_pages)
    d_v = v_pages.shape[3]
    if o is None:
        o = torch.empty((total_q, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((n_q, total_q), dtype=torch.float32, device=q.device)
    rc = lib().attn_fwd_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(cu_seqlens_q),
                              _ptr(seqlens_k), _ptr(o), _ptr(lse), B, int(max_seqlen_q), total_q, n_q, n_kv, d, d_v,
                              page_size, pages_per_seq, num_pages, *ks, *vs, int(bool(causal)), float(scale),
                              ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_fwd_paged")
    return o, lse


def device_status(stream=None) -> int:
    """Synchronise the stream, read and clear the device status word."""
    return int(lib().attn_device_status(ctypes.c_void_p(_stream(stream))))


def selftest_timeout(timeout_us: int, stream=None):
    _check(lib().attn_selftest_timeout(int(timeout_us), ctypes.c_void_p(_stream(stream))),
           "attn_selftest_timeout")


def selftest_ex2(x, stream=None):
    """(poly, sfu) base-2 exponentials of a float32 CUDA tensor x, as the
    prefill softmax evaluates them."""
    x = x.contiguous()
    yp, ys = torch.empty_like(x), torch.empty_like(x)
    _check(lib().attn_selftest_ex2(_ptr(x), _ptr(yp), _ptr(ys), x.numel(), ctypes.c_void_p(_stream(stream))),
           "attn_selftest_ex2")
    return yp, ys


def _tables(cos, sin):
    for t in (cos, sin):
        if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and t.dim() == 2):
            raise ValueError("rotary tables must be contiguous fp32 CUDA tensors [n_pos, d/2]")
    if cos.shape != sin.shape:
        raise ValueError("cos and sin tables differ in shape")
    return cos.shape[0], cos.shape[1]


def rope_tables(n_pos: int, d: int, base: float, device="cuda", stream=None):
    """cos, sin [n_pos, d/2] fp32 on the device (attn_rope_tables)."""
    cos = torch.empty((n_pos, d // 2), dtype=torch.float32, device=device)
    sin = torch.empty_like(cos)
    _check(lib().attn_rope_tables(_ptr(cos), _ptr(sin), int(n_pos), int(d), float(base),
                                  ctypes.c_void_p(_stream(stream))), "attn_rope_tables")
    return cos, sin


def rope_apply(x, cos, sin, pos0: int = 0, out=None, stream=None):
    """RoPE of x [B, H, S, d] bf16 (row s at position pos0 + s); returns out
    (a new tensor unless given; it may be x)."""
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 4):
        raise ValueError("x must be a contiguous bf16 CUDA tensor [B, H, S, d]")
    n_pos, _ = _tables(cos, sin)
    if out is None:
        out = torch.empty_like(x)
    B, H, S, d = x.shape
    _check(lib().attn_rope_apply(_ptr(x), _ptr(out), B, H, S, d, int(pos0), _ptr(cos), _ptr(sin), n_pos,
                                 ctypes.c_void_p(_stream(stream))), "attn_rope_apply")
    return out


def attn_fwd_rope(q, k, v, causal: bool, scale: float, cos, sin, k_rot=None, o=None, lse=None, stream=None,
                  want_lse=True):
    """attn_fwd on RoPE-rotated q and k (given unrotated); the rotated keys
    are written to k_rot (allocated unless given; it may be k). Returns
    (o, lse, k_rot)."""
    B, n_q, Sq, d_qk = q.shape
    _, n_kv, Skv, _ = k.shape
    d_v = v.shape[3]
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    n_pos, _ = _tables(cos, sin)
    if k_rot is None:
        k_rot = torch.empty_like(k)
    if o is None:
        o = torch.empty((B, n_q, Sq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Sq), dtype=torch.float32, device=q.device)
    rc = lib().attn_fwd_rope(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Sq, Skv, n_q, n_kv, d_qk, d_v,
                             int(bool(causal)), float(scale), _ptr(cos), _ptr(sin), n_pos, _ptr(k_rot),
                             ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_fwd_rope")
    return o, lse, k_rot


def attn_decode_rope(q, kcache, vcache, seqlens, scale: float, cos, sin, o=None, lse=None, workspace=None,
                     stream=None, want_lse=True):
    """attn_decode with q rotated at position seqlens[b] - 1 (the cache holds
    rotated keys). Arguments as attn_decode plus the tables (head dim 128)."""
    B, n_q, d_qk = q.shape
    _, n_kv, S_max, _ = kcache.shape
    d_v = vcache.shape[3]
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()):
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    if seqlens.dtype != torch.int32 or not seqlens.is_cuda:
        raise ValueError("seqlens must be an int32 CUDA tensor")
    n_pos, _ = _tables(cos, sin)
    ks, vs = _elem_strides(kcache), _elem_strides(vcache)
    if o is None:
        o = torch.empty((B, n_q, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = decode_workspace_bytes(B, n_q, n_kv, d_qk, d_v, S_max)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    rc = lib().attn_decode_rope(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(o), _ptr(lse),
                                B, n_q, n_kv, d_qk, d_v, S_max, *ks, *vs, _ptr(cos), _ptr(sin), n_pos,
                                float(scale), _ptr(workspace), workspace.numel(), ctypes.c_void_p(_stream(stream)))
    _check(rc, "attn_decode_rope")
    return o, lse
