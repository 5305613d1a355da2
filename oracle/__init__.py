"""fp64 CPU oracle for grouped-KV scaled-dot-product attention (forward).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The product path (the
CUDA library and its binding) never imports it, and this package never
imports the product.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only marshals arrays. Inputs of any float dtype are widened to
float64 exactly (bf16 -> fp64 is exact), so the oracle sees the very values
handed to the GPU.

Functions:
  sdpa(q, k, v, causal, scale, seqlens=None)      -> (o, lse)   full forward
  sdpa_rows(q_rows, rows, k, v, ...)             -> (o, lse)   sampled rows
  row_weights(q_row, b, h, i, k, v, ...)         -> (o, lse, w) one row + softmax weights
  online(q, k, v, causal, scale, block_r, block_c) -> (o, lse) FlashAttention-2 recurrence
  paged_to_cache(pages, block_table, seqlens)    -> cache      page-table gather (layout only)
  sdpa_varlen(q, k, v, cu_q, cu_k, causal, scale) -> (o, lse)  packed batch, one sdpa per sequence
  sdpa_window(q, k, v, causal, window, n_sink, scale, seqlens=None) -> (o, lse) sliding window + sinks
  dequant_e4m3(bytes, scale)                     -> fp64      FP8 (e4m3) cache values
  dequant_e4m3_tiles(bytes, scales, tile)        -> fp64      the same with one scale per token tile
  sdpa_fp8(q8, k8, v8, q_s, k_s, v_s, causal, scale) -> (o, lse) sdpa of per-tile dequantised e4m3 operands
  rope_tables(n_pos, d, base)                    -> (cos, sin) rotary tables [n_pos, d/2]
  rope(x, cos, sin, positions)                   -> fp64      rotary position embedding
  sdpa_rope(q, k, v, causal, scale, cos, sin)    -> (o, lse)  sdpa on rotated (bf16) queries and keys
  round_bf16(x)                                  -> fp64      nearest bf16 value, ties to even

Layouts: q [B, n_q, Sq, d_qk]; k [B, n_kv, Skv, d_k_row]; v [B, n_kv, Skv,
d_v_row] (any strides; the last dimension is read up to d_qk / d_v, so a
latent cache row of 576 can serve as key (all 576) and value (first 512)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.c_int64
_int = ctypes.c_int


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (-O2 -fopenmp, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _declare(lib):
    common = [_int] * 7 + [_i64] * 6 + [_i32p, _int, ctypes.c_double]
    lib.oracle_sdpa_fp64.argtypes = [_f64p] * 5 + common + [_int]
    lib.oracle_sdpa_fp64.restype = _int
    lib.oracle_sdpa_rows_fp64.argtypes = [_f64p] * 5 + [_i32p] * 3 + [_int] + common + [_int]
    lib.oracle_sdpa_rows_fp64.restype = _int
    lib.oracle_row_weights_fp64.argtypes = [_f64p] * 6 + [_int] * 3 + common
    lib.oracle_row_weights_fp64.restype = _i64
    lib.oracle_online_fp64.argtypes = [_f64p] * 5 + common + [_int, _int, _int]
    lib.oracle_online_fp64.restype = _int
    lib.oracle_sdpa_window_fp64.argtypes = ([_f64p] * 5 + [_int] * 7 + [_i64] * 6 +
                                            [_i32p, _int, _int, _int, ctypes.c_double, _int])
    lib.oracle_sdpa_window_fp64.restype = _int
    lib.oracle_rope_tables_fp64.argtypes = [_f64p, _f64p, _int, _int, ctypes.c_double]
    lib.oracle_rope_tables_fp64.restype = _int
    lib.oracle_rope_fp64.argtypes = [_f64p, _f64p, _i64, _int, _i32p, _f64p, _f64p, _int]
    lib.oracle_rope_fp64.restype = _int
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library. A non-default
    ``path`` loads another build of the same source (used by the mutation
    tests that plant mistakes in a copy of the oracle)."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _f64(x) -> np.ndarray:
    """Exact widening to a C-contiguous float64 array (torch or numpy in)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _kv_strides(t: np.ndarray):
    if t.ndim != 4:
        raise ValueError("k and v must be 4-D [B, n_kv, S, row]")
    es = t.itemsize
    return tuple(s // es for s in t.strides[:3])


def _ptr(a: np.ndarray, ty=_f64p):
    return a.ctypes.data_as(ty)


def _seq(seqlens):
    if seqlens is None:
        return None, None
    s = np.ascontiguousarray(np.asarray(
        seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
    return s, _ptr(s, _i32p)


def _nthreads(n):
    return int(n) if n else 0


def sdpa(q, k, v, causal: bool, scale: float, seqlens=None, d_qk=None, d_v=None,
         nthreads=None, lib=None):
    """Plain-definition forward. Returns (o [B,n_q,Sq,d_v], lse [B,n_q,Sq]) in fp64."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n_q, Sq, dq = q.shape
    _, n_kv, Skv, _ = k.shape
    d_qk = d_qk or dq
    d_v = d_v or v.shape[3]
    if d_qk != dq or d_qk > k.shape[3] or d_v > v.shape[3]:
        raise ValueError("head dims do not fit the given rows")
    o = np.zeros((B, n_q, Sq, d_v))
    lse = np.zeros((B, n_q, Sq))
    s_arr, s_ptr = _seq(seqlens)
    rc = lib.oracle_sdpa_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                              B, n_q, n_kv, Sq, Skv, d_qk, d_v,
                              *_kv_strides(k), *_kv_strides(v), s_ptr,
                              int(bool(causal)), float(scale), _nthreads(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o, lse


def sdpa_rows(q_rows, rows, k, v, B, n_q, Sq, causal: bool, scale: float,
              seqlens=None, d_v=None, nthreads=None, lib=None):
    """Sampled rows. ``rows`` is an int array [n, 3] of (b, h, i); ``q_rows``
    is [n, d_qk] (the query vectors of those rows). Returns (o [n, d_v], lse [n])."""
    lib = lib or load()
    q_rows, k, v = _f64(q_rows), _f64(k), _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    n, d_qk = q_rows.shape
    _, n_kv, Skv, _ = k.shape
    d_v = d_v or v.shape[3]
    rb = np.ascontiguousarray(rows[:, 0])
    rh = np.ascontiguousarray(rows[:, 1])
    ri = np.ascontiguousarray(rows[:, 2])
    o = np.zeros((n, d_v))
    lse = np.zeros((n,))
    s_arr, s_ptr = _seq(seqlens)
    rc = lib.oracle_sdpa_rows_fp64(_ptr(q_rows), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                   _ptr(rb, _i32p), _ptr(rh, _i32p), _ptr(ri, _i32p), n,
                                   B, n_q, n_kv, Sq, Skv, d_qk, d_v,
                                   *_kv_strides(k), *_kv_strides(v), s_ptr,
                                   int(bool(causal)), float(scale), _nthreads(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o, lse


def row_weights(q_row, b, h, i, k, v, B, n_q, Sq, causal: bool, scale: float,
                seqlens=None, d_v=None, lib=None):
    """One row: (o [d_v], lse, weights [Skv], n_visible)."""
    lib = lib or load()
    q_row, k, v = _f64(q_row).reshape(-1), _f64(k), _f64(v)
    _, n_kv, Skv, _ = k.shape
    d_qk = q_row.shape[0]
    d_v = d_v or v.shape[3]
    o = np.zeros((d_v,))
    lse = np.zeros((1,))
    w = np.zeros((max(Skv, 1),))
    s_arr, s_ptr = _seq(seqlens)
    nv = lib.oracle_row_weights_fp64(_ptr(q_row), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(w),
                                     int(b), int(h), int(i),
                                     B, n_q, n_kv, Sq, Skv, d_qk, d_v,
                                     *_kv_strides(k), *_kv_strides(v), s_ptr,
                                     int(bool(causal)), float(scale))
    if nv < 0:
        raise ValueError("oracle rejected the arguments")
    return o, float(lse[0]), w[:Skv], int(nv)


def online(q, k, v, causal: bool, scale: float, block_r: int, block_c: int,
           seqlens=None, d_v=None, nthreads=None, lib=None):
    """FlashAttention-2 tiled recurrence in fp64. Returns (o, lse)."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n_q, Sq, d_qk = q.shape
    _, n_kv, Skv, _ = k.shape
    d_v = d_v or v.shape[3]
    o = np.zeros((B, n_q, Sq, d_v))
    lse = np.zeros((B, n_q, Sq))
    s_arr, s_ptr = _seq(seqlens)
    rc = lib.oracle_online_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                B, n_q, n_kv, Sq, Skv, d_qk, d_v,
                                *_kv_strides(k), *_kv_strides(v), s_ptr,
                                int(bool(causal)), float(scale),
                                int(block_r), int(block_c), _nthreads(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o, lse


def paged_to_cache(pages, block_table, seqlens):
    """The logical cache a page table describes ("Attention deep dive",
    section 5: fixed-size pages addressed through a page table). pages is
    indexed [page, token in page, kv head, dim]; block_table [B, P] int;
    seqlens [B]. Token j of sequence b is token j % page_size of page
    block_table[b, j // page_size]. Returns float64 [B, n_kv, P*page_size,
    dim]: rows below the (clamped) length copied, rows at or past it zero, and
    rows of a page id outside the pool zero (the library reads such pages as
    zeros). No arithmetic: a gather written out row by row."""
    pages = _f64(pages)
    table = np.asarray(block_table.cpu().numpy() if hasattr(block_table, "cpu") else block_table, dtype=np.int64)
    lens = np.asarray(seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int64)
    num_pages, page_size, n_kv, dim = pages.shape
    B, P = table.shape
    cache = np.zeros((B, n_kv, P * page_size, dim))
    for b in range(B):
        n = min(max(int(lens[b]), 0), P * page_size)
        for j in range(n):
            pg = int(table[b, j // page_size])
            if 0 <= pg < num_pages:
                cache[b, :, j, :] = pages[pg, j % page_size]
    return cache


def sdpa_varlen(q, k, v, cu_q, cu_k, causal: bool, scale: float, nthreads=None, lib=None):
    """The plain definition over a packed batch: q [total_q, n_q, d], k/v
    [total_k, n_kv, d]; sequence b is rows cu_q[b]..cu_q[b+1]-1 of q and
    cu_k[b]..cu_k[b+1]-1 of k and v, attended on its own exactly as sdpa
    attends one batch element (causal alignment bottom-right per sequence).
    Returns (o [total_q, n_q, d_v], lse [n_q, total_q]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = np.asarray(cu_q.cpu().numpy() if hasattr(cu_q, "cpu") else cu_q, dtype=np.int64)
    ck = np.asarray(cu_k.cpu().numpy() if hasattr(cu_k, "cpu") else cu_k, dtype=np.int64)
    total_q, n_q, _ = q.shape
    d_v = v.shape[2]
    o = np.zeros((total_q, n_q, d_v))
    lse = np.full((n_q, total_q), -np.inf)
    for b in range(len(cq) - 1):
        qs, qe, ks_, ke = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if qe <= qs:
            continue
        qb = q[qs:qe].transpose(1, 0, 2)[None]           # [1, n_q, Sq_b, d]
        kb = k[ks_:ke].transpose(1, 0, 2)[None]          # [1, n_kv, Skv_b, d]
        vb = v[ks_:ke].transpose(1, 0, 2)[None]
        ob, lb = sdpa(qb, kb, vb, causal, scale, nthreads=nthreads, lib=lib)
        o[qs:qe] = ob[0].transpose(1, 0, 2)
        lse[:, qs:qe] = lb[0]
    return o, lse


def sdpa_window(q, k, v, causal: bool, window: int, n_sink: int, scale: float, seqlens=None, d_v=None,
                nthreads=None, lib=None):
    """Plain definition with a sliding window: of the visible keys of sdpa,
    key j stays only if p - j < window (p = the query's own position, the
    last visible key) or j < n_sink. Same layouts as sdpa."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n_q, Sq, d_qk = q.shape
    _, n_kv, Skv, _ = k.shape
    d_v = d_v or v.shape[3]
    o = np.zeros((B, n_q, Sq, d_v))
    lse = np.zeros((B, n_q, Sq))
    s_arr, s_ptr = _seq(seqlens)
    rc = lib.oracle_sdpa_window_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                     B, n_q, n_kv, Sq, Skv, d_qk, d_v,
                                     *_kv_strides(k), *_kv_strides(v), s_ptr,
                                     int(bool(causal)), int(window), int(n_sink), float(scale),
                                     _nthreads(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o, lse


def dequant_e4m3(raw, scale=None, head_axis=1):
    """Values of an FP8 e4m3 cache ("Flash Attention 3 and Multi-Headed Latent
    Attention", FP8 section: 8-bit e4m3 operands with scaling factors): each
    byte is 1 sign bit, 4 exponent bits (bias 7) and 3 mantissa bits;
    exponent 0 is subnormal (m * 2^-9), the pattern S.1111.111 is NaN and
    there are no infinities (largest finite 448). `scale` [n_kv] multiplies
    the values of each KV head (axis `head_axis`). Returns float64."""
    b = np.asarray(raw.cpu().numpy() if hasattr(raw, "cpu") else raw).view(np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * val
    val = np.where((e == 15) & (b & 7 == 7), np.nan, val)
    if scale is not None:
        sc = np.asarray(scale.cpu().numpy() if hasattr(scale, "cpu") else scale, dtype=np.float64)
        shape = [1] * val.ndim
        shape[head_axis] = -1
        val = val * sc.reshape(shape)
    return val


def dequant_e4m3_tiles(raw, scales, tile: int = 128):
    """Values of an e4m3 cache [B, n_kv, S, d] with one scale per tile of
    `tile` consecutive tokens of each (sequence, KV head) ("Flash Attention 3
    and Multi-Headed Latent Attention", FP8 section: per-tile scaling
    factors): token j of (b, g) is e4m3(byte) * scales[b, g, j // tile].
    `scales` [B, n_kv, ceil(S / tile)]. Returns float64."""
    val = dequant_e4m3(raw)
    sc = np.asarray(scales.cpu().numpy() if hasattr(scales, "cpu") else scales, dtype=np.float64)
    S = val.shape[2]
    tok_tile = np.arange(S) // tile                      # tile of each token
    return val * sc[:, :, tok_tile][..., None]


def sdpa_fp8(q8, k8, v8, q_scale, k_scale, v_scale, causal: bool, scale: float, tile: int = 128,
             nthreads=None, lib=None):
    """Attention over FP8 (e4m3) queries, keys and values with one scale per
    tile of `tile` rows of each (sequence, head) ("Flash Attention 3 and
    Multi-Headed Latent Attention", FP8 section: e4m3 operands with per-tile
    scaling factors): each operand is dequantised (dequant_e4m3_tiles), then
    the plain definition (sdpa) runs on the values. q8 [B, n_q, Sq, d],
    k8 / v8 [B, n_kv, Skv, d] bytes; q_scale [B, n_q, ceil(Sq / tile)],
    k_scale / v_scale [B, n_kv, ceil(Skv / tile)]."""
    q = dequant_e4m3_tiles(q8, q_scale, tile)
    k = dequant_e4m3_tiles(k8, k_scale, tile)
    v = dequant_e4m3_tiles(v8, v_scale, tile)
    return sdpa(q, k, v, causal, scale, nthreads=nthreads, lib=lib)


def rope_tables(n_pos: int, d: int, base: float, lib=None):
    """cos(m theta_j), sin(m theta_j) for m < n_pos, j < d/2, theta_j =
    base^(-2j/d) ("Attention Engineering: From MHA to GQA, MLA &
    FlashAttention", section 1: the geometric base frequencies and the
    [positions, d/2] cache tables). fp64, shape [n_pos, d/2] each."""
    lib = lib or load()
    c = np.zeros((n_pos, d // 2))
    s = np.zeros((n_pos, d // 2))
    if lib.oracle_rope_tables_fp64(_ptr(c), _ptr(s), int(n_pos), int(d), float(base)) != 0:
        raise ValueError("oracle rejected the arguments")
    return c, s


def rope(x, cos, sin, positions, lib=None):
    """Rotate every plane (x_{2j}, x_{2j+1}) of the last axis by its
    position's angle (section 1, real 2x2 block form). x [..., S, d];
    positions [S] (or broadcastable to x.shape[:-1]) index the tables
    cos/sin [n_pos, d/2] (fp32 values are widened exactly). Returns fp64."""
    lib = lib or load()
    x = _f64(x)
    d = x.shape[-1]
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(positions, dtype=np.int32), x.shape[:-1]))
    c = _f64(cos)
    s = _f64(sin)
    out = np.zeros_like(x)
    rc = lib.oracle_rope_fp64(_ptr(x), _ptr(out), int(np.prod(x.shape[:-1])), int(d), _ptr(pos, _i32p),
                              _ptr(c), _ptr(s), int(c.shape[0]))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (position outside the tables?)")
    return out


def round_bf16(x):
    """Round fp64 values to the nearest bf16 value (8 significant bits, ties
    to even), returned as fp64. Normal range only (|x| >= 2^-126 or 0)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                  # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def sdpa_rope(q, k, v, causal: bool, scale: float, cos, sin, operand_bf16: bool = True, nthreads=None,
              lib=None):
    """sdpa on rotated queries and keys (section 2, GQA formulation with
    RoPE(Q) RoPE(K)^T): key j at position j, query i at position
    Skv - Sq + i (the bottom-right alignment of the causal mask); values are
    not rotated. With operand_bf16 the rotated queries and keys are rounded
    to bf16 first: they are activations of a bf16 model, the operand type of
    the score contraction."""
    Sq, Skv = q.shape[2], k.shape[2]
    qr = rope(q, cos, sin, np.arange(Skv - Sq, Skv), lib=lib)
    kr = rope(k, cos, sin, np.arange(Skv), lib=lib)
    if operand_bf16:
        qr, kr = round_bf16(qr), round_bf16(kr)
    return sdpa(qr, kr, v, causal, scale, nthreads=nthreads, lib=lib)
