"""fp64 CPU oracle for VideoMLA latent-KV chunk attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline / reference arm may import this package.  The CUDA
library and its Python binding never import it, and it imports nothing from
them: the two share no code.  Inputs come from the seeded generators in
`workload`, which hold none of the method's arithmetic.

Source of every formula: VideoMLA, "Low-Rank Latent KV Cache for Minute-Scale
Autoregressive Video Diffusion".  The pages state the method in words only:
  * abstract: per-head keys and values are replaced by a head-shared low-rank
    content latent and a head-shared decoupled 3D-RoPE positional key, cutting
    per-token KV memory by 92.7%;
  * summary, "Approach": same statement, for chunk-causal autoregressive video
    diffusion on Wan2.1-T2V-1.3B;
  * summary, "Key results": 224 cached scalars per token against 3072, d_c = 192.
Multi-head latent attention itself is the DeepSeek-V2 construction the index
card lists under "Builds on".  The oracle writes out its plain definition:
explicit per-head keys K_h = [c . W_UK_h^T ; k_r] and values V_h = c . W_UV_h^T,
then ordinary max-subtracted softmax attention in fp64.

Readings where the pages are silent (each is also stated where it is used):
  * rope: 32 dims split (t 12, h 10, w 10); adjacent pairs; pair i of an axis
    with d_a dims turns at theta^(-2i/d_a) rad per position; theta = 1e4;
  * token n of a chunk starting at frame t0 sits at
    (t0 + n // (gh*gw), (n // gw) % gh, n % gw);
  * one call handles one chunk: every query sees every key in [0, n_kv)
    (cached frames plus its own chunk, bidirectional in the chunk);
  * the query's rope part q_r,h (32 dims per head) arrives unrotated and is
    rotated with the query's own position;
  * the softmax scale is an argument (the tests use 1/sqrt(128 + 32));
  * the query, rope-query and output projections around the attention are
    plain nn.Linear maps without bias (the pages name the Wan2.1 backbone and
    give no formula for them): `linear`.

Pins: tests/test_oracle_pins.py checks every function here against values
the pages print (the 224 / 3072 / 92.7% cache sizes), closed forms, invariants
of the rotary embedding, library routines (scaled-dot-product attention, a
complex-number rotation, mpmath cos/sin, torch's bf16 cast) and brute force
on tiny inputs.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

ROPE_SPLIT = (12, 10, 10)
ROPE_THETA = 1.0e4


# ---------------------------------------------------------------------------
# Sizes printed on the pages (abstract; summary "Key results")
# ---------------------------------------------------------------------------
def cache_scalars_per_token(d_c: int = 192, d_r: int = 32) -> int:
    """Latent cache: one head-shared content latent plus one head-shared rope key."""
    return d_c + d_r


def dense_scalars_per_token(heads: int = 12, d_head: int = 128) -> int:
    """Per-head cache: one key and one value of d_head per head."""
    return 2 * heads * d_head


def cache_reduction(d_c: int = 192, d_r: int = 32, heads: int = 12, d_head: int = 128) -> float:
    return 1.0 - cache_scalars_per_token(d_c, d_r) / dense_scalars_per_token(heads, d_head)


# ---------------------------------------------------------------------------
# bf16 decoding
# ---------------------------------------------------------------------------
def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# 3D rotary embedding (abstract: "decoupled 3D-RoPE positional key")
# ---------------------------------------------------------------------------
def rope_pair_axes(split=ROPE_SPLIT, theta=ROPE_THETA):
    """For each of the d_r/2 pairs: (axis index 0=t,1=h,2=w, angular frequency)."""
    out = []
    for axis, d_a in enumerate(split):
        for i in range(d_a // 2):
            out.append((axis, math.pow(theta, -2 * i / d_a)))
    return out


def token_positions(n_tok: int, t0: int, grid_h: int, grid_w: int):
    """(t, row, col) of the n_tok tokens of a chunk that starts at frame t0."""
    n = np.arange(n_tok, dtype=np.int64)
    per = grid_h * grid_w
    return t0 + n // per, (n // grid_w) % grid_h, n % grid_w


def rope3d(v: np.ndarray, t, row, col, split=ROPE_SPLIT, theta=ROPE_THETA) -> np.ndarray:
    """Rotate v[..., n, d_r] (float64) pairwise by the angles of positions (t, row, col)[n]."""
    v = np.asarray(v, dtype=np.float64)
    out = v.copy()
    pos = (np.asarray(t), np.asarray(row), np.asarray(col))
    for p, (axis, freq) in enumerate(rope_pair_axes(split, theta)):
        ang = pos[axis].astype(np.float64) * freq
        c, s = np.cos(ang), np.sin(ang)
        a, b = v[..., 2 * p], v[..., 2 * p + 1]
        out[..., 2 * p] = a * c - b * s
        out[..., 2 * p + 1] = a * s + b * c
    return out


# ---------------------------------------------------------------------------
# Cache append: ordered fp32, bit-exact target (C part, oracle/append_ref.c)
# ---------------------------------------------------------------------------
_lib = None


def _clib():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f32p = ctypes.POINTER(ctypes.c_float)
        i32p = ctypes.POINTER(ctypes.c_int)
        lib.oracle_cache_append.argtypes = [u16p, u16p, u16p, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                            i32p, ctypes.c_double, f32p, u16p]
        lib.oracle_cache_append.restype = None
        lib.oracle_ordered_dot.argtypes = [u16p, u16p, ctypes.c_int]
        lib.oracle_ordered_dot.restype = ctypes.c_float
        lib.oracle_round_bf16.argtypes = [f32p, u16p, ctypes.c_int64]
        lib.oracle_round_bf16.restype = None
        lib.oracle_rope_cos_sin.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int64, i32p, ctypes.c_double, f32p, f32p]
        lib.oracle_rope_cos_sin.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def cache_append(x_bits, w_dkv_bits, w_kr_bits, t0: int, grid_h: int, grid_w: int,
                 split=ROPE_SPLIT, theta=ROPE_THETA, want_fp32: bool = False):
    """Cache rows [c ; RoPE3D(k_r)] for tokens x[B, n_tok, D] (bf16 bits).

    Returns bf16 bits [B, n_tok, d_c + d_r] (and the fp32 values before rounding
    when want_fp32).  Token n sits at frame t0 + n // (gh*gw) (see token_positions).
    """
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if x.ndim == 2:
        x = x[None]
    wd = np.ascontiguousarray(w_dkv_bits, dtype=np.uint16)
    wk = np.ascontiguousarray(w_kr_bits, dtype=np.uint16)
    B, n_tok, D = x.shape
    d_c, d_r = wd.shape[0], wk.shape[0]
    assert wd.shape[1] == D and wk.shape[1] == D and d_c + d_r <= 1024 and d_r % 2 == 0
    out = np.empty((B, n_tok, d_c + d_r), dtype=np.uint16)
    out32 = np.empty((B, n_tok, d_c + d_r), dtype=np.float32) if want_fp32 else None
    sp = np.asarray(split, dtype=np.int32)
    _clib().oracle_cache_append(_ptr(x, ctypes.c_uint16), _ptr(wd, ctypes.c_uint16),
                                _ptr(wk, ctypes.c_uint16), B, n_tok, D, d_c, d_r,
                                int(t0), int(grid_h), int(grid_w), _ptr(sp, ctypes.c_int),
                                float(theta),
                                _ptr(out32, ctypes.c_float) if want_fp32 else None,
                                _ptr(out, ctypes.c_uint16))
    return (out, out32) if want_fp32 else out


def ordered_dot(a_bits, b_bits) -> float:
    a = np.ascontiguousarray(a_bits, dtype=np.uint16)
    b = np.ascontiguousarray(b_bits, dtype=np.uint16)
    return float(_clib().oracle_ordered_dot(_ptr(a, ctypes.c_uint16), _ptr(b, ctypes.c_uint16), a.size))


def round_bf16(a_f32) -> np.ndarray:
    a = np.ascontiguousarray(a_f32, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _clib().oracle_round_bf16(_ptr(a, ctypes.c_float), _ptr(out, ctypes.c_uint16), a.size)
    return out


def append_cos_sin(pair: int, t: int, row: int, col: int, split=ROPE_SPLIT, theta=ROPE_THETA):
    sp = np.asarray(split, dtype=np.int32)
    c = ctypes.c_float()
    s = ctypes.c_float()
    _clib().oracle_rope_cos_sin(pair, t, row, col, _ptr(sp, ctypes.c_int), theta,
                                ctypes.byref(c), ctypes.byref(s))
    return c.value, s.value


# ---------------------------------------------------------------------------
# Chunk attention over the latent cache (non-absorbed definition, fp64)
# ---------------------------------------------------------------------------
def _softmax_rows(s: np.ndarray) -> np.ndarray:
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=-1, keepdims=True)


def chunk_attention(q_bits, q_rope_bits, w_uk_bits, w_uv_bits, cache_bits, n_kv: int,
                    t0: int, grid_h: int, grid_w: int, scale: float, rows=None,
                    split=ROPE_SPLIT, theta=ROPE_THETA, row_block: int = 512) -> np.ndarray:
    """Per-head outputs out[b, i, h, :] for the queries of one chunk.

    q [B, Nq, H, d_h], q_rope [B, Nq, H, d_r] (unrotated), W_UK, W_UV [H*d_h, d_c],
    cache [B, cap, d_c + d_r] (rows [c ; rotated k_r]); keys are cache rows [0, n_kv).
    For head h:  K_h = [C . W_UK_h^T ; k_r],  V_h = C . W_UV_h^T,
                 Q_h = [q_h ; RoPE3D(q_rope_h, pos)],
                 out_h = softmax(scale * Q_h K_h^T) V_h.
    `rows` selects query indices (default: all).  Returns float64 [B, len(rows), H, d_h].
    """
    q = decode_bf16(q_bits)
    qr = decode_bf16(q_rope_bits)
    wuk = decode_bf16(w_uk_bits)
    wuv = decode_bf16(w_uv_bits)
    cache = decode_bf16(cache_bits)
    if q.ndim == 3:
        q, qr, cache = q[None], qr[None], cache[None]
    B, Nq, H, dh = q.shape
    d_r = qr.shape[-1]
    d_c = cache.shape[-1] - d_r
    rows = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    t, r, c = token_positions(Nq, t0, grid_h, grid_w)
    out = np.empty((B, len(rows), H, dh), dtype=np.float64)
    for b in range(B):
        C = cache[b, :n_kv, :d_c]
        kr = cache[b, :n_kv, d_c:]
        for h in range(H):
            K_h = np.concatenate([C @ wuk[h * dh:(h + 1) * dh].T, kr], axis=1)
            V_h = C @ wuv[h * dh:(h + 1) * dh].T
            for i0 in range(0, len(rows), row_block):
                sel = rows[i0:i0 + row_block]
                q_rot = rope3d(qr[b, sel, h], t[sel], r[sel], c[sel], split, theta)
                Q_h = np.concatenate([q[b, sel, h], q_rot], axis=1)
                P = _softmax_rows(scale * (Q_h @ K_h.T))
                out[b, i0:i0 + len(sel), h] = P @ V_h
    return out


def linear(x_bits, w_bits) -> np.ndarray:
    """y = x . W^T in float64 for x[..., in] and an nn.Linear weight W[out, in] (bf16 bits):
    the query, rope-query and output projections around the latent attention."""
    x = decode_bf16(x_bits)
    w = decode_bf16(w_bits)
    return x @ w.T


def materialized_kv(w_uk_bits, w_uv_bits, cache_bits, n_kv: int) -> np.ndarray:
    """Per-head content keys and values of cache rows [0, n_kv), float64
    [B, n_kv, 2H, d_h]: heads [0, H) hold K_h = C . W_UK_h^T, heads [H, 2H) hold
    V_h = C . W_UV_h^T (the non-absorbed keys/values of the abstract's shared latent)."""
    wuk = decode_bf16(w_uk_bits)
    wuv = decode_bf16(w_uv_bits)
    cache = decode_bf16(cache_bits)
    if cache.ndim == 2:
        cache = cache[None]
    d_c = wuk.shape[1]
    dh = 128
    H = wuk.shape[0] // dh
    C = cache[:, :n_kv, :d_c]
    out = np.empty((cache.shape[0], n_kv, 2 * H, dh), dtype=np.float64)
    for h in range(H):
        out[:, :, h] = C @ wuk[h * dh:(h + 1) * dh].T
        out[:, :, H + h] = C @ wuv[h * dh:(h + 1) * dh].T
    return out


def chunk_attention_absorbed(q_bits, q_rope_bits, w_uk_bits, w_uv_bits, cache_bits, n_kv: int,
                             t0: int, grid_h: int, grid_w: int, scale: float, rows=None,
                             split=ROPE_SPLIT, theta=ROPE_THETA) -> np.ndarray:
    """Same attention with W_UK absorbed into the queries and W_UV applied after P.C:
    s = scale * ((q_h W_UK_h) . c + RoPE(q_r) . k_r),  out_h = (softmax(s) . C) . W_UV_h^T."""
    q = decode_bf16(q_bits)
    qr = decode_bf16(q_rope_bits)
    wuk = decode_bf16(w_uk_bits)
    wuv = decode_bf16(w_uv_bits)
    cache = decode_bf16(cache_bits)
    if q.ndim == 3:
        q, qr, cache = q[None], qr[None], cache[None]
    B, Nq, H, dh = q.shape
    d_r = qr.shape[-1]
    d_c = cache.shape[-1] - d_r
    rows = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    t, r, c = token_positions(Nq, t0, grid_h, grid_w)
    out = np.empty((B, len(rows), H, dh), dtype=np.float64)
    for b in range(B):
        C = cache[b, :n_kv, :d_c]
        kr = cache[b, :n_kv, d_c:]
        for h in range(H):
            q_abs = q[b, rows, h] @ wuk[h * dh:(h + 1) * dh]
            q_rot = rope3d(qr[b, rows, h], t[rows], r[rows], c[rows], split, theta)
            P = _softmax_rows(scale * (q_abs @ C.T + q_rot @ kr.T))
            out[b, :, h] = (P @ C) @ wuv[h * dh:(h + 1) * dh].T
    return out


# ---------------------------------------------------------------------------
# Dense per-head attention (the 3072-scalar baseline layout)
# ---------------------------------------------------------------------------
def dense_attention(q_bits, k_bits, v_bits, scale: float, rows=None, row_block: int = 512):
    """out[b, i, h] = softmax(scale * q_h,i . K_h^T) V_h with q [B,Nq,H,d], k,v [B,Nk,H,d]."""
    q = decode_bf16(q_bits)
    k = decode_bf16(k_bits)
    v = decode_bf16(v_bits)
    if q.ndim == 3:
        q, k, v = q[None], k[None], v[None]
    B, Nq, H, d = q.shape
    rows = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((B, len(rows), H, v.shape[-1]), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            K = k[b, :, h]
            V = v[b, :, h]
            for i0 in range(0, len(rows), row_block):
                sel = rows[i0:i0 + row_block]
                P = _softmax_rows(scale * (q[b, sel, h] @ K.T))
                out[b, i0:i0 + len(sel), h] = P @ V
    return out
