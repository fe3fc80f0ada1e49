"""Pins for the fp64 oracle: each check ties it to something other than itself.

Sources: VideoMLA, "Low-Rank Latent KV Cache for Minute-Scale Autoregressive
Video Diffusion" (abstract; summary page "Approach" and "Key results").  The
pages give the method in words; the pins therefore use the printed cache sizes
(tests/golden/cache_size.txt), closed forms, invariants of the rotary
embedding, library routines (torch scaled-dot-product attention, complex
multiplication, mpmath, torch's bf16 cast) and brute force on tiny inputs.
The last group plants plausible mistakes in copies of oracle functions and
checks that the pins catch them.
"""
from __future__ import annotations

import cmath
import math
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle
import workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            vals[k] = float(v)
    return vals


# --------------------------------------------------------------------------
# Printed numbers
# --------------------------------------------------------------------------
def test_cache_size_matches_pages():
    g = _golden("cache_size.txt")
    assert oracle.cache_scalars_per_token(int(g["d_c"]), 32) == g["latent_scalars_per_token"]
    assert oracle.dense_scalars_per_token(12, 128) == g["dense_scalars_per_token"]
    assert round(100.0 * oracle.cache_reduction(), 1) == g["reduction_percent"]


def test_workload_shapes_match_pages():
    # 480P: 30 x 52 latent patches per frame; 21-frame window = 18 cached + 3 chunk frames.
    w = workload.CONFIGS["480p"]
    assert (w.n_q, w.n_cached, w.n_kv) == (4680, 28080, 32760)
    w = workload.CONFIGS["1080p"]
    assert (w.n_q, w.n_cached, w.n_kv) == (24480, 48960, 73440)
    w = workload.CONFIGS["tiny"]
    assert (w.n_q, w.n_kv) == (192, 576)
    assert w.d_c + w.d_r == 224 and 2 * w.heads * w.d_head == 3072


# --------------------------------------------------------------------------
# Rotary embedding
# --------------------------------------------------------------------------
def _complex_rope(v, t, r, c, split=(12, 10, 10), theta=1e4):
    """Independent statement: pair p is the complex number v[2p] + i v[2p+1],
    multiplied by exp(i * pos_axis * theta^(-2 i / d_axis))."""
    out = np.empty_like(v)
    p = 0
    for axis, d_a in enumerate(split):
        pos = (t, r, c)[axis]
        for i in range(d_a // 2):
            z = complex(v[2 * p], v[2 * p + 1]) * cmath.exp(1j * pos * theta ** (-2.0 * i / d_a))
            out[2 * p], out[2 * p + 1] = z.real, z.imag
            p += 1
    return out


def test_rope_frequencies_printed_values():
    axes = oracle.rope_pair_axes()
    assert len(axes) == 16
    assert [a for a, _ in axes] == [0] * 6 + [1] * 5 + [2] * 5
    # First pair of each axis turns at 1 rad/position; last t pair at 1e4^(-10/12) = 10^(-10/3).
    assert axes[0][1] == 1.0 and axes[6][1] == 1.0 and axes[11][1] == 1.0
    assert axes[5][1] == pytest.approx(10 ** (-10 / 3), rel=1e-15)
    assert axes[10][1] == pytest.approx(10 ** (-16 / 5), rel=1e-15)


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(1)
    for _ in range(20):
        v = rng.standard_normal(32)
        t, r, c = (int(x) for x in rng.integers(0, 200, size=3))
        got = oracle.rope3d(v[None], np.array([t]), np.array([r]), np.array([c]))[0]
        np.testing.assert_allclose(got, _complex_rope(v, t, r, c), rtol=0, atol=1e-12)


def test_rope_norm_identity_and_relative_offset():
    rng = np.random.default_rng(2)
    q = rng.standard_normal(32)
    k = rng.standard_normal(32)
    z = np.array([0])
    np.testing.assert_allclose(oracle.rope3d(q[None], z, z, z)[0], q, atol=0)
    for _ in range(20):
        p1 = rng.integers(0, 60, size=3)
        p2 = rng.integers(0, 60, size=3)
        s = rng.integers(0, 60, size=3)
        rq = oracle.rope3d(q[None], *[np.array([x]) for x in p1])[0]
        assert np.linalg.norm(rq) == pytest.approx(np.linalg.norm(q), rel=1e-13)
        d1 = rq @ oracle.rope3d(k[None], *[np.array([x]) for x in p2])[0]
        d2 = (oracle.rope3d(q[None], *[np.array([x]) for x in p1 + s])[0]
              @ oracle.rope3d(k[None], *[np.array([x]) for x in p2 + s])[0])
        assert d1 == pytest.approx(d2, rel=1e-10, abs=1e-10)
    # ... and it does depend on the offset
    a = oracle.rope3d(q[None], np.array([0]), np.array([0]), np.array([0]))[0] @ k
    b = oracle.rope3d(q[None], np.array([1]), np.array([0]), np.array([0]))[0] @ k
    assert abs(a - b) > 1e-3


def test_rope_axis_blocks():
    rng = np.random.default_rng(3)
    v = rng.standard_normal(32)
    base = oracle.rope3d(v[None], np.array([5]), np.array([5]), np.array([5]))[0]
    for axis, (lo, hi) in enumerate([(0, 12), (12, 22), (22, 32)]):
        pos = [np.array([5])] * 3
        pos[axis] = np.array([9])
        moved = oracle.rope3d(v[None], *pos)[0]
        changed = np.nonzero(np.abs(moved - base) > 1e-12)[0]
        assert changed.min() >= lo and changed.max() < hi


def test_token_positions_enumerate_frames_rows_cols():
    gh, gw, nf, t0 = 3, 4, 2, 7
    exp = [(t0 + f, r, c) for f in range(nf) for r in range(gh) for c in range(gw)]
    t, r, c = oracle.token_positions(nf * gh * gw, t0, gh, gw)
    assert list(zip(t.tolist(), r.tolist(), c.tolist())) == exp


# --------------------------------------------------------------------------
# Append (ordered fp32, bf16 RNE)
# --------------------------------------------------------------------------
def _bits(vals):
    return workload.bf16_bits(np.asarray(vals, dtype=np.float32))


def test_append_sum_order_is_sequential():
    # Terms 2^24, 1, 1, 1, -2^24: a left-to-right fp32 sum gives 0 (each +1 rounds
    # back to 2^24, ties to even); the exact sum is 3.
    a = _bits([1, 1, 1, 1, 1])
    b = _bits([2.0 ** 24, 1, 1, 1, -(2.0 ** 24)])
    assert oracle.ordered_dot(a, b) == 0.0
    # Terms 1, 1, 1, 2^24, -2^24: 3 + 2^24 rounds to 2^24 + 4, so the result is 4.
    b2 = _bits([1, 1, 1, 2.0 ** 24, -(2.0 ** 24)])
    assert oracle.ordered_dot(a, b2) == 4.0


def test_append_content_columns_through_full_path():
    # The content latent of the full append equals the ordered dot of each row.
    rng = np.random.default_rng(4)
    D = 64
    x = _bits(rng.standard_normal((1, 5, D)))
    wd = _bits(rng.standard_normal((6, D)) / 8)
    wk = _bits(rng.standard_normal((32, D)) / 8)
    _, out32 = oracle.cache_append(x, wd, wk, t0=3, grid_h=2, grid_w=3, want_fp32=True)
    for n in range(5):
        for j in range(6):
            assert out32[0, n, j] == np.float32(oracle.ordered_dot(x[0, n], wd[j]))


def test_append_error_bound_vs_fp64():
    rng = np.random.default_rng(5)
    D = 1536
    x = _bits(rng.standard_normal((1, 40, D)))
    wd = _bits(rng.standard_normal((192, D)) / math.sqrt(D))
    wk = _bits(rng.standard_normal((32, D)) / math.sqrt(D))
    bits, out32 = oracle.cache_append(x, wd, wk, t0=11, grid_h=4, grid_w=5, want_fp32=True)
    xd, wdd, wkd = oracle.decode_bf16(x[0]), oracle.decode_bf16(wd), oracle.decode_bf16(wk)
    u = 2.0 ** -24
    gam = D * u / (1 - D * u)
    exact_c = xd @ wdd.T
    bound_c = gam * (np.abs(xd) @ np.abs(wdd).T)
    assert np.all(np.abs(out32[0, :, :192] - exact_c) <= bound_c)
    # rope columns: fp64 rotation of the exact projection, within the summation bound
    # plus a few fp32 roundings of the rotation.
    t, r, c = oracle.token_positions(40, 11, 4, 5)
    exact_r = oracle.rope3d(xd @ wkd.T, t, r, c)
    mag = np.abs(xd) @ np.abs(wkd).T
    bound_r = 2 * gam * mag.max(axis=1, keepdims=True) + 8 * u * mag.max(axis=1, keepdims=True)
    assert np.all(np.abs(out32[0, :, 192:] - exact_r) <= bound_r)
    # final bits are the bf16 rounding of the fp32 values
    assert np.array_equal(bits, oracle.round_bf16(out32))


def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(6)
    v = rng.standard_normal(100000).astype(np.float32) * np.float32(37.0)
    # add exact ties: bf16 value + half an ulp, and values whose low 16 bits are 0x8000
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, -ties])
    ours = oracle.round_bf16(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_append_cos_sin_are_correctly_rounded():
    mpmath.mp.prec = 120
    rng = np.random.default_rng(7)
    for _ in range(300):
        pair = int(rng.integers(0, 16))
        t, r, c = (int(x) for x in rng.integers(0, 4000, size=3))
        cs, sn = oracle.append_cos_sin(pair, t, r, c)
        axis, _ = oracle.rope_pair_axes()[pair]
        d_a = (12, 10, 10)[axis]
        i = pair - (0, 6, 11)[axis]
        pos = (t, r, c)[axis]
        ang = mpmath.mpf(pos) * mpmath.power(10000, mpmath.mpf(-2 * i) / d_a)
        assert cs == np.float32(float(mpmath.cos(ang)))
        assert sn == np.float32(float(mpmath.sin(ang)))


def test_append_rope_uses_chunk_positions():
    rng = np.random.default_rng(8)
    D = 32
    gh, gw, t0 = 3, 5, 42
    n = 2 * gh * gw
    x = _bits(rng.standard_normal((1, n, D)))
    wd = _bits(rng.standard_normal((4, D)) / 4)
    wk = _bits(rng.standard_normal((32, D)) / 4)
    _, out32 = oracle.cache_append(x, wd, wk, t0=t0, grid_h=gh, grid_w=gw, want_fp32=True)
    pre = oracle.decode_bf16(x[0]) @ oracle.decode_bf16(wk).T
    for tok in range(n):
        f, rem = divmod(tok, gh * gw)
        rr, cc = divmod(rem, gw)
        ref = _complex_rope(pre[tok], t0 + f, rr, cc)
        np.testing.assert_allclose(out32[0, tok, 4:], ref, rtol=0, atol=2e-5)


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------
def _tiny_case(rng, B=1, Nq=6, n_kv=9, H=2, dh=8, d_c=12, cap=None, gh=2, gw=3):
    cap = cap or n_kv + 3
    q = _bits(rng.standard_normal((B, Nq, H, dh)))
    qr = _bits(rng.standard_normal((B, Nq, H, 32)))
    wuk = _bits(rng.standard_normal((H * dh, d_c)) / math.sqrt(d_c))
    wuv = _bits(rng.standard_normal((H * dh, d_c)) / math.sqrt(d_c))
    cache = _bits(rng.standard_normal((B, cap, d_c + 32)))
    return q, qr, wuk, wuv, cache


def test_attention_bruteforce_tiny():
    rng = np.random.default_rng(9)
    B, Nq, n_kv, H, dh, d_c, gh, gw, t0 = 1, 6, 9, 2, 8, 12, 2, 3, 4
    q, qr, wuk, wuv, cache = _tiny_case(rng, B, Nq, n_kv, H, dh, d_c, gh=gh, gw=gw)
    scale = 0.37
    got = oracle.chunk_attention(q, qr, wuk, wuv, cache, n_kv, t0, gh, gw, scale)
    Q, QR, WK, WV, C = (oracle.decode_bf16(a) for a in (q, qr, wuk, wuv, cache))
    for h in range(H):
        for i in range(Nq):
            f, rem = divmod(i, gh * gw)
            rq = _complex_rope(QR[0, i, h], t0 + f, rem // gw, rem % gw)
            s = []
            for j in range(n_kv):
                acc = 0.0
                for d in range(dh):
                    k_hd = sum(C[0, j, l] * WK[h * dh + d, l] for l in range(d_c))
                    acc += Q[0, i, h, d] * k_hd
                for e in range(32):
                    acc += rq[e] * C[0, j, d_c + e]
                s.append(scale * acc)
            m = max(s)
            w = [math.exp(x - m) for x in s]
            tot = sum(w)
            for e in range(dh):
                ref = sum(w[j] / tot * sum(C[0, j, l] * WV[h * dh + e, l] for l in range(d_c))
                          for j in range(n_kv))
                assert got[0, i, h, e] == pytest.approx(ref, rel=1e-10, abs=1e-12)


def test_absorbed_equals_nonabsorbed():
    rng = np.random.default_rng(10)
    w = workload.CONFIGS["tiny"].with_(heads=3)
    q, qr, wuk, wuv, cache = _tiny_case(rng, B=2, Nq=w.n_q, n_kv=w.n_kv, H=3, dh=128, d_c=192,
                                        gh=w.grid_h, gw=w.grid_w)
    a = oracle.chunk_attention(q, qr, wuk, wuv, cache, w.n_kv, 6, 8, 8, 160 ** -0.5)
    b = oracle.chunk_attention_absorbed(q, qr, wuk, wuv, cache, w.n_kv, 6, 8, 8, 160 ** -0.5)
    assert np.linalg.norm(a - b) <= 1e-12 * np.linalg.norm(a)


def test_materialized_kv_reproduces_attention():
    # softmax over [K_h ; k_r] with the materialised K_h, V_h (torch SDPA, fp64) equals
    # the absorbed formulation -- pins materialized_kv's head layout and transposes.
    rng = np.random.default_rng(19)
    B, Nq, n_kv, H, d_c, gh, gw, t0 = 2, 12, 30, 3, 20, 2, 3, 5
    q, qr, wuk, wuv, cache = _tiny_case(rng, B, Nq, n_kv, H, 128, d_c, cap=33, gh=gh, gw=gw)
    kv = oracle.materialized_kv(wuk, wuv, cache, n_kv)
    assert kv.shape == (B, n_kv, 2 * H, 128)
    ref = oracle.chunk_attention_absorbed(q, qr, wuk, wuv, cache, n_kv, t0, gh, gw, 0.3)
    Q, QR, C = (torch.from_numpy(oracle.decode_bf16(a)) for a in (q, qr, cache))
    t, r, c = oracle.token_positions(Nq, t0, gh, gw)
    for h in range(H):
        qrot = torch.from_numpy(oracle.rope3d(QR[:, :, h].numpy(), t, r, c))
        Qh = torch.cat([Q[:, :, h], qrot], dim=-1)
        Kh = torch.cat([torch.from_numpy(kv[:, :, h]), C[:, :n_kv, d_c:]], dim=-1)
        Vh = torch.from_numpy(kv[:, :, H + h])
        got = torch.nn.functional.scaled_dot_product_attention(Qh, Kh, Vh, scale=0.3)
        np.testing.assert_allclose(got.numpy(), ref[:, :, h], rtol=1e-11, atol=1e-12)


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(11)
    B, Nq, n_kv, H, dh, d_c, gh, gw, t0 = 2, 24, 40, 3, 16, 24, 2, 4, 9
    q, qr, wuk, wuv, cache = _tiny_case(rng, B, Nq, n_kv, H, dh, d_c, cap=50, gh=gh, gw=gw)
    scale = 0.21
    got = oracle.chunk_attention(q, qr, wuk, wuv, cache, n_kv, t0, gh, gw, scale, row_block=7)
    Q, QR, WK, WV, C = (torch.from_numpy(oracle.decode_bf16(a)) for a in (q, qr, wuk, wuv, cache))
    qrot = torch.empty_like(QR)
    for b in range(B):
        for i in range(Nq):
            f, rem = divmod(i, gh * gw)
            for h in range(H):
                qrot[b, i, h] = torch.from_numpy(_complex_rope(QR[b, i, h].numpy(), t0 + f,
                                                               rem // gw, rem % gw))
    Cc = C[:, :n_kv, :d_c]
    kr = C[:, :n_kv, d_c:]
    for h in range(H):
        Kh = torch.cat([torch.einsum("bjl,dl->bjd", Cc, WK[h * dh:(h + 1) * dh]), kr], dim=-1)
        Vh = torch.einsum("bjl,el->bje", Cc, WV[h * dh:(h + 1) * dh])
        Qh = torch.cat([Q[:, :, h], qrot[:, :, h]], dim=-1)
        ref = torch.nn.functional.scaled_dot_product_attention(Qh, Kh, Vh, scale=scale)
        np.testing.assert_allclose(got[:, :, h], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_attention_closed_forms():
    rng = np.random.default_rng(12)
    H, dh, d_c = 2, 8, 12
    q, qr, wuk, wuv, cache = _tiny_case(rng, 1, 6, 9, H, dh, d_c)
    WV = oracle.decode_bf16(wuv)
    C = oracle.decode_bf16(cache)
    # a single key: every query returns V of that key
    out = oracle.chunk_attention(q, qr, wuk, wuv, cache, 1, 0, 2, 3, 0.5)
    for h in range(H):
        ref = WV[h * dh:(h + 1) * dh] @ C[0, 0, :d_c]
        np.testing.assert_allclose(out[0, :, h], np.broadcast_to(ref, (6, dh)), rtol=1e-13, atol=1e-14)
    # identical keys: V of that key whatever the scores
    same = np.repeat(cache[:, 3:4], cache.shape[1], axis=1)
    out = oracle.chunk_attention(q * 0 + q, qr, wuk, wuv, same, 9, 0, 2, 3, 3.0)
    for h in range(H):
        ref = WV[h * dh:(h + 1) * dh] @ C[0, 3, :d_c]
        np.testing.assert_allclose(out[0, :, h], np.broadcast_to(ref, (6, dh)), rtol=1e-12, atol=1e-13)
    # zero queries: uniform weights -> mean of V over the keys
    zq, zqr = np.zeros_like(q), np.zeros_like(qr)
    out = oracle.chunk_attention(zq, zqr, wuk, wuv, cache, 9, 0, 2, 3, 1.0)
    for h in range(H):
        ref = WV[h * dh:(h + 1) * dh] @ C[0, :9, :d_c].mean(axis=0)
        np.testing.assert_allclose(out[0, :, h], np.broadcast_to(ref, (6, dh)), rtol=1e-12, atol=1e-13)


def test_attention_key_permutation_and_padding():
    rng = np.random.default_rng(13)
    q, qr, wuk, wuv, cache = _tiny_case(rng, 1, 6, 9, 2, 8, 12, cap=14)
    a = oracle.chunk_attention(q, qr, wuk, wuv, cache, 9, 1, 2, 3, 0.4)
    perm = cache.copy()
    perm[0, :9] = cache[0, rng.permutation(9)]
    perm[0, 9:] = _bits(rng.standard_normal((5, perm.shape[2])) * 100)  # slots past n_kv ignored
    b = oracle.chunk_attention(q, qr, wuk, wuv, perm, 9, 1, 2, 3, 0.4)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_attention_row_selection_matches_full():
    rng = np.random.default_rng(14)
    q, qr, wuk, wuv, cache = _tiny_case(rng, 2, 12, 20, 2, 8, 12, gh=2, gw=3)
    full = oracle.chunk_attention(q, qr, wuk, wuv, cache, 20, 5, 2, 3, 0.3)
    rows = np.array([11, 0, 7])
    part = oracle.chunk_attention(q, qr, wuk, wuv, cache, 20, 5, 2, 3, 0.3, rows=rows)
    np.testing.assert_array_equal(part, full[:, rows])


def test_dense_matches_torch_sdpa():
    rng = np.random.default_rng(15)
    B, Nq, Nk, H, d = 2, 17, 33, 3, 16
    q = _bits(rng.standard_normal((B, Nq, H, d)))
    k = _bits(rng.standard_normal((B, Nk, H, d)))
    v = _bits(rng.standard_normal((B, Nk, H, d)))
    got = oracle.dense_attention(q, k, v, 0.25, row_block=5)
    Q, K, V = (torch.from_numpy(oracle.decode_bf16(a)).transpose(1, 2) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=0.25).transpose(1, 2)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the checks above
# --------------------------------------------------------------------------
def _rope_sign_flipped(v, t, r, c):
    out = oracle.rope3d(v, -np.asarray(t), -np.asarray(r), -np.asarray(c))
    return out


def test_linear_hand_example_and_orientation():
    # A non-square weight [out=3, in=5]: a transposed operand cannot even produce [2, 3].
    x = np.array([[1, 2, 0, 0, 0], [0, 0, 0, 0, 1]], dtype=np.float32)
    W = np.array([[1, 0, 0, 0, 0], [0, 1, 0, 0, 0], [0, 0, 0, 0, 2]], dtype=np.float32)
    y = oracle.linear(workload.bf16_bits(x), workload.bf16_bits(W))
    assert y.shape == (2, 3)
    assert np.array_equal(y, np.array([[1.0, 2.0, 0.0], [0.0, 0.0, 2.0]]))


def test_linear_identity_and_bruteforce():
    rng = np.random.default_rng(21)
    xb = workload.bf16_bits(rng.standard_normal((4, 6)).astype(np.float32))
    eye = workload.bf16_bits(np.eye(6, dtype=np.float32))
    assert np.array_equal(oracle.linear(xb, eye), oracle.decode_bf16(xb))
    wb = workload.bf16_bits(rng.standard_normal((7, 6)).astype(np.float32))
    xs, ws = workload.bf16_to_f32(xb).tolist(), workload.bf16_to_f32(wb).tolist()
    y = oracle.linear(xb, wb)
    for i in range(4):
        for o in range(7):
            exact = math.fsum(xs[i][k] * ws[o][k] for k in range(6))
            assert abs(y[i, o] - exact) <= 1e-14 * (1 + abs(exact))


def test_linear_batched_leading_dims():
    # [B, n, D] inputs keep their leading dims; each token is projected on its own.
    rng = np.random.default_rng(22)
    xb = workload.bf16_bits(rng.standard_normal((2, 3, 8)).astype(np.float32))
    wb = workload.bf16_bits(rng.standard_normal((5, 8)).astype(np.float32))
    y = oracle.linear(xb, wb)
    assert y.shape == (2, 3, 5)
    for b in range(2):
        np.testing.assert_array_equal(y[b, 1], oracle.linear(xb[b, 1:2], wb)[0])


def test_planted_rope_sign_error_is_caught():
    rng = np.random.default_rng(16)
    v = rng.standard_normal(32)
    bad = _rope_sign_flipped(v[None], np.array([3]), np.array([2]), np.array([1]))[0]
    # norm and relative-offset invariants still hold for the flipped rotation,
    # but the complex-number statement does not:
    assert np.abs(bad - _complex_rope(v, 3, 2, 1)).max() > 1e-3


def test_planted_transposed_w_uk_is_caught():
    rng = np.random.default_rng(17)
    H, dh, d_c = 1, 12, 12  # square per-head block so the transposed use still type-checks
    q, qr, wuk, wuv, cache = _tiny_case(rng, 1, 6, 9, H, dh, d_c)
    wuk_t = oracle.decode_bf16(wuk).T.copy()
    good = oracle.chunk_attention(q, qr, wuk, wuv, cache, 9, 0, 2, 3, 0.5)
    bad = oracle.chunk_attention(q, qr, workload.bf16_bits(wuk_t.astype(np.float32)), wuv, cache,
                                 9, 0, 2, 3, 0.5)
    absorbed = oracle.chunk_attention_absorbed(q, qr, wuk, wuv, cache, 9, 0, 2, 3, 0.5)
    np.testing.assert_allclose(good, absorbed, rtol=1e-12, atol=1e-14)
    assert np.abs(bad - absorbed).max() > 1e-4


def test_planted_dropped_rope_term_is_caught():
    rng = np.random.default_rng(18)
    q, qr, wuk, wuv, cache = _tiny_case(rng, 1, 6, 9, 2, 8, 12)
    good = oracle.chunk_attention(q, qr, wuk, wuv, cache, 9, 0, 2, 3, 0.5)
    no_rope = oracle.chunk_attention(q, np.zeros_like(qr), wuk, wuv, cache, 9, 0, 2, 3, 0.5)
    assert np.abs(good - no_rope).max() > 1e-4


def test_input_generator_bf16_rounding_and_streams():
    # The seeded input generator (shared by the oracle and the GPU path) rounds to
    # bf16 like torch's cast, decodes exactly, and gives each named tensor its own
    # reproducible stream.
    rng = np.random.default_rng(7)
    v = rng.standard_normal(50000).astype(np.float32) * np.float32(11.0)
    ties = (np.arange(1, 1000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, -ties])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(workload.bf16_bits(v), ref)
    assert np.array_equal(workload.bf16_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16)
                          .float().numpy())
    a = workload.normal_bf16(5, (0, 1), (64, 8))
    assert np.array_equal(a, workload.normal_bf16(5, (0, 1), (64, 8)))
    assert not np.array_equal(a, workload.normal_bf16(5, (0, 2), (64, 8)))
    assert not np.array_equal(a, workload.normal_bf16(6, (0, 1), (64, 8)))
    f = workload.bf16_to_f32(workload.normal_bf16(3, (9,), (200000,), std=0.25)).astype(np.float64)
    assert abs(f.mean()) < 0.01 and abs(f.std() - 0.25) < 0.005
