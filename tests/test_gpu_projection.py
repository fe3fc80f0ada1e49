"""vmla_query_projection and vmla_output_projection on the GPU against the fp64 oracle.

Each output element is one fp32-accumulated dot product rounded once to bf16, so
the element-wise bound is the bf16 rounding (half an ulp, at most 2^-8 of the
value) plus an accumulation allowance of 2e-3 (fp32 sums of <= 1536 products of
N(0,1)-scaled terms stay far below it).  The global relative-L2 bound used
elsewhere (1e-2) is checked as well.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workload
from helpers import assert_close, sample_rows, to_dev, to_f64

pytestmark = pytest.mark.gpu

ACC_ALLOW = 2e-3


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


def _check(got, ref, what):
    bound = 2.0 ** -8 * np.abs(ref) + ACC_ALLOW
    worst = float(np.max(np.abs(got - ref) - bound))
    assert worst <= 0, f"{what}: element-wise bound exceeded by {worst:.3e}"
    assert_close(got, ref, what)


def _qproj(vm, w, rows=None):
    import torch
    iw = workload.io_weights(w)
    x = workload.batch_activations(w)["x"][:, -w.n_q:]  # the current chunk's hidden states
    q = torch.full((w.batch, w.n_q, w.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    qr = torch.full((w.batch, w.n_q, w.heads, 32), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_query_projection(to_dev(x), to_dev(iw["w_q"]), to_dev(iw["w_qr"]), q, qr)
    vm.vmla_get_device_status()
    gq, gr = to_f64(q), to_f64(qr)
    if rows is not None:
        x, gq, gr = x[:, rows], gq[:, rows], gr[:, rows]
    rq = oracle.linear(x, iw["w_q"]).reshape(gq.shape)
    rr = oracle.linear(x, iw["w_qr"]).reshape(gr.shape)
    _check(gq, rq, f"{w.name} q")
    _check(gr, rr, f"{w.name} q_rope")


def _oproj(vm, w, rows=None):
    import torch
    iw = workload.io_weights(w)
    o = workload.head_outputs(w)
    y = torch.full((w.batch, w.n_q, w.d_model), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_output_projection(to_dev(o), to_dev(iw["w_o"]), y)
    vm.vmla_get_device_status()
    gy = to_f64(y)
    if rows is not None:
        o, gy = o[:, rows], gy[:, rows]
    ref = oracle.linear(o.reshape(o.shape[0], o.shape[1], -1), iw["w_o"])
    _check(gy, ref, f"{w.name} y")


def test_query_projection_tiny(vm):
    _qproj(vm, workload.CONFIGS["tiny"])


def test_query_projection_ragged(vm):
    # 189 tokens (one full M tile + a ragged one); d_model 320 (5 k-blocks); 3 heads:
    # N = 384 + 96, so the second N tile holds the last content half and a part-filled
    # rope half.
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, heads=3, d_model=320)
    _qproj(vm, w)


@pytest.mark.parametrize("heads", [5, 7])
def test_query_projection_narrow_last_column(vm, heads):
    # N = 160 * heads = 800 or 1120: the last 256-column tile holds 32 or 96
    # columns, all of the rope half, and runs narrower MMAs (each CTA of the pair
    # stages 16 or 48 B rows; 1 or 3 column groups of 32).
    w = workload.CONFIGS["tiny"].with_(grid_h=10, grid_w=20, heads=heads, d_model=256)
    _qproj(vm, w)


def test_query_projection_480p_full(vm):
    _qproj(vm, workload.CONFIGS["480p"])


def test_query_projection_480p_b8_sampled(vm):
    w = workload.CONFIGS["480p_b8"]
    _qproj(vm, w, rows=sample_rows(w.n_q, 64, seed=3))


def test_output_projection_tiny(vm):
    _oproj(vm, workload.CONFIGS["tiny"])


def test_output_projection_ragged(vm):
    # d_model 384: the second N tile reads past W_O's last row (zero filled) and its
    # upper half is masked; K = 3 heads x 128.
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, heads=3, d_model=384)
    _oproj(vm, w)


def test_output_projection_480p_full(vm):
    _oproj(vm, workload.CONFIGS["480p"])


def test_output_projection_1080p_sampled(vm):
    w = workload.CONFIGS["1080p"]
    _oproj(vm, w, rows=sample_rows(w.n_q, 64, seed=4))


def test_layer_chain_480p_sampled(vm):
    """x -> (q, q_r) -> latent chunk attention -> W_O, all on the GPU, against the
    oracle's own chain on sampled query rows (every key, every head)."""
    import torch
    from helpers import SCALE, gpu_fill_window
    w = workload.CONFIGS["480p"]
    wts = workload.layer_weights(w)
    iw = workload.io_weights(w)
    x = workload.batch_activations(w)["x"]
    xd = to_dev(x)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, xd, to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    q = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    qr = torch.empty(w.batch, w.n_q, w.heads, 32, dtype=torch.bfloat16, device="cuda")
    vm.vmla_query_projection(xd[:, -w.n_q:].contiguous(), to_dev(iw["w_q"]), to_dev(iw["w_qr"]), q, qr)
    o = torch.empty_like(q)
    vm.vmla_chunk_attention(q, qr, to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, w.n_kv, w.chunk_t0,
                            w.grid_h, w.grid_w, SCALE, o)
    y = torch.empty(w.batch, w.n_q, w.d_model, dtype=torch.bfloat16, device="cuda")
    vm.vmla_output_projection(o, to_dev(iw["w_o"]), y)
    vm.vmla_get_device_status()

    rows = sample_rows(w.n_q, 24, seed=5)
    ref_cache = oracle.cache_append(x, wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    xq = x[:, -w.n_q:]
    # The oracle's chain keeps its own rounding points: q and q_r are rounded to bf16
    # as the GPU stores them, and so is the head output before W_O.
    rq = oracle.round_bf16(oracle.linear(xq, iw["w_q"])).reshape(w.batch, w.n_q, w.heads, 128)
    rr = oracle.round_bf16(oracle.linear(xq, iw["w_qr"])).reshape(w.batch, w.n_q, w.heads, 32)
    ro = oracle.chunk_attention(rq, rr, wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0, w.grid_h,
                                w.grid_w, SCALE, rows=rows)
    ry = oracle.linear(oracle.round_bf16(ro).reshape(w.batch, len(rows), -1), iw["w_o"])
    assert_close(to_f64(y)[:, rows], ry, "480p layer chain")


def test_projections_minimum_shapes(vm):
    """One token, one head, a single 64-wide k block (query side) and d_model 128
    (output side): one M tile, one N tile, a one-block pipeline."""
    import torch
    rng = np.random.default_rng(41)

    def bits(*shape, std=1.0):
        return workload.bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))

    x, wq, wqr = bits(1, 1, 64), bits(128, 64, std=0.125), bits(32, 64, std=0.125)
    q = torch.full((1, 1, 1, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    qr = torch.full((1, 1, 1, 32), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_query_projection(to_dev(x), to_dev(wq), to_dev(wqr), q, qr)
    o, wo = bits(1, 1, 1, 128), bits(128, 128, std=128 ** -0.5)
    y = torch.full((1, 1, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_output_projection(to_dev(o), to_dev(wo), y)
    vm.vmla_get_device_status()
    _check(to_f64(q), oracle.linear(x, wq).reshape(1, 1, 1, 128), "q, one token")
    _check(to_f64(qr), oracle.linear(x, wqr).reshape(1, 1, 1, 32), "q_rope, one token")
    _check(to_f64(y), oracle.linear(o.reshape(1, 1, 128), wo), "y, one token")


@pytest.mark.parametrize("tokens", [257, 272, 296, 356, 384, 385, 4680 + 256])
def test_projections_short_last_tile(vm, tokens):
    """Last M tile of 1, 16, 40, 100, 128, 129 and 72 rows (the pair tile's second
    CTA holding no rows, or only padding, for the shortest); 3 heads (N = 384 + 96,
    a partial last column), d_model 256 (query side) and 384 (output side)."""
    import torch
    rng = np.random.default_rng(tokens)

    def bits(*shape, std=1.0):
        return workload.bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))

    H = 3
    x, wq, wqr = bits(1, tokens, 256), bits(H * 128, 256, std=1 / 16), bits(H * 32, 256, std=1 / 16)
    q = torch.full((1, tokens, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    qr = torch.full((1, tokens, H, 32), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_query_projection(to_dev(x), to_dev(wq), to_dev(wqr), q, qr)
    o, wo = bits(1, tokens, H, 128), bits(384, H * 128, std=(H * 128) ** -0.5)
    y = torch.full((1, tokens, 384), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_output_projection(to_dev(o), to_dev(wo), y)
    vm.vmla_get_device_status()
    _check(to_f64(q), oracle.linear(x, wq).reshape(1, tokens, H, 128), f"q, {tokens} tokens")
    _check(to_f64(qr), oracle.linear(x, wqr).reshape(1, tokens, H, 32), f"q_rope, {tokens} tokens")
    _check(to_f64(y), oracle.linear(o.reshape(1, tokens, H * 128), wo), f"y, {tokens} tokens")
