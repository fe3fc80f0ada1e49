"""The latent-width variants (vmla_cache_append_dc / vmla_chunk_attention_dc) on the GPU.

d_c in {64, 128, 256} against the oracle, which takes d_c from its inputs' shapes:
the append bit-exact, the attention within relative L2 <= 1e-2 and max-abs
<= 3e-2 (full outputs on the tiny and ragged cases, sampled query rows -- all
heads, every key -- at 480P).  d_c = 192 through the _dc entry points must be
bit-identical to vmla_cache_append / vmla_chunk_attention.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workload
from helpers import SCALE, assert_close, sample_rows, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu

DCS = (64, 128, 256)


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


def _fill(vm, w, x_dev, wd, wk, cache):
    """Append the window chunk by chunk, as a rollout would."""
    per = w.tokens_per_frame
    for f0 in range(0, w.window_frames, w.chunk_frames):
        nf = min(w.chunk_frames, w.window_frames - f0)
        vm.vmla_cache_append_dc(x_dev[:, f0 * per:(f0 + nf) * per].contiguous(), wd, wk, cache,
                                (f0 * per) % cache.shape[1], f0, w.grid_h, w.grid_w)


def _case(vm, w, rows=None):
    import torch
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = torch.zeros(w.batch, w.n_kv, w.d_c + 32, dtype=torch.bfloat16, device="cuda")
    _fill(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    out = torch.full((w.batch, w.n_q, w.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention_dc(to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]), to_dev(wts["w_uv"]),
                               cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    got_cache = to_bits(cache)
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv,
                                 w.chunk_t0, w.grid_h, w.grid_w, SCALE, rows=rows)
    got = to_f64(out)
    if rows is not None:
        got = got[:, rows]
    return got_cache, ref_cache, got, ref


@pytest.mark.parametrize("d_c", DCS)
def test_dc_tiny_full(vm, d_c):
    w = workload.CONFIGS["tiny"].with_(d_c=d_c)
    gc, rc, got, ref = _case(vm, w)
    assert np.array_equal(gc, rc), f"d_c={d_c}: append not bit-exact"
    assert_close(got, ref, f"tiny d_c={d_c}")


@pytest.mark.parametrize("d_c", DCS)
def test_dc_ragged(vm, d_c):
    # 7x9 grid: 189-query chunk (a ragged query tile), 4 cached frames -> 441 keys
    # (a ragged key tile), 3 heads.
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3, d_c=d_c, seed=77)
    gc, rc, got, ref = _case(vm, w)
    assert np.array_equal(gc, rc), f"d_c={d_c}: append not bit-exact"
    assert_close(got, ref, f"ragged d_c={d_c}")


@pytest.mark.parametrize("d_c", DCS)
def test_dc_ragged_batch(vm, d_c):
    # three samples with their own seeds and a ragged query and key tile each: the
    # (sample, query tile, head) decode of every latent kernel
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3, d_c=d_c, batch=3, seed=78)
    gc, rc, got, ref = _case(vm, w)
    assert np.array_equal(gc, rc), f"d_c={d_c}: append not bit-exact"
    assert_close(got, ref, f"ragged batch 3 d_c={d_c}")


@pytest.mark.parametrize("d_c", (64, 128))
def test_dc_peaked(vm, d_c):
    # queries and rope queries x4: a peaked softmax that moves the running maximum
    # often, so the two-slot kernel rescales its accumulators and merges slots whose
    # maxima differ
    import torch
    w = workload.CONFIGS["tiny"].with_(heads=3, d_c=d_c, seed=79)
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    q = workload.bf16_bits(workload.bf16_to_f32(act["q"]) * np.float32(4.0))
    qr = workload.bf16_bits(workload.bf16_to_f32(act["q_rope"]) * np.float32(4.0))
    cache = torch.zeros(w.batch, w.n_kv, w.d_c + 32, dtype=torch.bfloat16, device="cuda")
    _fill(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    out = torch.full((w.batch, w.n_q, w.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention_dc(to_dev(q), to_dev(qr), to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, w.n_kv,
                               w.chunk_t0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    ref = oracle.chunk_attention(q, qr, wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0, w.grid_h,
                                 w.grid_w, SCALE)
    assert_close(to_f64(out), ref, f"peaked x4 d_c={d_c}")


@pytest.mark.parametrize("d_c", DCS)
def test_dc_480p_sampled(vm, d_c):
    w = workload.CONFIGS["480p"].with_(d_c=d_c)
    rows = sample_rows(w.n_q, 24, seed=d_c)
    gc, rc, got, ref = _case(vm, w, rows=rows)
    assert np.array_equal(gc, rc), f"d_c={d_c}: append not bit-exact"
    assert_close(got, ref, f"480p d_c={d_c}")


def test_dc_192_is_the_default_call(vm):
    import torch
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, heads=3, seed=5)
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    x, wd, wk = to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"])
    c1 = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    c2 = torch.zeros_like(c1)
    vm.vmla_cache_append(x, wd, wk, c1, 0, 0, w.grid_h, w.grid_w)
    vm.vmla_cache_append_dc(x, wd, wk, c2, 0, 0, w.grid_h, w.grid_w)
    assert torch.equal(c1.view(torch.int16), c2.view(torch.int16))
    q, qr, wuk, wuv = to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]), to_dev(wts["w_uv"])
    o1 = torch.empty_like(q)
    o2 = torch.empty_like(q)
    vm.vmla_chunk_attention(q, qr, wuk, wuv, c1, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, o1)
    vm.vmla_chunk_attention_dc(q, qr, wuk, wuv, c1, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, o2)
    vm.vmla_get_device_status()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
