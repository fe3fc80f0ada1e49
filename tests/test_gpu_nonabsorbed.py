"""Non-absorbed latent attention on the GPU: materialised per-head keys/values
(vmla_materialize_kv) against the oracle's definition, and attention over them
(vmla_chunk_attention_materialized / _nonabsorbed) against the fp64 oracle.
Tolerance: relative L2 <= 1e-2, max-abs <= 3e-2."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workload
from helpers import SCALE, assert_close, gpu_fill_window, sample_rows, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


def _setup(vm, w, cap_extra=0):
    import torch
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = torch.zeros(w.batch, w.n_kv + cap_extra, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    return wts, act, cache, ref_cache


def test_materialize_kv_matches_definition(vm):
    import torch
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3)
    wts, act, cache, ref_cache = _setup(vm, w, cap_extra=5)
    kv = torch.empty(w.batch, w.n_kv, 2 * w.heads, 128, dtype=torch.bfloat16, device="cuda")
    assert vm.vmla_materialized_kv_bytes(w.batch, w.heads, w.n_kv) == kv.numel() * 2
    vm.vmla_materialize_kv(to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, w.n_kv, kv)
    vm.vmla_get_device_status()
    ref = oracle.materialized_kv(wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv)
    got = to_f64(kv)
    # bf16 output of an fp32-accumulated product: within one bf16 rounding of the exact value
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3)


@pytest.mark.parametrize("name", ["tiny", "ragged", "ragged_batch"])
def test_materialized_attention_full(vm, name):
    import torch
    w = workload.CONFIGS["tiny"]
    if name == "ragged":
        w = w.with_(grid_h=7, grid_w=9, cached_frames=4, heads=3)
    if name == "ragged_batch":
        w = w.with_(grid_h=7, grid_w=9, cached_frames=4, heads=3, batch=3, seed=93)
    wts, act, cache, ref_cache = _setup(vm, w, cap_extra=3)
    kv = torch.empty(w.batch, w.n_kv, 2 * w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_materialize_kv(to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, w.n_kv, kv)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention_materialized(to_dev(act["q"]), to_dev(act["q_rope"]), kv, cache, w.n_kv, w.chunk_t0,
                                         w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE)
    assert_close(to_f64(out), ref, f"materialized {name}")


def test_nonabsorbed_480p_sampled_and_workspace(vm):
    import torch
    w = workload.CONFIGS["480p"]
    wts, act, cache, ref_cache = _setup(vm, w)
    need = vm.vmla_materialized_kv_bytes(w.batch, w.heads, w.n_kv)
    ws = torch.empty(need // 2, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    q, qr, wuk, wuv = to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]), to_dev(wts["w_uv"])
    vm.vmla_chunk_attention_nonabsorbed(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                        ws, out)
    vm.vmla_get_device_status()
    rows = sample_rows(w.n_q, 128, seed=11)
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE, rows=rows)
    assert_close(to_f64(out)[:, rows], ref, "nonabsorbed 480p")
    # the absorbed kernel agrees with it on the same rows
    out2 = torch.empty_like(out)
    vm.vmla_chunk_attention(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out2)
    vm.vmla_get_device_status()
    assert_close(to_f64(out2)[:, rows], ref, "absorbed 480p")
    # a workspace one byte too small is rejected before anything runs
    small = ws[: need // 2 - 8]
    with pytest.raises(vm.VmlaError) as ei:
        vm.vmla_chunk_attention_nonabsorbed(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                            small, out)
    assert ei.value.code == vm.VMLA_ERR_INVALID_ARG


def test_materialized_attention_b8_sampled(vm):
    import torch
    w = workload.CONFIGS["480p_b8"]
    wts, act, cache, ref_cache = _setup(vm, w)
    kv = torch.empty(w.batch, w.n_kv, 2 * w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_materialize_kv(to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, w.n_kv, kv)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention_materialized(to_dev(act["q"]), to_dev(act["q_rope"]), kv, cache, w.n_kv, w.chunk_t0,
                                         w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    rows = sample_rows(w.n_q, 32, seed=12)
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE, rows=rows)
    got = to_f64(out)[:, rows]
    for b in range(w.batch):
        assert_close(got[b], ref[b], f"materialized b8 sample {b}")


def test_materialize_kv_many_heads_per_cta(vm):
    """Batch 40 of a 144-key window (two key tiles, the second ragged) x 12 heads:
    960 work items over at most one CTA per SM, so each persistent CTA crosses
    several (sample, head) boundaries and reloads W_UK_h / W_UV_h each time."""
    import torch
    w = workload.CONFIGS["tiny"].with_(batch=40, grid_h=4, grid_w=4, seed=123)
    assert w.n_kv == 144
    wts, act, cache, ref_cache = _setup(vm, w, cap_extra=5)
    kv = torch.full((w.batch, w.n_kv, 2 * w.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_materialize_kv(to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, w.n_kv, kv)
    vm.vmla_get_device_status()
    ref = oracle.materialized_kv(wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv)
    got = to_f64(kv)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3)


def test_nonabsorbed_1080p_sampled(vm):
    import torch
    w = workload.CONFIGS["1080p"]
    wts, act, cache, ref_cache = _setup(vm, w)
    kv = torch.empty(w.batch, w.n_kv, 2 * w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_materialize_kv(to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, w.n_kv, kv)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention_materialized(to_dev(act["q"]), to_dev(act["q_rope"]), kv, cache, w.n_kv, w.chunk_t0,
                                         w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    rows = sample_rows(w.n_q, 24, seed=13)
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE, rows=rows)
    assert_close(to_f64(out)[:, rows], ref, "nonabsorbed 1080p")


@pytest.mark.parametrize("name", ["tiny", "480p"])
def test_dense_on_materialised_latent_equals_latent_attention(vm, name):
    """Cross-check of the two layouts: with zero rope queries, the latent attention
    over the cache equals dense per-head attention over the keys c.W_UK_h^T and
    values c.W_UV_h^T that k_materialize_kv writes from the same cache."""
    import torch
    w = workload.CONFIGS[name]
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    q = to_dev(act["q"])
    qr0 = torch.zeros(w.batch, w.n_q, w.heads, 32, dtype=torch.bfloat16, device="cuda")
    wuk, wuv = to_dev(wts["w_uk"]), to_dev(wts["w_uv"])
    out_l = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention(q, qr0, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out_l)
    kv = torch.empty(w.batch, w.n_kv, 2 * w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_materialize_kv(wuk, wuv, cache, w.n_kv, kv)
    k = kv[:, :, :w.heads].contiguous()
    v = kv[:, :, w.heads:].contiguous()
    out_d = torch.empty_like(out_l)
    vm.vmla_dense_attention(q, k, v, SCALE, out_d)
    vm.vmla_get_device_status()
    assert_close(to_f64(out_l), to_f64(out_d), f"{name}: latent vs dense on materialised K/V")
