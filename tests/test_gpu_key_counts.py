"""The per-head kernels (dense baseline and materialised keys/values) over key
counts that exercise how they share key tiles between their two softmax
warpgroups: one tile only (the second warpgroup has none), one key in the second
tile, odd and even tile counts, ragged last tiles.  Every output is compared with
the fp64 oracle at the stated tolerance (relative L2 <= 1e-2, max-abs <= 3e-2)."""
from __future__ import annotations

import pytest

import oracle
import workload
from helpers import SCALE, assert_close, gpu_fill_window, to_dev, to_f64

pytestmark = pytest.mark.gpu

KEY_COUNTS = [1, 77, 128, 129, 256, 300, 383, 512]


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


@pytest.mark.parametrize("n_kv", KEY_COUNTS)
def test_dense_key_counts(vm, n_kv):
    import torch
    w = workload.CONFIGS["tiny"].with_(heads=3)
    act = workload.batch_activations(w)
    kv = workload.batch_dense_kv(w)
    k, v = kv["k"][:, :n_kv].copy(), kv["v"][:, :n_kv].copy()
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_dense_attention(to_dev(act["q"]), to_dev(k), to_dev(v), SCALE, out)
    vm.vmla_get_device_status()
    assert_close(to_f64(out), oracle.dense_attention(act["q"], k, v, SCALE), f"dense n_kv={n_kv}")


@pytest.mark.parametrize("n_kv", KEY_COUNTS)
def test_materialized_key_counts(vm, n_kv):
    import torch
    w = workload.CONFIGS["tiny"].with_(heads=3)
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    kvm = torch.empty(w.batch, n_kv, 2 * w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_materialize_kv(to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache, n_kv, kvm)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention_materialized(to_dev(act["q"]), to_dev(act["q_rope"]), kvm, cache, n_kv, w.chunk_t0,
                                         w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE)
    assert_close(to_f64(out), ref, f"materialized n_kv={n_kv}")


@pytest.mark.parametrize("d_c", [64, 128, 192])
@pytest.mark.parametrize("n_kv", [1, 128, 129, 383, 512])
def test_latent_key_counts(vm, d_c, n_kv):
    # d_c <= 128 runs the two-slot latent kernel, 192 the column-split one
    import torch
    w = workload.CONFIGS["tiny"].with_(heads=3, d_c=d_c)
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = torch.zeros(w.batch, w.n_kv, d_c + 32, dtype=torch.bfloat16, device="cuda")
    per = w.tokens_per_frame
    for f0 in range(0, w.window_frames, w.chunk_frames):
        nf = min(w.chunk_frames, w.window_frames - f0)
        vm.vmla_cache_append_dc(to_dev(act["x"][:, f0 * per:(f0 + nf) * per].copy()), to_dev(wts["w_dkv"]),
                                to_dev(wts["w_kr"]), cache, f0 * per, f0, w.grid_h, w.grid_w)
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    out = torch.full((w.batch, w.n_q, w.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention_dc(to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]), to_dev(wts["w_uv"]),
                               cache, n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE)
    assert_close(to_f64(out), ref, f"latent d_c={d_c} n_kv={n_kv}")
