"""vmla_chunk_attention_nonabsorbed_noalloc: the allocation-free entry point.

For callers that cannot allocate device memory (a host program that only holds
tensors handed to it, a framework whose allocator owns the device budget, a loop
that cannot take cudaMalloc's device-wide synchronisation), the library keeps an
8 MiB scratch of its own.  These tests call the new entry point through the C ABI
(raw device pointers) and compare it with vmla_chunk_attention_nonabsorbed fed an
explicit workspace, and with the fp64 oracle, for two calls in a row with
different inputs, within the tolerance used throughout (relative L2 <= 1e-2,
max-abs <= 3e-2).  They also check that the calls leave the device's free memory
and torch's allocator untouched.  This file is collected last so that a run
stopping at its first failure has run everything else.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

import oracle
import workload
from helpers import SCALE, assert_close, gpu_fill_window, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


def _inputs(vm, w, layer):
    import torch
    wts = workload.layer_weights(w, layer)
    act = workload.batch_activations(w, layer)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    dev = (to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache)
    # The oracle forms its own cache from the same tokens (no input taken from the GPU).
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE)
    return dev, ref


def _noalloc_call(vm, w, q, qr, wuk, wuv, cache, out):
    P = ctypes.c_void_p
    return vm.lib.vmla_chunk_attention_nonabsorbed_noalloc(
        P(q.data_ptr()), P(qr.data_ptr()), P(wuk.data_ptr()), P(wuv.data_ptr()), P(cache.data_ptr()),
        w.batch, w.n_q, w.heads, cache.shape[1], w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, ctypes.c_float(SCALE),
        P(out.data_ptr()), P(0))


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_noalloc_matches_workspace_form_two_calls(vm, name):
    import torch
    w = workload.CONFIGS["tiny"]
    if name == "ragged":
        w = w.with_(grid_h=7, grid_w=9, cached_frames=4, heads=3)
    need = vm.vmla_materialized_kv_bytes(w.batch, w.heads, w.n_kv)
    assert 0 < need <= vm.NOALLOC_SCRATCH_BYTES
    ws = torch.empty(need // 2, dtype=torch.bfloat16, device="cuda")
    for layer in (0, 5):  # two calls in a row, different inputs: nothing stale may leak through
        (q, qr, wuk, wuv, cache), oracle_out = _inputs(vm, w, layer)
        out = torch.full((w.batch, w.n_q, w.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        ref = torch.empty_like(out)
        assert _noalloc_call(vm, w, q, qr, wuk, wuv, cache, out) == vm.VMLA_OK, vm.vmla_last_error()
        vm.vmla_chunk_attention_nonabsorbed(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                            ws, ref)
        vm.vmla_get_device_status()
        assert_close(to_f64(out), to_f64(ref), f"noalloc {name} layer {layer} vs workspace form")
        assert_close(to_f64(out), oracle_out, f"noalloc {name} layer {layer} vs oracle")


def test_noalloc_leaves_device_memory_unchanged(vm):
    """Once the library's kernels are loaded on the device (any first launch may
    make the driver load them), further calls change neither the device's free
    memory nor what torch's allocator holds."""
    import torch
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3)
    (q, qr, wuk, wuv, cache), oracle_out = _inputs(vm, w, 2)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    assert _noalloc_call(vm, w, q, qr, wuk, wuv, cache, out) == vm.VMLA_OK, vm.vmla_last_error()
    vm.vmla_get_device_status()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for _ in range(2):
        out.fill_(float("nan"))
        assert _noalloc_call(vm, w, q, qr, wuk, wuv, cache, out) == vm.VMLA_OK, vm.vmla_last_error()
        vm.vmla_get_device_status()
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0, f"device free memory changed by {free0 - free1} bytes across a call"
        assert torch.cuda.memory_allocated() == alloc0 and torch.cuda.memory_reserved() == reserved0
        assert_close(to_f64(out), oracle_out, "noalloc, repeated call vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch(vm):
    import torch
    w = workload.CONFIGS["480p"]  # 32760 keys x 12 heads: ~201 MB of keys/values
    assert vm.vmla_materialized_kv_bytes(w.batch, w.heads, w.n_kv) > vm.NOALLOC_SCRATCH_BYTES
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")  # never read: the call is refused first
    P = ctypes.c_void_p
    rc = vm.lib.vmla_chunk_attention_nonabsorbed_noalloc(
        P(t.data_ptr()), P(t.data_ptr()), P(t.data_ptr()), P(t.data_ptr()), P(t.data_ptr()), w.batch, w.n_q,
        w.heads, w.n_kv, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, ctypes.c_float(SCALE), P(t.data_ptr()), P(0))
    assert rc == vm.VMLA_ERR_UNSUPPORTED
    assert "scratch" in vm.vmla_last_error()
    vm.vmla_get_device_status()
