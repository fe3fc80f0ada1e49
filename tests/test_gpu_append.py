"""vmla_cache_append on the GPU: bit-exact against the ordered-fp32 oracle."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workload
from helpers import gpu_fill_window, to_bits, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


def _window_case(vm, w, slot_base=0, cap_extra=0):
    import torch
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cap = w.n_kv + cap_extra
    cache = torch.zeros(w.batch, cap, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache,
                    slot_base=slot_base)
    vm.vmla_get_device_status()
    got = to_bits(cache)
    ref = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    per_slot = np.zeros_like(got)
    slots = (slot_base + np.arange(w.n_kv)) % cap
    per_slot[:, slots] = ref
    return got, per_slot, slots


@pytest.mark.parametrize("name", ["tiny", "480p", "1080p"])
def test_append_bit_exact_full_window(vm, name):
    w = workload.CONFIGS[name]
    got, ref, slots = _window_case(vm, w)
    assert np.array_equal(got[:, slots], ref[:, slots])


def test_append_bit_exact_batch8(vm):
    w = workload.CONFIGS["480p_b8"]
    got, ref, slots = _window_case(vm, w)
    assert np.array_equal(got[:, slots], ref[:, slots])
    # samples differ from one another (independent seeds)
    assert not np.array_equal(got[0], got[1])


def test_append_ring_wraps_and_leaves_other_slots(vm):
    w = workload.CONFIGS["tiny"]
    got, ref, slots = _window_case(vm, w, slot_base=500, cap_extra=37)
    assert np.array_equal(got[:, slots], ref[:, slots])
    untouched = np.setdiff1d(np.arange(got.shape[1]), slots)
    assert np.all(got[:, untouched] == 0)


def test_append_ragged_and_single_token(vm):
    import torch
    w = workload.CONFIGS["tiny"].with_(grid_h=5, grid_w=7)
    wts = workload.layer_weights(w)
    x = workload.normal_bf16(9, (1,), (2, 33, 1536))
    for n_tok in (1, 33):
        cache = torch.zeros(2, 40, 224, dtype=torch.bfloat16, device="cuda")
        vm.vmla_cache_append(to_dev(x[:, :n_tok]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache,
                             3, 11, 5, 7)
        vm.vmla_get_device_status()
        ref = oracle.cache_append(x[:, :n_tok], wts["w_dkv"], wts["w_kr"], 11, 5, 7)
        got = to_bits(cache)
        assert np.array_equal(got[:, 3:3 + n_tok], ref)
        assert np.all(got[:, :3] == 0) and np.all(got[:, 3 + n_tok:] == 0)


@pytest.mark.parametrize("d_c", [64, 128, 192, 256])
def test_append_many_tiles_ragged(vm, d_c):
    """More 32-token tiles than SMs (300 tiles: the layout with 8 tokens per thread
    runs where two of its CTAs fit on an SM, d_c <= 192), a ragged last tile, a
    ring that wraps, and a first frame t0 > 0."""
    import torch
    w = workload.CONFIGS["480p"].with_(d_c=d_c)
    wts = workload.layer_weights(w)
    batch, n_tok, cap, slot0, t0 = 2, 4790, 4803, 4000, 5
    x = workload.normal_bf16(w.seed + 101, (3,), (batch, n_tok, w.d_model))
    cache = torch.zeros(batch, cap, d_c + 32, dtype=torch.bfloat16, device="cuda")
    vm.vmla_cache_append_dc(to_dev(x), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache, slot0, t0,
                            w.grid_h, w.grid_w)
    vm.vmla_get_device_status()
    ref = oracle.cache_append(x, wts["w_dkv"], wts["w_kr"], t0, w.grid_h, w.grid_w)
    got = to_bits(cache)
    slots = (slot0 + np.arange(n_tok)) % cap
    assert np.array_equal(got[:, slots], ref), f"d_c={d_c}: append not bit-exact"
    untouched = np.setdiff1d(np.arange(cap), slots)
    assert np.all(got[:, untouched] == 0)


@pytest.mark.parametrize("n_tok", [148 * 32, 148 * 32 + 1])
def test_append_layout_switch(vm, n_tok):
    """Either side of the layout switch on a 148-SM part: 148 tiles run the wide
    layout, 149 (one token more) the tall one; both bit-exact."""
    import torch
    w = workload.CONFIGS["480p"]
    wts = workload.layer_weights(w)
    x = workload.normal_bf16(w.seed + 211, (n_tok,), (1, n_tok, w.d_model))
    cache = torch.zeros(1, n_tok, 224, dtype=torch.bfloat16, device="cuda")
    vm.vmla_cache_append(to_dev(x), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache, 0, 2, w.grid_h, w.grid_w)
    vm.vmla_get_device_status()
    ref = oracle.cache_append(x, wts["w_dkv"], wts["w_kr"], 2, w.grid_h, w.grid_w)
    assert np.array_equal(to_bits(cache), ref)


@pytest.mark.parametrize("d_c,n_tok", [(128, 2304), (128, 2300), (192, 2304), (192, 2300), (256, 1600),
                                       (256, 1590)])
def test_append_two_slice_ctas_per_sm(vm, d_c, n_tok):
    """More slice CTAs than SMs but at most two per SM (d_c >= 128): the slice
    layout with two CTAs sharing an SM.  72 tiles x 3 or 4 slices, or 50 x 5 at
    d_c = 256 (148 < slices <= 296 on a 148-SM part), a ragged last tile, a ring
    that wraps, t0 > 0; bit-exact, nothing outside the written slots touched."""
    import torch
    w = workload.CONFIGS["480p"].with_(d_c=d_c)
    wts = workload.layer_weights(w)
    cap, t0 = n_tok + 13, 4
    slot0 = cap - 100
    x = workload.normal_bf16(w.seed + 307, (n_tok, d_c), (1, n_tok, w.d_model))
    cache = torch.zeros(1, cap, d_c + 32, dtype=torch.bfloat16, device="cuda")
    vm.vmla_cache_append_dc(to_dev(x), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache, slot0, t0,
                            w.grid_h, w.grid_w)
    vm.vmla_get_device_status()
    ref = oracle.cache_append(x, wts["w_dkv"], wts["w_kr"], t0, w.grid_h, w.grid_w)
    got = to_bits(cache)
    slots = (slot0 + np.arange(n_tok)) % cap
    assert np.array_equal(got[:, slots], ref), f"d_c={d_c}, {n_tok} tokens: append not bit-exact"
    untouched = np.setdiff1d(np.arange(cap), slots)
    assert np.all(got[:, untouched] == 0)
