"""vmla_chunk_attention_splitkv: the latent attention whose last partial wave of
(sample, query tile, head) units runs split over key ranges, each split unit merged
by its last part (parts keep at least 32 key tiles, so the split shapes here have
windows of more than 8192 keys).  Checked against the fp64 oracle (tolerance relative L2 <= 1e-2,
max-abs <= 3e-2) and against vmla_chunk_attention on the same inputs, on shapes
where every unit is split (fewer units than SMs), where only the tail wave is split
(1080P), where nothing is split (480P: the units fill exactly three waves), with a
ragged last key tile inside a part, and for two calls in a row on one workspace.
"""
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


def _inputs(vm, w, layer=0):
    import torch
    wts = workload.layer_weights(w, layer)
    act = workload.batch_activations(w, layer)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    dev = dict(q=to_dev(act["q"]), qr=to_dev(act["q_rope"]), wuk=to_dev(wts["w_uk"]), wuv=to_dev(wts["w_uv"]),
               cache=cache)
    return dev, wts, act


def _run(vm, w, d, split, workspace=None):
    import torch
    out = torch.full((w.batch, w.n_q, w.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    if split:
        vm.vmla_chunk_attention_splitkv(d["q"], d["qr"], d["wuk"], d["wuv"], d["cache"], w.n_kv, w.chunk_t0,
                                        w.grid_h, w.grid_w, SCALE, out, workspace=workspace)
    else:
        vm.vmla_chunk_attention(d["q"], d["qr"], d["wuk"], d["wuv"], d["cache"], w.n_kv, w.chunk_t0, w.grid_h,
                                w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    return to_f64(out)


def _oracle(w, wts, act, rows=None):
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    return oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv,
                                  w.chunk_t0, w.grid_h, w.grid_w, SCALE, rows=rows)


SMALL = {
    # 8x8 patches, a 136-frame window: 8704 keys = 68 key tiles; 2 query tiles x 3
    # heads = 6 units, every one split in 2 parts of 34 key tiles
    "long_window": workload.CONFIGS["tiny"].with_(cached_frames=133, heads=3, seed=94),
    # 7x9 patches, 134 frames: 8442 keys = 65 full key tiles + 122 keys, so the
    # second part of every unit ends in a ragged tile; 2 x 3 = 6 units
    "ragged": workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=131, heads=3, seed=95),
    # three samples of the ragged shape: 18 units, batch indexing of the split units
    "ragged_b3": workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=131, heads=3, batch=3, seed=96),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_splitkv_small_against_oracle_and_plain(vm, name):
    w = SMALL[name]
    assert vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv) > 0
    d, wts, act = _inputs(vm, w)
    got = _run(vm, w, d, True)
    ref = _oracle(w, wts, act)
    assert_close(got, ref, f"splitkv {name} vs oracle")
    plain = _run(vm, w, d, False)
    assert_close(got, plain, f"splitkv {name} vs vmla_chunk_attention")


def test_splitkv_two_calls_share_a_workspace(vm):
    # the second call starts from the first call's workspace contents
    import torch
    w = SMALL["ragged"]
    need = vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device="cuda")
    for layer in (0, 3):
        d, wts, act = _inputs(vm, w, layer)
        got = _run(vm, w, d, True, workspace=ws)
        assert_close(got, _oracle(w, wts, act), f"splitkv, layer {layer}, shared workspace")


def test_splitkv_1080p_tail_wave(vm):
    # 192 query tiles x 12 heads = 2304 units: 15 whole waves of 148 and 84 tail
    # units, each split over the keys; sampled rows include the last query tiles,
    # whose heads fall in the split tail.
    w = workload.CONFIGS["1080p"]
    assert vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv) > 0
    d, wts, act = _inputs(vm, w)
    got = _run(vm, w, d, True)
    plain = _run(vm, w, d, False)
    assert_close(got, plain, "1080p splitkv vs vmla_chunk_attention (every output)")
    tail_rows = np.arange(w.n_q - 128 * 8, w.n_q, 37)
    rows = np.union1d(sample_rows(w.n_q, 128, seed=11), tail_rows)
    ref = _oracle(w, wts, act, rows=rows)
    assert_close(got[:, rows], ref, "1080p splitkv vs oracle (sampled rows)")


def test_splitkv_480p_needs_no_split(vm):
    # 37 query tiles x 12 heads = 444 units = 3 whole waves: no workspace, same launch
    w = workload.CONFIGS["480p"]
    assert vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv) == 0
    d, _, _ = _inputs(vm, w)
    got = _run(vm, w, d, True)
    plain = _run(vm, w, d, False)
    assert np.array_equal(got, plain)


def test_splitkv_short_window_needs_no_split(vm):
    # 5 key tiles: too few for parts of 32 key tiles, so the launch is unsplit
    w = workload.CONFIGS["tiny"]
    assert vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv) == 0
    d, wts, act = _inputs(vm, w)
    got = _run(vm, w, d, True)
    assert np.array_equal(got, _run(vm, w, d, False))


def test_splitkv_rejects_a_small_workspace(vm):
    import torch
    w = SMALL["long_window"]
    need = vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv)
    d, _, _ = _inputs(vm, w)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(vm.VmlaError) as ei:
        vm.vmla_chunk_attention_splitkv(d["q"], d["qr"], d["wuk"], d["wuv"], d["cache"], w.n_kv, w.chunk_t0,
                                        w.grid_h, w.grid_w, SCALE, out, workspace=small)
    assert ei.value.code == vm.VMLA_ERR_INVALID_ARG and "workspace" in vm.vmla_last_error()
    vm.vmla_get_device_status()
