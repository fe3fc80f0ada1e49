"""vmla_chunk_attention and vmla_dense_attention on the GPU against the fp64 oracle.

Small cases compare every output; the full-size workloads (480P single layer,
batch 8, 1080P) compare sampled query rows, all heads, every key, in the same
launch configuration the benchmark times.  Tolerance: relative L2 <= 1e-2 and
max-abs <= 3e-2 (bf16 inputs, fp32 accumulation).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workload
from helpers import SCALE, assert_close, gpu_fill_window, sample_rows, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


def _mla_case(vm, w, layer=0, q_mult=1.0, rows=None, cap_extra=0, poison=False, cache_bits=None):
    """Fill the window on the GPU, run chunk attention, compare with the oracle.
    The oracle consumes its own append of the same tokens (bit-identical by the
    append tests) so no oracle input comes from the GPU."""
    import torch
    wts = workload.layer_weights(w, layer)
    act = workload.batch_activations(w, layer)
    q, qr = act["q"], act["q_rope"]
    if q_mult != 1.0:
        q = workload.bf16_bits(workload.bf16_to_f32(q) * np.float32(q_mult))
        qr = workload.bf16_bits(workload.bf16_to_f32(qr) * np.float32(q_mult))
    cap = w.n_kv + cap_extra
    if cache_bits is None:
        cache = torch.zeros(w.batch, cap, 224, dtype=torch.bfloat16, device="cuda")
        if poison:
            cache.view(torch.int16).fill_(0x7FC0)  # NaN in every slot the window does not cover
        gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
        ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    else:
        ref_cache = cache_bits
        full = np.zeros((w.batch, cap, 224), dtype=np.uint16)
        full[:, :w.n_kv] = cache_bits
        cache = to_dev(full)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention(to_dev(q), to_dev(qr), to_dev(wts["w_uk"]), to_dev(wts["w_uv"]), cache,
                            w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    ref = oracle.chunk_attention(q, qr, wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0,
                                 w.grid_h, w.grid_w, SCALE, rows=rows)
    got = to_f64(out)
    if rows is not None:
        got = got[:, rows]
    return got, ref


def test_chunk_attention_tiny_full(vm):
    got, ref = _mla_case(vm, workload.CONFIGS["tiny"])
    assert_close(got, ref, "tiny")


def test_chunk_attention_tiny_peaked(vm):
    # queries x4: peaked softmax, exercises the running-max rescale; full tolerance
    got, ref = _mla_case(vm, workload.CONFIGS["tiny"], q_mult=4.0)
    assert_close(got, ref, "tiny x4")


def test_chunk_attention_tiny_very_peaked(vm):
    """Queries x8 (scores ~8x the workload's, a near one-hot softmax).  Relative L2
    keeps the 1e-2 bound; max-abs is held to 8e-2.  Any form whose score product
    takes a bf16 operand formed from the latent carries that operand's rounding
    (2^-9 relative): the absorbed query q.W_UK here, the materialised key c.W_UK^T
    in the non-absorbed form and in a dense cache of those keys.  The CPU tests of
    tests/test_tolerance_reading.py show that this one rounding alone exceeds
    3e-2 at x8; this test shows the same on the three kernels, and that the
    latent kernel's error is no larger than the other two forms'."""
    import torch
    from helpers import errors
    w = workload.CONFIGS["tiny"]
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    q8 = workload.bf16_bits(workload.bf16_to_f32(act["q"]) * np.float32(8.0))
    qr8 = workload.bf16_bits(workload.bf16_to_f32(act["q_rope"]) * np.float32(8.0))
    qr0 = np.zeros_like(qr8)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    wuk, wuv = to_dev(wts["w_uk"]), to_dev(wts["w_uv"])
    shape = (w.batch, w.n_q, w.heads, 128)
    kv = torch.empty(w.batch, w.n_kv, 2 * w.heads, 128, dtype=torch.bfloat16, device="cuda")
    # Dense per-head cache holding the latent's keys and values rounded to bf16
    # (the rope queries are zero in this comparison: the dense kernel has no rope key).
    kv_bits = workload.bf16_bits(oracle.materialized_kv(wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv)
                                 .astype(np.float32))
    kd = to_dev(np.ascontiguousarray(kv_bits[:, :, :w.heads]))
    vd = to_dev(np.ascontiguousarray(kv_bits[:, :, w.heads:]))
    err = {}
    for rope_name, qr_bits in (("rope", qr8), ("no rope", qr0)):
        ref = oracle.chunk_attention(q8, qr_bits, wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv, w.chunk_t0,
                                     w.grid_h, w.grid_w, SCALE)
        q_d, qr_d = to_dev(q8), to_dev(qr_bits)
        out_a = torch.empty(*shape, dtype=torch.bfloat16, device="cuda")
        vm.vmla_chunk_attention(q_d, qr_d, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out_a)
        out_m = torch.empty_like(out_a)
        vm.vmla_materialize_kv(wuk, wuv, cache, w.n_kv, kv)
        vm.vmla_chunk_attention_materialized(q_d, qr_d, kv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                             out_m)
        outs = {"absorbed": out_a, "non-absorbed": out_m}
        if rope_name == "no rope":
            out_d = torch.empty_like(out_a)
            vm.vmla_dense_attention(q_d, kd, vd, SCALE, out_d)
            outs["dense bf16 K_h"] = out_d
        vm.vmla_get_device_status()
        for form, o in outs.items():
            got = to_f64(o)
            assert np.all(np.isfinite(got)), (rope_name, form)
            err[(rope_name, form)] = errors(got, ref)
    for key, (rel, mx) in err.items():
        assert rel <= 1e-2 and mx <= 8e-2, (key, rel, mx)
    for key in (("rope", "non-absorbed"), ("no rope", "non-absorbed"), ("no rope", "dense bf16 K_h")):
        assert err[key][1] > 3e-2, ("the bf16-key forms share the x8 excess", key, err[key])
    for r in ("rope", "no rope"):
        others = max(v[1] for k, v in err.items() if k[0] == r and k[1] != "absorbed")
        assert err[(r, "absorbed")][1] <= 1.25 * others, (r, err)


def test_chunk_attention_ragged_and_small(vm):
    # n_q, n_kv not multiples of 128; several query tiles and key tiles
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3)
    got, ref = _mla_case(vm, w)
    assert_close(got, ref, "ragged")


def test_chunk_attention_ragged_batch(vm):
    # three samples (independent seeds) of the ragged shape: batch indexing of
    # queries, cache rows and outputs with partial query and key tiles
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3, batch=3, seed=91)
    got, ref = _mla_case(vm, w)
    assert_close(got, ref, "ragged batch 3")
    assert not np.allclose(got[0], got[1])


def test_chunk_attention_poisoned_slots_ignored(vm):
    # slots past n_kv hold NaN; they must never reach the output
    got, ref = _mla_case(vm, workload.CONFIGS["tiny"], cap_extra=300, poison=True)
    assert_close(got, ref, "poisoned")


def test_chunk_attention_single_key(vm):
    w = workload.CONFIGS["tiny"].with_(heads=2)
    wts = workload.layer_weights(w)
    bits = oracle.cache_append(workload.normal_bf16(3, (0,), (1, 1, 1536)), wts["w_dkv"], wts["w_kr"],
                               0, w.grid_h, w.grid_w)
    w1 = w.with_(cached_frames=0)
    # n_kv = 1 key for all queries: out = W_UV_h . c of that key for every query
    import torch
    act = workload.batch_activations(w1)
    cache = to_dev(np.concatenate([bits, np.zeros((1, 7, 224), np.uint16)], axis=1))
    out = torch.empty(1, w1.n_q, 2, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_chunk_attention(to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]),
                            to_dev(wts["w_uv"]), cache, 1, 0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], bits, 1, 0,
                                 w.grid_h, w.grid_w, SCALE)
    assert_close(to_f64(out), ref, "single key")


def test_chunk_attention_identical_keys(vm):
    w = workload.CONFIGS["tiny"]
    wts = workload.layer_weights(w)
    row = oracle.cache_append(workload.normal_bf16(4, (0,), (1, 1, 1536)), wts["w_dkv"], wts["w_kr"],
                              0, w.grid_h, w.grid_w)
    bits = np.repeat(row, w.n_kv, axis=1)
    got, ref = _mla_case(vm, w, cache_bits=bits)
    assert_close(got, ref, "identical keys")
    # closed form: every query returns V of that key
    v = oracle.decode_bf16(wts["w_uv"]).reshape(w.heads, 128, 192) @ oracle.decode_bf16(row[0, 0, :192])
    np.testing.assert_allclose(got[0], np.broadcast_to(v, got[0].shape), atol=2e-2)


def test_chunk_attention_480p_sampled(vm):
    w = workload.CONFIGS["480p"]
    rows = sample_rows(w.n_q, 512, seed=1)
    got, ref = _mla_case(vm, w, rows=rows)
    assert_close(got, ref, "480p")


def test_chunk_attention_480p_b8_sampled(vm):
    w = workload.CONFIGS["480p_b8"]
    rows = sample_rows(w.n_q, 64, seed=2)
    got, ref = _mla_case(vm, w, rows=rows)
    assert_close(got, ref, "480p b8")
    # no cross-sample leakage: each sample's rows match its own oracle rows
    for b in range(w.batch):
        assert_close(got[b], ref[b], f"480p b8 sample {b}")


def test_chunk_attention_1080p_sampled(vm):
    w = workload.CONFIGS["1080p"]
    rows = sample_rows(w.n_q, 512, seed=3)
    got, ref = _mla_case(vm, w, rows=rows)
    assert_close(got, ref, "1080p")


def test_chunk_attention_other_layer_weights(vm):
    # a second layer of the per-chunk schedule (independent weights and activations)
    w = workload.CONFIGS["480p_chunk"]
    rows = sample_rows(w.n_q, 64, seed=4)
    got, ref = _mla_case(vm, w, layer=17, rows=rows)
    assert_close(got, ref, "480p layer 17")


# ---------------------------------------------------------------------------
# Dense per-head baseline
# ---------------------------------------------------------------------------
def _dense_case(vm, w, rows=None):
    import torch
    act = workload.batch_activations(w)
    kv = workload.batch_dense_kv(w)
    out = torch.empty(w.batch, w.n_q, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    vm.vmla_dense_attention(to_dev(act["q"]), to_dev(kv["k"]), to_dev(kv["v"]), SCALE, out)
    vm.vmla_get_device_status()
    ref = oracle.dense_attention(act["q"], kv["k"], kv["v"], SCALE, rows=rows)
    got = to_f64(out)
    return (got if rows is None else got[:, rows]), ref


def test_dense_attention_tiny_full(vm):
    got, ref = _dense_case(vm, workload.CONFIGS["tiny"])
    assert_close(got, ref, "dense tiny")


def test_dense_attention_ragged(vm):
    got, ref = _dense_case(vm, workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3))
    assert_close(got, ref, "dense ragged")


def test_dense_attention_ragged_batch(vm):
    w = workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3, batch=3, seed=92)
    got, ref = _dense_case(vm, w)
    assert_close(got, ref, "dense ragged batch 3")


def test_dense_attention_480p_sampled(vm):
    w = workload.CONFIGS["480p"]
    rows = sample_rows(w.n_q, 128, seed=5)
    got, ref = _dense_case(vm, w, rows=rows)
    assert_close(got, ref, "dense 480p")


def test_dense_attention_480p_b8_sampled(vm):
    # eight samples with their own K/V: no cross-sample leakage in the per-head kernel
    w = workload.CONFIGS["480p_b8"]
    rows = sample_rows(w.n_q, 64, seed=6)
    got, ref = _dense_case(vm, w, rows=rows)
    for b in range(w.batch):
        assert_close(got[b], ref[b], f"dense 480p b8 sample {b}")


def test_dense_attention_1080p_sampled(vm):
    # 574 key tiles, the last one holding 96 keys
    w = workload.CONFIGS["1080p"]
    rows = sample_rows(w.n_q, 128, seed=7)
    got, ref = _dense_case(vm, w, rows=rows)
    assert_close(got, ref, "dense 1080p")


# ---------------------------------------------------------------------------
# Failure path: a bounded wait that runs out is reported, and the context survives
# ---------------------------------------------------------------------------
def test_wait_timeout_is_reported_and_context_survives(vm):
    import torch
    vm.vmla_get_device_status()  # clean slate
    vm.vmla_selftest_wait_timeout(2_000_000)  # 2 ms
    with pytest.raises(vm.VmlaError) as ei:
        vm.vmla_get_device_status()
    assert ei.value.code == vm.VMLA_ERR_TIMEOUT
    vm.vmla_get_device_status()  # cleared
    got, ref = _mla_case(vm, workload.CONFIGS["tiny"])
    assert_close(got, ref, "after timeout")
    assert torch.cuda.is_available()
