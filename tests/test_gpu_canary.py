"""Guard regions around every output buffer: each call writes its output and
nothing before or after it.

Each output is a view into a larger allocation, with GUARD bf16 elements on both
sides (a multiple of 8, so the view stays 16-byte aligned) filled with a sentinel
bit pattern; after the call the guards must hold the sentinel still.  Sizes are
ragged (partial query, key and M tiles) so every masked tail is exercised.
"""
from __future__ import annotations

import pytest

import workload
from helpers import SCALE, gpu_fill_window, to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096           # bf16 elements on each side
SENTINEL = 0x5A5A      # an ordinary finite bf16 value no kernel produces by accident here


@pytest.fixture(scope="module")
def vm():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200 as vm
    return vm


def guarded(*shape):
    """A bf16 CUDA tensor of `shape` between two sentinel-filled guard regions."""
    import torch
    n = 1
    for s in shape:
        n *= s
    buf = torch.full((n + 2 * GUARD,), SENTINEL, dtype=torch.int16, device="cuda")
    view = buf[GUARD:GUARD + n].view(torch.bfloat16).view(*shape)
    return buf, view


def assert_guards(buf, what):
    import torch
    head = buf[:GUARD]
    tail = buf[-GUARD:]
    assert torch.all(head == SENTINEL), f"{what}: write before the buffer"
    assert torch.all(tail == SENTINEL), f"{what}: write after the buffer"


def _ragged():
    # 7x9 grid: 189 queries (one full and one partial 128-row tile), 441 keys
    # (three full and one partial 128-key tile), 3 heads.
    return workload.CONFIGS["tiny"].with_(grid_h=7, grid_w=9, cached_frames=4, heads=3, seed=31)


def test_canary_append(vm):
    w = _ragged()
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    buf, cache = guarded(w.batch, w.n_kv, 224)
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    vm.vmla_get_device_status()
    assert_guards(buf, "cache append")


def test_canary_attention_forms(vm):
    import torch
    w = _ragged()
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    q, qr = to_dev(act["q"]), to_dev(act["q_rope"])
    wuk, wuv = to_dev(wts["w_uk"]), to_dev(wts["w_uv"])
    shape = (w.batch, w.n_q, w.heads, 128)

    buf, out = guarded(*shape)
    vm.vmla_chunk_attention(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    assert_guards(buf, "chunk attention")

    kbuf, kv = guarded(w.batch, w.n_kv, 2 * w.heads, 128)
    vm.vmla_materialize_kv(wuk, wuv, cache, w.n_kv, kv)
    vm.vmla_get_device_status()
    assert_guards(kbuf, "materialize kv")

    buf, out = guarded(*shape)
    vm.vmla_chunk_attention_materialized(q, qr, kv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    assert_guards(buf, "materialized attention")

    kd = to_dev(workload.batch_dense_kv(w)["k"])
    vd = to_dev(workload.batch_dense_kv(w)["v"])
    buf, out = guarded(*shape)
    vm.vmla_dense_attention(q, kd, vd, SCALE, out)
    vm.vmla_get_device_status()
    assert_guards(buf, "dense attention")


@pytest.mark.parametrize("d_c", [64, 128, 256])  # two-slot kernel at 64 and 128
def test_canary_latent_widths(vm, d_c):
    w = _ragged().with_(d_c=d_c)
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cbuf, cache = guarded(w.batch, w.n_kv, d_c + 32)
    per = w.tokens_per_frame
    x = to_dev(act["x"])
    for f0 in range(0, w.window_frames, w.chunk_frames):
        nf = min(w.chunk_frames, w.window_frames - f0)
        vm.vmla_cache_append_dc(x[:, f0 * per:(f0 + nf) * per].contiguous(), to_dev(wts["w_dkv"]),
                                to_dev(wts["w_kr"]), cache, f0 * per, f0, w.grid_h, w.grid_w)
    buf, out = guarded(w.batch, w.n_q, w.heads, 128)
    vm.vmla_chunk_attention_dc(to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]), to_dev(wts["w_uv"]),
                               cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out)
    vm.vmla_get_device_status()
    assert_guards(cbuf, f"append d_c={d_c}")
    assert_guards(buf, f"chunk attention d_c={d_c}")


@pytest.mark.parametrize("d_c", [128, 192])
def test_canary_append_many_tiles(vm, d_c):
    # 2 x 150 tiles of 32 tokens, the last one ragged: the layout with 8 tokens
    # per thread, two CTAs per SM.
    w = workload.CONFIGS["480p"].with_(d_c=d_c)
    wts = workload.layer_weights(w)
    x = to_dev(workload.normal_bf16(w.seed + 7, (5,), (2, 4790, w.d_model)))
    cbuf, cache = guarded(2, 4790, d_c + 32)
    vm.vmla_cache_append_dc(x, to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache, 0, 0, w.grid_h, w.grid_w)
    vm.vmla_get_device_status()
    assert_guards(cbuf, f"append many tiles d_c={d_c}")


def test_canary_projections(vm):
    # 189 tokens (a partial M tile), d_model 384: N = 384 + 96 for the query
    # projection (a part-filled rope half) and N = 384 for the output projection.
    w = _ragged().with_(d_model=384)
    iw = workload.io_weights(w)
    x = to_dev(workload.batch_activations(w)["x"][:, -w.n_q:])
    qbuf, q = guarded(w.batch, w.n_q, w.heads, 128)
    rbuf, qr = guarded(w.batch, w.n_q, w.heads, 32)
    vm.vmla_query_projection(x, to_dev(iw["w_q"]), to_dev(iw["w_qr"]), q, qr)
    vm.vmla_get_device_status()
    assert_guards(qbuf, "query projection q")
    assert_guards(rbuf, "query projection q_rope")
    ybuf, y = guarded(w.batch, w.n_q, w.d_model)
    vm.vmla_output_projection(q, to_dev(iw["w_o"]), y)
    vm.vmla_get_device_status()
    assert_guards(ybuf, "output projection")


@pytest.mark.parametrize("d_c,n_tok", [(128, 2300), (192, 2300), (256, 1590)])
def test_canary_append_two_slice_ctas(vm, d_c, n_tok):
    # the slice layout at two CTAs per SM, with a ragged last tile
    w = workload.CONFIGS["480p"].with_(d_c=d_c)
    wts = workload.layer_weights(w)
    x = to_dev(workload.normal_bf16(w.seed + 9, (n_tok,), (1, n_tok, w.d_model)))
    cbuf, cache = guarded(1, n_tok, d_c + 32)
    vm.vmla_cache_append_dc(x, to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache, 0, 3, w.grid_h, w.grid_w)
    vm.vmla_get_device_status()
    assert_guards(cbuf, f"append two slice CTAs per SM d_c={d_c}")


def test_canary_splitkv(vm):
    # every unit split (fewer units than SMs, 66 key tiles with a ragged last one):
    # output and workspace between guards
    import torch
    w = _ragged().with_(cached_frames=131)
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device="cuda")
    gpu_fill_window(vm, w, to_dev(act["x"]), to_dev(wts["w_dkv"]), to_dev(wts["w_kr"]), cache)
    need = vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv)
    assert need > 0 and need % 2 == 0
    wbuf, ws = guarded(need // 2)
    buf, out = guarded(w.batch, w.n_q, w.heads, 128)
    vm.vmla_chunk_attention_splitkv(to_dev(act["q"]), to_dev(act["q_rope"]), to_dev(wts["w_uk"]),
                                    to_dev(wts["w_uv"]), cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out,
                                    workspace=ws)
    vm.vmla_get_device_status()
    assert_guards(buf, "splitkv output")
    assert_guards(wbuf, "splitkv workspace")
