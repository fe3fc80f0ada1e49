"""The per-chunk schedule (layers x [append + denoising-step attentions]) replayed
as one CUDA graph gives bit-identical results to eager launches, and a layer's
output matches the fp64 oracle (which builds its own cache from the same inputs).
Consecutive chunks slide the window: the second chunk's append evicts the oldest
frames, and its attention matches the oracle over the ring's contents."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workload
from helpers import SCALE, assert_close, to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bench
    import latent_kv_cache_b200 as vm
    return torch, bench, vm


def test_graph_replay_matches_eager_and_oracle(env):
    torch, bench, vm = env
    w = workload.CONFIGS["tiny"].with_(layers=3, steps=2, grid_h=7, grid_w=9, cached_frames=4)
    dev = torch.device("cuda", 0)
    op_lists, layers = bench.build_chunk_schedule(vm, w, dev, seed=7)
    ops = op_lists[0]
    for op in ops:
        op()
    vm.vmla_get_device_status()
    eager = [[o.clone() for o in L["out"]] for L in layers]
    caches = [L["cache"].clone() for L in layers]
    graph = bench.capture_graph(ops)
    for L in layers:
        for o in L["out"]:
            o.zero_()
    graph.replay()
    vm.vmla_get_device_status()
    for L, E, C in zip(layers, eager, caches):
        assert torch.equal(L["cache"], C)
        for o, e in zip(L["out"], E):
            assert torch.equal(o, e)

    # Oracle check of the last layer, last step: its cache comes from the oracle's own
    # append of the same window tokens (x is regenerated from the same seeded stream).
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    x_win = (torch.randn(w.batch, w.n_kv, w.d_model, generator=g, device=dev, dtype=torch.float32)).to(torch.bfloat16)
    L = layers[-1]
    bits = lambda t: to_bits(t)  # noqa: E731
    ref_cache = oracle.cache_append(bits(x_win), bits(L["wd"]), bits(L["wk"]), 0, w.grid_h, w.grid_w)
    assert np.array_equal(bits(L["cache"]), ref_cache)
    ref = oracle.chunk_attention(bits(L["q"][-1]), bits(L["qr"][-1]), bits(L["wuk"]), bits(L["wuv"]), ref_cache,
                                 w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE)
    assert_close(L["out"][-1].float().cpu().numpy().astype(np.float64), ref, "graph layer output")


def test_second_chunk_evicts_oldest_frames(env):
    torch, bench, vm = env
    # 7x9 grid, 4 cached frames + a 3-frame chunk: a 441-slot ring.  Chunk 0 (frames
    # 4-6) fills slots 252-440; chunk 1 (frames 7-9) wraps to slots 0-188, evicting
    # frames 0-2 and leaving frame 3 in slots 189-251.
    w = workload.CONFIGS["tiny"].with_(layers=2, steps=2, grid_h=7, grid_w=9, cached_frames=4)
    dev = torch.device("cuda", 0)
    op_lists, layers = bench.build_chunk_schedule(vm, w, dev, seed=9, chunks=2)
    for ops in op_lists:
        for op in ops:
            op()
    vm.vmla_get_device_status()

    g = torch.Generator(device=dev)
    g.manual_seed(9)
    x_win = (torch.randn(w.batch, w.n_kv, w.d_model, generator=g, device=dev, dtype=torch.float32)).to(torch.bfloat16)
    bits = lambda t: to_bits(t)  # noqa: E731
    L = layers[-1]
    xb = bits(x_win)
    per, nq = w.tokens_per_frame, w.n_q
    ref_cache = np.empty((w.batch, w.n_kv, 224), dtype=np.uint16)
    ref_cache[:, :w.n_cached] = oracle.cache_append(xb[:, :w.n_cached], bits(L["wd"]), bits(L["wk"]), 0,
                                                    w.grid_h, w.grid_w)
    chunk = xb[:, w.n_cached:]
    ref_cache[:, w.n_cached:] = oracle.cache_append(chunk, bits(L["wd"]), bits(L["wk"]), w.chunk_t0,
                                                    w.grid_h, w.grid_w)
    t1 = w.chunk_t0 + w.chunk_frames
    ref_cache[:, :nq] = oracle.cache_append(chunk, bits(L["wd"]), bits(L["wk"]), t1, w.grid_h, w.grid_w)
    assert np.array_equal(bits(L["cache"]), ref_cache)
    assert per * w.chunk_frames == nq
    ref = oracle.chunk_attention(bits(L["q"][-1]), bits(L["qr"][-1]), bits(L["wuk"]), bits(L["wuv"]), ref_cache,
                                 w.n_kv, t1, w.grid_h, w.grid_w, SCALE)
    assert_close(L["out"][-1].float().cpu().numpy().astype(np.float64), ref, "second chunk, sliding window")
