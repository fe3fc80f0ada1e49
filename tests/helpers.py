"""Shared helpers of the GPU tests: moving seeded inputs to the device, running
the append over a whole window, and the parity metrics."""
from __future__ import annotations

import numpy as np

RTOL_L2 = 1e-2   # relative L2 error bound for bf16 inputs with fp32 accumulation
ATOL_MAX = 3e-2  # max-abs error bound
SCALE = 160 ** -0.5  # 1 / sqrt(d_h + d_r): the per-head key is [content 128 ; rope 32]


def to_dev(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def to_bits(t) -> np.ndarray:
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.abs(got - ref).max())
    return rel, mx


def assert_close(got, ref, what=""):
    rel, mx = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert rel <= RTOL_L2 and mx <= ATOL_MAX, f"{what}: rel L2 {rel:.3e}, max abs {mx:.3e}"
    return rel, mx


def gpu_fill_window(vm, w, x_dev, wd, wk, cache, chunk_frames=None, slot_base=0):
    """Append every frame of the window in chunk-sized calls, as a rollout would:
    tokens of frames [t, t + chunk) go to slots (slot_base + t * per_frame) mod cap."""
    per = w.tokens_per_frame
    cf = chunk_frames or w.chunk_frames
    cap = cache.shape[1]
    for f0 in range(0, w.window_frames, cf):
        nf = min(cf, w.window_frames - f0)
        xs = x_dev[:, f0 * per:(f0 + nf) * per].contiguous()
        vm.vmla_cache_append(xs, wd, wk, cache, (slot_base + f0 * per) % cap, f0, w.grid_h, w.grid_w)


def sample_rows(n_q: int, k: int, seed: int = 0) -> np.ndarray:
    """k random query rows plus the first and last full/ragged tile edges."""
    rng = np.random.default_rng(seed)
    edge = {0, 1, 127, 128, n_q - 1, n_q - 2, (n_q // 128) * 128, min(n_q - 1, (n_q // 128) * 128 + 1)}
    rows = set(int(r) for r in rng.choice(n_q, size=min(k, n_q), replace=False)) | {e for e in edge if 0 <= e < n_q}
    return np.array(sorted(rows), dtype=np.int64)
