"""Seeded synthetic workloads for the VideoMLA latent-KV chunk attention path.

This module only *draws* inputs: shapes of the Wan2.1-T2V-1.3B-sized
workloads and seeded normal samples rounded to bf16.  It contains none of the
method's arithmetic (no projection, no rotary embedding, no attention), so
both the fp64 oracle and the CUDA path can consume the same bits from here
without sharing any code with each other.

Shapes (VideoMLA, "Low-Rank Latent KV Cache for Minute-Scale Autoregressive
Video Diffusion", abstract and key results): a head-shared content latent of
d_c = 192 plus a head-shared 3D-RoPE key of d_r = 32, i.e. 224 cached scalars
per token against 2 x 12 heads x 128 = 3072 for the dense per-head cache.
The backbone is Wan2.1-T2V-1.3B (model width 1536, 12 heads of 128), driven
chunk-causally: each chunk of 3 latent frames attends to a sliding window of
cached frames plus itself.

Value distributions: activations (x, q, q_rope, dense k/v) ~ N(0, 1);
projection weights ~ N(0, 1/fan_in) with fan_in = 1536 for W_DKV / W_KR and
fan_in = 192 for W_UK / W_UV.  All values are drawn in fp32 from numpy's
PCG64 (seeded through SeedSequence so every tensor has its own stream) and
rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np

# Stream ids: one independent random stream per named tensor.
_STREAM = {
    "x": 1,
    "q": 2,
    "q_rope": 3,
    "w_dkv": 11,
    "w_kr": 12,
    "w_uk": 13,
    "w_uv": 14,
    "w_q": 15,
    "w_qr": 16,
    "w_o": 17,
    "o": 18,
    "k_dense": 21,
    "v_dense": 22,
}


@dataclass(frozen=True)
class Workload:
    """One workload shape.  Token order inside a frame is row-major (row, col)."""

    name: str
    batch: int
    grid_h: int
    grid_w: int
    cached_frames: int
    chunk_frames: int = 3
    heads: int = 12
    d_model: int = 1536
    d_head: int = 128
    d_c: int = 192
    d_r: int = 32
    layers: int = 1
    steps: int = 1
    seed: int = 0
    rope_theta: float = 1.0e4
    rope_split: tuple = (12, 10, 10)  # (t, h, w) dims of the 32-dim rope key

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def n_q(self) -> int:
        return self.chunk_frames * self.tokens_per_frame

    @property
    def n_cached(self) -> int:
        return self.cached_frames * self.tokens_per_frame

    @property
    def n_kv(self) -> int:
        return self.n_cached + self.n_q

    @property
    def window_frames(self) -> int:
        return self.cached_frames + self.chunk_frames

    @property
    def chunk_t0(self) -> int:
        """Frame index of the first frame of the current chunk."""
        return self.cached_frames

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def attention_flops(self) -> float:
        """Absorbed-MLA tensor FLOPs of one chunk-attention call:
        2 * B * Nq * H * Nkv * (d_c + d_r)  (scores)  +  2 * B * Nq * H * Nkv * d_c  (P.C)."""
        per = 2.0 * self.batch * self.n_q * self.heads * self.n_kv
        return per * (self.d_c + self.d_r) + per * self.d_c

    def projection_flops(self) -> float:
        """Query absorption (q_h . W_UK_h) and the W_UV epilogue of one call."""
        return 2.0 * 2.0 * self.batch * self.n_q * self.heads * self.d_head * self.d_c

    def nonabsorbed_flops(self) -> float:
        """Attention over materialised per-head keys [K_h ; k_r] (160) and values V_h (128)."""
        return 2.0 * self.batch * self.n_q * self.heads * self.n_kv * (self.d_head + self.d_r + self.d_head)

    def dense_flops(self) -> float:
        """Dense per-head attention FLOPs (QK^T and PV, d = 128)."""
        return 2.0 * 2.0 * self.batch * self.n_q * self.heads * self.n_kv * self.d_head

    def io_projection_flops(self) -> float:
        """Query + rope-query projection (D -> H*160) and output projection (H*128 -> D)
        of the current chunk's tokens."""
        n = self.batch * self.n_q
        return 2.0 * n * self.d_model * self.heads * (self.d_head + self.d_r) + \
            2.0 * n * self.heads * self.d_head * self.d_model

    def append_flops(self, n_tok: int | None = None) -> float:
        n = self.n_q if n_tok is None else n_tok
        return 2.0 * self.batch * n * (self.d_c + self.d_r) * self.d_model


# The five workloads: a tiny case, the 480P single layer, the full per-chunk
# schedule at 480P, batch 8 at 480P and the 1080P single layer.
CONFIGS = {
    "tiny": Workload("tiny", batch=1, grid_h=8, grid_w=8, cached_frames=6, seed=0),
    "480p": Workload("480p", batch=1, grid_h=30, grid_w=52, cached_frames=18, seed=2000),
    "480p_chunk": Workload("480p_chunk", batch=1, grid_h=30, grid_w=52, cached_frames=18,
                           layers=30, steps=4, seed=3000),
    "480p_b8": Workload("480p_b8", batch=8, grid_h=30, grid_w=52, cached_frames=18, seed=4000),
    "1080p": Workload("1080p", batch=1, grid_h=68, grid_w=120, cached_frames=6, seed=5000),
}


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Decode bf16 bits to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed: int, key: tuple, shape: tuple, std: float = 1.0) -> np.ndarray:
    """Seeded N(0, std^2) samples rounded to bf16 (uint16 bits)."""
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, *[int(k) for k in key]])
    rng = np.random.Generator(np.random.PCG64(ss))
    v = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        v *= np.float32(std)
    return bf16_bits(v)


def layer_weights(w: Workload, layer: int = 0) -> dict:
    """Projection weights of one attention layer, nn.Linear layout [out, in]."""
    D, H, dh, dc, dr = w.d_model, w.heads, w.d_head, w.d_c, w.d_r
    s = w.seed
    return {
        "w_dkv": normal_bf16(s, (layer, _STREAM["w_dkv"]), (dc, D), std=D ** -0.5),
        "w_kr": normal_bf16(s, (layer, _STREAM["w_kr"]), (dr, D), std=D ** -0.5),
        # W_UK / W_UV map the 192-dim latent to the 12 x 128 heads: [H*128, 192].
        "w_uk": normal_bf16(s, (layer, _STREAM["w_uk"]), (H * dh, dc), std=dc ** -0.5),
        "w_uv": normal_bf16(s, (layer, _STREAM["w_uv"]), (H * dh, dc), std=dc ** -0.5),
    }


def io_weights(w: Workload, layer: int = 0) -> dict:
    """The projections around the attention of one layer, nn.Linear layout [out, in]:
    w_q [H*128, D] and w_qr [H*32, D] map hidden states to content / rope queries,
    w_o [D, H*128] maps the concatenated head outputs back to the model width."""
    D, H, dh, dr = w.d_model, w.heads, w.d_head, w.d_r
    s = w.seed
    return {
        "w_q": normal_bf16(s, (layer, _STREAM["w_q"]), (H * dh, D), std=D ** -0.5),
        "w_qr": normal_bf16(s, (layer, _STREAM["w_qr"]), (H * dr, D), std=D ** -0.5),
        "w_o": normal_bf16(s, (layer, _STREAM["w_o"]), (D, H * dh), std=(H * dh) ** -0.5),
    }


def head_outputs(w: Workload, layer: int = 0) -> np.ndarray:
    """A stand-in attention output o [B, n_q, H, 128] ~ N(0, 1) for testing W_O alone."""
    return np.stack([normal_bf16(w.seed + b * 7919, (layer, _STREAM["o"]), (w.n_q, w.heads, w.d_head))
                     for b in range(w.batch)])


def sample_activations(w: Workload, sample: int, layer: int = 0, step: int = 0) -> dict:
    """Activations of one batch sample:

    x      [n_kv, D]       hidden states of every token in the window (cached frames
                           first, then the current chunk), frame-major, row-major inside a frame
    q      [n_q, H, 128]   per-head content queries of the current chunk
    q_rope [n_q, H, 32]    per-head rope queries (not yet rotated)
    """
    D, H, dh, dr = w.d_model, w.heads, w.d_head, w.d_r
    s = w.seed + sample * 7919
    return {
        "x": normal_bf16(s, (layer, _STREAM["x"]), (w.n_kv, D)),
        "q": normal_bf16(s, (layer, step, _STREAM["q"]), (w.n_q, H, dh)),
        "q_rope": normal_bf16(s, (layer, step, _STREAM["q_rope"]), (w.n_q, H, dr)),
    }


def dense_kv(w: Workload, sample: int, layer: int = 0) -> dict:
    """Per-head dense K and V of the window, [n_kv, H, 128] each (the 3072-scalar cache)."""
    H, dh = w.heads, w.d_head
    s = w.seed + sample * 7919
    return {
        "k": normal_bf16(s, (layer, _STREAM["k_dense"]), (w.n_kv, H, dh)),
        "v": normal_bf16(s, (layer, _STREAM["v_dense"]), (w.n_kv, H, dh)),
    }


def batch_activations(w: Workload, layer: int = 0, step: int = 0) -> dict:
    """Stack sample_activations over the batch: x [B, n_kv, D], q [B, n_q, H, 128], ..."""
    parts = [sample_activations(w, b, layer, step) for b in range(w.batch)]
    return {k: np.stack([p[k] for p in parts]) for k in parts[0]}


def batch_dense_kv(w: Workload, layer: int = 0) -> dict:
    parts = [dense_kv(w, b, layer) for b in range(w.batch)]
    return {k: np.stack([p[k] for p in parts]) for k in parts[0]}
