"""Python binding of libvideomla.so, the B200 VideoMLA latent-KV chunk-attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI (include/videomla.h).  Functions carry the C names;
tensors are torch CUDA tensors (bf16, contiguous) whose device pointers are
passed through, on the given stream (default: torch's current stream).  Any
non-zero status raises VmlaError.  There is no fallback: if the shared library
is missing, importing this package fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvideomla.so")

VMLA_OK = 0
VMLA_ERR_INVALID_ARG = 1
VMLA_ERR_UNSUPPORTED = 2
VMLA_ERR_CUDA = 3
VMLA_ERR_TIMEOUT = 4

D_C, D_R, D_HEAD = 192, 32, 128


class VmlaError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{message} [{code}]")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python latent_kv_cache_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    lib.vmla_status_string.argtypes = [ctypes.c_int]
    lib.vmla_status_string.restype = ctypes.c_char_p
    lib.vmla_last_error.argtypes = []
    lib.vmla_last_error.restype = ctypes.c_char_p
    lib.vmla_cache_append.argtypes = [P, P, P, i32, i32, i32, P, i64, i64, i64, i32, i32, P]
    lib.vmla_cache_append.restype = ctypes.c_int
    lib.vmla_chunk_attention.argtypes = [P, P, P, P, P, i32, i32, i32, i64, i64, i64, i32, i32, f32, P, P]
    lib.vmla_chunk_attention.restype = ctypes.c_int
    lib.vmla_dense_attention.argtypes = [P, P, P, i32, i32, i64, i32, i32, f32, P, P]
    lib.vmla_dense_attention.restype = ctypes.c_int
    lib.vmla_get_device_status.argtypes = [P]
    lib.vmla_get_device_status.restype = ctypes.c_int
    lib.vmla_selftest_wait_timeout.argtypes = [i64, P]
    lib.vmla_selftest_wait_timeout.restype = ctypes.c_int
    lib.vmla_materialized_kv_bytes.argtypes = [i32, i32, i64]
    lib.vmla_materialized_kv_bytes.restype = i64
    lib.vmla_materialize_kv.argtypes = [P, P, P, i32, i32, i64, i64, P, P]
    lib.vmla_materialize_kv.restype = ctypes.c_int
    lib.vmla_chunk_attention_materialized.argtypes = [P, P, P, P, i32, i32, i32, i64, i64, i64, i32, i32, f32, P, P]
    lib.vmla_chunk_attention_materialized.restype = ctypes.c_int
    lib.vmla_chunk_attention_nonabsorbed.argtypes = [P, P, P, P, P, i32, i32, i32, i64, i64, i64, i32, i32, f32,
                                                     P, i64, P, P]
    lib.vmla_chunk_attention_nonabsorbed.restype = ctypes.c_int
    lib.vmla_cache_append_dc.argtypes = [P, P, P, i32, i32, i32, i32, P, i64, i64, i64, i32, i32, P]
    lib.vmla_cache_append_dc.restype = ctypes.c_int
    lib.vmla_chunk_attention_dc.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64, i64, i64, i32, i32, f32, P, P]
    lib.vmla_chunk_attention_dc.restype = ctypes.c_int
    lib.vmla_query_projection.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P]
    lib.vmla_query_projection.restype = ctypes.c_int
    lib.vmla_output_projection.argtypes = [P, P, i32, i32, i32, i32, P, P]
    lib.vmla_output_projection.restype = ctypes.c_int
    lib.vmla_chunk_attention_nonabsorbed_noalloc.argtypes = [P, P, P, P, P, i32, i32, i32, i64, i64, i64, i32, i32,
                                                             f32, P, P]
    lib.vmla_chunk_attention_nonabsorbed_noalloc.restype = ctypes.c_int
    lib.vmla_chunk_attention_splitkv_workspace_bytes.argtypes = [i32, i32, i32, i64]
    lib.vmla_chunk_attention_splitkv_workspace_bytes.restype = i64
    lib.vmla_chunk_attention_splitkv.argtypes = [P, P, P, P, P, i32, i32, i32, i64, i64, i64, i32, i32, f32, P, i64,
                                                 P, P]
    lib.vmla_chunk_attention_splitkv.restype = ctypes.c_int
    return lib


lib = _load()


def vmla_status_string(code: int) -> str:
    return lib.vmla_status_string(int(code)).decode()


def vmla_last_error() -> str:
    return lib.vmla_last_error().decode()


def _check(code: int) -> None:
    if code != VMLA_OK:
        raise VmlaError(code, f"{vmla_status_string(code)}: {vmla_last_error()}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bf16, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def vmla_cache_append(x, w_dkv, w_kr, cache, slot0: int, t0: int, grid_h: int, grid_w: int,
                      stream=None) -> None:
    """x [B, n_tok, D], w_dkv [192, D], w_kr [32, D], cache [B, cap, 224] (written in place)."""
    B, n_tok, D = x.shape
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D_C + D_R:
        raise ValueError("cache must be [B, cap, 224]")
    if tuple(w_dkv.shape) != (D_C, D) or tuple(w_kr.shape) != (D_R, D):
        raise ValueError("w_dkv must be [192, D] and w_kr [32, D]")
    _check(lib.vmla_cache_append(_ptr(x, "x"), _ptr(w_dkv, "w_dkv"), _ptr(w_kr, "w_kr"), B, n_tok, D,
                                 _ptr(cache, "cache"), cache.shape[1], int(slot0), int(t0),
                                 int(grid_h), int(grid_w), _stream(stream)))


def vmla_chunk_attention(q, q_rope, w_uk, w_uv, cache, n_kv: int, t0: int, grid_h: int, grid_w: int,
                         scale: float, out, stream=None) -> None:
    """q [B, Nq, H, 128], q_rope [B, Nq, H, 32], w_uk/w_uv [H*128, 192], cache [B, cap, 224],
    out [B, Nq, H, 128]; keys are cache rows [0, n_kv)."""
    B, Nq, H, dh = q.shape
    if dh != D_HEAD or tuple(q_rope.shape) != (B, Nq, H, D_R) or tuple(out.shape) != (B, Nq, H, D_HEAD):
        raise ValueError("q/q_rope/out shapes do not match [B, Nq, H, 128|32]")
    if tuple(w_uk.shape) != (H * D_HEAD, D_C) or tuple(w_uv.shape) != (H * D_HEAD, D_C):
        raise ValueError("w_uk / w_uv must be [H*128, 192]")
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D_C + D_R:
        raise ValueError("cache must be [B, cap, 224]")
    _check(lib.vmla_chunk_attention(_ptr(q, "q"), _ptr(q_rope, "q_rope"), _ptr(w_uk, "w_uk"),
                                    _ptr(w_uv, "w_uv"), _ptr(cache, "cache"), B, Nq, H, cache.shape[1],
                                    int(n_kv), int(t0), int(grid_h), int(grid_w), float(scale),
                                    _ptr(out, "out"), _stream(stream)))


def vmla_cache_append_dc(x, w_dkv, w_kr, cache, slot0: int, t0: int, grid_h: int, grid_w: int,
                         stream=None) -> None:
    """vmla_cache_append for latent width d_c = w_dkv.shape[0] (64, 128, 192 or 256):
    w_dkv [d_c, D], cache [B, cap, d_c + 32]."""
    B, n_tok, D = x.shape
    d_c = w_dkv.shape[0]
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != d_c + D_R:
        raise ValueError("cache must be [B, cap, d_c + 32]")
    if w_dkv.shape[1] != D or tuple(w_kr.shape) != (D_R, D):
        raise ValueError("w_dkv must be [d_c, D] and w_kr [32, D]")
    _check(lib.vmla_cache_append_dc(_ptr(x, "x"), _ptr(w_dkv, "w_dkv"), _ptr(w_kr, "w_kr"), B, n_tok, D, d_c,
                                    _ptr(cache, "cache"), cache.shape[1], int(slot0), int(t0),
                                    int(grid_h), int(grid_w), _stream(stream)))


def vmla_chunk_attention_dc(q, q_rope, w_uk, w_uv, cache, n_kv: int, t0: int, grid_h: int, grid_w: int,
                            scale: float, out, stream=None) -> None:
    """vmla_chunk_attention for latent width d_c = w_uk.shape[1]: w_uk/w_uv [H*128, d_c],
    cache [B, cap, d_c + 32]."""
    B, Nq, H, dh = q.shape
    d_c = w_uk.shape[1]
    if dh != D_HEAD or tuple(q_rope.shape) != (B, Nq, H, D_R) or tuple(out.shape) != (B, Nq, H, D_HEAD):
        raise ValueError("q/q_rope/out shapes do not match [B, Nq, H, 128|32]")
    if tuple(w_uk.shape) != (H * D_HEAD, d_c) or tuple(w_uv.shape) != (H * D_HEAD, d_c):
        raise ValueError("w_uk / w_uv must be [H*128, d_c]")
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != d_c + D_R:
        raise ValueError("cache must be [B, cap, d_c + 32]")
    _check(lib.vmla_chunk_attention_dc(_ptr(q, "q"), _ptr(q_rope, "q_rope"), _ptr(w_uk, "w_uk"),
                                       _ptr(w_uv, "w_uv"), _ptr(cache, "cache"), B, Nq, H, d_c, cache.shape[1],
                                       int(n_kv), int(t0), int(grid_h), int(grid_w), float(scale),
                                       _ptr(out, "out"), _stream(stream)))


def vmla_dense_attention(q, k, v, scale: float, out, stream=None) -> None:
    """q [B, Nq, H, 128], k/v [B, Nk, H, 128], out [B, Nq, H, 128]."""
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    if tuple(k.shape) != (B, Nk, H, d) or tuple(v.shape) != (B, Nk, H, d) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q/k/v/out shapes do not match")
    _check(lib.vmla_dense_attention(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), B, Nq, Nk, H, d,
                                    float(scale), _ptr(out, "out"), _stream(stream)))


def vmla_query_projection(x, w_q, w_qr, q, q_rope, stream=None) -> None:
    """x [B, n, D] -> q [B, n, H, 128] = x W_Q^T and q_rope [B, n, H, 32] = x W_QR^T (unrotated)."""
    B, n, D = x.shape
    H = q.shape[2]
    if tuple(q.shape) != (B, n, H, D_HEAD) or tuple(q_rope.shape) != (B, n, H, D_R):
        raise ValueError("q must be [B, n, H, 128] and q_rope [B, n, H, 32]")
    if tuple(w_q.shape) != (H * D_HEAD, D) or tuple(w_qr.shape) != (H * D_R, D):
        raise ValueError("w_q must be [H*128, D] and w_qr [H*32, D]")
    _check(lib.vmla_query_projection(_ptr(x, "x"), _ptr(w_q, "w_q"), _ptr(w_qr, "w_qr"), B, n, D, H,
                                     _ptr(q, "q"), _ptr(q_rope, "q_rope"), _stream(stream)))


def vmla_output_projection(o, w_o, y, stream=None) -> None:
    """o [B, n, H, 128] -> y [B, n, D] = o W_O^T with w_o [D, H*128]."""
    B, n, H, dh = o.shape
    D = y.shape[2]
    if dh != D_HEAD or tuple(y.shape) != (B, n, D) or tuple(w_o.shape) != (D, H * D_HEAD):
        raise ValueError("o must be [B, n, H, 128], w_o [D, H*128], y [B, n, D]")
    _check(lib.vmla_output_projection(_ptr(o, "o"), _ptr(w_o, "w_o"), B, n, H, D, _ptr(y, "y"), _stream(stream)))


def _check_latent_shapes(q, q_rope, cache, out):
    B, Nq, H, dh = q.shape
    if dh != D_HEAD or tuple(q_rope.shape) != (B, Nq, H, D_R) or tuple(out.shape) != (B, Nq, H, D_HEAD):
        raise ValueError("q/q_rope/out shapes do not match [B, Nq, H, 128|32]")
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D_C + D_R:
        raise ValueError("cache must be [B, cap, 224]")
    return B, Nq, H


def vmla_materialized_kv_bytes(batch: int, heads: int, n_kv: int) -> int:
    return int(lib.vmla_materialized_kv_bytes(int(batch), int(heads), int(n_kv)))


def vmla_materialize_kv(w_uk, w_uv, cache, n_kv: int, kv, stream=None) -> None:
    """kv [B, n_kv, 2H, 128]: K_h = c . W_UK_h^T in heads [0, H), V_h = c . W_UV_h^T in [H, 2H)."""
    B, cap = cache.shape[0], cache.shape[1]
    H = w_uk.shape[0] // D_HEAD
    if tuple(kv.shape) != (B, n_kv, 2 * H, D_HEAD):
        raise ValueError("kv must be [B, n_kv, 2H, 128]")
    _check(lib.vmla_materialize_kv(_ptr(w_uk, "w_uk"), _ptr(w_uv, "w_uv"), _ptr(cache, "cache"), B, H, cap,
                                   int(n_kv), _ptr(kv, "kv"), _stream(stream)))


def vmla_chunk_attention_materialized(q, q_rope, kv, cache, n_kv: int, t0: int, grid_h: int, grid_w: int,
                                      scale: float, out, stream=None) -> None:
    B, Nq, H = _check_latent_shapes(q, q_rope, cache, out)
    if kv.dim() != 4 or kv.shape[0] != B or kv.shape[1] < n_kv or kv.shape[2] != 2 * H:
        raise ValueError("kv must be [B, n_kv, 2H, 128]")
    _check(lib.vmla_chunk_attention_materialized(_ptr(q, "q"), _ptr(q_rope, "q_rope"), _ptr(kv, "kv"),
                                                 _ptr(cache, "cache"), B, Nq, H, cache.shape[1], int(n_kv), int(t0),
                                                 int(grid_h), int(grid_w), float(scale), _ptr(out, "out"),
                                                 _stream(stream)))


def vmla_chunk_attention_nonabsorbed(q, q_rope, w_uk, w_uv, cache, n_kv: int, t0: int, grid_h: int, grid_w: int,
                                     scale: float, workspace, out, stream=None) -> None:
    """workspace: a CUDA tensor of at least vmla_materialized_kv_bytes(B, H, n_kv) bytes."""
    B, Nq, H = _check_latent_shapes(q, q_rope, cache, out)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _check(lib.vmla_chunk_attention_nonabsorbed(_ptr(q, "q"), _ptr(q_rope, "q_rope"), _ptr(w_uk, "w_uk"),
                                                _ptr(w_uv, "w_uv"), _ptr(cache, "cache"), B, Nq, H, cache.shape[1],
                                                int(n_kv), int(t0), int(grid_h), int(grid_w), float(scale),
                                                workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                                _ptr(out, "out"), _stream(stream)))


def vmla_chunk_attention_splitkv_workspace_bytes(batch: int, n_q: int, heads: int, n_kv: int) -> int:
    """Workspace bytes vmla_chunk_attention_splitkv needs on the current device (0: none)."""
    n = lib.vmla_chunk_attention_splitkv_workspace_bytes(int(batch), int(n_q), int(heads), int(n_kv))
    if n < 0:
        raise ValueError("bad sizes or no current CUDA device")
    return n


def vmla_chunk_attention_splitkv(q, q_rope, w_uk, w_uv, cache, n_kv: int, t0: int, grid_h: int, grid_w: int,
                                 scale: float, out, workspace=None, stream=None) -> None:
    """vmla_chunk_attention whose last partial wave of (sample, query tile, head) units may
    run split over key ranges.  workspace: a contiguous CUDA tensor of at least
    vmla_chunk_attention_splitkv_workspace_bytes(B, Nq, H, n_kv) bytes; when None, one of
    that size is taken from torch's allocator for this call."""
    B, Nq, H, dh = q.shape
    if dh != D_HEAD or tuple(q_rope.shape) != (B, Nq, H, D_R) or tuple(out.shape) != (B, Nq, H, D_HEAD):
        raise ValueError("q/q_rope/out shapes do not match [B, Nq, H, 128|32]")
    if tuple(w_uk.shape) != (H * D_HEAD, D_C) or tuple(w_uv.shape) != (H * D_HEAD, D_C):
        raise ValueError("w_uk / w_uv must be [H*128, 192]")
    if cache.dim() != 3 or cache.shape[0] != B or cache.shape[2] != D_C + D_R:
        raise ValueError("cache must be [B, cap, 224]")
    if workspace is None:
        need = vmla_chunk_attention_splitkv_workspace_bytes(B, Nq, H, n_kv)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _check(lib.vmla_chunk_attention_splitkv(_ptr(q, "q"), _ptr(q_rope, "q_rope"), _ptr(w_uk, "w_uk"),
                                            _ptr(w_uv, "w_uv"), _ptr(cache, "cache"), B, Nq, H, cache.shape[1],
                                            int(n_kv), int(t0), int(grid_h), int(grid_w), float(scale),
                                            workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                            _ptr(out, "out"), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 8 << 20


def vmla_chunk_attention_nonabsorbed_noalloc(q, q_rope, w_uk, w_uv, cache, n_kv: int, t0: int, grid_h: int,
                                             grid_w: int, scale: float, out, stream=None) -> None:
    """Like vmla_chunk_attention_nonabsorbed, with the library's fixed scratch instead of a
    workspace (for callers that cannot allocate device memory); calls must not overlap."""
    B, Nq, H = _check_latent_shapes(q, q_rope, cache, out)
    _check(lib.vmla_chunk_attention_nonabsorbed_noalloc(_ptr(q, "q"), _ptr(q_rope, "q_rope"), _ptr(w_uk, "w_uk"),
                                                        _ptr(w_uv, "w_uv"), _ptr(cache, "cache"), B, Nq, H,
                                                        cache.shape[1], int(n_kv), int(t0), int(grid_h),
                                                        int(grid_w), float(scale), _ptr(out, "out"),
                                                        _stream(stream)))


def vmla_get_device_status(stream=None) -> None:
    _check(lib.vmla_get_device_status(_stream(stream)))


def vmla_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(lib.vmla_selftest_wait_timeout(int(limit_ns), _stream(stream)))
