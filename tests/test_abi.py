"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments before launching anything (no GPU needed: every call here fails
validation)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "videomla.h")


@pytest.fixture(scope="module")
def vm():
    import __graft_entry__
    __graft_entry__.build()
    import latent_kv_cache_b200 as vm
    return vm


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vmla_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_calls():
    names = _declared()
    for n in ("vmla_cache_append", "vmla_chunk_attention", "vmla_dense_attention",
              "vmla_get_device_status", "vmla_status_string", "vmla_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(vm):
    lib = ctypes.CDLL(vm.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n


def test_status_strings(vm):
    assert vm.vmla_status_string(0) == "VMLA_OK"
    assert vm.vmla_status_string(4) == "VMLA_ERR_TIMEOUT"
    assert vm.vmla_status_string(99) == "VMLA_ERR_UNKNOWN"


A = 0x10000  # 16-byte aligned fake address; never dereferenced (validation fails first)


def test_append_validation(vm):
    L = vm.lib
    assert L.vmla_cache_append(None, A, A, 1, 10, 1536, A, 100, 0, 0, 8, 8, None) == 1
    assert L.vmla_cache_append(A + 2, A, A, 1, 10, 1536, A, 100, 0, 0, 8, 8, None) == 1  # misaligned
    assert L.vmla_cache_append(A, A, A, 1, 10, 1500, A, 100, 0, 0, 8, 8, None) == 2      # d_model
    assert L.vmla_cache_append(A, A, A, 1, 10, 1536, A, 5, 0, 0, 8, 8, None) == 1        # n_tok > cap
    assert L.vmla_cache_append(A, A, A, 1, 10, 1536, A, 100, 100, 0, 8, 8, None) == 1    # slot0
    assert L.vmla_cache_append(A, A, A, 1, 10, 1536, A, 100, 0, 0, 0, 8, None) == 1      # grid
    assert L.vmla_cache_append(A, A, A, 1, 10, 1536, A, 100, 0, 0, 300, 8, None) == 2    # grid > 256
    assert L.vmla_cache_append(A, A, A, 1, 40, 1536, A, 100, 0, 0, 1, 1, None) == 2      # > 32 frames
    assert L.vmla_cache_append(A, A, A, 0, 10, 1536, A, 100, 0, 0, 8, 8, None) == 1      # batch
    assert "slot0" in vm.vmla_last_error() or "frames" in vm.vmla_last_error() or vm.vmla_last_error()


def test_attention_validation(vm):
    L = vm.lib
    f = ctypes.c_float
    assert L.vmla_chunk_attention(A, A, A, A, None, 1, 192, 12, 576, 576, 6, 8, 8, f(0.1), A, None) == 1
    assert L.vmla_chunk_attention(A, A, A, A, A, 1, 192, 12, 576, 577, 6, 8, 8, f(0.1), A, None) == 1
    assert L.vmla_chunk_attention(A, A, A, A, A, 1, 192, 12, 576, 0, 6, 8, 8, f(0.1), A, None) == 1
    assert L.vmla_chunk_attention(A, A, A, A, A, 1, 192, 12, 576, 576, 6, 8, 8, f(0.0), A, None) == 1
    assert L.vmla_chunk_attention(A, A, A, A, A, 1, 192, 12, 576, 576, 6, 8, 8, f(float("nan")), A, None) == 1
    assert L.vmla_chunk_attention(A, A, A, A, A, 1, 0, 12, 576, 576, 6, 8, 8, f(0.1), A, None) == 1
    assert L.vmla_chunk_attention(A, A, A, A, A, 1, 192, 12, 576, 576, -1, 8, 8, f(0.1), A, None) == 1
    assert L.vmla_chunk_attention(A, A, A, A, A, 1, 4000, 12, 5000, 576, 0, 2, 2, f(0.1), A, None) == 2
    assert L.vmla_dense_attention(A, A, A, 1, 192, 576, 12, 64, f(0.1), A, None) == 2
    assert L.vmla_dense_attention(A, None, A, 1, 192, 576, 12, 128, f(0.1), A, None) == 1
    assert L.vmla_dense_attention(A, A, A, 1, 192, 0, 12, 128, f(0.1), A, None) == 1
    assert L.vmla_selftest_wait_timeout(10, None) == 1


def test_latent_width_validation(vm):
    L = vm.lib
    f = ctypes.c_float
    assert L.vmla_cache_append_dc(A, A, A, 1, 10, 1536, 96, A, 100, 0, 0, 8, 8, None) == 2       # d_c
    assert L.vmla_cache_append_dc(A, A, A, 1, 10, 1536, 320, A, 100, 0, 0, 8, 8, None) == 2      # d_c
    assert "d_c" in vm.vmla_last_error()
    assert L.vmla_cache_append_dc(A, A, A, 1, 10, 1500, 64, A, 100, 0, 0, 8, 8, None) == 2       # d_model
    assert L.vmla_chunk_attention_dc(A, A, A, A, A, 1, 192, 12, 160, 576, 576, 6, 8, 8, f(0.1), A, None) == 2
    assert "d_c" in vm.vmla_last_error()
    assert L.vmla_chunk_attention_dc(A, A, A, A, None, 1, 192, 12, 64, 576, 576, 6, 8, 8, f(0.1), A, None) == 1


def test_projection_validation(vm):
    L = vm.lib
    assert L.vmla_query_projection(A, A, A, 1, 192, 1536, 12, A, None, None) == 1
    assert L.vmla_query_projection(A, A, A + 8, 1, 192, 1536, 12, A, A, None) == 1   # misaligned
    assert L.vmla_query_projection(A, A, A, 0, 192, 1536, 12, A, A, None) == 1       # batch
    assert L.vmla_query_projection(A, A, A, 1, 192, 1500, 12, A, A, None) == 2       # d_model % 64
    assert L.vmla_query_projection(A, A, A, 1, 192, 1536, 0, A, A, None) == 1        # heads
    assert L.vmla_output_projection(A, A, 1, 192, 12, 1536, None, None) == 1
    assert L.vmla_output_projection(A, A, 1, 0, 12, 1536, A, None) == 1              # n_tok
    assert L.vmla_output_projection(A, A, 1, 192, 12, 1600, A, None) == 2            # d_model % 128
    assert "d_model" in vm.vmla_last_error()


def test_binding_rejects_non_cuda_tensors(vm):
    import torch
    x = torch.zeros(1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises((TypeError, ValueError)):
        vm.vmla_cache_append(x, torch.zeros(192, 64, dtype=torch.bfloat16),
                             torch.zeros(32, 64, dtype=torch.bfloat16),
                             torch.zeros(1, 8, 224, dtype=torch.bfloat16), 0, 0, 2, 2)


def test_materialized_kv_bytes_overflow_is_rejected(vm):
    # batch 65535 x 512 heads x (2^31 - 1) keys x 512 bytes does not fit in int64:
    # the size query returns 0 and both non-absorbed forms refuse before any launch.
    L = vm.lib
    f = ctypes.c_float
    big = (1 << 31) - 1
    assert L.vmla_materialized_kv_bytes(65535, 512, big) == 0
    assert L.vmla_materialized_kv_bytes(1, 12, 32760) == 32760 * 2 * 12 * 128 * 2
    assert L.vmla_chunk_attention_nonabsorbed(A, A, A, A, A, 65535, 192, 512, big, big, 0, 8, 8, f(0.1), A,
                                              1 << 62, A, None) == 2
    assert "overflow" in vm.vmla_last_error()
    assert L.vmla_chunk_attention_nonabsorbed_noalloc(A, A, A, A, A, 65535, 192, 512, big, big, 0, 8, 8, f(0.1),
                                                      A, None) == 2
    assert "overflow" in vm.vmla_last_error()


def test_splitkv_validation(vm):
    L = vm.lib
    f = ctypes.c_float
    assert L.vmla_chunk_attention_splitkv_workspace_bytes(0, 192, 12, 576) == -1
    assert L.vmla_chunk_attention_splitkv_workspace_bytes(1, 192, 600, 576) == -1
    assert L.vmla_chunk_attention_splitkv_workspace_bytes(1, 192, 12, 0) == -1
    assert L.vmla_chunk_attention_splitkv(A, A, A, A, None, 1, 192, 12, 576, 576, 6, 8, 8, f(0.1), A, 1 << 20, A,
                                          None) == 1
    assert L.vmla_chunk_attention_splitkv(A, A, A, A, A, 1, 192, 12, 576, 577, 6, 8, 8, f(0.1), A, 1 << 20, A,
                                          None) == 1
    assert L.vmla_chunk_attention_splitkv(A, A, A, A, A, 1, 192, 12, 576, 576, 6, 8, 8, f(0.0), A, 1 << 20, A,
                                          None) == 1
