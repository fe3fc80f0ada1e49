"""The C ABI called from plain C: a small C program (tests/c/vmla_c_caller.c),
linked against libvideomla.so and the CUDA runtime only, appends a window,
runs the latent and the dense attention, and writes its outputs to files; they
are compared here with the oracle (append bit-exact, attention within the
tolerance).  No Python or PyTorch is in that process."""
from __future__ import annotations

import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import workload
from helpers import SCALE, assert_close

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "latent_kv_cache_b200")
CUDA = "/usr/local/cuda"


def _build(tmp):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    exe = os.path.join(tmp, "vmla_c_caller")
    cmd = [gcc, "-O2", "-std=c11", "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c", "vmla_c_caller.c"), "-o", exe,
           "-L", PKG, "-lvideomla", f"-Wl,-rpath,{PKG}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.parametrize("ragged", [False, True])
def test_c_caller_matches_oracle(tmp_path, ragged):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import latent_kv_cache_b200  # noqa: F401  (builds nothing; fails loudly if the library is missing)
    w = workload.CONFIGS["tiny"]
    if ragged:
        w = w.with_(grid_h=7, grid_w=9, cached_frames=4, heads=3, batch=2, seed=57)
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    kv = workload.batch_dense_kv(w)
    d = str(tmp_path)
    with open(os.path.join(d, "meta.txt"), "w") as f:
        f.write(f"{w.batch} {w.n_q} {w.n_kv} {w.heads} {w.d_model} {w.chunk_t0} {w.grid_h} {w.grid_w} {SCALE!r}\n")
    for name, arr in (("x", act["x"]), ("w_dkv", wts["w_dkv"]), ("w_kr", wts["w_kr"]), ("q", act["q"]),
                      ("q_rope", act["q_rope"]), ("w_uk", wts["w_uk"]), ("w_uv", wts["w_uv"]),
                      ("k", kv["k"]), ("v", kv["v"])):
        np.ascontiguousarray(arr, dtype=np.uint16).tofile(os.path.join(d, name + ".bin"))
    exe = _build(d)
    r = subprocess.run([exe, d], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr

    shape_out = (w.batch, w.n_q, w.heads, 128)
    cache = np.fromfile(os.path.join(d, "cache.bin"), dtype=np.uint16).reshape(w.batch, w.n_kv, 224)
    ref_cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    assert np.array_equal(cache, ref_cache)

    out = oracle.decode_bf16(np.fromfile(os.path.join(d, "out.bin"), dtype=np.uint16).reshape(shape_out))
    ref = oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], ref_cache, w.n_kv,
                                 w.chunk_t0, w.grid_h, w.grid_w, SCALE)
    assert_close(out, ref, "C caller, latent attention")

    out_d = oracle.decode_bf16(np.fromfile(os.path.join(d, "out_dense.bin"), dtype=np.uint16).reshape(shape_out))
    ref_d = oracle.dense_attention(act["q"], kv["k"], kv["v"], SCALE)
    assert_close(out_d, ref_d, "C caller, dense attention")
