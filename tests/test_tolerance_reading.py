"""How far a bf16 operand of the score product alone moves the attention output.

The method (VideoMLA abstract and summary "Approach") computes attention over
keys derived from the shared latent: in the absorbed form the score is
(q_h W_UK_h) . c, in the non-absorbed form q_h . (c W_UK_h^T).  On tensor cores
one factor of that product is a bf16 operand formed from an fp32 result (q_abs
or K_h), so it carries one bf16 rounding (relative 2^-9) that the fp64 oracle
does not.  These CPU tests take the oracle's own fp64 arithmetic, round only
that one operand to bf16 and keep every other step in fp64, and measure the
output error on the small workload:

  * at the workload's query scale both forms stay far inside the stated
    tolerance (relative L2 <= 1e-2, max-abs <= 3e-2);
  * with queries x8 (scores ~8x larger, a near one-hot softmax) both forms
    exceed max-abs 3e-2 while keeping relative L2 within 1e-2.

So the x8 case's max-abs excess belongs to bf16 score operands as such, not to
one kernel: the GPU tests hold the x8 case to relative L2 <= 1e-2 and max-abs
<= 8e-2 for every form, and check that the latent kernel's error there is no
larger than the non-absorbed and dense forms' on the same inputs.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workload
from helpers import SCALE, errors


def _bf16(a64: np.ndarray) -> np.ndarray:
    return oracle.decode_bf16(workload.bf16_bits(np.asarray(a64, dtype=np.float32)))


@pytest.fixture(scope="module")
def case():
    w = workload.CONFIGS["tiny"]
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache = oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)
    return w, wts, act, cache


def _scaled(bits, mult):
    return workload.bf16_bits(workload.bf16_to_f32(bits) * np.float32(mult))


def _one_operand_rounded(w, wts, act, cache, mult, form):
    """Attention in fp64 except for one bf16 rounding of the score operand built
    from the latent: q_abs = q_h W_UK_h ("absorbed") or K_h = c W_UK_h^T ("keys")."""
    q = oracle.decode_bf16(_scaled(act["q"], mult))[0]
    qr_bits = _scaled(act["q_rope"], mult)
    qr = oracle.decode_bf16(qr_bits)[0]
    wuk = oracle.decode_bf16(wts["w_uk"]).reshape(w.heads, 128, w.d_c)
    wuv = oracle.decode_bf16(wts["w_uv"]).reshape(w.heads, 128, w.d_c)
    cc = oracle.decode_bf16(cache)[0, :w.n_kv]
    c, kr = cc[:, :w.d_c], cc[:, w.d_c:]
    t, row, col = oracle.token_positions(w.n_q, w.chunk_t0, w.grid_h, w.grid_w)
    out = np.empty((w.n_q, w.heads, 128))
    for h in range(w.heads):
        rope = oracle.rope3d(qr[:, h], t, row, col) @ kr.T
        if form == "absorbed":
            s = _bf16(q[:, h] @ wuk[h]) @ c.T + rope
        else:
            s = q[:, h] @ _bf16(c @ wuk[h].T).T + rope
        s = SCALE * s
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        out[:, h] = (p @ c) @ wuv[h].T
    ref = oracle.chunk_attention(_scaled(act["q"], mult), qr_bits, wts["w_uk"], wts["w_uv"], cache, w.n_kv,
                                 w.chunk_t0, w.grid_h, w.grid_w, SCALE)[0]
    return errors(out, ref)


@pytest.mark.parametrize("form", ["absorbed", "keys"])
def test_workload_scale_is_well_inside_the_tolerance(case, form):
    rel, mx = _one_operand_rounded(*case, 1.0, form)
    assert rel <= 5e-3 and mx <= 1e-2, (rel, mx)


@pytest.mark.parametrize("form", ["absorbed", "keys"])
def test_queries_x8_exceed_max_abs_with_one_rounded_operand(case, form):
    rel, mx = _one_operand_rounded(*case, 8.0, form)
    assert rel <= 1e-2, rel
    assert 3e-2 < mx <= 8e-2, mx


def test_unrounded_arithmetic_matches_the_oracle(case):
    # Control: the same code with no rounding reproduces the oracle, so the
    # errors above come from the one rounded operand alone.
    w, wts, act, cache = case
    q = oracle.decode_bf16(_scaled(act["q"], 8.0))[0]
    qr_bits = _scaled(act["q_rope"], 8.0)
    qr = oracle.decode_bf16(qr_bits)[0]
    wuk = oracle.decode_bf16(wts["w_uk"]).reshape(w.heads, 128, w.d_c)
    wuv = oracle.decode_bf16(wts["w_uv"]).reshape(w.heads, 128, w.d_c)
    cc = oracle.decode_bf16(cache)[0, :w.n_kv]
    c, kr = cc[:, :w.d_c], cc[:, w.d_c:]
    t, row, col = oracle.token_positions(w.n_q, w.chunk_t0, w.grid_h, w.grid_w)
    ref = oracle.chunk_attention(_scaled(act["q"], 8.0), qr_bits, wts["w_uk"], wts["w_uv"], cache, w.n_kv,
                                 w.chunk_t0, w.grid_h, w.grid_w, SCALE)[0]
    for h in range(w.heads):
        s = SCALE * ((q[:, h] @ wuk[h]) @ c.T + oracle.rope3d(qr[:, h], t, row, col) @ kr.T)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        np.testing.assert_allclose((p @ c) @ wuv[h].T, ref[:, h], rtol=0, atol=1e-9)
