"""The fused path on inputs whose output is known in closed form (B200).

Same construction as the oracle's worked cases (tests/test_oracle_emulate_exact.py): exact INT8
codes, scores on log2-spaced levels, V exactly representable, so the output is a weighted mean
of V rows with weights 1, 1/2, 2, 1/4 (or 2^-2.5-scaled after the reference moves).  The GPU
output is compared with that weighted mean directly, not with the emulation; the tolerance is
the fp16 output rounding (2^-11 of values <= 1) plus the ex2.approx error.
"""
import numpy as np
import pytest
import torch

import quantized_attention_int8_b200 as qa
from tests.test_oracle_emulate_exact import LN2, _inputs, _weights

MODES = {0: ("fp8", "fp32"), 1: ("fp8", "fp16+fp32"), 2: ("fp16", "fp32"), 3: ("fp16", "fp16+fp32")}
FULL_LEVELS = [-1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0]
# fp16+fp32 with FP8 P.V: terms 112*v and 56*v with |v| <= 1/4 (and one 1) keep every fp16
# partial of the tile's P.V an exact even integer below 4096
SMALL_LEVELS = [-0.25, 0.0, 0.25]
CASES = [("one", [0.5], 0, [0, 1, 2, 3]), ("stay", [0.5, 1.5], 1, [0, 2, 3]), ("move", [0.5, 3.0], 2, [0, 2, 3])]


def _attn(q, k, v, mode, causal):
    pvd, acc = MODES[mode]
    return qa.sage_attn(q.cuda(), k.cuda(), v.cuda(), "HND", causal, LN2, acc, pv_dtype=pvd)


@pytest.mark.gpu
@pytest.mark.parametrize("name,deltas,seed,modes", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_closed_form_weights(name, deltas, seed, modes, mode):
    if mode not in modes:
        pytest.skip("fp16 tile partials are not exact for these weights")
    q, k, v, vnp = _inputs(deltas, SMALL_LEVELS if mode == 1 else FULL_LEVELS, seed)
    out = _attn(q, k, v, mode, False)[0, 0].float().cpu().numpy().astype(np.float64)
    w = _weights(deltas, tile=64 if mode & 2 else 128)
    want = (w[:, None] * vnp).sum(0) / w.sum()
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=1e-3)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [0, 2])
def test_closed_form_causal_prefixes(mode):
    q, k, v, vnp = _inputs([0.5], FULL_LEVELS, 0)
    out = _attn(q, k, v, mode, True)[0, 0].float().cpu().numpy().astype(np.float64)
    for i in range(128):
        w = np.where(np.arange(i + 1) < 64, 1.0, 0.5)
        want = (w[:, None] * vnp[:i + 1]).sum(0) / w.sum()
        np.testing.assert_allclose(out[i], want, rtol=0, atol=1e-3, err_msg=f"row {i}")
