"""The two readings of the online softmax in the method's emulation (CPU only).

* Plain (the default): the reference max is the running max, so P = E4M3(p * 448) with p <= 1,
  the blockwise online softmax as the pages describe it.
* Lazy (the reading the fused CUDA kernel takes): the reference moves only when the running max
  has grown by more than tau = 2, and P = E4M3(p * 448 / 4) with p <= 4.

Both share O and l's reference, so they compute the same weighted mean of the same V codes; they
differ only in how each P value rounds to its code.  These tests pin that: with one key tile the
plain reading is the one-pass quantized softmax written out from its definition, and on any input
the two readings stay within the sum of their P-rounding bounds, element by element.
"""
import numpy as np
import pytest

import workloads as W
from oracle import attention, emulate, fp8, quant


def _weights_and_codes(qz, causal, sm_scale):
    """Exact softmax weights of the dequantized INT8 scores (float64, (Hq, N, N), masked keys 0) and
    the decoded V codes times their channel scales (Hkv, N, d)."""
    B, Hq, Hkv, N, d = qz["B"], qz["Hq"], qz["Hkv"], qz["N"], qz["d"]
    assert B == 1
    G = Hq // Hkv
    w = np.zeros((Hq, N, N))
    for h in range(Hq):
        S = qz["q8"][0, h, :N].astype(np.int64) @ qz["k8"][0, h // G, :N].astype(np.int64).T
        qs = qz["qs"][0, h, np.arange(N) // 128].astype(np.float64)
        ks = qz["ks"][0, h // G, np.arange(N) // 128].astype(np.float64)
        s = S * qs[:, None] * ks[None, :] * sm_scale
        if causal:
            s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
        e = np.exp(s - s.max(1, keepdims=True))
        w[h] = e / e.sum(1, keepdims=True)
    v8 = qz["v8"][0, :, :N, :d]
    dec = v8.astype(np.float64) if qz["pv_mode"] & 2 else fp8.decode(v8)
    return w, dec * qz["vs"][0, :, None, :d].astype(np.float64)


def _code_error(w, scale, rel, sub_abs, sub_min):
    """Largest error, in softmax-weight units, of storing weight w as a code of p * scale.

    p = w * l with l >= 1 (the row sum against a reference at most the row max), so the error of
    the code relative to l is at most: rel * w when p * scale is a normal number (>= sub_min),
    else min(w, sub_abs / scale) (a subnormal code is off by at most half its step, sub_abs, and
    by at most the value itself).  Which case applies depends on l, so take the larger."""
    return np.maximum(rel * w, np.minimum(w, sub_abs / scale))


# E4M3: 3 mantissa bits (half-step 2^-4 relative), subnormals below 2^-6 with step 2^-9.
# fp16: 10 mantissa bits (2^-11), subnormals below 2^-14 with step 2^-24.
FORMATS = {0: (2.0 ** -4, 2.0 ** -10, 2.0 ** -6), 2: (2.0 ** -11, 2.0 ** -25, 2.0 ** -14)}


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mode", [0, 2])
def test_lazy_reading_within_p_rounding_of_plain(mode, causal):
    w_ = W.TINY.with_(name="readings", N=384, Hq=2, Hkv=1, causal=causal, pv_mode=mode)
    q, k, v = W.make_inputs(w_)
    scale = W.sm_scale_of(w_)
    qz = quant.quantize(q, k, v, "HND", mode)
    plain = emulate.emulate(qz, causal, scale).astype(np.float64)[:, :w_.N]
    lazy = emulate.emulate(qz, causal, scale, **emulate.lazy_reading(mode)).astype(np.float64)[:, :w_.N]
    wts, vdec = _weights_and_codes(qz, causal, scale)
    rel, sub_abs, sub_min = FORMATS[mode]
    p_scale = (448.0, 112.0) if mode == 0 else (1.0, 1.0)
    err_w = sum(_code_error(wts, s, rel, sub_abs, sub_min) for s in p_scale)   # (Hq, N, N)
    bound = np.einsum("hij,hjc->hic", err_w, np.abs(vdec)[np.arange(w_.Hq) // (w_.Hq // w_.Hkv)]) + 1e-5
    diff = np.abs(lazy - plain)
    assert (diff <= bound).all(), f"worst excess {float((diff - bound).max()):.3g}"
    # the bound is not vacuous: the readings do differ, by much less than it
    assert diff.max() > 0 and diff.max() < 0.5 * bound.max()


def test_plain_reading_with_one_key_tile_is_the_one_pass_quantized_softmax():
    # with one 128-key tile the online softmax has a single step: the reference is the row max M
    # and out = sum_j E4M3(448 * 2^(s_j - M)) v_j / (448 * sum_j 2^(s_j - M)), written out here in
    # float64 from the codes (s in log2 units: S * qs * ks * sm_scale * log2 e)
    w_ = W.TINY.with_(name="one_tile", N=128, Hq=2, Hkv=2)
    q, k, v = W.make_inputs(w_)
    scale = W.sm_scale_of(w_)
    qz = quant.quantize(q, k, v, "HND", 0)
    got = emulate.emulate(qz, False, scale).astype(np.float64)
    for h in range(2):
        S = qz["q8"][0, h].astype(np.int64) @ qz["k8"][0, h].astype(np.int64).T
        f = (qz["qs"][0, h, 0].astype(np.float32) * qz["ks"][0, h, 0].astype(np.float32)).astype(np.float64) * \
            np.float64(np.float32(np.float32(scale) * np.float32(emulate.LOG2E)))
        s = S * f
        p = np.exp2(s - s.max(1, keepdims=True))
        P = fp8.decode(fp8.encode(448.0 * p))
        vdec = fp8.decode(qz["v8"][0, h]) * qz["vs"][0, h].astype(np.float64)
        want = (P @ vdec) / (448.0 * p.sum(1, keepdims=True))
        # the emulation rounds s and p to float32 before coding: a code can move one E4M3 step when
        # 448 p falls within float32 rounding of a midpoint, so compare all but such rare elements
        # tightly and every element within one step of one key's weight
        d = np.abs(got[h, :128, :w_.d] - want[:, :w_.d])
        assert (d <= 1e-5).mean() >= 0.999, float(d.max())
        assert d.max() <= 2.0 ** -3 * float(np.abs(vdec).max())


def test_measured_method_error_of_both_readings_on_the_tiny_workload():
    # the lazy reading's coarser P codes (scale 112 instead of 448) cost accuracy on short rows:
    # on the tiny workload (256 keys) max |emulation - exact| is 0.0238 (plain) and 0.0281 (lazy)
    q, k, v = W.make_inputs(W.TINY)
    scale = W.sm_scale_of(W.TINY)
    qz = quant.quantize(q, k, v, "HND", 0)
    ref = attention.attention_f64(q, k, v, "HND", False, scale)
    e0 = np.abs(emulate.emulate(qz, False, scale).reshape(ref.shape) - ref).max()
    e2 = np.abs(emulate.emulate(qz, False, scale, **emulate.lazy_reading(0)).reshape(ref.shape) - ref).max()
    assert abs(e0 - 0.0238) < 5e-4 and abs(e2 - 0.0281) < 5e-4, (e0, e2)
