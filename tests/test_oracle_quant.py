"""Pins for the oracle's quantization emulation (CPU only).

Each check ties the emulation to something other than itself: the fp64
mean, the rounding bound of a symmetric INT8 code, exact integer
arithmetic done by brute force, or an exactly representable construction.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import fp8, quant

F32 = np.float32


def _rng(seed):
    return np.random.default_rng(seed)


def test_padded_dim():
    assert [quant.padded_dim(d) for d in (1, 64, 65, 96, 128, 129, 256)] == [64, 64, 128, 128, 128, 256, 256]
    with pytest.raises(ValueError):
        quant.padded_dim(257)


def test_k_mean_close_to_fp64_mean():
    # float32 summation of n terms in any order is within n * 2^-24 * sum|k| of the exact sum.
    k = (_rng(0).standard_normal((2, 3, 300, 40)) * 2 + 5).astype(F32)
    km = quant.k_token_mean(k)
    exact = k.astype(np.float64).mean(axis=2)
    bound = (300 + 3) * 2.0 ** -24 * np.abs(k.astype(np.float64)).sum(axis=2) / 300 + np.abs(exact) * 2.0 ** -23
    assert np.all(np.abs(km - exact) <= bound)


def test_k_mean_exact_when_sums_are_exact():
    # Small integers with N a power of two: every partial sum and the division are exact.
    k = _rng(1).integers(-50, 50, size=(1, 2, 512, 8)).astype(F32)
    assert np.array_equal(quant.k_token_mean(k), (k.astype(np.int64).sum(axis=2) / 512).astype(F32))


def test_k_mean_order_ragged_tail():
    # Brute-force the stated order with numpy float32 scalars (each + rounds to float32):
    # 16-token groups summed in order, a pairwise tree over the 8 groups of a block,
    # then the blocks in order.
    k = (_rng(2).standard_normal((1, 1, 300, 3)) * 1000).astype(F32)
    for c in range(3):
        total = F32(0)
        for b0 in range(0, 300, 128):
            g = []
            for g0 in range(b0, b0 + 128, 16):
                acc = F32(0)
                for n in range(g0, min(g0 + 16, 300)):
                    acc = F32(acc + k[0, 0, n, c])
                g.append(acc)
            part = F32(F32(F32(g[0] + g[1]) + F32(g[2] + g[3])) + F32(F32(g[4] + g[5]) + F32(g[6] + g[7])))
            total = F32(total + part)
        assert quant.k_token_mean(k)[0, 0, c] == F32(total / F32(300))


def test_int8_codes_bounds_and_extremes():
    x = (_rng(3).standard_normal((2, 2, 300, 40)) * 3).astype(F32)
    codes, scale = quant.int8_per_block(x, 64)
    assert codes.shape == (2, 2, 384, 64) and scale.shape == (2, 2, 3)
    assert np.all(codes[:, :, 300:] == 0) and np.all(codes[:, :, :, 40:] == 0)
    for b in range(3):
        blk = x[:, :, b * 128:(b + 1) * 128]
        cb = codes[:, :, b * 128:b * 128 + blk.shape[2], :40].astype(np.float64)
        s = scale[:, :, b].astype(np.float64)[:, :, None, None]
        # reconstruction error at most half a step (plus float32 slack)
        assert np.all(np.abs(cb * s - blk) <= s * (0.5 + 1e-5))
        # the element of largest magnitude maps to +-127
        amax = np.abs(blk).max(axis=(2, 3))
        assert np.allclose(scale[:, :, b], amax / 127, rtol=1e-7)
        assert np.all(np.abs(cb).max(axis=(2, 3)) == 127)


def test_int8_ties_to_even_and_zero_block():
    x = np.zeros((1, 1, 128, 64), F32)
    x[0, 0, 0, 0] = 127.0            # amax 127 -> inv 1 -> codes equal x exactly
    x[0, 0, 1, 0] = 2.5
    x[0, 0, 2, 0] = 3.5
    x[0, 0, 3, 0] = -2.5
    codes, scale = quant.int8_per_block(x, 64)
    assert scale[0, 0, 0] == 1.0
    assert list(codes[0, 0, :4, 0]) == [127, 2, 4, -2]
    z, zs = quant.int8_per_block(np.zeros((1, 1, 10, 8), F32), 64)
    assert zs[0, 0, 0] == 0 and not z.any()


def test_smoothing_removes_channel_offset_exactly():
    # Integer-valued K and a per-channel integer offset: the mean is exact,
    # so K and K + offset must give identical codes and scales.
    rng = _rng(4)
    k = rng.integers(-20, 20, size=(1, 2, 256, 16)).astype(np.float32)
    off = rng.integers(-100, 100, size=16).astype(np.float32)
    q = rng.standard_normal((1, 2, 256, 16)).astype(np.float32)
    a = quant.quantize(q, k, q, "HND")
    b = quant.quantize(q, k + off, q, "HND")
    assert np.array_equal(a["k8"], b["k8"]) and np.array_equal(a["ks"], b["ks"])
    assert np.allclose(b["km"][0, :, :16] - a["km"][0, :, :16], off)


def test_v_fp8_per_channel():
    v = (_rng(5).standard_normal((1, 2, 200, 20)) * 2).astype(F32)
    for mode, vmax, top in ((0, 448.0, 0x7E), (1, 1.0, 0x38)):
        codes, scale = quant.fp8_per_channel(v, 64, vmax)
        dec = fp8.decode(codes).astype(np.float64)
        assert np.allclose(scale[:, :, :20], np.abs(v).max(axis=2) / vmax, rtol=1e-7)
        assert np.all(scale[:, :, 20:] == 0) and np.all(codes[:, :, :, 20:] == 0)
        assert np.all(codes[:, :, 200:] == 0)
        rec = dec[:, :, :200, :20] * scale[:, :, None, :20]
        # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 in the normal range,
        # absolute error <= 2^-10 * scale in the subnormal range.
        err = np.abs(rec - v)
        assert np.all(err <= np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10 * scale[:, :, None, :20]) * (1 + 1e-6))
        mx = (codes[:, :, :200, :20] & 0x7F).max(axis=2)
        assert np.all(mx == top)


def test_qk_int32_brute_force():
    rng = _rng(6)
    a = rng.integers(-127, 128, size=(5, 7)).astype(np.int8)
    b = rng.integers(-127, 128, size=(4, 7)).astype(np.int8)
    s = quant.qk_int32(a, b)
    for i in range(5):
        for j in range(4):
            assert s[i, j] == sum(int(a[i, c]) * int(b[j, c]) for c in range(7))
    big = np.full((2, 256), 127, np.int8)
    assert quant.qk_int32(big, -big)[0, 0] == -256 * 127 * 127


def test_dequantized_scores_track_exact_scores():
    w = W.TINY
    q, k, v = W.make_inputs(w)
    qz = quant.quantize(q, k, v, w.layout)
    qf, kf = quant.to_hnd(q, "HND").astype(np.float64), quant.to_hnd(k, "HND").astype(np.float64)
    ks_mean = kf - kf.mean(axis=2, keepdims=True)
    for h in range(2):
        S = quant.qk_int32(qz["q8"][0, h], qz["k8"][0, h]).astype(np.float64)
        deq = S * np.repeat(qz["qs"][0, h], 128)[:, None] * np.repeat(qz["ks"][0, h], 128)[None, :]
        exact = qf[0, h] @ ks_mean[0, h].T
        # each code is off by at most half a step: |dS| <= sum_c (|q| dk + |k| dq + dq dk)
        dq = np.repeat(qz["qs"][0, h], 128)[:, None] / 2
        dk = np.repeat(qz["ks"][0, h], 128)[None, :] / 2
        bound = (np.abs(qf[0, h]).sum(1)[:, None] * dk + np.abs(ks_mean[0, h]).sum(1)[None, :] * dq
                 + 64 * dq * dk) * (1 + 1e-4) + 1e-3
        assert np.all(np.abs(deq - exact) <= bound)


def test_quantize_layouts_agree():
    w = W.TINY.with_(N=200, d=40, Hq=4, Hkv=2)
    q, k, v = W.make_inputs(w)
    a = quant.quantize(q, k, v, "HND")
    b = quant.quantize(q.transpose(1, 2).contiguous(), k.transpose(1, 2).contiguous(),
                       v.transpose(1, 2).contiguous(), "NHD")
    for key in ("q8", "qs", "k8", "ks", "km", "v8", "vs"):
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("rows", [32, 1])
def test_int8_finer_granularity_brute_force(rows):
    # one scale per `rows` tokens: brute force per group with python max / division
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((1, 2, 70, 5)) * np.exp(rng.uniform(-3, 3, (1, 2, 70, 1)))).astype(np.float32)
    codes, scale = quant.int8_per_block(x, 64, rows)
    assert codes.shape == (1, 2, 128, 64) and scale.shape == (1, 2, 128 // rows)
    for h in range(2):
        for g in range(128 // rows):
            blk = x[0, h, g * rows:(g + 1) * rows]
            am = float(np.max(np.abs(blk))) if blk.size else 0.0
            assert scale[0, h, g] == np.float32(np.float32(am) / np.float32(127.0))
            if am > 0:
                inv = np.float32(np.float32(127.0) / np.float32(am))
                ref = np.clip(np.rint((blk * inv).astype(np.float32)), -127, 127)
                assert np.array_equal(codes[0, h, g * rows:g * rows + len(blk), :5], ref)
    # the 128-token default is the same function
    c128, s128 = quant.int8_per_block(x, 64)
    c128b, s128b = quant.int8_per_block(x, 64, 128)
    assert np.array_equal(c128, c128b) and np.array_equal(s128, s128b)


def test_quantize_options_validate_and_record():
    w = W.TINY.with_(N=40, d=16)
    q, k, v = W.make_inputs(w)
    qz = quant.quantize(q, k, v, "HND", 0, q_gran=32, smooth_v=True)
    assert qz["qs"].shape == (1, 2, 4) and qz["q_gran"] == 32 and qz["smooth_v"]
    # the V mean is the same fixed-order mean as K's, and V - mean is what gets coded
    vm = quant.k_token_mean(quant.to_hnd(v, "HND"))
    assert np.array_equal(qz["vm"][:, :, :16], vm) and np.all(qz["vm"][:, :, 16:] == 0)
    ref = quant.quantize(q, k, (v.float() - torch.from_numpy(vm)[:, :, None, :]).numpy(), "HND", 0)
    assert np.array_equal(qz["v8"], ref["v8"]) and np.array_equal(qz["vs"], ref["vs"])
    with pytest.raises(ValueError):
        quant.quantize(q, k, v, "HND", 0, q_gran=64)
