"""GPU quantize/smooth pass vs the oracle's emulation: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import quant
from tests._support import cuda, opt_kw, pv_dtype, pv_name, slice_heads

pytestmark = pytest.mark.gpu

SMALL = [
    W.TINY,
    W.TINY.with_(name="ragged_d40_gqa_bf16", N=300, d=40, Hq=4, Hkv=2, dtype="bf16"),
    W.TINY.with_(name="single_token_d96", N=1, d=96),
    W.TINY.with_(name="nhd_koffset_fp16acc", N=700, d=128, layout="NHD", dist="normal_koffset", pv_mode=1),
    W.TINY.with_(name="d256_uniform", B=2, N=129, d=256, dist="uniform2"),
    W.TINY.with_(name="outlier_gqa4", N=640, d=64, Hq=8, Hkv=2, dist="normal_koutlier", dtype="bf16"),
    W.TINY.with_(name="d33_causal", N=257, d=33, Hq=3, Hkv=1, causal=True),
    W.TINY.with_(name="pv16_ragged_d40_gqa_bf16", N=300, d=40, Hq=4, Hkv=2, dtype="bf16", pv_mode=2),
    W.TINY.with_(name="pv16acc_nhd_koffset_d128", N=700, d=128, layout="NHD", dist="normal_koffset", pv_mode=3),
    W.TINY.with_(name="pv16_d256_outlier", B=2, N=129, d=256, dist="normal_koutlier", pv_mode=2),
    # Q scale granularity and V smoothing
    W.TINY.with_(name="qgran32_ragged_d40_gqa_bf16", N=300, d=40, Hq=4, Hkv=2, dtype="bf16", q_gran=32),
    W.TINY.with_(name="qgran1_d128_nhd", N=257, d=128, layout="NHD", q_gran=1),
    W.TINY.with_(name="qgran1_d256_smoothv", B=2, N=129, d=256, q_gran=1, smooth_v=True),
    W.TINY.with_(name="smoothv_koffset_d64", N=700, d=64, dist="normal_koffset", smooth_v=True),
    W.TINY.with_(name="smoothv_pv16acc_d96_ragged", N=333, d=96, pv_mode=3, smooth_v=True, q_gran=32),
    W.TINY.with_(name="smoothv_fp16acc_d33", N=257, d=33, Hq=3, Hkv=1, pv_mode=1, smooth_v=True),
]


def _gpu_codes(lib, w, q, k, v):
    z = lib.sage_quantize(cuda(q), cuda(k), cuda(v), w.layout, pv_name(w), pv_dtype(w), **opt_kw(w))
    lib.sage_check_status()
    out = {k2: z[k2].cpu().numpy() for k2 in ("q8", "qs", "k8", "ks", "km", "vs", "vm")}
    out["v8"] = z["v8t"].cpu().numpy().transpose(0, 1, 3, 2)
    return out


def _assert_same(got, ref, q_sel=slice(None), kv_sel=slice(None)):
    for key in ("q8", "qs"):
        assert np.array_equal(got[key][q_sel], ref[key]), key
    for key in ("k8", "ks", "km", "v8", "vs", "vm"):
        g, r = got[key][kv_sel], ref[key]
        if g.dtype == np.float32:
            ok = np.array_equal(g.view(np.uint32), r.view(np.uint32))
        elif g.dtype == np.float16:  # fp16 V codes, compared bit for bit
            ok = r.dtype == np.float16 and np.array_equal(g.view(np.uint16), r.view(np.uint16))
        else:
            ok = np.array_equal(g, r)
        if not ok:
            bad = np.argwhere(g != r)
            raise AssertionError(f"{key}: {len(bad)} mismatches, first at {bad[:3].tolist()}")


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_quantize_bit_exact_small(lib, w):
    q, k, v = W.make_inputs(w)
    got = _gpu_codes(lib, w, q, k, v)
    ref = quant.quantize(q, k, v, w.layout, w.pv_mode, w.q_gran, w.smooth_v)
    _assert_same(got, ref)


FULL = [W.IMAGE_DIT, W.VIDEO_DIT, W.LLM_GQA, W.BY_NAME["pad_sweep_b8_h16_n16384_d96_causal"], W.FP16_PV[1],
        # more than four waves of 128-token blocks: CTAs walk several blocks (ragged last block),
        # with the next tile prefetched (16-byte rows) or loaded synchronously (d = 33)
        W.TINY.with_(name="multiblock_prefetch_ragged_d64", B=4, Hq=8, Hkv=8, N=16381, d=64),
        W.TINY.with_(name="multiblock_sync_d33_nhd_smoothv", B=4, Hq=8, Hkv=8, N=16300, d=33, layout="NHD",
                     smooth_v=True, q_gran=32)]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_quantize_bit_exact_full_size_sampled_heads(lib, w):
    """Full-size launch on the GPU; the oracle recomputes two sampled (batch, kv-head) groups."""
    q, k, v = W.make_inputs(w)
    got = _gpu_codes(lib, w, q, k, v)
    G = w.Hq // w.Hkv
    for b, hk in {(0, 0), (w.B - 1, w.Hkv - 1)}:
        hq = list(range(hk * G, (hk + 1) * G))
        ref = quant.quantize(slice_heads(q, w.layout, b, hq), slice_heads(k, w.layout, b, [hk]),
                             slice_heads(v, w.layout, b, [hk]), w.layout, w.pv_mode, w.q_gran, w.smooth_v)
        _assert_same(got, ref, q_sel=(slice(b, b + 1), slice(hk * G, (hk + 1) * G)),
                     kv_sel=(slice(b, b + 1), slice(hk, hk + 1)))


def test_k_mean_follows_the_header_contract(lib):
    """km from sage_quantize through the C ABI, against the summation order include/sage.h states,
    written out here in plain Python float32 arithmetic on a ragged N (the last block holds 45 tokens,
    so its last groups are partial or empty): groups of 16 tokens summed in order from +0.0, the
    pairwise tree over a block's 8 groups, the block partials in block order, one division by N."""
    w = W.TINY.with_(name="km_contract", N=300, d=40, Hq=2, Hkv=1, dist="normal_koffset")
    q, k, v = W.make_inputs(w)
    z = lib.sage_quantize(cuda(q), cuda(k), cuda(v), w.layout, "fp32")
    lib.sage_check_status()
    got = z["km"].cpu().numpy()[0, 0, :w.d]
    f32 = np.float32
    kk = k[0, 0].float().numpy()  # (N, d), exact widening of the fp16 inputs
    for c in range(w.d):
        total = f32(0.0)
        for b0 in range(0, w.N, 128):
            g = []
            for g0 in range(b0, b0 + 128, 16):
                acc = f32(0.0)
                for n in range(g0, min(g0 + 16, w.N)):
                    acc = f32(acc + f32(kk[n, c]))
                g.append(acc)
            part = f32(f32(f32(g[0] + g[1]) + f32(g[2] + g[3])) + f32(f32(g[4] + g[5]) + f32(g[6] + g[7])))
            total = f32(total + part)
        want = f32(total / f32(w.N))
        assert got[c].view(np.uint32) == np.asarray(want).view(np.uint32), (c, got[c], want)
