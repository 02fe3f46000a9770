"""Fused attention on the GPU vs the oracle: the method's emulation (same codes) and exact fp64."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention, emulate, quant
from tests._support import (check_vs_emulation, check_vs_exact, cuda, nkeys, oracle_to_device, out_hnd,
                            opt_kw, pv_dtype, pv_name, slice_heads, vmax_of)

pytestmark = pytest.mark.gpu

SMALL = [
    W.TINY,
    W.TINY.with_(name="tiny_causal", causal=True),
    W.TINY.with_(name="ragged_d40_gqa_bf16", N=300, d=40, Hq=4, Hkv=2, dtype="bf16"),
    W.TINY.with_(name="single_token_d96", N=1, d=96),
    W.TINY.with_(name="nhd_koffset_fp16acc", N=700, d=128, layout="NHD", dist="normal_koffset", pv_mode=1,
                 sm_scale=None),
    W.TINY.with_(name="d256_uniform", B=2, N=129, d=256, dist="uniform2", sm_scale=None),
    W.TINY.with_(name="outlier_gqa4_causal_bf16", N=640, d=64, Hq=8, Hkv=2, dist="normal_koutlier", dtype="bf16",
                 causal=True),
    W.TINY.with_(name="d33_causal", N=257, d=33, Hq=3, Hkv=1, causal=True, sm_scale=None),
    W.TINY.with_(name="d96_causal_fp16acc", N=1000, d=96, causal=True, pv_mode=1, dist="uniform2", sm_scale=None),
    W.TINY.with_(name="d256_causal_fp16acc_nhd", N=300, d=256, causal=True, pv_mode=1, layout="NHD",
                 sm_scale=None),
    # INT8-QK / FP16-PV kernel (64-key tiles): fp32 and fp16+fp32 accumulation
    W.TINY.with_(name="pv16_tiny", pv_mode=2),
    W.TINY.with_(name="pv16acc_tiny_causal", causal=True, pv_mode=3),
    W.TINY.with_(name="pv16_ragged_d40_gqa_bf16", N=300, d=40, Hq=4, Hkv=2, dtype="bf16", pv_mode=2),
    W.TINY.with_(name="pv16_single_token_d96", N=1, d=96, pv_mode=2),
    W.TINY.with_(name="pv16acc_nhd_koffset_d128", N=700, d=128, layout="NHD", dist="normal_koffset", pv_mode=3,
                 sm_scale=None),
    W.TINY.with_(name="pv16_d256_uniform_causal", B=2, N=329, d=256, dist="uniform2", causal=True, pv_mode=2,
                 sm_scale=None),
    W.TINY.with_(name="pv16acc_d256_nhd", N=300, d=256, pv_mode=3, layout="NHD", sm_scale=None),
    W.TINY.with_(name="pv16_outlier_gqa4_causal_bf16", N=640, d=64, Hq=8, Hkv=2, dist="normal_koutlier",
                 dtype="bf16", causal=True, pv_mode=2),
    W.TINY.with_(name="pv16acc_d96_causal", N=1000, d=96, causal=True, pv_mode=3, dist="uniform2", sm_scale=None),
    # Q scale granularity and V smoothing
    W.TINY.with_(name="qgran32_causal_gqa_d64", N=640, Hq=8, Hkv=2, causal=True, q_gran=32),
    W.TINY.with_(name="qgran1_d128_nhd_bf16", N=300, d=128, layout="NHD", dtype="bf16", q_gran=1, sm_scale=None),
    W.TINY.with_(name="smoothv_koffset_d64_causal", N=700, d=64, dist="normal_koffset", causal=True, smooth_v=True),
    W.TINY.with_(name="smoothv_qgran1_pv16_d256", N=300, d=256, pv_mode=2, q_gran=1, smooth_v=True, sm_scale=None),
    W.TINY.with_(name="smoothv_qgran32_fp16acc_d96", N=513, d=96, pv_mode=1, q_gran=32, smooth_v=True,
                 sm_scale=None),
]


def _scale(w):
    return W.sm_scale_of(w)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_attention_kernel_reproduces_method(lib, w):
    """sage_attn_quantized on the oracle's own codes vs the CPU emulation of the method."""
    q, k, v = W.make_inputs(w)
    qz = quant.quantize(q, k, v, w.layout, w.pv_mode, w.q_gran, w.smooth_v)
    z = oracle_to_device(qz)
    out = lib.sage_attn_quantized(z, q.dtype, w.layout, w.causal, _scale(w), pv_name(w))
    lib.sage_check_status()
    em = emulate.emulate(qz, w.causal, _scale(w), **emulate.lazy_reading(w.pv_mode)).reshape(w.B, w.Hq, -1, w.d)
    check_vs_emulation(out_hnd(out, w.layout), em[:, :, :w.N].astype(np.float64), vmax_of(v), w.name)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_sage_attn_vs_exact_attention(lib, w):
    q, k, v = W.make_inputs(w)
    out = lib.sage_attn(cuda(q), cuda(k), cuda(v), w.layout, w.causal, _scale(w), pv_name(w), pv_dtype=pv_dtype(w),
                        **opt_kw(w))
    lib.sage_check_status()
    ref = attention.attention_f64(q, k, v, w.layout, w.causal, _scale(w))
    qz = quant.quantize(q, k, v, w.layout, w.pv_mode, w.q_gran, w.smooth_v)
    em = emulate.emulate(qz, w.causal, _scale(w), **emulate.lazy_reading(w.pv_mode)).reshape(w.B, w.Hq, -1, w.d)
    check_vs_exact(out_hnd(out, w.layout), ref, em[:, :, :w.N], nkeys(w.N, w.causal), vmax_of(v), w.name, w.dist,
                   w.pv_mode)


@pytest.mark.parametrize("w", SMALL[:6] + SMALL[10:13] + SMALL[-5:], ids=lambda w: w.name)
def test_end_to_end_equals_quantize_then_attend(lib, w):
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    a = lib.sage_attn(q, k, v, w.layout, w.causal, _scale(w), pv_name(w), pv_dtype=pv_dtype(w), **opt_kw(w))
    z = lib.sage_quantize(q, k, v, w.layout, pv_name(w), pv_dtype(w), **opt_kw(w))
    b = lib.sage_attn_quantized(z, q.dtype, w.layout, w.causal, _scale(w), pv_name(w))
    lib.sage_check_status()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_default_scale_and_no_write_past_output(lib):
    w = W.TINY.with_(name="ragged", N=200, d=72, sm_scale=None)
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    n = q.numel()
    buf = torch.full((n + 4096,), 7.0, dtype=q.dtype, device="cuda")
    out = buf[:n].view(q.shape)
    lib.sage_attn(q, k, v, "HND", False, None, out=out)          # None -> 1/sqrt(72) in float32
    ref = lib.sage_attn(q, k, v, "HND", False, float(np.float32(1.0) / np.sqrt(np.float32(72.0))))
    lib.sage_check_status()
    assert torch.equal(out, ref)
    assert bool((buf[n:] == 7.0).all())


def test_rejects_bad_inputs(lib):
    q = torch.zeros((1, 2, 64, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.SageError) as e:
        lib.sage_attn(q, q.clone(), q.clone())
    assert e.value.status == lib.SAGE_ERR_UNSUPPORTED
    h = torch.zeros((1, 3, 64, 64), dtype=torch.float16, device="cuda")
    kv = torch.zeros((1, 2, 64, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(lib.SageError) as e:
        lib.sage_attn(h, kv, kv.clone())
    assert e.value.status == lib.SAGE_ERR_INVALID_ARG


# every point of the head-dim padding sweep (N in {1K, 2K, 4K, 16K}, d in {96, 64}, both masks) at full size
FULL = [W.IMAGE_DIT, W.VIDEO_DIT, W.LLM_GQA] + list(W.pad_sweep()) + W.FP16_PV + W.OPTIONS + W.FP32_ACC + \
    W.HEAD_DIM_256


def _rows(out, layout, b, h, rows):
    t = out[b, h, rows] if layout == "HND" else out[b, rows, h]
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled_rows(lib, w):
    """The full-size launch the bench times; the oracle checks sampled heads and 128-row blocks."""
    q, k, v = W.make_inputs(w)
    out = lib.sage_attn(cuda(q), cuda(k), cuda(v), w.layout, w.causal, _scale(w), pv_name(w), pv_dtype=pv_dtype(w),
                        **opt_kw(w))
    lib.sage_check_status()
    G = w.Hq // w.Hkv
    nb = (w.N + 127) // 128
    qbs = sorted({0, 1, nb // 2, nb - 1})
    rows = np.concatenate([np.arange(i * 128, min((i + 1) * 128, w.N)) for i in qbs])
    heads = {(0, 0), (w.B - 1, w.Hq - 1)}
    if w.dist == "normal_koutlier":  # also a query head whose kv head has an outlier channel
        kf = k[0].float().abs().amax(dim=(1 if w.layout == "HND" else 0))
        hk_out = int(kf.amax(dim=-1).argmax())
        heads.add((0, hk_out * G))
    for b, hq in sorted(heads):
        hk = hq // G
        qs, ks, vs = (slice_heads(t, w.layout, b, [hh]) for t, hh in ((q, hq), (k, hk), (v, hk)))
        got = _rows(out, w.layout, b, hq, torch.as_tensor(rows))
        qz = quant.quantize(qs, ks, vs, w.layout, w.pv_mode, w.q_gran, w.smooth_v)
        em = emulate.emulate(qz, w.causal, _scale(w), heads=[(0, 0)], q_blocks=qbs, **emulate.lazy_reading(w.pv_mode))[0]
        em = np.concatenate([em[i * 128:i * 128 + min(128, w.N - qb * 128)] for i, qb in enumerate(qbs)])
        check_vs_emulation(got, em.astype(np.float64), vmax_of(vs), f"{w.name} b{b} h{hq}")
        ref = attention.attention_f64(qs, ks, vs, w.layout, w.causal, _scale(w), heads=[(0, 0)], rows=rows)[0]
        check_vs_exact(got, ref, em, nkeys(w.N, w.causal, rows), vmax_of(vs), f"{w.name} b{b} h{hq}", w.dist,
                       w.pv_mode)
