"""Different query / key lengths and packed (varlen) batches on the GPU vs the oracle.

Queries and keys of different lengths go through ``sage_attn`` (-> sage_attn_ex) with the causal
mask aligned bottom-right; packed batches through ``sage_attn_varlen``.  Each sequence of a packed
batch is checked against the oracle's emulation of that sequence alone (same codes: the GPU
quantizes every sequence on its own) and against exact fp64 attention.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention, emulate, quant
from tests._support import check_vs_emulation, check_vs_exact, cuda, out_hnd, pv_dtype, pv_name, vmax_of

pytestmark = pytest.mark.gpu


def _nkeys(nq, nk, causal, rows=None):
    r = np.arange(nq) if rows is None else np.asarray(rows)
    return np.clip(r + nk - nq + 1, 0, nk) if causal else np.full(len(r), nk)


RECT = [
    W.TINY.with_(name="nq200_nk700_causal_d64", N=200, Nk=700, causal=True),
    W.TINY.with_(name="nq700_nk300_causal_nhd_bf16_d128_fp16acc", N=700, Nk=300, d=128, causal=True, layout="NHD",
                 dtype="bf16", pv_mode=1, sm_scale=None),
    W.TINY.with_(name="nq1_nk1000_causal_d96", N=1, Nk=1000, d=96, causal=True, sm_scale=None),
    W.TINY.with_(name="nq300_nk129_d256_pv16", N=300, Nk=129, d=256, pv_mode=2, sm_scale=None),
    W.TINY.with_(name="nq513_nk100_causal_gqa_d40_pv16", N=513, Nk=100, d=40, Hq=4, Hkv=2, causal=True, pv_mode=2,
                 sm_scale=None),
    W.TINY.with_(name="nq130_nk1_causal", N=130, Nk=1, causal=True),
    W.TINY.with_(name="nq64_nk4096_causal_koffset_pv16acc", N=64, Nk=4096, causal=True, dist="normal_koffset",
                 pv_mode=3),
]


@pytest.mark.parametrize("w", RECT, ids=lambda w: w.name)
def test_rectangular_vs_method_and_exact(lib, w):
    q, k, v = W.make_inputs(w)
    scale = W.sm_scale_of(w)
    out = lib.sage_attn(cuda(q), cuda(k), cuda(v), w.layout, w.causal, scale, pv_name(w), pv_dtype=pv_dtype(w))
    lib.sage_check_status()
    got = out_hnd(out, w.layout)
    qz = quant.quantize(q, k, v, w.layout, w.pv_mode)
    em = emulate.emulate(qz, w.causal, scale, **emulate.lazy_reading(w.pv_mode)).reshape(w.B, w.Hq, -1, w.d)
    em = em[:, :, :w.N].astype(np.float64)
    check_vs_emulation(got, em, vmax_of(v), w.name)
    ref = attention.attention_f64(q, k, v, w.layout, w.causal, scale)
    nk = _nkeys(w.N, w.nk, w.causal)
    check_vs_exact(got, ref, em, nk, vmax_of(v), w.name, w.dist, w.pv_mode)
    assert np.all(got[:, :, nk == 0] == 0), "rows that see no key must be zero"


VARLEN = [
    W.TINY.with_(name="varlen_mixed_causal_d64", Hq=4, Hkv=2, causal=True,
                 varlen=((300, 300), (1, 77), (129, 129), (0, 50), (640, 1000), (5, 0), (128, 128))),
    W.TINY.with_(name="varlen_mixed_pv16acc_d128_bf16", d=128, dtype="bf16", pv_mode=3, sm_scale=None,
                 varlen=((700, 700), (64, 2000), (257, 1), (1, 1))),
    W.TINY.with_(name="varlen_gqa4_d96_koffset", d=96, Hq=8, Hkv=2, dist="normal_koffset", sm_scale=None,
                 varlen=((130, 260), (400, 400), (33, 17))),
    W.TINY.with_(name="varlen_d256_causal_pv16", d=256, causal=True, pv_mode=2, sm_scale=None,
                 varlen=((300, 200), (129, 129))),
]


def _varlen_run(lib, w):
    q, k, v, cq, ck = W.make_varlen_inputs(w)
    lens = w.seqlens()
    out = lib.sage_attn_varlen(cuda(q), cuda(k), cuda(v), cq.cuda(), ck.cuda(), max(a for a, _ in lens),
                               max(b for _, b in lens), w.causal, W.sm_scale_of(w), pv_name(w), pv_dtype=pv_dtype(w))
    lib.sage_check_status()
    return q, k, v, cq, ck, out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("w", VARLEN, ids=lambda w: w.name)
def test_varlen_per_sequence_vs_method_and_exact(lib, w):
    q, k, v, cq, ck, got = _varlen_run(lib, w)
    scale = W.sm_scale_of(w)
    for b, (nq, nk) in enumerate(w.seqlens()):
        if nq == 0:
            continue
        g = got[cq[b]:cq[b + 1]].transpose(1, 0, 2)[None]                       # (1, Hq, nq, d)
        if nk == 0:
            assert np.all(g == 0), f"{w.name} seq {b}: no keys -> zeros"
            continue
        qs, ks, vs = (t[c[b]:c[b + 1]][None] for t, c in ((q, cq), (k, ck), (v, ck)))  # (1, n, H, d)
        qz = quant.quantize(qs, ks, vs, "NHD", w.pv_mode)
        em = emulate.emulate(qz, w.causal, scale, **emulate.lazy_reading(w.pv_mode)).reshape(1, w.Hq, -1, w.d)
        em = em[:, :, :nq].astype(np.float64)
        check_vs_emulation(g, em, vmax_of(vs), f"{w.name} seq {b}")
        ref = attention.attention_f64(qs, ks, vs, "NHD", w.causal, scale)
        check_vs_exact(g, ref, em, _nkeys(nq, nk, w.causal), vmax_of(vs), f"{w.name} seq {b}", w.dist, w.pv_mode)
    # the whole packed output against the packed oracle definition as well
    ex = attention.attention_varlen_f64(q, k, v, cq.numpy(), ck.numpy(), w.causal, scale)
    assert np.abs(got - ex).max() <= 0.125 * float(v.float().abs().max())


@pytest.mark.parametrize("pv", [0, 2])
def test_varlen_equal_lengths_is_the_dense_nhd_batch(lib, pv):
    """A packed batch of equal-length sequences gives bit-identical results to the dense NHD call."""
    w = W.TINY.with_(name="dense", B=3, N=300, Hq=4, Hkv=2, layout="NHD", causal=True, pv_mode=pv)
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    dense = lib.sage_attn(q, k, v, "NHD", True, 0.125, pv_name(w), pv_dtype=pv_dtype(w))
    cu = torch.arange(4, dtype=torch.int32, device="cuda") * 300
    packed = lib.sage_attn_varlen(q.view(-1, 4, 64), k.view(-1, 2, 64), v.view(-1, 2, 64), cu, cu, 300, 300, True,
                                  0.125, pv_name(w), pv_dtype=pv_dtype(w))
    lib.sage_check_status()
    assert torch.equal(dense.view(-1, 4, 64).view(torch.int16), packed.view(torch.int16))
    # and Nq = Nk through sage_attn_ex is sage_attn
    ex = torch.empty_like(dense)
    st = lib.capi.sage_attn_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), ex.data_ptr(), 3, 4, 2, 300, 300, 64,
                               lib.SAGE_FP16, lib.SAGE_NHD, 1, 0.125, pv, None, torch.cuda.current_stream().cuda_stream)
    assert st == lib.SAGE_OK
    lib.sage_check_status()
    assert torch.equal(dense.view(torch.int16), ex.view(torch.int16))


@pytest.mark.parametrize("bad", ["decreasing", "too_long", "past_total", "negative"])
def test_varlen_bad_offsets_are_reported_and_write_nothing(lib, bad):
    q = torch.randn((300, 2, 64), device="cuda").half()
    k = torch.randn((300, 2, 64), device="cuda").half()
    cq = {"decreasing": [0, 200, 100, 300], "too_long": [0, 250, 260, 300], "past_total": [0, 100, 200, 301],
          "negative": [-5, 100, 200, 300]}[bad]
    cqd = torch.tensor(cq, dtype=torch.int32, device="cuda")
    ckd = torch.tensor([0, 100, 200, 300], dtype=torch.int32, device="cuda")
    out = torch.full_like(q, 7.0)
    lib.sage_attn_varlen(q, k, k.clone(), cqd, ckd, 200, 200, True, None, out=out)
    with pytest.raises(lib.SageError) as e:
        lib.sage_check_status()
    assert e.value.status == lib.SAGE_ERR_INVALID_ARG
    assert bool((out == 7.0).all())
    # the library stays usable
    good = lib.sage_attn_varlen(q, k, k.clone(), ckd, ckd, 100, 100, True, None)
    lib.sage_check_status()
    assert torch.isfinite(good).all()


FULL_VARLEN = W.TINY.with_(name="varlen_llm_causal_gqa_hq32_hkv8_d128", Hq=32, Hkv=8, d=128, causal=True,
                           dist="normal_koutlier", sm_scale=None,
                           varlen=((8192, 8192), (1000, 1000), (4096, 4096), (1, 3000), (2500, 2500), (777, 6000)))


def test_varlen_full_size_sampled_rows(lib):
    """A full-size packed LLM prefill batch; the oracle checks sampled heads and 128-row blocks."""
    w = FULL_VARLEN
    q, k, v, cq, ck, got = _varlen_run(lib, w)
    scale = W.sm_scale_of(w)
    G = w.Hq // w.Hkv
    for b, (nq, nk) in enumerate(w.seqlens()):
        nb = (nq + 127) // 128
        qbs = sorted({0, nb // 2, nb - 1})
        rows = np.concatenate([np.arange(i * 128, min((i + 1) * 128, nq)) for i in qbs])
        for hq in sorted({0, w.Hq - 1}):
            hk = hq // G
            qs = q[cq[b]:cq[b + 1], hq:hq + 1][None]
            ks, vs = (t[ck[b]:ck[b + 1], hk:hk + 1][None] for t in (k, v))
            qz = quant.quantize(qs, ks, vs, "NHD", w.pv_mode)
            em = emulate.emulate(qz, w.causal, scale, heads=[(0, 0)], q_blocks=qbs, **emulate.lazy_reading(w.pv_mode))[0]
            em = np.concatenate([em[i * 128:i * 128 + min(128, nq - qb * 128)] for i, qb in enumerate(qbs)])
            g = got[cq[b] + rows, hq]
            what = f"seq {b} ({nq}x{nk}) h{hq}"
            check_vs_emulation(g, em.astype(np.float64), vmax_of(vs), what)
            ref = attention.attention_f64(qs, ks, vs, "NHD", w.causal, scale, heads=[(0, 0)], rows=rows)[0]
            check_vs_exact(g, ref, em, _nkeys(nq, nk, w.causal, rows), vmax_of(vs), what, w.dist, w.pv_mode)
