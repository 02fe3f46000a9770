"""The checked build (libsage_b200_checked.so, compiled with -DSAGE_CHECKED) on small cases.

In that build every global store of the quantize and attention kernels first tests that its
bytes lie inside the buffer they belong to; a store outside is skipped and reported by
sage_check_status as SAGE_ERR_BOUNDS.  On every case here both builds must give the same bytes
and report no error (no store of a correct call leaves its buffer), and a narrowed output extent
must make the kernels skip, and report, exactly the stores past it.
"""
import pytest
import torch

import workloads as W
from tests._support import cuda, opt_kw, pv_dtype, pv_name

pytestmark = pytest.mark.gpu

T = W.TINY
CASES = [
    T,                                                                          # d 64, FP8 P.V, fp32
    T.with_(name="ragged_causal_gqa_d96_nhd", N=300, d=96, Hq=4, Hkv=2, causal=True, layout="NHD"),
    T.with_(name="d128_fp16fp32_causal", N=384, d=128, causal=True, pv_mode=1, sm_scale=None),
    T.with_(name="d128_pv16_fp32_bf16", N=200, d=128, pv_mode=2, dtype="bf16", sm_scale=None),
    T.with_(name="d80_pv16_fp16fp32_causal", N=260, d=80, pv_mode=3, causal=True, sm_scale=None),
    T.with_(name="d256_causal", N=300, d=256, causal=True, sm_scale=None),
    T.with_(name="d256_pv16", N=256, d=256, pv_mode=2, sm_scale=None),
    T.with_(name="per_thread_smooth_v", N=300, d=64, q_gran=1, smooth_v=True),
    T.with_(name="per_warp_koffset", N=256, d=128, q_gran=32, dist="normal_koffset", sm_scale=None),
    T.with_(name="nq_gt_nk_causal", N=384, Nk=200, d=64, causal=True),         # queries with no key: zero rows
]


@pytest.fixture(scope="module")
def checked(lib):
    c = lib.load_checked()
    assert c.sage_checked_build() == 1
    return c


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _with(lib, api, fn):
    """fn() with the package's Python entry points bound to `api` (one of the two libraries)."""
    saved = lib.capi
    lib.capi = api
    try:
        return fn()
    finally:
        lib.capi = saved


def _bits(t):
    """The tensor's bytes as one flat uint8 vector."""
    return t.contiguous().view(torch.uint8).reshape(-1)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_checked_build_matches_the_normal_build(lib, checked, w):
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    kw = dict(tensor_layout=w.layout, is_causal=w.causal, sm_scale=W.sm_scale_of(w), pv_accum_dtype=pv_name(w),
              pv_dtype=pv_dtype(w), **opt_kw(w))
    want = lib.sage_attn(q, k, v, **kw)
    assert lib.capi.sage_check_status(_stream()) == lib.SAGE_OK
    got = _with(lib, checked, lambda: lib.sage_attn(q, k, v, **kw))
    assert checked.sage_check_status(_stream()) == lib.SAGE_OK
    assert torch.equal(_bits(got), _bits(want)), w.name


def test_checked_build_quantize_matches(lib, checked):
    w = CASES[7]  # per-thread Q scales and V smoothing: every buffer sage_quantize writes
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    kw = dict(tensor_layout=w.layout, pv_dtype="fp8", **opt_kw(w))
    want = lib.sage_quantize(q, k, v, **kw)
    got = _with(lib, checked, lambda: lib.sage_quantize(q, k, v, **kw))
    assert checked.sage_check_status(_stream()) == lib.SAGE_OK
    for n in ("q8", "qs", "k8", "ks", "km", "v8t", "vs", "vm"):
        assert torch.equal(_bits(got[n]), _bits(want[n])), n


def test_checked_build_varlen_and_noalloc_match(lib, checked):
    w = T.with_(name="varlen", varlen=((130, 130), (1, 1), (300, 300)), Hq=4, Hkv=2, d=64, causal=True, B=3)
    q, k, v, cq, ck = W.make_varlen_inputs(w)
    q, k, v, cq, ck = (cuda(t) for t in (q, k, v, cq, ck))
    run = lambda: lib.sage_attn_varlen(q, k, v, cq, ck, 300, 300, True, None)
    want = run()
    got = _with(lib, checked, run)
    assert checked.sage_check_status(_stream()) == lib.SAGE_OK
    assert torch.equal(_bits(got), _bits(want))
    q, k, v = (cuda(t) for t in W.make_inputs(CASES[1]))
    run = lambda: lib.sage_attn_noalloc(q, k, v, "NHD", True)
    want = run()
    got = _with(lib, checked, run)
    assert checked.sage_check_status(_stream()) == lib.SAGE_OK
    assert torch.equal(_bits(got), _bits(want))


@pytest.mark.parametrize("d,mode", [(64, 0), (96, 1), (128, 2), (256, 0)])
def test_narrowed_output_extent_skips_and_reports_the_stores_past_it(lib, checked, d, mode):
    # HND output (1, 4, 300, d): the extent ends after head 1, in the middle of the call's work;
    # every byte before it must be the normal result and every byte after it left untouched
    w = T.with_(name="narrowed", Hq=4, Hkv=2, N=300, d=d, pv_mode=mode, sm_scale=None)
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    kw = dict(sm_scale=W.sm_scale_of(w), pv_accum_dtype=pv_name(w), pv_dtype=pv_dtype(w))
    want = lib.sage_attn(q, k, v, **kw)
    limit = 2 * w.N * d * 2
    out = torch.full_like(q, float("nan"))
    sentinel = _bits(out).clone()
    checked.sage_test_out_limit(limit)
    try:
        _with(lib, checked, lambda: lib.sage_attn(q, k, v, out=out, **kw))
        assert checked.sage_check_status(_stream()) == lib.SAGE_ERR_BOUNDS
    finally:
        checked.sage_test_out_limit(0)
    b = _bits(out)
    assert torch.equal(b[:limit], _bits(want)[:limit])
    assert torch.equal(b[limit:], sentinel[limit:])
    # the word was cleared by the read, and the full extent is back
    out2 = _with(lib, checked, lambda: lib.sage_attn(q, k, v, **kw))
    assert checked.sage_check_status(_stream()) == lib.SAGE_OK
    assert torch.equal(_bits(out2), _bits(want))
    # the normal build ignores the hook: it has no store checks
    lib.capi.sage_test_out_limit(limit)
    try:
        out3 = lib.sage_attn(q, k, v, **kw)
        assert lib.capi.sage_check_status(_stream()) == lib.SAGE_OK
    finally:
        lib.capi.sage_test_out_limit(0)
    assert torch.equal(_bits(out3), _bits(want))
