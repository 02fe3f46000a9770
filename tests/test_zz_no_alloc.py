"""The allocation-free entry point sage_attn_noalloc, called through the C ABI.

It is for callers that cannot allocate device memory at call time (a framework
or server that reserves all GPU memory up front, a runtime that forbids
allocation after start-up, a setup without stream-ordered memory pools); its
workspace is a static device array inside the library.  This file runs last so
that a failure here leaves every other test already run.  It passes alone in a
fresh process and after the other tests: the only state it relies on is the
per-device address lookup that the first call performs.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention, emulate, quant
from tests._support import check_vs_emulation, check_vs_exact, cuda, nkeys, out_hnd, vmax_of

pytestmark = pytest.mark.gpu

CASES = [
    W.IMAGE_DIT,                                                              # ~38 MiB of the 64 MiB workspace
    W.TINY.with_(name="ragged_causal_gqa_d96", N=300, d=96, Hq=4, Hkv=2, causal=True, sm_scale=None),
]


def _dt(lib, t):
    return lib.SAGE_BF16 if t.dtype == torch.bfloat16 else lib.SAGE_FP16


def _call(lib, fn, w, q, k, v, out):
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.B, w.Hq, w.Hkv, w.N, w.d, _dt(lib, q),
              lib.SAGE_HND if w.layout == "HND" else lib.SAGE_NHD, int(w.causal), float(W.sm_scale_of(w)),
              w.pv_mode, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_sage_attn_on_two_calls_in_a_row(lib):
    outs = []
    for w in CASES:  # two calls in a row, the second on a smaller problem than the first
        assert lib.sage_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d) <= lib.SAGE_NOALLOC_MAX_BYTES
        q, k, v = (cuda(t) for t in W.make_inputs(w))
        out = torch.empty_like(q)
        assert _call(lib, lib.capi.sage_attn_noalloc, w, q, k, v, out) == lib.SAGE_OK
        outs.append((w, q, k, v, out))
    assert lib.capi.sage_check_status(torch.cuda.current_stream().cuda_stream) == lib.SAGE_OK
    for w, q, k, v, out in outs:
        # the same kernels on the same workspace layout: bit for bit the pooled entry point's output
        ref = torch.empty_like(q)
        assert _call(lib, lib.capi.sage_attn, w, q, k, v, ref) == lib.SAGE_OK
        assert lib.capi.sage_check_status(torch.cuda.current_stream().cuda_stream) == lib.SAGE_OK
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), w.name
    # and the ragged causal case against the oracle: the method's emulation and exact attention
    w, q, k, v, out = outs[1]
    qc, kc, vc = (t.cpu() for t in (q, k, v))
    got = out_hnd(out, w.layout)
    qz = quant.quantize(qc, kc, vc, w.layout, w.pv_mode)
    em = emulate.emulate(qz, w.causal, W.sm_scale_of(w), **emulate.lazy_reading(w.pv_mode))
    em = em.reshape(w.B, w.Hq, -1, w.d)[:, :, :w.N].astype(np.float64)
    check_vs_emulation(got, em, vmax_of(vc), w.name)
    ref = attention.attention_f64(qc, kc, vc, w.layout, w.causal, W.sm_scale_of(w))
    check_vs_exact(got, ref, em, nkeys(w.N, w.causal), vmax_of(vc), w.name, w.dist, w.pv_mode)


def test_noalloc_rejects_workspace_beyond_the_static_array(lib):
    w = W.LLM_GQA  # needs ~200 MiB of workspace
    assert lib.sage_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d) > lib.SAGE_NOALLOC_MAX_BYTES
    fake = 0x100000
    st = lib.capi.sage_attn_noalloc(fake, fake + (1 << 34), fake + (2 << 34), fake + (3 << 34), w.B, w.Hq, w.Hkv,
                                    w.N, w.d, lib.SAGE_FP16, lib.SAGE_HND, 1, 0.0, 0, None)
    assert st == lib.SAGE_ERR_INVALID_ARG
