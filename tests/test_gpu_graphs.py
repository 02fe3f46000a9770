"""sage_attn inside a CUDA graph: its stream-ordered workspace allocation, the dependent launches of
the quantize pass and the fused kernel are all captured; replays match the eager call bit for bit
and follow new inputs written into the captured buffers."""
import pytest
import torch

import workloads as W
from tests._support import cuda, opt_kw, pv_dtype, pv_name

pytestmark = pytest.mark.gpu

CASES = [W.TINY.with_(name="graph_causal_gqa", N=1000, Hq=4, Hkv=2, causal=True),
         W.TINY.with_(name="graph_pv16_qthread_smoothv_nhd", N=777, d=128, layout="NHD", pv_mode=3, q_gran=1,
                      smooth_v=True)]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_sage_attn_captured_in_a_cuda_graph(lib, w):
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    kw = dict(pv_dtype=pv_dtype(w), **opt_kw(w))
    call = lambda o: lib.sage_attn(q, k, v, w.layout, w.causal, W.sm_scale_of(w), pv_name(w), out=o, **kw)
    out = torch.empty_like(q)
    call(out)  # warm-up outside the capture
    torch.cuda.synchronize()
    ref = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=torch.cuda.Stream()):
        call(out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    q.copy_(q.flip(2 if w.layout == "HND" else 1))  # new inputs in the captured buffers
    g.replay()
    torch.cuda.synchronize()
    eager = torch.empty_like(q)
    call(eager)
    lib.sage_check_status()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))


def test_readme_names_are_the_same_calls(lib):
    w = W.TINY.with_(name="names", N=300, Hq=4, Hkv=2, causal=True)
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    same = lambda a, b: torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert same(lib.sageattn(q, k, v, "HND", True), lib.sage_attn(q, k, v, "HND", True))
    assert same(lib.sageattn_qk_int8_pv_fp8_cuda(q, k, v, is_causal=True, pv_accum_dtype="fp32+fp16"),
                lib.sage_attn(q, k, v, "HND", True, None, "fp16+fp32"))
    assert same(lib.sageattn_qk_int8_pv_fp16_cuda(q, k, v, is_causal=True),
                lib.sage_attn(q, k, v, "HND", True, pv_dtype="fp16"))
    cu = torch.tensor([0, 100, 300], dtype=torch.int32, device="cuda")
    qp, kp, vp = (t[0].transpose(0, 1).contiguous() for t in (q, k, v))
    assert same(lib.sageattn_varlen(qp, kp, vp, cu, cu, 200, 200, True),
                lib.sage_attn_varlen(qp, kp, vp, cu, cu, 200, 200, True, pv_dtype="fp16"))
    lib.sage_check_status()
