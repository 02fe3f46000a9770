"""Failure detection on the GPU without a fault: a bounded wait that runs out is reported as
SAGE_ERR_TIMEOUT by sage_check_status, the flag clears, and the context stays usable."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention, emulate, quant
from tests._support import check_vs_exact, cuda, nkeys, out_hnd, vmax_of

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_survives(lib):
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.capi.sage_check_status(stream) == lib.SAGE_OK
    assert lib.capi.sage_selftest_wait_timeout(2000, stream) == lib.SAGE_OK  # ~2 ms of waiting, then gives up
    assert lib.capi.sage_check_status(stream) == lib.SAGE_ERR_TIMEOUT
    assert lib.capi.sage_check_status(stream) == lib.SAGE_OK                 # the flag was read and cleared
    # a full attention call on the same context still runs and is right
    w = W.TINY.with_(name="after_timeout", N=300, causal=True)
    q, k, v = W.make_inputs(w)
    out = lib.sage_attn(cuda(q), cuda(k), cuda(v), "HND", True, 0.125)
    lib.sage_check_status()
    em = emulate.emulate(quant.quantize(q, k, v, "HND", 0), True, 0.125, **emulate.lazy_reading(0))
    check_vs_exact(out_hnd(out, "HND"), attention.attention_f64(q, k, v, "HND", True, 0.125),
                   em.reshape(1, 2, -1, w.d)[:, :, :w.N], nkeys(w.N, True), vmax_of(v), w.name, w.dist, 0)
