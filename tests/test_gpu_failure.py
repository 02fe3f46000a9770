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


def test_injected_allocation_failure_is_reported_and_the_next_call_runs(lib):
    # the workspace allocation of the first call fails (host-side injection, nothing reaches the
    # device); the call reports SAGE_ERR_OOM and queues no work, and the next call is whole
    w = W.TINY.with_(name="after_oom", N=300)
    q, k, v = (cuda(t) for t in W.make_inputs(w))
    out = torch.full_like(q, 7.0)
    try:
        lib.capi.sage_test_inject(0, 1)
        with pytest.raises(lib.SageError) as e:
            lib.sage_attn(q, k, v, "HND", False, 0.125, out=out)
        assert e.value.status == lib.SAGE_ERR_OOM
    finally:
        lib.capi.sage_test_inject(0, 0)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was written
    assert lib.capi.sage_check_status(torch.cuda.current_stream().cuda_stream) == lib.SAGE_OK
    ref = lib.sage_attn(q, k, v, "HND", False, 0.125)
    lib.sage_check_status()
    again = lib.sage_attn(q, k, v, "HND", False, 0.125, out=out)
    lib.sage_check_status()
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))
