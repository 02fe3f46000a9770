"""sage_mma_probe on the GPU: the tcgen05.mma rate of each kind, the figure bench.py reports beside
the bf16-derived tensor peak.  The rate must be that of a B200 actually issuing the MMAs: above a
floor no CUDA-core path could reach, below the dense nominal ceiling with margin."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind,nominal", [(0, 4500.0), (1, 4500.0), (2, 2250.0)], ids=["i8", "f8f6f4", "f16"])
def test_mma_probe_rate_is_a_tensor_core_rate(lib, kind, nominal):
    st = torch.cuda.current_stream()
    ops = ctypes.c_double(0.0)
    best = 0.0
    for _ in range(4):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        assert lib.capi.sage_mma_probe(kind, 4000, ctypes.byref(ops), st.cuda_stream) == lib.SAGE_OK
        b.record(st)
        torch.cuda.synchronize()
        best = max(best, ops.value / (a.elapsed_time(b) * 1e-3) / 1e12)
    assert lib.capi.sage_check_status(st.cuda_stream) == lib.SAGE_OK
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert ops.value == sms * 4000 * 4 * 2 * 128 * 256 * (16 if kind == 2 else 32)
    assert 0.3 * nominal < best < 1.2 * nominal, best

