"""The C-ABI library on the host: it loads, exports what include/sage.h declares,
and rejects bad arguments before touching any GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x100000  # never dereferenced: every call below fails its argument checks first


def _declared():
    src = open(os.path.join(ROOT, "include", "sage.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(sage_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("sage_attn", "sage_quantize", "sage_attn_quantized", "sage_qk_int32", "sage_check_status",
              "sage_status_string", "sage_workspace_bytes", "sage_device_supported"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in _declared():
        assert hasattr(raw, n), n


def test_checked_build_exports_every_declared_symbol_and_says_so(lib):
    # the -DSAGE_CHECKED twin is a separate library with the same boundary
    checked = lib.load_checked()
    for n in _declared():
        assert hasattr(checked, n), n
    assert checked.sage_checked_build() == 1
    assert lib.capi.sage_checked_build() == 0
    assert checked.sage_status_string(lib.SAGE_ERR_BOUNDS).decode() == lib.sage_status_string(lib.SAGE_ERR_BOUNDS)
    # argument checks are the same host code in both
    assert checked.sage_attn(FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 256, 300, lib.SAGE_FP16, lib.SAGE_HND, 0, 0.0, 0,
                             None) == lib.SAGE_ERR_INVALID_ARG


def test_status_strings(lib):
    for s in range(8):
        assert lib.sage_status_string(s)
    assert "buffer" in lib.sage_status_string(lib.SAGE_ERR_BOUNDS)
    assert "fp16" in lib.sage_status_string(lib.SAGE_ERR_UNSUPPORTED)


def _attn(lib, **kw):
    a = dict(q=FAKE, k=FAKE + 0x100000000, v=FAKE + 0x200000000, out=FAKE + 0x300000000, B=1, Hq=2, Hkv=2, N=256,
             d=64, dtype=lib.SAGE_FP16, layout=lib.SAGE_HND, causal=0, scale=0.0, pv=0)
    a.update(kw)
    return lib.capi.sage_attn(a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                              a["dtype"], a["layout"], a["causal"], a["scale"], a["pv"], None)


def test_sage_attn_argument_checks(lib):
    E, U = lib.SAGE_ERR_INVALID_ARG, lib.SAGE_ERR_UNSUPPORTED
    assert _attn(lib, dtype=lib.SAGE_FP32) == U              # fp32 inputs are rejected like the reference
    assert _attn(lib, dtype=7) == E
    assert _attn(lib, q=None) == E and _attn(lib, out=None) == E
    assert _attn(lib, Hq=3, Hkv=2) == E                      # GQA needs Hq % Hkv == 0
    assert _attn(lib, d=257) == E and _attn(lib, d=0) == E
    assert _attn(lib, N=0) == E and _attn(lib, B=0) == E
    assert _attn(lib, layout=2) == E and _attn(lib, pv=4) == E and _attn(lib, pv=-1) == E
    assert _attn(lib, out=FAKE + 10) == E                     # out overlaps q
    assert _attn(lib, B=70000) == E                           # beyond the launch grid


def test_other_entry_points_argument_checks(lib):
    c, E = lib.capi, lib.SAGE_ERR_INVALID_ARG
    assert c.sage_quantize(FAKE, FAKE, FAKE, 1, 2, 2, 256, 64, lib.SAGE_FP32, 0, 0, None, *([FAKE] * 8), None) == \
        lib.SAGE_ERR_UNSUPPORTED
    assert c.sage_quantize(FAKE, FAKE, FAKE, 1, 2, 2, 256, 64, 0, 0, 0, None, None, *([FAKE] * 7), None) == E
    assert c.sage_quantize(FAKE, FAKE, FAKE, 1, 2, 2, 256, 64, 0, 0, 0, None, FAKE + 1, *([FAKE] * 7), None) == E
    assert c.sage_attn_quantized(*([FAKE] * 8), 1, 4, 3, 256, 64, 0, 0, 0, 0.0, 0, None, None) == E
    assert c.sage_attn_quantized(*([FAKE] * 7), None, 1, 4, 2, 256, 64, 0, 0, 0, 0.0, 0, None, None) == E
    # options: granularity must be 0, 128, 32 or 1; smooth_v 0 or 1; smoothing needs a vm buffer
    bad = [lib.SageOpts(64, 0), lib.SageOpts(128, 2), lib.SageOpts(-1, 0)]
    for o in bad:
        assert c.sage_attn_ex(FAKE, FAKE + (1 << 34), FAKE + (2 << 34), FAKE + (3 << 34), 1, 2, 2, 256, 256, 64,
                              0, 0, 0, 0.0, 0, ctypes.byref(o), None) == E
        assert c.sage_quantize(FAKE, FAKE, FAKE, 1, 2, 2, 256, 64, 0, 0, 0, ctypes.byref(o), *([FAKE] * 8),
                               None) == E
    sm = lib.SageOpts(1, 1)
    assert c.sage_quantize(FAKE, FAKE, FAKE, 1, 2, 2, 256, 64, 0, 0, 0, ctypes.byref(sm), *([FAKE] * 7), None,
                           None) == E
    assert c.sage_attn_quantized(*([FAKE] * 6), None, FAKE, 1, 2, 2, 256, 64, 0, 0, 0, 0.0, 0, ctypes.byref(sm),
                                 None) == E
    assert c.sage_qk_int32(FAKE, FAKE, 1, 2, 2, 256, 64, None, 1, FAKE, None) == E
    assert c.sage_qk_int32(FAKE, FAKE, 1, 2, 2, 256, 300, FAKE, 1, FAKE, None) == E
    assert c.sage_qk_int32(FAKE, FAKE, 1, 2, 2, 256, 64, FAKE, 0, FAKE, None) == lib.SAGE_OK  # nothing to do


def test_workspace_bytes(lib):
    assert lib.sage_workspace_bytes(1, 2, 2, 0, 64) == 0
    # q8 + k8 + V codes dominate: (Hq + Hkv + 2 Hkv) * Np * dp bytes (V codes counted at the
    # 2 bytes of the FP16 P.V modes, the largest), plus fp32 scales and partial sums
    ws = lib.sage_workspace_bytes(2, 8, 2, 1000, 96)
    codes = 2 * (8 + 2 + 2 * 2) * 1024 * 128
    # the rest: per-token Q scales (the finest granularity, 2*8*1024 floats), four K/V partial-sum
    # arrays (4 * 2*2*8 blocks * 128 floats), per-channel vectors and 1 KiB alignment per buffer
    assert codes < ws < codes + 2 * 8 * 1024 * 4 + 4 * 2 * 2 * 8 * 128 * 4 + 96 * 1024


def test_padded_dim(lib):
    assert [lib.padded_dim(d) for d in (1, 64, 65, 128, 129, 256)] == [64, 64, 128, 128, 256, 256]
    with pytest.raises(ValueError):
        lib.padded_dim(300)


def test_pv_mode_names(lib):
    assert lib.pv_mode() == lib.SAGE_PV_FP32 == 0
    assert lib.pv_mode("fp8", "fp16+fp32") == lib.pv_mode("fp8", "fp32+fp16") == lib.SAGE_PV_FP16_FP32 == 1
    assert lib.pv_mode("fp16", "fp32") == lib.SAGE_PV16_FP32 == 2
    assert lib.pv_mode("fp16", "fp16+fp32") == lib.SAGE_PV16_FP16_FP32 == 3
    assert lib.pv_mode("fp16", "fp16") == lib.SAGE_PV16_FP16 == 6  # named, and rejected by the library
    for bad in (("fp8", "fp16"), ("int8", "fp32"), ("fp16", "bf16")):
        with pytest.raises(ValueError):
            lib.pv_mode(*bad)


def test_pure_fp16_accumulation_is_rejected_not_substituted(lib):
    # pv_accum_dtype "fp16" with FP16 operands: SAGE_ERR_UNSUPPORTED from every entry point that
    # takes a P.V mode, before any GPU work (no silent fp32 accumulation in its place)
    U = lib.SAGE_ERR_UNSUPPORTED
    assert _attn(lib, pv=lib.SAGE_PV16_FP16) == U
    c = lib.capi
    assert c.sage_attn_noalloc(FAKE, FAKE + 0x100000000, FAKE + 0x200000000, FAKE + 0x300000000, 1, 2, 2, 256, 64,
                               lib.SAGE_FP16, lib.SAGE_HND, 0, 0.0, lib.SAGE_PV16_FP16, None) == U
    assert c.sage_attn_quantized(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE + 0x300000000, 1, 2, 2, 256, 64,
                                 lib.SAGE_FP16, lib.SAGE_HND, 0, 0.0, lib.SAGE_PV16_FP16, None, None) == U


def test_mma_probe_argument_checks(lib):
    ops = ctypes.c_double(0.0)
    E = lib.SAGE_ERR_INVALID_ARG
    assert lib.capi.sage_mma_probe(3, 10, ctypes.byref(ops), None) == E
    assert lib.capi.sage_mma_probe(0, 0, ctypes.byref(ops), None) == E
    assert lib.capi.sage_mma_probe(0, 10, None, None) == E


def test_injected_arch_and_allocation_failures(lib):
    """SAGE_ERR_ARCH and SAGE_ERR_OOM through the host-side test hook, with no GPU: the checks run in
    their documented order (arguments, device, workspace) and nothing reaches the device."""
    c = lib.capi
    try:
        c.sage_test_inject(90, 0)                         # an sm_90 device
        assert _attn(lib) == lib.SAGE_ERR_ARCH
        assert lib.sage_device_supported() is False
        assert _attn(lib, d=0) == lib.SAGE_ERR_INVALID_ARG  # argument checks still come first
        c.sage_test_inject(100, 2)                        # a B200 whose next two allocations fail
        assert c.sage_device_supported() == 1
        assert _attn(lib) == lib.SAGE_ERR_OOM
        fake = [FAKE + (i << 32) for i in range(9)]
        assert c.sage_quantize(fake[0], fake[1], fake[2], 1, 2, 2, 256, 64, lib.SAGE_FP16, lib.SAGE_HND, 0, None,
                               *fake[3:], FAKE, None, None) == lib.SAGE_ERR_OOM
    finally:
        c.sage_test_inject(0, 0)
    assert c.sage_device_supported() in (0, 1)


def test_selftest_budget_checks(lib):
    assert lib.capi.sage_selftest_wait_timeout(0, None) == lib.SAGE_ERR_INVALID_ARG
    assert lib.capi.sage_selftest_wait_timeout(100001, None) == lib.SAGE_ERR_INVALID_ARG


def test_opts_names(lib):
    assert (lib.opts().q_gran, lib.opts().smooth_v) == (128, 0)
    assert (lib.opts("per_warp", True).q_gran, lib.opts("per_warp", True).smooth_v) == (32, 1)
    assert lib.opts("per_thread").q_gran == 1
    with pytest.raises(ValueError):
        lib.opts("per_channel")


def test_readme_entry_point_names(lib):
    import inspect
    for name in ("sageattn", "sageattn_qk_int8_pv_fp8_cuda", "sageattn_qk_int8_pv_fp16_cuda", "sageattn_varlen"):
        assert callable(getattr(lib, name)) and name in lib.__all__
    sig = inspect.signature(lib.sageattn)
    assert list(sig.parameters)[:6] == ["q", "k", "v", "tensor_layout", "is_causal", "sm_scale"]
    assert sig.parameters["tensor_layout"].default == "HND" and sig.parameters["is_causal"].default is False
    assert inspect.signature(lib.sageattn_varlen).parameters["pv_dtype"].default == "fp16"
