"""INT8-QK / FP8-PV quantized attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/sage.h`` (``libsage_b200.so``,
built in-tree by ``python quantized_attention_int8_b200/build_lib.py``).  The
functions keep the C entry points' names and only marshal arguments: torch
supplies device memory and the current CUDA stream, and every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback: if
the library is missing, importing this package fails.

    from quantized_attention_int8_b200 import sage_attn
    out = sage_attn(q, k, v, tensor_layout="HND", is_causal=False)

mirrors the ``sageattn(q, k, v, tensor_layout, is_causal, sm_scale)`` call of
the SageAttention README ("How to Use"); ``pv_accum_dtype`` selects "fp32" or
"fp16+fp32" accumulation of the P.V product (qwbw.cn article, pitfalls) and
``pv_dtype`` its operands: "fp8" (E4M3, the INT8-QK / FP8-PV kernel) or "fp16"
(the INT8-QK / FP16-PV kernel of the README's "Available APIs"); ``qk_quant_gran``
the Q scale granularity ("per_block", "per_warp", "per_thread") and ``smooth_v``
optional V smoothing (see ``sage_opts`` in include/sage.h).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "SageError", "sage_attn", "sage_quantize", "sage_attn_quantized", "sage_qk_int32", "sage_check_status",
    "sage_workspace_bytes", "sage_device_supported", "sage_status_string", "padded_dim", "LIB_PATH", "capi",
    "sage_attn_noalloc", "SAGE_NOALLOC_MAX_BYTES", "load_checked", "CHECKED_LIB_PATH", "pv_mode", "sage_attn_varlen", "SageOpts", "opts",
    "sageattn", "sageattn_qk_int8_pv_fp8_cuda", "sageattn_qk_int8_pv_fp16_cuda", "sageattn_varlen",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsage_b200.so")
# the same library compiled with -DSAGE_CHECKED: every kernel store tests its extent first
CHECKED_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsage_b200_checked.so")

SAGE_OK, SAGE_ERR_INVALID_ARG, SAGE_ERR_UNSUPPORTED, SAGE_ERR_ARCH, SAGE_ERR_CUDA, SAGE_ERR_OOM, \
    SAGE_ERR_TIMEOUT, SAGE_ERR_BOUNDS = range(8)
SAGE_HND, SAGE_NHD = 0, 1
SAGE_FP16, SAGE_BF16, SAGE_FP32 = 0, 1, 2
SAGE_PV_FP32, SAGE_PV_FP16_FP32, SAGE_PV16_FP32, SAGE_PV16_FP16_FP32, SAGE_PV16_FP16 = 0, 1, 2, 3, 6

_LAYOUTS = {"HND": SAGE_HND, "NHD": SAGE_NHD}
_DTYPES = {torch.float16: SAGE_FP16, torch.bfloat16: SAGE_BF16, torch.float32: SAGE_FP32}
_PV = {("fp8", "fp32"): SAGE_PV_FP32, ("fp8", "fp16+fp32"): SAGE_PV_FP16_FP32,
       ("fp8", "fp32+fp16"): SAGE_PV_FP16_FP32,
       ("fp16", "fp32"): SAGE_PV16_FP32, ("fp16", "fp16+fp32"): SAGE_PV16_FP16_FP32,
       ("fp16", "fp16"): SAGE_PV16_FP16}


def pv_mode(pv_dtype: str = "fp8", pv_accum_dtype: str = "fp32") -> int:
    """The sage_pv_mode value for P.V operands ``pv_dtype`` and accumulation ``pv_accum_dtype``.

    "fp32+fp16" is the README's spelling of the two-level (fp16 tile, fp32 total)
    accumulation of the FP8 kernel.  "fp16" (pure fp16 accumulation with FP16 operands,
    the fastest and least overflow-safe option on the GPUs the pages target) maps to
    SAGE_PV16_FP16, which the library rejects with SAGE_ERR_UNSUPPORTED: on sm_100a a
    tcgen05 MMA issues at the same rate with an F16 or an F32 accumulator, so fp16
    accumulation would buy no speed and only add error and overflow risk.
    """
    try:
        return _PV[(pv_dtype, pv_accum_dtype)]
    except KeyError:
        raise ValueError(f"unsupported pv_dtype / pv_accum_dtype {pv_dtype!r} / {pv_accum_dtype!r}") from None


class SageOpts(ctypes.Structure):
    """The C ``sage_opts``: query tokens per Q scale (128, 32 or 1) and V smoothing (0 / 1)."""
    _fields_ = [("q_gran", ctypes.c_int), ("smooth_v", ctypes.c_int)]


_GRANS = {"per_block": 128, "per_warp": 32, "per_thread": 1}


def opts(qk_quant_gran: str = "per_block", smooth_v: bool = False) -> SageOpts:
    """SageOpts for a granularity name ("per_block", "per_warp", "per_thread") and V smoothing."""
    if qk_quant_gran not in _GRANS:
        raise ValueError(f"qk_quant_gran must be one of {sorted(_GRANS)}, got {qk_quant_gran!r}")
    return SageOpts(_GRANS[qk_quant_gran], 1 if smooth_v else 0)


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is not built; run `python quantized_attention_int8_b200/build_lib.py` "
            "(this package has no CPU fallback)")
    lib = ctypes.CDLL(path)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "sage_attn": ([P, P, P, P, I, I, I, I, I, I, I, I, F, I, P], I),
        "sage_workspace_bytes": ([I, I, I, I, I], Z),
        "sage_quantize": ([P, P, P, I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P], I),
        "sage_attn_quantized": ([P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, P, P], I),
        "sage_qk_int32": ([P, P, I, I, I, I, I, P, I, P, P], I),
        "sage_check_status": ([P], I),
        "sage_status_string": ([I], ctypes.c_char_p),
        "sage_device_supported": ([], I),
        "sage_attn_noalloc": ([P, P, P, P, I, I, I, I, I, I, I, I, F, I, P], I),
        "sage_attn_ex": ([P, P, P, P, I, I, I, I, I, I, I, I, I, F, I, P, P], I),
        "sage_selftest_wait_timeout": ([I, P], I),
        "sage_mma_probe": ([I, I, ctypes.POINTER(ctypes.c_double), P], I),
        "sage_test_inject": ([I, I], None),
        "sage_test_out_limit": ([ctypes.c_longlong], None),
        "sage_checked_build": ([], I),
        "sage_attn_varlen": ([P, P, P, P, P, P, I, I, I, ctypes.c_longlong, ctypes.c_longlong, I, I, I, I, I, F, I, P,
                              P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, res
    return lib


capi = _load()


def load_checked() -> ctypes.CDLL:
    """The checked build (``libsage_b200_checked.so``) with the same signatures as ``capi``.

    Its kernels test every global store against the buffer it belongs to, skip one that falls
    outside and report it through ``sage_check_status`` (SAGE_ERR_BOUNDS).  A second, independent
    copy of the library: its device state (error words, no-alloc workspace) is its own."""
    return _load(CHECKED_LIB_PATH)


class SageError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {sage_status_string(status)} (status {status})")


def sage_status_string(status: int) -> str:
    return capi.sage_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != SAGE_OK:
        raise SageError(status, where)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def padded_dim(d: int) -> int:
    if d > 256:
        raise ValueError("head_dim > 256 is not supported")
    return 64 if d <= 64 else (128 if d <= 128 else 256)


def _shape(q: torch.Tensor, k: torch.Tensor, layout: str):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    if layout == "HND":
        B, Hq, N, d = q.shape
        Hkv, Nk = k.shape[1], k.shape[2]
    elif layout == "NHD":
        B, N, Hq, d = q.shape
        Hkv, Nk = k.shape[2], k.shape[1]
    else:
        raise ValueError(f"tensor_layout must be 'HND' or 'NHD', got {layout!r}")
    return B, Hq, Hkv, N, Nk, d


def _check_tensors(q, k, v):
    for t in (q, k, v):
        if not t.is_cuda:
            raise ValueError("q, k, v must be CUDA tensors (no CPU path exists)")
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share one dtype")
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {q.dtype}")


def _check_inputs_nk(q, k, v, layout):
    """(B, Hq, Hkv, Nq, Nk, d) of q and k, v, which may differ in length."""
    _check_tensors(q, k, v)
    B, Hq, Hkv, N, Nk, d = _shape(q, k, layout)
    kshape = (B, Hkv, Nk, d) if layout == "HND" else (B, Nk, Hkv, d)
    if tuple(k.shape) != kshape:
        raise ValueError(f"k has shape {tuple(k.shape)}, expected {kshape}")
    return B, Hq, Hkv, N, Nk, d


def _check_inputs(q, k, v, layout):
    """(B, Hq, Hkv, N, d) of q, k, v of one length."""
    B, Hq, Hkv, N, Nk, d = _check_inputs_nk(q, k, v, layout)
    if Nk != N:
        raise ValueError(f"q has {N} tokens and k, v {Nk}; this entry point needs equal lengths")
    return B, Hq, Hkv, N, d


def sage_attn(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None, pv_accum_dtype="fp32", out=None,
              pv_dtype="fp8", qk_quant_gran="per_block", smooth_v=False):
    """Quantized attention of fp16/bf16 q (B,Hq,Nq,d), k/v (B,Hkv,Nk,d) (HND; NHD stores (B,N,H,d)).

    Nq may differ from Nk (then the causal mask is aligned bottom-right); non-default
    qk_quant_gran / smooth_v, or Nq != Nk, go through sage_attn_ex."""
    B, Hq, Hkv, N, Nk, d = _check_inputs_nk(q, k, v, tensor_layout)
    o = opts(qk_quant_gran, smooth_v)
    if out is None:
        out = torch.empty_like(q)
    scale = float(sm_scale) if sm_scale is not None else 0.0
    mode = pv_mode(pv_dtype, pv_accum_dtype)
    if Nk == N and o.q_gran == 128 and not o.smooth_v:
        st = capi.sage_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, N, d,
                            _DTYPES[q.dtype], _LAYOUTS[tensor_layout], int(bool(is_causal)), scale, mode, _stream())
        _check(st, "sage_attn")
    else:
        st = capi.sage_attn_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, N, Nk, d,
                               _DTYPES[q.dtype], _LAYOUTS[tensor_layout], int(bool(is_causal)), scale, mode,
                               ctypes.byref(o), _stream())
        _check(st, "sage_attn_ex")
    return out


def sage_attn_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, is_causal=False,
                     sm_scale=None, pv_accum_dtype="fp32", out=None, pv_dtype="fp8", qk_quant_gran="per_block",
                     smooth_v=False):
    """Packed batch: q (total_q, Hq, d), k/v (total_k, Hkv, d), cu_seqlens_* int32 CUDA tensors of
    B + 1 offsets (sequence b = tokens cu[b] .. cu[b+1]-1).  Each sequence attends to its own keys
    (causal: aligned bottom-right per sequence).  A bad offset table raises SageError from the
    status check after the launch."""
    _check_tensors(q, k, v)
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("varlen q, k, v must be 3-D (tokens, heads, head_dim)")
    total_q, Hq, d = q.shape
    total_k, Hkv, dk = k.shape
    if dk != d:
        raise ValueError("q and k must have the same head_dim")
    for c in (cu_seqlens_q, cu_seqlens_k):
        if not (c.is_cuda and c.dtype == torch.int32 and c.dim() == 1 and c.is_contiguous()):
            raise ValueError("cu_seqlens must be contiguous 1-D int32 CUDA tensors")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 >= 2 offsets")
    B = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    st = capi.sage_attn_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), cu_seqlens_q.data_ptr(),
                               cu_seqlens_k.data_ptr(), B, int(max_seqlen_q), int(max_seqlen_k), total_q, total_k,
                               Hq, Hkv, d, _DTYPES[q.dtype], int(bool(is_causal)),
                               float(sm_scale) if sm_scale is not None else 0.0, pv_mode(pv_dtype, pv_accum_dtype),
                               ctypes.byref(opts(qk_quant_gran, smooth_v)), _stream())
    _check(st, "sage_attn_varlen")
    return out


SAGE_NOALLOC_MAX_BYTES = 64 << 20


def sage_attn_noalloc(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None, pv_accum_dtype="fp32", out=None,
                      pv_dtype="fp8"):
    """sage_attn with no device allocation inside the library (for callers that cannot
    allocate at call time); the caller supplies ``out`` or torch allocates it here.  The
    library's static workspace holds problems up to SAGE_NOALLOC_MAX_BYTES of workspace
    (larger ones raise SageError with SAGE_ERR_INVALID_ARG); calls that may overlap on the
    GPU must be ordered by the caller."""
    B, Hq, Hkv, N, d = _check_inputs(q, k, v, tensor_layout)
    if out is None:
        out = torch.empty_like(q)
    st = capi.sage_attn_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, N, d,
                                _DTYPES[q.dtype], _LAYOUTS[tensor_layout], int(bool(is_causal)),
                                float(sm_scale) if sm_scale is not None else 0.0, pv_mode(pv_dtype, pv_accum_dtype),
                        _stream())
    _check(st, "sage_attn_noalloc")
    return out


def sage_workspace_bytes(B, Hq, Hkv, N, d) -> int:
    return int(capi.sage_workspace_bytes(B, Hq, Hkv, N, d))


def sage_quantize(q, k, v, tensor_layout="HND", pv_accum_dtype="fp32", pv_dtype="fp8", qk_quant_gran="per_block",
                  smooth_v=False) -> dict:
    """The quantize/smooth pass alone; returns the codes and scales as CUDA tensors.

    Layouts (Np = 128*ceil(N/128), dp = padded head dim): q8 int8 (B,Hq,Np,dp),
    qs f32 (B,Hq,Np/128), k8 int8 (B,Hkv,Np,dp), ks f32 (B,Hkv,Np/128),
    km f32 (B,Hkv,dp), v8t (B,Hkv,dp,Np) uint8 E4M3 codes (pv_dtype "fp8") or
    float16 codes (pv_dtype "fp16"), vs f32 (B,Hkv,dp), vm f32 (B,Hkv,dp) (V's token mean
    with smooth_v, else zeros); qs has Np / q_gran entries per head.
    """
    mode = pv_mode(pv_dtype, pv_accum_dtype)
    o = opts(qk_quant_gran, smooth_v)
    B, Hq, Hkv, N, d = _check_inputs(q, k, v, tensor_layout)
    dp, nb = padded_dim(d), (N + 127) // 128
    Np = nb * 128
    dev = q.device
    z = dict(
        q8=torch.empty((B, Hq, Np, dp), dtype=torch.int8, device=dev),
        qs=torch.empty((B, Hq, Np // o.q_gran), dtype=torch.float32, device=dev),
        k8=torch.empty((B, Hkv, Np, dp), dtype=torch.int8, device=dev),
        ks=torch.empty((B, Hkv, nb), dtype=torch.float32, device=dev),
        km=torch.empty((B, Hkv, dp), dtype=torch.float32, device=dev),
        v8t=torch.empty((B, Hkv, dp, Np), dtype=torch.float16 if pv_dtype == "fp16" else torch.uint8, device=dev),
        vs=torch.empty((B, Hkv, dp), dtype=torch.float32, device=dev),
        vm=torch.zeros((B, Hkv, dp), dtype=torch.float32, device=dev),
    )
    st = capi.sage_quantize(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv, N, d, _DTYPES[q.dtype],
                            _LAYOUTS[tensor_layout], mode, ctypes.byref(o),
                            *(z[n].data_ptr() for n in ("q8", "qs", "k8", "ks", "km", "v8t", "vs", "vm")), _stream())
    _check(st, "sage_quantize")
    z.update(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, pv_dtype=pv_dtype, qk_quant_gran=qk_quant_gran, smooth_v=bool(smooth_v))
    return z


def sage_attn_quantized(z: dict, out_dtype=torch.float16, tensor_layout="HND", is_causal=False, sm_scale=None,
                        pv_accum_dtype="fp32", out=None):
    """The fused attention kernel alone on quantized buffers (the dict sage_quantize returns;
    its ``pv_dtype`` entry selects the P.V operands)."""
    B, Hq, Hkv, N, d = (z[n] for n in ("B", "Hq", "Hkv", "N", "d"))
    if out is None:
        shape = (B, Hq, N, d) if tensor_layout == "HND" else (B, N, Hq, d)
        out = torch.empty(shape, dtype=out_dtype, device=z["q8"].device)
    o = opts(z.get("qk_quant_gran", "per_block"), z.get("smooth_v", False))
    vm = z.get("vm")
    st = capi.sage_attn_quantized(*(z[n].data_ptr() for n in ("q8", "qs", "k8", "ks", "v8t", "vs")),
                                  vm.data_ptr() if vm is not None else None,
                                  out.data_ptr(), B, Hq, Hkv, N, d, _DTYPES[out.dtype], _LAYOUTS[tensor_layout],
                                  int(bool(is_causal)), float(sm_scale) if sm_scale is not None else 0.0,
                                  pv_mode(z.get("pv_dtype", "fp8"), pv_accum_dtype), ctypes.byref(o), _stream())
    _check(st, "sage_attn_quantized")
    return out


def sage_qk_int32(z: dict, tiles) -> torch.Tensor:
    """int32 Q8.K8^T of 128x128 tiles; tiles = list of (b, hq, q_tile, k_tile)."""
    t = torch.as_tensor(tiles, dtype=torch.int32).reshape(-1, 4).to(z["q8"].device).contiguous()
    out = torch.empty((t.shape[0], 128, 128), dtype=torch.int32, device=z["q8"].device)
    st = capi.sage_qk_int32(z["q8"].data_ptr(), z["k8"].data_ptr(), z["B"], z["Hq"], z["Hkv"], z["N"], z["d"],
                            t.data_ptr(), t.shape[0], out.data_ptr(), _stream())
    _check(st, "sage_qk_int32")
    return out


def sage_check_status() -> None:
    _check(capi.sage_check_status(_stream()), "sage_check_status")


def sage_device_supported() -> bool:
    return bool(capi.sage_device_supported())


# ---------------------------------------------------------------------------------------------
# The entry-point names of the SageAttention README ("How to Use": sageattn(q, k, v,
# tensor_layout="HND", is_causal=False); "Available APIs": the INT8-QK kernels with FP8 or FP16
# P.V and the varlen one), mapped onto the calls above.
# ---------------------------------------------------------------------------------------------
def sageattn(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None, **kw):
    """sage_attn under the README's name (FP8 P.V with fp32 accumulation unless told otherwise)."""
    return sage_attn(q, k, v, tensor_layout, is_causal, sm_scale, **kw)


def sageattn_qk_int8_pv_fp8_cuda(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None,
                                 pv_accum_dtype="fp32", qk_quant_gran="per_block", smooth_v=False, out=None):
    """INT8 Q.K^T and FP8 (E4M3) P.V; pv_accum_dtype "fp32" or "fp16+fp32" / "fp32+fp16"."""
    return sage_attn(q, k, v, tensor_layout, is_causal, sm_scale, pv_accum_dtype, out=out, pv_dtype="fp8",
                     qk_quant_gran=qk_quant_gran, smooth_v=smooth_v)


def sageattn_qk_int8_pv_fp16_cuda(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None,
                                  pv_accum_dtype="fp32", qk_quant_gran="per_block", smooth_v=False, out=None):
    """INT8 Q.K^T and FP16 P.V; pv_accum_dtype "fp32", "fp16+fp32" or "fp16" (see pv_mode)."""
    return sage_attn(q, k, v, tensor_layout, is_causal, sm_scale, pv_accum_dtype, out=out, pv_dtype="fp16",
                     qk_quant_gran=qk_quant_gran, smooth_v=smooth_v)


def sageattn_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, is_causal=False, sm_scale=None,
                    pv_dtype="fp16", **kw):
    """sage_attn_varlen under the README's name; FP16 P.V by default, as the README lists it."""
    return sage_attn_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, is_causal, sm_scale,
                            pv_dtype=pv_dtype, **kw)
