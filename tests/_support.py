"""Shared helpers for the GPU parity tests: moving oracle results to the
device layouts, slicing heads, and the tolerance checks (derived below)."""
from __future__ import annotations

import numpy as np
import torch

import workloads as W
from oracle import quant

# ---------------------------------------------------------------------------------------------
# Tolerances
#
# Against the CPU emulation of the method (same codes, the fused kernel's lazy-reference reading:
# emulate(..., **emulate.lazy_reading(mode))): the only differences are the output rounding (bf16
# half ulp = 2^-9 relative), float32 summation order and the GPU's ex2.approx (a few ulp).  The
# last one can, rarely, move p*448 across an E4M3 rounding boundary (probability ~2^-17 per
# score), changing one P code by one step (<= 2^-3 of that p).  So >= 99.99% of elements must lie
# within 2^-7 |emul| + 2e-3, and every element within 2^-3 max|V| (one flipped code of a key whose
# weight is close to 1).
#
# Against exact fp64 attention, anchored on the method's own error on the same rows:
# * every element: |gpu - exact| <= |emul - exact| + 2^-7 |emul| + 2e-3 (>= 99.99% of elements;
#   the rest within |emul - exact| + 2^-3 max|V|, the code flips above);
# * cosine similarity >= 0.999 (inputs with x8 K outlier channels: the method itself can fall
#   below it, as the shared per-block K scale grows; there >= cos(emul, exact) - 2e-4);
# * the target accuracy, max |gpu - exact| <= 2e-2, for unit-variance inputs (Q, K, V ~ N(0, 1),
#   K also with a per-channel offset, which smoothing removes), on rows that see enough keys: >= 256
#   with FP16 P.V, >= 1024 with FP8 P.V.  The relaxation on shorter rows is the method's, not the
#   kernel's, and the emulation alone shows it (max over rows by visible keys, causal N(0,1) cases):
#   FP16 P.V 0.027 (1-31 keys), 0.019 (32-127), 0.023 (128-255), then <= 0.010 -- on short rows the
#   INT8 Q/K score error moves a peaked softmax; FP8 P.V 0.11 (1-31), 0.03-0.05 (32-255), 0.021
#   (256-511), 0.023 (512-1023), then <= 0.012 -- each E4M3 code of P and V is off by up to 2^-4
#   relative, and a row averages that error over its keys.
# Quantization codes, scales, K mean and int32 scores: bit-exact (other tests).
# ---------------------------------------------------------------------------------------------
COS_MIN = 0.999
TARGET_MAX_ABS = 2e-2
FP8_TARGET_MIN_KEYS, FP16_TARGET_MIN_KEYS = 1024, 256
TIGHT_REL, TIGHT_ABS, TIGHT_FRAC = 2.0 ** -7, 2e-3, 0.9999
UNIT_VARIANCE = ("normal", "normal_koffset")


def cos_sim(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def check_vs_exact(out, ref, emul, nkeys, vmax, what="", dist="normal", pv_mode=0):
    """out, ref, emul: (..., rows, d) float64 -- the GPU output, exact attention and the method's
    emulation (lazy reading) on the same rows; nkeys: (rows,) visible keys of each row; dist: the
    inputs' value recipe (workloads.py); pv_mode: the P.V mode.  Returns the measured figures."""
    out, ref, emul = (np.asarray(x, np.float64) for x in (out, ref, emul))
    err = np.abs(out - ref)
    own = np.abs(emul - ref)
    c = cos_sim(out, ref)
    cmin = COS_MIN if dist != "normal_koutlier" else min(COS_MIN, cos_sim(emul, ref) - 2e-4)
    assert c >= cmin, f"{what}: cosine {c:.6f} < {cmin:.6f}"
    band = own + TIGHT_REL * np.abs(emul) + TIGHT_ABS
    frac = float((err <= band).mean())
    assert frac >= TIGHT_FRAC, f"{what}: only {frac:.6f} of elements within the method's own error + " \
                               f"2^-7|emul| + 2e-3 (worst excess {float((err - band).max()):.4g})"
    worst = float((err - own).max())
    assert worst <= 0.125 * vmax, f"{what}: {worst:.4f} beyond the method's own error > 2^-3 max|V|"
    nk = np.asarray(nkeys)
    min_keys = FP16_TARGET_MIN_KEYS if pv_mode & 2 else FP8_TARGET_MIN_KEYS
    rows = nk >= min_keys
    target = None
    if dist in UNIT_VARIANCE and rows.any():
        target = float(err[..., rows, :].max())
        assert target <= TARGET_MAX_ABS, f"{what}: max abs {target:.4f} > {TARGET_MAX_ABS} on rows with >= " \
                                         f"{min_keys} keys"
    return dict(cos=c, max_abs=float(err.max()), max_abs_target_rows=target, frac_in_band=frac)


def check_vs_emulation(out, emul, vmax, what=""):
    err = np.abs(out - emul)
    tight = err <= TIGHT_REL * np.abs(emul) + TIGHT_ABS
    frac = tight.mean()
    assert frac >= TIGHT_FRAC, f"{what}: only {frac:.6f} of elements agree with the emulation " \
                               f"(worst {err.max():.4g} at {np.unravel_index(err.argmax(), err.shape)})"
    assert err.max() <= 0.125 * vmax, f"{what}: {err.max():.4f} > 2^-3 max|V|"
    return float(frac)


# ---------------------------------------------------------------------------------------------
def cuda(t: torch.Tensor) -> torch.Tensor:
    return t.cuda().contiguous()


def slice_heads(t: torch.Tensor, layout: str, b: int, heads) -> torch.Tensor:
    """Keep batch b and the given heads (keeps the layout)."""
    t = t[b:b + 1]
    return (t[:, heads] if layout == "HND" else t[:, :, heads]).contiguous()


def oracle_to_device(qz: dict) -> dict:
    """Oracle codes/scales -> CUDA tensors in the library's layouts (V transposed)."""
    v8t = np.ascontiguousarray(qz["v8"].transpose(0, 1, 3, 2))
    z = {k: torch.from_numpy(np.ascontiguousarray(qz[k])).cuda() for k in ("q8", "qs", "k8", "ks", "km", "vs", "vm")}
    z["v8t"] = torch.from_numpy(v8t).cuda()
    z.update({k: qz[k] for k in ("B", "Hq", "Hkv", "N", "d")})
    z["pv_dtype"] = "fp16" if qz["pv_mode"] & 2 else "fp8"
    z["qk_quant_gran"] = {128: "per_block", 32: "per_warp", 1: "per_thread"}[qz.get("q_gran", 128)]
    z["smooth_v"] = bool(qz.get("smooth_v", False))
    return z


def out_hnd(out: torch.Tensor, layout: str) -> np.ndarray:
    return quant.to_hnd(out.float().cpu(), layout).astype(np.float64)


def nkeys(N: int, causal: bool, rows=None) -> np.ndarray:
    r = np.arange(N) if rows is None else np.asarray(rows)
    return r + 1 if causal else np.full(len(r), N)


def vmax_of(v) -> float:
    return float(v.float().abs().max())


def pv_name(w: W.Workload) -> str:
    """pv_accum_dtype of the workload's P.V mode."""
    return "fp16+fp32" if w.pv_mode & 1 else "fp32"


GRAN_NAME = {128: "per_block", 32: "per_warp", 1: "per_thread"}


def opt_kw(w: W.Workload) -> dict:
    """Keyword options of the Python binding for the workload's Q granularity and V smoothing."""
    return dict(qk_quant_gran=GRAN_NAME[w.q_gran], smooth_v=w.smooth_v)


def pv_dtype(w: W.Workload) -> str:
    """pv_dtype (P.V operands) of the workload's P.V mode."""
    return "fp16" if w.pv_mode & 2 else "fp8"
