"""Derives the polynomial the fused kernel uses for part of its exponentials.

The kernel computes 2^x as 2^n * 2^r with n = round(x) and r = x - n in
[-1/2, 1/2]; 2^r is approximated by a degree-4 polynomial whose coefficients
are fitted here: a least-squares fit of the RELATIVE error on Chebyshev nodes of
[-1/2, 1/2] (which is close to the minimax fit), with the constant term pinned to
1 so that 2^0 is exact.  Run it to print the float32 constants pasted into
attn.cu; tests/test_exp2_poly.py checks that the two agree and that the
polynomial's relative error, evaluated the way the kernel does it in float32,
stays below 2^-17 over [-1/2, 1/2].

    python quantized_attention_int8_b200/csrc/exp2_poly.py
"""
from __future__ import annotations

import numpy as np

DEGREE = 4


def fit(degree: int = DEGREE, nodes: int = 4001) -> np.ndarray:
    """Coefficients c[0..degree] (c[0] = 1) of sum c_k r^k ~ 2^r on [-1/2, 1/2]."""
    k = np.arange(nodes)
    r = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)          # Chebyshev nodes
    target = np.exp2(r)
    # minimise sum ((1 + sum_{k>=1} c_k r^k) / 2^r - 1)^2
    A = np.stack([r ** j / target for j in range(1, degree + 1)], axis=1)
    b = 1.0 - 1.0 / target
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    return np.concatenate([[1.0], c])


def coefficients_f32() -> np.ndarray:
    return fit().astype(np.float32)


def eval_f32(r: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Horner in float32 with one rounding per step, as the kernel's fused multiply-adds do."""
    r = np.asarray(r, np.float32)
    acc = np.full_like(r, c[-1], dtype=np.float32)
    for ck in c[-2::-1]:
        acc = (acc.astype(np.float64) * r.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return acc


def max_rel_error(c: np.ndarray, n: int = 200001) -> float:
    r = np.linspace(-0.5, 0.5, n).astype(np.float32)
    return float(np.max(np.abs(eval_f32(r, c).astype(np.float64) / np.exp2(r.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = coefficients_f32()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r:>24}  (0x{np.float32(v).view(np.uint32):08X})")
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c):.3e} (2^{np.log2(max_rel_error(c)):.1f})")
