"""The quantized attention method end to end, in float32 on the CPU.

Test infrastructure only (see the package docstring).  This is a diagnostic:
it predicts the error the method itself makes against exact attention, so a
test can tell a kernel bug from the cost of 8-bit arithmetic.

Steps, per (batch, query head, 128-row query block), over the key tiles in
increasing order (the blockwise online softmax; SageAttention README,
"Current Features"; qwbw.cn article, pitfalls, for the ``pv_accum_dtype``
options).  A key tile is ``tile`` keys, 128 by default: one INT8 K block.

1. S = Q8 . K8^T exactly in integers (K8 holds codes of K - mean(K)).
2. Dequantize in the log2 domain: s = S * f with
   f = (qs * ks) * (sm_scale * log2(e)), all float32 (qs of the query row's
   Q-scale group: its 128-, 32- or 1-token block).  Keys j >= Nk, and
   j > i + (Nk - Nq) under the (bottom-right aligned) causal mask, are
   excluded; a row that sees no key at all outputs zeros.
3. Online softmax against a reference max m: the reference moves to
   m' = max(m, row max of s) when that exceeds m by more than ``tau``
   (log2 units), else it stays (m' = m); p = 2^(s - m') <= 2^tau;
   alpha = 2^(m - m') (1 when it stays); l = l * alpha + sum(p).
   tau = 0 (the default) is the plain online softmax: the reference is
   always the running max.  A larger tau is a lazy reference, which moves
   (and rescales O) only when the running max has grown by more than tau;
   O and l share the reference, so the result differs only in how P rounds.
4. P is stored as E4M3(p * 448 * 2^-tau), so codes stay within +-448 (FP8
   P.V modes 0, 1), or as fp16(p) (FP16 P.V modes 2, 3).
5. PV: modes 0 and 2 (fp32 accumulation) O = O * alpha + P . V;
   modes 1 and 3 (fp16+fp32, "two-level accumulation") the tile's P . V is first
   rounded to float16 (a fresh fp16 accumulator per tile), then
   O = O * alpha + T.
6. out = O * vs / (P scale * l) (+ vm, V's token mean, when V was smoothed),
   P scale being 448 * 2^-tau (FP8) or 1 (FP16), rounded to the output dtype
   by the caller.
"""
from __future__ import annotations

import numpy as np

from . import fp8
from .quant import BLOCK, P_SCALE, PV_FP16, F32

LOG2E = 1.4426950408889634
TAU = 0.0  # the plain online softmax: the reference is the running max


def lazy_reading(pv_mode: int) -> dict:
    """The lazy-reference reading of steps 3-5 that the fused CUDA kernel takes: tau = 2 (O is
    rescaled only when the running max has grown by more than 2 in log2 units) and key tiles of
    128 keys for FP8 P.V, 64 for FP16 P.V (where a P row of fp16 values and a V^T row are each
    128 bytes).  The pages fix neither; pass it as ``emulate(..., **lazy_reading(mode))``."""
    return dict(tau=2.0, tile=64 if pv_mode in PV_FP16 else BLOCK)


def emulate(qz: dict, causal: bool, sm_scale: float, heads=None, q_blocks=None, tau: float = TAU,
            tile: int = BLOCK):
    """Emulated output float32 (len(heads), len(q_blocks) * 128, d) in HND row order.

    ``qz`` is the dict from ``quant.quantize``.  ``heads`` lists (b, hq) pairs
    (default: all), ``q_blocks`` the 128-row query blocks (default: all).
    ``tau`` and ``tile``: steps 3-5 (default: the plain online softmax over
    128-key tiles).  Rows beyond N are returned as NaN.
    """
    if tile not in (64, BLOCK):
        raise ValueError("tile must be 64 or 128 keys")
    B, Hq, Hkv, N, d = qz["B"], qz["Hq"], qz["Hkv"], qz["N"], qz["d"]
    Nk = qz.get("Nk", N)
    off = Nk - N                      # causal: query i sees keys j <= i + off
    G = Hq // Hkv
    nb = (N + BLOCK - 1) // BLOCK
    nbk = (Nk + BLOCK - 1) // BLOCK
    mode = qz["pv_mode"]
    hs = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else list(heads)
    qbs = list(range(nb)) if q_blocks is None else list(q_blocks)
    c = F32(F32(sm_scale) * F32(LOG2E))
    fp16_pv = mode in PV_FP16
    T = tile
    pscale = F32(1.0) if fp16_pv else F32(P_SCALE * 2.0 ** -tau)  # exact: 448 * 2^-tau
    out = np.full((len(hs), len(qbs) * BLOCK, d), np.nan, F32)
    for n, (b, h) in enumerate(hs):
        hk = h // G
        if fp16_pv:
            v8 = qz["v8"][b, hk].astype(np.float64)             # fp16 codes (Np, dp)
        else:
            v8 = fp8.decode(qz["v8"][b, hk]).astype(np.float64)  # E4M3 codes (Np, dp)
        for r, qb in enumerate(qbs):
            rows = qb * BLOCK + np.arange(BLOCK)
            q8 = qz["q8"][b, h, qb * BLOCK:(qb + 1) * BLOCK].astype(np.int64)
            qg = qz.get("q_gran", BLOCK)
            qsr = qz["qs"][b, h, rows // qg].astype(F32)           # Q scale of every row
            m = np.full(BLOCK, -np.inf, F32)
            l = np.zeros(BLOCK, F32)
            O = np.zeros((BLOCK, qz["dp"]), F32)
            n_tiles = nbk * BLOCK // T
            if causal:  # tiles up to the one holding the block's last visible key
                n_tiles = min(n_tiles, max(0, (qb * BLOCK + BLOCK - 1 + off) // T + 1))
            for j in range(n_tiles):
                keys = j * T + np.arange(T)
                if keys[0] >= Nk:
                    break
                k8 = qz["k8"][b, hk, j * T:(j + 1) * T].astype(np.int64)
                S = q8 @ k8.T
                valid = (keys[None, :] < Nk) & np.ones((BLOCK, 1), bool)
                if causal:
                    valid &= keys[None, :] <= rows[:, None] + off
                f = ((qsr * F32(qz["ks"][b, hk, keys[0] // BLOCK])).astype(F32) * c).astype(F32)  # (BLOCK,)
                smax = np.where(valid, S, np.iinfo(np.int64).min).max(axis=1)
                has = valid.any(axis=1)
                tmax = np.where(has, smax.astype(F32) * f, F32(-np.inf)).astype(F32)
                mc = np.maximum(m, tmax)
                upd = mc > (m + F32(tau)).astype(F32)             # the reference max moves
                m_new = np.where(upd, mc, m).astype(F32)
                with np.errstate(invalid="ignore"):
                    arg = (S.astype(np.float64) * f[:, None].astype(np.float64)
                           - m_new[:, None].astype(np.float64)).astype(F32)
                p = np.where(valid, np.exp2(arg), F32(0)).astype(F32)
                with np.errstate(invalid="ignore"):
                    alpha = np.where(np.isneginf(m), F32(0), np.exp2((m - m_new).astype(F32))).astype(F32)
                alpha = np.where(upd, alpha, F32(1)).astype(F32)
                l = (l * alpha + p.sum(axis=1, dtype=F32)).astype(F32)
                if fp16_pv:
                    p8 = p.astype(np.float16).astype(np.float64)
                else:
                    p8 = fp8.decode(fp8.encode((p * pscale).astype(F32)))
                pv = p8 @ v8[j * T:(j + 1) * T]                          # exact in float64
                if mode in (1, 3):
                    pv = pv.astype(np.float16)
                O = (O * alpha[:, None] + pv.astype(F32)).astype(F32)
                m = m_new
            vs = qz["vs"][b, hk].astype(F32)
            with np.errstate(divide="ignore", invalid="ignore"):
                o = (O * vs[None, :] / (pscale * l[:, None])).astype(F32)
            o[l == 0] = 0.0                                   # rows that saw no key
            if qz.get("smooth_v"):
                o = np.where((l > 0)[:, None], (o + qz["vm"][b, hk][None, :]).astype(F32), o)
            ok = rows < N
            out[n, r * BLOCK:(r + 1) * BLOCK][ok] = o[ok, :d]
    return out
