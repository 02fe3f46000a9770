"""Exact scaled-dot-product attention in float64.

Test infrastructure only (see the package docstring).

This is the definition the quantized method approximates: the two stages
"scores = Q K^T, then softmax(scores) times V" (trdm.cn article on building
SageAttention for the RX 9070XT, section 2.2), with ``sm_scale`` and
``is_causal`` behaving as in SDPA (qwbw.cn article, "one-line replacement"
section), fp16/bf16 q, k, v in the HND (B, H, N, d) or NHD (B, N, H, d)
layout (SageAttention README, "How to Use"), and grouped-query attention
with num_qo_heads divisible by num_kv_heads (qwbw.cn article, pitfalls).

Readings: query head h uses kv head h // (Hq / Hkv) (contiguous groups, the
SDPA repeat_interleave convention); the causal mask keeps key j for query i
iff j <= i (Nq = Nk); the unpadded head dim d is used throughout, since
padding with zeros changes no dot product.
"""
from __future__ import annotations

import numpy as np

from .quant import to_hnd


def _head_rows(qh, kh, vh, rows, causal, sm_scale):
    """Attention for the selected query rows of one head, all in float64."""
    s = (qh[rows] @ kh.T) * sm_scale                      # (r, N)
    if causal:
        j = np.arange(kh.shape[0])[None, :]
        s = np.where(j <= np.asarray(rows)[:, None], s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return (p @ vh) / p.sum(axis=1, keepdims=True)


def attention_f64(q, k, v, layout="HND", causal=False, sm_scale=None, heads=None, rows=None,
                  chunk=512):
    """out[b, h, i, :] = sum_j softmax_j(sm_scale * q_i . k_j [masked]) v_j, float64.

    q: (B, Hq, N, d), k/v: (B, Hkv, N, d) in ``layout``.  ``heads`` is an
    optional list of (b, hq) pairs and ``rows`` an optional list of query rows;
    the result is then an array (len(heads), len(rows), d) for those only.
    Without them the full (B, Hq, N, d) output in HND order is returned.
    """
    qf, kf, vf = (to_hnd(t, layout).astype(np.float64) for t in (q, k, v))
    B, Hq, N, d = qf.shape
    Hkv = kf.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be divisible by Hkv")
    G = Hq // Hkv
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    full = heads is None and rows is None
    hs = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else list(heads)
    rs = np.arange(N) if rows is None else np.asarray(rows)
    out = np.empty((len(hs), len(rs), d))
    for n, (b, h) in enumerate(hs):
        kh, vh = kf[b, h // G], vf[b, h // G]
        for c in range(0, len(rs), chunk):
            out[n, c:c + chunk] = _head_rows(qf[b, h], kh, vh, rs[c:c + chunk], causal, sm_scale)
    if full:
        return out.reshape(B, Hq, N, d)
    return out
