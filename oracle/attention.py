"""Exact scaled-dot-product attention in float64.

Test infrastructure only (see the package docstring).

This is the definition the quantized method approximates: the two stages
"scores = Q K^T, then softmax(scores) times V" (trdm.cn article on building
SageAttention for the RX 9070XT, section 2.2), with ``sm_scale`` and
``is_causal`` behaving as in SDPA (qwbw.cn article, "one-line replacement"
section), fp16/bf16 q, k, v in the HND (B, H, N, d) or NHD (B, N, H, d)
layout (SageAttention README, "How to Use"), and grouped-query attention
with num_qo_heads divisible by num_kv_heads (qwbw.cn article, pitfalls).

q and k, v may have different sequence lengths, and a batch may hold
sequences of different lengths packed token by token (SageAttention README,
news of 2024-11-11 and 2024-11-12: different sequence lengths between q and
k, v; ``sageattn_varlen``).

Readings: query head h uses kv head h // (Hq / Hkv) (contiguous groups, the
SDPA repeat_interleave convention); the causal mask keeps key j for query i
iff j <= i + (Nk - Nq), i.e. the last query sees every key (bottom-right
alignment; the pages do not say, and with Nq = Nk both alignments agree); a
query row that sees no key at all outputs zeros; the unpadded head dim d is
used throughout, since padding with zeros changes no dot product.  A packed
(varlen) batch is one independent attention per sequence.
"""
from __future__ import annotations

import numpy as np

from .quant import to_hnd


def _head_rows(qh, kh, vh, rows, causal, sm_scale):
    """Attention for the selected query rows of one head, all in float64."""
    if kh.shape[0] == 0:                                  # no keys: every row sees nothing
        return np.zeros((len(rows), vh.shape[1]))
    s = (qh[rows] @ kh.T) * sm_scale                      # (r, Nk)
    if causal:
        j = np.arange(kh.shape[0])[None, :]
        s = np.where(j <= np.asarray(rows)[:, None] + (kh.shape[0] - qh.shape[0]), s, -np.inf)
    seen = np.isfinite(s).any(axis=1)                     # rows that see at least one key
    m = np.where(seen[:, None], s.max(axis=1, keepdims=True), 0.0)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return np.where(seen[:, None], (p @ vh) / np.where(l > 0, l, 1.0), 0.0)


def attention_f64(q, k, v, layout="HND", causal=False, sm_scale=None, heads=None, rows=None,
                  chunk=512):
    """out[b, h, i, :] = sum_j softmax_j(sm_scale * q_i . k_j [masked]) v_j, float64.

    q: (B, Hq, Nq, d), k/v: (B, Hkv, Nk, d) in ``layout``.  ``heads`` is an
    optional list of (b, hq) pairs and ``rows`` an optional list of query rows;
    the result is then an array (len(heads), len(rows), d) for those only.
    Without them the full (B, Hq, Nq, d) output in HND order is returned.
    """
    qf, kf, vf = (to_hnd(t, layout).astype(np.float64) for t in (q, k, v))
    B, Hq, N, d = qf.shape
    Hkv = kf.shape[1]
    if kf.shape[2] != vf.shape[2]:
        raise ValueError("k and v must have the same length")
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


def attention_varlen_f64(q, k, v, cu_seqlens_q, cu_seqlens_k, causal=False, sm_scale=None):
    """Packed batch: q (total_q, Hq, d), k/v (total_k, Hkv, d); sequence b owns query tokens
    cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1 and key tokens cu_seqlens_k[b] .. cu_seqlens_k[b+1] - 1.
    Returns float64 (total_q, Hq, d): each sequence's attention on its own tokens."""
    qf, kf, vf = (np.asarray(t.float().numpy() if hasattr(t, "float") else t, np.float64) for t in (q, k, v))
    cq, ck = np.asarray(cu_seqlens_q, np.int64), np.asarray(cu_seqlens_k, np.int64)
    out = np.zeros(qf.shape)
    for b in range(len(cq) - 1):
        qs, ks = slice(cq[b], cq[b + 1]), slice(ck[b], ck[b + 1])
        if cq[b + 1] == cq[b]:
            continue
        o = attention_f64(qf[None, qs], kf[None, ks], vf[None, ks], "NHD", causal, sm_scale)
        out[qs] = o[0].transpose(1, 0, 2)
    return out
