"""Seeded synthetic inputs for the quantized-attention path.

This module only draws random numbers and arranges them in the shapes and
layouts of the attention workloads; it holds none of the method's
arithmetic.  Both the CPU oracle (through the tests) and the CUDA path (through
the tests and the bench) are fed from here, so the two always see identical
fp16/bf16 bits.

Recipe (every draw is fp32 from a torch CPU generator, then rounded to the
workload dtype with round-to-nearest-even):

* ``normal``         Q, K, V i.i.d. N(0, 1).
* ``normal_koffset`` as ``normal``, plus one per-channel offset vector
  o ~ N(0, 3^2) of shape (d,) added to every K token of every batch and head
  (the "K has a channel-wise bias" case that mean-smoothing targets).
* ``normal_koutlier`` as ``normal``, then round(0.01 * Hkv * d) distinct
  (kv-head, channel) pairs, chosen by the seed, have K multiplied by 8 on all
  tokens and batches (outlier channels).
* ``uniform2``       Q, K, V i.i.d. U(-2, 2).

Each tensor has its own generator stream so that changing one tensor's shape
never changes another's values: stream 0 = Q, 1 = K, 2 = V, 3 = K offset,
4 = outlier choice.
"""
from __future__ import annotations

import dataclasses
from typing import Iterator

import torch

STREAM_Q, STREAM_K, STREAM_V, STREAM_OFFSET, STREAM_OUTLIER = 0, 1, 2, 3, 4

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, layout, mask and value recipe."""
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    dtype: str = "fp16"           # "fp16" | "bf16"
    layout: str = "HND"           # "HND" = (B,H,N,d), "NHD" = (B,N,H,d)
    causal: bool = False
    dist: str = "normal"          # see module docstring
    pv_mode: int = 0              # P.V: 0 = FP8, fp32 accumulation; 1 = FP8, fp16+fp32;
                                  # 2 = FP16 operands, fp32; 3 = FP16 operands, fp16+fp32
    seed: int = 0
    sm_scale: float | None = None  # None -> 1/sqrt(d)
    Nk: int | None = None          # key / value length when it differs from N (the query length)
    varlen: tuple = ()             # packed batch: ((nq, nk), ...) per sequence; then B = len(varlen)
    q_gran: int = 128              # query tokens per Q scale: 128 (per block), 32 (per warp), 1 (per thread)
    smooth_v: bool = False         # code V - mean_tokens(V), add the mean back

    @property
    def nk(self) -> int:
        return self.N if self.Nk is None else self.Nk

    def seqlens(self):
        """[(nq, nk)] of every sequence."""
        return list(self.varlen) if self.varlen else [(self.N, self.nk)] * self.B

    def ops(self) -> float:
        """Algorithmic attention operations: 4*Hq*d per visible (query, key) pair, i.e.
        4*B*Hq*Nq*Nk*d, and under the (bottom-right) causal mask only the visible pairs."""
        total = 0
        for nq, nk in self.seqlens():
            if self.causal:
                # query i sees min(nk, max(0, i + nk - nq + 1)) keys
                pairs = sum(min(nk, max(0, i + nk - nq + 1)) for i in range(nq)) if nq != nk else nq * (nq + 1) // 2
            else:
                pairs = nq * nk
            total += pairs
        v = 4.0 * self.Hq * self.d * total
        if self.causal and not self.varlen and self.Nk is None:
            v = 4.0 * self.B * self.Hq * self.N * self.N * self.d / 2  # the pages' convention: half of N^2
        return v

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the method is exercised on (image/video DiT self-attention,
# causal LLM prefill with GQA, head-dim padding sweep) plus the tiny one.
TINY = Workload("tiny_b1_h2_n256_d64", 1, 2, 2, 256, 64, "fp16", "HND", False, "normal", 0, 0, 1.0 / 8.0)
IMAGE_DIT = Workload("image_dit_b2_h24_n4096_d64", 2, 24, 24, 4096, 64, "bf16", "HND", False, "normal_koffset", 0, 2)
VIDEO_DIT = Workload("video_dit_b1_h24_n32768_d128_nhd", 1, 24, 24, 32768, 128, "bf16", "NHD", False,
                     "normal_koffset", 1, 3)
LLM_GQA = Workload("llm_causal_gqa_b4_hq32_hkv8_n8192_d128", 4, 32, 8, 8192, 128, "fp16", "HND", True,
                   "normal_koutlier", 0, 4)


def pad_sweep() -> Iterator[Workload]:
    """B=8, H=16, N in {1K,2K,4K,16K}, d in {96, 64}, causal and not, U(-2,2)."""
    for n in (1024, 2048, 4096, 16384):
        for d in (96, 64):
            for causal in (False, True):
                yield Workload(f"pad_sweep_b8_h16_n{n}_d{d}_{'causal' if causal else 'full'}",
                               8, 16, 16, n, d, "fp16", "HND", causal, "uniform2", 0, 5)


# The same inputs through the INT8-QK / FP16-PV kernel (fp32 and fp16+fp32 accumulation).
FP16_PV = [IMAGE_DIT.with_(name="image_dit_b2_h24_n4096_d64_pv16", pv_mode=2),
           VIDEO_DIT.with_(name="video_dit_b1_h24_n32768_d128_nhd_pv16", pv_mode=3),
           LLM_GQA.with_(name="llm_causal_gqa_b4_hq32_hkv8_n8192_d128_pv16", pv_mode=2)]

# The same inputs with finer Q scales and V smoothing.
OPTIONS = [IMAGE_DIT.with_(name="image_dit_b2_h24_n4096_d64_qthread_smoothv", q_gran=1, smooth_v=True),
           LLM_GQA.with_(name="llm_causal_gqa_b4_hq32_hkv8_n8192_d128_qwarp", q_gran=32)]

# The video-DiT inputs with fp32 P.V accumulation (the default mode) instead of fp16+fp32.
FP32_ACC = [VIDEO_DIT.with_(name="video_dit_b1_h24_n32768_d128_nhd_fp32acc", pv_mode=0)]

# Head dim 256 (the largest padded size): the kernel's 256-column output tile.
HEAD_DIM_256 = [Workload("d256_b2_h16_n8192", 2, 16, 16, 8192, 256, "fp16", "HND", False, "normal", 0, 6),
                Workload("d256_b2_h16_n8192_causal", 2, 16, 16, 8192, 256, "fp16", "HND", True, "normal", 0, 6)]

ALL = [TINY, IMAGE_DIT, VIDEO_DIT, LLM_GQA] + list(pad_sweep()) + FP16_PV + OPTIONS + FP32_ACC + HEAD_DIM_256

# Short video-DiT cases (8192 tokens, inputs still larger than L2) for detailed profiles of the
# fused kernel, whose counters take dozens of replays per launch.
PROFILE = [VIDEO_DIT.with_(name="video_dit_b1_h24_n8192_d128_nhd", N=8192),
           VIDEO_DIT.with_(name="video_dit_b1_h24_n8192_d128_nhd_fp32acc", N=8192, pv_mode=0)]
BY_NAME = {w.name: w for w in ALL + PROFILE}


def _gen(w: Workload, stream: int, seq: int = 0) -> torch.Generator:
    # One independent, reproducible stream per (workload seed, shape, tensor[, sequence]).
    key = (w.seed * 1_000_003 + stream * 7919 + w.N * 31 + w.d * 131 + w.B * 17 + w.Hq * 3
           + w.Hkv * 5 + (1 if w.causal else 0) + (w.Nk or 0) * 37 + seq * 104_729)
    return torch.Generator().manual_seed(key & 0x7FFF_FFFF_FFFF)


def _draw(w: Workload, stream: int, shape, seq: int = 0) -> torch.Tensor:
    g = _gen(w, stream, seq)
    if w.dist == "uniform2":
        return torch.rand(shape, generator=g, dtype=torch.float32) * 4.0 - 2.0
    return torch.randn(shape, generator=g, dtype=torch.float32)


def make_inputs(w: Workload):
    """Return (q, k, v) as contiguous CPU tensors of w.dtype in w.layout.

    Logical shapes are (B, Hq, N, d) for q and (B, Hkv, Nk, d) for k, v; for
    the NHD layout the same logical tensors are stored as (B, N, H, d).
    """
    if w.varlen:
        raise ValueError("packed workloads: use make_varlen_inputs")
    q, k, v = _logical(w, w.B, w.N, w.nk)
    dt = DTYPES[w.dtype]
    out = []
    for t in (q, k, v):
        t = t.to(dt)
        if w.layout == "NHD":
            t = t.transpose(1, 2)
        out.append(t.contiguous())
    return tuple(out)


def _logical(w: Workload, B: int, nq: int, nk: int, seq: int = 0):
    """float32 (B, Hq, nq, d), (B, Hkv, nk, d) x 2 of the workload's value recipe."""
    if w.dist not in ("normal", "normal_koffset", "normal_koutlier", "uniform2"):
        raise ValueError(f"unknown value recipe {w.dist!r}")
    q = _draw(w, STREAM_Q, (B, w.Hq, nq, w.d), seq)
    k = _draw(w, STREAM_K, (B, w.Hkv, nk, w.d), seq)
    v = _draw(w, STREAM_V, (B, w.Hkv, nk, w.d), seq)
    if w.dist == "normal_koffset":
        off = torch.randn((w.d,), generator=_gen(w, STREAM_OFFSET), dtype=torch.float32) * 3.0
        k += off
    elif w.dist == "normal_koutlier":
        n_out = max(1, round(0.01 * w.Hkv * w.d))
        pick = torch.randperm(w.Hkv * w.d, generator=_gen(w, STREAM_OUTLIER))[:n_out]
        for p in pick.tolist():
            k[:, p // w.d, :, p % w.d] *= 8.0
    return q, k, v


def make_varlen_inputs(w: Workload):
    """Packed batch of w.varlen's sequences: q (total_q, Hq, d), k and v (total_k, Hkv, d) of w.dtype
    (sequence b's tokens after those of b - 1; each sequence drawn from its own streams, the K
    offset / outlier channels shared), and cu_seqlens_q, cu_seqlens_k as int32 CPU tensors."""
    qs, ks, vs = [], [], []
    cq, ck = [0], [0]
    dt = DTYPES[w.dtype]
    for b, (nq, nk) in enumerate(w.varlen):
        q, k, v = _logical(w, 1, nq, nk, seq=b)
        qs.append(q[0].transpose(0, 1))
        ks.append(k[0].transpose(0, 1))
        vs.append(v[0].transpose(0, 1))
        cq.append(cq[-1] + nq)
        ck.append(ck[-1] + nk)
    pack = lambda ts: torch.cat(ts, 0).to(dt).contiguous()
    return (pack(qs), pack(ks), pack(vs), torch.tensor(cq, dtype=torch.int32), torch.tensor(ck, dtype=torch.int32))


def sm_scale_of(w: Workload) -> float:
    return w.sm_scale if w.sm_scale is not None else 1.0 / (w.d ** 0.5)
