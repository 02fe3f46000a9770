"""Quantization step of SageAttention-style attention, emulated on the CPU.

Test infrastructure only (see the package docstring).

What the pages fix (SageAttention README, "Current Features"; qwbw.cn
article, pitfalls section):

* Q K^T runs on INT8 codes, with "smoothing" of K and scales at "varying
  granularities";
* P V runs in FP8;
* head_dim is zero-padded to 64, 128 or 256 when it is none of those.

Readings adopted where the pages give no formula or number (each one is a
choice a reader can check here, and the CUDA path implements the same one):

* Smoothing subtracts the per-channel mean of K over all N tokens of a
  (batch, kv-head) (softmax is invariant to it: every score of query row i
  shifts by q_i . mean(K)).  The pages give no summation order; the mean is
  summed in float32 in this fixed order: each 128-token block is split into
  8 groups of 16 consecutive tokens, each group is summed token by token from
  +0.0 (tokens >= N skipped, so an empty group is +0.0), the block partial is
  the pairwise tree ((g0 + g1) + (g2 + g3)) + ((g4 + g5) + (g6 + g7)), the
  block partials are added one by one in block order from +0.0, and the total
  is divided by float(N) with one IEEE division.
* Q and K - mean(K) get symmetric INT8 codes per (batch, head, 128-token
  block) over all channels: amax = max |x| over the block's real tokens and
  channels; inv = 127 / amax (one IEEE float32 division; 0 when amax = 0);
  code = clamp(rint(x * inv), -127, 127) with rint rounding half to even;
  scale = amax / 127.  Padded tokens and channels get code 0.
* V gets FP8 E4M3 codes per (batch, kv-head, channel) over all tokens:
  inv = VMAX / amax, code = E4M3_rne_satfinite(v * inv), scale = amax / VMAX.
  VMAX is 448 for fp32 PV accumulation and 1 for the fp16+fp32 (two-level)
  accumulation, so that one 128-key tile's fp16 partial sum is bounded by
  128 * 448 * 1 = 57344 < 65504 and cannot overflow.
* For the FP16 P.V variant (README "Available APIs": sageattn_qk_int8_pv_fp16_cuda)
  V is kept in fp16 with the same per-channel scaling to [-1, 1]: inv = 1 / amax,
  code = fp16_rne(v * inv), scale = amax.  (Q and K are quantized as above.)
* "Varying granularities" for Q (README "Current Features"; "per-thread
  quantization", news of 2024-12-20): Q may take one scale per 128 tokens
  (per block, the default), per 32 tokens (per warp: the rows one warp of the
  CUDA kernel owns) or per token (per thread: one thread of the kernel owns
  one query row).  The codes and scales follow the INT8 rule above with the
  block of that many tokens.  K keeps one scale per 128-token block.
* Optional V smoothing (the "thorough outlier smoothing" of the SageAttention2
  title): V - mean_tokens(V) is coded instead of V, the mean summed in the same
  fixed order as K's, and the mean is added back to the output (each row of
  softmax weights sums to 1, so the result is unchanged in exact arithmetic).
* All float arithmetic is IEEE float32 with round-to-nearest-even and no
  fused multiply-add; numpy float32 operations satisfy this.
"""
from __future__ import annotations

import numpy as np

from . import fp8

BLOCK = 128              # tokens per Q/K scale block and per KV tile
P_SCALE = 448.0          # p in [0, 1] is stored as E4M3(p * 448)
# PV modes: 0 = FP8 P.V, fp32 accumulation; 1 = FP8 P.V, fp16+fp32; 2 = FP16 P.V, fp32;
# 3 = FP16 P.V, fp16+fp32.  V code range per mode:
VMAX = {0: 448.0, 1: 1.0, 2: 1.0, 3: 1.0}
PV_FP16 = (2, 3)
F32 = np.float32


def padded_dim(d: int) -> int:
    """Smallest of 64, 128, 256 that holds d (qwbw.cn article, pitfalls: pad_qkv)."""
    for p in (64, 128, 256):
        if d <= p:
            return p
    raise ValueError(f"head_dim {d} > 256 is not supported")


def n_blocks(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK


def to_hnd(x, layout: str) -> np.ndarray:
    """Any fp16/bf16 tensor or array -> float32 numpy (B, H, N, d); widening is exact."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.float().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x, dtype=np.float32)
    if layout == "NHD":
        x = x.transpose(0, 2, 1, 3)
    elif layout != "HND":
        raise ValueError(layout)
    return np.ascontiguousarray(x)


GROUPS, GROUP = 8, 16     # a 128-token block = 8 groups of 16 consecutive tokens


def k_token_mean(k: np.ndarray) -> np.ndarray:
    """Per-channel mean of K over tokens, in the fixed float32 order described above.

    k: float32 (B, H, N, d) -> float32 (B, H, d).
    """
    B, H, N, d = k.shape
    nb = n_blocks(N)
    kp = np.zeros((B, H, nb * BLOCK, d), F32)
    kp[:, :, :N] = k
    kg = kp.reshape(B, H, nb, GROUPS, GROUP, d)
    tok = (np.arange(nb)[:, None, None] * BLOCK + np.arange(GROUPS)[None, :, None] * GROUP
           + np.arange(GROUP)[None, None, :])                # token index of (block, group, t)
    gs = np.zeros((B, H, nb, GROUPS, d), F32)
    for t in range(GROUP):
        valid = tok[:, :, t] < N                          # skip tokens beyond N
        gs = np.where(valid[None, None, :, :, None], gs + kg[:, :, :, :, t, :], gs)
    part = ((gs[:, :, :, 0] + gs[:, :, :, 1]) + (gs[:, :, :, 2] + gs[:, :, :, 3])) + \
           ((gs[:, :, :, 4] + gs[:, :, :, 5]) + (gs[:, :, :, 6] + gs[:, :, :, 7]))
    total = np.zeros((B, H, d), F32)
    for b in range(nb):
        total = total + part[:, :, b, :]
    return total / F32(N)


def int8_per_block(x: np.ndarray, dp: int, rows: int = BLOCK):
    """Symmetric INT8 codes of x (float32 (B,H,N,d)) with one scale per (b, h, block of
    ``rows`` tokens) (128: per block; 32: per warp; 1: per token).

    Returns codes int8 (B, H, N_pad, dp) and scales float32 (B, H, N_pad / rows).
    """
    B, H, N, d = x.shape
    nb = n_blocks(N)
    xp = np.zeros((B, H, nb * BLOCK, dp), F32)
    xp[:, :, :N, :d] = x                               # padding is exact zeros
    xb = xp.reshape(B, H, nb * BLOCK // rows, rows, dp)
    amax = np.abs(xb).max(axis=(3, 4))                 # zeros cannot raise the max
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, F32(127.0) / amax, F32(0.0)).astype(F32)
    prod = (xb * inv[:, :, :, None, None]).astype(F32)
    codes = np.clip(np.rint(prod), -127, 127).astype(np.int8)
    scale = (amax / F32(127.0)).astype(F32)
    return codes.reshape(B, H, nb * BLOCK, dp), scale


def fp8_per_channel(v: np.ndarray, dp: int, vmax: float):
    """Per-(b, h, channel) E4M3 codes of v (float32 (B,H,N,d)) over all tokens.

    Returns codes uint8 (B, H, N_pad, dp) and scales float32 (B, H, dp).
    """
    B, H, N, d = v.shape
    nb = n_blocks(N)
    amax = np.zeros((B, H, dp), F32)
    amax[:, :, :d] = np.abs(v).max(axis=2)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, F32(vmax) / amax, F32(0.0)).astype(F32)
    vp = np.zeros((B, H, nb * BLOCK, dp), F32)
    vp[:, :, :N, :d] = v
    prod = (vp * inv[:, :, None, :]).astype(F32)
    codes = fp8.encode(prod)
    # padded tokens are +0.0 * inv = +0.0 -> code 0; padded channels have inv 0
    scale = (amax / F32(vmax)).astype(F32)
    return codes, scale


def fp16_per_channel(v: np.ndarray, dp: int):
    """Per-(b, h, channel) fp16 codes of v / amax (float32 (B,H,N,d)) over all tokens.

    Returns codes float16 (B, H, N_pad, dp) and scales float32 (B, H, dp) = amax.
    """
    B, H, N, d = v.shape
    nb = n_blocks(N)
    amax = np.zeros((B, H, dp), F32)
    amax[:, :, :d] = np.abs(v).max(axis=2)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, F32(1.0) / amax, F32(0.0)).astype(F32)
    vp = np.zeros((B, H, nb * BLOCK, dp), F32)
    vp[:, :, :N, :d] = v
    codes = (vp * inv[:, :, None, :]).astype(F32).astype(np.float16)   # one RNE rounding to fp16
    return codes, amax.copy()


Q_GRANS = (128, 32, 1)   # query tokens per Q scale: per block, per warp, per thread


def quantize(q, k, v, layout: str = "HND", pv_mode: int = 0, q_gran: int = BLOCK, smooth_v: bool = False) -> dict:
    """The whole quantization step for one attention call.

    q: (B, Hq, Nq, d), k and v: (B, Hkv, Nk, d) in ``layout`` (fp16/bf16 torch
    tensors or arrays).  Returns a dict of numpy arrays:
      q8 int8 (B,Hq,Nq_pad,dp), qs f32 (B,Hq,nbq), k8 int8 (B,Hkv,Nk_pad,dp),
      ks f32 (B,Hkv,nbk), km f32 (B,Hkv,dp), v8 (B,Hkv,Nk_pad,dp) V codes (uint8 E4M3
      for PV modes 0/1, float16 for the FP16 P.V modes 2/3), vs f32 (B,Hkv,dp),
      plus the sizes (N = Nq, Nk).  Q and K are quantized on their own lengths.
    q_gran: query tokens per Q scale (qs then has Nq_pad / q_gran entries per head).
    smooth_v: code V - vm (vm f32 (B,Hkv,dp), the token mean; zeros when off).
    """
    if q_gran not in Q_GRANS:
        raise ValueError(f"q_gran must be one of {Q_GRANS}")
    qf, kf, vf = (to_hnd(t, layout) for t in (q, k, v))
    B, Hq, N, d = qf.shape
    Hkv = kf.shape[1]
    dp = padded_dim(d)
    km = k_token_mean(kf)
    ksm = (kf - km[:, :, None, :]).astype(F32)        # one float32 subtraction
    q8, qs = int8_per_block(qf, dp, q_gran)
    k8, ks = int8_per_block(ksm, dp)
    vm = np.zeros((B, Hkv, dp), F32)
    if smooth_v:
        vmean = k_token_mean(vf)                      # same fixed summation order as K's mean
        vm[:, :, :d] = vmean
        vf = (vf - vmean[:, :, None, :]).astype(F32)  # one float32 subtraction
    if pv_mode in PV_FP16:
        v8, vs = fp16_per_channel(vf, dp)      # "v8" holds the fp16 codes in these modes
    else:
        v8, vs = fp8_per_channel(vf, dp, VMAX[pv_mode])
    kmp = np.zeros((B, Hkv, dp), F32)
    kmp[:, :, :d] = km
    return dict(q8=q8, qs=qs, k8=k8, ks=ks, km=kmp, v8=v8, vs=vs, vm=vm,
                B=B, Hq=Hq, Hkv=Hkv, N=N, Nk=kf.shape[2], d=d, dp=dp, pv_mode=pv_mode, q_gran=q_gran,
                smooth_v=bool(smooth_v))


def qk_int32(q8: np.ndarray, k8: np.ndarray) -> np.ndarray:
    """Exact integer scores S = Q8 . K8^T for one head: (Nq, dp) x (Nk, dp) -> int32.

    |S| <= 256 * 127^2 < 2^31, so int32 holds every value exactly.
    """
    s = q8.astype(np.int64) @ k8.astype(np.int64).T
    assert np.abs(s).max(initial=0) < 2 ** 31
    return s.astype(np.int32)
