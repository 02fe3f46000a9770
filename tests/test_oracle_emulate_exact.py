"""Worked cases for the method's emulation (CPU only), with outputs known in closed form.

The inputs are built so that every quantization step is exact:
- Q rows are A * e_0 (channel 0 only): one INT8 code, 127, per row.
- K's channel 0 is c + delta or c - delta, in equal numbers per 128-key block, so the token mean
  is c exactly and every K code is +-127.
- V holds values that its per-channel scale maps exactly onto E4M3 (or fp16) codes.
With sm_scale = ln 2 the dequantized score of a key is +-delta in log2 units, so the online softmax
weights are exact powers of two and every P code is exact.  The output is then a weighted mean
of V rows whose weights follow from the method's definition: p = 2^(s - m) against the reference
max m, which moves when a tile's max exceeds it by more than tau (0: the plain online softmax,
whose reference is the running max; 2: the lazy reading of the fused kernel), and O and l
rescaled by alpha = 2^(m_old - m_new) when it moves.  The expected values below are written from
those weights alone, so a wrong P scale (448 * 2^-tau), V scale, row sum, rescale factor, tile
order or mask index in the emulation fails them.  Every case runs under both readings.
"""
import math

import numpy as np
import pytest
import torch

from oracle import emulate, quant

LN2 = math.log(2.0)
D = 64
C = 2.0  # K's channel-0 centre (its token mean)


def _inputs(deltas, v_levels, seed, n_q=128):
    """Q (n_q rows), K (128 keys per entry of `deltas`: the first 64 at C + delta, the next 64 at
    C - delta) and V (values drawn from `v_levels`, with |v| = 1 at key 0 of every channel)."""
    n = 128 * len(deltas)
    q = torch.zeros(1, 1, n_q, D)
    q[..., 0] = 1.0
    k = torch.zeros(1, 1, n, D)
    for t, dl in enumerate(deltas):
        k[0, 0, t * 128:t * 128 + 64, 0] = C + dl
        k[0, 0, t * 128 + 64:t * 128 + 128, 0] = C - dl
    rng = np.random.default_rng(seed)
    v = rng.choice(np.asarray(v_levels, np.float64), size=(n, D))
    v[0] = np.where(rng.random(D) < 0.5, -1.0, 1.0)  # channel amax exactly 1
    vt = torch.from_numpy(v).view(1, 1, n, D)
    return q.half(), k.half(), vt.half(), v


def _weights(deltas, tau=2.0, tile=128):
    """Per-key weight (p relative to the final reference) and the row sum, from the method's rules,
    for a row that sees every key.  Keys come in tiles of `tile`; score = +delta for the first
    half of each 128-key block, -delta for the second."""
    n = 128 * len(deltas)
    x = np.array([deltas[j // 128] * (1 if j % 128 < 64 else -1) for j in range(n)], np.float64)
    m = -math.inf
    w = np.zeros(n)
    for t0 in range(0, n, tile):
        xs = x[t0:t0 + tile]
        mc = max(m, xs.max())
        if mc > m + tau:  # the reference moves: everything so far scales by 2^(m - mc)
            w[:t0] *= 0.0 if m == -math.inf else 2.0 ** (m - mc)
            m = mc
        w[t0:t0 + tile] = 2.0 ** (xs - m)
    return w


PLAIN = dict(tau=0.0, tile=128)
READINGS = {"plain": lambda mode: PLAIN, "lazy": emulate.lazy_reading}


def _run(deltas, mode, v_levels, reading, causal=False, seed=0):
    q, k, v, vnp = _inputs(deltas, v_levels, seed)
    qz = quant.quantize(q, k, v, "HND", mode)
    # preconditions of the construction: every code is the intended exact value
    assert (np.abs(qz["q8"][0, 0, :128, 0]) == 127).all()
    n = 128 * len(deltas)
    assert (np.abs(qz["k8"][0, 0, :n, 0]) == 127).all() and (qz["k8"][0, 0, :n, 1:] == 0).all()
    assert qz["km"][0, 0, 0] == C
    return emulate.emulate(qz, causal, LN2, **READINGS[reading](mode))[0, :128].astype(np.float64), vnp


@pytest.mark.parametrize("reading", sorted(READINGS))
@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_one_tile_weights_one_and_half(mode, reading):
    # 64 keys at weight 1 and 64 at weight 1/2 (lazy FP16 P.V: two 64-key tiles, same weights)
    levels = [-0.25, 0.0, 0.25] if mode == 1 else [-1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0]
    out, v = _run([0.5], mode, levels, reading)
    want = (v[:64].sum(0) + 0.5 * v[64:128].sum(0)) / 96.0
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=2e-6)


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_one_tile_causal_prefix_weights(reading):
    # row i sees keys 0..i: rows < 64 average their prefix; later rows add keys at weight 1/2
    out, v = _run([0.5], 0, [-1.0, -0.5, 0.0, 0.5, 1.0], reading, causal=True)
    for i in range(128):
        w = np.where(np.arange(i + 1) < 64, 1.0, 0.5)
        want = (w[:, None] * v[:i + 1]).sum(0) / w.sum()
        np.testing.assert_allclose(out[i], want, rtol=0, atol=2e-6, err_msg=f"row {i}")


@pytest.mark.parametrize("mode", [0, 2, 3])
def test_two_tiles_reference_stays_lazy_moves_plain(mode):
    # second block's scores +-1.5: its max exceeds the first's (0.5) by 1.  Lazy reading (tau = 2):
    # the reference stays at 0.5 and the weights are 1, 1/2, 2, 1/4 (P codes 112, 56, 224, 28 in
    # the FP8 modes).  Plain online softmax: the reference moves to 1.5 and the first block's
    # weights halve: 1/2, 1/4, 1, 1/8 (P codes 448, 224 before the move, then 448, 112)
    for reading, w_want, total in (("lazy", [1.0, 0.5, 2.0, 0.25], 240.0), ("plain", [0.5, 0.25, 1.0, 0.125], 120.0)):
        out, v = _run([0.5, 1.5], mode, [-1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0], reading, seed=1)
        rd = READINGS[reading](mode)
        w = _weights([0.5, 1.5], tau=rd["tau"], tile=rd["tile"])
        np.testing.assert_allclose(w, np.repeat(w_want, 64))
        want = (w[:, None] * v).sum(0) / w.sum()
        assert w.sum() == total
        np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=2e-6, err_msg=reading)


@pytest.mark.parametrize("reading", sorted(READINGS))
@pytest.mark.parametrize("mode", [0, 2, 3])
def test_two_tiles_reference_moves(mode, reading):
    # second block's scores +-3: its max exceeds the reference 0.5 by 2.5 > tau (either reading),
    # so the reference moves to 3 and the first block's weights scale by alpha = 2^-2.5 (O and l alike)
    out, v = _run([0.5, 3.0], mode, [-1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0], reading, seed=2)
    a = 2.0 ** -2.5
    w = np.repeat([a, 0.5 * a, 1.0, 2.0 ** -6], 64)
    rd = READINGS[reading](mode)
    np.testing.assert_allclose(_weights([0.5, 3.0], tau=rd["tau"], tile=rd["tile"]), w, rtol=1e-15)
    want = (w[:, None] * v).sum(0) / w.sum()
    # fp16+fp32 over 128-key tiles: the second tile's fp16 partial (64 keys at weight 1, 64 at
    # 2^-6, |partial| <= 65) rounds to fp16, half an ulp <= 2^-11 * 65, divided by the row sum
    # (> 80): within 4e-4.  Every other case is exact up to float32 rounding.
    atol = 4e-4 if (mode == 3 and rd["tile"] == 128) else 2e-6
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=atol)


@pytest.mark.parametrize("reading,p8", [("lazy", [112.0, 56.0, 224.0, 28.0]), ("plain", [448.0, 224.0, 448.0, 56.0])])
def test_two_tiles_fp16_partials_two_level(reading, p8):
    # fp16+fp32 with FP8 P.V: each tile's P.V sum is exactly representable in fp16 here, so its
    # fp16 rounding is exact and the result equals the fp32-accumulation weights.  P codes per
    # tile: lazy 112, 56 | 224, 28 (reference stays at 0.5); plain 448, 224 | 448, 56 (the
    # reference moves to 1.5 and the first tile's partial is halved in O)
    out, v = _run([0.5, 1.5], 1, [-0.25, 0.0, 0.25], reading, seed=3)
    p8 = np.repeat(p8, 64)
    for t in range(2):
        sums = (p8[t * 128:(t + 1) * 128, None] * v[t * 128:(t + 1) * 128]).sum(0)
        assert (sums.astype(np.float16).astype(np.float64) == sums).all()
    w = p8 / 448.0 if reading == "plain" else p8 / 112.0
    if reading == "plain":
        w[:128] *= 0.5
    want = (w[:, None] * v).sum(0) / w.sum()
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=2e-6)
