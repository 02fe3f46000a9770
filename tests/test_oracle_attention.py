"""Pins for the oracle's exact float64 attention (CPU only).

Brute force on tiny inputs, closed forms, invariants, and torch's SDPA in
float64 as an independent library routine.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention, emulate, fp8, quant


def _brute(q, k, v, causal, scale):
    # pure-python loops, no numpy linear algebra
    N, d = len(q), len(q[0])
    out = []
    for i in range(N):
        js = [j for j in range(N) if (j <= i or not causal)]
        s = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in js]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        out.append([sum(e[t] * v[js[t]][c] for t in range(len(js))) / z for c in range(d)])
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(causal):
    rng = np.random.default_rng(0)
    q, k, v = (rng.standard_normal((1, 1, 7, 3)).astype(np.float32) for _ in range(3))
    got = attention.attention_f64(q, k, v, "HND", causal, 0.7)[0, 0]
    ref = _brute(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), causal, 0.7)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_closed_forms():
    rng = np.random.default_rng(1)
    v = rng.standard_normal((1, 1, 9, 4)).astype(np.float32)
    k = rng.standard_normal((1, 1, 9, 4)).astype(np.float32)
    q0 = np.zeros_like(k)
    vf = v[0, 0].astype(np.float64)
    # Q = 0: uniform weights -> mean of V; causal -> prefix means
    assert np.allclose(attention.attention_f64(q0, k, v, causal=False)[0, 0], vf.mean(0)[None, :].repeat(9, 0))
    pref = np.cumsum(vf, 0) / np.arange(1, 10)[:, None]
    assert np.allclose(attention.attention_f64(q0, k, v, causal=True)[0, 0], pref)
    # row 0 under the causal mask sees only key 0
    q = rng.standard_normal((1, 1, 9, 4)).astype(np.float32)
    assert np.allclose(attention.attention_f64(q, k, v, causal=True)[0, 0, 0], vf[0])
    # sm_scale -> 0 gives the mean; a huge sm_scale picks the argmax key
    assert np.allclose(attention.attention_f64(q, k, v, sm_scale=1e-12)[0, 0], vf.mean(0)[None].repeat(9, 0))
    s = q[0, 0].astype(np.float64) @ k[0, 0].astype(np.float64).T
    hard = vf[s.argmax(1)]
    assert np.allclose(attention.attention_f64(q, k, v, sm_scale=1e4)[0, 0], hard, atol=1e-6)


def test_rows_sum_and_matches_torch_sdpa_f64():
    w = W.TINY.with_(N=100, d=24, Hq=4, Hkv=2)
    q, k, v = W.make_inputs(w)
    for causal in (False, True):
        got = attention.attention_f64(q, k, v, "HND", causal, 0.3)
        kk = k.double().repeat_interleave(2, dim=1)
        vv = v.double().repeat_interleave(2, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(q.double(), kk, vv, is_causal=causal, scale=0.3)
        assert np.allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12)
    # V = 1 gives 1 everywhere: the weights of every row sum to one
    ones = torch.ones_like(v)
    assert np.allclose(attention.attention_f64(q, k, ones, "HND", True, 0.3), 1.0)


def test_invariances():
    w = W.TINY.with_(N=64, d=16, Hq=4, Hkv=2)
    q, k, v = (t.double().numpy() for t in W.make_inputs(w))
    base = attention.attention_f64(q, k, v, "HND", False, 0.25)
    # permuting keys together with values changes nothing without the mask
    perm = np.random.default_rng(2).permutation(64)
    assert np.allclose(attention.attention_f64(q, k[:, :, perm], v[:, :, perm], "HND", False, 0.25), base)
    # subtracting the token mean of K changes nothing (each row of scores shifts)
    km = k.mean(axis=2, keepdims=True)
    for causal in (False, True):
        assert np.allclose(attention.attention_f64(q, k - km, v, "HND", causal, 0.25),
                           attention.attention_f64(q, k, v, "HND", causal, 0.25))
    # GQA equals MHA with K and V repeated per group
    mha = attention.attention_f64(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1), "HND", False, 0.25)
    assert np.allclose(mha, base)
    # NHD storage of the same tensors gives the same result
    nhd = attention.attention_f64(*(t.transpose(0, 2, 1, 3) for t in (q, k, v)), "NHD", False, 0.25)
    assert np.allclose(nhd, base)
    # zero-padding d to 128 with sm_scale 1/sqrt(96) equals the unpadded result
    w2 = W.TINY.with_(N=50, d=96)
    q2, k2, v2 = (t.double().numpy() for t in W.make_inputs(w2))
    pad = lambda t: np.concatenate([t, np.zeros(t.shape[:3] + (32,))], axis=3)
    a = attention.attention_f64(q2, k2, v2, "HND", True, 1 / math.sqrt(96))
    b = attention.attention_f64(pad(q2), pad(k2), pad(v2), "HND", True, 1 / math.sqrt(96))
    assert np.allclose(b[..., :96], a) and np.allclose(b[..., 96:], 0)
    # rows/heads selection returns the same numbers as the full call
    sel = attention.attention_f64(q, k, v, "HND", False, 0.25, heads=[(0, 3)], rows=[5, 60])
    assert np.allclose(sel[0], base[0, 3, [5, 60]])


def test_emulation_constant_scores_give_mean_of_v():
    # Q = 0 makes every score 0, so every p is exactly 1 and P8 = 448 exactly;
    # V values +-1, +-0.5 with amax 1 are exact in E4M3 after scaling by 448.
    rng = np.random.default_rng(3)
    N = 300
    q = np.zeros((1, 1, N, 8), np.float32)
    k = rng.standard_normal((1, 1, N, 8)).astype(np.float32)
    v = rng.choice([-1.0, -0.5, 0.5, 1.0], size=(1, 1, N, 8)).astype(np.float32)
    v[0, 0, 0] = 1.0
    qz = quant.quantize(q, k, v, "HND", 0)
    em = emulate.emulate(qz, False, 0.35)[0, :N]
    assert np.allclose(em, v[0, 0].mean(0)[None].repeat(N, 0), rtol=1e-6, atol=1e-7)
    emc = emulate.emulate(qz, True, 0.35)[0, :N]
    pref = np.cumsum(v[0, 0].astype(np.float64), 0) / np.arange(1, N + 1)[:, None]
    assert np.allclose(emc, pref, rtol=1e-6, atol=1e-7)


def test_emulation_causal_row0_is_dequantized_v0():
    w = W.TINY.with_(causal=True)
    q, k, v = W.make_inputs(w)
    for mode in (0, 1):
        qz = quant.quantize(q, k, v, "HND", mode)
        em = emulate.emulate(qz, True, 0.125, heads=[(0, 1)], q_blocks=[0])[0, 0]
        vhat = fp8.decode(qz["v8"][0, 1, 0, :64]) * qz["vs"][0, 1, :64]
        assert np.allclose(em, vhat, rtol=1e-6)


def test_emulation_tracks_exact_attention():
    # The method's own error on the tiny workload: cosine similarity >= 0.999
    # and max abs error inside the 1e-1 bound the 9070XT bench reports.
    w = W.TINY
    q, k, v = W.make_inputs(w)
    for mode in (0, 1):
        qz = quant.quantize(q, k, v, "HND", mode)
        em = emulate.emulate(qz, False, 0.125).reshape(1, 2, 256, 64).astype(np.float64)
        ref = attention.attention_f64(q, k, v, "HND", False, 0.125)
        cos = (em * ref).sum() / np.sqrt((em ** 2).sum() * (ref ** 2).sum())
        assert cos >= 0.999 and np.abs(em - ref).max() < 0.1


def test_emulation_fp16_pv_modes():
    # FP16 P.V: Q = 0 gives p = 1 exactly (fp16 1.0), V codes v/amax are exact in fp16 for
    # these values, so every row is the (prefix) mean of V; causal row 0 is fp16(v0/amax)*amax.
    rng = np.random.default_rng(4)
    N = 300
    q = np.zeros((1, 1, N, 8), np.float32)
    k = rng.standard_normal((1, 1, N, 8)).astype(np.float32)
    v = rng.choice([-1.0, -0.5, 0.5, 1.0, 0.25], size=(1, 1, N, 8)).astype(np.float32)
    v[0, 0, 0] = 1.0
    for mode in (2, 3):
        qz = quant.quantize(q, k, v, "HND", mode)
        assert qz["v8"].dtype == np.float16 and np.allclose(qz["vs"][0, 0, :8], 1.0)
        em = emulate.emulate(qz, False, 0.35)[0, :N]
        assert np.allclose(em, v[0, 0].mean(0)[None].repeat(N, 0), rtol=1e-6, atol=1e-7)
        emc = emulate.emulate(qz, True, 0.35)[0, :N]
        pref = np.cumsum(v[0, 0].astype(np.float64), 0) / np.arange(1, N + 1)[:, None]
        assert np.allclose(emc, pref, rtol=1e-6, atol=1e-7)
    # and the method stays within the target cosine (0.999) on the tiny workload
    w = W.TINY
    q, k, v = W.make_inputs(w)
    for mode in (2, 3):
        qz = quant.quantize(q, k, v, "HND", mode)
        em = emulate.emulate(qz, False, 0.125).reshape(1, 2, 256, 64).astype(np.float64)
        ref = attention.attention_f64(q, k, v, "HND", False, 0.125)
        cos = (em * ref).sum() / np.sqrt((em ** 2).sum() * (ref ** 2).sum())
        assert cos >= 0.9999 and np.abs(em - ref).max() < 0.02


def test_fp16_v_codes_bound():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((1, 2, 200, 20)) * 3).astype(np.float32)
    codes, scale = quant.fp16_per_channel(v, 64)
    assert np.allclose(scale[:, :, :20], np.abs(v).max(axis=2)) and np.all(scale[:, :, 20:] == 0)
    rec = codes[:, :, :200, :20].astype(np.float64) * scale[:, :, None, :20]
    # fp16 keeps 11 significant bits: relative error <= 2^-11 (subnormals: 2^-25 absolute)
    assert np.all(np.abs(rec - v) <= np.maximum(np.abs(v) * 2.0 ** -11, 2.0 ** -25 * scale[:, :, None, :20]) * (1 + 1e-6))
    assert np.all(np.abs(codes[:, :, :200, :20]).max(axis=2) == 1.0)


def _brute_rect(q, k, v, causal, scale):
    # pure-python loops; causal keeps key j for query i iff j <= i + (Nk - Nq); rows that see no key -> 0
    Nq, Nk, d = len(q), len(k), len(v[0])
    out = []
    for i in range(Nq):
        js = [j for j in range(Nk) if (not causal or j <= i + Nk - Nq)]
        if not js:
            out.append([0.0] * d)
            continue
        s = [scale * sum(q[i][c] * k[j][c] for c in range(len(q[0]))) for j in js]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        out.append([sum(e[t] * v[js[t]][c] for t in range(len(js))) / z for c in range(d)])
    return out


@pytest.mark.parametrize("nq,nk", [(5, 9), (9, 5), (1, 7), (7, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular_brute_force(nq, nk, causal):
    rng = np.random.default_rng(10 + nq * 10 + nk)
    q = rng.standard_normal((1, 1, nq, 3)).astype(np.float32)
    k, v = (rng.standard_normal((1, 1, nk, 3)).astype(np.float32) for _ in range(2))
    got = attention.attention_f64(q, k, v, "HND", causal, 0.6)[0, 0]
    ref = _brute_rect(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), causal, 0.6)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_rectangular_matches_sdpa_with_bottom_right_mask():
    rng = np.random.default_rng(11)
    for nq, nk in ((40, 100), (100, 40), (33, 33)):
        # float32-representable values (the oracle widens its inputs from float32, like fp16/bf16)
        q = torch.from_numpy(rng.standard_normal((2, 4, nq, 16)).astype(np.float32)).double()
        k, v = (torch.from_numpy(rng.standard_normal((2, 2, nk, 16)).astype(np.float32)).double() for _ in range(2))
        got = attention.attention_f64(q, k, v, "HND", True, 0.25)
        i = torch.arange(nq)[:, None]
        j = torch.arange(nk)[None, :]
        mask = j <= i + (nk - nq)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), attn_mask=mask, scale=0.25)
        seen = mask.any(1)                    # SDPA gives NaN on rows with no key; the reading is 0
        assert np.allclose(got[:, :, seen.numpy()], ref[:, :, seen].numpy(), rtol=1e-10, atol=1e-12)
        assert np.all(got[:, :, ~seen.numpy()] == 0)
    # one query row with the causal mask sees every key (bottom-right alignment)
    q1 = q[:, :, -1:]
    assert np.allclose(attention.attention_f64(q1, k, v, "HND", True, 0.25),
                       attention.attention_f64(q1, k, v, "HND", False, 0.25))


def test_varlen_matches_block_diagonal_sdpa():
    rng = np.random.default_rng(12)
    lq, lk = [37, 1, 130, 0, 64], [50, 3, 130, 7, 1]
    cq, ck = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    q = torch.from_numpy(rng.standard_normal((cq[-1], 4, 8)).astype(np.float32)).double()
    k, v = (torch.from_numpy(rng.standard_normal((ck[-1], 2, 8)).astype(np.float32)).double() for _ in range(2))
    for causal in (False, True):
        got = attention.attention_varlen_f64(q, k, v, cq, ck, causal, 0.3)
        mask = torch.zeros((cq[-1], ck[-1]), dtype=torch.bool)
        for b in range(len(lq)):
            i = torch.arange(lq[b])[:, None]
            j = torch.arange(lk[b])[None, :]
            mask[cq[b]:cq[b + 1], ck[b]:ck[b + 1]] = (j <= i + lk[b] - lq[b]) if causal else True
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.permute(1, 0, 2)[None], k.permute(1, 0, 2).repeat_interleave(2, 0)[None],
            v.permute(1, 0, 2).repeat_interleave(2, 0)[None], attn_mask=mask, scale=0.3)[0].permute(1, 0, 2)
        seen = mask.any(1).numpy()
        assert np.allclose(got[seen], ref[seen].numpy(), rtol=1e-10, atol=1e-12)
        assert np.all(got[~seen] == 0)
    # equal lengths: the packed batch is the dense NHD batch
    w = W.TINY.with_(N=70, d=16, Hq=4, Hkv=2, B=3, layout="NHD")
    qd, kd, vd = W.make_inputs(w)
    cu = np.arange(4) * 70
    dense = attention.attention_f64(qd, kd, vd, "NHD", True, 0.3)          # (B, Hq, N, d)
    packed = attention.attention_varlen_f64(qd.reshape(-1, 4, 16), kd.reshape(-1, 2, 16), vd.reshape(-1, 2, 16),
                                            cu, cu, True, 0.3)
    assert np.allclose(packed.reshape(3, 70, 4, 16).transpose(0, 2, 1, 3), dense)


@pytest.mark.parametrize("mode", [0, 2])
def test_emulation_rectangular_closed_forms(mode):
    # Q = 0 with exactly representable V: row i is the mean of v[0 .. i + Nk - Nq] (causal), or of all V
    rng = np.random.default_rng(13)
    for nq, nk in ((200, 300), (300, 140)):
        q = np.zeros((1, 1, nq, 8), np.float32)
        k = rng.standard_normal((1, 1, nk, 8)).astype(np.float32)
        v = rng.choice([-1.0, -0.5, 0.5, 1.0], size=(1, 1, nk, 8)).astype(np.float32)
        v[0, 0, 0] = 1.0
        qz = quant.quantize(q, k, v, "HND", mode)
        assert qz["N"] == nq and qz["Nk"] == nk
        em = emulate.emulate(qz, False, 0.35)[0, :nq]
        assert np.allclose(em, v[0, 0].mean(0)[None].repeat(nq, 0), rtol=1e-6, atol=1e-7)
        emc = emulate.emulate(qz, True, 0.35)[0, :nq]
        cum = np.cumsum(v[0, 0].astype(np.float64), 0) / np.arange(1, nk + 1)[:, None]
        last = np.arange(nq) + nk - nq                     # last visible key of each row
        ref = np.where(last[:, None] >= 0, cum[np.clip(last, 0, None)], 0.0)
        assert np.allclose(emc, ref, rtol=1e-6, atol=1e-7)
        # and the method tracks exact attention on random Q
        qr = rng.standard_normal((1, 2, nq, 64)).astype(np.float32)
        kr, vr = (rng.standard_normal((1, 2, nk, 64)).astype(np.float32) for _ in range(2))
        qz = quant.quantize(qr, kr, vr, "HND", mode)
        for causal in (False, True):
            em = emulate.emulate(qz, causal, 0.125).reshape(1, 2, -1, 64)[:, :, :nq].astype(np.float64)
            ex = attention.attention_f64(qr, kr, vr, "HND", causal, 0.125)
            assert (em * ex).sum() / np.sqrt((em ** 2).sum() * (ex ** 2).sum()) >= 0.999


def test_v_smoothing_identity_in_exact_attention():
    # softmax rows sum to one: attention(V - mu) + mu = attention(V) for any per-channel mu
    w = W.TINY.with_(N=90, d=12, Hq=4, Hkv=2)
    q, k, v = (t.double().numpy() for t in W.make_inputs(w))
    # the oracle widens its inputs through float32, so v - mu carries one float32 rounding
    # (<= 2^-24 * 32 for |mu| < 16): the identity holds to that
    mu = np.round(np.random.default_rng(22).standard_normal((1, 2, 1, 12)) * 5 * 16) / 16
    for causal in (False, True):
        a = attention.attention_f64(q, k, v, "HND", causal, 0.3)
        b = attention.attention_f64(q, k, v - mu, "HND", causal, 0.3) + np.repeat(mu, 2, axis=1)
        assert np.allclose(a, b, rtol=0, atol=2e-6)


def test_emulation_v_smoothing_and_q_granularity():
    rng = np.random.default_rng(23)
    # V with large per-channel offsets: smoothing must not change the result beyond rounding, and
    # must shrink the error of the FP8 codes
    w = W.TINY.with_(N=384, d=64)
    q, k, v = W.make_inputs(w)
    v = (v.float() + torch.from_numpy(rng.standard_normal(64).astype(np.float32) * 20)).half()
    ref = attention.attention_f64(q, k, v, "HND", False, 0.125)
    errs = {}
    for sv in (False, True):
        for mode in (0, 2):
            qz = quant.quantize(q, k, v, "HND", mode, smooth_v=sv)
            em = emulate.emulate(qz, False, 0.125).reshape(1, 2, -1, 64)[:, :, :384].astype(np.float64)
            errs[(sv, mode)] = np.abs(em - ref).max() / np.abs(ref).max()
    # FP8 codes gain most (measured 54x smaller error); fp16 codes already carry the offset
    assert errs[(True, 0)] < 0.25 * errs[(False, 0)] and errs[(True, 2)] < 1.1 * errs[(False, 2)]
    # V constant over tokens: smoothed codes carry ~nothing, the output is the mean itself
    vc = torch.from_numpy(np.broadcast_to(rng.standard_normal(64).astype(np.float32), (1, 2, 384, 64)).copy()).half()
    qz = quant.quantize(q, k, vc, "HND", 0, smooth_v=True)
    em = emulate.emulate(qz, True, 0.125).reshape(1, 2, -1, 64)[:, :, :384]
    assert np.allclose(em, vc.float().numpy(), rtol=1e-5, atol=1e-5)
    # Q rows of very different magnitude: per-token scales track exact attention at least as well
    qv = (q.float() * torch.from_numpy(np.exp(rng.uniform(-4, 1, (1, 2, 384, 1))).astype(np.float32))).half()
    ref = attention.attention_f64(qv, k, v, "HND", True, 0.125)
    cos = {}
    for g in quant.Q_GRANS:
        qz = quant.quantize(qv, k, v, "HND", 2, q_gran=g, smooth_v=True)
        em = emulate.emulate(qz, True, 0.125).reshape(1, 2, -1, 64)[:, :, :384].astype(np.float64)
        cos[g] = float((em * ref).sum() / np.sqrt((em ** 2).sum() * (ref ** 2).sum()))
        assert cos[g] >= 0.999
    assert cos[1] >= cos[32] - 1e-6 and cos[32] >= cos[128] - 1e-6
