"""Property-based pins for the oracle's quantizers (CPU only, hypothesis).

Random shapes (ragged token counts, head dims below the padded width) and magnitudes over many
decades; the properties follow from the definitions: symmetric INT8 with one scale per block
reconstructs every element within half a step, maps the block's largest magnitude to +-127 and
leaves padding at 0; E4M3 encoding is monotonic and returns the nearest representable value.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import fp8, quant

F32 = np.float32
ALL_E4M3 = np.sort(np.unique(fp8.decode(np.arange(256, dtype=np.uint8))[np.isfinite(fp8.decode(np.arange(256, dtype=np.uint8)))]))


@settings(max_examples=40, deadline=None)
@given(n=st.integers(1, 300), d=st.integers(1, 128), log_scale=st.floats(-20, 20), seed=st.integers(0, 2**31 - 1),
       rows=st.sampled_from([128, 32, 1]))
def test_int8_per_block_properties(n, d, log_scale, seed, rows):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((1, 1, n, d)) * 2.0 ** log_scale).astype(F32)
    dp = quant.padded_dim(d)
    codes, scale = quant.int8_per_block(x, dp, rows)
    npad = -(-n // 128) * 128
    assert codes.shape == (1, 1, npad, dp) and codes.dtype == np.int8
    assert (codes[:, :, n:] == 0).all() and (codes[:, :, :, d:] == 0).all()
    assert (np.abs(codes.astype(np.int32)) <= 127).all()
    for g in range(-(-n // rows)):
        blk = x[0, 0, g * rows:(g + 1) * rows].astype(np.float64)
        c = codes[0, 0, g * rows:g * rows + len(blk), :d].astype(np.float64)
        s = float(scale[0, 0, g])
        amax = np.abs(blk).max()
        if amax == 0:
            assert s == 0 and not c.any()
            continue
        assert np.abs(c).max() == 127
        assert abs(s - amax / 127) <= 1e-6 * s
        assert (np.abs(c * s - blk) <= s * (0.5 + 1e-5)).all()


@settings(max_examples=60, deadline=None)
@given(st.lists(st.floats(-500, 500, allow_nan=False, width=32), min_size=2, max_size=64))
def test_e4m3_encode_is_monotonic_and_nearest(xs):
    x = np.asarray(sorted(xs), F32)
    y = fp8.decode(fp8.encode(x)).astype(np.float64)
    assert (np.diff(y) >= 0).all()  # monotonic
    xc = np.clip(x.astype(np.float64), -448, 448)  # saturating
    dist = np.abs(ALL_E4M3[None, :].astype(np.float64) - xc[:, None]).min(axis=1)
    assert (np.abs(y - xc) <= dist + 1e-12).all()  # no representable value is nearer


@settings(max_examples=30, deadline=None)
@given(n=st.integers(1, 600), d=st.integers(1, 96), seed=st.integers(0, 2**31 - 1), vmax=st.sampled_from([448.0, 1.0]))
def test_fp8_per_channel_properties(n, d, seed, vmax):
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal((1, 1, n, d)) * rng.uniform(0.01, 100.0, size=d)).astype(F32)
    dp = quant.padded_dim(d)
    codes, vs = quant.fp8_per_channel(v, dp, vmax)
    dec = fp8.decode(codes[0, 0, :n, :d]).astype(np.float64)
    s = vs[0, 0, :d].astype(np.float64)
    # every channel's largest magnitude maps to +-vmax; the codes stay within +-vmax
    assert np.allclose(np.abs(dec).max(axis=0), vmax, rtol=0, atol=0)
    assert (np.abs(dec) <= vmax).all()
    err = np.abs(dec * s - v[0, 0].astype(np.float64))
    # dequantized values within half of E4M3's relative step (2^-4 of the value), or half of its
    # subnormal step (2^-9 in code units) times the channel scale
    assert (err <= np.maximum(np.abs(v[0, 0]) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)).all()
    assert (codes[0, 0, n:] == 0).all() and (codes[0, 0, :, d:] == 0).all()
