"""int32 Q8.K8^T tiles from the tcgen05 kind::i8 path vs exact integer products (bit-exact)."""
import numpy as np
import pytest

import workloads as W
from oracle import quant
from tests._support import oracle_to_device, slice_heads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [
    W.TINY,
    W.TINY.with_(name="d96_ragged", N=300, d=96, Hq=4, Hkv=2, dist="uniform2"),
    W.TINY.with_(name="d256", N=256, d=256, dist="normal_koutlier"),
    W.TINY.with_(name="d128_nhd", N=384, d=128, layout="NHD", dist="normal_koffset", dtype="bf16"),
], ids=lambda w: w.name)
def test_qk_int32_all_tiles(lib, w):
    q, k, v = W.make_inputs(w)
    qz = quant.quantize(q, k, v, w.layout, w.pv_mode)
    z = oracle_to_device(qz)
    nb = (w.N + 127) // 128
    tiles = [(b, h, i, j) for b in range(w.B) for h in range(w.Hq) for i in range(nb) for j in range(nb)]
    s = lib.sage_qk_int32(z, tiles).cpu().numpy()
    lib.sage_check_status()
    G = w.Hq // w.Hkv
    for t, (b, h, i, j) in enumerate(tiles):
        ref = quant.qk_int32(qz["q8"][b, h, i * 128:(i + 1) * 128], qz["k8"][b, h // G, j * 128:(j + 1) * 128])
        assert np.array_equal(s[t], ref), (b, h, i, j)


def test_qk_int32_full_size_sampled_tiles(lib):
    """Config-3 sizes (N = 32768, d = 128): the Q/K codes of one head, tiles across the sequence."""
    w = W.VIDEO_DIT
    q, k, v = W.make_inputs(w)
    qz = quant.quantize(slice_heads(q, w.layout, 0, [5]), slice_heads(k, w.layout, 0, [5]),
                        slice_heads(v, w.layout, 0, [5]), w.layout, w.pv_mode)
    z = oracle_to_device(qz)
    rng = np.random.default_rng(0)
    tiles = [(0, 0, int(i), int(j)) for i, j in rng.integers(0, 256, size=(24, 2))] + [(0, 0, 255, 255), (0, 0, 0, 255)]
    s = lib.sage_qk_int32(z, tiles).cpu().numpy()
    lib.sage_check_status()
    for t, (_, _, i, j) in enumerate(tiles):
        ref = quant.qk_int32(qz["q8"][0, 0, i * 128:(i + 1) * 128], qz["k8"][0, 0, j * 128:(j + 1) * 128])
        assert np.array_equal(s[t], ref), (i, j)
