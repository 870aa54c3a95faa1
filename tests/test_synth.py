"""The seeded input generator: determinism and the workload's distributions."""
import numpy as np

import dfssm_synth as synth

M64 = 2**64 - 1


def splitmix_mix(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def test_counter_mode_splitmix64():
    # SplitMix64 from seed 0: the first outputs of the published generator
    g = 0x9E3779B97F4A7C15
    assert splitmix_mix(g) == 0xE220A8397B1DCDAF
    sid = synth.stream_id(1, 2, 3, 4, 5)
    k = synth.key(123, sid)
    assert k == splitmix_mix((123 + splitmix_mix((sid + g) & M64)) & M64)
    r = synth.raw(123, sid, 10, 5)
    for i in range(5):
        assert int(r[i]) == splitmix_mix((k + (10 + i + 1) * g) & M64)


def test_x_distribution_and_outliers():
    m, d_in = 64, 4096
    x = synth.activations(synth.MASTER_SEED, 3, 0, m, d_in)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    cols = synth.outlier_cols(synth.MASTER_SEED, 3, m, 0, d_in)
    assert len(cols) == 41 and len(set(cols.tolist())) == 41
    mask = np.zeros(d_in, bool)
    mask[cols] = True
    assert abs(xf[:, ~mask].std() - 1.0) < 0.02
    assert abs(xf[:, mask].std() - 20.0) < 1.5
    assert abs(xf[:, ~mask].mean()) < 0.02
    # deterministic, and independent of thread count (pure function of the counter)
    x2 = synth.activations(synth.MASTER_SEED, 3, 0, m, d_in)
    np.testing.assert_array_equal(x, x2)
    assert len(synth.outlier_cols(1, 0, 1, 0, 2048)) == 20


def test_weight_distributions():
    w = synth.linear_weights(synth.MASTER_SEED, 2, 0, 2048, 8512)
    bits = np.unpackbits(w["sign"])
    assert abs(bits.mean() - 0.5) < 0.002
    assert 0.005 <= w["alpha"].min() and w["alpha"].max() <= 0.05
    assert 1e-4 <= w["sa"].min() and w["sa"].max() <= 1e-3
    assert 1e-4 <= w["sb"].min() and w["sb"].max() <= 1e-3
    for k in ("wa", "wb"):
        v = w[k].astype(int)
        assert v.min() == -127 and v.max() == 127
        assert abs(v.mean()) < 1.5
    # different linears draw different weights
    w2 = synth.linear_weights(synth.MASTER_SEED, 2, 1, 2048, 8512)
    assert not np.array_equal(w["sign"], w2["sign"])
