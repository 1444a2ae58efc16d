"""The seeded input generator: published SplitMix64 vector, stream
independence, Box-Muller moments, bf16 rounding and the outlier recipe."""
import numpy as np

from bitlinear_w1_a8_03_b200 import synth


def test_splitmix64_published_vector():
    # SplitMix64 (Steele, Lea, Flood 2014; Vigna's reference C) seeded with
    # 1234567 starts 6457827717110365317, 3203168211198807973, ...
    z = np.array([(1234567 + (i + 1) * 0x9E3779B97F4A7C15) & (2**64 - 1) for i in range(5)], dtype=np.uint64)
    with np.errstate(over="ignore"):
        got = synth._mix64(z).tolist()
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_streams_are_independent():
    a = synth.weights(0, 64, 64, 1.0).ravel()
    b = synth.activations(0, 64, 64).ravel()
    c = synth.weights(1, 64, 64, 1.0).ravel()
    for u, v in ((a, b), (a, c), (b, c)):
        assert abs(float(np.corrcoef(u, v)[0, 1])) < 0.05
        assert abs(float(np.corrcoef(u[1:], v[:-1])[0, 1])) < 0.05


def test_normal_moments_and_determinism():
    x = synth.normal_f32(synth.stream_key(5, 2), 1 << 20, 0.02)
    assert abs(float(x.mean())) < 1e-4
    assert abs(float(x.std()) / 0.02 - 1) < 0.005
    assert np.array_equal(x[:1000], synth.normal_f32(synth.stream_key(5, 2), 1000, 0.02))
    # the threaded block split gives the same numbers as one block
    big = synth.normal_f32(synth.stream_key(6, 1), (1 << 23) + 3, 1.0)
    assert np.array_equal(big[-5:], synth._normal_block(synth.stream_key(6, 1), 0, ((1 << 23) + 4) // 2)[(1 << 23) - 2:(1 << 23) + 3].astype(np.float32))


def test_bf16_round_to_nearest_even():
    f = np.array([1.0, 1.00390625, 1.01171875, 1.0 + 2**-8 + 2**-20, -2.5, 3.0e38], dtype=np.float32)
    b = synth.f32_to_bf16_bits(f)
    back = synth.bf16_bits_to_f32(b)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa → 1.0
    assert back.tolist()[:4] == [1.0, 1.0, 1.015625, 1.0078125]
    assert back[4] == -2.5


def test_outliers_recipe():
    K = 4096
    idx = synth.outlier_channels(2000, K)
    assert len(idx) == 4 and len(set(idx.tolist())) == 4
    x = synth.activations(2000, 3, K, outliers=True)
    base = synth.activations(2000, 3, K, outliers=False)
    assert np.array_equal(x[:, idx], base[:, idx] * np.float32(20))
    mask = np.ones(K, bool)
    mask[idx] = False
    assert np.array_equal(x[:, mask], base[:, mask])
    assert len(synth.outlier_channels(1, 256)) == 1 and len(synth.outlier_channels(1, 11008)) == 11
