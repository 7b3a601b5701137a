"""The seeded input generator: determinism, distribution, bias recipe."""
import numpy as np

import synth


def test_deterministic_and_seed_sensitive():
    a = synth.expert(0, 0, 3, 128, 64)
    b = synth.expert(0, 0, 3, 128, 64)
    c = synth.expert(1, 0, 3, 128, 64)
    d = synth.expert(0, 1, 3, 128, 64)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[0], c[0]) and not np.array_equal(a[0], d[0])
    x1 = synth.x_f32(5, 2, 3, 256)
    assert np.array_equal(x1, synth.x_f32(5, 2, 3, 256))
    assert not np.array_equal(x1, synth.x_f32(5, 3, 3, 256))


def test_gaussian_approximation_moments_and_exactness():
    z = synth.x_f32(0, 0, 64, 16384).ravel().astype(np.float64)
    assert abs(z.mean()) < 5e-3
    assert abs(z.var() - 1.0) < 5e-3
    assert np.abs(z).max() <= 6.0
    # every value is an integer multiple of 2^-16 (exact Irwin-Hall offset)
    assert np.all(np.rint(z * 65536) == z * 65536)
    # fourth moment of the 12-term Irwin-Hall sum: 3 - 1.2/12 = 2.9
    assert abs((z ** 4).mean() - 2.9) < 0.05


def test_bf16_activations_round_the_fp32_ones_to_nearest_even():
    xf = synth.x_f32(9, 1, 4, 512)
    xb = synth.x_bf16(9, 1, 4, 512)
    back = (xb.astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.abs(back - xf) <= np.abs(xf) * 2.0 ** -8)
    # round to nearest: no bf16 neighbour is closer
    up = ((xb.astype(np.uint32) + 1) << 16).view(np.float32)
    dn = ((xb.astype(np.uint32) - 1) << 16).view(np.float32)
    err = np.abs(back - xf)
    assert np.all(err <= np.abs(up - xf)) and np.all(err <= np.abs(dn - xf))


def test_router_weights_scale():
    wr = synth.router(0, 0, 64, 1024)
    assert abs(wr.std() - 0.02) < 5e-4


def test_zipf_bias_is_a_mean_centred_log_power_law_over_a_permutation():
    b, r = synth.zipf_bias(0, 0, 256, kappa=0.7)
    assert sorted(r.tolist()) == list(range(1, 257))
    assert abs(float(b.astype(np.float64).sum())) < 1e-3
    # b_e = kappa * (-1.1 ln rank + c): differences between experts follow the law
    e1, e2 = int(np.argmin(r)), int(np.argmax(r))
    assert abs((b[e1] - b[e2]) - 0.7 * 1.1 * np.log(256.0)) < 1e-4
    b2, r2 = synth.zipf_bias(0, 1, 256, kappa=0.7)
    assert not np.array_equal(r, r2)  # each layer draws its own popularity order
