"""The seeded generator: determinism, row addressing, value ranges, rounding."""
import numpy as np
import pytest

from bit_weight_gemv_q4_b200 import synth


def test_deterministic_and_row_addressable():
    q_full = synth.weights(4, 0, 5, 256, 0, 40)
    q_rows = synth.weights(4, 0, 5, 256, 17, 9)
    assert np.array_equal(q_full[17:26], q_rows)
    assert np.array_equal(q_full, synth.weights(4, 0, 5, 256, 0, 40))
    q8_full = synth.weights(8, 0, 6, 96, 0, 20)
    assert np.array_equal(q8_full[3:7], synth.weights(8, 0, 6, 96, 3, 4))
    s_full = synth.scales(0, 7, 96, 0, 20)
    assert np.array_equal(s_full[11:20], synth.scales(0, 7, 96, 11, 9))
    # different streams and seeds differ
    assert not np.array_equal(q_full, synth.weights(4, 0, 9, 256, 0, 40))
    assert not np.array_equal(q_full, synth.weights(4, 1, 5, 256, 0, 40))


def test_q4_uniform_over_all_sixteen_codes():
    q = synth.weights(4, 0, 1, 4096, 0, 64)
    nib = np.concatenate([q & 0xF, q >> 4]).ravel()
    counts = np.bincount(nib, minlength=16)
    expect = nib.size / 16
    chi2 = ((counts - expect) ** 2 / expect).sum()
    assert chi2 < 60  # 15 d.o.f.; p ~ 1e-7 at 60


def test_q8_range_and_uniformity():
    q = synth.weights(8, 0, 2, 4096, 0, 64).astype(np.int64).ravel()
    assert q.min() == -127 and q.max() == 127
    counts = np.bincount(q + 127, minlength=255)
    expect = q.size / 255
    chi2 = ((counts - expect) ** 2 / expect).sum()
    assert chi2 < 400  # 254 d.o.f.


def test_normals_moments():
    z = synth.normals_f64(0, 3, 0, 200_000)
    assert abs(z.mean()) < 0.01
    assert abs(z.std() - 1) < 0.01
    assert abs((np.abs(z) < 1).mean() - 0.6827) < 0.005


def test_scale_distribution():
    s = synth.scales(0, 11, 4096, 0, 64).view(np.float16).astype(np.float64)
    assert np.all(s >= 0)
    # E|0.02 z| = 0.02 * sqrt(2/pi)
    assert abs(s.mean() - 0.02 * np.sqrt(2 / np.pi)) < 3e-4


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000) * 0.02,
        rng.standard_normal(5000) * 1e-6,  # subnormal range
        rng.standard_normal(5000) * 1e4,
        np.array([65504.0, 65519.99, 65520.0, 1e9, 2.0**-24, 2.0**-25, 3 * 2.0**-26, 0.0, -0.0]),
        # exact halfway cases between fp16 neighbours
        (1024 + np.arange(0, 64) + 0.5) * 2.0**-10,
    ])
    got = synth.f64_to_f16_bits(vals)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def _bf16_value(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000),
        rng.standard_normal(2000) * 1e-39,  # bf16 subnormal range
        (128 + np.arange(0, 64) + 0.5) * 2.0**-7,  # halfway cases
    ])
    got = synth.f64_to_bf16_bits(vals)
    # sign is kept; compare magnitudes with the two neighbouring magnitudes
    assert np.all((got >> 15) == np.signbit(vals))
    mag = (got & 0x7FFF).astype(np.int64)
    a = np.abs(vals)
    v = _bf16_value(mag.astype(np.uint16))
    up = _bf16_value((mag + 1).astype(np.uint16))
    dn = np.where(mag > 0, _bf16_value(np.maximum(mag - 1, 0).astype(np.uint16)), np.inf)
    err = np.abs(v - a)
    # no neighbour is strictly closer
    assert np.all(err <= np.abs(up - a))
    assert np.all(err <= np.abs(dn - a))
    # ties go to the even pattern
    tie = (err == np.abs(up - a)) | (err == np.abs(dn - a))
    assert tie.sum() >= 64
    assert np.all(mag[tie] % 2 == 0)


def test_activation_rows():
    x = synth.activations(0, synth.act_stream(0), 4, 5120)
    assert x.shape == (4, 5120) and x.dtype == np.uint16
    v = _bf16_value(x)
    assert abs(v.mean()) < 0.03 and abs(v.std() - 1) < 0.03
    # the first row of an M=4 block equals the M=1 block
    assert np.array_equal(synth.activations(0, synth.act_stream(0), 1, 5120)[0], x[0])


@pytest.mark.parametrize("K", [0, 16, 33])
def test_bad_shapes_rejected(K):
    with pytest.raises(ValueError):
        synth.weights(4, 0, 0, K, 0, 1)
