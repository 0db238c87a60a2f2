"""The seeded input generator: shapes, dtypes, determinism, structure."""
import numpy as np

import synth


def test_tiny_layer_shapes_and_determinism():
    a = synth.config_layers(0)[0]
    b = synth.config_layers(0)[0]
    assert (a.K, a.N, a.group_size, a.krot) == (256, 512, 128, 8)
    assert a.pairs.dtype == np.int16 and a.pairs.shape == (8, 256)
    assert a.theta.dtype == np.float32 and a.theta.shape == (8, 128)
    assert a.channel_scales.dtype == np.float32 and a.channel_scales.shape == (256,)
    assert a.codes.dtype == np.uint8 and a.codes.shape == (512, 256)
    assert a.zero_codes.shape == (512, 2) and np.all(a.zero_codes == 8)
    assert a.scales.dtype == np.float16 and a.scales.shape == (2, 512)
    assert a.bias is None
    for f in ("pairs", "theta", "channel_scales", "codes", "scales"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    x = synth.make_activations(a, 4)
    assert x.dtype == np.float16 and x.shape == (4, 256)
    assert np.array_equal(x, synth.make_activations(b, 4))


def test_pairs_are_group_local_perfect_matchings():
    lay = synth.config_layers(0)[0]
    G = lay.group_size
    for s in range(lay.krot):
        for g in range(lay.K // G):
            assert sorted(lay.pairs[s, g * G:(g + 1) * G].tolist()) == list(range(G))
    assert np.all(np.abs(lay.theta) <= np.pi)
    assert np.all((lay.channel_scales >= 0.5) & (lay.channel_scales <= 2.0))
    assert lay.codes.max() <= 15
    assert np.all((lay.scales >= 0.00499) & (lay.scales <= 0.0201))


def test_active_pair_fraction():
    lay = synth.make_layer("q", 512, 64, 5, active_pairs=6)
    nz = (lay.theta != 0).reshape(lay.krot, -1, 64).sum(axis=2)
    assert np.all(nz == 6)
    full = synth.make_layer("q", 512, 64, 5)
    assert np.all((full.theta != 0).reshape(full.krot, -1, 64).sum(axis=2) == 64)


def test_outliers_and_bias():
    lay = synth.make_layer("g", 4096, 64, 9, n_outliers=synth.one_percent(4096), bias_std=0.01)
    assert lay.outlier_channels.size == 41
    x = synth.make_activations(lay, 256).astype(np.float64)
    rms = np.sqrt((x ** 2).mean(axis=0))
    assert np.all(rms[lay.outlier_channels] > 10)
    mask = np.ones(4096, bool)
    mask[lay.outlier_channels] = False
    assert np.all(rms[mask] < 2)
    assert lay.bias.dtype == np.float16 and 0.005 < float(np.std(lay.bias.astype(np.float64))) < 0.02


def test_config_shapes_listing():
    assert [s[1:] for s in synth.config_layer_shapes(4)] == [
        (4096, 4096), (4096, 1024), (4096, 1024), (4096, 4096),
        (4096, 14336), (4096, 14336), (14336, 4096)]
    assert synth.CONFIG_M[1] == [1, 4, 16]


def test_float_weight_inputs_are_seeded_and_typed():
    lay = synth.make_layer("w", 256, 64, 5)
    W1, s1 = synth.make_float_weight(lay)
    W2, s2 = synth.make_float_weight(lay)
    assert W1.dtype == np.float16 and W1.shape == (64, 256)
    assert s1.dtype == np.float16 and s1.shape == (2, 64)
    assert np.array_equal(W1, W2) and np.array_equal(s1, s2)
    assert np.all(s1 > 0)
