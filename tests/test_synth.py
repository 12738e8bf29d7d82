"""The seeded input generator: published test vectors, determinism, slices, distributions."""
import numpy as np

import synth


def test_splitmix64_published_vectors():
    # SplitMix64 seeded with state 0: first two outputs (Vigna's splitmix64.c)
    assert synth.mix(0) == 0xE220A8397B1DCDAF
    assert synth.mix(0x9E3779B97F4A7C15) == 0x6E789E6AA1B965F4
    assert synth.mix((2 * 0x9E3779B97F4A7C15) % 2**64) == 0x06C45D188009454F


def test_counter_based_slices_match_full_draw():
    full = synth.normal(3, 2, 0, 10000)
    part = synth.normal(3, 2, 1234, 777)
    np.testing.assert_array_equal(part, full[1234:1234 + 777])
    assert synth.normal_one(3, 2, 1234) == np.float64(synth.normal_one(3, 2, 1234))
    assert np.float32(synth.normal_one(3, 2, 1234)) == full[1234]
    rows = synth.unit_rows(5, 1, 0, 50, 16)
    np.testing.assert_array_equal(synth.unit_rows(5, 1, 20, 10, 16), rows[20:30])


def test_threads_do_not_change_values():
    a = synth.normal(9, 0, 0, 200000)  # threaded
    b = np.concatenate([synth.normal(9, 0, i, 1000) for i in range(0, 200000, 1000)])  # single-threaded pieces
    np.testing.assert_array_equal(a, b)


def test_distributions():
    x = synth.normal(1, 0, 0, 2_000_000).astype(np.float64)
    assert abs(x.mean()) < 3e-3 and abs(x.std() - 1) < 3e-3
    # tails of a normal: P(|x| > 3) ~ 0.0027
    assert abs((np.abs(x) > 3).mean() - 0.0027) < 4e-4
    y = synth.normal(1, 3, 0, 100000, mean=-2.0)
    assert abs(y.mean() + 2.0) < 0.02
    u = synth.unit_rows(2, 1, 0, 4000, 112).astype(np.float64)
    np.testing.assert_allclose(np.linalg.norm(u, axis=1), 1.0, atol=1e-6)
    # isotropy: mean ~ 0, covariance ~ I/d
    assert np.abs(u.mean(axis=0)).max() < 0.01
    c = u.T @ u / len(u)
    assert np.abs(np.diag(c) - 1 / 112).max() < 2e-3


def test_different_streams_differ():
    assert not np.array_equal(synth.normal(0, 0, 0, 100), synth.normal(0, 1, 0, 100))
    assert not np.array_equal(synth.normal(0, 0, 0, 100), synth.normal(1, 0, 0, 100))


def test_workload_inputs_heads_slice():
    w = synth.WORKLOADS["gdn_480p_5s"].with_(F=3, L=7, H=3)
    full = synth.inputs(w)
    part = synth.inputs(w, heads=[2])
    for key in "qkvab":
        np.testing.assert_array_equal(part[key][0], full[key].reshape((w.B * w.H,) + full[key].shape[2:])[2])
    assert full["q"].shape == (1, 3, 21, 112) and full["a"].shape == (1, 3, 3)
    s0 = synth.inputs(synth.WORKLOADS["gdn_stream_720p"].with_(L=5, H=2), call=0)
    s1 = synth.inputs(synth.WORKLOADS["gdn_stream_720p"].with_(L=5, H=2), call=1)
    assert s0["q"].shape == (1, 2, 5, 112) and not np.array_equal(s0["q"], s1["q"])


def test_leading_frames_match_full_draw():
    w = synth.WORKLOADS["gdn_480p_5s"].with_(F=4, L=5, H=3)
    full = synth.inputs(w)
    part = synth.inputs(w, frames=2)
    for key in "qkvb":
        np.testing.assert_array_equal(part[key], full[key][:, :, :10])
    np.testing.assert_array_equal(part["a"], full["a"][:, :, :2])
