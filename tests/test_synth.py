"""The seeded generator against the published SplitMix64 definition."""
import numpy as np

from linear_complexity_vision_b200 import synth


def test_splitmix64_first_outputs_of_seed_zero():
    # SplitMix64 (Steele, Lea, Flood 2014) started from state 0 produces
    # 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F first.
    state = np.uint64(0)
    outs = []
    for i in range(1, 4):
        with np.errstate(over="ignore"):
            z = np.array([state + np.uint64(i) * synth._GOLDEN], dtype=np.uint64)
        outs.append(int(synth._mix(z)[0]))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_streams_are_deterministic_and_distinct():
    a = synth.uniform(7, 2, 1000)
    b = synth.uniform(7, 2, 1000)
    c = synth.uniform(7, 3, 1000)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    assert a.min() >= 0.0 and a.max() < 1.0
    # counter offsets address the same stream
    np.testing.assert_array_equal(synth.uniform(7, 2, 10, offset=990), a[990:])


def test_moments():
    n = synth.normal(11, 0, 200000)
    assert abs(n.mean()) < 0.01 and abs(n.std() - 1.0) < 0.01
    x = synth.draw(11, "w", (100000,), ("uniform", -8, 8))
    assert x.min() >= -8 and x.max() < 8 and abs(x.mean()) < 0.1
    y = synth.draw(11, "k", (100000,), ("normal", 2.0))
    assert abs(y.std() - 2.0) < 0.03


def test_workload_shapes():
    wl = synth.workload(5, B=1, H=4, W=4, C=8)
    inp = wl.generate()
    assert inp["x"].shape == (1, 16, 8) and inp["mu_k"].shape == (8,)
    assert synth.WORKLOADS[4].T == 4096 and synth.WORKLOADS[5].N == 8 * 4096 * 1024
