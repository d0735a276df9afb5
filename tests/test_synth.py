"""The seeded input generator (not part of the method): SplitMix64 reference
values, counter-based random access, and the distributions it promises."""
import numpy as np

import synth


def test_splitmix64_reference_values():
    # SplitMix64 (Steele, Lea, Flood 2014) from state 0: the widely published
    # first output of the generator seeded with 0.
    assert int(synth.raw_u64(0, 0, 1)[0]) == 0xE220A8397B1DCDAF


def test_random_access_equals_sequential():
    a = synth.normal(5, 1000, 64)
    b = synth.normal_at(5, np.arange(1000, 1064, dtype=np.uint64))
    assert np.array_equal(a, b)
    dims = synth.TINY
    w = synth.model_weights_f32(dims)
    name, layer, shape, off = synth.weight_layout(dims)[6]
    assert (name, layer) == ("wu", 0)
    rows = synth.weight_rows_f32(0, off, shape, [0, 3, 687])
    assert np.array_equal(rows, w["layers"][0]["wu"][[0, 3, 687]])


def test_distributions():
    z = synth.normal(9, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    ids = synth.prompt_ids(synth.TINY, 4, 1000)
    assert ids.min() >= 0 and ids.max() <= 1022 and 1023 not in ids
    x, hc, conf = synth.micro_inputs(2, 500, 64)
    changed = np.abs(x - hc).max(axis=-1) > 0.1
    assert 0.05 < changed.mean() < 0.15
    assert abs(conf.mean() - 5 / 6) < 0.02 and conf.min() >= 0 and conf.max() <= 1
