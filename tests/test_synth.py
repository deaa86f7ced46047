"""The seeded input generator (host side) against numpy's Philox4x64-10 and its recipe."""
import math

import numpy as np

import synth


def test_philox_matches_numpy():
    # numpy's Philox (4x64, 10 rounds) increments the counter before each block
    for key, ctr in [((0, 0), (0, 0, 0, 0)), ((5, 7), (3, 0, 0, 0)), ((2**63 + 11, 99), (12345, 6, 0, 1))]:
        g = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(ctr, dtype=np.uint64))
        want = g.random_raw(4)
        c = list(ctr)
        c[0] += 1
        assert np.array_equal(synth.philox_block(c, key), want)


def test_known_answer_zero():
    # published known-answer vector of Philox4x64-10 for counter 0, key 0
    got = synth.philox_block([0, 0, 0, 0], [0, 0])
    assert [int(v) for v in got] == [0x16554d9eca36314c, 0xdb20fe9d672d0fdc,
                                     0xd7e772cee186176b, 0x7e68b68aec7ba23b]


def test_normal_recipe_and_moments():
    n = 1 << 20
    st = synth.stream_id(synth.KIND_EXPERT, 3, 17, 1)
    v = synth.normal_host(n, 42, st, sigma=0.02)
    assert abs(v.mean()) < 3 * 0.02 / math.sqrt(n) * 2
    assert abs(v.std() / 0.02 - 1) < 0.005
    assert np.abs(v).max() < 0.02 * 5.0
    # offsets address the same stream
    tail = synth.normal_host(1000, 42, st, offset=n - 1000, sigma=0.02)
    assert np.array_equal(tail, v[-1000:])
    # recompute a few values from the recipe (the block function is checked against numpy above)
    c = synth.scale_for(0.02)
    for i in (0, 1, 2, 12345):
        blk = synth.philox_block([i >> 1, st, 0, 0], [42, 0])
        a, b = int(blk[2 * (i & 1)]), int(blk[2 * (i & 1) + 1])
        s = sum((a >> (16 * j)) & 0xffff for j in range(4)) + sum((b >> (16 * j)) & 0xffff for j in range(4))
        assert v[i] == np.float32(np.float32(s - 4 * 65535) * np.float32(c))


def test_forced_routing_uniform():
    wl = synth.WORKLOADS["full_q4"]
    f = synth.forced_experts(wl, tokens=256)
    assert f.shape == (256, 1, 4)
    counts = np.bincount(f.reshape(-1), minlength=512)
    assert counts.min() == counts.max() == 2          # 256*4/512 each, exactly
    b = synth.logit_bias(wl, tokens=3)
    assert b.shape == (3, 1, 512) and np.count_nonzero(b[0, 0]) == 4


def test_forced_routing_skewed():
    wl = synth.WORKLOADS["stack_q4_skewed"]
    f = synth.forced_experts(wl, tokens=256)
    assert f.shape == (256, 24, 4)
    for l in (0, 23):
        assert all(len(set(row)) == 4 for row in f[:, l].tolist())
        counts = np.bincount(f[:, l].reshape(-1), minlength=512)
        hot = np.argsort(-counts)[:32]
        share = counts[hot].sum() / counts.sum()
        assert 0.6 < share < 0.8
