"""The seeded input generator (host side): published test vector, determinism,
random access, distribution."""
import os

import numpy as np

import pins
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_splitmix64_published_sequence():
    exp = [int(v) for v in open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt"))
           if v.strip() and not v.startswith("#")]
    n = np.arange(1, 6, dtype=np.uint64)
    with np.errstate(over="ignore"):
        got = synth.mix64(np.uint64(1234567) + n * synth.GAMMA)
    assert [int(v) for v in got] == exp


def test_normal_moments_and_range():
    z = synth.normal_f32(3, 0, np.arange(1 << 20, dtype=np.uint64)).astype(np.float64)
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    assert np.abs(z).max() <= 6.0
    # exact multiples of 2**-16
    assert np.all(z * 65536 == np.round(z * 65536))


def test_random_access_and_subsets():
    E, H, I = 6, 64, 32
    full = synth.weights_gate_up(9, E, H, I)
    sub = synth.weights_gate_up(9, E, H, I, experts=[4, 1])
    assert np.array_equal(sub[0], full[4]) and np.array_equal(sub[1], full[1])
    dn = synth.weights_down(9, E, I, H)
    dn_sub = synth.weights_down(9, E, I, H, experts=[5])
    assert np.array_equal(dn_sub[0], dn[5])
    # gate and up halves are different tensors
    assert not np.array_equal(full[:, :, :I], full[:, :, I:])
    again = synth.weights_gate_up(9, E, H, I)
    assert np.array_equal(full, again)
    other_seed = synth.weights_gate_up(10, E, H, I)
    assert not np.array_equal(full, other_seed)


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(300).astype(np.float32),
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)])
    got = synth.bf16_bits_rne(v)
    for a, b in zip(v, got):
        assert int(b) == pins.nearest_bf16_bits(np.float32(a))


def test_zipf_bias_skews_routing():
    cfg = synth.WORKLOADS["decode_e128_t64_zipf"]
    lg = synth.router_logits(cfg["seeds"][0], cfg["T"], cfg["E"], zipf_s=cfg["zipf"])
    top = np.argsort(-lg, axis=1, kind="stable")[:, :cfg["top_k"]]
    counts = np.bincount(top.reshape(-1), minlength=cfg["E"])
    assert (counts == 0).sum() > 20          # some experts receive no token
    assert counts.max() >= 48                # the hottest expert takes most tokens


def test_host_c_generator_equals_numpy_definition():
    """The C copy of the generator (used to draw the oracle's weights quickly)
    gives the numpy definition's values bit for bit."""
    assert synth._host_lib() is not None, "gcc build of synth_host.c failed"
    E, H, I = 7, 96, 64
    ex = [6, 0, 3]
    assert np.array_equal(synth.weights_gate_up(21, E, H, I, experts=ex).view(np.uint32),
                          synth._weights_gate_up_np(21, E, H, I, experts=ex).view(np.uint32))
    assert np.array_equal(synth.weights_down(21, E, I, H, experts=ex).view(np.uint32),
                          synth._weights_down_np(21, E, I, H, experts=ex).view(np.uint32))
    got = synth.normal_range_f32(5, synth.TID_LOGITS, 1000, 4096)
    ref = synth.normal_f32(5, synth.TID_LOGITS, np.arange(1000, 5096, dtype=np.uint64))
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # a full-size expert at the 30B-like shape, spot-checked against the definition
    W = synth.weights_gate_up(1000, 128, 2048, 768, experts=[77])
    rows = np.array([0, 1, 1023, 2047], dtype=np.uint64)
    flat = np.uint64(77 * 2048 * 768) + rows[:, None] * np.uint64(768) + np.arange(768, dtype=np.uint64)[None, :]
    assert np.array_equal(W[0, rows.astype(np.int64), 768:],
                          synth.normal_f32(1000, synth.TID_UP, flat) * synth.WEIGHT_STD)
