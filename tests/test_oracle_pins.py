"""The oracle against its pins (no GPU): see pins.py for what each pin rests on."""
import numpy as np
import pytest

import pins


@pytest.mark.parametrize("name,check", pins.ALL_CHECKS, ids=[n for n, _ in pins.ALL_CHECKS])
def test_pin(orc, name, check):
    check(orc, np.random.default_rng(2024))


def test_tiny_workload_dense_bruteforce(orc):
    """The tiny workload (E=8, H=256, I=128, top-2, T=4, seed 0), quantised by the
    oracle, against the unpermuted dense loop written in pins.py."""
    import synth
    cfg = synth.WORKLOADS["tiny"]
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    seed = cfg["seeds"][0]
    Wgu = synth.weights_gate_up(seed, E, H, I)
    Wdn = synth.weights_down(seed, E, I, H)
    x = synth.activations_bf16(seed, T, H)
    logits = synth.router_logits(seed, T, E)
    gc, gs = orc.quantize(Wgu)
    dc, ds = orc.quantize(Wdn)
    ew = orc.quantized_experts(E, Wgu, Wdn, range(E))
    y64, yb = orc.moe_forward(ew, x, logits, k)
    ref = pins.dense_layer_reference(x, logits, k, gc, gs, dc, ds)
    assert np.abs(y64 - ref).max() <= 1e-10 * np.abs(ref).max()
    # the stored bf16 copy is the once-rounded fp64 value
    for t in range(T):
        for h in (0, 17, H - 1):
            assert int(yb[t, h]) == orc.f64_to_bf16(y64[t, h])
    # quantisation error of the packed weights is small against the weights themselves
    deq = pins.dequant_dense(gc, gs)
    rel = np.linalg.norm(deq - Wgu) / np.linalg.norm(Wgu)
    assert rel < 0.15


def test_zero_tokens_and_bad_args(orc):
    ew = orc.quantized_experts(2, np.zeros((2, 32, 64), np.float32), np.zeros((2, 32, 32), np.float32),
                               range(2))
    y64, yb = orc.moe_forward(ew, np.zeros((0, 32), np.uint16), np.zeros((0, 2), np.float32), 1)
    assert y64.shape == (0, 32)
    with pytest.raises(ValueError):
        orc.route(np.zeros((1, 4), np.float32), 5)
    with pytest.raises(ValueError):
        orc.group(np.array([[0, 7]], np.int32), 4)


def test_unmaterialised_expert_is_an_error(orc):
    import oracle
    ew = oracle.ExpertWeights(4, 32, 32)
    ew.set(0, np.zeros((16, 64), np.uint8), np.zeros((1, 64), np.uint16),
           np.zeros((16, 32), np.uint8), np.zeros((1, 32), np.uint16))
    logits = np.array([[0.0, 5.0, 0.0, 0.0]], np.float32)   # routes to expert 1
    with pytest.raises(ValueError):
        orc.moe_forward(ew, np.zeros((1, 32), np.uint16), logits, 1)
