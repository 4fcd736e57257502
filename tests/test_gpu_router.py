"""The router GEMM fused with the top-k (fe_moe_router) and the layer from x
alone (fe_moe_forward_router), against the oracle.

* logits: the oracle's fp64 sum_h x[t][h] W_r[e][h], within the bound of any
  fp32 summation order, H * 2^-24 * sum_h |x W_r| (the products of two bf16
  values are exact in fp32);
* routing: the oracle's top-k and softmax of the DEVICE's fp32 logits, so that
  the choice of experts is taken in the kernel's precision on both sides:
  expert ids exactly, weights within the routing tolerance of the layer tests;
* layer: y against the oracle's layer on the device's logits.
"""
import numpy as np
import pytest

import harness
import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def check_logits(lg, x_bits, wr_bits, what):
    orc = oracle.default()
    ref = orc.router_logits(x_bits, wr_bits)
    xa = np.abs(harness.bf16_to_f64(x_bits))
    wa = np.abs(harness.bf16_to_f64(wr_bits))
    H = x_bits.shape[1]
    bound = H * 2.0 ** -24 * (xa @ wa.T) + 1e-30
    err = np.abs(lg.astype(np.float64) - ref)
    assert np.all(err <= bound), f"{what}: worst error / bound {float((err / bound).max()):.3f}"


# E, H, top_k, T: the decode layer's router (T = 1, a few tokens, a full tile, ragged
# tiles, many tiles), the 512-expert router, and small shapes with ragged expert
# chunks (E not a multiple of 32), K not a power-of-two multiple of 64, k = E.
CASES = [
    (128, 2048, 8, 1), (128, 2048, 8, 5), (128, 2048, 8, 16), (128, 2048, 8, 37), (128, 2048, 8, 300),
    (512, 2048, 8, 3), (8, 256, 2, 19), (40, 192, 4, 70), (32, 64, 32, 9),
]


@pytest.mark.parametrize("E,H,k,T", CASES)
def test_router_matches_oracle(torch_cuda, E, H, k, T):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    layer = fe.MoELayer(E, H, 64, T, k)
    x = synth.activations_bf16(900 + T, T, H)
    wr = synth.router_weights_bf16(901 + E, E, H)
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    wd = torch.from_numpy(wr.view(np.int16)).cuda()
    lg, idx, w = layer.router(xd, wd, k)
    # a second launch: the per-tile tickets were reset; the same bits come back
    lg2, idx2, w2 = layer.router(xd, wd, k)
    torch.cuda.synchronize()
    assert torch.equal(lg, lg2) and torch.equal(idx, idx2) and torch.equal(w, w2)
    lg, idx, w = lg.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    check_logits(lg, x, wr, f"E={E} H={H} T={T}")
    ridx, rw = oracle.default().route(lg, k)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=1e-6, atol=1e-7)
    st, bits = layer.status()
    assert st == fe.FE_OK and bits == 0


def test_router_edges(torch_cuda):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    E, H, k = 128, 2048, 8
    layer = fe.MoELayer(E, H, 64, 4, k)
    x = torch.zeros((4, H), dtype=torch.int16, device="cuda")
    wr = torch.zeros((E, H), dtype=torch.int16, device="cuda")
    lg = torch.full((4, E), 7.0, dtype=torch.float32, device="cuda")
    # T = 0: nothing is written
    assert fe.fe_moe_router(layer.h, x.data_ptr(), wr.data_ptr(), 0, k, lg.data_ptr(), None, None, None) == fe.FE_OK
    torch.cuda.synchronize()
    assert bool((lg == 7.0).all())
    # misaligned operands, T above the reservation, k too large
    assert fe.fe_moe_router(layer.h, x.data_ptr() + 2, wr.data_ptr(), 1, k, lg.data_ptr(), None, None,
                            None) == fe.FE_ERR_INVALID_ARG
    assert fe.fe_moe_router(layer.h, x.data_ptr(), wr.data_ptr(), 5, k, lg.data_ptr(), None, None,
                            None) == fe.FE_ERR_CAPACITY
    assert fe.fe_moe_router(layer.h, x.data_ptr(), wr.data_ptr(), 1, 33, lg.data_ptr(), None, None,
                            None) == fe.FE_ERR_UNSUPPORTED
    # all-zero router: every logit 0, the lowest k expert ids, equal weights
    l2, idx, w = layer.router(x[:3], wr, k)
    torch.cuda.synchronize()
    assert bool((l2 == 0).all())
    assert idx.cpu().numpy().tolist() == [list(range(k))] * 3
    np.testing.assert_allclose(w.cpu().numpy(), 1.0 / k, rtol=1e-6)


@pytest.mark.parametrize("E,H,I,k,T", [(128, 2048, 768, 8, 1), (128, 2048, 768, 8, 64), (8, 256, 128, 2, 37)])
def test_forward_router_matches_oracle(torch_cuda, E, H, I, k, T):
    """The layer from x alone: router GEMM, top-k, layer.  y against the oracle's layer
    on the device's logits; the logits against the oracle's router GEMM."""
    torch = torch_cuda
    src = "host" if H <= 256 else "device"
    gl = harness.GpuLayer(E, H, I, 77, max_T=T, max_k=k, source=src)
    x = synth.activations_bf16(910 + T, T, H)
    wr = synth.router_weights_bf16(911, E, H)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    wd = torch.from_numpy(wr.view(np.int16)).cuda()
    y, lg = gl.layer.forward_router(xd, wd, k)
    torch.cuda.synchronize()
    lg = lg.cpu().numpy()
    check_logits(lg, x, wr, f"layer E={E} T={T}")
    rows = np.arange(T) if T <= 8 else np.unique(np.linspace(0, T - 1, 16).astype(np.int64))
    osd = harness.OracleSide(E, H, I, 77)
    ref, _ = osd.forward(x[rows], lg[rows], k)
    harness.assert_output_close(y.view(torch.int16).cpu().numpy().view(np.uint16)[rows], ref,
                                f"forward_router E={E} T={T}")
    # the same layer called with those logits gives the same bits
    y2 = gl.layer.forward(xd, torch.from_numpy(lg).cuda(), k)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
