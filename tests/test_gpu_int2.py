"""Layers whose experts mix E2M1 and INT2 codes (fe_moe_load_int2) against the
oracle's layer with a format per expert, the INT2 packers against the oracle's
INT2 quantiser, and the paths such a layer is refused on."""
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


def mixed_layer(E, H, I, seed, fmt, max_T, max_k, source):
    """A handle with every expert's E2M1 weights, then INT2 weights for fmt[e] = 1 (the same
    seeded float weights, quantised to INT2)."""
    import torch

    import fp4_expert_gemv_b200 as fe
    gl = harness.GpuLayer(E, H, I, seed, max_T=max_T, max_k=max_k, source=source)
    if source == "device":
        st = torch.cuda.current_stream().cuda_stream
        W = torch.empty((E, H, 2 * I), dtype=torch.float32, device="cuda")
        synth.device_gate_up(W.data_ptr(), seed, E, H, I, st)
        gc, gs = fe.pack_int2_device(W)
        del W
        W = torch.empty((E, I, H), dtype=torch.float32, device="cuda")
        synth.device_down(W.data_ptr(), seed, E, I, H, st)
        dc, ds = fe.pack_int2_device(W)
        del W
    else:
        gc, gs = fe.pack_int2_host(synth.weights_gate_up(seed, E, H, I))
        dc, ds = fe.pack_int2_host(synth.weights_down(seed, E, I, H))
    gl.layer.load_int2(fmt, gc, gs, dc, ds)
    torch.cuda.synchronize()
    return gl


def test_pack_int2_device_matches_host_and_oracle(torch_cuda):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((3, 96, 40)) * 0.02).astype(np.float32)
    W[1, 32:64, 7] = 0.0                                          # an all-zero group
    W[2, 0:4, 3] = [1.5, -1.0, 0.0, 1.0]                          # midpoints at scale 1
    c_dev, s_dev = fe.pack_int2_device(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    c_host, s_host = fe.pack_int2_host(W)
    c_ref, s_ref = oracle.default().quantize_int2(W)
    assert np.array_equal(c_dev.cpu().numpy(), c_host) and np.array_equal(c_host, c_ref)
    assert np.array_equal(s_dev.cpu().numpy().view(np.uint16), s_host) and np.array_equal(s_host, s_ref)


# E, H, I, top_k, T, format rule, weights source: the 30B-like decode layer with every
# other expert INT2 at T = 1 (top-8) and T = 2 (top-4, so that the pairs fit the
# single-launch kernel), the 512-expert layer with every third expert INT2, and a tiny
# layer with every expert INT2 (four tokens, eight pairs)
CASES = [
    (128, 2048, 768, 8, 1, "odd", "device"),
    (128, 2048, 768, 4, 2, "odd", "device"),
    (512, 2048, 512, 10, 1, "third", "device"),
    (8, 256, 128, 2, 4, "all", "host"),
]


@pytest.mark.parametrize("E,H,I,k,T,rule,source", CASES)
def test_mixed_layer_matches_oracle(torch_cuda, E, H, I, k, T, rule, source):
    import fp4_expert_gemv_b200 as fe
    fmt = [1 if (rule == "all" or (rule == "odd" and e % 2) or (rule == "third" and e % 3 == 0)) else 0
           for e in range(E)]
    seed = 41
    gl = mixed_layer(E, H, I, seed, fmt, max_T=max(T, 8), max_k=k, source=source)
    x = synth.activations_bf16(seed + T, T, H)
    lg = synth.router_logits(seed + T, T, E)
    idx_ref, _ = oracle.default().route(lg, k)
    routed = set(int(e) for e in idx_ref.reshape(-1))
    assert any(fmt[e] for e in routed), "the batch should reach an INT2 expert"
    if rule != "all":
        assert any(not fmt[e] for e in routed), "and an E2M1 one"
    y, idx, w, off, sp = gl.forward(x, lg, k)
    assert gl.layer.last_forward_info()[0] == fe.PATH_FUSED_DECODE
    assert np.array_equal(idx, idx_ref)
    osd = harness.OracleSide(E, H, I, seed, fmt=fmt)
    ref, _ = osd.forward(x, lg, k)
    harness.assert_output_close(y, ref, f"mixed E={E} T={T} ({rule} INT2)")
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0


def test_int2_layer_runs_only_on_the_decode_path(torch_cuda):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    E, H, I, k = 8, 256, 128, 2
    fmt = [e % 2 for e in range(E)]
    gl = mixed_layer(E, H, I, 43, fmt, max_T=64, max_k=k, source="host")
    x = torch.from_numpy(synth.activations_bf16(5, 64, H).view(np.int16)).cuda().view(torch.bfloat16)
    lg = torch.from_numpy(synth.router_logits(5, 64, E)).cuda()
    y = torch.empty_like(x)
    # more pairs than the single-launch kernel takes: refused before anything runs
    assert fe.fe_moe_forward(gl.layer.h, x.data_ptr(), lg.data_ptr(), 64, k, y.data_ptr(), None) == \
        fe.FE_ERR_UNSUPPORTED
    # another path forced at T = 1: refused
    gl.layer.set_path(fe.PATH_GEMV)
    assert fe.fe_moe_forward(gl.layer.h, x.data_ptr(), lg.data_ptr(), 1, k, y.data_ptr(), None) == \
        fe.FE_ERR_UNSUPPORTED
    gl.layer.set_path(0)
    # a stack of such layers runs one launch per layer, equal to the layers called in turn
    gl2 = mixed_layer(E, H, I, 44, fmt, max_T=64, max_k=k, source="host")
    stack = fe.Stack([gl.layer, gl2.layer])
    xs = torch.from_numpy(np.stack([synth.activations_bf16(6 + l, 1, H) for l in range(2)]).view(np.int16)).cuda()
    lgs = torch.from_numpy(np.stack([synth.router_logits(6 + l, 1, E) for l in range(2)])).cuda()
    ys = torch.empty_like(xs)
    stack.forward(xs.view(torch.bfloat16), lgs, k, ys.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert stack.last_launches() == 2
    for l, layer in enumerate((gl.layer, gl2.layer)):
        yl = layer.forward(xs[l].view(torch.bfloat16), lgs[l], k)
        torch.cuda.synchronize()
        assert torch.equal(yl.view(torch.int16), ys[l])
    stack.close()
