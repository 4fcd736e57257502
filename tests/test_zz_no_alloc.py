"""The allocation-free entry point, fe_moe_forward_noalloc, through the C ABI.

It serves callers that may not allocate device memory when they run the layer
(an external memory manager owns every device byte, or no allocating call is
allowed at that point): its scratch is one static device array instead of a
reserved workspace.  Its output must match the regular entry point,
fe_moe_forward, within the acceptance tolerance of the other tests, on two
calls in a row, since every call shares and reuses the same static array.

This file's name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest

import harness
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _device_layer(torch, fe, E, H, I, seed):
    """Packed weights in the public format on the device, and a handle loaded with them."""
    st = torch.cuda.current_stream().cuda_stream
    W = torch.empty((E, H, 2 * I), dtype=torch.float32, device="cuda")
    synth.device_gate_up(W.data_ptr(), seed, E, H, I, st)
    gc, gs = fe.pack_device(W)
    W = torch.empty((E, I, H), dtype=torch.float32, device="cuda")
    synth.device_down(W.data_ptr(), seed, E, I, H, st)
    dc, ds = fe.pack_device(W)
    del W
    layer = fe.MoELayer(E, H, I, max_T=8, max_top_k=min(16, E))
    layer.load_packed(gc, gs, dc, ds)
    torch.cuda.synchronize()
    return (gc, gs, dc, ds), layer


def _noalloc(fe, torch, E, H, I, packed, x, lg, k):
    gc, gs, dc, ds = packed
    T = x.shape[0]
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    st = fe.fe_moe_forward_noalloc(E, H, I, gc.data_ptr(), gs.data_ptr(), dc.data_ptr(), ds.data_ptr(),
                                   x.data_ptr(), lg.data_ptr(), T, k, y.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    fe.check(st, "fe_moe_forward_noalloc")
    return y


@pytest.mark.parametrize("name", ["tiny", "decode_e128_t1"])
def test_noalloc_matches_forward_twice(torch_cuda, name):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    cfg = synth.WORKLOADS[name]
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    packed, layer = _device_layer(torch, fe, E, H, I, cfg["seeds"][0])
    for call, (T, seed) in enumerate([(cfg["T"], 90), (3, 91)]):   # two calls in a row, different sizes
        xh = synth.activations_bf16(seed, T, H)
        lh = synth.router_logits(seed, T, E)
        x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
        lg = torch.from_numpy(lh).cuda()
        y_na = _noalloc(fe, torch, E, H, I, packed, x, lg, k)
        y_ref = layer.forward(x, lg, k)
        torch.cuda.synchronize()
        a = y_na.view(torch.int16).cpu().numpy().view(np.uint16)
        b = harness.bf16_to_f64(y_ref.view(torch.int16).cpu().numpy().view(np.uint16))
        harness.assert_output_close(a, b, f"{name} call {call}")
    layer.close()


def test_noalloc_rejects_sizes_beyond_its_array(torch_cuda):
    import fp4_expert_gemv_b200 as fe
    E, H, I = 128, 2048, 768
    # 64 tokens * top-8 = 512 pairs need 512 * (768 + 2048) * 4 bytes > 4 MiB
    st = fe.fe_moe_forward_noalloc(E, H, I, 256, 256, 256, 256, 256, 256, 64, 8, 512, None)
    assert st == fe.FE_ERR_CAPACITY
    assert b"static" in fe.fe_moe_last_error()
