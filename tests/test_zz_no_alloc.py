"""The allocation-free entry point, fe_moe_forward_noalloc, through the C ABI.

It serves callers that may not allocate device memory when they run the layer
(an external memory manager owns every device byte, or no allocating call is
allowed at that point): its scratch is one static device array instead of a
reserved workspace.  Its output must match the regular entry point,
fe_moe_forward, and the CPU oracle within the acceptance tolerance of the other
tests, on calls in a row, since every call shares and reuses the same static
array; its routing and grouping must equal the oracle's bit for bit.

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
    layer = fe.MoELayer(E, H, I, max_T=64, max_top_k=min(16, E))
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


def _noalloc_routing(fe, torch, E, T, k):
    dev = torch.device("cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sp = torch.empty(T * k, dtype=torch.int32, device=dev)
    pr = torch.empty(T * k, dtype=torch.int32, device=dev)
    fe.check(fe.fe_moe_noalloc_get_routing(E, T, k, idx.data_ptr(), w.data_ptr(), counts.data_ptr(), off.data_ptr(),
                                           sp.data_ptr(), pr.data_ptr(), torch.cuda.current_stream().cuda_stream),
             "fe_moe_noalloc_get_routing")
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (idx, w, counts, off, sp, pr)]


# (workload, [(T, top_k, input seed), ...]): two or more calls in a row on one
# set of weights.  T=32 on the tiny layer puts about 8 pairs on each expert,
# more than one staged chunk of the projection kernels; the 512-expert layer
# runs top-10 at T=4.
CASES = [
    ("tiny", [(4, 2, 90), (3, 2, 91), (32, 2, 92)]),
    ("decode_e128_t1", [(1, 8, 93), (3, 8, 94)]),
    ("decode_e512_t4", [(4, 10, 95), (1, 10, 96)]),
]


@pytest.mark.parametrize("name,calls", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_forward_and_oracle(torch_cuda, name, calls):
    """Calls in a row through the static array: y against the regular entry
    point (fe_moe_forward) and against the CPU oracle within the acceptance
    tolerance; routing and grouping bit-exact against the oracle."""
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    import oracle
    cfg = synth.WORKLOADS[name]
    E, H, I = cfg["E"], cfg["H"], cfg["I"]
    seed = cfg["seeds"][0]
    packed, layer = _device_layer(torch, fe, E, H, I, seed)
    osd = harness.OracleSide(E, H, I, seed)
    orc = oracle.default()
    for call, (T, k, s_in) in enumerate(calls):
        xh = synth.activations_bf16(s_in, T, H)
        lh = synth.router_logits(s_in, T, E)
        x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
        lg = torch.from_numpy(lh).cuda()
        y_na = _noalloc(fe, torch, E, H, I, packed, x, lg, k)
        idx, w, counts, off, sp, pr = _noalloc_routing(fe, torch, E, T, k)
        y_ref = layer.forward(x, lg, k)
        torch.cuda.synchronize()
        a = y_na.view(torch.int16).cpu().numpy().view(np.uint16)
        b = harness.bf16_to_f64(y_ref.view(torch.int16).cpu().numpy().view(np.uint16))
        harness.assert_output_close(a, b, f"{name} call {call}: against fe_moe_forward")
        y64, _ = osd.forward(xh, lh, k)
        harness.assert_output_close(a, y64, f"{name} call {call}: against the oracle")
        idx_ref, w_ref = orc.route(lh, k)
        c_ref, off_ref, sp_ref, pr_ref = orc.group(idx_ref, E)
        assert np.array_equal(idx, idx_ref) and np.array_equal(off, off_ref)
        assert np.array_equal(sp, sp_ref) and np.array_equal(pr, pr_ref) and np.array_equal(counts, c_ref)
        np.testing.assert_allclose(w, w_ref, rtol=1e-6, atol=1e-7)
        assert fe.noalloc_status() == (fe.FE_OK, 0)
    layer.close()


def test_noalloc_reports_and_clears_device_status(torch_cuda):
    """A NaN logit is flagged in the array's status word, read (and cleared)
    by fe_moe_noalloc_get_status; the next call starts from a clear word."""
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    cfg = synth.WORKLOADS["tiny"]
    E, H, I = cfg["E"], cfg["H"], cfg["I"]
    packed, layer = _device_layer(torch, fe, E, H, I, cfg["seeds"][0])
    xh = synth.activations_bf16(97, 2, H)
    lh = synth.router_logits(97, 2, E)
    lh[1, 3] = np.nan
    x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
    _noalloc(fe, torch, E, H, I, packed, x, torch.from_numpy(lh).cuda(), 2)
    st, bits = fe.noalloc_status()
    assert st == fe.FE_ERR_DEVICE_STATUS and bits & fe.FE_DEVICE_NAN_LOGIT
    assert fe.noalloc_status() == (fe.FE_OK, 0)
    lh[1, 3] = 0.5
    # a call after a flagged one (its word left set on purpose) starts clean
    _noalloc(fe, torch, E, H, I, packed, x, torch.from_numpy(lh).cuda().clone().fill_(float("nan")), 2)
    _noalloc(fe, torch, E, H, I, packed, x, torch.from_numpy(lh).cuda(), 2)
    assert fe.noalloc_status() == (fe.FE_OK, 0)
    layer.close()


def test_noalloc_rejects_sizes_beyond_its_array(torch_cuda):
    import fp4_expert_gemv_b200 as fe
    E, H, I = 128, 2048, 768
    # 64 tokens * top-8 = 512 pairs need 512 * (768 + 2048) * 4 bytes > 4 MiB
    st = fe.fe_moe_forward_noalloc(E, H, I, 256, 256, 256, 256, 256, 256, 64, 8, 512, None)
    assert st == fe.FE_ERR_CAPACITY
    assert b"static" in fe.fe_moe_last_error()
