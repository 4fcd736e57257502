"""The 48-layer stacks the benchmark times (fe_moe_stack_forward captured in
one CUDA graph, built by the benchmark's own code), against the CPU oracle,
and the stack entry points' chaining and host-buffer forms.

Each benchmark layer has its own seeded weights, x and logits (seed
1000 + l), so the first and the last layer of the timed graph are compared
with the oracle directly.
"""
import numpy as np
import pytest

import bench
import harness
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@pytest.mark.parametrize("name", ["decode_e128_t1", "prefill_e128_t4096"])
def test_stack_graph_layers_0_and_last_match_oracle(torch_cuda, name):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    cfg = synth.WORKLOADS[name]
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    layers = bench.LAYERS
    device = torch.device("cuda", 0)
    handles = bench.build_stack(cfg, layers, device)
    stack = fe.Stack(handles)
    x, lg = bench.stack_inputs(cfg, layers)
    x_dev = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    lg_dev = torch.from_numpy(lg).to(device)
    y_dev = torch.empty((layers, T, H), dtype=torch.bfloat16, device=device)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        stack.forward(x_dev, lg_dev, k, y_dev, stream=s)
    torch.cuda.synchronize()
    y_direct = y_dev.view(torch.int16).cpu().numpy().copy()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        stack.forward(x_dev, lg_dev, k, y_dev, stream=s)
    y_dev.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    y = y_dev.view(torch.int16).cpu().numpy()
    assert np.array_equal(y, y_direct), "graph replay differs from the direct stack forward"
    y = y.view(np.uint16)
    rows = np.arange(T) if T <= 8 else np.unique(np.linspace(0, T - 1, 24).astype(np.int64))
    for l in (0, layers - 1):
        osd = harness.OracleSide(E, H, I, synth.STACK_SEED0 + l)
        ref, _ = osd.forward(x[l][rows], lg[l][rows], k)
        harness.assert_output_close(y[l][rows], ref, f"{name}: layer {l} of the timed graph")
    del g
    stack.close()
    for m in handles:
        m.close()
    torch.cuda.empty_cache()


def test_stack_chaining_and_host_forms(torch_cuda):
    """y = x shifted by one layer chains the layers: the result equals calling
    each handle in turn; the host-buffer forms (independent and chained) equal
    the device forms bit for bit; layer 0 matches the oracle."""
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    E, H, I, k, T, n = 8, 256, 128, 2, 5, 3
    layers = []
    for l in range(n):
        gl = harness.GpuLayer(E, H, I, 300 + l, max_T=8, max_k=4, source="host")
        layers.append(gl.layer)
    stack = fe.Stack(layers)
    xs = np.stack([synth.activations_bf16(310 + l, T, H) for l in range(n)])
    lg = np.ascontiguousarray(np.stack([synth.router_logits(320 + l, T, E) for l in range(n)]), dtype=np.float32)
    lg_dev = torch.from_numpy(lg).cuda()
    # chained on the device: one buffer of n + 1 layers' rows
    buf = torch.zeros((n + 1, T, H), dtype=torch.int16, device="cuda")
    buf[0].copy_(torch.from_numpy(xs[0].view(np.int16)))
    stack.forward(buf[0:].view(torch.bfloat16), lg_dev, k, buf[1:].view(torch.bfloat16))
    # the same by hand
    cur = buf[0].view(torch.bfloat16).clone()
    for l in range(n):
        cur = layers[l].forward(cur, lg_dev[l], k)
    torch.cuda.synchronize()
    assert np.array_equal(buf[n].cpu().numpy(), cur.view(torch.int16).cpu().numpy())
    # host, chained
    y_host = np.empty((T, H), dtype=np.uint16)
    stack.forward_host(np.ascontiguousarray(xs[0]), lg, k, y_host, chained=True)
    assert np.array_equal(y_host.view(np.int16), buf[n].cpu().numpy())
    # independent layers, device and host forms
    x_dev = torch.from_numpy(xs.view(np.int16)).cuda()
    y_dev = torch.empty_like(x_dev)
    stack.forward(x_dev.view(torch.bfloat16), lg_dev, k, y_dev.view(torch.bfloat16))
    y_ind = np.empty((n, T, H), dtype=np.uint16)
    stack.forward_host(xs, lg, k, y_ind, chained=False)
    torch.cuda.synchronize()
    assert np.array_equal(y_ind.view(np.int16), y_dev.cpu().numpy())
    osd = harness.OracleSide(E, H, I, 300)
    harness.assert_output_close(y_ind[0], osd.forward(xs[0], lg[0], k)[0], "stack layer 0")
    # y overlapping x of the same layer is refused before anything runs
    assert fe.fe_moe_stack_forward(stack.h, x_dev.data_ptr(), lg_dev.data_ptr(), T, k, x_dev.data_ptr() + 2,
                                   None) == fe.FE_ERR_INVALID_ARG
    stack.close()
