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
    if T == 1:
        assert stack.last_launches() == 1, "the one-token stack should run as one persistent launch"
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
    if T == 1:
        # one launch per layer instead of the persistent launch: the same layer, the
        # cross-CTA sums grouped differently (the persistent split rotates per layer)
        stack.set_prefetch(False)
        with torch.cuda.stream(s):
            stack.forward(x_dev, lg_dev, k, y_dev, stream=s)
        torch.cuda.synchronize()
        y_per = y_dev.view(torch.int16).cpu().numpy().view(np.uint16)
        for l in range(layers):
            harness.assert_output_close(y.view(np.uint16)[l], harness.bf16_to_f64(y_per[l]),
                                        f"{name}: persistent against per-layer launches, layer {l}")
        stack.set_prefetch(True)
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


@pytest.mark.parametrize("E,H,I,k", [(8, 256, 128, 2), (128, 2048, 768, 8)])
def test_persistent_stack_one_token(torch_cuda, E, H, I, k):
    """At T = 1 the stack runs as one persistent launch (every layer routed up
    front, the weights streamed through a shared-memory ring across layer
    boundaries).  Independent and chained layers, against the oracle layer by
    layer (chained: the first two layers, whose inputs are still far from
    zero), and against one launch per layer."""
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    n = 6
    layers = []
    for l in range(n):
        if H <= 256:
            gl = harness.GpuLayer(E, H, I, 500 + l, max_T=1, max_k=k, source="host")
        else:
            gl = harness.GpuLayer(E, H, I, 500 + l, max_T=1, max_k=k)
        layers.append(gl.layer)
    stack = fe.Stack(layers)
    xs = np.stack([synth.activations_bf16(510 + l, 1, H) for l in range(n)])
    lg = np.ascontiguousarray(np.stack([synth.router_logits(520 + l, 1, E) for l in range(n)]), dtype=np.float32)
    lg_dev = torch.from_numpy(lg).cuda()
    x_dev = torch.from_numpy(xs.view(np.int16)).cuda()
    # independent layers: one launch
    y1 = torch.empty_like(x_dev)
    for _ in range(3):   # repeated launches: tags and counters of later launches
        stack.forward(x_dev.view(torch.bfloat16), lg_dev, k, y1.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert stack.last_launches() == 1
    ya = y1.cpu().numpy().view(np.uint16)
    for l in range(n):
        osd = harness.OracleSide(E, H, I, 500 + l)
        harness.assert_output_close(ya[l], osd.forward(xs[l], lg[l], k)[0], f"persistent, layer {l}")
    # the same with one launch per layer
    stack.set_prefetch(False)
    y2 = torch.empty_like(x_dev)
    stack.forward(x_dev.view(torch.bfloat16), lg_dev, k, y2.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert stack.last_launches() == n
    yb = y2.cpu().numpy().view(np.uint16)
    for l in range(n):
        harness.assert_output_close(ya[l], harness.bf16_to_f64(yb[l]), f"persistent against per-layer, layer {l}")
    stack.set_prefetch(True)
    # chained: y = x shifted by one layer
    buf = torch.zeros((n + 1, 1, H), dtype=torch.int16, device="cuda")
    buf[0].copy_(x_dev[0])
    for _ in range(2):
        stack.forward(buf[0:].view(torch.bfloat16), lg_dev, k, buf[1:].view(torch.bfloat16))
    torch.cuda.synchronize()
    assert stack.last_launches() == 1
    yc = buf.cpu().numpy().view(np.uint16)
    chain = harness.oracle_chain(500, 2, xs[0][0], lg[:2, 0, :], k, E, H, I)
    for l in range(2):
        harness.assert_output_close(yc[l + 1], chain[l][0].reshape(1, H), f"persistent chained, layer {l}")
    # and against one launch per layer, chained the same way
    stack.set_prefetch(False)
    buf2 = torch.zeros_like(buf)
    buf2[0].copy_(x_dev[0])
    stack.forward(buf2[0:].view(torch.bfloat16), lg_dev, k, buf2[1:].view(torch.bfloat16))
    torch.cuda.synchronize()
    yd = buf2.cpu().numpy().view(np.uint16)
    harness.assert_output_close(yc[1], harness.bf16_to_f64(yd[1]), "chained, layer 0 against per-layer")
    st, bits = layers[0].status()
    assert st == fe.FE_OK and bits == 0, f"device status bits {bits:#x}"
    stack.close()


@pytest.mark.parametrize("T", [2, 4])
def test_persistent_stack_few_sparse_tokens(torch_cuda, T):
    """A few tokens with sparse routing (the 512-expert layer, top-10) run as one persistent
    launch per token: against one launch per layer, the oracle on layer 0, and every layer's
    routing and grouping of all T tokens bit for bit; independent and chained layers."""
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    import oracle
    E, H, I, k, n = 512, 2048, 512, 10, 3
    layers = [harness.GpuLayer(E, H, I, 600 + l, max_T=T, max_k=k).layer for l in range(n)]
    stack = fe.Stack(layers)
    xs = np.stack([synth.activations_bf16(610 + l, T, H) for l in range(n)])
    lg = np.ascontiguousarray(np.stack([synth.router_logits(620 + l, T, E) for l in range(n)]), dtype=np.float32)
    x_dev = torch.from_numpy(xs.view(np.int16)).cuda()
    lg_dev = torch.from_numpy(lg).cuda()
    y1 = torch.empty_like(x_dev)
    for _ in range(2):
        stack.forward(x_dev.view(torch.bfloat16), lg_dev, k, y1.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert stack.last_launches() == T
    ya = y1.cpu().numpy().view(np.uint16)
    orc = oracle.default()
    for l, layer in enumerate(layers):
        idx, w, off, sp = layer.routing(T, k)
        counts, pr = layer.grouping(T, k)
        torch.cuda.synchronize()
        idx_ref, w_ref = orc.route(lg[l], k)
        c_ref, off_ref, sp_ref, pr_ref = orc.group(idx_ref, E)
        assert np.array_equal(idx.cpu().numpy(), idx_ref) and np.array_equal(off.cpu().numpy(), off_ref)
        assert np.array_equal(sp.cpu().numpy(), sp_ref) and np.array_equal(pr.cpu().numpy(), pr_ref)
        assert np.array_equal(counts.cpu().numpy(), c_ref)
        np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=1e-6, atol=1e-7)
    osd = harness.OracleSide(E, H, I, 600)
    harness.assert_output_close(ya[0], osd.forward(xs[0], lg[0], k)[0], f"persistent T={T}, layer 0")
    stack.set_prefetch(False)
    y2 = torch.empty_like(x_dev)
    stack.forward(x_dev.view(torch.bfloat16), lg_dev, k, y2.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert stack.last_launches() > T
    yb = y2.cpu().numpy().view(np.uint16)
    for l in range(n):
        harness.assert_output_close(ya[l], harness.bf16_to_f64(yb[l]), f"T={T} persistent against per-layer, layer {l}")
    # chained: y = x shifted by one layer, per token
    buf = torch.zeros((n + 1, T, H), dtype=torch.int16, device="cuda")
    buf[0].copy_(x_dev[0])
    stack.forward(buf[0:].view(torch.bfloat16), lg_dev, k, buf[1:].view(torch.bfloat16))
    torch.cuda.synchronize()
    yc_per = buf.cpu().numpy().view(np.uint16).copy()
    stack.set_prefetch(True)
    buf2 = torch.zeros_like(buf)
    buf2[0].copy_(x_dev[0])
    stack.forward(buf2[0:].view(torch.bfloat16), lg_dev, k, buf2[1:].view(torch.bfloat16))
    torch.cuda.synchronize()
    assert stack.last_launches() == T
    yc = buf2.cpu().numpy().view(np.uint16)
    harness.assert_output_close(yc[1], harness.bf16_to_f64(yc_per[1]), f"T={T} chained, layer 0 against per-layer")
    st, bits = layers[0].status()
    assert st == fe.FE_OK and bits == 0, f"device status bits {bits:#x}"
    stack.close()
