"""GPU parity of the fe_moe layer against the CPU oracle, through the C ABI.

Routing indices and the grouping are compared bit for bit, slot weights to
1e-6, and y within max|y - y_ref| <= 1e-2 max|y_ref| and
||y - y_ref|| / ||y_ref|| <= 5e-3 against the oracle's fp64 output.
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


def check_routing(orc, logits, k, E, idx, w, off, sp, counts=None, pair_row=None):
    idx_ref, w_ref = orc.route(logits, k)
    counts_ref, off_ref, sp_ref, pr_ref = orc.group(idx_ref, E)
    assert np.array_equal(idx, idx_ref), "router indices differ"
    np.testing.assert_allclose(w, w_ref, rtol=1e-6, atol=1e-7)
    assert np.array_equal(off, off_ref), "expert offsets differ"
    assert np.array_equal(sp, sp_ref), "grouped pair order differs"
    if counts is not None:
        assert np.array_equal(counts, counts_ref), "per-expert pair counts differ"
    if pair_row is not None:
        assert np.array_equal(pair_row, pr_ref), "inverse permutation (pair -> grouped row) differs"


def run_and_check(gl, osd, x, lg, k, sample=None, what="", y_ref=None):
    orc = oracle.default()
    y, idx, w, off, sp = gl.forward(x, lg, k)
    check_routing(orc, lg, k, gl.E, idx, w, off, sp, *gl.last_grouping)
    rows = np.arange(x.shape[0]) if sample is None else np.asarray(sample)
    if y_ref is None:
        y_ref, _ = osd.forward(x[rows], lg[rows], k)
    return harness.assert_output_close(y[rows], y_ref, what)


def covering_rows(logits, k, E, tile=256, group=32, at_least=256, seed=0):
    """Token rows whose pairs touch, for every expert, its first and last
    grouped row and every 32-row epilogue group of every 256-row tile (so a
    second tile of an expert with more than 256 pairs is covered), topped up
    with random rows to at least `at_least`.  Chosen from the oracle's routing."""
    orc = oracle.default()
    idx, _ = orc.route(logits, k)
    counts, off, sp, _ = orc.group(idx, E)
    chosen = set()
    covered = set()
    pos_cell = {}
    for e in range(E):
        o, c = int(off[e]), int(counts[e])
        for r in range(c):
            pos_cell[o + r] = (e, r // tile, (r % tile) // group)
    # cells a token covers, through the inverse permutation
    _, _, _, pr = orc.group(idx, E)
    def cells_of(tok):
        return {pos_cell[int(pr[tok * k + j])] for j in range(k)}
    for e in range(E):
        o, c = int(off[e]), int(counts[e])
        if c == 0:
            continue
        for pos in (o, o + c - 1):
            t = int(sp[pos]) // k
            chosen.add(t)
            covered |= cells_of(t)
    for pos in sorted(pos_cell):
        if pos_cell[pos] not in covered:
            t = int(sp[pos]) // k
            chosen.add(t)
            covered |= cells_of(t)
    rng = np.random.default_rng(seed)
    T = logits.shape[0]
    while len(chosen) < min(at_least, T):
        chosen.add(int(rng.integers(0, T)))
    assert covered == set(pos_cell.values())
    return np.array(sorted(chosen))


def test_device_generator_matches_host(torch_cuda):
    torch = torch_cuda
    E, H, I, seed = 3, 64, 96, 11
    st = torch.cuda.current_stream().cuda_stream
    W = torch.empty((E, H, 2 * I), dtype=torch.float32, device="cuda")
    synth.device_gate_up(W.data_ptr(), seed, E, H, I, st)
    D = torch.empty((E, I, H), dtype=torch.float32, device="cuda")
    synth.device_down(D.data_ptr(), seed, E, I, H, st)
    z = torch.empty(1000, dtype=torch.float32, device="cuda")
    synth.device_normal(z.data_ptr(), seed, synth.TID_X, 1000, 1.0, st)
    torch.cuda.synchronize()
    assert np.array_equal(W.cpu().numpy().view(np.uint32),
                          synth.weights_gate_up(seed, E, H, I).view(np.uint32))
    assert np.array_equal(D.cpu().numpy().view(np.uint32), synth.weights_down(seed, E, I, H).view(np.uint32))
    assert np.array_equal(z.cpu().numpy(), synth.normal_f32(seed, synth.TID_X, np.arange(1000)))


def quantiser_probe(rng):
    E, K, N = 2, 96, 48
    W = (rng.standard_normal((E, K, N)) * 0.02).astype(np.float32)
    W[0, 0:32, 0] = 0.0
    W[1, 32:64, 5] = np.float32(-0.25)
    # exact E2M1 midpoints: the group max 3.0 gives scale bf16(3/6) = 0.5 exactly,
    # so these weights divide to the midpoints 0.25, 0.75, ..., 5
    mids = np.array([3.0, 0.125, 0.375, 0.625, 0.875, 1.25, 1.75, 2.5], dtype=np.float32)
    W[0, 0:8, 7] = mids
    W[0, 8:32, 7] = 0.0
    W[1, 0:8, 3] = -mids
    W[1, 8:32, 3] = 0.0
    W[0, 32:64, 9] = np.float32(1e30)
    return W


def test_pack_device_matches_oracle(torch_cuda):
    import fp4_expert_gemv_b200 as fe
    torch = torch_cuda
    rng = np.random.default_rng(7)
    for W in [quantiser_probe(rng), (rng.standard_normal((3, 256, 64)) * 3).astype(np.float32)]:
        c_ref, s_ref = oracle.default().quantize(W)
        c, s = fe.pack_device(torch.from_numpy(W).cuda())
        torch.cuda.synchronize()
        assert np.array_equal(s.cpu().numpy().view(np.uint16), s_ref)
        assert np.array_equal(c.cpu().numpy(), c_ref)


@pytest.mark.parametrize("path", ["auto", "gemv"])
def test_tiny_layer_host_packed(torch_cuda, path):
    cfg, seed, x, lg = harness.workload_inputs("tiny")
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    gl = harness.GpuLayer(E, H, I, seed, max_T=64, max_k=8, source="host", path=PATHS[path])
    osd = harness.OracleSide(E, H, I, seed)
    run_and_check(gl, osd, x, lg, k, what="tiny")
    # a second batch of other sizes through the same handle: ragged token counts
    for T, kk, s2 in [(1, 2, 21), (7, 3, 22), (33, 8, 23), (64, 1, 24)]:
        x2 = synth.activations_bf16(s2, T, H)
        lg2 = synth.router_logits(s2, T, E)
        run_and_check(gl, osd, x2, lg2, kk, what=f"tiny T={T} k={kk}")


def test_tiny_layer_device_packed_equals_host_packed(torch_cuda):
    torch = torch_cuda
    cfg, seed, x, lg = harness.workload_inputs("tiny")
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    gd = harness.GpuLayer(E, H, I, seed, max_T=8, max_k=8, source="device", keep_packed=True)
    gh = harness.GpuLayer(E, H, I, seed, max_T=8, max_k=8, source="host", keep_packed=True)
    for a, b in zip(gd.packed, gh.packed):
        assert np.array_equal(a.cpu().numpy().view(b.dtype), b)
    ya = gd.forward(x, lg, k)[0]
    yb = gh.forward(x, lg, k)[0]
    assert np.array_equal(ya, yb)


PATHS = {"auto": 0, "gemv": 1, "tc": 2}


@pytest.mark.parametrize("path", ["auto", "gemv"])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_decode_e128_t1(torch_cuda, seed, path):
    cfg, seed, x, lg = harness.workload_inputs("decode_e128_t1", seed=seed)
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    gl = harness.GpuLayer(E, H, I, seed, max_T=64, max_k=16, source="device", keep_packed=True,
                          path=PATHS[path])
    osd = harness.OracleSide(E, H, I, seed)
    run_and_check(gl, osd, x, lg, k, what=f"decode_e128_t1 seed {seed} path {path}")
    import fp4_expert_gemv_b200 as fe
    taken, kernels = gl.layer.last_forward_info()
    assert taken == (fe.PATH_FUSED_DECODE if path == "auto" else fe.PATH_GEMV), taken
    # the device-generated, device-packed bytes of the touched experts equal the oracle's
    idx, _ = oracle.default().route(lg, k)
    for e in np.unique(idx)[:3]:
        gc, gs, dc, ds = (t[e].cpu().numpy() for t in gl.packed)
        rc, rs, rdc, rds = osd.packed[int(e)]
        assert np.array_equal(gc, rc) and np.array_equal(gs.view(np.uint16), rs)
        assert np.array_equal(dc, rdc) and np.array_equal(ds.view(np.uint16), rds)
    if seed == 1:
        # more token counts through the same full-size layer
        for T, s2 in [(2, 31), (5, 32)]:
            x2 = synth.activations_bf16(s2, T, H)
            lg2 = synth.router_logits(s2, T, E)
            run_and_check(gl, osd, x2, lg2, k, what=f"decode_e128 T={T}")


def test_decode_e128_t64_zipf(torch_cuda):
    cfg, seed, x, lg = harness.workload_inputs("decode_e128_t64_zipf")
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    gl = harness.GpuLayer(E, H, I, seed, max_T=64, max_k=8)
    osd = harness.OracleSide(E, H, I, seed)
    idx, _ = oracle.default().route(lg, k)
    counts = np.bincount(idx.reshape(-1), minlength=E)
    assert (counts == 0).sum() > 0 and counts.max() > 32   # skewed, some experts empty
    run_and_check(gl, osd, x, lg, k, what="t64 zipf (all 64 rows)")


@pytest.mark.parametrize("seed,T", [(4, 1), (5, 1), (4, 4), (5, 4)])
def test_decode_e512(torch_cuda, seed, T):
    cfg, seed, x, lg = harness.workload_inputs("decode_e512_t1", seed=seed, T=T)
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    gl = _cached_layer(E, H, I, seed)
    osd = _cached_oracle(E, H, I, seed)
    for path in ("auto", "gemv"):
        gl.layer.set_path(PATHS[path])
        run_and_check(gl, osd, x, lg, k, what=f"e512 seed {seed} T={T} path {path}")
    gl.layer.set_path(0)


_LAYERS, _ORACLES = {}, {}


def _cached_layer(E, H, I, seed):
    key = (E, H, I, seed)
    if key not in _LAYERS:
        _LAYERS.clear()
        _LAYERS[key] = harness.GpuLayer(E, H, I, seed, max_T=16, max_k=16)
    return _LAYERS[key]


def _cached_oracle(E, H, I, seed):
    key = (E, H, I, seed)
    if key not in _ORACLES:
        _ORACLES[key] = harness.OracleSide(E, H, I, seed)
    return _ORACLES[key]


_PREFILL_REF = {}


@pytest.mark.parametrize("path", ["gemv", "tc"])
def test_prefill_t4096_covering_rows(torch_cuda, path):
    """T=4096: routing and grouping compared on all 4096 tokens; y on a row set
    that touches every expert's first and last grouped row and every 32-row
    epilogue group of every 256-row tile (several hundred rows)."""
    import fp4_expert_gemv_b200 as fe
    cfg, seed, x, lg = harness.workload_inputs("prefill_e128_t4096")
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    gl = harness.GpuLayer(E, H, I, seed, max_T=T, max_k=k, path=PATHS[path])
    if "rows" not in _PREFILL_REF:
        rows = covering_rows(lg, k, E)
        assert len(rows) >= 256
        osd = harness.OracleSide(E, H, I, seed)
        _PREFILL_REF["rows"] = rows
        _PREFILL_REF["y"] = osd.forward(x[rows], lg[rows], k)[0]
    rows = _PREFILL_REF["rows"]
    run_and_check(gl, None, x, lg, k, sample=rows, y_ref=_PREFILL_REF["y"],
                  what=f"prefill, {len(rows)} covering rows, path {path}")
    if path == "tc":
        assert gl.layer.last_forward_info()[0] == fe.PATH_TCGEN05
    _LAYERS.clear()


def test_tcgen05_tiles(torch_cuda):
    """Tensor-core tiles: partial tiles, experts without tokens, several
    tiles for one expert, all tokens on one expert."""
    import fp4_expert_gemv_b200 as fe
    E, H, I, seed = 8, 256, 128, 0
    gl = harness.GpuLayer(E, H, I, seed, max_T=600, max_k=8, source="host", path=fe.PATH_TCGEN05)
    osd = harness.OracleSide(E, H, I, seed)
    x = synth.activations_bf16(90, 600, H)
    lg = synth.router_logits(90, 600, E)
    run_and_check(gl, osd, x[:5], lg[:5], 1, what="tc T=5 k=1 (most experts empty)")
    assert gl.layer.last_forward_info()[0] == fe.PATH_TCGEN05
    run_and_check(gl, osd, x[:40], lg[:40], 2, what="tc T=40 k=2")
    run_and_check(gl, osd, x[:64], lg[:64], 8, what="tc T=64 k=8 (every expert, 64 rows)")
    lg_hot = lg.copy()
    lg_hot[:, 3] += 100.0
    run_and_check(gl, osd, x, lg_hot, 1, sample=list(range(0, 600, 37)) + [599],
                  what="tc 600 tokens on one expert: tiles of 256, 256, 88")
    run_and_check(gl, osd, x[:300], lg[:300], 8, sample=list(range(0, 300, 23)) + [299],
                  what="tc T=300 k=8 (2400 pairs, ~300 rows per expert)")
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0


def test_streaming_chunks(torch_cuda):
    """Streaming (moderate-T) kernels with more tokens on one expert than one
    staged chunk holds: gate_up makes one pass over the expert's units per
    16-row chunk, down stages several 64-row chunks per round of units."""
    import fp4_expert_gemv_b200 as fe
    E, H, I, seed, T = 8, 256, 128, 3, 200
    gl = harness.GpuLayer(E, H, I, seed, max_T=T, max_k=2, source="host")
    osd = harness.OracleSide(E, H, I, seed)
    x = synth.activations_bf16(60, T, H)
    lg = synth.router_logits(60, T, E)
    lg[:, 2] += 100.0          # every token's first expert: 200 pairs on expert 2
    lg[: T // 2, 6] += 50.0    # half the tokens' second expert: 100 pairs on expert 6
    rows = np.arange(0, T, 7)
    run_and_check(gl, osd, x, lg, 2, sample=rows, what="one expert over many chunks")
    assert gl.layer.last_forward_info()[0] == fe.PATH_GEMV
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0


@pytest.mark.parametrize("path", ["auto", "gemv"])
def test_edge_cases(torch_cuda, path):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    E, H, I, seed = 8, 256, 128, 0
    gl = harness.GpuLayer(E, H, I, seed, max_T=40, max_k=8, source="host", path=PATHS[path])
    osd = harness.OracleSide(E, H, I, seed)
    x = synth.activations_bf16(50, 40, H)
    # k = 1 and k = E
    lg = synth.router_logits(50, 40, E)
    run_and_check(gl, osd, x, lg, 1, what="k=1")
    run_and_check(gl, osd, x[:5], lg[:5], E, what="k=E")
    # every token to the same experts (one expert holds all pairs), others empty
    lg_hot = lg.copy()
    lg_hot[:, 5] += 100.0
    run_and_check(gl, osd, x, lg_hot, 1, what="all tokens to one expert")
    run_and_check(gl, osd, x, lg_hot, 2, what="one hot expert, k=2")
    # 8 tokens on one expert through the single-launch kernel: a full 8-column block
    run_and_check(gl, osd, x[:8], lg_hot[:8], 1, what="one hot expert, T=8, k=1")
    if path == "auto":
        assert gl.layer.last_forward_info()[0] == fe.PATH_FUSED_DECODE
    # ties: equal logits everywhere, and pairwise ties
    lg_tie = np.zeros((6, E), np.float32)
    lg_tie[1, :] = 1.0
    lg_tie[2, [1, 6]] = 3.0
    lg_tie[3, ::2] = -2.0
    run_and_check(gl, osd, x[:6], lg_tie, 3, what="ties")
    # T = 0 is a no-op
    y = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    fe.check(fe.fe_moe_forward(gl.layer.h, 16, 16, 0, 2, 16, None))
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0
    # bit-reproducible: no atomics decide an order anywhere on this path
    a = gl.forward(x[:300], lg[:300], 8)[0]
    b = gl.forward(x[:300], lg[:300], 8)[0]
    assert np.array_equal(a, b)


def fused_routing_cases(E, k, T):
    """Router logits [T, E] that stress the single-launch kernel's top-k
    selection: the per-lane maxima threshold (lane l holds experts l, l+32, ...),
    its fallback when more than 128 keys tie above it, ties, signed zeros and
    -inf rows."""
    rng = np.random.default_rng(1000 * E + 10 * k + T)
    out = []
    base = rng.standard_normal((T, E)).astype(np.float32)
    out.append(("random", base))
    one_lane = base.copy()
    one_lane[:, ::32] += 10.0          # one lane holds every large key
    out.append(("one lane holds the top", one_lane))
    if E >= 512:
        many = base.copy()
        for lane in range(16):         # lanes 0..15: all 16 keys above the 16th lane maximum
            for j in range(E // 32):
                many[:, lane + 32 * j] = np.float32(100.0 + lane + 0.01 * j)
        out.append(("more than 128 candidates", many))
    out.append(("all equal", np.zeros((T, E), np.float32)))
    ints = rng.integers(-2, 3, (T, E)).astype(np.float32)
    ints[ints == 0] = np.where(rng.random(int((ints == 0).sum())) < 0.5, np.float32(0.0), np.float32(-0.0))
    out.append(("integer ties and signed zeros", ints))
    ninf = np.full((T, E), -np.inf, np.float32)
    ninf[:, rng.integers(0, E, 2)] = 1.0
    out.append(("-inf rows with two finite", ninf))
    return out


@pytest.mark.parametrize("E,k,T", [(512, 10, 1), (512, 16, 1), (128, 8, 2), (20, 4, 4), (8, 2, 8)])
def test_fused_routing_cases(torch_cuda, E, k, T):
    import fp4_expert_gemv_b200 as fe
    H, I, seed = 256, 128, 31
    gl = harness.GpuLayer(E, H, I, seed, max_T=T, max_k=k)
    osd = harness.OracleSide(E, H, I, seed)
    x = synth.activations_bf16(70, T, H)
    for what, lg in fused_routing_cases(E, k, T):
        run_and_check(gl, osd, x, lg, k, what=f"E={E} k={k} T={T}: {what}")
        assert gl.layer.last_forward_info()[0] == fe.PATH_FUSED_DECODE, what


@pytest.mark.parametrize("path", ["auto", "gemv", "tc"])
@pytest.mark.parametrize("scale", [3e5, 1e-4, 1e-8])
def test_activation_magnitudes_use_power_of_two_shift(torch_cuda, scale, path):
    """x far from unit scale: rows are staged in fp16 with a power-of-two shift
    that puts each row's maximum in [2^14, 2^15), so |x| ~ 1e6 does not
    overflow and |x| ~ 1e-8 (act ~ 1e-17) keeps fp16's precision."""
    E, H, I, seed = 8, 256, 128, 0
    T = 40 if path == "tc" else 4
    gl = harness.GpuLayer(E, H, I, seed, max_T=T, max_k=2, source="host", path=PATHS[path])
    osd = harness.OracleSide(E, H, I, seed)
    x = synth.activations_bf16(60, T, H)
    xs = synth.bf16_bits_rne(synth.bf16_bits_to_f32(x) * np.float32(scale))
    lg = synth.router_logits(60, T, E)
    run_and_check(gl, osd, xs, lg, 2, what=f"|x| ~ {scale:g}, path {path}")


def test_nan_logit_sets_status(torch_cuda):
    import fp4_expert_gemv_b200 as fe
    E, H, I, seed = 8, 256, 128, 0
    gl = harness.GpuLayer(E, H, I, seed, max_T=4, max_k=2, source="host")
    x = synth.activations_bf16(61, 2, H)
    lg = synth.router_logits(61, 2, E)
    lg[1, 3] = np.nan
    gl.forward(x, lg, 2)
    st, bits = gl.layer.status()
    assert st == fe.FE_ERR_DEVICE_STATUS and bits & fe.FE_DEVICE_NAN_LOGIT
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0


def test_deterministic(torch_cuda):
    cfg, seed, x, lg = harness.workload_inputs("decode_e128_t64_zipf")
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    gl = harness.GpuLayer(E, H, I, 99, max_T=64, max_k=8)
    a = gl.forward(x, lg, k)[0]
    b = gl.forward(x, lg, k)[0]
    assert np.array_equal(a, b)
    # the fused single-token kernel too (its combine is ordered, no atomics)
    a1 = gl.forward(x[:1], lg[:1], k)[0]
    for _ in range(3):
        assert np.array_equal(gl.forward(x[:1], lg[:1], k)[0], a1)


@pytest.mark.parametrize("path", ["auto", "gemv", "tc"])
def test_graph_replay_with_changing_inputs(torch_cuda, path):
    torch = torch_cuda
    E, H, I, seed, k = 8, 256, 128, 0, 2
    T = 40 if path == "tc" else 4   # tc: GPU-wide routing and the tensor-core tiles inside the graph
    gl = harness.GpuLayer(E, H, I, seed, max_T=T, max_k=k, source="host", path=PATHS[path])
    osd = harness.OracleSide(E, H, I, seed)
    xs = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ls = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ys = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    x0 = synth.activations_bf16(70, T, H)
    l0 = synth.router_logits(70, T, E)
    xs.copy_(torch.from_numpy(x0.view(np.int16)).view(torch.bfloat16))
    ls.copy_(torch.from_numpy(l0))
    with torch.cuda.stream(s):
        gl.layer.forward(xs, ls, k, ys, stream=s)   # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        gl.layer.forward(xs, ls, k, ys, stream=s)
    for sd in (71, 72, 73):
        xn = synth.activations_bf16(sd, T, H)
        ln = synth.router_logits(sd, T, E)
        xs.copy_(torch.from_numpy(xn.view(np.int16)).view(torch.bfloat16))
        ls.copy_(torch.from_numpy(ln))
        g.replay()
        torch.cuda.synchronize()
        y = ys.view(torch.int16).cpu().numpy().view(np.uint16)
        y_ref, _ = osd.forward(xn, ln, k)
        harness.assert_output_close(y, y_ref, f"graph replay seed {sd}")
    del g


def test_forward_host_matches_device_forward(torch_cuda):
    E, H, I, seed, T, k = 8, 256, 128, 0, 5, 2
    gl = harness.GpuLayer(E, H, I, seed, max_T=T, max_k=k, source="host")
    x = synth.activations_bf16(80, T, H)
    lg = synth.router_logits(80, T, E)
    y_dev = gl.forward(x, lg, k)[0]
    y_host = np.empty((T, H), dtype=np.uint16)
    gl.layer.forward_host(x, lg, k, y_host)
    assert np.array_equal(y_dev, y_host)


def test_argument_errors(torch_cuda):
    import ctypes

    import fp4_expert_gemv_b200 as fe
    h = ctypes.c_void_p()
    assert fe.fe_moe_create(8, 256, 128, 16, ctypes.byref(h)) == fe.FE_ERR_UNSUPPORTED
    assert fe.fe_moe_create(8, 250, 128, 32, ctypes.byref(h)) == fe.FE_ERR_INVALID_ARG
    assert fe.fe_moe_create(0, 256, 128, 32, ctypes.byref(h)) == fe.FE_ERR_INVALID_ARG
    assert fe.fe_moe_create(8, 256, 128, 32, ctypes.byref(h)) == fe.FE_OK
    try:
        assert fe.fe_moe_forward(h, 16, 16, 1, 2, 32, None) == fe.FE_ERR_NOT_LOADED
        assert fe.fe_moe_reserve(h, 4, 9) == fe.FE_ERR_INVALID_ARG
        assert fe.fe_moe_reserve(h, 4, 2) == fe.FE_OK
        z = np.zeros(1 << 20, np.uint8)
        assert fe.fe_moe_load_packed(h, z.ctypes.data, z.ctypes.data, z.ctypes.data, z.ctypes.data, 0, None) == 0
        assert fe.fe_moe_forward(h, 16, 16, 5, 2, 32, None) == fe.FE_ERR_CAPACITY
        assert fe.fe_moe_forward(h, 16, 16, 1, 3, 32, None) == fe.FE_ERR_CAPACITY
        assert fe.fe_moe_forward(h, 16, 16, 1, 0, 32, None) == fe.FE_ERR_INVALID_ARG
        assert fe.fe_moe_forward(h, None, 16, 1, 2, 32, None) == fe.FE_ERR_INVALID_ARG
        assert fe.fe_moe_forward(h, 16, 16, 1, 2, 16, None) == fe.FE_ERR_INVALID_ARG   # y aliases x
        assert fe.fe_moe_forward(h, 16, 16, -1, 2, 32, None) == fe.FE_ERR_INVALID_ARG
        assert fe.fe_moe_set_path(h, fe.PATH_NVFP4 + 1) == fe.FE_ERR_INVALID_ARG
        assert fe.fe_moe_set_path(h, -1) == fe.FE_ERR_INVALID_ARG
        assert fe.fe_moe_set_path(h, fe.PATH_AUTO) == fe.FE_OK
        st, = [fe.fe_moe_get_status(h, None)]
        assert st == fe.FE_OK
    finally:
        fe.fe_moe_destroy(h)
    # the tensor-core tiles need I % 128 == 0: asking for them on I = 64 is refused
    # before anything is launched
    h2 = ctypes.c_void_p()
    assert fe.fe_moe_create(8, 256, 64, 32, ctypes.byref(h2)) == fe.FE_OK
    try:
        assert fe.fe_moe_reserve(h2, 4, 2) == fe.FE_OK
        z = np.zeros(1 << 20, np.uint8)
        assert fe.fe_moe_load_packed(h2, z.ctypes.data, z.ctypes.data, z.ctypes.data, z.ctypes.data, 0, None) == 0
        assert fe.fe_moe_set_path(h2, fe.PATH_TCGEN05) == fe.FE_OK
        assert fe.fe_moe_forward(h2, 16, 16, 1, 2, 32, None) == fe.FE_ERR_UNSUPPORTED
    finally:
        fe.fe_moe_destroy(h2)


def test_exchange_timeout_reports_and_recovers(torch_cuda):
    """The single-launch kernel's wait for the other CTAs runs out (it waits for
    an arrival that never comes, bounded at 20 us): the status reports
    FE_DEVICE_EXCHANGE_TIMEOUT and the next normal forward is oracle-correct."""
    import fp4_expert_gemv_b200 as fe
    cfg, seed, x, lg = harness.workload_inputs("decode_e128_t1")
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    gl = harness.GpuLayer(E, H, I, seed, max_T=1, max_k=k)
    osd = harness.OracleSide(E, H, I, seed)
    fe.check(fe.fe_moe_set_exchange_test(gl.layer.h, 1, 20000))
    gl.forward(x, lg, k)
    assert gl.layer.last_forward_info()[0] == fe.PATH_FUSED_DECODE
    st, bits = gl.layer.status()
    assert st == fe.FE_ERR_DEVICE_STATUS and bits & fe.FE_DEVICE_EXCHANGE_TIMEOUT
    fe.check(fe.fe_moe_set_exchange_test(gl.layer.h, 0, 1))
    run_and_check(gl, osd, x, lg, k, what="decode after a timed-out exchange")
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0
