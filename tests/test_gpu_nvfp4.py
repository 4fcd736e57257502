"""The block-scaled FP4 (NVFP4) variant of the layer (fe_moe_load_nvfp4, FE_PATH_NVFP4):
the device row encoder against the oracle's encoder bit for bit, and the variant layer
against the oracle's variant layer on the same seeded inputs, every token row at small
sizes and sampled rows of the full-size prefill workload.  The variant is an
approximation of the layer; its distance to the exact layer is printed and only
bounded loosely."""
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


def encoder_rows(rng, K):
    rows = [rng.standard_normal(K) * s for s in (0.02, 1.0, 30.0, 1e-5, 3e3)]
    rows.append(np.zeros(K))
    one = np.zeros(K)
    one[K // 3] = -2.5
    rows.append(one)
    rows.append(np.where(rng.random(K) < 0.2, rng.standard_normal(K), 0.0))
    rows.append(rng.standard_normal(K) * np.repeat(10.0 ** rng.uniform(-7, 3, K // 16), 16))
    r = rng.standard_normal(K) * 0.1
    r[0] = 1.0
    r[1:8] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) / 6.0   # E2M1 decision points
    rows.append(r)
    rows += list(rng.standard_normal((54, K)) * np.exp(rng.uniform(-4, 4, (54, 1))))
    return np.array(rows, dtype=np.float32)


@pytest.mark.parametrize("K", [16, 256, 2048])
def test_nvfp4_encoder_matches_oracle(torch_cuda, K):
    torch = torch_cuda
    import fp4_expert_gemv_b200 as fe
    V = encoder_rows(np.random.default_rng(K), K)
    codes, sf, g = fe.nvfp4_quantize_device(torch.from_numpy(V).cuda())
    torch.cuda.synchronize()
    c_ref, s_ref, g_ref = oracle.default().nvfp4_quantize(V)
    assert np.array_equal(g.cpu().numpy().view(np.uint32), g_ref.view(np.uint32))
    assert np.array_equal(sf.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def nvfp4_layer(E, H, I, seed, max_T, k, source):
    import torch

    import fp4_expert_gemv_b200 as fe
    gl = harness.GpuLayer(E, H, I, seed, max_T=max_T, max_k=k, source=source, keep_packed=True,
                          path=fe.PATH_NVFP4)
    gl.layer.load_nvfp4(*gl.packed)
    torch.cuda.synchronize()
    return gl


# E, H, I, top_k, T, weights source: a tiny layer (partial tiles), a layer whose hot
# experts take more than 256 rows (two tiles), the 30B-like layer at T = 64
CASES = [
    (8, 256, 256, 2, 64, "host"),
    (16, 512, 256, 4, 300, "host"),
    (128, 2048, 768, 8, 64, "device"),
]


@pytest.mark.parametrize("E,H,I,k,T,source", CASES)
def test_nvfp4_layer_matches_variant_oracle(torch_cuda, E, H, I, k, T, source):
    import fp4_expert_gemv_b200 as fe
    seed = 61
    gl = nvfp4_layer(E, H, I, seed, T, k, source)
    x = synth.activations_bf16(seed + T, T, H)
    lg = synth.router_logits(seed + T, T, E, zipf_s=1.1 if T >= 64 else 0.0)
    y, idx, w, off, sp = gl.forward(x, lg, k)
    assert gl.layer.last_forward_info()[0] == fe.PATH_NVFP4
    idx_ref, _ = oracle.default().route(lg, k)
    assert np.array_equal(idx, idx_ref)
    osd = harness.OracleSide(E, H, I, seed)
    ref_v, _ = osd.forward_nvfp4(x, lg, k)
    harness.assert_output_close(y, ref_v, f"NVFP4 variant E={E} T={T}")
    ref, _ = osd.forward(x, lg, k)
    max_rel, l2_rel = harness.output_errors(y, ref)
    print(f"NVFP4 variant vs exact layer E={E} H={H} I={I} T={T}: max-rel {max_rel:.3e} l2-rel {l2_rel:.3e}")
    assert l2_rel < 0.3
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0


def test_nvfp4_prefill_sampled(torch_cuda):
    """The full-size prefill workload (E=128, T=4096, top-8) on the variant, against the
    oracle's variant on sampled token rows that together reach many experts."""
    import fp4_expert_gemv_b200 as fe
    cfg, seed, x, lg = harness.workload_inputs("prefill_e128_t4096")
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    gl = nvfp4_layer(E, H, I, seed, T, k, "device")
    y, idx, w, off, sp = gl.forward(x, lg, k)
    assert gl.layer.last_forward_info()[0] == fe.PATH_NVFP4
    rows = np.unique(np.concatenate([[0, 1, T // 2, T - 1], np.random.default_rng(5).choice(T, 28, replace=False)]))
    osd = harness.OracleSide(E, H, I, seed)
    ref_v, _ = osd.forward_nvfp4(x[rows], lg[rows], k)
    harness.assert_output_close(y[rows], ref_v, "NVFP4 variant, prefill rows")
    ref, _ = osd.forward(x[rows], lg[rows], k)
    max_rel, l2_rel = harness.output_errors(y[rows], ref)
    print(f"NVFP4 variant vs exact layer, prefill rows: max-rel {max_rel:.3e} l2-rel {l2_rel:.3e}")
    assert l2_rel < 0.3
    st, bits = gl.layer.status()
    assert st == fe.FE_OK and bits == 0


def test_nvfp4_refusals(torch_cuda):
    import fp4_expert_gemv_b200 as fe
    # I % 256 != 0: the variant cannot be loaded
    gl = harness.GpuLayer(8, 256, 128, 3, max_T=8, max_k=2, source="host", keep_packed=True)
    with pytest.raises(fe.FeMoeError) as ei:
        gl.layer.load_nvfp4(*gl.packed)
    assert ei.value.status == fe.FE_ERR_UNSUPPORTED
    # forced without loading it: refused before anything runs
    gl.layer.set_path(fe.PATH_NVFP4)
    x = synth.activations_bf16(3, 4, 256)
    lg = synth.router_logits(3, 4, 8)
    with pytest.raises(fe.FeMoeError) as ei:
        gl.forward(x, lg, 2)
    assert ei.value.status == fe.FE_ERR_UNSUPPORTED
