"""Host logic of bench.py (no GPU): the roofline's byte counts, the hash-gated
ncu traffic record, and the count of distinct routed experts."""
import json

import numpy as np

import bench
import oracle
import synth


def test_algorithmic_bytes_match_the_stated_figures():
    # per expert: gate_up codes + scales + down codes + scales (H 2048, I 768 and I 512)
    assert bench.bytes_per_expert(2048, 768) == 2_654_208
    assert bench.bytes_per_expert(2048, 512) == 1_769_472
    # the decode layer at one token: 8 experts, x, logits, y
    assert bench.algorithmic_bytes_per_layer(128, 2048, 768, 1, 8) == 21_242_368
    # INT2: two bits per code, the same bf16 scales
    H, I = 2048, 768
    assert bench.int2_bytes_per_expert(H, I) == H * 2 * I // 4 + (H // 32) * 2 * I * 2 + I * H // 4 + (I // 32) * H * 2


def test_distinct_routed_matches_the_oracle_routing():
    lg = synth.router_logits(17, 64, 128, zipf_s=1.1)
    idx, _ = oracle.default().route(lg, 8)
    assert bench.distinct_routed(lg, 8) == len(np.unique(idx))


def test_traffic_is_reported_only_while_the_sources_match(tmp_path, monkeypatch):
    files = ["stack_decode.cuh", "common.cuh"]
    good = bench.source_hash(files)
    rec = {"entries": [{"workload": "decode_e128_t1", "kernel": "stack_decode_kernel", "sources": files,
                        "sources_sha256_16": good, "dram_bytes_per_layer": 1000.0}]}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.ncu_traffic("decode_e128_t1", 48) == (48000.0, "stack_decode_kernel")
    assert bench.ncu_traffic("prefill_e128_t4096", 1) == (None, None)
    rec["entries"][0]["sources_sha256_16"] = "0" * 16   # the kernel changed since the capture
    path.write_text(json.dumps(rec))
    assert bench.ncu_traffic("decode_e128_t1", 48) == (None, "stack_decode_kernel")



def test_kernel_label_follows_the_launch_count():
    assert "stack_decode_kernel" in bench.kernel_label(3, 1, 1)
    assert "per token" in bench.kernel_label(3, 4, 4)
    assert "decode_kernel" in bench.kernel_label(3, 48, 1) and "stack" not in bench.kernel_label(3, 48, 1)
    assert "sg_kernel" in bench.kernel_label(1, 336, 64)


def test_nvfp4_roofline_arithmetic():
    """The block-scaled FP4 record: 309.24 GFLOP per prefill layer, the FP4 peak as 4 x the
    measured sustained bf16 rate."""
    import bench
    peaks = {"bf16_tflops_sustained": 1400.0}
    r = bench.nvfp4_roofline(1000.0, 4096, 8, 2048, 768, peaks, "measured")
    flops = 2.0 * 4096 * 8 * 3 * 2048 * 768
    assert abs(flops - 309.237645312e9) < 1.0
    assert abs(r["achieved"] - flops / 1e-3 / 1e12) < 1e-9
    assert r["peak"] == 5600.0 and abs(r["frac"] - r["achieved"] / 5600.0) < 1e-12
    assert abs(r["frac_of_nominal_fp4_9pflops"] - r["achieved"] / 9000.0) < 1e-12
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
