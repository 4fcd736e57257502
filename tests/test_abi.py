"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, and its host packer reproduces the oracle's quantiser."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fe_moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?(fe_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ["fe_moe_create", "fe_moe_load_packed", "fe_moe_forward", "fe_moe_destroy",
                     "fe_moe_reserve", "fe_moe_get_routing", "fe_moe_get_status", "fe_moe_pack_host"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    import fp4_expert_gemv_b200 as fe
    lib = ctypes.CDLL(fe.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    # the binding wraps each of them under the same name
    for n in declared_functions():
        assert hasattr(fe, n), n


def test_status_strings():
    import fp4_expert_gemv_b200 as fe
    for code in range(0, -8, -1):
        assert fe.fe_moe_status_string(code)
    assert fe.fe_moe_status_string(-4) == b"T or top_k above the reserved workspace"


def test_pack_host_matches_oracle_quantiser():
    import fp4_expert_gemv_b200 as fe
    rng = np.random.default_rng(5)
    cases = [(rng.standard_normal((2, 64, 40)) * 0.02).astype(np.float32),
             (rng.standard_normal((1, 96, 8)) * 5).astype(np.float32)]
    W = np.zeros((2, 64, 16), np.float32)
    W[0, 0:8, 3] = [3.0, 0.125, 0.375, 0.625, 0.875, 1.25, 1.75, 2.5]   # exact midpoints
    W[1, 0:8, 4] = [-3.0, -0.125, -0.375, -0.625, -0.875, -1.25, -1.75, -2.5]
    W[1, 32:64, 9] = 1e-3
    cases.append(W)
    # every ratio the encoder can see, through a constant scale of 1 (group max 6)
    r = pins.encode_probe_values(rng)
    r = r[np.abs(r) <= 6.0]
    n = (r.size + 30) // 31
    V = np.zeros((1, 32, n), np.float32)
    V[0, 0, :] = 6.0
    V[0, 1:, :].reshape(-1)[: r.size] = r
    V[0, 1:, :] = np.pad(r, (0, 31 * n - r.size)).reshape(31, n)
    cases.append(V)
    orc = oracle.default()
    for W in cases:
        c, s = fe.pack_host(W)
        c_ref, s_ref = orc.quantize(W)
        assert np.array_equal(s, s_ref)
        assert np.array_equal(c, c_ref)


def test_pack_int2_host_matches_oracle_quantiser():
    import fp4_expert_gemv_b200 as fe
    rng = np.random.default_rng(6)
    cases = [(rng.standard_normal((2, 64, 40)) * 0.02).astype(np.float32),
             (rng.standard_normal((1, 96, 8)) * 5).astype(np.float32)]
    # exact midpoints between levels (r = -1, 0, 1 with the group max 1.5 -> scale 1)
    W = np.zeros((1, 32, 4), np.float32)
    W[0, 0, :] = 1.5
    W[0, 1:8, 0] = [-1.0, 0.0, 1.0, -0.5, 0.5, -1.5, 0.999]
    W[0, 1:8, 1] = [-1.0001, -0.9999, 1.0001, 0.9999, -0.0001, 0.0001, 2.0]
    cases.append(W)
    cases.append(np.zeros((1, 64, 3), np.float32))   # all-zero groups: scale 0, codes 2
    orc = oracle.default()
    for W in cases:
        c, s = fe.pack_int2_host(W)
        c_ref, s_ref = orc.quantize_int2(W)
        assert np.array_equal(s, s_ref)
        assert np.array_equal(c, c_ref)


def test_synth_device_library_is_built():
    path = os.path.join(ROOT, "synth", "libfe_synth.so")
    assert os.path.exists(path)
    lib = ctypes.CDLL(path)
    for n in ("fe_synth_gate_up", "fe_synth_down", "fe_synth_normal"):
        assert hasattr(lib, n)


def test_nvfp4_entry_points_refuse_bad_arguments_on_the_host():
    """The block-scaled FP4 entry points validate before touching the device (no GPU needed):
    null or misaligned pointers, K not a multiple of 16, negative rows, a null handle."""
    import fp4_expert_gemv_b200 as fe
    q = fe.fe_moe_nvfp4_quantize_device
    A = 1 << 20   # aligned fake addresses: never dereferenced, every call here is refused first
    assert q(None, 1, 16, A, A, A, None) == fe.FE_ERR_INVALID_ARG
    assert q(A, 1, 16, None, A, A, None) == fe.FE_ERR_INVALID_ARG
    assert q(A, 1, 15, A, A, A, None) == fe.FE_ERR_INVALID_ARG
    assert q(A, 1, 0, A, A, A, None) == fe.FE_ERR_INVALID_ARG
    assert q(A, -1, 16, A, A, A, None) == fe.FE_ERR_INVALID_ARG
    assert q(A + 8, 1, 16, A, A, A, None) == fe.FE_ERR_INVALID_ARG      # src not 16-byte aligned
    assert q(A, 1, 16, A + 4, A, A, None) == fe.FE_ERR_INVALID_ARG      # codes not 8-byte aligned
    assert q(A, 0, 16, A, A, A, None) == fe.FE_OK                        # nothing to do
    assert fe.fe_moe_load_nvfp4(None, A, A, A, A, 1, None) == fe.FE_ERR_INVALID_ARG
    assert fe.fe_moe_set_path(None, fe.PATH_NVFP4) == fe.FE_ERR_INVALID_ARG
