"""Seeded synthetic inputs for the packed FP4 MoE layer (host side, numpy).

This module is the one piece shared by the CPU oracle's tests and the CUDA
path's tests and benchmark. It holds no arithmetic of the layer itself (no
quantiser, no routing, no matmul): it only turns (seed, tensor id, flat index)
into numbers.

Generator definition (counter based, so any element can be drawn on its own
and the device copy in ``synth.cu`` reproduces every value bit for bit):

* ``mix64`` is the SplitMix64 output function (Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014): xor-shift 30,
  multiply 0xBF58476D1CE4E5B9, xor-shift 27, multiply 0x94D049BB133111EB,
  xor-shift 31, all modulo 2**64.
* stream base ``b = mix64(seed * 256 + tensor_id)``.
* draw ``j`` (0, 1, 2) of element ``i`` is ``mix64(b + (3 i + j + 1) * G)``
  with ``G = 0x9E3779B97F4A7C15`` (the SplitMix64 increment).
* one standard-normal variate per element is the classic twelve-uniform
  (Irwin-Hall) approximation: the twelve 16-bit fields of the three draws are
  summed to ``S`` and ``z = (S - 393210) / 65536``, which has mean 0 and
  variance 1 - 2**-32 and is exact in float32 (|S - 393210| < 2**19).

Tensor ids: 0 = W_gate [E,H,I], 1 = W_up [E,H,I], 2 = W_down [E,I,H],
3 = x [T,H], 4 = router logits [T,E].

Derived values (each a single IEEE operation, identical on CPU and GPU):
weights ``w = float32(z) * float32(0.02)``; activations ``x = bf16_rne(z)``;
logits ``z`` in float32, plus an optional Zipf bias
``float32(z) + float32(-s * ln(e + 1))`` for the skewed-load workload.
"""
from __future__ import annotations

import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
S_CENTER = 393210          # 12 * (2**16 - 1) / 2
WEIGHT_STD = np.float32(0.02)

TID_GATE, TID_UP, TID_DOWN, TID_X, TID_LOGITS = 0, 1, 2, 3, 4
TID_ROUTER = 5

_CHUNK = 1 << 22


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wraps modulo 2**64)."""
    z = np.asarray(z, dtype=np.uint64)
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_base(seed: int, tid: int) -> np.uint64:
    if not (0 <= seed < (1 << 55)) or not (0 <= tid < 256):
        raise ValueError("seed must be in [0, 2**55) and tensor id in [0, 256)")
    return mix64(np.array([seed * 256 + tid], dtype=np.uint64))[0]


def normal_f32(seed: int, tid: int, idx: np.ndarray) -> np.ndarray:
    """Approximate N(0,1) float32 for each flat index in ``idx`` (any shape)."""
    idx = np.asarray(idx, dtype=np.uint64)
    flat = idx.reshape(-1)
    out = np.empty(flat.shape, dtype=np.float32)
    base = stream_base(seed, tid)
    mask = np.uint64(0xFFFF)
    with np.errstate(over="ignore"):
        for s in range(0, flat.size, _CHUNK):
            i3 = flat[s:s + _CHUNK] * np.uint64(3)
            acc = np.zeros(i3.shape, dtype=np.int64)
            for j in range(3):
                d = mix64(base + (i3 + np.uint64(j + 1)) * GAMMA)
                for q in range(4):
                    acc += ((d >> np.uint64(16 * q)) & mask).astype(np.int64)
            out[s:s + _CHUNK] = (acc - S_CENTER).astype(np.float32) / np.float32(65536.0)
    return out.reshape(idx.shape)


def bf16_bits_rne(v: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _experts(E: int, experts) -> np.ndarray:
    if experts is None:
        return np.arange(E, dtype=np.int64)
    ex = np.asarray(experts, dtype=np.int64).reshape(-1)
    if ex.size and (ex.min() < 0 or ex.max() >= E):
        raise ValueError("expert id out of range")
    return ex


def _weights_gate_up_np(seed: int, E: int, H: int, I: int, experts=None) -> np.ndarray:
    """The numpy definition of weights_gate_up (see there)."""
    ex = _experts(E, experts)
    out = np.empty((ex.size, H, 2 * I), dtype=np.float32)
    kn = (np.arange(H, dtype=np.uint64)[:, None] * np.uint64(I)
          + np.arange(I, dtype=np.uint64)[None, :])
    for a, e in enumerate(ex):
        flat = np.uint64(int(e) * H * I) + kn
        out[a, :, :I] = normal_f32(seed, TID_GATE, flat) * WEIGHT_STD
        out[a, :, I:] = normal_f32(seed, TID_UP, flat) * WEIGHT_STD
    return out


def _weights_down_np(seed: int, E: int, I: int, H: int, experts=None) -> np.ndarray:
    """The numpy definition of weights_down (see there)."""
    ex = _experts(E, experts)
    out = np.empty((ex.size, I, H), dtype=np.float32)
    kn = (np.arange(I, dtype=np.uint64)[:, None] * np.uint64(H)
          + np.arange(H, dtype=np.uint64)[None, :])
    for a, e in enumerate(ex):
        flat = np.uint64(int(e) * I * H) + kn
        out[a] = normal_f32(seed, TID_DOWN, flat) * WEIGHT_STD
    return out


def weights_gate_up(seed: int, E: int, H: int, I: int, experts=None) -> np.ndarray:
    """Unquantised fused gate_up weights, float32 [n_experts, H, 2I].

    Columns [0, I) are W_gate[e] (tensor 0), columns [I, 2I) are W_up[e]
    (tensor 1); element (e, k, n) of either has flat index (e*H + k)*I + n.
    Drawn by the host C copy of the generator when it is built (identical
    values, pinned against the numpy definition), else by numpy.
    """
    ex = _experts(E, experts)
    lib = _host_lib()
    if lib is None:
        return _weights_gate_up_np(seed, E, H, I, experts)
    out = np.empty((ex.size, H, 2 * I), dtype=np.float32)
    exa = np.ascontiguousarray(ex, dtype=np.int64)
    lib.synth_host_gate_up(out.ctypes.data, seed, H, I, exa.ctypes.data, ex.size)
    return out


def weights_down(seed: int, E: int, I: int, H: int, experts=None) -> np.ndarray:
    """Unquantised down weights, float32 [n_experts, I, H]; flat index (e*I + k)*H + n."""
    ex = _experts(E, experts)
    lib = _host_lib()
    if lib is None:
        return _weights_down_np(seed, E, I, H, experts)
    out = np.empty((ex.size, I, H), dtype=np.float32)
    exa = np.ascontiguousarray(ex, dtype=np.int64)
    lib.synth_host_down(out.ctypes.data, seed, I, H, exa.ctypes.data, ex.size)
    return out


def activations_bf16(seed: int, T: int, H: int) -> np.ndarray:
    """x as bfloat16 bit patterns, uint16 [T, H]."""
    z = normal_range_f32(seed, TID_X, 0, T * H).reshape(T, H)
    return bf16_bits_rne(z)


def router_logits(seed: int, T: int, E: int, zipf_s: float | None = None) -> np.ndarray:
    """Router logits float32 [T, E]; optional Zipf(s) per-expert bias -s*ln(e+1)."""
    z = normal_range_f32(seed, TID_LOGITS, 0, T * E).reshape(T, E)
    if zipf_s is not None:
        bias = np.array([-zipf_s * math.log(e + 1) for e in range(E)], dtype=np.float64)
        z = (z + bias.astype(np.float32)[None, :]).astype(np.float32)
    return np.ascontiguousarray(z, dtype=np.float32)


def router_weights_bf16(seed: int, E: int, H: int) -> np.ndarray:
    """Router rows W_r as bfloat16 bit patterns, uint16 [E, H]: N(0, 1) / sqrt(H), so that
    with N(0, 1) activations the logits are about N(0, 1)."""
    z = normal_range_f32(seed, TID_ROUTER, 0, E * H).reshape(E, H)
    return bf16_bits_rne((z * np.float32(1.0 / math.sqrt(H))).astype(np.float32))


# Workload recipes: shapes, seeds and value distributions of the five layer
# configurations (tiny check layer, 30B-A3B-like decode layer at T=1, the same
# layer at T=64 with Zipf-skewed routing, a 512-expert layer at T=1/4, and a
# T=4096 prefill layer). Seeds 6 and 7 and the stack seeds 1000+l are this
# project's choice.
WORKLOADS = {
    "tiny": dict(E=8, H=256, I=128, top_k=2, T=4, seeds=(0,), zipf=None),
    "decode_e128_t1": dict(E=128, H=2048, I=768, top_k=8, T=1, seeds=(1, 2, 3), zipf=None),
    "decode_e128_t64_zipf": dict(E=128, H=2048, I=768, top_k=8, T=64, seeds=(6,), zipf=1.1),
    "decode_e512_t1": dict(E=512, H=2048, I=512, top_k=10, T=1, seeds=(4, 5), zipf=None),
    "decode_e512_t4": dict(E=512, H=2048, I=512, top_k=10, T=4, seeds=(4, 5), zipf=None),
    "prefill_e128_t4096": dict(E=128, H=2048, I=768, top_k=8, T=4096, seeds=(7,), zipf=None),
}
STACK_LAYERS = 48
STACK_SEED0 = 1000


# -- host C copy of the generator (synth_host.c, built into libfe_synth_host.so) ----

_HOST_SRC = None
_HOST_LIB = None
_HOST_TRIED = False


def build_host(force: bool = False) -> str:
    """Compile synth_host.c with gcc (OpenMP, no FMA contraction, no fast-math)."""
    import os
    import subprocess
    here = os.path.dirname(os.path.abspath(__file__))
    src = os.path.join(here, "synth_host.c")
    out = os.path.join(here, "libfe_synth_host.so")
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, src])
        os.replace(tmp, out)
    return out


def _host_lib():
    """The host C generator, built on first use; None if it cannot be built."""
    global _HOST_LIB, _HOST_TRIED
    if _HOST_LIB is None and not _HOST_TRIED:
        _HOST_TRIED = True
        try:
            import ctypes
            lib = ctypes.CDLL(build_host())
            P, u64, i64 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64
            lib.synth_host_gate_up.argtypes = [P, u64, i64, i64, P, i64]
            lib.synth_host_down.argtypes = [P, u64, i64, i64, P, i64]
            lib.synth_host_normal.argtypes = [P, u64, u64, u64, i64]
            for f in (lib.synth_host_gate_up, lib.synth_host_down, lib.synth_host_normal):
                f.restype = ctypes.c_int
            _HOST_LIB = lib
        except (OSError, FileNotFoundError, Exception):   # no compiler: numpy definition only
            _HOST_LIB = None
    return _HOST_LIB


def normal_range_f32(seed: int, tid: int, first: int, count: int) -> np.ndarray:
    """normal_f32(seed, tid, first .. first + count - 1), by the C copy when built."""
    lib = _host_lib()
    if lib is None:
        return normal_f32(seed, tid, np.arange(first, first + count, dtype=np.uint64))
    out = np.empty(count, dtype=np.float32)
    lib.synth_host_normal(out.ctypes.data, seed, tid, first, count)
    return out


# -- device copy of the generator (synth.cu, built into libfe_synth.so) ----------

_DEVICE_LIB = None


def _device_lib():
    global _DEVICE_LIB
    if _DEVICE_LIB is None:
        import ctypes
        import os
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfe_synth.so")
        if not os.path.exists(path):
            raise ImportError(f"{path} is not built; run `python fp4_expert_gemv_b200/build.py`")
        lib = ctypes.CDLL(path)
        P, u64, i64 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64
        lib.fe_synth_gate_up.argtypes = [P, u64, i64, i64, i64, P]
        lib.fe_synth_down.argtypes = [P, u64, i64, i64, i64, P]
        lib.fe_synth_normal.argtypes = [P, u64, u64, i64, ctypes.c_float, P]
        for f in (lib.fe_synth_gate_up, lib.fe_synth_down, lib.fe_synth_normal):
            f.restype = ctypes.c_int
        _DEVICE_LIB = lib
    return _DEVICE_LIB


def device_gate_up(dst_ptr: int, seed: int, E: int, H: int, I: int, stream_ptr: int) -> None:
    """Fill float32 device memory [E, H, 2I] with weights_gate_up(seed, E, H, I)."""
    if _device_lib().fe_synth_gate_up(dst_ptr, seed, E, H, I, stream_ptr) != 0:
        raise RuntimeError("fe_synth_gate_up launch failed")


def device_down(dst_ptr: int, seed: int, E: int, I: int, H: int, stream_ptr: int) -> None:
    """Fill float32 device memory [E, I, H] with weights_down(seed, E, I, H)."""
    if _device_lib().fe_synth_down(dst_ptr, seed, E, I, H, stream_ptr) != 0:
        raise RuntimeError("fe_synth_down launch failed")


def device_normal(dst_ptr: int, seed: int, tid: int, count: int, scale: float, stream_ptr: int) -> None:
    """Fill float32 device memory [count] with normal_f32(seed, tid, i) * float32(scale)."""
    if _device_lib().fe_synth_normal(dst_ptr, seed, tid, count, scale, stream_ptr) != 0:
        raise RuntimeError("fe_synth_normal launch failed")
