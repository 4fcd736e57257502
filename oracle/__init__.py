"""ctypes front end for the C oracle in ``oracle.c``.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may use this module; the CUDA
library never does.  The two share no code.

Functions take and return numpy arrays.  bfloat16 values travel as their
uint16 bit patterns.  ``Oracle(path)`` wraps one build of oracle.c, so that a
test can also load a deliberately altered build and check that the pins
reject it; ``default()`` is the build of the committed source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False, src: str = SOURCE, out: str = _LIB) -> str:
    """Compile oracle.c with gcc (-O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


class ExpertWeights:
    """Per-expert packed buffers handed to the oracle (None = not materialised).

    gate_up codes uint8 [H/2, 2I] (gate columns, then up columns), scales
    bf16 bits [H/32, 2I]; down codes uint8 [I/2, H], scales [I/32, H].  An
    expert set with fmt=1 holds INT2 codes instead: [H/4, 2I] and [I/4, H].
    """

    def __init__(self, E: int, H: int, I: int):
        self.E, self.H, self.I = E, H, I
        self.fmt = np.zeros(E, dtype=np.uint8)
        self.gu_codes = [None] * E
        self.gu_scales = [None] * E
        self.dn_codes = [None] * E
        self.dn_scales = [None] * E

    def set(self, e: int, gu_codes, gu_scales, dn_codes, dn_scales, fmt: int = 0):
        H, I = self.H, self.I
        per = 4 if fmt else 2
        assert gu_codes.shape == (H // per, 2 * I) and gu_scales.shape == (H // 32, 2 * I)
        assert dn_codes.shape == (I // per, H) and dn_scales.shape == (I // 32, H)
        self.fmt[e] = 1 if fmt else 0
        self.gu_codes[e] = np.ascontiguousarray(gu_codes, dtype=np.uint8)
        self.gu_scales[e] = np.ascontiguousarray(gu_scales, dtype=np.uint16)
        self.dn_codes[e] = np.ascontiguousarray(dn_codes, dtype=np.uint8)
        self.dn_scales[e] = np.ascontiguousarray(dn_scales, dtype=np.uint16)

    def _ptrs(self, lst):
        arr = (ctypes.c_void_p * self.E)()
        for e, a in enumerate(lst):
            arr[e] = None if a is None else a.ctypes.data
        return arr


class Oracle:
    """One loaded build of oracle.c."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        lib.orc_e2m1_decode.argtypes = [i32]
        lib.orc_e2m1_decode.restype = ctypes.c_double
        lib.orc_e2m1_encode.argtypes = [ctypes.c_float]
        lib.orc_e2m1_encode.restype = i32
        lib.orc_f64_to_bf16_rne.argtypes = [ctypes.c_double]
        lib.orc_f64_to_bf16_rne.restype = ctypes.c_uint16
        lib.orc_quantize.argtypes = [P, i64, i64, i64, P, P]
        lib.orc_quantize.restype = i32
        lib.orc_dequant.argtypes = [P, P, i64, i64, i64]
        lib.orc_dequant.restype = ctypes.c_float
        lib.orc_route.argtypes = [P, i32, i32, i32, P, P]
        lib.orc_route.restype = i32
        lib.orc_group.argtypes = [P, i32, i32, i32, P, P, P, P]
        lib.orc_group.restype = i32
        lib.orc_int2_decode.argtypes = [i32]
        lib.orc_int2_decode.restype = ctypes.c_double
        lib.orc_int2_encode.argtypes = [ctypes.c_float]
        lib.orc_int2_encode.restype = i32
        lib.orc_quantize_int2.argtypes = [P, i64, i64, i64, P, P]
        lib.orc_quantize_int2.restype = i32
        lib.orc_dequant_int2.argtypes = [P, P, i64, i64, i64]
        lib.orc_dequant_int2.restype = ctypes.c_float
        lib.orc_moe_forward_fmt.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P]
        lib.orc_moe_forward_fmt.restype = i32
        lib.orc_router_logits.argtypes = [P, P, i32, i32, i32, P]
        lib.orc_router_logits.restype = i32
        lib.orc_moe_forward.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P]
        lib.orc_moe_forward.restype = i32
        lib.orc_e4m3_decode.argtypes = [i32]
        lib.orc_e4m3_decode.restype = ctypes.c_double
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode.restype = i32
        lib.orc_nvfp4_quantize.argtypes = [P, i64, i64, P, P, P]
        lib.orc_nvfp4_quantize.restype = i32
        lib.orc_moe_forward_nvfp4.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P]
        lib.orc_moe_forward_nvfp4.restype = i32
        self.lib = lib
        self.path = path

    def e2m1_decode(self, code: int) -> float:
        return self.lib.orc_e2m1_decode(int(code))

    def e2m1_encode(self, r: float) -> int:
        return self.lib.orc_e2m1_encode(float(r))

    def f64_to_bf16(self, v: float) -> int:
        return int(self.lib.orc_f64_to_bf16_rne(float(v)))

    def quantize(self, W: np.ndarray):
        """float32 W [E, K, N] -> (codes uint8 [E, K/2, N], scales uint16 [E, K/32, N])."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        E, K, N = W.shape
        codes = np.empty((E, K // 2, N), dtype=np.uint8)
        scales = np.empty((E, K // 32, N), dtype=np.uint16)
        _check(self.lib.orc_quantize(_ptr(W), E, K, N, _ptr(codes), _ptr(scales)), "quantize")
        return codes, scales

    def int2_decode(self, code: int) -> float:
        return self.lib.orc_int2_decode(int(code))

    def int2_encode(self, r: float) -> int:
        return self.lib.orc_int2_encode(float(r))

    def quantize_int2(self, W: np.ndarray):
        """float32 W [E, K, N] -> (INT2 codes uint8 [E, K/4, N], scales uint16 [E, K/32, N])."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        E, K, N = W.shape
        codes = np.empty((E, K // 4, N), dtype=np.uint8)
        scales = np.empty((E, K // 32, N), dtype=np.uint16)
        _check(self.lib.orc_quantize_int2(_ptr(W), E, K, N, _ptr(codes), _ptr(scales)), "quantize_int2")
        return codes, scales

    def dequant_int2(self, codes: np.ndarray, scales: np.ndarray, k: int, n: int) -> float:
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        return self.lib.orc_dequant_int2(_ptr(codes), _ptr(scales), codes.shape[-1], int(k), int(n))

    def dequant(self, codes: np.ndarray, scales: np.ndarray, k: int, n: int) -> float:
        """One dequantised weight of a single expert's [K/2, N] codes / [K/32, N] scales."""
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        return self.lib.orc_dequant(_ptr(codes), _ptr(scales), codes.shape[-1], int(k), int(n))

    def route(self, logits: np.ndarray, k: int):
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        T, E = logits.shape
        idx = np.empty((T, k), dtype=np.int32)
        w = np.empty((T, k), dtype=np.float32)
        _check(self.lib.orc_route(_ptr(logits), T, E, k, _ptr(idx), _ptr(w)), "route")
        return idx, w

    def router_logits(self, x_bf16: np.ndarray, w_router_bf16: np.ndarray) -> np.ndarray:
        """The router GEMM: x [T, H] (bf16 bits) times W_r [E, H] (bf16 bits, one row per
        expert), transposed: float64 logits [T, E]."""
        x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        w = np.ascontiguousarray(w_router_bf16, dtype=np.uint16)
        T, H = x_bf16.shape
        E = w.shape[0]
        assert w.shape == (E, H)
        out = np.empty((T, E), dtype=np.float64)
        _check(self.lib.orc_router_logits(_ptr(x_bf16), _ptr(w), T, H, E, _ptr(out)), "router_logits")
        return out

    def group(self, idx: np.ndarray, E: int):
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        T, k = idx.shape
        counts = np.empty(E, dtype=np.int32)
        offsets = np.empty(E + 1, dtype=np.int32)
        sp = np.empty(T * k, dtype=np.int32)
        pr = np.empty(T * k, dtype=np.int32)
        _check(self.lib.orc_group(_ptr(idx), T, k, E, _ptr(counts), _ptr(offsets), _ptr(sp),
                                  _ptr(pr)), "group")
        return counts, offsets, sp, pr

    def moe_forward(self, weights: ExpertWeights, x_bf16: np.ndarray, logits: np.ndarray, k: int,
                    want_act: bool = False):
        """The layer: (y64 [T,H] float64, y_bf16 [T,H] uint16[, act64 [T*k, I]])."""
        E, H, I = weights.E, weights.H, weights.I
        x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        T = x_bf16.shape[0]
        assert x_bf16.shape == (T, H) and logits.shape == (T, E)
        y64 = np.zeros((T, H), dtype=np.float64)
        yb = np.zeros((T, H), dtype=np.uint16)
        act = np.zeros((T * k, I), dtype=np.float64) if want_act else None
        rc = self.lib.orc_moe_forward_fmt(E, H, I, T, k, _ptr(x_bf16), _ptr(logits), _ptr(weights.fmt),
                                      weights._ptrs(weights.gu_codes), weights._ptrs(weights.gu_scales),
                                      weights._ptrs(weights.dn_codes), weights._ptrs(weights.dn_scales),
                                      _ptr(y64), _ptr(yb), _ptr(act))
        _check(rc, "moe_forward")
        return (y64, yb, act) if want_act else (y64, yb)

    def e4m3_decode(self, byte: int) -> float:
        return self.lib.orc_e4m3_decode(int(byte))

    def e4m3_encode(self, t: float) -> int:
        return self.lib.orc_e4m3_encode(float(t))

    def nvfp4_quantize(self, V: np.ndarray):
        """NVFP4 encoding of the rows of float32 V [R, K]: (codes uint8 [R, K/2], E4M3 scale
        factors uint8 [R, K/16], row scales float32 [R])."""
        V = np.ascontiguousarray(V, dtype=np.float32)
        R, K = V.shape
        codes = np.empty((R, K // 2), dtype=np.uint8)
        sf = np.empty((R, K // 16), dtype=np.uint8)
        g = np.empty(R, dtype=np.float32)
        _check(self.lib.orc_nvfp4_quantize(_ptr(V), R, K, _ptr(codes), _ptr(sf), _ptr(g)), "nvfp4_quantize")
        return codes, sf, g

    def moe_forward_nvfp4(self, weights: ExpertWeights, x_bf16: np.ndarray, logits: np.ndarray, k: int,
                          want_act: bool = False):
        """The block-scaled FP4 (NVFP4) variant of the layer: (y64, y_bf16[, act64]), act64 the
        bf16-rounded act in pair order."""
        E, H, I = weights.E, weights.H, weights.I
        assert not weights.fmt.any(), "the NVFP4 variant re-encodes E2M1 experts"
        x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        T = x_bf16.shape[0]
        assert x_bf16.shape == (T, H) and logits.shape == (T, E)
        y64 = np.zeros((T, H), dtype=np.float64)
        yb = np.zeros((T, H), dtype=np.uint16)
        act = np.zeros((T * k, I), dtype=np.float64) if want_act else None
        rc = self.lib.orc_moe_forward_nvfp4(E, H, I, T, k, _ptr(x_bf16), _ptr(logits),
                                            weights._ptrs(weights.gu_codes), weights._ptrs(weights.gu_scales),
                                            weights._ptrs(weights.dn_codes), weights._ptrs(weights.dn_scales),
                                            _ptr(y64), _ptr(yb), _ptr(act))
        _check(rc, "moe_forward_nvfp4")
        return (y64, yb, act) if want_act else (y64, yb)

    def quantized_experts(self, E: int, Wgu: np.ndarray, Wdn: np.ndarray, experts, fmt=None) -> ExpertWeights:
        """Quantise dense float32 gate_up [n, H, 2I] and down [n, I, H] weights of the listed
        expert ids (row a belongs to experts[a]) with this oracle's quantisers: E2M1, or INT2
        for the experts e with fmt[e] = 1 (fmt: None or a length-E sequence)."""
        n, H, I2 = Wgu.shape
        I = I2 // 2
        experts = list(experts)
        assert len(experts) == n and Wdn.shape == (n, I, H)
        ew = ExpertWeights(E, H, I)
        for a, e in enumerate(experts):
            f = int(fmt[e]) if fmt is not None else 0
            q = self.quantize_int2 if f else self.quantize
            gc, gs = q(Wgu[a:a + 1])
            dc, ds = q(Wdn[a:a + 1])
            ew.set(e, gc[0], gs[0], dc[0], ds[0], fmt=f)
        return ew


_default = None


def default() -> Oracle:
    """The oracle built from oracle.c as committed."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default
