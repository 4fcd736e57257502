"""Python binding of the fe_moe C ABI (include/fe_moe.h): argument marshalling only.

Every function named ``fe_moe_*`` here calls the C entry point of the same
name in ``libfe_moe.so``; all computation runs in the library's CUDA kernels.
The library must have been built (``python -m fp4_expert_gemv_b200.build``);
importing this package without it raises ImportError: there is no fallback.

``MoELayer`` is a convenience wrapper that takes torch tensors (device memory
and streams only) and checks status codes.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfe_moe.so")

FE_OK = 0
FE_ERR_INVALID_ARG = -1
FE_ERR_UNSUPPORTED = -2
FE_ERR_NOT_LOADED = -3
FE_ERR_CAPACITY = -4
FE_ERR_OOM = -5
FE_ERR_CUDA = -6
FE_ERR_DEVICE_STATUS = -7
FE_DEVICE_BAD_EXPERT = 0x1
FE_DEVICE_NAN_LOGIT = 0x2
FE_DEVICE_EXCHANGE_TIMEOUT = 0x4
FE_DEVICE_LOAD_TIMEOUT = 0x8
FE_DEVICE_TC_TIMEOUT = 0x10

PATH_AUTO, PATH_GEMV, PATH_TCGEN05, PATH_FUSED_DECODE, PATH_NVFP4 = 0, 1, 2, 3, 4

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python fp4_expert_gemv_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_i32 = ctypes.c_int
_i64 = ctypes.c_int64
_st = ctypes.c_int

_SIGS = {
    "fe_moe_create": (_st, [_i32, _i32, _i32, _i32, ctypes.POINTER(_P)]),
    "fe_moe_reserve": (_st, [_P, _i32, _i32]),
    "fe_moe_load_packed": (_st, [_P, _P, _P, _P, _P, _i32, _P]),
    "fe_moe_forward": (_st, [_P, _P, _P, _i32, _i32, _P, _P]),
    "fe_moe_forward_host": (_st, [_P, _P, _P, _i32, _i32, _P, _P]),
    "fe_moe_get_routing": (_st, [_P, _P, _P, _P, _P, _P]),
    "fe_moe_get_status": (_st, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "fe_moe_set_path": (_st, [_P, _i32]),
    "fe_moe_last_forward_info": (_st, [_P, ctypes.POINTER(_i32), ctypes.POINTER(_i32)]),
    "fe_moe_set_trace": (_st, [_P, _P]),
    "fe_moe_status_string": (ctypes.c_char_p, [_st]),
    "fe_moe_destroy": (None, [_P]),
    "fe_moe_pack_host": (_st, [_P, _i64, _i64, _i64, _P, _P]),
    "fe_moe_pack_device": (_st, [_P, _i64, _i64, _i64, _P, _P, _P]),
    "fe_moe_device_bytes": (ctypes.c_size_t, [_P]),
    "fe_moe_last_error": (ctypes.c_char_p, []),
    "fe_moe_forward_noalloc": (_st, [_i32, _i32, _i32, _P, _P, _P, _P, _P, _P, _i32, _i32, _P, _P]),
    "fe_moe_get_grouping": (_st, [_P, _P, _P, _P]),
    "fe_moe_noalloc_get_status": (_st, [ctypes.POINTER(ctypes.c_uint32)]),
    "fe_moe_noalloc_get_routing": (_st, [_i32, _i32, _i32, _P, _P, _P, _P, _P, _P, _P]),
    "fe_moe_stack_create": (_st, [ctypes.POINTER(_P), _i32, ctypes.POINTER(_P)]),
    "fe_moe_stack_forward": (_st, [_P, _P, _P, _i32, _i32, _P, _P]),
    "fe_moe_stack_forward_host": (_st, [_P, _P, _P, _i32, _i32, _P, _i32, _P]),
    "fe_moe_stack_destroy": (None, [_P]),
    "fe_moe_stack_set_prefetch": (_st, [_P, _i32]),
    "fe_moe_stack_last_launches": (_i32, [_P]),
    "fe_moe_set_exchange_test": (_st, [_P, _i32, ctypes.c_uint64]),
    "fe_moe_router": (_st, [_P, _P, _P, _i32, _i32, _P, _P, _P, _P]),
    "fe_moe_load_int2": (_st, [_P, _P, _P, _P, _P, _P, _i32, _P]),
    "fe_moe_pack_int2_host": (_st, [_P, _i64, _i64, _i64, _P, _P]),
    "fe_moe_pack_int2_device": (_st, [_P, _i64, _i64, _i64, _P, _P, _P]),
    "fe_moe_forward_router": (_st, [_P, _P, _P, _i32, _i32, _P, _P, _P]),
    "fe_moe_load_nvfp4": (_st, [_P, _P, _P, _P, _P, _i32, _P]),
    "fe_moe_nvfp4_quantize_device": (_st, [_P, _i64, _i64, _P, _P, _P, _P]),
}

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args
    globals()[_name] = _f


class FeMoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = fe_moe_status_string(status)
        detail = ""
        if status in (FE_ERR_CUDA, FE_ERR_OOM):
            detail = " [" + (fe_moe_last_error() or b"").decode(errors="replace") + "]"
        super().__init__(f"{what}: {msg.decode() if msg else status} ({status}){detail}")


def check(status: int, what: str = "fe_moe") -> None:
    if status != FE_OK:
        raise FeMoeError(status, what)


def _dptr(t) -> int:
    """Device address of a torch tensor (or an int address)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_ptr(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class MoELayer:
    """One fe_moe handle: create + reserve, load packed weights, forward."""

    def __init__(self, E: int, H: int, I: int, max_T: int, max_top_k: int, group: int = 32):
        h = _P()
        check(fe_moe_create(E, H, I, group, ctypes.byref(h)), "fe_moe_create")
        self.h = h
        self.E, self.H, self.I = E, H, I
        self.max_T, self.max_top_k = max_T, max_top_k
        try:
            check(fe_moe_reserve(self.h, max_T, max_top_k), "fe_moe_reserve")
        except Exception:
            fe_moe_destroy(self.h)
            self.h = None
            raise

    def load_packed(self, gu_codes, gu_scales, dn_codes, dn_scales, stream=None):
        """Device torch tensors (uint8 codes, int16/uint16/bfloat16 scales) or host numpy arrays."""
        import numpy as np
        if isinstance(gu_codes, np.ndarray):
            arrs = [np.ascontiguousarray(a) for a in (gu_codes, gu_scales, dn_codes, dn_scales)]
            check(fe_moe_load_packed(self.h, *[a.ctypes.data for a in arrs], 0, _stream_ptr(stream)),
                  "fe_moe_load_packed")
            import torch
            torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
        else:
            for t in (gu_codes, gu_scales, dn_codes, dn_scales):
                assert t.is_cuda and t.is_contiguous()
            check(fe_moe_load_packed(self.h, _dptr(gu_codes), _dptr(gu_scales), _dptr(dn_codes), _dptr(dn_scales),
                                     1, _stream_ptr(stream)), "fe_moe_load_packed")

    def forward(self, x_bf16, logits, top_k: int, y_bf16=None, stream=None):
        import torch
        T = x_bf16.shape[0]
        if y_bf16 is None:
            y_bf16 = torch.empty((T, self.H), dtype=torch.bfloat16, device=x_bf16.device)
        check(fe_moe_forward(self.h, _dptr(x_bf16), _dptr(logits), T, top_k, _dptr(y_bf16), _stream_ptr(stream)),
              "fe_moe_forward")
        return y_bf16

    def load_int2(self, formats, gu_codes, gu_scales, dn_codes, dn_scales, stream=None):
        """INT2 weights for the experts e with formats[e] = 1 (host numpy arrays or device
        torch tensors, full size [E, ...]); synchronous."""
        import numpy as np
        fmt = np.ascontiguousarray(np.asarray(formats, dtype=np.uint8))
        assert fmt.shape == (self.E,)
        if isinstance(gu_codes, np.ndarray):
            arrs = [np.ascontiguousarray(a) for a in (gu_codes, gu_scales, dn_codes, dn_scales)]
            check(fe_moe_load_int2(self.h, fmt.ctypes.data, *[a.ctypes.data for a in arrs], 0, _stream_ptr(stream)),
                  "fe_moe_load_int2")
        else:
            check(fe_moe_load_int2(self.h, fmt.ctypes.data, _dptr(gu_codes), _dptr(gu_scales), _dptr(dn_codes),
                                   _dptr(dn_scales), 1, _stream_ptr(stream)), "fe_moe_load_int2")

    def load_nvfp4(self, gu_codes, gu_scales, dn_codes, dn_scales, stream=None):
        """The block-scaled FP4 re-encoding of the packed weights (the arrays of load_packed:
        host numpy arrays or device torch tensors); then set_path(PATH_NVFP4) runs the variant."""
        import numpy as np
        if isinstance(gu_codes, np.ndarray):
            arrs = [np.ascontiguousarray(a) for a in (gu_codes, gu_scales, dn_codes, dn_scales)]
            check(fe_moe_load_nvfp4(self.h, *[a.ctypes.data for a in arrs], 0, _stream_ptr(stream)),
                  "fe_moe_load_nvfp4")
            import torch
            torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
        else:
            for t in (gu_codes, gu_scales, dn_codes, dn_scales):
                assert t.is_cuda and t.is_contiguous()
            check(fe_moe_load_nvfp4(self.h, _dptr(gu_codes), _dptr(gu_scales), _dptr(dn_codes), _dptr(dn_scales),
                                    1, _stream_ptr(stream)), "fe_moe_load_nvfp4")

    def router(self, x_bf16, w_router_bf16, top_k: int, logits=None, idx=None, w=None, stream=None):
        """The router GEMM fused with the top-k: (logits [T, E] f32, idx [T, k] i32, w [T, k] f32)."""
        import torch
        T = x_bf16.shape[0]
        dev = x_bf16.device
        if logits is None:
            logits = torch.empty((T, self.E), dtype=torch.float32, device=dev)
        if idx is None:
            idx = torch.empty((T, top_k), dtype=torch.int32, device=dev)
        if w is None:
            w = torch.empty((T, top_k), dtype=torch.float32, device=dev)
        check(fe_moe_router(self.h, _dptr(x_bf16), _dptr(w_router_bf16), T, top_k, _dptr(logits), _dptr(idx),
                            _dptr(w), _stream_ptr(stream)), "fe_moe_router")
        return logits, idx, w

    def forward_router(self, x_bf16, w_router_bf16, top_k: int, y_bf16=None, logits=None, stream=None):
        """The layer from x alone (router GEMM, top-k, layer): (y [T, H] bf16, logits [T, E] f32)."""
        import torch
        T = x_bf16.shape[0]
        if y_bf16 is None:
            y_bf16 = torch.empty((T, self.H), dtype=torch.bfloat16, device=x_bf16.device)
        if logits is None:
            logits = torch.empty((T, self.E), dtype=torch.float32, device=x_bf16.device)
        check(fe_moe_forward_router(self.h, _dptr(x_bf16), _dptr(w_router_bf16), T, top_k, _dptr(y_bf16),
                                    _dptr(logits), _stream_ptr(stream)), "fe_moe_forward_router")
        return y_bf16, logits

    def forward_host(self, x_bf16_host, logits_host, top_k: int, y_bf16_host, stream=None):
        """Host (ideally pinned) numpy/torch CPU buffers in and out; synchronous."""
        def hp(a):
            return a.ctypes.data if hasattr(a, "ctypes") else a.data_ptr()
        T = x_bf16_host.shape[0]
        check(fe_moe_forward_host(self.h, hp(x_bf16_host), hp(logits_host), T, top_k, hp(y_bf16_host),
                                  _stream_ptr(stream)), "fe_moe_forward_host")
        return y_bf16_host

    def routing(self, T: int, top_k: int, stream=None):
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        idx = torch.empty((T, top_k), dtype=torch.int32, device=dev)
        w = torch.empty((T, top_k), dtype=torch.float32, device=dev)
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=dev)
        sp = torch.empty(T * top_k, dtype=torch.int32, device=dev)
        check(fe_moe_get_routing(self.h, _dptr(idx), _dptr(w), _dptr(offsets), _dptr(sp), _stream_ptr(stream)),
              "fe_moe_get_routing")
        return idx, w, offsets, sp

    def grouping(self, T: int, top_k: int, stream=None):
        """(counts int32 [E], pair_row int32 [T*top_k]) of the last forward, as device tensors."""
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        counts = torch.empty(self.E, dtype=torch.int32, device=dev)
        pair_row = torch.empty(T * top_k, dtype=torch.int32, device=dev)
        check(fe_moe_get_grouping(self.h, _dptr(counts), _dptr(pair_row), _stream_ptr(stream)), "fe_moe_get_grouping")
        return counts, pair_row

    def status(self):
        bits = ctypes.c_uint32(0)
        st = fe_moe_get_status(self.h, ctypes.byref(bits))
        return st, bits.value

    def set_path(self, path: int):
        check(fe_moe_set_path(self.h, path), "fe_moe_set_path")

    def last_forward_info(self):
        path, kernels = _i32(0), _i32(0)
        check(fe_moe_last_forward_info(self.h, ctypes.byref(path), ctypes.byref(kernels)), "fe_moe_last_forward_info")
        return path.value, kernels.value

    def device_bytes(self) -> int:
        return fe_moe_device_bytes(self.h)

    def close(self):
        if getattr(self, "h", None):
            fe_moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Stack:
    """fe_moe_stack over MoELayer objects (kept alive here): n layers back to back on one stream."""

    def __init__(self, layers):
        self.layers = list(layers)
        arr = (_P * len(self.layers))(*[m.h for m in self.layers])
        h = _P()
        check(fe_moe_stack_create(arr, len(self.layers), ctypes.byref(h)), "fe_moe_stack_create")
        self.h = h
        self.n = len(self.layers)
        self.E, self.H = self.layers[0].E, self.layers[0].H

    def forward(self, x_bf16, logits, top_k: int, y_bf16, stream=None):
        """x device bf16 [n, T, H] (layer l reads x[l]), logits device float32 [n, T, E], y device bf16
        [n, T, H] (layer l writes y[l]); pass y = a view of x shifted by one layer to chain them."""
        T = logits.shape[1]
        check(fe_moe_stack_forward(self.h, _dptr(x_bf16), _dptr(logits), T, top_k, _dptr(y_bf16),
                                   _stream_ptr(stream)), "fe_moe_stack_forward")
        return y_bf16

    def forward_host(self, x_bf16_host, logits_host, top_k: int, y_bf16_host, chained=False, stream=None):
        """Host buffers (numpy or CPU torch, ideally pinned), bf16 as int16/uint16 bits; logits [n, T, E].
        chained=False: x, y [n, T, H]; chained=True: x [T, H] into layer 0, y [T, H] out of the last."""
        def hp(a):
            return a.ctypes.data if hasattr(a, "ctypes") else a.data_ptr()
        T = logits_host.shape[1]
        check(fe_moe_stack_forward_host(self.h, hp(x_bf16_host), hp(logits_host), T, top_k, hp(y_bf16_host),
                                        1 if chained else 0, _stream_ptr(stream)), "fe_moe_stack_forward_host")
        return y_bf16_host

    def set_prefetch(self, on: bool):
        """Cross-layer streaming (one persistent launch at T=1) on or off."""
        check(fe_moe_stack_set_prefetch(self.h, 1 if on else 0), "fe_moe_stack_set_prefetch")

    def last_launches(self) -> int:
        return fe_moe_stack_last_launches(self.h)

    def close(self):
        if getattr(self, "h", None):
            fe_moe_stack_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def noalloc_status():
    """(status, bits) of the last fe_moe_forward_noalloc call on the current device."""
    bits = ctypes.c_uint32(0)
    st = fe_moe_noalloc_get_status(ctypes.byref(bits))
    return st, bits.value


def pack_host(W):
    """numpy float32 [E, K, N] -> (codes uint8 [E, K/2, N], scales uint16 [E, K/32, N]) via fe_moe_pack_host."""
    import numpy as np
    W = np.ascontiguousarray(W, dtype=np.float32)
    E, K, N = W.shape
    codes = np.empty((E, K // 2, N), dtype=np.uint8)
    scales = np.empty((E, K // 32, N), dtype=np.uint16)
    check(fe_moe_pack_host(W.ctypes.data, E, K, N, codes.ctypes.data, scales.ctypes.data), "fe_moe_pack_host")
    return codes, scales


def pack_int2_host(W):
    """numpy float32 [E, K, N] -> (INT2 codes uint8 [E, K/4, N], scales uint16 [E, K/32, N])."""
    import numpy as np
    W = np.ascontiguousarray(W, dtype=np.float32)
    E, K, N = W.shape
    codes = np.empty((E, K // 4, N), dtype=np.uint8)
    scales = np.empty((E, K // 32, N), dtype=np.uint16)
    check(fe_moe_pack_int2_host(W.ctypes.data, E, K, N, codes.ctypes.data, scales.ctypes.data),
          "fe_moe_pack_int2_host")
    return codes, scales


def pack_int2_device(W, codes=None, scales=None, stream=None):
    """torch float32 CUDA [E, K, N] -> (INT2 codes uint8 [E, K/4, N], scales int16 bf16-bits)."""
    import torch
    E, K, N = W.shape
    if codes is None:
        codes = torch.empty((E, K // 4, N), dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty((E, K // 32, N), dtype=torch.int16, device=W.device)
    check(fe_moe_pack_int2_device(_dptr(W), E, K, N, _dptr(codes), _dptr(scales), _stream_ptr(stream)),
          "fe_moe_pack_int2_device")
    return codes, scales


def nvfp4_quantize_device(V, stream=None):
    """torch float32 CUDA [R, K] -> NVFP4 (codes uint8 [R, K/2], E4M3 scale factors uint8 [R, K/16],
    row scales float32 [R])."""
    import torch
    R, K = V.shape
    assert V.is_cuda and V.is_contiguous() and V.dtype == torch.float32
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device=V.device)
    sf = torch.empty((R, K // 16), dtype=torch.uint8, device=V.device)
    g = torch.empty((R,), dtype=torch.float32, device=V.device)
    check(fe_moe_nvfp4_quantize_device(_dptr(V), R, K, _dptr(codes), _dptr(sf), _dptr(g), _stream_ptr(stream)),
          "fe_moe_nvfp4_quantize_device")
    return codes, sf, g


def pack_device(W, codes=None, scales=None, stream=None):
    """torch float32 CUDA [E, K, N] -> (codes uint8, scales int16 bf16-bits) via fe_moe_pack_device."""
    import torch
    E, K, N = W.shape
    if codes is None:
        codes = torch.empty((E, K // 2, N), dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty((E, K // 32, N), dtype=torch.int16, device=W.device)
    check(fe_moe_pack_device(_dptr(W), E, K, N, _dptr(codes), _dptr(scales), _stream_ptr(stream)),
          "fe_moe_pack_device")
    return codes, scales
