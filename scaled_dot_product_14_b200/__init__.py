"""B200-native fused scaled-dot-product attention forward (sm_100a).

Thin binding over the C ABI in ``include/sdpa.h`` (``libsdpa_b200.so``, built
in-tree by ``scaled_dot_product_14_b200.build``).  The functions named like the
C entry points only marshal arguments; every step of the attention runs in the
library's CUDA kernels.  There is no Python or CPU fallback: if the library is
missing, the first call raises.

``attention(q, k, v, ...)`` is a convenience wrapper for torch tensors given as
logical ``[B, H, L, D]`` views with any strides (pass ``x.transpose(1, 2)`` for
a ``[B, L, H, D]`` buffer); the strides go to the library unchanged.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdpa_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "sdpa.h")

# sdpa_dtype / sdpa_mask_kind / sdpa_path / sdpa_status (include/sdpa.h)
SDPA_F32, SDPA_F16, SDPA_BF16 = 0, 1, 2
SDPA_MASK_NONE, SDPA_MASK_ADDITIVE, SDPA_MASK_BOOL, SDPA_MASK_CAUSAL, SDPA_MASK_SLIDING = 0, 1, 2, 3, 4
SDPA_PATH_NONE, SDPA_PATH_PREFILL, SDPA_PATH_DECODE = 0, 1, 2
STATUS = {0: "SDPA_OK", 1: "SDPA_ERR_INVALID_ARG", 2: "SDPA_ERR_UNSUPPORTED_DIM", 3: "SDPA_ERR_UNSUPPORTED_STRIDE",
          4: "SDPA_ERR_MISALIGNED", 5: "SDPA_ERR_LAUNCH_CONFIG", 6: "SDPA_ERR_CUDA", 7: "SDPA_ERR_TIMEOUT",
          8: "SDPA_ERR_NO_MEMORY", 9: "SDPA_ERR_NULL_POINTER", 10: "SDPA_ERR_TOO_LARGE"}


class SdpaError(RuntimeError):
    def __init__(self, status: int, where: str = "sdpa_forward"):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}: {sdpa_error_string(status)}"
        if status == 6:
            msg += f" ({sdpa_last_cuda_error()})"
        super().__init__(msg)


class _Counters(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "calls", "prefill_calls", "decode_calls", "empty_calls", "rejected_calls", "prefill_tcgen05_launches",
        "prefill_ffma_launches", "decode_mma_launches", "decode_ffma_launches", "combine_launches",
        "prefill_tf32_launches")]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m scaled_dot_product_14_b200.build` (there is no fallback path)")
            L = ctypes.CDLL(LIB_PATH)
            i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
            P64 = ctypes.POINTER(ctypes.c_int64)
            L.sdpa_forward.restype = i32
            L.sdpa_forward.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, P64, ctypes.c_float, i32,
                                       vp, P64, i32, vp]
            L.sdpa_forward_noalloc.restype = i32
            L.sdpa_forward_noalloc.argtypes = list(L.sdpa_forward.argtypes)
            L.sdpa_forward_window.restype = i32
            L.sdpa_forward_window.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, P64,
                                              ctypes.c_float, i64, i32, vp]
            L.sdpa_supported.restype = i32
            L.sdpa_supported.argtypes = [i64, i64, i64, i64, i64, i64, i64, P64, i32, P64, i32,
                                         ctypes.POINTER(ctypes.c_int)]
            L.sdpa_error_string.restype = ctypes.c_char_p
            L.sdpa_error_string.argtypes = [i32]
            L.sdpa_last_cuda_error.restype = ctypes.c_char_p
            L.sdpa_get_counters.restype = None
            L.sdpa_get_counters.argtypes = [ctypes.POINTER(_Counters)]
            L.sdpa_reset_counters.restype = None
            L.sdpa_last_launch_count.restype = i32
            L.sdpa_check_device_error.restype = i32
            L.sdpa_check_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
            L.sdpa_shutdown.restype = i32
            L.sdpa_abi_version.restype = i32
            L.sdpa_profile_enable.restype = i32
            L.sdpa_profile_enable.argtypes = [i32]
            L.sdpa_profile_collect.restype = i32
            L.sdpa_profile_collect.argtypes = [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_double)]
            L.sdpa_debug_set.restype = i32
            L.sdpa_debug_set.argtypes = [i32, i64]
            L.sdpa_workspace_bytes.restype = i64
            L.sdpa_workspace_bytes.argtypes = []
            _lib = L
    return _lib


def _i64array(vals, n):
    if vals is None:
        return None
    vals = [int(x) for x in vals]
    if len(vals) != n:
        raise ValueError(f"expected {n} strides, got {len(vals)}")
    return (ctypes.c_int64 * n)(*vals)


# ------------------------------------------------------------------ C ABI, one to one
def sdpa_forward(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, scale, mask_kind, mask, mask_strides,
                 dtype, stream) -> int:
    """Calls the C entry point; pointers are ints (device addresses), strides sequences."""
    return lib().sdpa_forward(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, _i64array(strides, 16),
                              ctypes.c_float(scale), mask_kind, mask, _i64array(mask_strides, 4), dtype, stream)


def sdpa_forward_window(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, scale, window, dtype, stream) -> int:
    """Causal sliding-window attention over the `window` most recent keys."""
    return lib().sdpa_forward_window(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, _i64array(strides, 16),
                                     ctypes.c_float(scale), int(window), dtype, stream)


def sdpa_forward_noalloc(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, scale, mask_kind, mask,
                         mask_strides, dtype, stream) -> int:
    """The allocation-free decode entry point (same arguments as sdpa_forward)."""
    return lib().sdpa_forward_noalloc(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, _i64array(strides, 16),
                                      ctypes.c_float(scale), mask_kind, mask, _i64array(mask_strides, 4), dtype,
                                      stream)


def sdpa_supported(B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, mask_kind, mask_strides, dtype):
    """Returns (status, path)."""
    path = ctypes.c_int(0)
    st = lib().sdpa_supported(B, Hq, Hkv, Lq, Lk, Dqk, Dv, _i64array(strides, 16), mask_kind,
                              _i64array(mask_strides, 4), dtype, ctypes.byref(path))
    return st, path.value


def sdpa_error_string(status: int) -> str:
    return lib().sdpa_error_string(status).decode()


def sdpa_last_cuda_error() -> str:
    return lib().sdpa_last_cuda_error().decode()


def sdpa_get_counters() -> dict:
    c = _Counters()
    lib().sdpa_get_counters(ctypes.byref(c))
    return {n: getattr(c, n) for n, _ in _Counters._fields_}


def sdpa_reset_counters() -> None:
    lib().sdpa_reset_counters()


def sdpa_last_launch_count() -> int:
    return lib().sdpa_last_launch_count()


def sdpa_check_device_error(stream=None):
    code = ctypes.c_int(0)
    st = lib().sdpa_check_device_error(stream, ctypes.byref(code))
    return st, code.value


def sdpa_shutdown() -> int:
    return lib().sdpa_shutdown()


def sdpa_abi_version() -> int:
    return lib().sdpa_abi_version()


# sdpa_debug_knob (include/sdpa.h): test hooks for the failure paths
SDPA_DEBUG_WAIT_LIMIT_NS, SDPA_DEBUG_DECODE_BARRIER_EXTRA, SDPA_DEBUG_FAIL_ALLOCS = 0, 1, 2


def sdpa_debug_set(knob: int, value: int) -> int:
    return lib().sdpa_debug_set(knob, int(value))


def sdpa_workspace_bytes() -> int:
    return lib().sdpa_workspace_bytes()


KERNEL_FAMILIES = ("prefill_tcgen05", "prefill_ffma", "decode_mma", "decode_ffma", "combine", "zero_fill",
                   "prefill_tf32")


def sdpa_profile_enable(on: bool) -> int:
    return lib().sdpa_profile_enable(1 if on else 0)


def sdpa_profile_collect() -> dict:
    """{family: (launches, total_ms)} for the kernels timed since the last collect."""
    n = len(KERNEL_FAMILIES)
    launches = (ctypes.c_uint64 * n)()
    ms = (ctypes.c_double * n)()
    st = lib().sdpa_profile_collect(launches, ms)
    if st != 0:
        raise SdpaError(st, "sdpa_profile_collect")
    return {f: (launches[i], ms[i]) for i, f in enumerate(KERNEL_FAMILIES)}


# ------------------------------------------------------------------ torch convenience
def _dtype_code(t):
    import torch
    codes = {torch.float32: SDPA_F32, torch.float16: SDPA_F16, torch.bfloat16: SDPA_BF16}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def attention(q, k, v, *, scale=None, mask=None, causal=False, window=None, out=None, stream=None):
    """out = softmax(scale q k^T + mask) v for CUDA tensors given as logical [B, H, L, D] views.

    ``mask``: None; a bool tensor (True = attend) or a tensor of q's dtype
    (additive), 4-D and broadcastable to [B, Hq, Lq, Lk] through zero strides
    (``expand``).  ``causal=True`` uses bottom-right alignment; with ``window``
    it is limited to the ``window`` most recent keys (sliding window).
    Returns ``out`` ([B, Hq, Lq, Dv], contiguous unless given).
    """
    import torch
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D logical [B, H, L, D] views")
    B, Hq, Lq, Dqk = q.shape
    Hkv, Lk, Dv = k.shape[1], k.shape[2], v.shape[3]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, Hq, Lq, Dv), dtype=q.dtype, device=q.device)
    if scale is None:
        scale = float(Dqk) ** -0.5
    mk, mptr, mst = SDPA_MASK_NONE, None, None
    if causal:
        if mask is not None:
            raise ValueError("causal and an explicit mask are exclusive")
        mk = SDPA_MASK_CAUSAL
    elif mask is not None:
        if mask.dim() != 4:
            raise ValueError("mask must be 4-D (use expand for broadcasting)")
        mask = mask.expand(B, Hq, Lq, Lk)
        if mask.dtype == torch.bool:
            mk, mptr = SDPA_MASK_BOOL, mask.data_ptr()
        else:
            if mask.dtype != q.dtype:
                raise TypeError("additive mask must have q's dtype")
            mk, mptr = SDPA_MASK_ADDITIVE, mask.data_ptr()
        mst = list(mask.stride())
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    strides = list(q.stride()) + list(k.stride()) + list(v.stride()) + list(out.stride())
    if window is not None:
        if not causal:
            raise ValueError("a sliding window is causal: pass causal=True with window")
        st = sdpa_forward_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, Lq, Lk,
                                 Dqk, Dv, strides, float(scale), int(window), dt, stream)
        if st != 0:
            raise SdpaError(st, "sdpa_forward_window")
        return out
    st = sdpa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq, Hkv, Lq, Lk, Dqk, Dv,
                      strides, float(scale), mk, mptr, mst, dt, stream)
    if st != 0:
        raise SdpaError(st)
    return out
