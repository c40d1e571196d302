"""Float64 CPU oracle for scaled-dot-product attention (test infrastructure).

TEST INFRASTRUCTURE ONLY: the product library never imports, links or runs
anything in this directory.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` call it.  It
shares no code with the CUDA path.

The arithmetic lives in ``sdpa_oracle.c`` (plain C, float64, sequential
loops); this module only compiles it with gcc, marshals numpy buffers and
splits the requested query rows over host threads (the rows are independent
by definition, so the split changes no arithmetic).

Definition: MLX issue #3585 "mx.fast.scaled_dot_product_attention produces
incorrect attention scores (MLX 0.31.2)", section "Reproduction" (softmax of
scale * q k^T along the key axis, times v); GQA grouping from MLX issue #3885
"Metal SDPA: no fused path for head_dim=512", section "Measured impact".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sdpa_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle_sdpa.so")

F32, F16, BF16 = 0, 1, 2
MASK_NONE, MASK_ADDITIVE, MASK_BOOL, MASK_CAUSAL, MASK_SLIDING = 0, 1, 2, 3, 4

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc if the shared object is missing or stale."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i64, p = ctypes.c_int64, ctypes.c_void_p
            lib.oracle_sdpa_rows.restype = ctypes.c_int
            lib.oracle_sdpa_rows.argtypes = [p, p, p, i64, i64, i64, i64, i64, i64, i64, p,
                                             ctypes.c_double, ctypes.c_int, p, p, i64, ctypes.c_int,
                                             p, i64, p, p]
            lib.oracle_version.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def sdpa_rows(q, k, v, *, B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, scale, dtype,
              mask_kind=MASK_NONE, mask=None, mask_strides=(0, 0, 0, 0), rows=None,
              threads=None, want_probs=False, window=0):
    """Attention for selected query rows, in float64.

    q, k, v, mask: 1-D numpy storage buffers (float32 for fp32, uint16 bit
    patterns for fp16 / bf16, uint8 for a boolean mask); ``strides`` holds the
    12 element strides (b, h, l, d) of q, k and v into those buffers.
    ``rows`` is an (n, 3) int64 array of (b, h, i); None means every row in
    (b, h, i) order.  ``window``: the key count of the sliding-window mask kind.  Returns (n, Dv) float64 (and (n, Lk) weights if asked).
    """
    lib = _load()
    if rows is None:
        bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(Lq), indexing="ij")
        rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    n = rows.shape[0]
    out = np.zeros((n, Dv), dtype=np.float64)
    probs = np.zeros((n, Lk), dtype=np.float64) if want_probs else None
    st = np.ascontiguousarray(strides, dtype=np.int64)
    mst = np.ascontiguousarray(mask_strides, dtype=np.int64)
    if threads is None:
        threads = os.cpu_count() or 1
    threads = max(1, min(threads, n)) if n else 1

    def run(lo, hi):
        o = out[lo:hi]
        pr = probs[lo:hi] if probs is not None else None
        rc = lib.oracle_sdpa_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Lq, Lk, Dqk, Dv,
                                  _ptr(st), float(scale), int(mask_kind), _ptr(mask), _ptr(mst),
                                  int(window), int(dtype), _ptr(rows[lo:hi]), hi - lo, _ptr(o), _ptr(pr))
        if rc != 0:
            raise ValueError("oracle rejected its arguments")

    if n:
        bounds = np.linspace(0, n, threads + 1).astype(int)
        if threads == 1:
            run(0, n)
        else:
            with ThreadPoolExecutor(threads) as ex:
                list(ex.map(lambda t: run(bounds[t], bounds[t + 1]), range(threads)))
    return (out, probs) if want_probs else out


def sdpa_full(q, k, v, *, B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, scale, dtype,
              mask_kind=MASK_NONE, mask=None, mask_strides=(0, 0, 0, 0), threads=None, window=0):
    """Every row; returns float64 [B, Hq, Lq, Dv]."""
    o = sdpa_rows(q, k, v, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, Dqk=Dqk, Dv=Dv, strides=strides,
                  scale=scale, dtype=dtype, mask_kind=mask_kind, mask=mask,
                  mask_strides=mask_strides, threads=threads, window=window)
    return o.reshape(B, Hq, Lq, Dv)
