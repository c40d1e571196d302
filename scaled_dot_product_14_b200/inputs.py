"""Seeded synthetic inputs for attention, shared by tests, smoke check and bench.

This module holds random-number generation, rounding to a storage dtype and
memory layout only.  It contains none of the attention arithmetic, so both the
float64 oracle and the CUDA path may be fed from it.

Recipe (stated once, used everywhere):
  * ``numpy.random.default_rng(seed)``; draws in the order Q, K, V, mask;
  * values ``standard_normal`` in float32, rounded to the run's dtype with
    round-to-nearest-even (bf16 by bit arithmetic, fp16 by numpy's cast);
  * additive decode mask ``[1,1,1,kL]``: U(-1, 0) with the last floor(0.1 kL)
    keys set to -inf; boolean mask ``[1,1,Lq,Lk]``: keep with probability
    ``p_keep`` (uint8, 1 = attend);
  * the deterministic MLX issue #3585 input: ``linspace(-0.5, 0.5, n,
    endpoint=False)`` in float32 reshaped to [B, L, H, D] (section "Minimal
    reproduction with deterministic inputs").
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F32, F16, BF16 = 0, 1, 2
DTYPE_NAMES = {F32: "f32", F16: "f16", BF16: "bf16"}
DTYPE_BY_NAME = {"f32": F32, "fp32": F32, "f16": F16, "fp16": F16, "bf16": BF16}
ELEM_SIZE = {F32: 4, F16: 2, BF16: 2}
MASK_NONE, MASK_ADDITIVE, MASK_BOOL, MASK_CAUSAL, MASK_SLIDING = 0, 1, 2, 3, 4


# ----------------------------------------------------------------------------- dtype storage
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    # finite and infinite values stay below 2^32 after the rounding increment
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_storage(x: np.ndarray, dtype: int) -> np.ndarray:
    """float32 values -> storage array (float32, or uint16 bit patterns for fp16/bf16)."""
    x = np.asarray(x, dtype=np.float32)
    if dtype == F32:
        return np.ascontiguousarray(x)
    if dtype == F16:
        return np.ascontiguousarray(x.astype(np.float16)).view(np.uint16)
    if dtype == BF16:
        return f32_to_bf16_bits(x)
    raise ValueError(dtype)


def storage_to_f32(s: np.ndarray, dtype: int) -> np.ndarray:
    """Exact widening of a storage array to float32 (for test-side comparisons)."""
    if dtype == F32:
        return np.asarray(s, dtype=np.float32)
    if dtype == F16:
        return np.asarray(s, dtype=np.uint16).view(np.float16).astype(np.float32)
    return bf16_bits_to_f32(s)


# ----------------------------------------------------------------------------- layouts
def strides_for(layout: str, B: int, H: int, L: int, D: int):
    """Element strides (b, h, l, d) of a contiguous buffer in the given layout."""
    if layout == "bhld":
        return (H * L * D, L * D, D, 1)
    if layout == "blhd":
        return (L * H * D, D, H * D, 1)
    raise ValueError(layout)


def place(x_bhld: np.ndarray, layout: str) -> np.ndarray:
    """Store logical [B,H,L,D] values as a flat contiguous buffer in ``layout``."""
    if layout == "bhld":
        return np.ascontiguousarray(x_bhld).reshape(-1)
    return np.ascontiguousarray(x_bhld.transpose(0, 2, 1, 3)).reshape(-1)


def page1_linspace(shape=(2, 82, 8, 64)) -> np.ndarray:
    """The deterministic input of MLX issue #3585 (float32, given shape)."""
    n = int(np.prod(shape))
    return np.linspace(-0.5, 0.5, n, endpoint=False, dtype=np.float32).reshape(shape)


# ----------------------------------------------------------------------------- cases
@dataclass
class Case:
    """One attention problem: storage buffers plus every size and stride."""
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    Dqk: int
    Dv: int
    dtype: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    strides: tuple                      # 12 element strides: q, k, v x (b, h, l, d)
    out_strides: tuple                  # 4 element strides of the output (b, h, l, d)
    scale: float
    mask_kind: int = MASK_NONE
    mask: np.ndarray | None = None
    mask_strides: tuple = (0, 0, 0, 0)
    layout: str = "bhld"
    meta: dict = field(default_factory=dict)
    window: int = 0                     # sliding-window mask: keys each query sees (0 = not that kind)

    @property
    def all_strides16(self):
        return tuple(self.strides) + tuple(self.out_strides)


def default_scale(Dqk: int) -> float:
    """float(Dqk) ** -0.5 in float64, rounded to float32 (the ABI takes a float)."""
    return float(np.float32(float(Dqk) ** -0.5))


def make_case(seed: int, B: int, Hq: int, Hkv: int, Lq: int, Lk: int, Dqk: int, Dv: int | None = None,
              dtype: int = BF16, mask: str = "none", layout: str = "bhld", p_keep: float = 0.9,
              scale: float | None = None, window: int = 0) -> Case:
    """Seeded N(0,1) case.  mask in {"none", "causal", "decode_additive",
    "additive" ([B,1,Lq,Lk] U(-1,0)), "additive_bcast" ([1,1,Lq,Lk]), "additive_full" ([B,Hq,Lq,Lk]),
    "bool" ([1,1,Lq,Lk]),
    "bool_full" ([B,Hq,Lq,Lk]), "sliding" (causal limited to the `window` most recent keys)}."""
    Dv = Dqk if Dv is None else Dv
    rng = np.random.default_rng(seed)
    qf = rng.standard_normal((B, Hq, Lq, Dqk), dtype=np.float32)
    kf = rng.standard_normal((B, Hkv, Lk, Dqk), dtype=np.float32)
    vf = rng.standard_normal((B, Hkv, Lk, Dv), dtype=np.float32)
    q = to_storage(place(qf, layout), dtype)
    k = to_storage(place(kf, layout), dtype)
    v = to_storage(place(vf, layout), dtype)
    strides = strides_for(layout, B, Hq, Lq, Dqk) + strides_for(layout, B, Hkv, Lk, Dqk) + \
        strides_for(layout, B, Hkv, Lk, Dv)
    out_strides = strides_for(layout, B, Hq, Lq, Dv)
    mk, mbuf, mst = MASK_NONE, None, (0, 0, 0, 0)
    if mask == "causal":
        mk = MASK_CAUSAL
    elif mask == "sliding":
        if window < 1:
            raise ValueError("the sliding-window mask needs window >= 1")
        mk = MASK_SLIDING
    elif mask == "decode_additive":
        m = rng.uniform(-1.0, 0.0, size=(Lk,)).astype(np.float32)
        n_inf = int(np.floor(0.1 * Lk))
        if n_inf:
            m[Lk - n_inf:] = -np.inf
        mk, mbuf, mst = MASK_ADDITIVE, to_storage(m, dtype), (0, 0, 0, 1)
    elif mask == "additive":
        m = rng.uniform(-1.0, 0.0, size=(B, 1, Lq, Lk)).astype(np.float32)
        mk, mbuf, mst = MASK_ADDITIVE, to_storage(m.reshape(-1), dtype), (Lq * Lk, 0, Lk, 1)
    elif mask == "additive_bcast":
        m = rng.uniform(-1.0, 0.0, size=(Lq, Lk)).astype(np.float32)
        mk, mbuf, mst = MASK_ADDITIVE, to_storage(m.reshape(-1), dtype), (0, 0, Lk, 1)
    elif mask == "additive_full":
        m = rng.uniform(-1.0, 0.0, size=(B, Hq, Lq, Lk)).astype(np.float32)
        mk, mbuf, mst = MASK_ADDITIVE, to_storage(m.reshape(-1), dtype), (Hq * Lq * Lk, Lq * Lk, Lk, 1)
    elif mask == "bool":
        m = (rng.random((Lq, Lk)) < p_keep).astype(np.uint8)
        mk, mbuf, mst = MASK_BOOL, m.reshape(-1), (0, 0, Lk, 1)
    elif mask == "bool_full":
        m = (rng.random((B, Hq, Lq, Lk)) < p_keep).astype(np.uint8)
        mk, mbuf, mst = MASK_BOOL, m.reshape(-1), (Hq * Lq * Lk, Lq * Lk, Lk, 1)
    elif mask != "none":
        raise ValueError(mask)
    return Case(B, Hq, Hkv, Lq, Lk, Dqk, Dv, dtype, q, k, v, strides, out_strides,
                default_scale(Dqk) if scale is None else float(np.float32(scale)),
                mk, mbuf, mst, layout, {"seed": seed, "mask": mask}, window if mk == MASK_SLIDING else 0)


def sample_rows(seed: int, B: int, Hq: int, Lq: int, n: int, include_edges: bool = True) -> np.ndarray:
    """Seeded (b, h, i) rows for sampled parity checks at large sizes; always
    includes the first and last query row of the first and last head."""
    rng = np.random.default_rng(seed + 7919)
    rows = np.stack([rng.integers(0, B, n), rng.integers(0, Hq, n), rng.integers(0, Lq, n)], axis=1)
    if include_edges:
        edges = np.array([[0, 0, 0], [0, 0, Lq - 1], [B - 1, Hq - 1, 0], [B - 1, Hq - 1, Lq - 1]])
        rows = np.concatenate([edges, rows], axis=0)
    return np.unique(rows.astype(np.int64), axis=0)
