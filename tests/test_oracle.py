"""Pins for the float64 oracle, checked against things other than itself.

* The values MLX issue #3585 prints for its deterministic linspace input.
* Closed forms (single visible key, constant V, zero scale, causal row 0, Lk = 1).
* Invariants (rows of weights sum to 1, mask shift, joint K/V permutation,
  chunked queries, GQA = repeated KV heads, [B,L,H,D] = [B,H,L,D]).
* The library special case: torch CPU float64 scaled_dot_product_attention.
* Exact dtype decoding: with one key the output is that key's V row, so every
  finite fp16 / bf16 bit pattern must come back as numpy widens it.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from scaled_dot_product_14_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mlx3585_linspace.json")


def run(oracle_mod, c: I.Case, rows=None, want_probs=False):
    return oracle_mod.sdpa_rows(c.q, c.k, c.v, B=c.B, Hq=c.Hq, Hkv=c.Hkv, Lq=c.Lq, Lk=c.Lk,
                                Dqk=c.Dqk, Dv=c.Dv, strides=c.strides, scale=c.scale, dtype=c.dtype,
                                mask_kind=c.mask_kind, mask=c.mask, mask_strides=c.mask_strides,
                                rows=rows, want_probs=want_probs, window=c.window)


def full(oracle_mod, c: I.Case):
    return run(oracle_mod, c).reshape(c.B, c.Hq, c.Lq, c.Dv)


def logical(c: I.Case, which: str) -> np.ndarray:
    """Logical float64 [B,H,L,D] view of a case's stored q/k/v (test-side widening)."""
    buf = {"q": c.q, "k": c.k, "v": c.v}[which]
    H = c.Hq if which == "q" else c.Hkv
    L = c.Lq if which == "q" else c.Lk
    D = c.Dv if which == "v" else c.Dqk
    st = {"q": c.strides[0:4], "k": c.strides[4:8], "v": c.strides[8:12]}[which]
    f = I.storage_to_f32(buf, c.dtype).astype(np.float64)
    idx = (np.arange(c.B)[:, None, None, None] * st[0] + np.arange(H)[None, :, None, None] * st[1]
           + np.arange(L)[None, None, :, None] * st[2] + np.arange(D)[None, None, None, :] * st[3])
    return f[idx]


def with_values(c: I.Case, q=None, k=None, v=None) -> I.Case:
    """Replace logical [B,H,L,D] tensors of a case (stored contiguous [B,H,L,D])."""
    import dataclasses
    qq = logical(c, "q") if q is None else q
    kk = logical(c, "k") if k is None else k
    vv = logical(c, "v") if v is None else v
    st = I.strides_for("bhld", c.B, c.Hq, c.Lq, c.Dqk) + I.strides_for("bhld", c.B, c.Hkv, c.Lk, c.Dqk) + \
        I.strides_for("bhld", c.B, c.Hkv, c.Lk, c.Dv)
    return dataclasses.replace(c, q=I.to_storage(qq.reshape(-1), c.dtype), k=I.to_storage(kk.reshape(-1), c.dtype),
                               v=I.to_storage(vv.reshape(-1), c.dtype), strides=st, layout="bhld")


# --------------------------------------------------------------------------- MLX issue #3585 pins
def _page1(oracle_mod):
    B, S, H, D = 2, 82, 8, 64
    x = I.page1_linspace((B, S, H, D))                  # [B, L, H, D] buffer, float32
    buf = x.reshape(-1)
    scale = float(D) ** -0.5
    # C: correct attention, the buffer read with [B,L,H,D] strides
    st = I.strides_for("blhd", B, H, S, D)
    C = oracle_mod.sdpa_full(buf, buf, buf, B=B, Hq=H, Hkv=H, Lq=S, Lk=S, Dqk=D, Dv=D, strides=st * 3,
                             scale=scale, dtype=I.F32)          # [B,H,L,D]
    C_blhd = C.transpose(0, 2, 1, 3)
    # M: the same contiguous buffer declared as [B, H=82, L=8, D] (the misread layout)
    stm = I.strides_for("bhld", B, S, H, D)
    M = oracle_mod.sdpa_full(buf, buf, buf, B=B, Hq=S, Hkv=S, Lq=H, Lk=H, Dqk=D, Dv=D, strides=stm * 3,
                             scale=scale, dtype=I.F32)          # indexed [2, 82, 8, 64] like the buffer
    # G: the repro's "manual": mx.softmax without an axis is a softmax over the whole array.
    xt = x.astype(np.float64).transpose(0, 2, 1, 3)
    sc = xt @ xt.transpose(0, 1, 3, 2) * scale
    w = np.exp(sc - sc.max())
    w /= w.sum()
    G = (w @ xt).transpose(0, 2, 1, 3)                  # back to [B, L, H, D]
    return x, C, C_blhd, M, G


def test_page1_input_generator_matches_printed_array():
    g = json.load(open(GOLDEN))["printed_input"]
    x = I.page1_linspace((2, 82, 8, 64))
    n = x.size
    assert n == 83968
    np.testing.assert_allclose(x[0, 0, 0, :3], g["first_row_head"], atol=5e-7)
    np.testing.assert_allclose(x[0, 0, 0, -3:], g["first_row_tail"], atol=5e-7)
    np.testing.assert_allclose(x[1, 0, 0, :3], g["batch1_first_row_head"], atol=5e-11)
    np.testing.assert_allclose(x[-1, -1, -1, -3:], g["last_row_tail"], atol=5e-7)
    assert x[1, 0, 0, 0] == 0.0 and x[0, 0, 0, 0] == -0.5


def test_page1_printed_differences(oracle_mod):
    gold = json.load(open(GOLDEN))["printed"]
    x, C, C_blhd, M, G = _page1(oracle_mod)
    d_gm = np.abs(G - M)
    # 7 printed significant digits: half a unit in the last place is 5e-8.
    assert abs(d_gm.max() - gold["manual_vs_fused_max_diff"]) <= 6e-8
    worst = np.unravel_index(np.argmax(d_gm), d_gm.shape)
    assert abs(G[worst] - gold["worst_element_manual"]) <= 6e-7
    assert abs(M[worst] - gold["worst_element_fused"]) <= 6e-7
    d_gc = np.abs(G - C_blhd)
    assert abs(d_gc.max() - gold["manual_vs_pytorch_fused_max_diff"]) <= 6e-8


def test_page1_layouts_agree(oracle_mod):
    """C (strided [B,L,H,D]) equals the oracle on a contiguous [B,H,L,D] copy."""
    x, C, C_blhd, M, G = _page1(oracle_mod)
    xt = np.ascontiguousarray(x.transpose(0, 2, 1, 3)).reshape(-1)
    B, S, H, D = x.shape
    C2 = oracle_mod.sdpa_full(xt, xt, xt, B=B, Hq=H, Hkv=H, Lq=S, Lk=S, Dqk=D, Dv=D,
                              strides=I.strides_for("bhld", B, H, S, D) * 3, scale=D ** -0.5, dtype=I.F32)
    assert np.abs(C - C2).max() <= 1e-12
    # the library computes the same thing on the transposed view (the maintainer's PyTorch check)
    t = torch.from_numpy(x.astype(np.float64)).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(t, t, t, scale=D ** -0.5).numpy()
    assert np.abs(C - ref).max() <= 1e-12


# --------------------------------------------------------------------------- closed forms
@pytest.mark.parametrize("dtype", [I.F32, I.BF16, I.F16])
def test_single_visible_key_returns_its_value_row(oracle_mod, dtype):
    c = I.make_case(11, 1, 2, 1, 3, 9, 64, dtype=dtype, mask="bool_full")
    m = np.zeros((1, 2, 3, 9), np.uint8)
    keep = [[4, 0, 8], [2, 2, 7]]
    for h in range(2):
        for i in range(3):
            m[0, h, i, keep[h][i]] = 1
    c.mask = m.reshape(-1)
    o = full(oracle_mod, c)
    v = logical(c, "v")
    for h in range(2):
        for i in range(3):
            np.testing.assert_array_equal(o[0, h, i], v[0, 0, keep[h][i]])


def test_constant_v_gives_the_constant(oracle_mod):
    c = I.make_case(12, 2, 4, 2, 5, 33, 72, dtype=I.F32, mask="additive")
    c = with_values(c, v=np.full((2, 2, 33, 72), 0.625))
    o = full(oracle_mod, c)
    assert np.abs(o - 0.625).max() <= 1e-15


def test_zero_scale_gives_mean_of_visible_rows(oracle_mod):
    c = I.make_case(13, 1, 2, 2, 6, 6, 64, dtype=I.F32, mask="causal", scale=0.0)
    o = full(oracle_mod, c)
    v = logical(c, "v")
    for h in range(2):
        for i in range(6):
            np.testing.assert_allclose(o[0, h, i], v[0, h, :i + 1].mean(0), atol=1e-14)


def test_causal_row0_and_single_key(oracle_mod):
    c = I.make_case(14, 2, 4, 4, 7, 7, 80, dtype=I.F16, mask="causal")
    o = full(oracle_mod, c)
    v = logical(c, "v")
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    c1 = I.make_case(15, 2, 4, 2, 5, 1, 96, dtype=I.BF16)
    o1 = full(oracle_mod, c1)
    v1 = logical(c1, "v")
    for h in range(4):
        for i in range(5):
            np.testing.assert_array_equal(o1[:, h, i], v1[:, h // 2, 0])


def test_fully_masked_rows_are_zero(oracle_mod):
    # Lq > Lk causal: rows i < Lq - Lk see no key under bottom-right alignment
    c = I.make_case(16, 1, 2, 1, 9, 4, 64, dtype=I.F32, mask="causal")
    o = full(oracle_mod, c)
    assert np.all(o[:, :, :5] == 0.0)
    assert np.all(np.isfinite(o))
    np.testing.assert_array_equal(o[0, 0, 5], logical(c, "v")[0, 0, 0])


# --------------------------------------------------------------------------- invariants
def test_weight_rows_sum_to_one(oracle_mod):
    c = I.make_case(21, 2, 4, 2, 9, 40, 128, dtype=I.BF16, mask="bool")
    _, p = run(oracle_mod, c, want_probs=True)
    s = p.sum(1)
    assert np.abs(s - 1.0).max() <= 1e-13
    assert np.all(p >= 0)


def test_additive_mask_row_shift_changes_nothing(oracle_mod):
    c = I.make_case(22, 1, 2, 2, 6, 17, 64, dtype=I.F32, mask="additive_full")
    # put the mask on a 2^-10 grid so that the per-row shift below is exact in fp32
    m0 = np.floor(I.storage_to_f32(c.mask, c.dtype) * 1024) / 1024
    c.mask = I.to_storage(m0, c.dtype)
    o1 = full(oracle_mod, c)
    m = m0.reshape(1, 2, 6, 17) + np.float32(0.25) * np.arange(6)[None, None, :, None]
    c.mask = I.to_storage(m.reshape(-1), c.dtype)
    o2 = full(oracle_mod, c)
    assert np.abs(o1 - o2).max() <= 1e-12


def test_joint_kv_permutation_changes_nothing(oracle_mod):
    c = I.make_case(23, 2, 2, 1, 5, 23, 64, dtype=I.F32)
    o1 = full(oracle_mod, c)
    perm = np.random.default_rng(0).permutation(23)
    c2 = with_values(c, k=logical(c, "k")[:, :, perm], v=logical(c, "v")[:, :, perm])
    o2 = full(oracle_mod, c2)
    assert np.abs(o1 - o2).max() <= 1e-12


@pytest.mark.parametrize("lq", [4, 16])
@pytest.mark.parametrize("mask", ["none", "causal", "additive"])
def test_chunked_queries_equal_unchunked(oracle_mod, lq, mask):
    """mlxcel issue #1065 ("f32 matmul and single-query SDPA lose ~fp16 precision"),
    section "The four failing tests": chunked query attention must equal the
    unchunked call.  A chunk of queries [a, a+n) attends to keys [0, Lk - Lq + a + n)
    under bottom-right causal alignment."""
    Lk = lq + 9
    c = I.make_case(24, 1, 4, 2, lq, Lk, 64, dtype=I.F32, mask=mask)
    ref = full(oracle_mod, c)
    q = logical(c, "q")
    mfull = None if c.mask is None else I.storage_to_f32(c.mask, c.dtype).reshape(1, 1, lq, Lk)
    for chunk in [1, 2, 3, 4, 5]:
        got = np.zeros_like(ref)
        for a in range(0, lq, chunk):
            n = min(chunk, lq - a)
            kv_len = Lk - lq + a + n if mask == "causal" else Lk
            sub = I.make_case(24, 1, 4, 2, n, kv_len, 64, dtype=I.F32, mask=mask)
            sub = with_values(sub, q=q[:, :, a:a + n], k=logical(c, "k")[:, :, :kv_len],
                              v=logical(c, "v")[:, :, :kv_len])
            if mfull is not None:
                sub.mask = I.to_storage(np.ascontiguousarray(mfull[:, :, a:a + n, :kv_len]).reshape(-1), c.dtype)
                sub.mask_strides = (n * kv_len, 0, kv_len, 1)
            got[:, :, a:a + n] = full(oracle_mod, sub)
        assert np.abs(got - ref).max() <= 1e-12, chunk


def test_gqa_equals_repeated_kv(oracle_mod):
    c = I.make_case(25, 2, 8, 2, 5, 11, 64, dtype=I.F32, mask="bool_full")
    o1 = full(oracle_mod, c)
    k = np.repeat(logical(c, "k"), 4, axis=1)
    v = np.repeat(logical(c, "v"), 4, axis=1)
    import dataclasses
    c2 = dataclasses.replace(c, Hkv=8)
    c2 = with_values(c2, q=logical(c, "q"), k=k, v=v)
    o2 = full(oracle_mod, c2)
    assert np.abs(o1 - o2).max() <= 1e-12


@pytest.mark.parametrize("dtype", [I.F32, I.BF16])
def test_layouts_agree(oracle_mod, dtype):
    a = I.make_case(26, 2, 4, 2, 7, 13, 96, dtype=dtype, layout="bhld")
    b = I.make_case(26, 2, 4, 2, 7, 13, 96, dtype=dtype, layout="blhd")
    assert np.abs(full(oracle_mod, a) - full(oracle_mod, b)).max() <= 1e-12


# --------------------------------------------------------------------------- library special case
def _torch_ref(c: I.Case):
    q = torch.from_numpy(logical(c, "q"))
    k = torch.from_numpy(logical(c, "k")).repeat_interleave(c.Hq // c.Hkv, dim=1)
    v = torch.from_numpy(logical(c, "v")).repeat_interleave(c.Hq // c.Hkv, dim=1)
    mask, causal = None, False
    if c.mask_kind == I.MASK_CAUSAL:
        assert c.Lq == c.Lk
        causal = True
    elif c.mask_kind in (I.MASK_ADDITIVE, I.MASK_BOOL):
        ms = c.mask_strides
        f = I.storage_to_f32(c.mask, c.dtype).astype(np.float64) if c.mask_kind == I.MASK_ADDITIVE else c.mask
        idx = (np.arange(c.B)[:, None, None, None] * ms[0] + np.arange(c.Hq)[None, :, None, None] * ms[1]
               + np.arange(c.Lq)[None, None, :, None] * ms[2] + np.arange(c.Lk)[None, None, None, :] * ms[3])
        m = f[idx]
        mask = torch.from_numpy(m) if c.mask_kind == I.MASK_ADDITIVE else torch.from_numpy(m != 0)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, is_causal=causal,
                                                            scale=c.scale).numpy()


@pytest.mark.parametrize("D,Dv", [(64, 64), (72, 72), (80, 80), (96, 96), (128, 128), (192, 128), (256, 256), (512, 512)])
@pytest.mark.parametrize("mask", ["none", "additive", "bool", "causal"])
def test_matches_torch_float64(oracle_mod, D, Dv, mask):
    c = I.make_case(30 + D, 2, 4, 2, 9, 9, D, Dv, dtype=I.BF16, mask=mask, p_keep=0.8)
    if c.mask_kind == I.MASK_BOOL:      # torch returns NaN for rows with no key; keep one key per row
        m = c.mask.reshape(c.Lq, c.Lk)
        m[:, 0] = 1
    o = full(oracle_mod, c)
    ref = _torch_ref(c)
    assert np.abs(o - ref).max() <= 1e-12


def test_matches_torch_decode_mask_with_minus_inf(oracle_mod):
    c = I.make_case(40, 1, 8, 2, 1, 50, 256, dtype=I.BF16, mask="decode_additive")
    assert np.isneginf(I.storage_to_f32(c.mask, c.dtype)[-5:]).all()
    assert np.abs(full(oracle_mod, c) - _torch_ref(c)).max() <= 1e-12


# --------------------------------------------------------------------------- exact dtype decoding
@pytest.mark.parametrize("dtype", [I.F16, I.BF16])
def test_every_finite_bit_pattern_decodes_exactly(oracle_mod, dtype):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = I.storage_to_f32(bits, dtype)
    bits = bits[np.isfinite(vals)]
    vals = I.storage_to_f32(bits, dtype).astype(np.float64)
    Dv = bits.size
    q = I.to_storage(np.ones(64, np.float32), dtype)
    k = I.to_storage(np.ones(64, np.float32), dtype)
    st = (64, 64, 64, 1, 64, 64, 64, 1, Dv, Dv, Dv, 1)
    o = oracle_mod.sdpa_rows(q, k, bits, B=1, Hq=1, Hkv=1, Lq=1, Lk=1, Dqk=64, Dv=Dv, strides=st,
                             scale=0.125, dtype=dtype)
    np.testing.assert_array_equal(o[0], vals)


def test_fp32_path_is_not_reduced_precision(oracle_mod):
    """mlxcel issue #1065: an error near 2^-10 in fp32 marks reduced internal
    precision.  The oracle on fp32 inputs must agree with torch float64 far below it."""
    c = I.make_case(41, 1, 4, 4, 4, 4, 64, dtype=I.F32, mask="causal")
    assert np.abs(full(oracle_mod, c) - _torch_ref(c)).max() < 1e-12 < 2.0 ** -10


# --------------------------------------------------------------------------- sliding window
# The pages name Gemma 4's sliding (local) attention layers (MLX issue #3885,
# "Current routing") without their rule; the reading pinned here: with the
# causal bottom-right alignment own = i + Lk - Lq, key j is visible iff
# own - W < j <= own.
@pytest.mark.parametrize("Lq,Lk", [(7, 7), (3, 9), (9, 5)])
def test_window_of_one_returns_the_own_key(oracle_mod, Lq, Lk):
    """W = 1: each query sees exactly its own (bottom-right aligned) key, so the
    row is that key's V row exactly; queries whose own position is before key 0
    see nothing and give zeros."""
    c = I.make_case(50, 1, 4, 2, Lq, Lk, 64, dtype=I.BF16, mask="sliding", window=1)
    o, v = full(oracle_mod, c), logical(c, "v")
    for h in range(4):
        for i in range(Lq):
            own = i + Lk - Lq
            if own < 0:
                assert np.all(o[0, h, i] == 0.0)
            else:
                np.testing.assert_array_equal(o[0, h, i], v[0, h // 2, own])


def test_window_of_two_is_a_two_key_softmax(oracle_mod):
    """W = 2: the row is the softmax-weighted mean of the V rows at own - 1 and
    own, weights 1 / (1 + e^(s_other - s_self)) worked out per row here."""
    c = I.make_case(51, 1, 2, 1, 6, 10, 64, dtype=I.F32, mask="sliding", window=2)
    o, q, k, v = full(oracle_mod, c), logical(c, "q"), logical(c, "k"), logical(c, "v")
    for h in range(2):
        for i in range(6):
            own = i + 4
            s_prev = c.scale * float(q[0, h, i] @ k[0, 0, own - 1])
            s_own = c.scale * float(q[0, h, i] @ k[0, 0, own])
            w_own = 1.0 / (1.0 + math.exp(s_prev - s_own))
            expect = w_own * v[0, 0, own] + (1.0 - w_own) * v[0, 0, own - 1]
            assert np.abs(o[0, h, i] - expect).max() <= 1e-12


@pytest.mark.parametrize("W", [9, 10, 1000])
def test_window_covering_every_key_is_causal(oracle_mod, W):
    c = I.make_case(52, 2, 4, 2, 9, 9, 80, dtype=I.F16, mask="sliding", window=W)
    import dataclasses
    causal = dataclasses.replace(c, mask_kind=I.MASK_CAUSAL, window=0)
    assert np.abs(full(oracle_mod, c) - _torch_ref(causal)).max() <= 1e-12


@pytest.mark.parametrize("W", [1, 3, 8])
@pytest.mark.parametrize("Lq,Lk", [(12, 12), (5, 17)])
def test_window_matches_torch_with_a_band_matrix(oracle_mod, W, Lq, Lk):
    """torch float64 SDPA with an explicit boolean band built as a matrix (lower
    triangle of the shifted causal mask minus the triangle W below it); rows
    with an empty band are excluded (torch gives NaN there)."""
    c = I.make_case(53 + W, 2, 4, 2, Lq, Lk, 128, dtype=I.BF16, mask="sliding", window=W)
    ones = np.ones((Lq, Lk), dtype=bool)
    band = np.tril(ones, k=Lk - Lq) & ~np.tril(ones, k=Lk - Lq - W)
    q = torch.from_numpy(logical(c, "q"))
    k = torch.from_numpy(logical(c, "k")).repeat_interleave(2, dim=1)
    v = torch.from_numpy(logical(c, "v")).repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(band),
                                                           scale=c.scale).numpy()
    o = full(oracle_mod, c)
    rows = band.any(axis=1)
    assert np.abs(o[:, :, rows] - ref[:, :, rows]).max() <= 1e-12
    assert np.all(o[:, :, ~rows] == 0.0)


def test_window_chunked_queries_equal_unchunked(oracle_mod):
    """Bottom-right alignment makes a chunk of the last queries see the same
    keys as in the whole call (mlxcel issue #1065's chunked-prefill check)."""
    c = I.make_case(54, 1, 2, 2, 8, 20, 64, dtype=I.F32, mask="sliding", window=5)
    whole = full(oracle_mod, c)
    for a in range(8):
        sub = I.make_case(54, 1, 2, 2, 1, 20 - 7 + a, 64, dtype=I.F32, mask="sliding", window=5)
        sub = with_values(sub, q=logical(c, "q")[:, :, a:a + 1], k=logical(c, "k")[:, :, :20 - 7 + a],
                          v=logical(c, "v")[:, :, :20 - 7 + a])
        assert np.abs(full(oracle_mod, sub)[:, :, 0] - whole[:, :, a]).max() <= 1e-12
