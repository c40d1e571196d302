"""GPU parity: the CUDA path through the C ABI against the float64 oracle, on
the same seeded stored inputs, element by element (every row at sizes the
oracle finishes in seconds; seeded sampled rows at full sizes).

Workloads follow the pages: the MLX issue #3585 linspace case, the decode
shapes of MLX issue #3885 (d=256 32q/8kv and d=512 32q/4kv, additive mask, qL=1,
seqK 1k/4k; d=512 prefill), the head-dim-72 prefill of MLX PR #4330 (B=1, 16
heads, N=8192), and that PR's coverage sweep (dtypes x masks, aligned and
unaligned lengths)."""
import json
import os

import numpy as np
import pytest
import torch

import scaled_dot_product_14_b200 as S
from scaled_dot_product_14_b200 import inputs as I

from gpu_util import GpuCase, compare, oracle_rows, run_and_check, TOL

pytestmark = pytest.mark.gpu

DIMS = [(64, 64), (72, 72), (80, 80), (96, 96), (128, 128), (192, 128), (256, 256), (512, 512)]
DTYPES = [I.F32, I.F16, I.BF16]
MASKS = ["none", "additive", "bool", "causal"]


@pytest.fixture(scope="module", autouse=True)
def built():
    from scaled_dot_product_14_b200 import build
    import oracle
    build.build()
    oracle.build()
    assert torch.cuda.is_available()
    cap = torch.cuda.get_device_capability()
    assert cap == (10, 0), f"expected a B200 (sm_100), got {cap}"


def path_of(c):
    st, path = S.sdpa_supported(c.B, c.Hq, c.Hkv, c.Lq, c.Lk, c.Dqk, c.Dv, c.all_strides16, c.mask_kind,
                                c.mask_strides if c.mask is not None else None, c.dtype)
    assert st == 0
    return path


# ---------------------------------------------------------------- MLX issue #3585 linspace case
def _page1_case(layout_view: str, values: np.ndarray):
    """values: float32 [B, L, H, D]."""
    B, L, H, D = values.shape
    if layout_view == "blhd_strided":        # the [B,L,H,D] buffer passed with its own strides
        buf, st = values.reshape(-1), I.strides_for("blhd", B, H, L, D)
        ost = I.strides_for("blhd", B, H, L, D)
    else:                                    # a contiguous [B,H,L,D] copy
        buf = np.ascontiguousarray(values.transpose(0, 2, 1, 3)).reshape(-1)
        st = ost = I.strides_for("bhld", B, H, L, D)
    return I.Case(B, H, H, L, L, D, D, I.F32, buf, buf.copy(), buf.copy(), st * 3, ost, I.default_scale(D),
                  layout="blhd" if layout_view == "blhd_strided" else "bhld")


@pytest.mark.parametrize("view", ["blhd_strided", "bhld_copy"])
def test_page1_linspace(view):
    x = I.page1_linspace((2, 82, 8, 64))
    c = _page1_case(view, x)
    (mx, mean), got = run_and_check(c, label=f"page1 {view}")
    assert path_of(c) == S.SDPA_PATH_PREFILL


def test_page1_normal_copy():
    x = np.random.default_rng(1000).standard_normal((2, 82, 8, 64), dtype=np.float32)
    run_and_check(_page1_case("blhd_strided", x), label="page1 N(0,1)")


def test_page1_printed_differences_through_gpu():
    """The GPU reproduces both printed max-differences of MLX issue #3585: fed the
    buffer with its true [B,L,H,D] strides it gives correct attention (0.3308013
    from the whole-array-softmax "manual"), and fed the same buffer declared as
    [B, H=82, L=8, D] it gives the misread-layout output (0.4969254)."""
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "mlx3585_linspace.json")))["printed"]
    x = I.page1_linspace((2, 82, 8, 64))
    xt = x.astype(np.float64).transpose(0, 2, 1, 3)
    sc = xt @ xt.transpose(0, 1, 3, 2) * (64 ** -0.5)
    w = np.exp(sc - sc.max())
    G = ((w / w.sum()) @ xt).transpose(0, 2, 1, 3)
    g = GpuCase(_page1_case("blhd_strided", x))
    assert g.run() == 0
    C = g.output().transpose(0, 2, 1, 3)
    assert abs(np.abs(G - C).max() - gold["manual_vs_pytorch_fused_max_diff"]) < 1e-5
    buf = x.reshape(-1)
    st = I.strides_for("bhld", 2, 82, 8, 64)
    mis = I.Case(2, 82, 82, 8, 8, 64, 64, I.F32, buf, buf, buf, st * 3, st, I.default_scale(64))
    gm = GpuCase(mis)
    assert gm.run() == 0
    M = gm.output()
    assert abs(np.abs(G - M).max() - gold["manual_vs_fused_max_diff"]) < 1e-5


# ---------------------------------------------------------------- decode workloads (MLX issue #3885)
@pytest.mark.parametrize("kL", [1024, 4096])
def test_decode_d256_gqa4_additive(kL):
    c = I.make_case(1001, 1, 32, 8, 1, kL, 256, dtype=I.BF16, mask="decode_additive")
    assert path_of(c) == S.SDPA_PATH_DECODE
    before = S.sdpa_get_counters()
    run_and_check(c, label=f"decode d256 kL={kL}")
    after = S.sdpa_get_counters()
    assert after["decode_mma_launches"] == before["decode_mma_launches"] + 1


@pytest.mark.parametrize("kL", [1024, 4096])
@pytest.mark.parametrize("mask", ["none", "decode_additive"])
def test_decode_d512_gqa8(kL, mask):
    c = I.make_case(1002, 1, 32, 4, 1, kL, 512, dtype=I.BF16, mask=mask)
    run_and_check(c, label=f"decode d512 kL={kL} {mask}")


@pytest.mark.parametrize("splits", [1, 4, 16, "one wave"])
@pytest.mark.parametrize("D,Hkv", [(512, 4), (256, 8), (64, 8)])
@pytest.mark.parametrize("mask", ["none", "decode_additive"])
def test_decode_ring_reuse(monkeypatch, splits, D, Hkv, mask):
    """Few splits give each CTA many key slots, so every ring position of the
    decode kernel is reused many times (at D = 512 the ring has 3 positions of
    2 sub-blocks for 7 consumer warps, so a warp's first sub-block can already
    sit in a position's second use).  Repeated calls: a race would show as a
    mismatch in some of them."""
    if splits == "one wave":   # as many splits as fill the SMs
        splits = torch.cuda.get_device_properties(0).multi_processor_count // Hkv
    monkeypatch.setenv("SDPA_DECODE_SPLITS", str(splits))
    c = I.make_case(1003, 1, 32, Hkv, 1, 4096, D, dtype=I.BF16, mask=mask)
    g = GpuCase(c)
    ref = oracle_rows(c).reshape(-1, D)
    for _ in range(3):
        assert g.run() == 0
        got = g.output().reshape(-1, D)
        err = np.abs(got - ref)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (splits, D, mask, float(err.max()), float(err.mean()))
    assert S.sdpa_check_device_error() == (0, 0)


def test_prefill_d512_causal_4096():
    c = I.make_case(1002, 1, 32, 4, 4096, 4096, 512, dtype=I.BF16, mask="causal")
    rows = I.sample_rows(1002, 1, 32, 4096, 96)
    run_and_check(c, rows=rows, label="prefill d512 causal L=4096")


# ---------------------------------------------------------------- head dim 72 prefill (MLX PR #4330)
@pytest.mark.parametrize("dtype,mask", [(I.BF16, "none"), (I.F16, "none"), (I.BF16, "bool")])
def test_prefill_d72_8192(dtype, mask):
    c = I.make_case(1003, 1, 16, 16, 8192, 8192, 72, dtype=dtype, mask=mask, layout="blhd", p_keep=0.9)
    rows = I.sample_rows(1003, 1, 16, 8192, 256)
    run_and_check(c, rows=rows, label=f"prefill d72 {dtype} {mask}")


# ---------------------------------------------------------------- the coverage sweep
def _sweep_case(D, Dv, dtype, mask, L, seed, B=2):
    return I.make_case(seed, B, 32, 8, L, L, D, Dv, dtype=dtype, mask=mask)


@pytest.mark.parametrize("D,Dv", DIMS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("mask", MASKS)
def test_sweep_L128_full(D, Dv, dtype, mask):
    c = _sweep_case(D, Dv, dtype, mask, 128, 1004)
    run_and_check(c, label=f"sweep L=128 D={D} dt={dtype} {mask}")


@pytest.mark.parametrize("D,Dv", DIMS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("mask", MASKS)
def test_sweep_L2048_sampled(D, Dv, dtype, mask):
    c = _sweep_case(D, Dv, dtype, mask, 2048, 1005)
    rows = I.sample_rows(1005, 2, 32, 2048, 48)
    run_and_check(c, rows=rows, label=f"sweep L=2048 D={D} dt={dtype} {mask}")


_L16K_MASKS = {}


def _l16k_masks(dtype):
    """The configured masks of the L=16384 sweep for one dtype: additive
    [B,1,Lq,Lk] U(-1,0) and boolean [1,1,Lq,Lk] (p_keep 0.9), each drawn once
    from its own seeded generator and shared by every head dim (one draw of the
    1.07 G-element additive mask takes seconds on the host)."""
    if dtype not in _L16K_MASKS:
        _L16K_MASKS.clear()
        L = 16384
        add = np.random.default_rng(1006 + 50000).uniform(-1.0, 0.0, size=(2, 1, L, L)).astype(np.float32)
        keep = (np.random.default_rng(1006 + 60000).random((L, L)) < 0.9).astype(np.uint8)
        _L16K_MASKS[dtype] = (I.to_storage(add.reshape(-1), dtype), keep.reshape(-1))
    return _L16K_MASKS[dtype]


@pytest.mark.parametrize("dtype,D,Dv", [(dt, D, Dv) for dt in DTYPES for (D, Dv) in DIMS])
def test_sweep_L16384_sampled(dtype, D, Dv):
    """Every (head dim, dtype, mask) cell of the sweep at L=16384, B=2, Hq=32,
    Hkv=8, on seeded sampled rows (plus the first and last rows): the same
    Q/K/V for the four masks, the additive mask [B,1,Lq,Lk] as configured."""
    import dataclasses
    L = 16384
    base = I.make_case(1006, 2, 32, 8, L, L, D, Dv, dtype=dtype, mask="none")
    add, keep = _l16k_masks(dtype)
    variants = {
        "none": base,
        "causal": dataclasses.replace(base, mask_kind=I.MASK_CAUSAL),
        "additive": dataclasses.replace(base, mask_kind=I.MASK_ADDITIVE, mask=add, mask_strides=(L * L, 0, L, 1)),
        "bool": dataclasses.replace(base, mask_kind=I.MASK_BOOL, mask=keep, mask_strides=(0, 0, L, 1)),
    }
    rows = I.sample_rows(1006 + D, 2, 32, L, 32)
    for mask in MASKS:
        run_and_check(variants[mask], rows=rows, label=f"sweep L=16384 D={D} dt={dtype} {mask}")


@pytest.mark.parametrize("D,Dv", DIMS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("mask", MASKS)
def test_chunked_query_consistency(D, Dv, dtype, mask):
    """mlxcel issue #1065, "The four failing tests": qL=4 in chunks of 1 must equal
    the unchunked call; each chunk is a decode call on a key prefix (causal,
    bottom-right) and every result is checked against the oracle."""
    lq, lk = 4, 300
    c = I.make_case(1007, 2, 32, 8, lq, lk, D, Dv, dtype=dtype,
                    mask={"additive": "additive", "bool": "bool_full"}.get(mask, mask))
    (_, _), full = run_and_check(c, label="unchunked")
    tmax, _ = TOL[dtype]
    for a in range(lq):
        import dataclasses
        kv = lk - lq + a + 1 if mask == "causal" else lk
        st = c.strides
        sub = dataclasses.replace(
            c, Lq=1, Lk=kv, q=c.q[a * st[2]:], mask_kind=c.mask_kind,
            mask=None if c.mask is None else c.mask[a * c.mask_strides[2]:])
        (_, _), part = run_and_check(sub, label=f"chunk {a}")
        assert np.abs(part[:, :, 0] - full[:, :, a]).max() <= 2 * tmax


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("Lq", [1, 2, 7, 8, 9, 16, 17, 127, 129])
@pytest.mark.parametrize("Lk", [1, 7, 127, 129])
@pytest.mark.parametrize("dtype,D,mask", [(I.BF16, 128, "causal"), (I.F16, 72, "none"), (I.F32, 96, "bool_full"),
                                          (I.BF16, 512, "additive")])
def test_ragged_lengths(Lq, Lk, dtype, D, mask):
    c = I.make_case(1100 + Lq * 7 + Lk, 2, 4, 2, Lq, Lk, D, dtype=dtype, mask=mask, p_keep=0.7)
    run_and_check(c, label=f"Lq={Lq} Lk={Lk}")


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32])
@pytest.mark.parametrize("Lq", [1, 8, 40])
def test_gqa_ratios(G, Lq):
    c = I.make_case(1200 + G, 2, 2 * G, 2, Lq, 333, 128, dtype=I.BF16, mask="causal" if Lq > 1 else "none")
    run_and_check(c, label=f"G={G} Lq={Lq}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_many_decode_rows(dtype):
    # 64 query heads on one KV head, 8 queries: 512 rows per group -> several row groups per CTA grid
    c = I.make_case(1300, 2, 64, 1, 8, 1000, 128, dtype=dtype, mask="causal")
    run_and_check(c, label="MQA qL=8")


@pytest.mark.parametrize("Lq", [1, 33])
def test_no_keys_gives_zeros(Lq):
    c = I.make_case(1400, 1, 4, 2, Lq, 0, 64, dtype=I.BF16)
    g = GpuCase(c)
    assert g.run() == 0
    assert np.all(g.output() == 0.0)


def test_empty_batch_launches_nothing():
    c = I.make_case(1401, 0, 4, 2, 16, 16, 64, dtype=I.BF16)
    before = S.sdpa_get_counters()
    g = GpuCase(c)
    assert g.run() == 0
    after = S.sdpa_get_counters()
    assert after["empty_calls"] == before["empty_calls"] + 1
    assert S.sdpa_last_launch_count() == 0


@pytest.mark.parametrize("Lq", [8, 40])
@pytest.mark.parametrize("dtype", DTYPES)
def test_causal_more_queries_than_keys(Lq, dtype):
    """Bottom-right alignment: queries i < Lq - Lk see no key and output zeros."""
    c = I.make_case(1402, 1, 4, 2, Lq, 5, 64, dtype=dtype, mask="causal")
    (_, _), got = run_and_check(c, label="causal Lq>Lk")
    assert np.all(got[:, :, :Lq - 5] == 0.0)


@pytest.mark.parametrize("Lq", [1, 24])
def test_fully_masked_rows_are_zero(Lq):
    c = I.make_case(1403, 1, 4, 2, Lq, 100, 256, dtype=I.BF16, mask="bool")
    c.mask.reshape(Lq, 100)[0, :] = 0
    (_, _), got = run_and_check(c, label="masked row")
    assert np.all(got[:, :, 0] == 0.0)
    c2 = I.make_case(1404, 1, 4, 2, Lq, 100, 64, dtype=I.F16, mask="additive")
    m = I.storage_to_f32(c2.mask, c2.dtype).reshape(1, 1, Lq, 100)
    m[0, 0, 0, :] = -np.inf
    c2.mask = I.to_storage(m.reshape(-1), c2.dtype)
    (_, _), got2 = run_and_check(c2, label="-inf row")
    assert np.all(got2[:, :, 0] == 0.0)


@pytest.mark.parametrize("Lq", [1, 100])
def test_strided_views(Lq):
    """q as a head-slice of a wider tensor, out into a strided sub-view."""
    B, Hq, Hkv, Lk, D = 2, 8, 4, 150, 128
    big = I.make_case(1500, B, 2 * Hq, Hkv, Lq, Lk, D, dtype=I.BF16, layout="blhd")
    import dataclasses
    st = list(big.strides)
    # take every other query head: head stride doubles, count halves
    st[1] = 2 * st[1]
    ost = (Lq * Hq * 2 * D, 2 * D, Hq * 2 * D, 1)   # out: [B, L, 2*Hq, D] buffer, every other head
    c = dataclasses.replace(big, Hq=Hq, strides=tuple(st), out_strides=ost)
    run_and_check(c, label="strided view")


def test_layouts_agree_on_gpu():
    a = I.make_case(1600, 2, 8, 2, 200, 200, 96, dtype=I.BF16, layout="bhld", mask="causal")
    b = I.make_case(1600, 2, 8, 2, 200, 200, 96, dtype=I.BF16, layout="blhd", mask="causal")
    (_, _), ga = run_and_check(a, label="bhld")
    (_, _), gb = run_and_check(b, label="blhd")
    assert np.abs(ga - gb).max() <= 1e-6


TF32_DIMS = [(40, 32), (64, 64), (72, 72), (80, 80), (96, 96)]


@pytest.mark.parametrize("D,Dv", [(64, 64), (72, 72), (80, 80), (96, 96), (128, 128), (192, 128)])
@pytest.mark.parametrize("mask", MASKS)
def test_fp32_prefill_tiles(D, Dv, mask):
    """fp32 prefill: the tcgen05 three-term TF32 kernel at head dims up to 96
    (128-row query tiles, 64-key tiles), the register-tiled FFMA kernel above
    (128 group rows per CTA, 64-key tiles): Lq=100 with 4 query heads per KV
    head puts rows of two heads in one FFMA row tile, and Lk=200 leaves a ragged
    last key tile on both."""
    c = I.make_case(1900 + D, 2, 8, 2, 100, 200, D, Dv, dtype=I.F32, mask=mask, layout="blhd", p_keep=0.7)
    before = S.sdpa_get_counters()
    run_and_check(c, label=f"fp32 D={D} {mask}")
    after = S.sdpa_get_counters()
    fam = "prefill_tf32_launches" if (D, Dv) in TF32_DIMS else "prefill_ffma_launches"
    assert after[fam] == before[fam] + 1


@pytest.mark.parametrize("D,Dv", TF32_DIMS)
@pytest.mark.parametrize("mask", MASKS + ["sliding"])
@pytest.mark.parametrize("Lq,Lk", [(129, 129), (300, 1000), (1000, 300), (2048, 2048)])
def test_fp32_three_term_tf32_holds_fp32_accuracy(D, Dv, mask, Lq, Lk):
    """mlxcel issue #1065: TF32 inside an fp32 path must not show up as error;
    the three-term split keeps max-abs <= 1e-5 against the float64 oracle (far
    below the 2^-10 fingerprint of plain TF32) over ragged tiles, Lq != Lk and
    every mask kind; sampled rows at the larger sizes."""
    c = I.make_case(2600 + D + Lq, 1, 8, 2, Lq, Lk, D, Dv, dtype=I.F32, mask=mask, p_keep=0.7, window=150)
    before = S.sdpa_get_counters()
    rows = None if Lq * Lk <= 300_000 else I.sample_rows(2600 + D, 1, 8, Lq, 96)
    (mx, _), _ = run_and_check(c, rows=rows, label=f"tf32x3 D={D} {mask} {Lq}x{Lk}")
    after = S.sdpa_get_counters()
    assert after["prefill_tf32_launches"] == before["prefill_tf32_launches"] + 1
    assert mx <= 1e-5 < 2.0 ** -10


def test_fp32_keeps_fp32_precision():
    """mlxcel issue #1065: fp32 error near 2^-10 = 9.77e-4 would mean reduced
    internal precision; the fp32 path must stay far below it on both paths."""
    for Lq in (1, 64):
        c = I.make_case(1700 + Lq, 1, 8, 2, Lq, 4096, 128, dtype=I.F32, mask="causal")
        (mx, mean), _ = run_and_check(c, label=f"fp32 Lq={Lq}")
        assert mx < 1e-5 < 2.0 ** -10


def test_repeat_calls_are_deterministic():
    c = I.make_case(1800, 1, 32, 8, 1, 4096, 256, dtype=I.BF16, mask="decode_additive")
    g = GpuCase(c)
    assert g.run() == 0
    a = g.output().copy()
    assert g.run() == 0
    b = g.output()
    assert np.array_equal(a, b)


def test_counters_invariant():
    c = S.sdpa_get_counters()
    assert c["calls"] == c["prefill_calls"] + c["decode_calls"] + c["empty_calls"] + c["rejected_calls"]


# ---------------------------------------------------------------- sliding window (NEXT: local attention)
# Gemma 4's sliding layers (MLX issue #3885, "Current routing": n_q=32, n_kv=16,
# d=256) next to its global ones; the rule is the reading documented with the
# oracle: with own = i + Lk - Lq, key j is visible iff own - W < j <= own.
@pytest.mark.parametrize("D,Dv", DIMS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("W", [1, 77, 300])
def test_sliding_window_prefill(D, Dv, dtype, W):
    """Lq < Lk with ragged tiles: windows narrower than one key tile, spanning
    a few tiles, and wider than most rows' history; every row checked."""
    c = I.make_case(2100 + W, 1, 8, 2, 333, 517, D, Dv, dtype=dtype, mask="sliding", window=W)
    assert path_of(c) == S.SDPA_PATH_PREFILL
    run_and_check(c, label=f"sliding W={W} D={D} dt={dtype}")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("D,Dv", [(72, 72), (128, 128), (256, 256), (512, 512)])
def test_sliding_window_long_prefill_skips_tiles(D, Dv, dtype):
    """L = 4096 with a 256-key window: most key tiles of a query tile lie
    outside every row's window and are never loaded; sampled rows, including
    the first rows (whose windows are cut at key 0)."""
    c = I.make_case(2200, 1, 8, 4, 4096, 4096, D, Dv, dtype=dtype, mask="sliding", window=256)
    rows = np.concatenate([I.sample_rows(2200, 1, 8, 4096, 48),
                           np.array([[0, 3, i] for i in (1, 2, 255, 256, 257)])])
    run_and_check(c, rows=np.unique(rows, axis=0), label=f"sliding long D={D} dt={dtype}")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("Lq", [1, 4, 8])
@pytest.mark.parametrize("W", [1, 100, 1024, 5000])
def test_sliding_window_decode_gemma4_shape(dtype, Lq, W):
    """The decode path on the sliding-layer shape (32 q / 16 kv heads, d=256),
    kL=4096: the splits divide the window's keys only."""
    c = I.make_case(2300 + W, 1, 32, 16, Lq, 4096, 256, dtype=dtype, mask="sliding", window=W)
    assert path_of(c) == S.SDPA_PATH_DECODE
    run_and_check(c, label=f"sliding decode W={W} Lq={Lq} dt={dtype}")


@pytest.mark.parametrize("D,Dv", DIMS)
def test_sliding_window_equals_causal_when_it_covers_every_key(D, Dv):
    import dataclasses
    c = I.make_case(2400, 2, 8, 2, 129, 129, D, Dv, dtype=I.BF16, mask="sliding", window=129)
    (_, _), a = run_and_check(c, label="window = Lk")
    (_, _), b = run_and_check(dataclasses.replace(c, mask_kind=I.MASK_CAUSAL, window=0), label="causal")
    assert np.abs(a - b).max() <= 1e-6


def test_sliding_window_abi_rules():
    c = I.make_case(2500, 1, 4, 2, 16, 16, 64, dtype=I.BF16)
    g = GpuCase(c)
    out = g.out_buf.data_ptr() + g.pad * g.out_buf.element_size()
    args = (g.q.data_ptr(), g.k.data_ptr(), g.v.data_ptr(), out, c.B, c.Hq, c.Hkv, c.Lq, c.Lk, c.Dqk, c.Dv,
            c.all_strides16, c.scale)
    s = torch.cuda.current_stream().cuda_stream
    assert S.sdpa_forward_window(*args, 0, c.dtype, s) == 1                       # window >= 1
    assert S.sdpa_forward(*args, S.SDPA_MASK_SLIDING, None, None, c.dtype, s) == 1  # needs the window entry
    assert S.sdpa_supported(c.B, c.Hq, c.Hkv, c.Lq, c.Lk, c.Dqk, c.Dv, c.all_strides16, S.SDPA_MASK_SLIDING,
                            None, c.dtype) == (0, S.SDPA_PATH_PREFILL)
    assert S.sdpa_forward_window(*args, 5, c.dtype, s) == 0
    torch.cuda.synchronize()


# ---------------------------------------------------------------- many heads, GQA, ragged (head dims 64-96)
# The 96-key-tile kernel on grids of 16, 160 and 240 two-tile CTAs (on 148 SMs:
# under one wave, one wave and a little, one and a half waves), with GQA
# groups of 1, 3 and 8, ragged query and key lengths, every mask kind; all rows
# are checked.
@pytest.mark.parametrize("D", [64, 72, 96])
@pytest.mark.parametrize("dtype", [I.BF16, I.F16])
@pytest.mark.parametrize("shape", [
    dict(Hq=4, Hkv=4, Lq=1000, Lk=1000),
    dict(Hq=80, Hkv=10, Lq=500, Lk=509),
    dict(Hq=120, Hkv=40, Lq=512, Lk=384),
])
@pytest.mark.parametrize("mask", ["none", "bool", "additive", "causal"])
def test_prefill_many_heads_ragged(D, dtype, shape, mask):
    seed = 5100 + D + 7 * shape["Hq"] + (mask == "bool") * 3 + (mask == "additive") * 5 + (mask == "causal") * 11
    c = I.make_case(seed, 1, shape["Hq"], shape["Hkv"], shape["Lq"], shape["Lk"], D, dtype=dtype, mask=mask,
                    layout="blhd")
    run_and_check(c, None, label=f"many heads D={D} {shape} {mask}")


# ---------------------------------------------------------------- decode split plan
# The decode plan gives every (batch, KV head, row group) the same split count:
# at most the SMs' share per group and half the key slots, then the fewest
# splits that reach the smallest largest share.  These shapes land on each
# branch (one split; capped by the slots; capped by the SMs; more groups than
# SMs, in waves) with ragged key counts; all rows against the oracle.
@pytest.mark.parametrize("D", [64, 256, 512])
@pytest.mark.parametrize("B,Hkv,group", [(1, 1, 4), (1, 8, 4), (2, 40, 2), (4, 48, 1)])
@pytest.mark.parametrize("Lk", [1, 33, 95, 200, 1000, 5000])
def test_decode_split_plan(D, B, Hkv, group, Lk):
    mask = "decode_additive" if Lk % 2 == 1 else "none"
    c = I.make_case(6100 + D + Hkv + Lk, B, Hkv * group, Hkv, 1, Lk, D, dtype=I.BF16, mask=mask)
    run_and_check(c, None, label=f"decode split plan D={D} B={B} Hkv={Hkv} G={group} Lk={Lk}")


# The split counts the decode plan picks for the measured decode shapes on a
# 148-SM B200 (read from the SDPA_LOG line of each call): every KV head gets the
# same count, the one the split-count sweep found fastest or within 1 % of it.
@pytest.mark.parametrize("D,Hkv,Lk,splits", [(256, 8, 4096, 16), (256, 8, 1024, 16),
                                             (512, 4, 1024, 16), (512, 4, 4096, 32)])
def test_decode_plan_split_counts(monkeypatch, capfd, D, Hkv, Lk, splits):
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("split counts pinned for 148 SMs")
    monkeypatch.setenv("SDPA_LOG", "1")
    c = I.make_case(6400 + D + Lk, 1, 32, Hkv, 1, Lk, D, dtype=I.BF16, mask="none")
    rows = I.sample_rows(6400 + D, 1, 32, 1, 8)
    run_and_check(c, rows, label=f"plan D={D} Lk={Lk}")
    err = capfd.readouterr().err
    lines = [l for l in err.splitlines() if l.startswith("[sdpa]") and f"Lk={Lk} Dqk={D}" in l]
    assert lines, err
    import re
    m = re.search(r"grid=\((\d+),1,1\).*splits=(\d+)", lines[-1])
    assert m, lines[-1]
    assert int(m.group(2)) == splits and int(m.group(1)) == Hkv * splits, lines[-1]
